"""The layer under torch.autograd against the fp64 oracle.

Forward: the layer output within the forward tolerance (max-abs 2e-2,
mean-abs 2e-3).  Backward: d(qkv) within the backward tolerance of
test_gpu_backward (per gradient plane, max <= 2e-2 max|ref|, mean <= 5e-3
mean|ref|); gate planes and pad rows get exactly zero.
"""
import math

import numpy as np
import pytest
from _parity import check_attention

from oracle import ulysses_oracle as orc

pytestmark = pytest.mark.gpu


def _close(got, ref, what, max_rel=2e-2, mean_rel=5e-3):
    err = np.abs(got - ref)
    assert err.max() <= max_rel * np.abs(ref).max(), (what, float(err.max()))
    assert err.mean() <= mean_rel * np.abs(ref).mean(), (what, float(err.mean()))
    check_attention(f"autograd {what}", got, ref, max_abs=None, mean_abs=None)


@pytest.mark.parametrize("P,N,H,C,layout,cu,causal", [
    (2, 1000, 4, 3, "token", None, False),
    (4, 777, 8, 4, "token", None, False),
    (2, 640, 4, 3, "plane", None, False),
    (2, 900, 4, 3, "token", [0, 300, 900], True),
])
def test_autograd_layer_against_oracle(gpu, P, N, H, C, layout, cu, causal):
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs
    from ulysses_sequence_attention_repack_b200.autograd import ulysses_attention
    Np = inputs.padded(N, P)
    ts, ps = (0, 0) if layout == "token" else (H * 128, Np * H * 128)
    plan = U.ulysses_plan(N, H, 128, P, C, ts, ps, 0, cu, causal=causal)
    S = inputs.qkv_seq(N, H, P, C, 80 + N, gpu, layout=layout)
    x = S if layout == "token" else S.transpose(0, 1)          # [Np, C, H, D] view either way
    x = x.detach().requires_grad_(True)
    out = ulysses_attention(x, plan)
    g = torch.Generator(device=gpu)
    g.manual_seed(81 + N)
    G = torch.randn((Np, H, 128), generator=g, device=gpu).to(torch.bfloat16)
    G[N:] = 0
    out.backward(G)
    torch.cuda.synchronize()
    assert U.ulysses_last_device_error(plan) == 0
    S_bits = inputs.host_bits(x)                                 # token-major bits
    scale = 1.0 / math.sqrt(128)
    ref_out = orc.layer_fwd(S_bits, P, N, scale, cu_seqlens=cu, causal=causal)
    err = np.abs(out.detach().float().cpu().numpy() - ref_out)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3
    ref = orc.layer_bwd(S_bits, inputs.host_bits(G), P, N, scale, cu, causal)
    got = x.grad.float().cpu().numpy().astype(np.float64)
    for c, name in enumerate(("dQ", "dK", "dV")):
        _close(got[:N, c], ref[:N, c], name)
    assert np.all(got[N:] == 0)
    if C > 3:
        assert np.all(got[:, 3:] == 0)                           # the gate is not attended


def test_autograd_rejects_wrong_input(gpu):
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200.autograd import ulysses_attention
    plan = U.ulysses_plan(256, 4, 128, 2, 3)
    with pytest.raises(TypeError):
        ulysses_attention(torch.zeros((256, 3, 4, 128), device=gpu), plan)        # fp32
    with pytest.raises(ValueError):
        ulysses_attention(torch.zeros((255, 3, 4, 128), dtype=torch.bfloat16, device=gpu), plan)
