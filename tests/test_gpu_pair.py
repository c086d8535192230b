"""The CTA-pair attention kernel (ULYSSES_PLAN_PAIR_ATTENTION) against the
fp64 oracle and against the default one-CTA-per-SM kernel.

The pair kernel computes every output row with the same arithmetic as the
default kernel (the same MMA shapes per SM, the same softmax code on its TMEM
rows), so the two give identical bits; both are also checked against the
oracle with the layer's gates, and the fused and multi-GPU push launches of
the pair kernel must equal its unfused output bit for bit.
"""
import math

import numpy as np
import pytest
from _parity import check_attention

from oracle import ulysses_oracle as orc

pytestmark = pytest.mark.gpu

# (P, N, H, C, cu_seqlens, causal, seed)
CASES = [
    pytest.param(2, 1024, 8, 3, None, False, 50, id="tiny"),
    pytest.param(4, 1001, 8, 4, None, False, 51, id="ragged-qkvg"),
    pytest.param(8, 2048, 16, 3, [0, 1024, 1536, 2048], False, 52, id="varlen-P8"),
    pytest.param(2, 1000, 4, 3, [0, 300, 300, 777, 1000], False, 53, id="varlen-empty-segment"),
    pytest.param(2, 1024, 8, 3, None, True, 54, id="causal"),
    pytest.param(2, 1000, 4, 3, [0, 300, 301, 777, 1000], True, 55, id="causal-varlen"),
    pytest.param(4, 5, 4, 3, None, False, 56, id="N5"),
    pytest.param(1, 1, 1, 3, None, False, 57, id="N1"),
    pytest.param(56, 1000, 56, 3, None, False, 58, id="P56-Hl1"),
    pytest.param(2, 3000, 8, 3, None, False, 59, id="several-units-per-pair"),
]


def _bits(t):
    from ulysses_sequence_attention_repack_b200 import inputs
    return inputs.host_bits(t)


def _layer(gpu, P, N, H, C, cu, causal, seed, pair):
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs
    plan = U.ulysses_plan(N, H, 128, P, C, 0, 0, 0, cu, causal=causal, pair_cta=pair)
    Np, Hl = plan.padded_tokens, H // P
    S = inputs.qkv_seq(N, H, P, C, seed, gpu)
    T = torch.empty((P, C, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
    OT = torch.empty((P, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
    OSf = torch.empty((Np, H, 128), dtype=torch.bfloat16, device=gpu)
    scale = 1.0 / math.sqrt(128)
    U.ulysses_repack_fwd(plan, S, T)
    U.ulysses_attn_fwd(plan, T, OT, scale)
    U.ulysses_layer_fwd(plan, S, OSf, None, fused=1)
    # the multi-GPU push launch with the ranks emulated
    Nl = plan.rows_per_rank
    OSp = torch.full_like(OSf, float("nan"))
    outs = [OSp[q * Nl:(q + 1) * Nl] for q in range(P)]
    for r in range(P):
        U.ulysses_attn_fwd_push(plan, r, T[r], outs, scale)
    torch.cuda.synchronize()
    assert U.ulysses_last_device_error(plan) == 0
    return S, T, OT, OSf, OSp


@pytest.mark.parametrize("P,N,H,C,cu,causal,seed", CASES)
def test_pair_kernel_against_oracle_and_default_kernel(gpu, P, N, H, C, cu, causal, seed):
    S, T, OT, OSf, OSp = _layer(gpu, P, N, H, C, cu, causal, seed, pair=True)
    ref = orc.attention_heads(_bits(T), N, 1.0 / math.sqrt(128), cu_seqlens=cu, causal=causal)
    got = OT.float().cpu().numpy().astype(np.float64)
    check_attention(f"pair kernel P={P} N={N} H={H} cu={cu} causal={causal}", got, ref)
    assert np.all(got[:, N:] == 0)
    lay = orc.repack_bwd(_bits(OT)[:, None])[:, 0]
    assert np.array_equal(_bits(OSf), lay)          # fused == unfused
    assert np.array_equal(_bits(OSp), lay)          # push epilogue == unfused
    _, _, OT1, OSf1, _ = _layer(gpu, P, N, H, C, cu, causal, seed, pair=False)
    assert np.array_equal(_bits(OT), _bits(OT1))    # same bits as one CTA per SM
    assert np.array_equal(_bits(OSf), _bits(OSf1))


@pytest.mark.slow
def test_pair_kernel_dit19k_equals_default_kernel(gpu):
    """Video-DiT size: the pair kernel's output equals the default kernel's
    bit for bit (which the full-size tests check against the oracle)."""
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs
    P, N, H, C = 4, 19_394, 56, 3
    S = inputs.qkv_seq(N, H, P, C, 1, gpu)
    outs = []
    for pair in (True, False):
        plan = U.ulysses_plan(N, H, 128, P, C, pair_cta=pair)
        OS = torch.empty((plan.padded_tokens, H, 128), dtype=torch.bfloat16, device=gpu)
        U.ulysses_layer_fwd(plan, S, OS, None, fused=1)
        torch.cuda.synchronize()
        assert U.ulysses_last_device_error(plan) == 0
        outs.append(OS)
    assert torch.equal(outs[0], outs[1])
