"""QKV prologue fused into the repack, against the fp64 oracle.

Planes 2.. (V, gate) are copied: bit-exact.  Planes 0 / 1 (Q, K) are
computed in fp32 and rounded once to bf16, so each element must lie within
half a bf16 ulp of the fp64 value (2^-9 relative) plus the fp32 error of the
norm and rotation (bounded here by 1e-5 of the terms' magnitude), i.e.
|gpu - ref| <= 2^-8 |ref| + 1e-4 for O(1) inputs.
"""
import numpy as np
import pytest
from _parity import check_attention

from oracle import ulysses_oracle as orc

pytestmark = pytest.mark.gpu

REL = 2.0 ** -8
ABS = 1e-4


def _make(gpu, P, N, H, C, rd, seed, layout="token"):
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs
    Np = inputs.padded(N, P)
    ts, ps = (0, 0) if layout == "token" else (H * 128, Np * H * 128)
    plan = U.ulysses_plan(N, H, 128, P, C, ts, ps)
    S = inputs.qkv_seq(N, H, P, C, seed, gpu, layout=layout)
    g = torch.Generator(device=gpu)
    g.manual_seed(seed + 500)
    wq = torch.randn(128, generator=g, device=gpu).to(torch.bfloat16)
    wk = torch.randn(128, generator=g, device=gpu).to(torch.bfloat16)
    ang = torch.rand((Np, max(rd // 2, 1)), generator=g, device=gpu) * 6.2832
    cos = torch.cat([torch.cos(ang), torch.cos(ang)], 1)[:, :rd].to(torch.bfloat16).contiguous()
    sin = torch.cat([torch.sin(ang), torch.sin(ang)], 1)[:, :rd].to(torch.bfloat16).contiguous()
    if rd == 0:
        cos = sin = None
    return plan, S, wq, wk, cos, sin


def _check(plan, S, T, wq, wk, cos, sin, rd, P, layout, tokens=None):
    from ulysses_sequence_attention_repack_b200 import inputs
    S_bits = inputs.host_bits(S)
    if layout != "token":
        S_bits = np.ascontiguousarray(S_bits.transpose(1, 0, 2, 3))
    Np = S_bits.shape[0]
    rdz = max(rd, 16)
    cb = inputs.host_bits(cos) if cos is not None else np.zeros((Np, rdz), np.uint16)
    sb = inputs.host_bits(sin) if sin is not None else np.zeros((Np, rdz), np.uint16)
    T_bits = inputs.host_bits(T)
    if tokens is None:
        ref = orc.prologue_repack_fwd(S_bits, P, inputs.host_bits(wq), inputs.host_bits(wk), cb[:, :rd], sb[:, :rd], rd)
        got = orc.bf16_bits_to_f64(T_bits)
        # V / gate planes: exact copies
        assert np.array_equal(T_bits[:, 2:], orc.repack_fwd(S_bits, P)[:, 2:])
        err = np.abs(got[:, :2] - ref[:, :2])
        bound = REL * np.abs(ref[:, :2]) + ABS
        assert np.all(err <= bound), float((err - bound).max())
        return
    # sampled tokens: the prologue is per token, the repack a permutation
    H = S_bits.shape[2]
    Hl = H // P
    y = orc.qkv_prologue(S_bits[tokens], inputs.host_bits(wq), inputs.host_bits(wk), cb[tokens, :rd],
                         sb[tokens, :rd], rd)                                   # [R, C, H, D]
    got = orc.bf16_bits_to_f64(T_bits[:, :, tokens])                            # [P, C, R, Hl, D]
    want = y.reshape(len(tokens), y.shape[1], P, Hl, 128).transpose(2, 1, 0, 3, 4)
    err = np.abs(got[:, :2] - want[:, :2])
    assert np.all(err <= REL * np.abs(want[:, :2]) + ABS)
    assert np.array_equal(got[:, 2:], want[:, 2:])


@pytest.mark.parametrize("P,N,H,C,rd,layout", [
    (2, 1000, 8, 3, 96, "token"), (4, 777, 8, 4, 96, "token"), (1, 300, 2, 3, 128, "token"),
    (2, 640, 4, 3, 0, "token"), (2, 513, 6, 3, 64, "plane"), (8, 1024, 56, 3, 96, "token")])
def test_prologue_repack_against_oracle(gpu, P, N, H, C, rd, layout):
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    plan, S, wq, wk, cos, sin = _make(gpu, P, N, H, C, rd, 60 + N, layout)
    Np = plan.padded_tokens
    T = torch.empty((P, C, Np, H // P, 128), dtype=torch.bfloat16, device=gpu)
    U.ulysses_prologue_repack_fwd(plan, S, T, wq, wk, cos, sin, rd, 1e-5)
    torch.cuda.synchronize()
    _check(plan, S, T, wq, wk, cos, sin, rd, P, layout)


def test_prologue_feeds_attention(gpu):
    """Prologue -> attention -> inverse repack equals the oracle chain on the same bytes."""
    import math

    import torch
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs
    P, N, H, C, rd = 2, 1024, 8, 3, 96
    plan, S, wq, wk, cos, sin = _make(gpu, P, N, H, C, rd, 71)
    T = torch.empty((P, C, N, H // P, 128), dtype=torch.bfloat16, device=gpu)
    U.ulysses_prologue_repack_fwd(plan, S, T, wq, wk, cos, sin, rd)
    OT = torch.empty((P, N, H // P, 128), dtype=torch.bfloat16, device=gpu)
    U.ulysses_attn_fwd(plan, T, OT, 1.0 / math.sqrt(128))
    torch.cuda.synchronize()
    ref = orc.attention_heads(inputs.host_bits(T), N, 1.0 / math.sqrt(128))
    check_attention(f"prologue -> attention P={P} N={N} H={H}", OT.float().cpu().numpy(), ref)


def test_prologue_argument_checks(gpu):
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    plan, S, wq, wk, cos, sin = _make(gpu, 2, 256, 4, 3, 96, 72)
    T = torch.empty((2, 3, 256, 2, 128), dtype=torch.bfloat16, device=gpu)
    with pytest.raises(U.UlyssesError) as e:
        U.ulysses_prologue_repack_fwd(plan, S, T, wq, wk, cos, sin, 40)     # not a multiple of 16
    assert e.value.code == 8
    with pytest.raises(U.UlyssesError) as e:
        U.ulysses_prologue_repack_fwd(plan, S, T, wq, wk, cos, sin, 96, -1.0)
    assert e.value.code == 1


@pytest.mark.slow
def test_prologue_repack_dit19k(gpu):
    """Video-DiT size (P=4, N=19,394, H=56): V plane bit-exact everywhere, Q/K on 2048 sampled tokens."""
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs
    P, N, H, C, rd = 4, 19_394, 56, 3, 96
    plan, S, wq, wk, cos, sin = _make(gpu, P, N, H, C, rd, 1)
    Np = plan.padded_tokens
    T = torch.empty((P, C, Np, H // P, 128), dtype=torch.bfloat16, device=gpu)
    U.ulysses_prologue_repack_fwd(plan, S, T, wq, wk, cos, sin, rd)
    T2 = torch.empty_like(T)
    U.ulysses_repack_fwd(plan, S, T2)
    torch.cuda.synchronize()
    assert torch.equal(T[:, 2], T2[:, 2])
    tokens = orc.sample_rows(N, 2048, 1)
    _check(plan, S, T, wq, wk, cos, sin, rd, P, "token", tokens=tokens)
