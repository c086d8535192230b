"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Small cases span several tiles and ragged tails; the oracle finishes them in
seconds.  Repack: bit-exact.  Attention: max-abs <= 2e-2 and mean-abs <= 2e-3
against the fp64 oracle (the layer's stated tolerance); pad rows exactly zero.
"""
import math

import numpy as np
import pytest
from _parity import MAX_ABS, MEAN_ABS, check_attention

from oracle import ulysses_oracle as orc

pytestmark = pytest.mark.gpu

# (P, N, H, C, layout, cu_seqlens, seed)
CASES = [
    pytest.param(2, 1024, 8, 3, "token", None, 0, id="tiny-P2-N1024-H8"),
    pytest.param(4, 1001, 8, 3, "token", None, 5, id="ragged-P4-N1001"),
    pytest.param(1, 300, 2, 3, "token", None, 6, id="P1-N300"),
    pytest.param(4, 777, 8, 4, "token", None, 7, id="qkvg-P4-N777"),
    pytest.param(2, 640, 4, 3, "plane", None, 8, id="plane-major-P2"),
    pytest.param(2, 1000, 4, 3, "token", [0, 300, 301, 777, 1000], 9, id="varlen-4seq"),
    pytest.param(8, 2048, 16, 3, "token", [0, 1024, 1536, 2048], 10, id="varlen-P8"),
    pytest.param(2, 1000, 4, 3, "token", [0, 300, 300, 777, 1000, 1000], 37, id="varlen-empty-segments"),
    pytest.param(1, 1, 1, 3, "token", None, 11, id="N1"),
    pytest.param(4, 5, 4, 3, "token", None, 12, id="N5-P4"),
    # one head per rank across 56 ranks (the Video-DiT head count): 56 runs per row
    pytest.param(56, 1000, 56, 3, "token", None, 38, id="P56-Hl1"),
]


def _torch():
    import torch
    return torch


def _strides(layout, N, P, C, H):
    Np = orc.padded_tokens(N, P)
    if layout == "token":
        return 0, 0
    return H * 128, Np * H * 128


def _seq_as_token_major(bits, layout):
    # oracle input is always [Np, C, H, D]
    return bits if layout == "token" else np.ascontiguousarray(bits.transpose(1, 0, 2, 3))


def _run(P, N, H, C, layout, cu, seed):
    torch = _torch()
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs
    dev = torch.device("cuda", 0)
    ts, ps = _strides(layout, N, P, C, H)
    plan = U.ulysses_plan(N, H, 128, P, C, ts, ps, 0, cu)
    Np = plan.padded_tokens
    S = inputs.qkv_seq(N, H, P, C, seed, dev, layout=layout)
    Hl = H // P
    T = torch.empty((P, C, Np, Hl, 128), dtype=torch.bfloat16, device=dev)
    U.ulysses_repack_fwd(plan, S, T)
    OT = torch.empty((P, Np, Hl, 128), dtype=torch.bfloat16, device=dev)
    U.ulysses_attn_fwd(plan, T, OT, 1.0 / math.sqrt(128))
    back = torch.empty_like(S)
    U.ulysses_repack_bwd(plan, T, back, C)
    OS = torch.empty((Np, H, 128), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=dev)
    U.ulysses_layer_fwd(plan, S, OS, ws, fused=0)
    OSf = torch.empty((Np, H, 128), dtype=torch.bfloat16, device=dev)
    U.ulysses_layer_fwd(plan, S, OSf, None, fused=1)
    torch.cuda.synchronize()
    assert U.ulysses_last_device_error(plan) == 0
    return plan, S, T, OT, back, OS, OSf


def _bits(t):
    from ulysses_sequence_attention_repack_b200 import inputs
    return inputs.host_bits(t)


def _f32(t):
    return t.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("P,N,H,C,layout,cu,seed", CASES)
def test_repack_attention_layer_against_oracle(gpu, P, N, H, C, layout, cu, seed):
    plan, S, T, OT, back, OS, OSf = _run(P, N, H, C, layout, cu, seed)
    S_bits = _seq_as_token_major(_bits(S), layout)
    # step 1: bit-exact
    T_ref = orc.repack_fwd(S_bits, P)
    assert np.array_equal(_bits(T), T_ref)
    # step 3 on all planes: exact round trip
    assert np.array_equal(_bits(back), _bits(S))
    # step 2 against fp64 attention on the same bytes
    scale = 1.0 / math.sqrt(128)
    O_ref = orc.attention_heads(T_ref, N, scale, cu_seqlens=cu)
    O_gpu = _f32(OT)
    check_attention(f"attn P={P} N={N} H={H} C={C} {layout} cu={cu}", O_gpu, O_ref)
    assert np.all(O_gpu[:, N:] == 0)
    # the whole layer: oracle composition, and fused == unfused bit for bit
    L_ref = orc.output_repack_bwd(O_ref)
    check_attention(f"layer P={P} N={N} H={H} C={C} {layout} cu={cu}", _f32(OS), L_ref)
    assert np.array_equal(_bits(OS), _bits(OSf))
    # step 3 on the attention output equals the layer output bit for bit
    assert np.array_equal(_bits(OS), orc.repack_bwd(_bits(OT)[:, None])[:, 0])


CAUSAL_CASES = [
    pytest.param(2, 1024, 8, None, 13, id="causal-tiny"),
    pytest.param(4, 1001, 8, None, 14, id="causal-ragged"),
    pytest.param(1, 300, 2, None, 15, id="causal-P1"),
    pytest.param(2, 1000, 4, [0, 300, 301, 777, 1000], 16, id="causal-varlen"),
    pytest.param(2, 700, 4, [0, 256, 512, 700], 17, id="causal-varlen-aligned"),
    pytest.param(2, 700, 4, [0, 0, 256, 256, 700], 18, id="causal-varlen-empty-segments"),
]


@pytest.mark.parametrize("P,N,H,cu,seed", CAUSAL_CASES)
def test_causal_attention_against_oracle(gpu, P, N, H, cu, seed):
    torch = _torch()
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs
    plan = U.ulysses_plan(N, H, 128, P, 3, 0, 0, 0, cu, causal=True)
    Np, Hl = plan.padded_tokens, H // P
    S = inputs.qkv_seq(N, H, P, 3, seed, gpu)
    T = torch.empty((P, 3, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
    U.ulysses_repack_fwd(plan, S, T)
    OT = torch.empty((P, Np, Hl, 128), dtype=torch.bfloat16, device=gpu)
    U.ulysses_attn_fwd(plan, T, OT, 1.0 / math.sqrt(128))
    OS = torch.empty((Np, H, 128), dtype=torch.bfloat16, device=gpu)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=gpu)
    U.ulysses_layer_fwd(plan, S, OS, ws, fused=0)
    OSf = torch.empty_like(OS)
    U.ulysses_layer_fwd(plan, S, OSf, None, fused=1)
    torch.cuda.synchronize()
    assert U.ulysses_last_device_error(plan) == 0
    ref = orc.attention_heads(_bits(T), N, 1.0 / math.sqrt(128), cu_seqlens=cu, causal=True)
    check_attention(f"causal P={P} N={N} H={H} cu={cu}", _f32(OT), ref)
    assert np.all(_f32(OT)[:, N:] == 0)
    assert np.array_equal(_bits(OS), _bits(OSf))
    assert np.array_equal(_bits(OS), orc.repack_bwd(_bits(OT)[:, None])[:, 0])
    # the first row of every segment is exactly its own value row, rounded to bf16
    segs = [(0, N)] if cu is None else list(zip(cu, cu[1:]))
    for a, b in segs:
        if b > a:
            np.testing.assert_array_equal(_bits(OS[a]), _bits(S[a, 2]))


def test_sharp_softmax_diagnostic(gpu):
    """Q scaled by 8: peaked rows exercise the running-max rescale path."""
    torch = _torch()
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs
    dev = torch.device("cuda", 0)
    P, N, H = 2, 1024, 4
    plan = U.ulysses_plan(N, H, 128, P, 3)
    S = inputs.qkv_seq(N, H, P, 3, 21, dev)
    S[:, 0] *= 8
    OS = torch.empty((N, H, 128), dtype=torch.bfloat16, device=dev)
    U.ulysses_layer_fwd(plan, S, OS, None, fused=1)
    torch.cuda.synchronize()
    ref = orc.layer_fwd(_bits(S), P, N, 1.0 / math.sqrt(128))
    check_attention("sharp softmax (Q x 8) P=2 N=1024 H=4", _f32(OS), ref, max_abs=4 * MAX_ABS)


def test_uniform_keys_give_mean_of_v(gpu):
    torch = _torch()
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs
    dev = torch.device("cuda", 0)
    P, N, H = 2, 700, 4
    plan = U.ulysses_plan(N, H, 128, P, 3)
    S = inputs.qkv_seq(N, H, P, 3, 22, dev)
    S[:N, 1] = S[0:1, 1]      # every key equal
    OS = torch.empty((N, H, 128), dtype=torch.bfloat16, device=dev)
    U.ulysses_layer_fwd(plan, S, OS, None, fused=1)
    torch.cuda.synchronize()
    v = _f32(S[:N, 2])                                 # [N, H, D]
    want = np.broadcast_to(v.mean(axis=0, keepdims=True), v.shape)
    check_attention("uniform keys P=2 N=700 H=4", _f32(OS), want)


HOST_CASES = [
    pytest.param(2, 1024, 8, 3, "token", None, False, 30, id="tiny"),
    pytest.param(4, 1001, 8, 3, "token", None, False, 31, id="ragged-P4"),
    pytest.param(4, 777, 8, 4, "token", None, False, 32, id="qkvg-P4"),
    pytest.param(2, 640, 4, 3, "plane", None, False, 33, id="plane-major"),
    pytest.param(8, 2048, 16, 3, "token", [0, 1024, 1536, 2048], False, 34, id="varlen-P8"),
    pytest.param(4, 1001, 8, 3, "token", None, True, 35, id="causal-P4"),
    # 223 work units per head: the pipeline splits each rank's 4 heads into 2 groups
    pytest.param(2, 57_001, 8, 3, "token", None, False, 36, id="head-groups"),
]


@pytest.mark.parametrize("P,N,H,C,layout,cu,causal,seed", HOST_CASES)
def test_host_layer_streams_ranks_exactly(gpu, P, N, H, C, layout, cu, causal, seed):
    """ulysses_layer_fwd_host (copies and kernels streamed rank by rank) equals
    the device layer bit for bit, fused and unfused, on two calls in a row
    with a non-default stream that is the only thing synchronised."""
    torch = _torch()
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs
    ts, ps = _strides(layout, N, P, C, H)
    plan = U.ulysses_plan(N, H, 128, P, C, ts, ps, 0, cu, causal=causal)
    Np = plan.padded_tokens
    S = inputs.qkv_seq(N, H, P, C, seed, gpu, layout=layout)
    want = torch.empty((Np, H, 128), dtype=torch.bfloat16, device=gpu)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=gpu)
    U.ulysses_layer_fwd(plan, S, want, ws, fused=0)
    torch.cuda.synchronize()
    want_bits = _bits(want)
    host_in = S.cpu().pin_memory()
    dev_in = torch.empty_like(S)
    dev_out = torch.empty_like(want)
    stream = torch.cuda.Stream(device=gpu)
    for fused in (0, 1, 0):
        host_out = torch.full(want.shape, float("nan"), dtype=torch.bfloat16).pin_memory()
        dev_in.zero_()
        dev_out.zero_()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            U.ulysses_layer_fwd_host(plan, host_in, host_out, dev_in, dev_out, ws if fused == 0 else None,
                                     fused=fused, stream=stream)
        stream.synchronize()
        assert U.ulysses_last_device_error(plan, stream) == 0
        assert np.array_equal(host_out.view(torch.int16).numpy().view("uint16"), want_bits), fused
        assert torch.equal(dev_in, S)
    if N <= 4096:   # the device layer at larger N is checked against the oracle in the full-size tests
        ref = orc.layer_fwd(_seq_as_token_major(_bits(S), layout), P, N, 1.0 / math.sqrt(128), cu_seqlens=cu,
                            causal=causal)
        check_attention(f"host layer P={P} N={N} H={H} causal={causal}", _f32(want), ref)
