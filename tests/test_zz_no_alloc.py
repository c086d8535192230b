"""The allocation-free entry point against the regular fused layer.

ulysses_layer_fwd_fused_noalloc serves callers that cannot call cudaMalloc
(and therefore cannot create a plan, which allocates a device error word).
It must produce what ulysses_layer_fwd(fused=1) produces.  Two calls in a
row check that the shared file-scope scratch left by the first call does not
leak into the second.  This file is collected last on purpose, so a run that
stops at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
from _parity import check_attention

pytestmark = pytest.mark.gpu


def _call(lib, S, out, N, H, P, C, cu):
    if cu is None:
        arr, ns = None, 0
    else:
        arr = (ctypes.c_int32 * len(cu))(*cu)
        ns = len(cu) - 1
    status = ctypes.c_int32(-1)
    import torch
    code = lib.ulysses_layer_fwd_fused_noalloc(S.data_ptr(), out.data_ptr(), N, H, 128, P, C, 0, 0, arr, ns,
                                               ctypes.byref(status), torch.cuda.current_stream().cuda_stream)
    return code, status.value


def test_no_alloc_matches_fused_layer_on_two_calls(gpu):
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs
    lib = U.load()
    cases = [(2, 1000, 8, 3, None, 31), (4, 2053, 8, 4, [0, 700, 701, 2053], 32)]   # P, N, H, C, cu, seed
    for P, N, H, C, cu, seed in cases:
        S = inputs.qkv_seq(N, H, P, C, seed, gpu)
        Np = S.shape[0]
        plan = U.ulysses_plan(N, H, 128, P, C, 0, 0, 0, cu)
        ref = torch.empty((Np, H, 128), dtype=torch.bfloat16, device=gpu)
        U.ulysses_layer_fwd(plan, S, ref, None, fused=1)
        out = torch.full((Np, H, 128), float("nan"), dtype=torch.bfloat16, device=gpu)
        code, status = _call(lib, S, out, N, H, P, C, cu)
        torch.cuda.synchronize()
        assert code == 0 and status == 0, (code, status)
        check_attention(f"no-alloc vs fused layer P={P} N={N}", out.float().cpu().numpy(),
                        ref.float().cpu().numpy())
        assert torch.equal(out, ref)      # same kernel, same tile order: identical bits


def test_no_alloc_leaves_device_memory_untouched(gpu):
    """After a first call (which looks up the scratch address in this
    context), further calls change neither the device's free memory nor
    torch's allocation counters."""
    import torch
    from ulysses_sequence_attention_repack_b200 import inputs
    lib = __import__("ulysses_sequence_attention_repack_b200").load()
    P, N, H, C = 2, 1000, 8, 3
    S = inputs.qkv_seq(N, H, P, C, 33, gpu)
    out = torch.empty((S.shape[0], H, 128), dtype=torch.bfloat16, device=gpu)
    first = _call(lib, S, out, N, H, P, C, None)
    torch.cuda.synchronize()
    assert first == (0, 0)
    free0, _ = torch.cuda.mem_get_info(gpu)
    stats0 = torch.cuda.memory_stats(gpu)
    for _ in range(2):
        assert _call(lib, S, out, N, H, P, C, None) == (0, 0)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info(gpu)
    stats1 = torch.cuda.memory_stats(gpu)
    assert free1 == free0
    for key in ("allocation.all.allocated", "segment.all.allocated", "reserved_bytes.all.current"):
        assert stats1.get(key, 0) == stats0.get(key, 0), key


def test_no_alloc_call_in_a_cuda_graph(gpu):
    """After a first call in this context (the header's rule), an asynchronous
    call (host_status NULL) can be captured into a CUDA graph on a side
    stream; each replay reproduces the fused layer bit for bit."""
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    from ulysses_sequence_attention_repack_b200 import inputs
    lib = U.load()
    P, N, H, C = 2, 1000, 8, 3
    S = inputs.qkv_seq(N, H, P, C, 34, gpu)
    Np = S.shape[0]
    plan = U.ulysses_plan(N, H, 128, P, C)
    ref = torch.empty((Np, H, 128), dtype=torch.bfloat16, device=gpu)
    U.ulysses_layer_fwd(plan, S, ref, None, fused=1)
    out = torch.empty_like(ref)
    assert _call(lib, S, out, N, H, P, C, None) == (0, 0)      # the first call, outside any capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=side):
        code = lib.ulysses_layer_fwd_fused_noalloc(S.data_ptr(), out.data_ptr(), N, H, 128, P, C, 0, 0, None, 0,
                                                   None, side.cuda_stream)
    assert code == 0
    for _ in range(2):
        out.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    del graph


def test_no_alloc_rejects_bad_arguments(gpu):
    import ulysses_sequence_attention_repack_b200 as U
    lib = U.load()
    from ulysses_sequence_attention_repack_b200 import _lib
    st = ctypes.c_int32(0)
    # D != 128, heads not divisible by ranks, gate-less pack, too many sequences
    assert lib.ulysses_layer_fwd_fused_noalloc(0x10000, 0x90000000, 64, 8, 64, 2, 3, 0, 0, None, 0,
                                               ctypes.byref(st), None) == _lib.ULYSSES_ERR_UNSUPPORTED
    assert lib.ulysses_layer_fwd_fused_noalloc(0x10000, 0x90000000, 64, 6, 128, 4, 3, 0, 0, None, 0,
                                               ctypes.byref(st), None) == _lib.ULYSSES_ERR_DIVISIBILITY
    assert lib.ulysses_layer_fwd_fused_noalloc(0x10000, 0x90000000, 64, 8, 128, 2, 2, 0, 0, None, 0,
                                               ctypes.byref(st), None) == _lib.ULYSSES_ERR_ARG
    many = (ctypes.c_int32 * 66)(*range(66))
    assert lib.ulysses_layer_fwd_fused_noalloc(0x10000, 0x90000000, 65, 8, 128, 1, 3, 0, 0, many, 65,
                                               ctypes.byref(st), None) == _lib.ULYSSES_ERR_UNSUPPORTED
