"""Device helpers of the attention kernel checked on their own."""
import _selftest_lib
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def test_fma_pipe_exp2_relative_error(gpu):
    import torch
    x = torch.cat([torch.linspace(-125.0, 8.0, 1_000_001, dtype=torch.float32),
                   torch.tensor([0.0, -0.5, 0.5, -1.0, 1.0, 7.999, -124.5], dtype=torch.float32)]).to(gpu)
    y = torch.empty_like(x)
    _selftest_lib.exp2_poly(x, y)
    torch.cuda.synchronize()
    xs = x.cpu().numpy().astype(np.float64)
    ref = np.exp2(xs)
    rel = np.abs(y.cpu().numpy().astype(np.float64) / ref - 1.0)
    # polynomial error 7.5e-5 plus fp32 rounding of the Horner steps
    assert rel.max() < 1.0e-4, rel.max()
    # integer arguments are exact powers of two up to the polynomial's value at 0
    ints = np.arange(-125, 9, dtype=np.float32)
    xi = torch.from_numpy(ints).to(gpu)
    yi = torch.empty_like(xi)
    _selftest_lib.exp2_poly(xi, yi)
    torch.cuda.synchronize()
    assert np.allclose(yi.cpu().numpy() / np.exp2(ints.astype(np.float64)), 9.999280572e-01, rtol=1e-7)


def test_fma_pipe_exp2_clamps_below_range(gpu):
    import torch
    x = torch.tensor([-126.0, -200.0, -1e30, float("-inf")], dtype=torch.float32, device=gpu)
    y = torch.empty_like(x)
    _selftest_lib.exp2_poly(x, y)
    torch.cuda.synchronize()
    got = y.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got)) and np.all(got > 0) and np.all(got <= 2.0 ** -124)


def test_bounded_wait_gives_up_and_reports(gpu):
    """A wait on a phase nothing completes returns after its limit with the error bits set."""
    import math
    import time

    import torch
    import ulysses_sequence_attention_repack_b200 as U
    lib = _selftest_lib.load()
    err = torch.zeros(4, dtype=torch.int32, device=gpu)
    t0 = time.time()
    assert lib.ulysses_selftest_wait_timeout(err.data_ptr(), 20_000, torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    word = int(err[0].item())
    assert word & 1, word                      # kErrWaitTimeout
    assert word & 0x100 and word & 0x200, hex(word)
    assert elapsed < 5.0
    # the context is still usable: a small layer still matches the fused path
    from ulysses_sequence_attention_repack_b200 import inputs
    plan = U.ulysses_plan(300, 4, 128, 2, 3)
    S = inputs.qkv_seq(300, 4, 2, 3, 3, gpu)
    a = torch.empty((300, 4, 128), dtype=torch.bfloat16, device=gpu)
    b = torch.empty_like(a)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=gpu)
    U.ulysses_layer_fwd(plan, S, a, ws, fused=0)
    U.ulysses_layer_fwd(plan, S, b, None, fused=1)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and U.ulysses_last_device_error(plan) == 0
    assert math.isfinite(float(a.float().abs().sum()))
