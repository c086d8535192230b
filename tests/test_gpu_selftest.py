"""Device helpers of the attention kernel checked on their own."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def test_fma_pipe_exp2_relative_error(gpu):
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    x = torch.cat([torch.linspace(-125.0, 8.0, 1_000_001, dtype=torch.float32),
                   torch.tensor([0.0, -0.5, 0.5, -1.0, 1.0, 7.999, -124.5], dtype=torch.float32)]).to(gpu)
    y = torch.empty_like(x)
    U.ulysses_selftest_exp2_poly(x, y)
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
    U.ulysses_selftest_exp2_poly(xi, yi)
    torch.cuda.synchronize()
    assert np.allclose(yi.cpu().numpy() / np.exp2(ints.astype(np.float64)), 9.999280572e-01, rtol=1e-7)


def test_fma_pipe_exp2_clamps_below_range(gpu):
    import torch
    import ulysses_sequence_attention_repack_b200 as U
    x = torch.tensor([-126.0, -200.0, -1e30, float("-inf")], dtype=torch.float32, device=gpu)
    y = torch.empty_like(x)
    U.ulysses_selftest_exp2_poly(x, y)
    torch.cuda.synchronize()
    got = y.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got)) and np.all(got > 0) and np.all(got <= 2.0 ** -124)
