"""Loader of libulysses_selftest.so, the library of test hooks (device helpers
of the kernels run on their own), built beside libulysses.so by the package's
build step.  Test infrastructure only."""
import ctypes

SELFTEST_EXPORTS = ("ulysses_selftest_exp2_poly", "ulysses_selftest_wait_timeout", "ulysses_selftest_bounds_check")


def load():
    from ulysses_sequence_attention_repack_b200 import build
    build.ensure_built()
    lib = ctypes.CDLL(build.SELFTEST_LIB)
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    lib.ulysses_selftest_exp2_poly.argtypes = [vp, vp, i64, vp]
    lib.ulysses_selftest_exp2_poly.restype = ctypes.c_int
    lib.ulysses_selftest_wait_timeout.argtypes = [vp, i64, vp]
    lib.ulysses_selftest_wait_timeout.restype = ctypes.c_int
    lib.ulysses_selftest_bounds_check.argtypes = [vp, vp]
    lib.ulysses_selftest_bounds_check.restype = ctypes.c_int
    return lib


def exp2_poly(x, y):
    """y = 2^x with the attention kernel's FMA-pipe exponential (float32 device tensors)."""
    import torch
    code = load().ulysses_selftest_exp2_poly(x.data_ptr(), y.data_ptr(), int(x.numel()),
                                             torch.cuda.current_stream().cuda_stream)
    if code != 0:
        raise RuntimeError(f"ulysses_selftest_exp2_poly: error {code}")
