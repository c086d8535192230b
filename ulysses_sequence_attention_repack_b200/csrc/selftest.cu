// Self-test entry points: device helpers of the attention kernel exposed on
// their own so tests can check them against reference values.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/ulysses_selftest.h"
#include "bounds.cuh"
#include "exp2_poly.cuh"

namespace {

__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
  const int64_t i = 2 * (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const ulysses::f2 r = ulysses::exp2_poly2(ulysses::f2{x[i], x[i + 1]});
    y[i] = r.x;
    y[i + 1] = r.y;
  } else if (i < n) {
    y[i] = ulysses::exp2_poly2(ulysses::f2{x[i], x[i]}).x;
  }
}

// One CTA waits on an mbarrier phase that nothing completes, once with the
// single-thread wait and once with the warp-collective wait, each bounded by
// limit_ns.  Both must give up, set kErrWaitTimeout in *err, and return.
__global__ void wait_timeout_kernel(unsigned int* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ulysses::mbar_init(ulysses::smem_u32(&bar), 1);
    abort_flag = 0;
    ulysses::fence_mbar_init();
  }
  __syncthreads();
  ulysses::WaitGuard g{&abort_flag, err, limit_ns};
  if (threadIdx.x == 0) {
    if (!ulysses::mbar_wait(ulysses::smem_u32(&bar), 0, g)) atomicOr(err, 0x100u);
    abort_flag = 0;   // re-arm so the warp-wide wait also runs its own limit
  }
  __syncwarp();
  if (!ulysses::mbar_wait_warp(ulysses::smem_u32(&bar), 0, g) && threadIdx.x == 0) atomicOr(err, 0x200u);
}

}  // namespace

extern "C" int ulysses_selftest_wait_timeout(unsigned int* dev_err, int64_t limit_us, void* stream) {
  if (!dev_err || limit_us < 1 || limit_us > 1000000) return 1;
  wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(dev_err,
                                                                      static_cast<uint64_t>(limit_us) * 1000u);
  return cudaGetLastError() == cudaSuccess ? 0 : 6;
}

extern "C" int ulysses_selftest_exp2_poly(const float* x, float* y, int64_t n, void* stream) {
  if (!x || !y || n < 0) return 1;
  if (n == 0) return 0;
  const int64_t pairs = (n + 1) / 2;
  const int threads = 256;
  const int64_t blocks = (pairs + threads - 1) / threads;
  if (blocks > 0x7fffffff) return 1;
  exp2_poly_kernel<<<static_cast<unsigned>(blocks), threads, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? 0 : 6;
}

namespace {

// The range check of the bounds-checked build, forced on: three offsets
// against an extent of 100 elements, of which only the first is inside.  No
// memory is touched; the results land in *err next to kErrBounds.
__global__ void bounds_check_kernel(unsigned int* err) {
  if (threadIdx.x != 0) return;
  if (ulysses::in_bounds<true>(0, 8, 100, err)) atomicOr(err, 0x10u);
  if (!ulysses::in_bounds<true>(-8, 8, 100, err)) atomicOr(err, 0x20u);
  if (!ulysses::in_bounds<true>(96, 8, 100, err)) atomicOr(err, 0x40u);
}

}  // namespace

extern "C" int ulysses_selftest_bounds_check(unsigned int* dev_err, void* stream) {
  if (!dev_err) return 1;
  bounds_check_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(dev_err);
  return cudaGetLastError() == cudaSuccess ? 0 : 6;
}
