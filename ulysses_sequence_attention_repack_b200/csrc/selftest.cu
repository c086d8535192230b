// Self-test entry points: device helpers of the attention kernel exposed on
// their own so tests can check them against reference values.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/ulysses_selftest.h"
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

}  // namespace

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
