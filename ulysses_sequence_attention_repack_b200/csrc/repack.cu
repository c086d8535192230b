// Ulysses repack on one GPU: the all-to-all index map between the
// sequence-sharded layout and the head-sharded layout.
//
//   mode 0 (dir = 0): T[r, c, n, j, d] = S[n, c, r*Hl + j, d]
//   mode 1 (dir = 1): S[n, c, r*Hl + j, d] = T[r, c, n, j, d]
//
// Shapes follow the mode comment above ulysses_a2a_tuned ("hao-ai-lab
// FastVideo, compare main...perf/ulysses-h3-adaptive",
// csrc/comm/ulysses_all_to_all.cu): [B, S_local, H, D] <-> [B, S_global, H_local, D],
// with each of the P source slabs contributing its rows in rank order.
//
// Pure data movement, HBM bound.  For one (token n, plane c) the sequence side
// is one contiguous run of H*D*2 bytes; it splits into P contiguous runs of
// Hl*D*2 bytes on the head side.  One warp moves one (n, c) run with 16-byte
// vector loads and stores: 32 lanes cover 512 contiguous bytes per step on
// both sides, and every lane keeps kUnroll loads in flight before storing.
// Destination offsets of each head are precomputed in shared memory so the
// inner loop has no division.
#include <cuda_runtime.h>

#include <cstdint>

#include "bounds.cuh"
#include "internal.h"

namespace ulysses {
namespace {

constexpr int kRepackThreads = 256;
// 16 loads in flight per lane (~100 registers, no spills): 3.6% faster at
// the Video-DiT size than 8 (64 registers, with spills in two kernels)
constexpr int kUnroll = 16;
constexpr int kMaxHeads = 1024;

__device__ __forceinline__ int4 ld_stream(const int4* p) {
  int4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.s32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_stream(int4* p, int4 v) {
  asm volatile("st.global.cs.v4.s32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// Element offsets are int64 throughout: the largest head-sharded buffer holds
// 7.2e9 elements.  src_ext / dst_ext are the buffers' extents in elements,
// used by the bounds-checked build only (bounds.cuh).
template <int DIR>
__global__ void __launch_bounds__(kRepackThreads) repack_kernel(const int4* __restrict__ src,
                                                                int4* __restrict__ dst, int64_t Np, int32_t H,
                                                                int32_t Hl, int32_t Ctot, int32_t c0, int32_t cc,
                                                                int64_t tok_stride, int64_t plane_stride,
                                                                int64_t src_ext, int64_t dst_ext,
                                                                unsigned int* err) {
  // head_off[h]: element offset of head h's run inside a head-sharded row,
  // relative to T[0, c, n, 0, 0]: r*Ctot*Np*Hl*D + j*D with r = h / Hl, j = h % Hl.
  __shared__ int64_t head_off[kMaxHeads];
  constexpr int D = 128;
  const int64_t rank_stride = static_cast<int64_t>(Ctot) * Np * Hl * D;
  for (int h = threadIdx.x; h < H; h += blockDim.x) {
    const int r = h / Hl, j = h - (h / Hl) * Hl;
    head_off[h] = r * rank_stride + static_cast<int64_t>(j) * D;
  }
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int64_t rows = Np * cc;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int vec_per_row = H * (D / 8);   // 16-byte vectors in one (n, c) run

  for (int64_t row = warp0; row < rows; row += nwarps) {
    // plane-major over the chunk: consecutive warps take consecutive tokens
    const int c = c0 + static_cast<int>(row / Np);
    const int64_t n = row - (row / Np) * Np;
    const int64_t seq_base = n * tok_stride + c * plane_stride;                 // elements
    const int64_t head_base = (static_cast<int64_t>(c) * Np + n) * Hl * D;       // elements, + head_off[h]
    for (int k0 = 0; k0 < vec_per_row; k0 += 32 * kUnroll) {
      int4 v[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int k = k0 + u * 32 + lane;
        if (k < vec_per_row) {
          const int h = k >> 4;
          const int64_t seq_off = seq_base + static_cast<int64_t>(k) * 8;
          const int64_t head_el = head_base + head_off[h] + (k & 15) * 8;
          const int64_t s_el = DIR == 0 ? seq_off : head_el;
          v[u] = make_int4(0, 0, 0, 0);
          if (in_bounds(s_el, 8, src_ext, err)) v[u] = ld_stream(src + (s_el >> 3));
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int k = k0 + u * 32 + lane;
        if (k < vec_per_row) {
          const int h = k >> 4;
          const int64_t seq_off = seq_base + static_cast<int64_t>(k) * 8;
          const int64_t head_el = head_base + head_off[h] + (k & 15) * 8;
          const int64_t d_el = DIR == 0 ? head_el : seq_off;
          if (in_bounds(d_el, 8, dst_ext, err)) st_stream(dst + (d_el >> 3), v[u]);
        }
      }
    }
  }
}

// Mode 0 with the E4M3 cast of the FP8 attention variant:
//   T8[r, c, n, j, d] = e4m3(S[n, c, r*Hl + j, d])
// Same traversal as repack_kernel<0>; each 16-byte load of 8 bf16 values
// becomes one 8-byte store of 8 E4M3 codes (round to nearest even,
// saturating at +-448: cvt.rn.satfinite).
__device__ __forceinline__ uint32_t e4m3x4(uint32_t w01, uint32_t w23) {
  uint16_t a, b;
  // each 32-bit word holds two bf16 values, the lower-indexed one in bits 0-15;
  // cvt puts its first source in the high byte
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
      : "=h"(a)
      : "f"(__uint_as_float(w01 & 0xFFFF0000u)), "f"(__uint_as_float(w01 << 16)));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
      : "=h"(b)
      : "f"(__uint_as_float(w23 & 0xFFFF0000u)), "f"(__uint_as_float(w23 << 16)));
  return static_cast<uint32_t>(a) | (static_cast<uint32_t>(b) << 16);
}

__global__ void __launch_bounds__(kRepackThreads) repack_fp8_kernel(const int4* __restrict__ src,
                                                                    uint2* __restrict__ dst, int64_t Np,
                                                                    int32_t H, int32_t Hl, int32_t Ctot,
                                                                    int32_t c0, int32_t cc, int64_t tok_stride,
                                                                    int64_t plane_stride, int64_t src_ext,
                                                                    int64_t dst_ext, unsigned int* err) {
  __shared__ int64_t head_off[kMaxHeads];
  constexpr int D = 128;
  const int64_t rank_stride = static_cast<int64_t>(Ctot) * Np * Hl * D;
  for (int h = threadIdx.x; h < H; h += blockDim.x) {
    const int r = h / Hl, j = h - (h / Hl) * Hl;
    head_off[h] = r * rank_stride + static_cast<int64_t>(j) * D;
  }
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int64_t rows = Np * cc;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int vec_per_row = H * (D / 8);

  for (int64_t row = warp0; row < rows; row += nwarps) {
    const int c = c0 + static_cast<int>(row / Np);
    const int64_t n = row - (row / Np) * Np;
    const int64_t seq_base = n * tok_stride + c * plane_stride;
    const int64_t head_base = (static_cast<int64_t>(c) * Np + n) * Hl * D;
    for (int k0 = 0; k0 < vec_per_row; k0 += 32 * kUnroll) {
      int4 v[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int k = k0 + u * 32 + lane;
        if (k < vec_per_row) {
          const int64_t s_el = seq_base + static_cast<int64_t>(k) * 8;
          v[u] = make_int4(0, 0, 0, 0);
          if (in_bounds(s_el, 8, src_ext, err)) v[u] = ld_stream(src + (s_el >> 3));
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int k = k0 + u * 32 + lane;
        if (k < vec_per_row) {
          const int64_t head_el = head_base + head_off[k >> 4] + (k & 15) * 8;   // one byte per element
          uint2 o;
          o.x = e4m3x4(static_cast<uint32_t>(v[u].x), static_cast<uint32_t>(v[u].y));
          o.y = e4m3x4(static_cast<uint32_t>(v[u].z), static_cast<uint32_t>(v[u].w));
          if (in_bounds(head_el, 8, dst_ext, err)) dst[head_el >> 3] = o;
        }
      }
    }
  }
}

// Extents (elements) of the two sides of one repack launch: the
// sequence-sharded buffer as its strides span it over Ctot planes, and the
// head-sharded [P, Ctot, Np, Hl, D] buffer.
inline int64_t seq_extent(int64_t Np, int32_t H, int32_t Ctot, int64_t tok_stride, int64_t plane_stride) {
  return (Np - 1) * tok_stride + static_cast<int64_t>(Ctot - 1) * plane_stride + static_cast<int64_t>(H) * 128;
}
inline int64_t head_extent(int64_t Np, int32_t H, int32_t Ctot) {
  return static_cast<int64_t>(Ctot) * Np * H * 128;
}

}  // namespace

cudaError_t launch_repack_fp8(const void* src, void* dst, int64_t Np, int32_t H, int32_t P, int32_t Ctot,
                              int32_t c0, int32_t cc, int64_t tok_stride, int64_t plane_stride,
                              cudaStream_t stream, unsigned int* err) {
  if (H > kMaxHeads || P < 1 || H % P != 0) return cudaErrorInvalidValue;
  const int64_t rows = Np * cc;
  if (rows == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int warps_per_cta = kRepackThreads / 32;
  const int64_t want = (rows + warps_per_cta - 1) / warps_per_cta;
  const int grid = static_cast<int>(want < static_cast<int64_t>(sms) * 8 ? want : static_cast<int64_t>(sms) * 8);
  repack_fp8_kernel<<<grid, kRepackThreads, 0, stream>>>(static_cast<const int4*>(src), static_cast<uint2*>(dst),
                                                         Np, H, H / P, Ctot, c0, cc, tok_stride, plane_stride,
                                                         seq_extent(Np, H, Ctot, tok_stride, plane_stride),
                                                         head_extent(Np, H, Ctot), err);
  return cudaGetLastError();
}

cudaError_t launch_repack(int dir, const void* src, void* dst, int64_t Np, int32_t H, int32_t P, int32_t Ctot,
                          int32_t c0, int32_t cc, int64_t tok_stride, int64_t plane_stride, cudaStream_t stream,
                          unsigned int* err) {
  if (H > kMaxHeads || P < 1 || H % P != 0) return cudaErrorInvalidValue;
  const int64_t rows = Np * cc;
  if (rows == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int warps_per_cta = kRepackThreads / 32;
  // persistent grid: 8 resident CTAs of 256 threads per SM
  const int64_t want = (rows + warps_per_cta - 1) / warps_per_cta;
  const int grid = static_cast<int>(want < static_cast<int64_t>(sms) * 8 ? want : static_cast<int64_t>(sms) * 8);
  const int Hl = H / P;
  const int64_t seq_ext = seq_extent(Np, H, Ctot, tok_stride, plane_stride);
  const int64_t head_ext = head_extent(Np, H, Ctot);
  if (dir == 0) {
    repack_kernel<0><<<grid, kRepackThreads, 0, stream>>>(static_cast<const int4*>(src), static_cast<int4*>(dst),
                                                          Np, H, Hl, Ctot, c0, cc, tok_stride, plane_stride,
                                                          seq_ext, head_ext, err);
  } else {
    repack_kernel<1><<<grid, kRepackThreads, 0, stream>>>(static_cast<const int4*>(src), static_cast<int4*>(dst),
                                                          Np, H, Hl, Ctot, c0, cc, tok_stride, plane_stride,
                                                          head_ext, seq_ext, err);
  }
  return cudaGetLastError();
}

}  // namespace ulysses
