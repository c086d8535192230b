// Ulysses exchange across P real GPUs, one process per GPU: each rank pushes
// its rows into the other ranks' buffers with plain 16-byte stores through
// peer pointers (CUDA IPC mappings over NVLink, or local buffers when the
// ranks are emulated on one GPU).  This is the all-to-all of "Ulysses
// performance on GB200" (fine-grained remote stores into each peer's window,
// one plane at a time), written for NVSwitch, where every peer is reached at
// full bandwidth: no staging buffer, no TMA and no multicast on peer memory.
//
//   mode 0, pushed by rank q (shard S_q [Nl, C, H, D], rows q*Nl + i):
//       T_r[c, q*Nl + i, j, d] = S_q[i, c, r*Hl + j, d]        for every r
//   mode 1, pushed by rank r (head rows O_r [Cp, Np, Hl, D]):
//       O_q[i, c, r*Hl + j, d] = O_r[c, q*Nl + i, j, d]        for every q
//
// One warp moves one contiguous source run (a token's H*D values in mode 0,
// a token's Hl*D values in mode 1) with 16-byte loads, UNROLL in flight per
// lane, and 16-byte stores to the destination rank's buffer.
#include <cuda_runtime.h>

#include <cstdint>

#include "bounds.cuh"
#include "internal.h"

namespace ulysses {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 8;
constexpr int kMaxHeads = 1024;

__device__ __forceinline__ int4 ld_stream(const int4* p) {
  int4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.s32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_vec(int4* p, int4 v) {
  asm volatile("st.global.v4.s32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// mode 0: rows = Nl * cc runs of H*D elements; head h of (i, c) goes to
// rank h / Hl at element ((c*Np + q*Nl + i)*Hl + h % Hl)*D.  src_vecs /
// dst_vecs: extents in 16-byte vectors of the shard and of each rank's
// destination, for the bounds-checked build only (bounds.cuh).
__global__ void __launch_bounds__(kThreads) push_fwd_kernel(const int4* __restrict__ src, PushTable dst,
                                                            int64_t Nl, int64_t Np, int32_t H, int32_t Hl,
                                                            int32_t C, int32_t c0, int32_t cc, int32_t rank,
                                                            int64_t src_vecs, int64_t dst_vecs, unsigned int* err) {
  __shared__ int4* head_base[kMaxHeads];   // rank r's buffer + j*D (16-byte units)
  constexpr int D = 128;
  for (int h = threadIdx.x; h < H; h += blockDim.x) {
    const int r = h / Hl, j = h - (h / Hl) * Hl;
    head_base[h] = static_cast<int4*>(dst.p[r]) + j * (D / 8);
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t rows = Nl * cc;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int vec_per_row = H * (D / 8);
  for (int64_t row = warp0; row < rows; row += nwarps) {
    const int c = c0 + static_cast<int>(row / Nl);
    const int64_t i = row - (row / Nl) * Nl;
    const int64_t src_vec = (i * C + c) * static_cast<int64_t>(H) * (D / 8);
    const int64_t dst_vec = (static_cast<int64_t>(c) * Np + static_cast<int64_t>(rank) * Nl + i) * Hl * (D / 8);
    for (int k0 = 0; k0 < vec_per_row; k0 += 32 * kUnroll) {
      int4 v[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int k = k0 + u * 32 + lane;
        if (k < vec_per_row) {
          v[u] = make_int4(0, 0, 0, 0);
          if (in_bounds(src_vec + k, 1, src_vecs, err)) v[u] = ld_stream(src + src_vec + k);
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int k = k0 + u * 32 + lane;
        if (k < vec_per_row) {
          const int h = k >> 4;
          const int64_t rel = static_cast<int64_t>(h - (h / Hl) * Hl) * (D / 8) + dst_vec + (k & 15);
          if (in_bounds(rel, 1, dst_vecs, err)) st_vec(head_base[h] + dst_vec + (k & 15), v[u]);
        }
      }
    }
  }
}

// mode 1: rows = Np * cc runs of Hl*D elements (source [Cp, Np, Hl, D]); row n
// of plane c goes to rank q = n / Nl at element (((n - q*Nl)*Cp + c)*H + r*Hl)*D.
__global__ void __launch_bounds__(kThreads) push_bwd_kernel(const int4* __restrict__ src, PushTable dst,
                                                            int64_t Nl, int64_t Np, int32_t H, int32_t Hl,
                                                            int32_t Cp, int32_t c0, int32_t cc, int32_t rank,
                                                            int32_t nranks, int64_t src_vecs, int64_t dst_vecs,
                                                            unsigned int* err) {
  constexpr int D = 128;
  const int lane = threadIdx.x & 31;
  const int64_t rows = Np * cc;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int vec_per_row = Hl * (D / 8);
  for (int64_t row = warp0; row < rows; row += nwarps) {
    const int c = c0 + static_cast<int>(row / Np);
    const int64_t n = row - (row / Np) * Np;
    const int q = static_cast<int>(n / Nl);
    const int64_t i = n - q * Nl;
    const int64_t src_vec = (static_cast<int64_t>(c) * Np + n) * vec_per_row;
    const int64_t out_vec = ((i * Cp + c) * H + static_cast<int64_t>(rank) * Hl) * (D / 8);
    if (!in_bounds(q, 1, nranks, err)) continue;   // a table entry past the ranks in use
    int4* out = static_cast<int4*>(dst.p[q]) + out_vec;
    for (int k0 = 0; k0 < vec_per_row; k0 += 32 * kUnroll) {
      int4 v[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int k = k0 + u * 32 + lane;
        if (k < vec_per_row) {
          v[u] = make_int4(0, 0, 0, 0);
          if (in_bounds(src_vec + k, 1, src_vecs, err)) v[u] = ld_stream(src + src_vec + k);
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int k = k0 + u * 32 + lane;
        if (k < vec_per_row && in_bounds(out_vec + k, 1, dst_vecs, err)) st_vec(out + k, v[u]);
      }
    }
  }
}

int grid_for(int64_t rows) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int warps_per_cta = kThreads / 32;
  const int64_t want = (rows + warps_per_cta - 1) / warps_per_cta;
  return static_cast<int>(want < static_cast<int64_t>(sms) * 8 ? want : static_cast<int64_t>(sms) * 8);
}

}  // namespace

cudaError_t launch_push(int dir, const void* src, const PushTable& dst, int64_t Nl, int64_t Np, int32_t H,
                        int32_t P, int32_t C, int32_t c0, int32_t cc, int32_t rank, cudaStream_t stream,
                        unsigned int* err) {
  if (H > kMaxHeads || P < 1 || P > ULYSSES_MAX_PUSH_RANKS || H % P != 0 || rank < 0 || rank >= P)
    return cudaErrorInvalidValue;
  const int64_t rows = (dir == 0 ? Nl : Np) * cc;
  if (rows == 0) return cudaSuccess;
  const int grid = grid_for(rows);
  const int64_t Hl = H / P;
  // extents in 16-byte vectors: shard [Nl, C, H, D] and head slab [C, Np, Hl, D]
  const int64_t shard_vecs = Nl * C * H * 16, slab_vecs = static_cast<int64_t>(C) * Np * Hl * 16;
  if (dir == 0)
    push_fwd_kernel<<<grid, kThreads, 0, stream>>>(static_cast<const int4*>(src), dst, Nl, Np, H, H / P, C, c0,
                                                   cc, rank, shard_vecs, slab_vecs, err);
  else
    push_bwd_kernel<<<grid, kThreads, 0, stream>>>(static_cast<const int4*>(src), dst, Nl, Np, H, H / P, C, c0,
                                                   cc, rank, P, slab_vecs, shard_vecs, err);
  return cudaGetLastError();
}

}  // namespace ulysses
