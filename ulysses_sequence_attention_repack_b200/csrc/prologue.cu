// QKV prologue fused into the Ulysses repack (mode 0): per-head RMSNorm and
// partial rotate-half RoPE on the Q and K planes, V (and a gate plane) copied,
// written straight into the head-sharded layout
//
//   T[r, c, n, j, :] = prologue(S[n, c, r*Hl + j, :])
//
// The prologue is the one of "hao-ai-lab FastVideo, compare
// aryan/h3-nvfp4-stack-speedups...main", mk/qkv_prologue.py: for one 128-wide
// (token, head) row of Q or K,
//   y = x / sqrt(mean(x^2) + eps) * w
//   y[i] <- y[i] cos[n, i] - y[i + rd/2] sin[n, i]          i <  rd/2
//   y[i] <- y[i] cos[n, i] + y[i - rd/2] sin[n, i]          rd/2 <= i < rd
// with channels >= rd untouched; fp32 arithmetic, one bf16 rounding at the
// store.  Fusing it with the repack removes a full read and write of Q and K:
// the kernel moves exactly the bytes the plain repack moves.
//
// Work layout: one warp per (token, plane) row, as in repack.cu.  For the Q
// and K planes each half-warp owns one head (16 lanes x 8 channels = 128):
// the sum of squares is reduced with four xor-shuffles inside the half-warp
// and the rotate-half partner of a lane's 8 channels lives rd/16 lanes away
// in the same half-warp, so it is one shuffle per value.  cos / sin / weights
// are loaded once per row and reused for all heads.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "bounds.cuh"
#include "internal.h"

namespace ulysses {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxHeads = 1024;
constexpr int HD = 128;

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

__device__ __forceinline__ void unpack8(int4 v, float (&f)[8]) {
  const uint32_t w[4] = {static_cast<uint32_t>(v.x), static_cast<uint32_t>(v.y), static_cast<uint32_t>(v.z),
                         static_cast<uint32_t>(v.w)};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

struct PrologueArgs {
  const int4* src;
  int4* dst;
  const uint16_t* wq;
  const uint16_t* wk;
  const uint16_t* cos;
  const uint16_t* sin;
  int64_t Np;
  int64_t tok_stride, plane_stride;   // elements, sequence side
  int32_t H, Hl, Ctot, c0, cc;
  int32_t rd;                         // rotary dims (multiple of 16, <= 128)
  float eps;
  // extents in elements, for the bounds-checked build only (bounds.cuh):
  // sequence side, head side, and the cos / sin tables [Np, rd]
  int64_t src_ext, dst_ext, table_ext;
  unsigned int* err;
};

__global__ void __launch_bounds__(kThreads) prologue_repack_kernel(const PrologueArgs a) {
  __shared__ int64_t head_off[kMaxHeads];
  const int64_t rank_stride = static_cast<int64_t>(a.Ctot) * a.Np * a.Hl * HD;
  for (int h = threadIdx.x; h < a.H; h += blockDim.x) {
    const int r = h / a.Hl, j = h - (h / a.Hl) * a.Hl;
    head_off[h] = r * rank_stride + static_cast<int64_t>(j) * HD;
  }
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int half = lane >> 4;          // which head of the pair
  const int ch = lane & 15;            // 8-channel chunk of the head
  const int rd8 = a.rd >> 3;           // chunks under RoPE
  const int hd8 = a.rd >> 4;           // partner distance in chunks (rd/2 / 8)
  const bool rot_lo = ch < hd8, rot_hi = ch >= hd8 && ch < rd8;
  const int partner = rot_lo ? lane + hd8 : (rot_hi ? lane - hd8 : lane);

  const int64_t rows = a.Np * a.cc;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;

  for (int64_t row = warp0; row < rows; row += nwarps) {
    const int c = a.c0 + static_cast<int>(row / a.Np);
    const int64_t n = row - (row / a.Np) * a.Np;
    const int64_t seq_base = n * a.tok_stride + c * a.plane_stride;
    const int64_t head_base = (static_cast<int64_t>(c) * a.Np + n) * a.Hl * HD;

    if (c >= 2) {   // V / gate: plain 16-byte copy, as in the repack
      const int vec_per_row = a.H * (HD / 8);
      for (int k0 = 0; k0 < vec_per_row; k0 += 32 * 8) {
        int4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int k = k0 + u * 32 + lane;
          if (k < vec_per_row) {
            const int64_t s_el = seq_base + static_cast<int64_t>(k) * 8;
            v[u] = make_int4(0, 0, 0, 0);
            if (in_bounds(s_el, 8, a.src_ext, a.err)) v[u] = ld_stream(a.src + (s_el >> 3));
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int k = k0 + u * 32 + lane;
          if (k < vec_per_row) {
            const int64_t d_el = head_base + head_off[k >> 4] + (k & 15) * 8;
            if (in_bounds(d_el, 8, a.dst_ext, a.err)) st_stream(a.dst + (d_el >> 3), v[u]);
          }
        }
      }
      continue;
    }

    // Q or K: this lane's norm weights and its token's cos / sin chunk
    float w[8], cs[8], sn[8];
    {
      const uint16_t* wp = (c == 0 ? a.wq : a.wk) + ch * 8;
      unpack8(*reinterpret_cast<const int4*>(wp), w);
      if (ch < rd8) {
        const int64_t t_el = n * a.rd + ch * 8;
        const bool ok = in_bounds(t_el, 8, a.table_ext, a.err);
        unpack8(ok ? *reinterpret_cast<const int4*>(a.cos + t_el) : make_int4(0, 0, 0, 0), cs);
        unpack8(ok ? *reinterpret_cast<const int4*>(a.sin + t_el) : make_int4(0, 0, 0, 0), sn);
        if (rot_lo) {
#pragma unroll
          for (int e = 0; e < 8; ++e) sn[e] = -sn[e];   // y[i] cos - y[i + rd/2] sin
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          cs[e] = 1.0f;
          sn[e] = 0.0f;
        }
      }
    }
    constexpr int kPairs = 8;   // head pairs in flight per lane (4: 359 us, 8: 303 us, 14: 411 us at dit19k)
    for (int hp0 = 0; hp0 < a.H; hp0 += 2 * kPairs) {
      int4 v[kPairs];
#pragma unroll
      for (int u = 0; u < kPairs; ++u) {
        const int h = hp0 + 2 * u + half;
        v[u] = make_int4(0, 0, 0, 0);
        const int64_t s_el = seq_base + static_cast<int64_t>(h) * HD + ch * 8;
        if (h < a.H && in_bounds(s_el, 8, a.src_ext, a.err)) v[u] = ld_stream(a.src + (s_el >> 3));
      }
#pragma unroll
      for (int u = 0; u < kPairs; ++u) {
        const int h = hp0 + 2 * u + half;
        float x[8];
        unpack8(v[u], x);
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
        ss += __shfl_xor_sync(0xffffffffu, ss, 8);
        ss += __shfl_xor_sync(0xffffffffu, ss, 4);
        ss += __shfl_xor_sync(0xffffffffu, ss, 2);
        ss += __shfl_xor_sync(0xffffffffu, ss, 1);
        const float inv = rsqrtf(ss * (1.0f / HD) + a.eps);
        float y[8], pr[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] = x[e] * inv * w[e];
#pragma unroll
        for (int e = 0; e < 8; ++e) pr[e] = __shfl_sync(0xffffffffu, y[e], partner);
        int4 o;
        o.x = static_cast<int>(pack2(fmaf(pr[0], sn[0], y[0] * cs[0]), fmaf(pr[1], sn[1], y[1] * cs[1])));
        o.y = static_cast<int>(pack2(fmaf(pr[2], sn[2], y[2] * cs[2]), fmaf(pr[3], sn[3], y[3] * cs[3])));
        o.z = static_cast<int>(pack2(fmaf(pr[4], sn[4], y[4] * cs[4]), fmaf(pr[5], sn[5], y[5] * cs[5])));
        o.w = static_cast<int>(pack2(fmaf(pr[6], sn[6], y[6] * cs[6]), fmaf(pr[7], sn[7], y[7] * cs[7])));
        if (h < a.H) {
          const int64_t d_el = head_base + head_off[h] + ch * 8;
          if (in_bounds(d_el, 8, a.dst_ext, a.err)) st_stream(a.dst + (d_el >> 3), o);
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_prologue_repack(const void* src, void* dst, const void* wq, const void* wk, const void* cos,
                                   const void* sin, int32_t rd, float eps, int64_t Np, int32_t H, int32_t P,
                                   int32_t Ctot, int32_t c0, int32_t cc, int64_t tok_stride, int64_t plane_stride,
                                   cudaStream_t stream, unsigned int* err) {
  if (H > kMaxHeads || P < 1 || H % P != 0) return cudaErrorInvalidValue;
  const int64_t rows = Np * cc;
  if (rows == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int warps_per_cta = kThreads / 32;
  const int64_t want = (rows + warps_per_cta - 1) / warps_per_cta;
  const int grid = static_cast<int>(want < static_cast<int64_t>(sms) * 8 ? want : static_cast<int64_t>(sms) * 8);
  PrologueArgs a;
  a.src = static_cast<const int4*>(src);
  a.dst = static_cast<int4*>(dst);
  a.wq = static_cast<const uint16_t*>(wq);
  a.wk = static_cast<const uint16_t*>(wk);
  a.cos = static_cast<const uint16_t*>(cos);
  a.sin = static_cast<const uint16_t*>(sin);
  a.Np = Np;
  a.tok_stride = tok_stride;
  a.plane_stride = plane_stride;
  a.H = H;
  a.Hl = H / P;
  a.Ctot = Ctot;
  a.c0 = c0;
  a.cc = cc;
  a.rd = rd;
  a.eps = eps;
  a.src_ext = (Np - 1) * tok_stride + static_cast<int64_t>(Ctot - 1) * plane_stride + static_cast<int64_t>(H) * HD;
  a.dst_ext = static_cast<int64_t>(Ctot) * Np * H * HD;
  a.table_ext = Np * rd;
  a.err = err;
  prologue_repack_kernel<<<grid, kThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace ulysses
