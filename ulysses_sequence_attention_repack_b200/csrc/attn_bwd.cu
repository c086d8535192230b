// Backward of the layer's attention step on sm_100a: given Q, K, V (head-
// sharded T), the output O, the output gradient dO and the forward's
// log-sum-exp, compute dQ, dK, dV of O = softmax(s Q K^T) V:
//
//   P = exp2(s log2e Q K^T - lse2)      (lse2 = m + log2 l from the forward)
//   dV = P^T dO,   dP = dO V^T,   dS = P o (dP - D),   D = rowsum(dO o O)
//   dQ = s dS K,   dK = s dS^T Q
//
// This is the gradient the Ulysses transport carries back: the FastVideo
// transport's _FusedUlyssesA2A.backward runs the inverse map on it under the
// forward's plan ("hao-ai-lab FastVideo, compare main...perf/ulysses-h3-
// adaptive", ulysses_a2a.py).
//
// Two passes, no atomics:
//   pass A (one CTA unit = 128 keys of one head and sequence, loop over query
//           blocks): S^T = K Q^T and dP^T = V dO^T into TMEM, then
//           P^T and dS^T (bf16, aliased over them), then
//           dV += P^T dO and dK += dS^T Q with A read from TMEM;
//   pass B (unit = 128 queries, loop over key blocks): S = Q K^T and
//           dP = dO V^T, then dS, then dQ += dS K.
// Both reuse the forward's machinery: TMA-fed 128B-swizzled tiles, grouped
// tcgen05 MMAs issued by one thread, one thread per TMEM lane for the
// elementwise step, bounded mbarrier waits.  Warps: 0-3 elementwise and
// epilogue, 4 MMA issuer, 5 TMA producer.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace ulysses {
namespace {

constexpr int kThreads = 256;
constexpr int kMmaWarp = 4;
constexpr int kTmaWarp = 5;
constexpr int BT = 128;                               // rows per tile (keys or queries)
constexpr int HD = 128;
constexpr uint32_t kHalfBytes = BT * 64 * 2;          // 16 KB swizzled box
constexpr uint32_t kTileBytes = 2 * kHalfBytes;       // 32 KB
constexpr int kStages = 2;
constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;

// shared memory map
constexpr uint32_t kOffF0 = 0;                                // fixed tile 0
constexpr uint32_t kOffF1 = kTileBytes;                       // fixed tile 1
constexpr uint32_t kOffX = 2 * kTileBytes;                    // [stage][X0, X1]
// pass A: per stage, 132 lse floats then 132 D floats, copied from the block
// start rounded down to a multiple of 4 (16-byte aligned bulk copies)
constexpr uint32_t kRowFloats = 132;
constexpr uint32_t kRowStageBytes = 2 * kRowFloats * 4;                // 1056
constexpr uint32_t kOffRow = kOffX + kStages * 2 * kTileBytes;
constexpr uint32_t kOffBar = kOffRow + kStages * kRowStageBytes;
enum {
  B_FFULL = 0, B_FEMPTY, B_XFULL0, B_XFULL1, B_XEMPTY0, B_XEMPTY1, B_SFULL, B_PFULL, B_OFULL, B_OEMPTY, B_DONE,
  B_COUNT
};
constexpr uint32_t kOffSlot = kOffBar + B_COUNT * 8;
constexpr uint32_t kOffAbort = kOffSlot + 4;
constexpr uint32_t kSmemBytes = kOffAbort + 4 + 1024;

// TMEM columns: A0 (S or S^T, then P^T / dS bf16), A1 (dP or dP^T, then dS^T), accumulators
constexpr uint32_t kColA0 = 0, kColA1 = 128, kColAcc0 = 256, kColAcc1 = 384;
constexpr uint32_t kIdescSS = idesc_bf16_f32(BT, BT, 0, 0);
constexpr uint32_t kIdescTS = idesc_bf16_f32(BT, HD, 0, 1);

struct SegB {
  int32_t start, end;      // the segment's rows [start, end)
  int32_t tile_end;        // rows this segment's units cover (Np for the segment ending at N)
  int32_t ntile;           // 128-row units per (rank, head)
  int32_t unit_base;
};

struct BwdParams {
  __nv_bfloat16* dqkv;     // [P, 3, Np, Hl, D]
  const float* lse;        // [P*Hl][ls]
  const float* delta;      // [P*Hl][ls]
  int64_t ls;              // row stride of lse / delta
  unsigned int* err;
  int32_t N, Np, Hl, P, causal;
  int32_t num_units, nseg;
  float scale, scale_log2;
  SegB seg[ULYSSES_MAX_SEQS];
};

struct UnitB {
  int seg, r, j, row0;     // row0: first key (pass A) or query (pass B) of the unit
};

__device__ __forceinline__ bool decode_b(const BwdParams& p, int u, UnitB& w) {
  int s = 0;
  while (s + 1 < p.nseg && u >= p.seg[s + 1].unit_base) ++s;
  const int local = u - p.seg[s].unit_base;
  const int nt = p.seg[s].ntile;
  const int rh = local / nt;
  const int tb = local - rh * nt;
  w.seg = s;
  w.r = rh / p.Hl;
  w.j = rh - w.r * p.Hl;
  w.row0 = p.seg[s].start + tb * BT;
  return local >= 0 && w.r < p.P;
}

// Streamed blocks of a unit: pass A visits query blocks [first, start + ceil((end - start)/128)),
// causal: only blocks holding queries >= the unit's first key; pass B visits
// key blocks of the segment, causal: up to the unit's last query.
template <bool kPassA>
__device__ __forceinline__ void stream_range(const BwdParams& p, const SegB& sd, const UnitB& w, int& first,
                                             int& count) {
  const int nblk = (sd.end - sd.start + BT - 1) / BT;
  if (kPassA) {
    first = p.causal ? (w.row0 - sd.start) / BT : 0;
    count = w.row0 < sd.end ? nblk - first : 0;       // pad-only units have nothing to accumulate
  } else {
    first = 0;
    const int hi = p.causal ? min(sd.end, w.row0 + BT) : sd.end;
    count = w.row0 < sd.end ? (hi - sd.start + BT - 1) / BT : 0;
  }
}

__device__ __forceinline__ bool drain_wait_b(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

// D[(r*Hl + j) * ls + n] = sum_d dO[r, n, j, d] * O[r, n, j, d] for n < Np.
// One half-warp per row: 16 lanes x 8 channels.
__global__ void __launch_bounds__(256) bwd_delta_kernel(const int4* __restrict__ out, const int4* __restrict__ dout,
                                                        float* __restrict__ delta, int64_t rows, int32_t Np,
                                                        int32_t Hl, int64_t ls) {
  const int64_t hw = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 4;
  const int64_t nhw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 4;
  const int ch = threadIdx.x & 15;
  for (int64_t row = hw; row < rows; row += nhw) {   // row = (r*Np + n)*Hl + j
    const int4 a = out[row * 16 + ch];
    const int4 b = dout[row * 16 + ch];
    const uint32_t wa[4] = {static_cast<uint32_t>(a.x), static_cast<uint32_t>(a.y), static_cast<uint32_t>(a.z),
                            static_cast<uint32_t>(a.w)};
    const uint32_t wb[4] = {static_cast<uint32_t>(b.x), static_cast<uint32_t>(b.y), static_cast<uint32_t>(b.z),
                            static_cast<uint32_t>(b.w)};
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc = fmaf(__uint_as_float(wa[i] << 16), __uint_as_float(wb[i] << 16), acc);
      acc = fmaf(__uint_as_float(wa[i] & 0xFFFF0000u), __uint_as_float(wb[i] & 0xFFFF0000u), acc);
    }
    // the two half-warps may run different trip counts: shuffle within the half only
    const unsigned hmask = 0xFFFFu << (threadIdx.x & 16);
    acc += __shfl_xor_sync(hmask, acc, 8);
    acc += __shfl_xor_sync(hmask, acc, 4);
    acc += __shfl_xor_sync(hmask, acc, 2);
    acc += __shfl_xor_sync(hmask, acc, 1);
    if (ch == 0) {
      const int64_t j = row % Hl;
      const int64_t rn = row / Hl;
      const int64_t n = rn % Np, r = rn / Np;
      delta[(r * Hl + j) * ls + n] = acc;
    }
  }
}

template <bool kPassA>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kOffBar;
  auto BAR = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffSlot);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  WaitGuard g{abort_flag, p.err, kWaitLimitNs};

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(BAR(B_FFULL), 1);
    mbar_init(BAR(B_FEMPTY), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(BAR(B_XFULL0 + s), 1);
      mbar_init(BAR(B_XEMPTY0 + s), 1);
    }
    mbar_init(BAR(B_SFULL), 1);
    mbar_init(BAR(B_PFULL), BT);
    mbar_init(BAR(B_OFULL), 1);
    mbar_init(BAR(B_OEMPTY), BT);
    mbar_init(BAR(B_DONE), 1);
    fence_mbar_init();
  }
  if (warp == kTmaWarp && lane == 0) {
    prefetch_tmap(&tm_qkv);
    prefetch_tmap(&tm_do);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t xc = 0, uc = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x, ++uc) {
        UnitB w;
        if (!decode_b(p, u, w)) {
          atomicOr(p.err, kErrBadUnit);
          break;
        }
        const SegB& sd = p.seg[w.seg];
        int first, count;
        stream_range<kPassA>(p, sd, w, first, count);
        if (uc > 0 && !(ok = mbar_wait(BAR(B_FEMPTY), (uc - 1) & 1, g))) break;
        mbar_arrive_expect_tx(BAR(B_FFULL), 2 * kTileBytes);
        for (int h = 0; h < 2; ++h) {
          if (kPassA) {   // fixed: K and V rows of the unit
            tma_load_5d(sbase + kOffF0 + h * kHalfBytes, &tm_qkv, BAR(B_FFULL), 64 * h, w.j, w.row0, 1, w.r);
            tma_load_5d(sbase + kOffF1 + h * kHalfBytes, &tm_qkv, BAR(B_FFULL), 64 * h, w.j, w.row0, 2, w.r);
          } else {        // fixed: Q and dO rows of the unit
            tma_load_5d(sbase + kOffF0 + h * kHalfBytes, &tm_qkv, BAR(B_FFULL), 64 * h, w.j, w.row0, 0, w.r);
            tma_load_5d(sbase + kOffF1 + h * kHalfBytes, &tm_do, BAR(B_FFULL), 64 * h, w.j, w.row0, 0, w.r);
          }
        }
        for (int i = 0; i < count; ++i) {
          const int r0 = sd.start + (first + i) * BT;
          const uint32_t s = xc % kStages, ph = (xc / kStages) & 1;
          if (xc >= kStages && !(ok = mbar_wait(BAR(B_XEMPTY0 + s), ph ^ 1, g))) break;
          const uint32_t x0 = sbase + kOffX + s * 2 * kTileBytes, x1 = x0 + kTileBytes;
          if (kPassA) {   // streamed: Q and dO of a query block, its lse and D
            mbar_arrive_expect_tx(BAR(B_XFULL0 + s), 2 * kTileBytes + kRowStageBytes);
            for (int h = 0; h < 2; ++h) {
              tma_load_5d(x0 + h * kHalfBytes, &tm_qkv, BAR(B_XFULL0 + s), 64 * h, w.j, r0, 0, w.r);
              tma_load_5d(x1 + h * kHalfBytes, &tm_do, BAR(B_XFULL0 + s), 64 * h, w.j, r0, 0, w.r);
            }
            const int64_t roff = (static_cast<int64_t>(w.r) * p.Hl + w.j) * p.ls + (r0 & ~3);
            bulk_load(sbase + kOffRow + s * kRowStageBytes, p.lse + roff, kRowFloats * 4, BAR(B_XFULL0 + s));
            bulk_load(sbase + kOffRow + s * kRowStageBytes + kRowFloats * 4, p.delta + roff, kRowFloats * 4,
                      BAR(B_XFULL0 + s));
          } else {        // streamed: K and V of a key block
            mbar_arrive_expect_tx(BAR(B_XFULL0 + s), 2 * kTileBytes);
            for (int h = 0; h < 2; ++h) {
              tma_load_5d(x0 + h * kHalfBytes, &tm_qkv, BAR(B_XFULL0 + s), 64 * h, w.j, r0, 1, w.r);
              tma_load_5d(x1 + h * kHalfBytes, &tm_qkv, BAR(B_XFULL0 + s), 64 * h, w.j, r0, 2, w.r);
            }
          }
          ++xc;
        }
      }
      if (uc > 0) drain_wait_b(BAR(B_FFULL), (uc - 1) & 1);
      for (uint32_t n = (xc > kStages ? xc - kStages : 0); n < xc; ++n)
        drain_wait_b(BAR(B_XFULL0 + n % kStages), (n / kStages) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ tcgen05 issuer
    if (lane == 0) {
      uint32_t xc = 0, uc = 0, pc = 0;
      bool ok = true;
      const uint64_t dF0 = desc_sw128(sbase + kOffF0, 16, 1024), dF1 = desc_sw128(sbase + kOffF1, 16, 1024);
      for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x, ++uc) {
        UnitB w;
        if (!decode_b(p, u, w)) break;
        const SegB& sd = p.seg[w.seg];
        int first, count;
        stream_range<kPassA>(p, sd, w, first, count);
        if (!(ok = mbar_wait(BAR(B_FFULL), uc & 1, g))) break;
        tc_fence_after();
        for (int i = 0; ok && i < count; ++i) {
          const uint32_t s = xc % kStages;
          const uint32_t x0 = sbase + kOffX + s * 2 * kTileBytes, x1 = x0 + kTileBytes;
          if (!(ok = mbar_wait(BAR(B_XFULL0 + s), (xc / kStages) & 1, g))) break;
          tc_fence_after();
          // pass A: S^T = K Q^T, dP^T = V dO^T;  pass B: S = Q K^T, dP = dO V^T
          mma_ss_k128(tmem + kColA0, dF0, desc_sw128(x0, 16, 1024), kIdescSS, 0);
          mma_ss_k128(tmem + kColA1, dF1, desc_sw128(x1, 16, 1024), kIdescSS, 0);
          mma_commit(BAR(B_SFULL));
          if (i == 0 && uc > 0 && !(ok = mbar_wait(BAR(B_OEMPTY), (uc - 1) & 1, g))) break;
          if (!(ok = mbar_wait(BAR(B_PFULL), pc & 1, g))) break;
          ++pc;
          tc_fence_after();
          if (kPassA) {
            // dV += P^T dO, dK += dS^T Q (B operands read MN-major from the stage)
            mma_ts_k128(tmem + kColAcc0, tmem + kColA0, desc_sw128(x1, kHalfBytes, 1024), kIdescTS, i > 0);
            mma_ts_k128(tmem + kColAcc1, tmem + kColA1, desc_sw128(x0, kHalfBytes, 1024), kIdescTS, i > 0);
          } else {
            // dQ += dS K
            mma_ts_k128(tmem + kColAcc0, tmem + kColA0, desc_sw128(x0, kHalfBytes, 1024), kIdescTS, i > 0);
          }
          mma_commit(BAR(B_XEMPTY0 + s));
          ++xc;
        }
        if (!ok) break;
        mma_commit(BAR(B_OFULL));
        mma_commit(BAR(B_FEMPTY));
      }
      mma_commit(BAR(B_DONE));
      drain_wait_b(BAR(B_DONE), 0);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ elementwise + epilogue
    const int row = threadIdx.x;                       // TMEM lane == row of the unit's tile
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tA0 = tmem + lane_base + kColA0, tA1 = tmem + lane_base + kColA1;
    const float sl2 = p.scale_log2;
    const float* srow = reinterpret_cast<const float*>(smem + kOffRow);
    uint32_t sc = 0, uc = 0, xc = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x, ++uc) {
      UnitB w;
      if (!decode_b(p, u, w)) break;
      const SegB& sd = p.seg[w.seg];
      int first, count;
      stream_range<kPassA>(p, sd, w, first, count);
      const int my = w.row0 + row;                     // key (pass A) or query (pass B) index
      float lse_row = 0.f, d_row = 0.f;
      if (!kPassA && my < p.Np) {
        const int64_t off = (static_cast<int64_t>(w.r) * p.Hl + w.j) * p.ls + my;
        lse_row = p.lse[off];
        d_row = p.delta[off];
      }
      for (int i = 0; i < count; ++i) {
        if (!(ok = mbar_wait_warp(BAR(B_SFULL), sc & 1, g))) break;
        ++sc;
        tc_fence_after();
        const int r0 = sd.start + (first + i) * BT;    // first streamed index of this block
        const uint32_t s = xc % kStages;
        ++xc;
        // pass A: lse / D of the 128 streamed queries (the copy starts at r0 rounded down to 4)
        const float* lse_s = srow + s * (kRowStageBytes / 4) + (r0 & 3);
        const float* dlt_s = lse_s + kRowFloats;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t sv[32], dv[32];
          tmem_ld32(tA0 + 32 * c, sv);
          tmem_ld32(tA1 + 32 * c, dv);
          tmem_wait_ld();
          tmem_regs_ready(sv);
          tmem_regs_ready(dv);
          uint32_t pk_p[16], pk_ds[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float pv[2], ds[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int col = 32 * c + e + h;
              const int other = r0 + col;              // query (pass A) or key (pass B) index
              float lse_q, d_q;
              bool valid;
              if (kPassA) {
                lse_q = lse_s[col];
                d_q = dlt_s[col];
                valid = other < sd.end && my < sd.end && (!p.causal || other >= my);
              } else {
                lse_q = lse_row;
                d_q = d_row;
                valid = other < sd.end && my < sd.end && (!p.causal || other <= my);
              }
              const float x = fmaf(__uint_as_float(sv[e + h]), sl2, -lse_q);
              const float pe = ex2_approx(x);
              pv[h] = valid ? pe : 0.f;
              ds[h] = valid ? pe * (__uint_as_float(dv[e + h]) - d_q) : 0.f;
            }
            pk_p[e >> 1] = pack_bf16x2(pv[0], pv[1]);
            pk_ds[e >> 1] = pack_bf16x2(ds[0], ds[1]);
          }
          if (kPassA) {
            tmem_st16(tA0 + 16 * c, pk_p);    // P^T over the first 64 columns of A0
            tmem_st16(tA1 + 16 * c, pk_ds);   // dS^T over the first 64 columns of A1
          } else {
            tmem_st16(tA0 + 16 * c, pk_ds);   // dS over the first 64 columns of A0
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(BAR(B_PFULL));
      }
      if (!ok) break;
      // epilogue: accumulators -> bf16 rows of dQ / dK / dV (pad rows: zeros)
      if (!(ok = mbar_wait_warp(BAR(B_OFULL), uc & 1, g))) break;
      tc_fence_after();
      const bool live = count > 0 && my < sd.end;
      const bool write = my < sd.tile_end && my < p.Np;
      const int nacc = kPassA ? 2 : 1;
      for (int a = 0; a < nacc; ++a) {
        // pass A: acc0 = dV (plane 2), acc1 = dK (plane 1, times scale); pass B: acc0 = dQ (plane 0)
        const int plane = kPassA ? (a == 0 ? 2 : 1) : 0;
        const float f = (kPassA && a == 0) ? 1.0f : p.scale;
        uint32_t ov[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_base + (a == 0 ? kColAcc0 : kColAcc1) + 32 * c, ov[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_regs_ready(ov[c]);
        if (write) {
          uint4* dst = reinterpret_cast<uint4*>(
              p.dqkv + ((((static_cast<int64_t>(w.r) * 3 + plane) * p.Np + my) * p.Hl + w.j) * HD));
          const float* o = reinterpret_cast<const float*>(&ov[0][0]);
#pragma unroll
          for (int v = 0; v < 16; ++v) {
            uint4 q = make_uint4(0u, 0u, 0u, 0u);
            if (live) {
              q.x = pack_bf16x2(o[8 * v + 0] * f, o[8 * v + 1] * f);
              q.y = pack_bf16x2(o[8 * v + 2] * f, o[8 * v + 3] * f);
              q.z = pack_bf16x2(o[8 * v + 4] * f, o[8 * v + 5] * f);
              q.w = pack_bf16x2(o[8 * v + 6] * f, o[8 * v + 7] * f);
            }
            dst[v] = q;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(BAR(B_OEMPTY));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- host side

using EncodeTiledFnB = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                    const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFnB encode_fn() {
  static EncodeTiledFnB fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFnB>(ptr);
  }
  return fn;
}

// 5-D view (d, local head, token, plane, rank) of a head-sharded [P, C, Np, Hl, D] buffer.
bool head_map(CUtensorMap* m, const void* base, int64_t P, int64_t C, int64_t Np, int64_t Hl) {
  EncodeTiledFnB encode = encode_fn();
  if (!encode) return false;
  cuuint64_t dims[5] = {HD, static_cast<cuuint64_t>(Hl), static_cast<cuuint64_t>(Np), static_cast<cuuint64_t>(C),
                        static_cast<cuuint64_t>(P)};
  cuuint64_t strides[4] = {HD * 2, static_cast<cuuint64_t>(Hl) * HD * 2, static_cast<cuuint64_t>(Np * Hl) * HD * 2,
                           static_cast<cuuint64_t>(C * Np * Hl) * HD * 2};
  cuuint32_t box[5] = {64, 1, BT, 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kPassA>
cudaError_t launch_pass(const CUtensorMap& tq, const CUtensorMap& td, const BwdParams& p, int sms,
                        cudaStream_t stream) {
  static bool attr_set[2][64] = {{false}};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[kPassA][dev]) {
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_kernel<kPassA>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[kPassA][dev] = true;
  }
  const int grid = std::min(p.num_units, sms);
  attn_bwd_kernel<kPassA><<<grid, kThreads, kSmemBytes, stream>>>(tq, td, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bwd(const AttnBwdLaunch& a, cudaStream_t stream) {
  const ulysses_plan_t* pl = a.plan;
  const int64_t P = pl->P, Hl = pl->Hl, Np = pl->Np;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t ls = lse_row_stride(Np);

  // D = rowsum(dO o O)
  {
    const int64_t rows = P * Np * Hl;
    const int64_t want = (rows * 16 + 255) / 256;
    const int grid = static_cast<int>(std::min<int64_t>(want, static_cast<int64_t>(sms) * 8));
    if (grid > 0)
      bwd_delta_kernel<<<grid, 256, 0, stream>>>(static_cast<const int4*>(a.out), static_cast<const int4*>(a.dout),
                                                 a.delta, rows, static_cast<int32_t>(Np), static_cast<int32_t>(Hl),
                                                 ls);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }

  CUtensorMap tq, td;
  if (!head_map(&tq, a.qkv, P, pl->C, Np, Hl) || !head_map(&td, a.dout, P, 1, Np, Hl)) return cudaErrorInvalidValue;

  BwdParams p;
  std::memset(&p, 0, sizeof(p));
  p.dqkv = static_cast<__nv_bfloat16*>(a.dqkv);
  p.lse = a.lse;
  p.delta = a.delta;
  p.ls = ls;
  p.err = pl->dev_err;
  p.N = static_cast<int32_t>(pl->N);
  p.Np = static_cast<int32_t>(Np);
  p.Hl = static_cast<int32_t>(Hl);
  p.P = static_cast<int32_t>(P);
  p.causal = pl->causal;
  p.scale = a.scale;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  // segments longest first; the segment ending at N also covers the pad rows
  int order[ULYSSES_MAX_SEQS];
  int nseg = 0;
  for (int s = 0; s < pl->num_seqs; ++s)
    if (pl->segs[s].end > pl->segs[s].start) order[nseg++] = s;
  std::stable_sort(order, order + nseg, [&](int x, int y) {
    return (pl->segs[x].end - pl->segs[x].start) > (pl->segs[y].end - pl->segs[y].start);
  });
  int units = 0;
  for (int k = 0; k < nseg; ++k) {
    const ulysses::Segment& sg = pl->segs[order[k]];
    SegB& d = p.seg[k];
    d.start = sg.start;
    d.end = sg.end;
    d.tile_end = (sg.end == pl->N) ? static_cast<int32_t>(Np) : sg.end;
    d.ntile = (d.tile_end - d.start + BT - 1) / BT;
    d.unit_base = units;
    units += d.ntile * static_cast<int>(P * Hl);
  }
  p.nseg = nseg;
  p.num_units = units;
  if (units == 0) return cudaSuccess;
  cudaError_t e = launch_pass<true>(tq, td, p, sms, stream);    // dK, dV
  if (e != cudaSuccess) return e;
  return launch_pass<false>(tq, td, p, sms, stream);           // dQ
}

}  // namespace ulysses
