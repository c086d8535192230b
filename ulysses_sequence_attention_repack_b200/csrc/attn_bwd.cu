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
// Default, one pass over the keys (kModeAQ): one CTA unit = 128 keys of one
// head and sequence, looping over the query blocks: S^T = K Q^T and
// dP^T = V dO^T into TMEM, then P^T and dS^T (bf16, aliased over them),
// dV += P^T dO and dK += dS^T Q with A read from TMEM, and dQ^T = K^T dS^T
// with dS also stored to shared memory; a fourth warpgroup adds each dQ^T
// block into an fp32 accumulator in global memory (reductions performed in
// L2, so the order of the additions, and the last bits of dQ, vary from run
// to run), which a last kernel scales and rounds to bf16.
//
// Deterministic, two passes, no atomics (plan flag DETERMINISTIC):
//   pass A (kModeA, the loop above without dQ), then
//   pass B (kModeB, unit = 128 queries, loop over key blocks): S = Q K^T and
//           dP = dO V^T, then dS (bf16, over dP), then dQ += dS K.
// All reuse the forward's machinery: TMA-fed 128B-swizzled tiles, grouped
// tcgen05 MMAs issued by one thread, bounded mbarrier waits.  Warps: 0-7
// elementwise and epilogue (two warpgroups, each one thread per TMEM lane and
// 64 of the 128 columns), 8 MMA issuer, 9 TMA producer; kModeAQ adds warps
// 12-15 (dQ reduction; 10 and 11 only complete their warpgroup).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>

#include "bounds.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace ulysses {
namespace {

constexpr int kModeA = 0;    // dK, dV (loop over query blocks)
constexpr int kModeB = 1;    // dQ (loop over key blocks)
constexpr int kModeAQ = 2;   // dK, dV and dQ in one loop over query blocks
constexpr int kEwWarps = 8;                           // two warpgroups, 64 columns each
constexpr int kMmaWarp = kEwWarps;
constexpr int kTmaWarp = kEwWarps + 1;
constexpr int kDqWarp0 = 12;                          // kModeAQ: warps 12-15 reduce dQ
template <int kMode>
constexpr int threads_of() {
  return kMode == kModeAQ ? 512 : 32 * (kEwWarps + 2);
}
// kModeAQ register split (setmaxnreg), against the 128 per thread a 512-thread
// CTA is launched with: 256 x 168 + 128 x 80 + 128 x 96 = 512 x 128.
constexpr uint32_t kEwRegs = 168, kCtlRegs = 80, kDqRegs = 96;
static_assert(256 * kEwRegs + 128 * kCtlRegs + 128 * kDqRegs == 512 * 128, "register split");
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
// pass A: per stage, 132 floats of -lse then 132 of -D, copied from the
// block start rounded down to a multiple of 4 (16-byte aligned bulk copies)
constexpr uint32_t kRowFloats = 132;
constexpr uint32_t kRowStageBytes = 2 * kRowFloats * 4;                // 1056
constexpr uint32_t kOffRow = kOffX + kStages * 2 * kTileBytes;
// kModeAQ only: 64 rows of 512 bytes (fp32 dQ of 64 queries) staged for the
// bulk reduce-adds, after the row stages.
constexpr uint32_t kOffDqStage = (kOffRow + kStages * kRowStageBytes + 127) / 128 * 128;
constexpr uint32_t kDqStageRows = 64;
constexpr uint32_t kDqStageBytes = kDqStageRows * HD * 4;
// Streamed tiles: X0 (pass A: Q, pass B: K) and X1 (dO / V) arrive on their
// own barriers, so the MMA that needs X0 first does not wait for X1.  Pass A
// frees both with one commit after dK; kModeAQ frees Q with that commit and
// dO's slot (which then holds dS, and after dQ^T the first half of the
// block's dQ rows) when the dQ warps' bulk copies have read it; pass B frees
// V as soon as dP is done (an elementwise thread arrives) and K with a commit
// after dQ.
enum {
  B_FFULL = 0, B_FEMPTY, B_X0FULL0, B_X0FULL1, B_X1FULL0, B_X1FULL1, B_X0EMPTY0, B_X0EMPTY1, B_X1EMPTY0,
  B_X1EMPTY1, B_SFULL, B_DPFULL, B_PFULL, B_DSFULL, B_OFULL, B_OEMPTY, B_DONE,
  B_DVDONE, B_DQFULL, B_DQEMPTY,   // kModeAQ: dV has read dO; dQ^T is in TMEM; dQ^T has been read out
  B_DQSTAGED,                      // kModeAQ: every dQ warp has written its channels of the staged rows
  B_DQFREE,                        // kModeAQ: every dQ warp's bulk copies have read the staged rows
  B_COUNT
};
// Barriers, TMEM slot and abort flag after the tiles.  Modes A and B leave
// 1 KB of slack to round the dynamic shared memory base up to 1024 bytes;
// kModeAQ needs that kilobyte for its staging rows, so it runs only on a
// base that is already 1024-byte aligned (checked; error bit kErrSmemAlign).
template <int kMode>
__host__ __device__ constexpr uint32_t off_bar() {
  return kMode == kModeAQ ? kOffDqStage + kDqStageBytes : kOffRow + kStages * kRowStageBytes;
}
template <int kMode>
__host__ __device__ constexpr uint32_t smem_bytes() {
  return off_bar<kMode>() + B_COUNT * 8 + 8 + (kMode == kModeAQ ? 0u : 1024u);
}
static_assert(smem_bytes<kModeAQ>() <= 232448, "kModeAQ shared memory");
static_assert(smem_bytes<kModeA>() <= 232448, "pass shared memory");

// TMEM columns: A0 (S or S^T, then P^T / dS bf16), A1 (dP or dP^T, then dS^T), accumulators
constexpr uint32_t kColA0 = 0, kColA1 = 128, kColAcc0 = 256, kColAcc1 = 384;
constexpr uint32_t kIdescSS = idesc_bf16_f32(BT, BT, 0, 0);
constexpr uint32_t kIdescTS = idesc_bf16_f32(BT, HD, 0, 1);
// dQ^T = K^T dS^T: M = D (A = K^T, MN-major in the K tile), N = 128 queries
// (B = dS^T, MN-major: key rows of 128 query columns)
constexpr uint32_t kIdescDq = idesc_bf16_f32(HD, BT, 1, 1);

struct SegB {
  int32_t start, end;      // the segment's rows [start, end)
  int32_t tile_end;        // rows this segment's units cover (Np for the segment ending at N)
  int32_t ntile;           // 128-row units per (rank, head)
  int32_t unit_base;
  int32_t pair_base;       // causal schedule: first pair of units of this segment
};

struct BwdParams {
  __nv_bfloat16* dqkv;     // [P, 3, Np, Hl, D]
  const float* nlse;       // [P*Hl][ls]: -lse
  const float* nd;         // [P*Hl][ls]: -rowsum(dO o O)
  float* dqacc;            // kModeAQ: [P*Hl][Np][D] fp32 sum of dS K (zeroed by bwd_delta_kernel)
  int64_t dqkv_ext;        // elements of dqkv (range checks of the bounds-checked build)
  int64_t dqacc_ext;       // elements of dqacc
  int64_t ls;              // row stride of both
  unsigned int* err;
  int32_t N, Np, Hl, P, causal;
  int32_t num_units, nseg;
  int32_t num_pairs, paired;   // causal schedule (see unit_of_cta_b)
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

// The k-th work unit of this CTA: 1 (w filled), 0 (no units left), 2 (an
// empty slot: skip), -1 (decodes outside the problem).  With the causal mask
// a unit's cost is linear in its tile index (pass A: the query blocks at or
// after its keys; pass B: the key blocks up to its queries), so the tiles of
// each (segment, rank, head) are paired as (ntile - 1 - i, i), pairs of equal
// cost, and CTA b takes pairs b, b + G, ...; the middle tile of an odd count
// leaves an empty slot.  Otherwise CTA b takes units b, b + G, ... .
__device__ __forceinline__ int unit_of_cta_b(const BwdParams& p, int k, UnitB& w) {
  if (!p.paired) {
    const int u = blockIdx.x + k * gridDim.x;
    if (u >= p.num_units) return 0;
    return decode_b(p, u, w) ? 1 : -1;
  }
  const int pp = blockIdx.x + (k >> 1) * gridDim.x;
  if (pp >= p.num_pairs) return 0;
  int s = 0;
  while (s + 1 < p.nseg && pp >= p.seg[s + 1].pair_base) ++s;
  const int nt = p.seg[s].ntile;
  const int half = (nt + 1) >> 1;
  const int local = pp - p.seg[s].pair_base;
  const int rh = local / half;
  const int i = local - rh * half;
  const int tb = (k & 1) ? i : nt - 1 - i;
  if ((k & 1) && tb >= nt - 1 - i) return 2;   // the unpaired middle tile
  return decode_b(p, p.seg[s].unit_base + rh * nt + tb, w) ? 1 : -1;
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

// kModeAQ starts a unit's loop over query blocks at its own key-tile index
// (mod the block count), so the CTAs working on one head add into different
// dQ tiles at any moment rather than all into the same one.  Block i of the
// loop is query block first + rot_block(i, rot, count).
template <int kMode>
__device__ __forceinline__ int block_rot(const SegB& sd, const UnitB& w, int count) {
  if (kMode != kModeAQ || count <= 0) return 0;
  return ((w.row0 - sd.start) / BT) % count;
}
__device__ __forceinline__ int rot_block(int i, int rot, int count) {
  const int k = i + rot;
  return k >= count ? k - count : k;
}

__device__ __forceinline__ bool drain_wait_b(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

// nd[(r*Hl + j) * ls + n] = -sum_d dO[r, n, j, d] * O[r, n, j, d] and
// nlse[...] = -lse[...] for n < Np: the row terms the elementwise step
// subtracts, stored negated so that it adds them.  With dqacc (one-pass
// backward) it also zeroes the row's fp32 dQ accumulator
// dqacc[((r*Hl + j) * Np + n) * D ..].  One half-warp per row: 16 lanes x 8
// channels.
__global__ void __launch_bounds__(256) bwd_delta_kernel(const int4* __restrict__ out, const int4* __restrict__ dout,
                                                        const float* __restrict__ lse, float* __restrict__ nd,
                                                        float* __restrict__ nlse, float4* __restrict__ dqacc,
                                                        int64_t rows, int32_t Np, int32_t Hl, int64_t ls) {
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
    const int64_t j = row % Hl;
    const int64_t rn = row / Hl;
    const int64_t n = rn % Np, r = rn / Np;
    if (dqacc) {
      float4* z = dqacc + ((r * Hl + j) * Np + n) * (HD / 4) + 2 * ch;
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (ch == 0) {
      const int64_t o = (r * Hl + j) * ls + n;
      nd[o] = -acc;
      nlse[o] = -lse[o];
    }
  }
}

// dQ = scale * dqacc, rounded to bf16, into plane 0 of dqkv [P, 3, Np, Hl, D];
// dqacc is [P*Hl][Np][D] fp32.  One thread per 8 channels.
__global__ void __launch_bounds__(256) dq_convert_kernel(const float4* __restrict__ dqacc, uint4* __restrict__ dqkv,
                                                         int64_t rows, int32_t Np, int32_t Hl, float scale) {
  const int64_t total = rows * 16;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = t >> 4;    // (r*Hl + j)*Np + n
    const int ch = static_cast<int>(t & 15);
    const int64_t n = row % Np, rj = row / Np;
    const int64_t j = rj % Hl, r = rj / Hl;
    const float4 a = dqacc[row * 32 + 2 * ch];
    const float4 b = dqacc[row * 32 + 2 * ch + 1];
    uint4 q;
    q.x = pack_bf16x2(a.x * scale, a.y * scale);
    q.y = pack_bf16x2(a.z * scale, a.w * scale);
    q.z = pack_bf16x2(b.x * scale, b.y * scale);
    q.w = pack_bf16x2(b.z * scale, b.w * scale);
    dqkv[(((r * 3) * Np + n) * Hl + j) * 16 + ch] = q;
  }
}

// Elementwise step of one streamed block for one thread: its TMEM lane (a key
// in pass A, a query in pass B) against the 64 columns of its warpgroup.
//   P  = exp2(s log2e S - lse)             (0 where the pair is masked)
// Pass A takes -lse per column from shared memory (nl_s), pass B one value
// per row (nl_row).  kMask: the block straddles a segment end or the causal
// diagonal, or (pass A) its rows are not 16-byte aligned in shared memory;
// otherwise the columns are read four at a time.
template <bool kPassA, bool kMask>
__device__ __forceinline__ void p_block(const uint32_t (&sv)[2][32], float (&pr)[64], float sl2,
                                        const float* nl_s, uint32_t nl_sa, float nl_row, int col0, int my, int end,
                                        int causal) {
  auto sval = [&](int e) { return __uint_as_float(sv[e >> 5][e & 31]); };
  if (kPassA && !kMask) {
#pragma unroll
    for (int e = 0; e < 64; e += 4) {
      const float4 l = lds128(nl_sa + 4 * e);
      const f2 x0 = ffma2(f2{sval(e), sval(e + 1)}, f2{sl2, sl2}, f2{l.x, l.y});
      const f2 x1 = ffma2(f2{sval(e + 2), sval(e + 3)}, f2{sl2, sl2}, f2{l.z, l.w});
      pr[e] = ex2_approx(x0.x);
      pr[e + 1] = ex2_approx(x0.y);
      pr[e + 2] = ex2_approx(x1.x);
      pr[e + 3] = ex2_approx(x1.y);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 64; e += 2) {
      const f2 nl = kPassA ? f2{nl_s[e], nl_s[e + 1]} : f2{nl_row, nl_row};
      const f2 x = ffma2(f2{sval(e), sval(e + 1)}, f2{sl2, sl2}, nl);
      pr[e] = ex2_approx(x.x);
      pr[e + 1] = ex2_approx(x.y);
    }
  }
  if (kMask) {
    const bool row_ok = my < end;
#pragma unroll
    for (int e = 0; e < 64; ++e) {
      const int other = col0 + e;                      // query (pass A) or key (pass B) index
      const bool valid = row_ok && other < end && (!causal || (kPassA ? other >= my : other <= my));
      pr[e] = valid ? pr[e] : 0.f;
    }
  }
}

//   dS = P o (dP - D) over 32 columns, packed to bf16 pairs (pk[k] holds
// columns 2k, 2k + 1); -D per column (pass A, nd_s) or per row (pass B, nd_row)
template <bool kPassA, bool kMask>
__device__ __forceinline__ void ds_half(const uint32_t (&dv)[32], const float* pr, const float* nd_s, uint32_t nd_sa,
                                        float nd_row, uint32_t (&pk)[16]) {
#pragma unroll
  for (int e = 0; e < 32; e += 4) {
    f2 n0, n1;
    if (kPassA && !kMask) {
      const float4 d = lds128(nd_sa + 4 * e);
      n0 = f2{d.x, d.y};
      n1 = f2{d.z, d.w};
    } else if (kPassA) {
      n0 = f2{nd_s[e], nd_s[e + 1]};
      n1 = f2{nd_s[e + 2], nd_s[e + 3]};
    } else {
      n0 = n1 = f2{nd_row, nd_row};
    }
    f2 d0 = fmul2(f2{pr[e], pr[e + 1]}, fadd2(f2{__uint_as_float(dv[e]), __uint_as_float(dv[e + 1])}, n0));
    f2 d1 = fmul2(f2{pr[e + 2], pr[e + 3]}, fadd2(f2{__uint_as_float(dv[e + 2]), __uint_as_float(dv[e + 3])}, n1));
    if (kMask) {   // D past the segment end may be anything: masked entries stay exactly 0
      d0.x = pr[e] == 0.f ? 0.f : d0.x;
      d0.y = pr[e + 1] == 0.f ? 0.f : d0.y;
      d1.x = pr[e + 2] == 0.f ? 0.f : d1.x;
      d1.y = pr[e + 3] == 0.f ? 0.f : d1.y;
    }
    pk[e >> 1] = pack_bf16x2(d0.x, d0.y);
    pk[(e >> 1) + 1] = pack_bf16x2(d1.x, d1.y);
  }
}

template <int kMode>
__global__ void __launch_bounds__(threads_of<kMode>(), 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ BwdParams p) {
  constexpr bool kPassA = kMode != kModeB;
  constexpr bool kDq = kMode == kModeAQ;
  constexpr uint32_t kOffBar = off_bar<kMode>();
  constexpr uint32_t kOffSlot = kOffBar + B_COUNT * 8;
  constexpr uint32_t kOffAbort = kOffSlot + 4;
  extern __shared__ uint8_t smem_raw[];
  if (kDq && (smem_u32(smem_raw) & 1023u) != 0) {   // the layout has no slack to align it
    if (threadIdx.x == 0 && p.err) atomicOr(p.err, kErrSmemAlign);
    return;
  }
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
      mbar_init(BAR(B_X0FULL0 + s), 1);
      mbar_init(BAR(B_X1FULL0 + s), 1);
      mbar_init(BAR(B_X0EMPTY0 + s), 1);
      mbar_init(BAR(B_X1EMPTY0 + s), kDq ? 4 : 1);   // kModeAQ: the dQ warps release dO's slot
    }
    mbar_init(BAR(B_SFULL), 1);
    mbar_init(BAR(B_DPFULL), 1);
    mbar_init(BAR(B_PFULL), kEwWarps);      // one elected arrival per elementwise warp
    mbar_init(BAR(B_DSFULL), kEwWarps);
    mbar_init(BAR(B_OFULL), 1);
    mbar_init(BAR(B_OEMPTY), kEwWarps);
    mbar_init(BAR(B_DONE), 1);
    mbar_init(BAR(B_DVDONE), 1);
    mbar_init(BAR(B_DQFULL), 1);
    mbar_init(BAR(B_DQEMPTY), 4);           // one elected arrival per dQ warp
    mbar_init(BAR(B_DQSTAGED), 4);
    mbar_init(BAR(B_DQFREE), 4);
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
  if (kDq) {   // whole warpgroups: 0-1 elementwise, 2 MMA / TMA (+ two idle warps), 3 dQ
    if (warp < kEwWarps)
      regs_inc<kEwRegs>();
    else if (warp < kDqWarp0)
      regs_dec<kCtlRegs>();
    else
      regs_dec<kDqRegs>();
  }

  if (kDq && warp >= kDqWarp0) {
    // ------------------------------------------------------------ dQ reduction (kModeAQ)
    // Thread (warp w, lane l) owns TMEM lane d = 32 (w % 4) + l of dQ^T, i.e.
    // channel d of the block's 128 queries.  dQ^T goes out as fp32 rows [q][d]
    // (512 bytes per query) in two rounds of 64 queries: round 0 into the
    // block's dO slot (free once dQ^T is complete: it held dS), round 1 into
    // registers, after which A1 is free for the next dP; then round 1 into a
    // 32 KB staging area once the previous block's round 1 has been read out
    // of it.  Each round is handed to the TMA engine as bulk reduce-adds into
    // dqacc[(r*Hl + j)*Np + q][..] (warp w: 16 of the 64 queries, those inside
    // the segment); dO's slot returns to the producer when round 0 has been
    // read.
    const int dq_w = warp - kDqWarp0;
    const int dl = 32 * (warp & 3) + lane;
    const uint32_t tq = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + kColA1;
    const uint32_t sbuf = sbase + kOffDqStage;
    uint32_t qc = 0, rc = 0, xc = 0;   // blocks, staged rounds, stage slots used
    bool ok = true;
    // Round n of 64 rows staged at `rows` (queries q0 .. q0 + 63): once every
    // warp's channels are in place, warp w reduce-adds its 16 rows (those
    // before `end`) into dqacc.
    auto dq_rows_reduce = [&](uint32_t n, uint32_t rows, int q0, int end, int64_t head_row) -> bool {
      fence_proxy_async_smem();                      // the rows are for the TMA engine to read
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(B_DQSTAGED));
      if (!mbar_wait_warp(BAR(B_DQSTAGED), n & 1, g)) return false;   // every channel is in place
      if (lane == 0) {
        const int qw = q0 + 16 * dq_w;
        const int nq = min(16, end - qw);            // rows of this warp inside the segment
        if (nq > 0) {
          const int64_t off = (head_row + qw) * HD;
          if (in_bounds(off, static_cast<int64_t>(nq) * HD, p.dqacc_ext, p.err))
            bulk_reduce_add_f32(p.dqacc + off, rows + dq_w * 16 * 512, static_cast<uint32_t>(nq) * 512);
        }
        bulk_commit();
      }
      __syncwarp();
      return true;
    };
    for (int k = 0; ok; ++k) {
      UnitB w;
      const int st = unit_of_cta_b(p, k, w);
      if (st == 0 || st < 0) break;
      if (st == 2) continue;
      const SegB& sd = p.seg[w.seg];
      int first, count;
      stream_range<true>(p, sd, w, first, count);
      const int rot = block_rot<kMode>(sd, w, count);
      const int64_t head_row = (static_cast<int64_t>(w.r) * p.Hl + w.j) * p.Np;
      for (int i = 0; ok && i < count; ++i, ++xc) {
        const int r0 = sd.start + (first + rot_block(i, rot, count)) * BT;
        const uint32_t s = xc % kStages;
        const uint32_t dslot = sbase + kOffX + s * 2 * kTileBytes + kTileBytes;
        if (!(ok = mbar_wait_warp(BAR(B_DQFULL), qc & 1, g))) break;
        ++qc;
        tc_fence_after();
        uint32_t v[2][32];
        tmem_ld32(tq, v[0]);
        tmem_ld32(tq + 32, v[1]);
        tmem_wait_ld();
        tmem_regs_ready(v[0]);
        tmem_regs_ready(v[1]);
#pragma unroll
        for (int c = 0; c < 64; ++c) sts32(dslot + c * 512 + 4 * dl, v[c >> 5][c & 31]);
        tmem_ld32(tq + 64, v[0]);
        tmem_ld32(tq + 96, v[1]);
        tmem_wait_ld();
        tmem_regs_ready(v[0]);
        tmem_regs_ready(v[1]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(B_DQEMPTY));   // all of dQ^T is out of TMEM: A1 may take the next dP
        if (!(ok = dq_rows_reduce(rc++, dslot, r0, sd.end, head_row))) break;
        if (qc > 1) {   // the previous block's round 1 must have been read out of the staging area
          if (lane == 0) {
            bulk_wait_read_but_newest();
            mbar_arrive(BAR(B_DQFREE));
          }
          if (!(ok = mbar_wait_warp(BAR(B_DQFREE), (qc - 2) & 1, g))) break;
        }
#pragma unroll
        for (int c = 0; c < 64; ++c) sts32(sbuf + c * 512 + 4 * dl, v[c >> 5][c & 31]);
        if (!(ok = dq_rows_reduce(rc++, sbuf, r0 + 64, sd.end, head_row))) break;
        if (lane == 0) {   // round 0 has been read: dO's slot goes back to the producer
          bulk_wait_read_but_newest();
          mbar_arrive(BAR(B_X1EMPTY0 + s));
        }
        __syncwarp();
      }
    }
    if (lane == 0) bulk_wait_all();
  } else if (warp >= kEwWarps) {
   if (warp == kTmaWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t xc = 0, uc = 0, x0c = 0, x1c = 0;   // blocks, units, copies issued per tile barrier
      bool ok = true;
      for (int k = 0; ok; ++k) {
        UnitB w;
        const int st = unit_of_cta_b(p, k, w);
        if (st == 0) break;
        if (st == 2) continue;
        if (st < 0) {
          atomicOr(p.err, kErrBadUnit);
          break;
        }
        const SegB& sd = p.seg[w.seg];
        int first, count;
        stream_range<kPassA>(p, sd, w, first, count);
        const int rot = block_rot<kMode>(sd, w, count);
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
          const int r0 = sd.start + (first + rot_block(i, rot, count)) * BT;
          const uint32_t s = xc % kStages, ph = (xc / kStages) & 1;
          const uint32_t x0 = sbase + kOffX + s * 2 * kTileBytes, x1 = x0 + kTileBytes;
          if (kPassA) {   // streamed: Q with its -lse / -D rows, then dO, of a query block
            if (xc >= kStages && !(ok = mbar_wait(BAR(B_X0EMPTY0 + s), ph ^ 1, g))) break;
            mbar_arrive_expect_tx(BAR(B_X0FULL0 + s), kTileBytes + kRowStageBytes);
            for (int h = 0; h < 2; ++h)
              tma_load_5d(x0 + h * kHalfBytes, &tm_qkv, BAR(B_X0FULL0 + s), 64 * h, w.j, r0, 0, w.r);
            const int64_t roff = (static_cast<int64_t>(w.r) * p.Hl + w.j) * p.ls + (r0 & ~3);
            bulk_load(sbase + kOffRow + s * kRowStageBytes, p.nlse + roff, kRowFloats * 4, BAR(B_X0FULL0 + s));
            bulk_load(sbase + kOffRow + s * kRowStageBytes + kRowFloats * 4, p.nd + roff, kRowFloats * 4,
                      BAR(B_X0FULL0 + s));
            ++x0c;
            // kModeAQ: dO's slot also stages half of a dQ^T block and comes back later
            if (kDq && xc >= kStages && !(ok = mbar_wait(BAR(B_X1EMPTY0 + s), ph ^ 1, g))) break;
            mbar_arrive_expect_tx(BAR(B_X1FULL0 + s), kTileBytes);
            for (int h = 0; h < 2; ++h)
              tma_load_5d(x1 + h * kHalfBytes, &tm_do, BAR(B_X1FULL0 + s), 64 * h, w.j, r0, 0, w.r);
            ++x1c;
          } else {        // streamed: V as soon as its slot is free (after dP), then K (after dQ)
            if (xc >= kStages && !(ok = mbar_wait(BAR(B_X1EMPTY0 + s), ph ^ 1, g))) break;
            mbar_arrive_expect_tx(BAR(B_X1FULL0 + s), kTileBytes);
            for (int h = 0; h < 2; ++h)
              tma_load_5d(x1 + h * kHalfBytes, &tm_qkv, BAR(B_X1FULL0 + s), 64 * h, w.j, r0, 2, w.r);
            ++x1c;
            if (xc >= kStages && !(ok = mbar_wait(BAR(B_X0EMPTY0 + s), ph ^ 1, g))) break;
            mbar_arrive_expect_tx(BAR(B_X0FULL0 + s), kTileBytes);
            for (int h = 0; h < 2; ++h)
              tma_load_5d(x0 + h * kHalfBytes, &tm_qkv, BAR(B_X0FULL0 + s), 64 * h, w.j, r0, 1, w.r);
            ++x0c;
          }
          ++xc;
        }
        ++uc;
      }
      // no copy may be in flight when the CTA exits
      if (uc > 0) drain_wait_b(BAR(B_FFULL), (uc - 1) & 1);
      for (uint32_t n = (x0c > kStages ? x0c - kStages : 0); n < x0c; ++n)
        drain_wait_b(BAR(B_X0FULL0 + n % kStages), (n / kStages) & 1);
      for (uint32_t n = (x1c > kStages ? x1c - kStages : 0); n < x1c; ++n)
        drain_wait_b(BAR(B_X1FULL0 + n % kStages), (n / kStages) & 1);
    }
   } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ tcgen05 issuer
    // Per block i (pass A):  [P^T(i) ready] dV += P^T dO, S(i+1), [dS^T(i) ready] dK += dS^T Q, dP(i+1)
    //           (pass B):  [S(i) read]      S(i+1),          [dS(i) ready]   dQ += dS K,   dP(i+1)
    //          (kModeAQ):  [P^T(i) ready] dV += P^T dO, S(i+1), [dS(i) ready] dK += dS^T Q,
    //                      dQ^T = K^T dS^T over A1, [dQ^T read out] dP(i+1)
    // so the next block's S is computed while the elementwise warps form dS.
    // The bf16 operands P^T / dS come in two halves of 32 TMEM columns, one per
    // elementwise warpgroup, at column offsets 0 and 64 of their region.
    if (lane == 0) {
      uint32_t xc = 0, uc = 0, pc = 0, qfull = 0, qempty = 0;
      bool ok = true;
      const uint64_t dF0 = desc_sw128(sbase + kOffF0, 16, 1024), dF1 = desc_sw128(sbase + kOffF1, 16, 1024);
      const uint64_t dKT = desc_sw128(sbase + kOffF0, kHalfBytes, 1024);   // K^T as an MN-major A operand
      auto xdesc = [&](uint32_t s, int t, uint32_t lbo) {
        return desc_sw128(sbase + kOffX + s * 2 * kTileBytes + t * kTileBytes, lbo, 1024);
      };
      // kModeAQ: A1 may take the next dP only once the last dQ^T has been read out of it
      auto a1_free = [&]() -> bool {
        if (!kDq || qempty == qfull) return true;
        if (!mbar_wait(BAR(B_DQEMPTY), qempty & 1, g)) return false;
        ++qempty;
        tc_fence_after();
        return true;
      };
      for (int k = 0; ok; ++k) {
        UnitB w;
        const int st = unit_of_cta_b(p, k, w);
        if (st == 0 || st < 0) break;
        if (st == 2) continue;
        const SegB& sd = p.seg[w.seg];
        int first, count;
        stream_range<kPassA>(p, sd, w, first, count);
        if (!(ok = mbar_wait(BAR(B_FFULL), uc & 1, g))) break;
        // the accumulators are free once the previous unit's epilogue has read them
        if (uc > 0 && !(ok = mbar_wait(BAR(B_OEMPTY), (uc - 1) & 1, g))) break;
        tc_fence_after();
        if (count > 0) {
          const uint32_t s = xc % kStages, ph = (xc / kStages) & 1;
          if (!(ok = mbar_wait(BAR(B_X0FULL0 + s), ph, g))) break;
          tc_fence_after();
          // pass A: S^T = K Q^T, dP^T = V dO^T;  pass B: S = Q K^T, dP = dO V^T
          mma_ss_k128(tmem + kColA0, dF0, xdesc(s, 0, 16), kIdescSS, 0);
          mma_commit(BAR(B_SFULL));
          ok = a1_free();
          if (!ok) break;
          if (!(ok = mbar_wait(BAR(B_X1FULL0 + s), ph, g))) break;
          tc_fence_after();
          mma_ss_k128(tmem + kColA1, dF1, xdesc(s, 1, 16), kIdescSS, 0);
          mma_commit(BAR(B_DPFULL));
        }
        for (int i = 0; ok && i < count; ++i) {
          const uint32_t xi = xc + i, s = xi % kStages, sn = (xi + 1) % kStages;
          const bool more = i + 1 < count;
          if (!(ok = mbar_wait(BAR(B_PFULL), pc & 1, g))) break;
          tc_fence_after();
          if (kPassA) {   // dV += P^T dO (B: dO read MN-major from the stage)
            mma_ts_k64(tmem + kColAcc0, tmem + kColA0, xdesc(s, 1, kHalfBytes), kIdescTS, i > 0);
            mma_ts_k64(tmem + kColAcc0, tmem + kColA0 + 64, xdesc(s, 1, kHalfBytes) + 512, kIdescTS, 1);
            if (kDq) mma_commit(BAR(B_DVDONE));   // dO's slot may now take dS
          }
          if (more) {     // S of the next block over A0 (in order after the MMAs that read it)
            if (!(ok = mbar_wait(BAR(B_X0FULL0 + sn), ((xi + 1) / kStages) & 1, g))) break;
            tc_fence_after();
            mma_ss_k128(tmem + kColA0, dF0, xdesc(sn, 0, 16), kIdescSS, 0);
            mma_commit(BAR(B_SFULL));
          }
          if (!(ok = mbar_wait(BAR(B_DSFULL), pc & 1, g))) break;
          tc_fence_after();
          ++pc;
          // pass A: dK += dS^T Q (B: Q MN-major);  pass B: dQ += dS K (B: K MN-major)
          const uint32_t acc = kPassA ? kColAcc1 : kColAcc0;
          mma_ts_k64(tmem + acc, tmem + kColA1, xdesc(s, 0, kHalfBytes), kIdescTS, i > 0);
          mma_ts_k64(tmem + acc, tmem + kColA1 + 64, xdesc(s, 0, kHalfBytes) + 512, kIdescTS, 1);
          if (kDq) {      // dQ^T = K^T dS^T over A1 (after dK has read dS^T), dS from dO's slot
            mma_commit(BAR(B_X0EMPTY0 + s));       // dK was the last reader of the Q slot
            mma_ss_k128_mn(tmem + kColA1, dKT, xdesc(s, 1, kHalfBytes), kIdescDq, 0);
            mma_commit(BAR(B_DQFULL));
            ++qfull;
          } else {
            mma_commit(BAR(B_X0EMPTY0 + s));
          }
          if (more) {     // dP of the next block over A1
            ok = a1_free();
            if (!ok) break;
            if (!(ok = mbar_wait(BAR(B_X1FULL0 + sn), ((xi + 1) / kStages) & 1, g))) break;
            tc_fence_after();
            mma_ss_k128(tmem + kColA1, dF1, xdesc(sn, 1, 16), kIdescSS, 0);
            mma_commit(BAR(B_DPFULL));
          }
        }
        if (!ok) break;
        xc += count;
        mma_commit(BAR(B_OFULL));
        mma_commit(BAR(B_FEMPTY));
        ++uc;
      }
      mma_commit(BAR(B_DONE));
      drain_wait_b(BAR(B_DONE), 0);
    }
   }
  } else {
    // ------------------------------------------------------------ elementwise + epilogue
    // Warp w owns TMEM lanes 32 (w % 4) .. +31 (one row of the unit's tile per
    // thread) and, with its warpgroup w / 4, 64 of the 128 columns.
    const int wg = warp >> 2;
    const int row = 32 * (warp & 3) + lane;
    const int c0 = 64 * wg;
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const uint32_t tA0 = tmem + lane_base + kColA0 + c0, tA1 = tmem + lane_base + kColA1 + c0;
    const float sl2 = p.scale_log2;
    const float* srow = reinterpret_cast<const float*>(smem + kOffRow);
    uint32_t sc = 0, uc = 0, xc = 0, dvc = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      UnitB w;
      const int st = unit_of_cta_b(p, k, w);
      if (st == 0 || st < 0) break;
      if (st == 2) continue;
      const SegB& sd = p.seg[w.seg];
      const int end = sd.end;
      int first, count;
      stream_range<kPassA>(p, sd, w, first, count);
      const int rot = block_rot<kMode>(sd, w, count);
      const int my = w.row0 + row;                     // key (pass A) or query (pass B) index
      float nl_row = 0.f, nd_row = 0.f;               // pass B: -lse and -D of this thread's query
      if (!kPassA && my < p.Np) {
        const int64_t off = (static_cast<int64_t>(w.r) * p.Hl + w.j) * p.ls + my;
        nl_row = p.nlse[off];
        nd_row = p.nd[off];
      }
      for (int i = 0; i < count; ++i) {
        if (!(ok = mbar_wait_warp(BAR(B_SFULL), sc & 1, g))) break;
        ++sc;
        tc_fence_after();
        const int r0 = sd.start + (first + rot_block(i, rot, count)) * BT;    // first streamed index of this block
        const uint32_t s = xc % kStages;
        // pass A reads the block's lse / D rows, which arrive with the stage
        const uint32_t ph = (xc / kStages) & 1;
        if (kPassA && !(ok = mbar_wait_warp(BAR(B_X0FULL0 + s), ph, g))) break;
        ++xc;
        // lse / D of the warpgroup's 64 streamed queries (the copy starts at r0 rounded down to 4)
        const float* nl_s = srow + s * (kRowStageBytes / 4) + (r0 & 3) + c0;
        const float* nd_s = nl_s + kRowFloats;
        const uint32_t nl_sa = sbase + kOffRow + s * kRowStageBytes + 4 * ((r0 & 3) + c0);   // same, shared window
        const uint32_t nd_sa = nl_sa + 4 * kRowFloats;
        // the whole 128 x 128 block is inside the segment and off the causal diagonal
        // (pass A also needs its shared-memory rows 16-byte aligned: blocks start at
        // the segment start plus multiples of 128)
        const bool full = w.row0 + BT <= end && r0 + BT <= end &&
                          (!p.causal || (kPassA ? r0 > w.row0 : r0 < w.row0)) && (!kPassA || (r0 & 3) == 0);
        // phase 1 (S ready): P in fp32, kept for phase 2; pass A stores P^T (bf16) for dV += P^T dO
        float pr[64];
        {
          uint32_t sv[2][32];
          tmem_ld32(tA0, sv[0]);
          tmem_ld32(tA0 + 32, sv[1]);
          tmem_wait_ld();
          tmem_regs_ready(sv[0]);
          tmem_regs_ready(sv[1]);
          if (full)
            p_block<kPassA, false>(sv, pr, sl2, nl_s, nl_sa, nl_row, r0 + c0, my, end, p.causal);
          else
            p_block<kPassA, true>(sv, pr, sl2, nl_s, nl_sa, nl_row, r0 + c0, my, end, p.causal);
        }
        if (kPassA) {
          uint32_t pk[2][16];
#pragma unroll
          for (int e = 0; e < 32; ++e) pk[e >> 4][e & 15] = pack_bf16x2(pr[2 * e], pr[2 * e + 1]);
          tmem_st16(tA0, pk[0]);                       // P^T over columns c0 .. c0 + 31 of A0
          tmem_st16(tA0 + 16, pk[1]);
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(B_PFULL));     // pass B: S has been read
        // phase 2 (dP ready): dS = P o (dP - D) over columns c0 .. c0 + 31 of A1
        if (!(ok = mbar_wait_warp(BAR(B_DPFULL), (sc - 1) & 1, g))) break;
        tc_fence_after();
        if (!kPassA && threadIdx.x == 0) mbar_arrive(BAR(B_X1EMPTY0 + s));   // dP done: V's slot is free
        uint32_t dsk[2][16];
#pragma unroll
        for (int h = 0; h < 2; ++h) {    // two halves of 32 columns: dS of half 0 lands before half 1 is read
          uint32_t dv[32];
          tmem_ld32(tA1 + 32 * h, dv);
          tmem_wait_ld();
          tmem_regs_ready(dv);
          if (full)
            ds_half<kPassA, false>(dv, pr + 32 * h, nd_s + 32 * h, nd_sa + 128 * h, nd_row, dsk[h]);
          else
            ds_half<kPassA, true>(dv, pr + 32 * h, nd_s + 32 * h, nd_sa + 128 * h, nd_row, dsk[h]);
          tmem_st16(tA1 + 16 * h, dsk[h]);
        }
        if (kDq) {
          // dS (bf16) also into shared memory for dQ^T = K^T dS^T, over the block's
          // dO tile once dV has read it: key row `row` of the warpgroup's 64-query
          // half, 128 bytes in 16-byte chunks at the 128B-swizzled positions
          if (!(ok = mbar_wait_warp(BAR(B_DVDONE), dvc & 1, g))) break;
          ++dvc;
          const uint32_t drow = sbase + kOffX + s * 2 * kTileBytes + kTileBytes + wg * kHalfBytes + row * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            sts128(drow + ((c ^ (row & 7)) << 4), dsk[c >> 2][4 * (c & 3)], dsk[c >> 2][4 * (c & 3) + 1],
                   dsk[c >> 2][4 * (c & 3) + 2], dsk[c >> 2][4 * (c & 3) + 3]);
          fence_proxy_async_smem();
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(B_DSFULL));
      }
      if (!ok) break;
      // epilogue: this warpgroup's 64 accumulator columns -> bf16 rows of dQ / dK / dV (pad rows: zeros)
      if (!(ok = mbar_wait_warp(BAR(B_OFULL), uc & 1, g))) break;
      tc_fence_after();
      const bool live = count > 0 && my < end;
      const bool write = my < sd.tile_end && my < p.Np;
      const int nacc = kPassA ? 2 : 1;
      for (int a = 0; a < nacc; ++a) {
        // pass A: acc0 = dV (plane 2), acc1 = dK (plane 1, times scale); pass B: acc0 = dQ (plane 0)
        const int plane = kPassA ? (a == 0 ? 2 : 1) : 0;
        const float f = (kPassA && a == 0) ? 1.0f : p.scale;
        uint32_t ov[2][32];
        const uint32_t tacc = tmem + lane_base + (a == 0 ? kColAcc0 : kColAcc1) + c0;
        tmem_ld32(tacc, ov[0]);
        tmem_ld32(tacc + 32, ov[1]);
        tmem_wait_ld();
        tmem_regs_ready(ov[0]);
        tmem_regs_ready(ov[1]);
        const int64_t doff = (((static_cast<int64_t>(w.r) * 3 + plane) * p.Np + my) * p.Hl + w.j) * HD + c0;
        if (write && in_bounds(doff, 64, p.dqkv_ext, p.err)) {
          uint4* dst = reinterpret_cast<uint4*>(p.dqkv + doff);
          const float* o = reinterpret_cast<const float*>(&ov[0][0]);
#pragma unroll
          for (int v = 0; v < 8; ++v) {
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
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(B_OEMPTY));
      ++uc;
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
  static const EncodeTiledFnB fn = [] {   // initialised once, thread-safe
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFnB>(ptr);
    cudaGetLastError();
    return static_cast<EncodeTiledFnB>(nullptr);
  }();
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

template <int kMode>
cudaError_t launch_pass(const CUtensorMap& tq, const CUtensorMap& td, const BwdParams& p, int sms,
                        cudaStream_t stream) {
  static PerDeviceOnce setup;
  int dev = 0;
  cudaGetDevice(&dev);
  cudaError_t e = setup.run(dev, [] {
    return cudaFuncSetAttribute(attn_bwd_kernel<kMode>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                smem_bytes<kMode>());
  });
  if (e != cudaSuccess) return e;
  const int grid = std::min(p.num_units, sms);
  attn_bwd_kernel<kMode><<<grid, threads_of<kMode>(), smem_bytes<kMode>(), stream>>>(tq, td, p);
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
                                                 a.lse, a.delta, a.delta + P * Hl * ls,
                                                 reinterpret_cast<float4*>(a.dq_acc), rows,
                                                 static_cast<int32_t>(Np), static_cast<int32_t>(Hl), ls);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }

  CUtensorMap tq, td;
  if (!head_map(&tq, a.qkv, P, pl->C, Np, Hl) || !head_map(&td, a.dout, P, 1, Np, Hl)) return cudaErrorInvalidValue;

  BwdParams p;
  std::memset(&p, 0, sizeof(p));
  p.dqkv = static_cast<__nv_bfloat16*>(a.dqkv);
  p.nd = a.delta;
  p.nlse = a.delta + P * Hl * ls;
  p.dqacc = a.dq_acc;
  p.dqkv_ext = P * 3 * Np * Hl * HD;
  p.dqacc_ext = a.dq_acc ? P * Hl * Np * HD : 0;
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
  int units = 0, pairs = 0;
  for (int k = 0; k < nseg; ++k) {
    const ulysses::Segment& sg = pl->segs[order[k]];
    SegB& d = p.seg[k];
    d.start = sg.start;
    d.end = sg.end;
    d.tile_end = (sg.end == pl->N) ? static_cast<int32_t>(Np) : sg.end;
    d.ntile = (d.tile_end - d.start + BT - 1) / BT;
    d.unit_base = units;
    d.pair_base = pairs;
    units += d.ntile * static_cast<int>(P * Hl);
    pairs += (d.ntile + 1) / 2 * static_cast<int>(P * Hl);
  }
  p.nseg = nseg;
  p.num_units = units;
  p.num_pairs = pairs;
  p.paired = (p.causal && units >= 2 * sms) ? 1 : 0;   // two units per SM at least, or the pairs idle SMs
  if (units == 0) return cudaSuccess;
  if (!a.dq_acc) {   // deterministic: two passes
    cudaError_t e = launch_pass<kModeA>(tq, td, p, sms, stream);    // dK, dV
    if (e != cudaSuccess) return e;
    return launch_pass<kModeB>(tq, td, p, sms, stream);            // dQ
  }
  cudaError_t e = launch_pass<kModeAQ>(tq, td, p, sms, stream);     // dK, dV, and dQ into dq_acc
  if (e != cudaSuccess) return e;
  const int64_t rows = P * Hl * Np;
  const int grid = static_cast<int>(std::min<int64_t>((rows * 16 + 255) / 256, static_cast<int64_t>(sms) * 8));
  dq_convert_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const float4*>(a.dq_acc),
                                              static_cast<uint4*>(a.dqkv), rows, static_cast<int32_t>(Np),
                                              static_cast<int32_t>(Hl), a.scale);
  return cudaGetLastError();
}

}  // namespace ulysses
