// Softmax attention for the Ulysses layer on sm_100a.
//
//   O[n, :] = sum_{m in K(n)} softmax_m(scale * <Q_n, K_m>) V_m
//
// (the FA4 backend call of flash_attn_cute.py in "hao-ai-lab FastVideo,
// compare aryan/h3-nvfp4-stack-speedups...main": softmax_scale, non-causal,
// varlen through cu_seqlens).  K(n) is the key range of the packed sequence
// holding row n; with the causal option (the trainer's causal Ulysses flash
// wrapper in the prime-rl Ulysses context-parallelism pull request) only the
// keys m <= n of that range.  Computed flash-style: keys are visited in tiles of 128 and
// the softmax is kept online (running max and sum), so the N x N score matrix
// never leaves the SM.
//
// Design (one persistent CTA per SM, 12 warps):
//   warp 9      TMA producer: Q tiles (2 x 128 rows) and a 2-stage K ring and
//               V ring, 128-byte swizzled, completion counted on mbarriers.
//   warp 8      tcgen05 issuer (one lane): S_i = Q_i K^T into TMEM (fp32),
//               then O_i += P_i V with P_i read from TMEM (bf16, aliased over
//               S_i) and V from shared memory, each group of MMAs one asm
//               block with precomputed descriptors.  Two Q tiles ping-pong so
//               the tensor core works on one tile while the other is in
//               softmax (one issuer per tile was measured slower: the
//               interleaving delays each tile's S).
//   warps 0-7   two softmax warpgroups, one per Q tile; thread t of a group
//               owns query row t, so row max and row sum need no shuffles.
//               P is handed over in two halves (keys 0-63, then 64-127).
//               The running max is only moved (and O rescaled in TMEM) when
//               it grows by more than 8 in log2 units; the final 1/l uses the
//               same stale max, so the result is unchanged.  The first thread
//               of group 1 releases the K/V ring slots.
// TMEM: S0 | S1 | O0 | O1, 128 fp32 columns each (all 512 columns).
//
// FP8 variant (template flag kFp8): Q, K, V arrive as E4M3 codes (cast in the
// repack), the two products are tcgen05 kind::f8f6f4 MMAs, and P is stored as
// E4M3 (four codes per TMEM column).  Everything else is shared.
//
// Every wait is bounded: on timeout the kernel sets an error bit, skips the
// remaining work, waits (bounded) for its own in-flight copies and MMAs,
// frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>

#include "bounds.cuh"
#include "exp2_poly.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

// With ULY_EMU_EVERY = k > 0, one pair in k of each row's exponentials is
// computed on the FMA pipe (exp2_poly2) instead of the MUFU unit.  Off by
// default: on B200 the MUFU unit is not what limits this loop, and the extra
// FMA-pipe instructions made it slower (k = 8, 4, 2 all measured slower).
#ifndef ULY_EMU_EVERY
#define ULY_EMU_EVERY 0
#endif

namespace ulysses {
namespace {

constexpr int kThreads = 384;      // 3 warpgroups
constexpr int kMmaWarp = 8;
constexpr int kTmaWarp = 9;
constexpr int kFwdWarp = 10;        // CTA pairs: forwards the odd CTA's completed fills
constexpr int kHandWarp = 11;       // CTA pairs: forwards the odd CTA's P and O hand-offs
// Register split: the kernel is launched with kLaunchRegs per thread
// (384 x 168 = 64512); warpgroup 2 (TMA, MMA, two spare warps) drops to
// kProducerRegs and the two softmax warpgroups rise to kSoftmaxRegs:
// 128 x 72 + 256 x 216 = 64512.  The host refuses to launch if the compiled
// register count differs, so the increase can never wait for registers that
// were not released.
constexpr uint32_t kLaunchRegs = 168;
constexpr uint32_t kProducerRegs = 72;
constexpr uint32_t kSoftmaxRegs = 216;
static_assert(128 * kProducerRegs + 256 * kSoftmaxRegs <= kThreads * kLaunchRegs, "register split");
constexpr int BM = 128;            // query rows per tile
constexpr int BN = 128;            // keys per tile
constexpr int HD = 128;            // head dim
constexpr int kUnitRows = 2 * BM;  // query rows per work unit (two tiles)
constexpr int kPairUnitRows = 4 * BM;   // CTA pairs: two tiles of 256 rows (128 in each CTA)
constexpr uint32_t kBoxBytes = BM * 128;  // one TMA box: 128 rows x 128 bytes, 128B-swizzled (16 KB)
constexpr int kStages = 2;
constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;   // 1 s per wait

// Tile geometry per element type.  A 128 x 128 tile is two boxes of 64 bf16
// columns (32 KB) or one box of 128 E4M3 columns (16 KB).  In a CTA pair each
// CTA holds half of every K tile (64 keys, two boxes of 64 rows) and half of
// every V tile (64 head-dim columns, one box of 128 rows): 16 KB each.
template <bool kFp8, bool kPair = false>
struct Geo {
  static constexpr int kBoxes = kFp8 ? 1 : 2;
  static constexpr uint32_t kTileBytes = kBoxes * kBoxBytes;              // one CTA's Q tile
  static constexpr uint32_t kKBytes = kPair ? kTileBytes / 2 : kTileBytes;   // one K stage
  static constexpr uint32_t kVBytes = kPair ? kTileBytes / 2 : kTileBytes;   // one V stage
  // shared memory map (offsets from a 1024-aligned base)
  static constexpr uint32_t kOffQ = 0;                                  // [2 tiles]
  static constexpr uint32_t kOffK = kOffQ + 2 * kTileBytes;             // [stages]
  static constexpr uint32_t kOffV = kOffK + kStages * kKBytes;          // [stages]
  static constexpr uint32_t kOffBar = kOffV + kStages * kVBytes;
};
// barrier indices
enum {
  B_QFULL0 = 0, B_QFULL1, B_QEMPTY,
  B_KFULL0, B_KFULL1, B_KEMPTY0, B_KEMPTY1,
  B_VFULL0, B_VFULL1, B_VEMPTY0, B_VEMPTY1,
  B_SFULL0, B_SFULL1, B_PFULL0, B_PFULL1,
  B_OFULL0, B_OFULL1, B_OEMPTY0, B_OEMPTY1,
  B_PHALF0, B_PHALF1,
  B_DONE, B_COUNT
};
template <bool kFp8, bool kPair = false>
struct Smem {
  static constexpr uint32_t kOffBar = Geo<kFp8, kPair>::kOffBar;
  static constexpr uint32_t kOffSlot = kOffBar + B_COUNT * 8;     // TMEM base address
  static constexpr uint32_t kOffAbort = kOffSlot + 4;
  static constexpr uint32_t kBytes = kOffAbort + 4 + 1024;        // + alignment slack
};

// TMEM columns
constexpr uint32_t kColS0 = 0, kColO0 = 256;

constexpr uint32_t kIdescS = idesc_bf16_f32(BM, BN, 0, 0);    // Q, K both K-major (head dim contiguous)
constexpr uint32_t kIdescPV = idesc_bf16_f32(BM, HD, 0, 1);   // P from TMEM, V MN-major (head dim contiguous)
constexpr uint32_t kIdescS8 = idesc_e4m3_f32(BM, BN, 0, 0);   // the same for E4M3 operands
constexpr uint32_t kIdescPV8 = idesc_e4m3_f32(BM, HD, 0, 1);
constexpr uint32_t kIdescS2 = idesc_bf16_f32(2 * BM, BN, 0, 0);   // CTA pairs: M = 256
constexpr uint32_t kIdescPV2 = idesc_bf16_f32(2 * BM, HD, 0, 1);

struct SegDesc {
  int32_t start;       // first query row and first key
  int32_t kv_end;      // one past the last key
  int32_t q_end;       // one past the last query row this segment writes (Np for the last segment)
  int32_t nqb;         // query blocks of one work unit's rows (256, or 512 for CTA pairs)
  int32_t unit_base;   // first work unit of this segment
  int32_t pair_base;   // causal schedule: first pair of query blocks of this segment
};

struct AttnParams {
  __nv_bfloat16* out;
  float* lse;                      // optional: log2-domain log-sum-exp per row (m + log2 l)
  int64_t lse_stride;              // floats between (rank, head) rows of lse
  unsigned int* err;
  int64_t o_stride_r, o_stride_n, o_stride_j;
  int32_t N, Np;
  int32_t Hl, P, fused;
  int32_t causal;                  // query n sees keys m <= n only
  int32_t num_units, nseg;
  int32_t num_pairs;               // causal schedule: pairs of query blocks over all segments and heads
  int32_t paired;                  // 1: the causal pair schedule (enough units for two per CTA)
  float scale_log2;
  int64_t push_rows;               // > 0: row n is stored to push.p[n / push_rows] (multi-GPU push)
  int32_t push_ranks;              // table entries in use
  int64_t out_ext, lse_ext;        // elements, for the bounds-checked build only (bounds.cuh)
  SegDesc seg[ULYSSES_MAX_SEQS];   // longest first
  PushTable push;
};

struct Unit {
  int seg, r, j, q0;
};

template <int kRows>
__device__ __forceinline__ bool decode_unit(const AttnParams& p, int u, Unit& w) {
  int s = 0;
  while (s + 1 < p.nseg && u >= p.seg[s + 1].unit_base) ++s;
  const int local = u - p.seg[s].unit_base;
  const int nqb = p.seg[s].nqb;
  const int rh = local / nqb;         // (rank, head) major, query block minor: CTAs running
  const int qb = local - rh * nqb;    // side by side share one head's K/V in L2
  w.seg = s;
  w.r = rh / p.Hl;
  w.j = rh - w.r * p.Hl;
  w.q0 = p.seg[s].start + qb * kRows;
  return local >= 0 && w.r < p.P;
}

// The k-th work unit of this CTA.  Returns 1 with w filled, 0 when the CTA
// has no units left, 2 for an empty slot of the schedule (skip it), -1 if a
// unit decodes outside the problem.
//   Non-causal: every unit of a segment visits the same key tiles, and CTA b
//   takes units b, b + G, b + 2G, ... (G = gridDim.x).
//   Causal: a unit visits the key tiles up to its last query row, so its cost
//   grows with its query block qb.  The blocks of each (segment, rank, head)
//   are paired as (nqb - 1 - i, i), pairs of equal total cost, and CTA b takes
//   pairs b, b + G, ... (both units of a pair, the costlier first); the middle
//   block of an odd count has no partner, which leaves an empty slot.  Plain
//   round robin would leave the busiest CTA with ~1.2x the average work at
//   the Video-DiT size.  With fewer than two units per SM the pairs would
//   idle half the SMs, so small causal problems keep the plain schedule.
//   cta / ncta: this CTA's index and the grid size, or the pair's index and
//   the number of pairs.
template <int kRows>
__device__ __forceinline__ int unit_of_cta(const AttnParams& p, int k, Unit& w, int cta, int ncta) {
  if (!p.paired) {
    const int u = cta + k * ncta;
    if (u >= p.num_units) return 0;
    return decode_unit<kRows>(p, u, w) ? 1 : -1;
  }
  const int pp = cta + (k >> 1) * ncta;
  if (pp >= p.num_pairs) return 0;
  int s = 0;
  while (s + 1 < p.nseg && pp >= p.seg[s + 1].pair_base) ++s;
  const int nqb = p.seg[s].nqb;
  const int half = (nqb + 1) >> 1;
  const int local = pp - p.seg[s].pair_base;
  const int rh = local / half;
  const int i = local - rh * half;
  const int qb = (k & 1) ? i : nqb - 1 - i;
  if ((k & 1) && qb >= nqb - 1 - i) return 2;   // the unpaired middle block
  return decode_unit<kRows>(p, p.seg[s].unit_base + rh * nqb + qb, w) ? 1 : -1;
}

// P = exp2(s * scale_log2 - m) for columns [64 half, 64 half + 64) of one row,
// stored to TMEM as 32 bf16 pairs at P columns [32 half, 32 half + 32); the
// row sum accumulates in acc.
template <bool kEmu>
__device__ __forceinline__ void exp_store_half(const float* s, int half, f2 scale2, f2 negm2, f2 (&acc)[4],
                                               uint32_t tS) {
  uint32_t pk[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    const f2 x = ffma2(f2{s[64 * half + 2 * c], s[64 * half + 2 * c + 1]}, scale2, negm2);
    f2 e;
    if (kEmu && ULY_EMU_EVERY > 0 && (c % (ULY_EMU_EVERY > 0 ? ULY_EMU_EVERY : 1)) == ULY_EMU_EVERY - 1) {
      e = exp2_poly2(x);
    } else {
      e.x = ex2_approx(x.x);
      e.y = ex2_approx(x.y);
    }
    acc[c & 3] = fadd2(acc[c & 3], e);
    pk[c] = pack_bf16x2(e.x, e.y);
  }
  tmem_st32(tS + 32 * half, pk);
}

// The E4M3 variant of exp_store_half: the same 64 probabilities, stored as
// 16 columns of four E4M3 codes at P columns [16 half, 16 half + 16).  The
// row sum uses the fp32 values.  P stays below 2^8 (the running max moves
// when it grows by more than 8), inside E4M3's range of 448.  With E4M3
// operands the tensor core needs half the cycles of bf16 and the MUFU unit
// limits the loop, so with kEmu one group of four keys in kFp8EmuEvery is
// exponentiated on the FMA pipe (exp2_poly2, relative error 7.5e-5, far below
// E4M3's 2^-4).  Measured against no emulation at the Video-DiT size
// (19,394 tokens) and the 104k-token size: 1 in 8 is 7.3% and 3.6% faster,
// 1 in 4 4.3% and 0%, 1 in 16 1.4% and 0%, 1 in 3 or 2 slower than 1 in 4.
constexpr int kFp8EmuEvery = 8;
template <bool kEmu>
__device__ __forceinline__ void exp_store_half_fp8(const float* s, int half, f2 scale2, f2 negm2, f2 (&acc)[4],
                                                   uint32_t tS) {
  uint32_t pk[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const float* sc = s + 64 * half + 4 * c;
    const f2 x0 = ffma2(f2{sc[0], sc[1]}, scale2, negm2);
    const f2 x1 = ffma2(f2{sc[2], sc[3]}, scale2, negm2);
    f2 e0, e1;
    if (kEmu && c % kFp8EmuEvery == kFp8EmuEvery - 1) {
      e0 = exp2_poly2(x0);
      e1 = exp2_poly2(x1);
    } else {
      e0.x = ex2_approx(x0.x);
      e0.y = ex2_approx(x0.y);
      e1.x = ex2_approx(x1.x);
      e1.y = ex2_approx(x1.y);
    }
    acc[(2 * c) & 3] = fadd2(acc[(2 * c) & 3], e0);
    acc[(2 * c + 1) & 3] = fadd2(acc[(2 * c + 1) & 3], e1);
    pk[c] = pack_e4m3x4(e0.x, e0.y, e1.x, e1.y);
  }
  tmem_st16(tS + 16 * half, pk);
}

// Number of 128-key tiles a unit visits: the whole segment, or (causal) the
// keys up to the unit's last query row.
template <int kRows>
__device__ __forceinline__ int unit_kv_tiles(const AttnParams& p, const SegDesc& sd, const Unit& w) {
  const int hi = p.causal ? min(sd.kv_end, w.q0 + kRows) : sd.kv_end;
  return (hi - sd.start + BN - 1) / BN;
}

// waits that ignore the abort flag (used for draining in-flight work)
__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

// kFp8: Q, K, V are E4M3 codes (one byte per element) and P is stored as
// E4M3 for the P V product; otherwise everything is bf16.
//
// kPair: the kernel runs as clusters of two CTAs on neighbouring SMs.  A work
// unit is 512 query rows of one (rank, head, sequence); tile i (i = 0, 1) of
// the pair is rows q0 + 256 i .. q0 + 256 i + 255, the even CTA holding the
// first 128 of them in its shared memory and TMEM and the odd CTA the other
// 128.  One thread of the even CTA issues every MMA as a cta_group::2
// operation of M = 256: S_i = Q_i K^T reads each CTA's 64 keys of the K tile
// (B split by N) and O_i += P_i V each CTA's 64 head-dim columns of V.  So
// each SM copies into shared memory half of every K and V tile, and the
// B-operand reads of both products are split between the two SMs.  Each
// CTA's softmax warps work on their own TMEM rows exactly as in the
// single-CTA kernel; their P and O hand-offs arrive (one arrival per warp)
// on the even CTA's barriers, and the MMA thread's commits arrive on the
// barriers of both CTAs.  Every CTA's copies complete on its own barriers,
// and warp 10 of the odd CTA forwards each completed fill to the even CTA's
// barrier, so each producer can wait for its own copies before its CTA exits.
template <bool kFp8, bool kPair>
__device__ __forceinline__ void attn_body(const CUtensorMap* tmap, const CUtensorMap* tmapK, const AttnParams& p) {
  using G = Geo<kFp8, kPair>;
  constexpr int kRows = kPair ? kPairUnitRows : kUnitRows;
  constexpr uint32_t kTileBytes = G::kTileBytes;
  constexpr uint32_t kOffQ = G::kOffQ, kOffK = G::kOffK, kOffV = G::kOffV, kOffBar = G::kOffBar;
  constexpr uint32_t kOffSlot = Smem<kFp8, kPair>::kOffSlot, kOffAbort = Smem<kFp8, kPair>::kOffAbort;
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
  // the CTA (or pair) index and count the work units are dealt over
  const uint32_t cr = kPair ? cluster_ctarank() : 0u;   // 0: the CTA whose thread issues the MMAs
  const bool leader = cr == 0;
  const int cta = kPair ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int ncta = kPair ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  // shared::cluster addresses of barrier 0 in the even (L) and the odd (O) CTA of a pair
  const uint32_t lbar0 = kPair ? mapa_shared(bar0, 0) : bar0;
  const uint32_t obar0 = kPair ? mapa_shared(bar0, 1) : bar0;
  auto LBAR = [&](int i) { return lbar0 + 8u * static_cast<uint32_t>(i); };
  auto OBAR = [&](int i) { return obar0 + 8u * static_cast<uint32_t>(i); };
  // tcgen05 completion of everything this thread issued, on barrier i of both CTAs
  auto commit = [&](int i) {
    if constexpr (kPair) {
      mma_commit_pair(LBAR(i));
      mma_commit_pair(OBAR(i));
    } else {
      mma_commit(BAR(i));
    }
  };
  // a P or O hand-off of this softmax thread: a CTA-scope arrival on its own
  // CTA's barrier (in a pair, the odd CTA's completed phases are forwarded to
  // the even CTA by warp kHandWarp, so no softmax thread pays a cluster-scope
  // release)
  auto hand_off = [&](int i) { mbar_arrive(BAR(i)); };

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    // the even CTA's fill and hand-off barriers also take the odd CTA's
    // forwarded arrival
    const uint32_t fills = (kPair && leader) ? 2 : 1;
    const uint32_t hands = (kPair && leader) ? BM + 1 : BM;
    mbar_init(BAR(B_QFULL0), fills);
    mbar_init(BAR(B_QFULL1), fills);
    mbar_init(BAR(B_QEMPTY), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(BAR(B_KFULL0 + s), fills);
      mbar_init(BAR(B_KEMPTY0 + s), 1);
      mbar_init(BAR(B_VFULL0 + s), fills);
      mbar_init(BAR(B_VEMPTY0 + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(B_SFULL0 + i), 1);
      mbar_init(BAR(B_PFULL0 + i), hands);
      mbar_init(BAR(B_OFULL0 + i), 1);
      mbar_init(BAR(B_OEMPTY0 + i), hands);
      mbar_init(BAR(B_PHALF0 + i), hands);
    }
    mbar_init(BAR(B_DONE), 1);
    fence_mbar_init();
  }
  if (warp == kTmaWarp && lane == 0) {
    prefetch_tmap(tmap);
    if (kPair) prefetch_tmap(tmapK);
  }
  if (warp == kMmaWarp) {
    if constexpr (kPair) {
      tmem_alloc_pair(smem_u32(tmem_slot), 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), 512);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) cluster_sync();   // both CTAs' barriers initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp >= 8) {
   regs_dec<kProducerRegs>();
   if (warp == kTmaWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t kc = 0, vc = 0, uc = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        Unit w;
        const int st = unit_of_cta<kRows>(p, k, w, cta, ncta);
        if (st == 0) break;
        if (st == 2) continue;
        if (st < 0) {
          atomicOr(p.err, kErrBadUnit);
          break;
        }
        const SegDesc& sd = p.seg[w.seg];
        const int hc = p.fused ? w.r * p.Hl + w.j : w.j;   // head coordinate
        const int rc = p.fused ? 0 : w.r;                  // rank coordinate
        if (uc > 0 && !(ok = mbar_wait<kPair>(BAR(B_QEMPTY), (uc - 1) & 1, g))) break;
        for (int i = 0; i < 2; ++i) {
          const int q_row = w.q0 + (kPair ? i * 2 * BM + static_cast<int>(cr) * BM : i * BM);
          mbar_arrive_expect_tx(BAR(B_QFULL0 + i), kTileBytes);
          for (int h = 0; h < G::kBoxes; ++h)
            tma_load_5d(sbase + kOffQ + i * kTileBytes + h * kBoxBytes, tmap, BAR(B_QFULL0 + i), 64 * h, hc, q_row,
                        0, rc);
        }
        const int nkv = unit_kv_tiles<kRows>(p, sd, w);
        for (int t = 0; t < nkv; ++t) {
          const int kv0 = sd.start + t * BN;
          {
            const uint32_t s = kc % kStages, ph = (kc / kStages) & 1;
            if (kc >= kStages && !(ok = mbar_wait(BAR(B_KEMPTY0 + s), ph ^ 1, g))) break;
            mbar_arrive_expect_tx(BAR(B_KFULL0 + s), G::kKBytes);
            if constexpr (kPair) {   // this CTA's 64 keys, both 64-column boxes (64 rows each)
              for (int h = 0; h < 2; ++h)
                tma_load_5d(sbase + kOffK + s * G::kKBytes + h * (G::kKBytes / 2), tmapK, BAR(B_KFULL0 + s),
                            64 * h, hc, kv0 + 64 * static_cast<int>(cr), 1, rc);
            } else {
              for (int h = 0; h < G::kBoxes; ++h)
                tma_load_5d(sbase + kOffK + s * G::kKBytes + h * kBoxBytes, tmap, BAR(B_KFULL0 + s), 64 * h, hc,
                            kv0, 1, rc);
            }
            ++kc;
          }
          {
            const uint32_t s = vc % kStages, ph = (vc / kStages) & 1;
            if (vc >= kStages && !(ok = mbar_wait(BAR(B_VEMPTY0 + s), ph ^ 1, g))) break;
            mbar_arrive_expect_tx(BAR(B_VFULL0 + s), G::kVBytes);
            if constexpr (kPair) {   // this CTA's 64 head-dim columns of all 128 keys: one box
              tma_load_5d(sbase + kOffV + s * G::kVBytes, tmap, BAR(B_VFULL0 + s), 64 * static_cast<int>(cr), hc,
                          kv0, 2, rc);
            } else {
              for (int h = 0; h < G::kBoxes; ++h)
                tma_load_5d(sbase + kOffV + s * G::kVBytes + h * kBoxBytes, tmap, BAR(B_VFULL0 + s), 64 * h, hc,
                            kv0, 2, rc);
            }
            ++vc;
          }
        }
        ++uc;
      }
      // drain: every copy this thread issued has landed before the CTA exits
      if (uc > 0) {
        drain_wait(BAR(B_QFULL0), (uc - 1) & 1);
        drain_wait(BAR(B_QFULL1), (uc - 1) & 1);
      }
      for (uint32_t n = (kc > kStages ? kc - kStages : 0); n < kc; ++n)
        drain_wait(BAR(B_KFULL0 + n % kStages), (n / kStages) & 1);
      for (uint32_t n = (vc > kStages ? vc - kStages : 0); n < vc; ++n)
        drain_wait(BAR(B_VFULL0 + n % kStages), (n / kStages) & 1);
    }
   } else if (kPair && warp == kFwdWarp) {
    // ------------------------------------------------------------ fill forwarder (odd CTA of a pair)
    // Follows the producer's fills in order: once this CTA's half of a fill
    // has landed, arrive on the even CTA's barrier of that fill.
    if (!leader && lane == 0) {
      uint32_t kc = 0, vc = 0, uc = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        Unit w;
        const int st = unit_of_cta<kRows>(p, k, w, cta, ncta);
        if (st == 0 || st < 0) break;
        if (st == 2) continue;
        const int nkv = unit_kv_tiles<kRows>(p, p.seg[w.seg], w);
        for (int i = 0; ok && i < 2; ++i) {
          if (!(ok = mbar_wait(BAR(B_QFULL0 + i), uc & 1, g))) break;
          mbar_arrive_cluster(LBAR(B_QFULL0 + i));
        }
        for (int t = 0; ok && t < nkv; ++t) {
          if (!(ok = mbar_wait(BAR(B_KFULL0 + kc % kStages), (kc / kStages) & 1, g))) break;
          mbar_arrive_cluster(LBAR(B_KFULL0 + kc % kStages));
          ++kc;
          if (!(ok = mbar_wait(BAR(B_VFULL0 + vc % kStages), (vc / kStages) & 1, g))) break;
          mbar_arrive_cluster(LBAR(B_VFULL0 + vc % kStages));
          ++vc;
        }
        ++uc;
      }
    }
   } else if (kPair && warp == kHandWarp) {
    // ------------------------------------------------------------ hand-off forwarder (odd CTA of a pair)
    // Forwards this CTA's completed P and O hand-off phases to the even CTA,
    // in the order the MMA thread consumes them (O of the previous unit, then
    // P by halves, tile 0 before tile 1), so this CTA's barrier is never more
    // than one phase ahead of the forwarder.
    if (!leader && lane == 0) {
      uint32_t pc = 0, uc = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        Unit w;
        const int st = unit_of_cta<kRows>(p, k, w, cta, ncta);
        if (st == 0 || st < 0) break;
        if (st == 2) continue;
        const int nkv = unit_kv_tiles<kRows>(p, p.seg[w.seg], w);
        for (int t = 0; ok && t < nkv; ++t) {
          for (int i = 0; ok && i < 2; ++i) {
            if (t == 0 && uc > 0) {
              if (!(ok = mbar_wait(BAR(B_OEMPTY0 + i), (uc - 1) & 1, g))) break;
              mbar_arrive_cluster(LBAR(B_OEMPTY0 + i));
            }
            if (!(ok = mbar_wait(BAR(B_PHALF0 + i), pc & 1, g))) break;
            mbar_arrive_cluster(LBAR(B_PHALF0 + i));
            if (!(ok = mbar_wait(BAR(B_PFULL0 + i), pc & 1, g))) break;
            mbar_arrive_cluster(LBAR(B_PFULL0 + i));
          }
          ++pc;
        }
        ++uc;
      }
    }
   } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ tcgen05 issuer
    if (lane == 0 && leader) {
      uint32_t kc = 0, vc = 0, uc = 0, pc = 0;
      bool ok = true;
      // descriptors computed once; each group of 8 MMAs is one asm block.  In
      // a pair the same shared-memory offsets hold the odd CTA's halves.
      const uint64_t dQ0 = desc_sw128(sbase + kOffQ, 16, 1024);
      const uint64_t dQ1 = desc_sw128(sbase + kOffQ + kTileBytes, 16, 1024);
      const uint64_t dK0 = desc_sw128(sbase + kOffK, 16, 1024);
      const uint64_t dK1 = desc_sw128(sbase + kOffK + G::kKBytes, 16, 1024);
      // V is read MN-major: the leading byte offset steps to the second
      // 64-column box of a bf16 tile (an E4M3 tile's 128 columns are one box;
      // a pair's CTA holds one 64-column box)
      const uint64_t dV0 = desc_sw128(sbase + kOffV, kBoxBytes, 1024);
      const uint64_t dV1 = desc_sw128(sbase + kOffV + G::kVBytes, kBoxBytes, 1024);
      auto issue_s = [&](int i, uint32_t ks) {
        if (kPair)
          mma_ss_k128_pair(tmem + kColS0 + 128 * i, i ? dQ1 : dQ0, ks ? dK1 : dK0, kIdescS2, 0);
        else if (kFp8)
          mma_ss_f8_k128(tmem + kColS0 + 128 * i, i ? dQ1 : dQ0, ks ? dK1 : dK0, kIdescS8, 0);
        else
          mma_ss_k128(tmem + kColS0 + 128 * i, i ? dQ1 : dQ0, ks ? dK1 : dK0, kIdescS, 0);
      };
      // O_i (+)= P_i V over keys [64 h, 64 h + 64): P columns [32 h, 32 h + 32)
      // (bf16 pairs) or [16 h, 16 h + 16) (E4M3 quads), V rows 64 h.. (8 KB
      // further in each 128-byte-wide box: +512 descriptor units)
      auto issue_pv_half = [&](int i, uint32_t vs, int h, uint32_t acc) {
        if (kPair)
          mma_ts_k64_pair(tmem + kColO0 + 128 * i, tmem + kColS0 + 128 * i + 32 * h, (vs ? dV1 : dV0) + 512 * h,
                          kIdescPV2, acc);
        else if (kFp8)
          mma_ts_f8_k64(tmem + kColO0 + 128 * i, tmem + kColS0 + 128 * i + 16 * h, (vs ? dV1 : dV0) + 512 * h,
                        kIdescPV8, acc);
        else
          mma_ts_k64(tmem + kColO0 + 128 * i, tmem + kColS0 + 128 * i + 32 * h, (vs ? dV1 : dV0) + 512 * h,
                     kIdescPV, acc);
      };
      for (int k = 0; ok; ++k) {
        Unit w;
        const int st = unit_of_cta<kRows>(p, k, w, cta, ncta);
        if (st == 0 || st < 0) break;
        if (st == 2) continue;
        const SegDesc& sd = p.seg[w.seg];
        const int nkv = unit_kv_tiles<kRows>(p, sd, w);
        if (!(ok = mbar_wait<kPair>(BAR(B_QFULL0), uc & 1, g))) break;
        if (!(ok = mbar_wait<kPair>(BAR(B_QFULL1), uc & 1, g))) break;
        uint32_t ks = kc % kStages;
        if (!(ok = mbar_wait<kPair>(BAR(B_KFULL0 + ks), (kc / kStages) & 1, g))) break;
        tc_fence_after();
        issue_s(0, ks);
        commit(B_SFULL0);
        issue_s(1, ks);
        commit(B_SFULL1);
        ++kc;
        if (nkv == 1) commit(B_QEMPTY);
        for (int t = 0; ok && t < nkv; ++t) {
          const uint32_t vs = vc % kStages;
          if (!(ok = mbar_wait<kPair>(BAR(B_VFULL0 + vs), (vc / kStages) & 1, g))) break;
          for (int i = 0; i < 2; ++i) {
            if (t == 0 && uc > 0 && !(ok = mbar_wait<kPair>(BAR(B_OEMPTY0 + i), (uc - 1) & 1, g))) break;
            if (!(ok = mbar_wait<kPair>(BAR(B_PHALF0 + i), pc & 1, g))) break;
            tc_fence_after();
            issue_pv_half(i, vs, 0, t > 0);
            if (!(ok = mbar_wait<kPair>(BAR(B_PFULL0 + i), pc & 1, g))) break;
            tc_fence_after();
            issue_pv_half(i, vs, 1, 1);
            if (t == nkv - 1) {
              commit(B_OFULL0 + i);
            } else if (i == 0) {
              ks = kc % kStages;
              if (!(ok = mbar_wait<kPair>(BAR(B_KFULL0 + ks), (kc / kStages) & 1, g))) break;
              tc_fence_after();
              issue_s(0, ks);
              commit(B_SFULL0);
            } else {
              issue_s(1, ks);
              commit(B_SFULL1);
              ++kc;
              if (t + 1 == nkv - 1) commit(B_QEMPTY);
            }
          }
          ++pc;
          if (!ok) break;
          ++vc;
        }
        ++uc;
      }
      // drain: all MMAs this thread issued are complete before TMEM is freed
      if constexpr (kPair)
        mma_commit_pair(LBAR(B_DONE));
      else
        mma_commit(BAR(B_DONE));
      drain_wait(BAR(B_DONE), 0);
    }
   }
  } else {
    regs_inc<kSoftmaxRegs>();
    // ------------------------------------------------------------ softmax warpgroups
    const int wg = warp >> 2;                  // Q tile 0 or 1
    const int row = threadIdx.x & 127;         // query row inside the tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + kColS0 + 128 * wg;
    const uint32_t tO = tmem + lane_base + kColO0 + 128 * wg;
    const float sl2 = p.scale_log2;
    uint32_t sc = 0, uc = 0;
    uint32_t kslot = 0, vslot = 0;   // K / V ring fills consumed (warpgroup 1 releases them)
    bool ok = true;
    for (int k = 0; ok; ++k) {
      Unit w;
      const int st = unit_of_cta<kRows>(p, k, w, cta, ncta);
      if (st == 0 || st < 0) break;
      if (st == 2) continue;
      const SegDesc& sd = p.seg[w.seg];
      const int nkv = unit_kv_tiles<kRows>(p, sd, w);
      // first query row of this thread's tile in this CTA
      const int tile_row0 = w.q0 + (kPair ? wg * 2 * BM + static_cast<int>(cr) * BM : wg * BM);
      float m_used = -INFINITY;   // running max, log2 units (scaled)
      float l = 0.f;              // running sum of exp2(x - m_used)
      for (int t = 0; t < nkv; ++t) {
        if (!(ok = mbar_wait_warp<kPair>(BAR(B_SFULL0 + wg), sc & 1, g))) break;
        ++sc;
        if (wg == 1 && row == 0) {
          // S1(t) complete => S0(t) complete (same issuer, issued earlier):
          // K(t) is free.  S1(t) was issued after P1(t-1) V(t-1), the last
          // use of V(t-1).  Releasing here saves two tcgen05.commit per step.
          mbar_arrive(BAR(B_KEMPTY0 + kslot % kStages));
          ++kslot;
          if (t > 0) mbar_arrive(BAR(B_VEMPTY0 + vslot++ % kStages));
        }
        tc_fence_after();
        uint32_t sraw[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, sraw[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_regs_ready(sraw[c]);
        float* s = reinterpret_cast<float*>(&sraw[0][0]);
        // keys past the segment end, and (causal) past this row, are masked
        const int kv0 = sd.start + t * BN;
        const int row_n = tile_row0 + row;
        const int valid = (p.causal ? min(sd.kv_end, row_n + 1) : sd.kv_end) - kv0;   // may be <= 0
        const bool masked = __any_sync(0xffffffffu, valid < BN);
        if (masked) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= valid) s[c] = -INFINITY;
        }
        // row max: eight independent 3-input max chains, then a short tree
        float mxa[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mxa[k] = fmax3(s[16 * k], s[16 * k + 1], s[16 * k + 2]);
#pragma unroll
        for (int i = 3; i < 15; i += 2)
#pragma unroll
          for (int k = 0; k < 8; ++k) mxa[k] = fmax3(mxa[k], s[16 * k + i], s[16 * k + i + 1]);
#pragma unroll
        for (int k = 0; k < 8; ++k) mxa[k] = fmaxf(mxa[k], s[16 * k + 15]);
        const float mx = fmax3(fmax3(mxa[0], mxa[1], mxa[2]), fmax3(mxa[3], mxa[4], mxa[5]), fmaxf(mxa[6], mxa[7]));
        const float m_new = fmaxf(m_used, mx * sl2);
        // Move the running max only when it grew by more than 8 (log2 units):
        // probabilities stay below 2^8 and O is rescaled rarely.
        bool need = false;
        float f = 1.0f;
        if (t == 0) {
          m_used = m_new;
        } else if (m_new - m_used > 8.0f) {
          need = true;
          f = ex2_approx(m_used - m_new);
          l *= f;
          m_used = m_new;
        }
        if (__any_sync(0xffffffffu, need)) {
          // O holds the sum of earlier tiles (complete: S of this tile was
          // issued after them); scale it to the new max before the next P V.
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + 32 * c, o);
            tmem_wait_ld();
            tmem_regs_ready(o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
            tmem_st32(tO + 32 * c, o);
          }
        }
        const f2 scale2{sl2, sl2}, negm2{-m_used, -m_used};
        f2 acc[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
        // P (bf16 pairs) over the first 64 columns of S, in two halves; the
        // first half is handed to the MMA warp before the second is computed.
        // Masked tiles use MUFU ex2 only, so masked keys give exact zeros.
        const bool emu = !masked;
        if (kFp8 && emu)
          exp_store_half_fp8<true>(s, 0, scale2, negm2, acc, tS);
        else if (kFp8)
          exp_store_half_fp8<false>(s, 0, scale2, negm2, acc, tS);
        else if (emu)
          exp_store_half<true>(s, 0, scale2, negm2, acc, tS);
        else
          exp_store_half<false>(s, 0, scale2, negm2, acc, tS);
        tmem_wait_st();
        tc_fence_before();
        hand_off(B_PHALF0 + wg);
        if (kFp8 && emu)
          exp_store_half_fp8<true>(s, 1, scale2, negm2, acc, tS);
        else if (kFp8)
          exp_store_half_fp8<false>(s, 1, scale2, negm2, acc, tS);
        else if (emu)
          exp_store_half<true>(s, 1, scale2, negm2, acc, tS);
        else
          exp_store_half<false>(s, 1, scale2, negm2, acc, tS);
        {
          const f2 a01 = fadd2(acc[0], acc[1]), a23 = fadd2(acc[2], acc[3]);
          const f2 a = fadd2(a01, a23);
          l += a.x + a.y;
        }
        tmem_wait_st();
        tc_fence_before();
        hand_off(B_PFULL0 + wg);
      }
      if (!ok) break;
      // epilogue: O / l -> bf16 -> global
      if (!(ok = mbar_wait_warp<kPair>(BAR(B_OFULL0 + wg), uc & 1, g))) break;
      if (wg == 1 && row == 0) mbar_arrive(BAR(B_VEMPTY0 + vslot++ % kStages));   // last V of the unit
      tc_fence_after();
      uint32_t oraw[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tO + 32 * c, oraw[c]);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_regs_ready(oraw[c]);
      tc_fence_before();
      hand_off(B_OEMPTY0 + wg);
      const int n = tile_row0 + row;
      if (p.lse && n < sd.q_end && n < p.Np) {
        const int64_t li = (static_cast<int64_t>(w.r) * p.Hl + w.j) * p.lse_stride + n;
        if (in_bounds(li, 1, p.lse_ext, p.err)) p.lse[li] = m_used + log2f(l);
      }
      if (n < sd.q_end && n < p.Np) {
        __nv_bfloat16* obase = p.out;
        int64_t ooff = w.r * p.o_stride_r + n * p.o_stride_n + w.j * p.o_stride_j;
        bool ok = true;
        if (p.push_rows > 0) {   // the owning rank's shard, through its peer pointer
          const int64_t q = n / p.push_rows;
          ok = in_bounds(q, 1, p.push_ranks, p.err);
          obase = static_cast<__nv_bfloat16*>(p.push.p[ok ? q : 0]);
          ooff = (n - q * p.push_rows) * p.o_stride_n + w.j * p.o_stride_j;
        }
        ok = ok && in_bounds(ooff, HD, p.out_ext, p.err);
        uint4* dst = reinterpret_cast<uint4*>(obase + ooff);
        const bool pad = n >= p.N;   // pad rows are written as zeros
        const float inv = 1.0f / l;
        const float* o = reinterpret_cast<const float*>(&oraw[0][0]);
#pragma unroll
        for (int v = 0; v < 16; ++v) {
          uint4 q;
          q.x = pack_bf16x2(o[8 * v + 0] * inv, o[8 * v + 1] * inv);
          q.y = pack_bf16x2(o[8 * v + 2] * inv, o[8 * v + 3] * inv);
          q.z = pack_bf16x2(o[8 * v + 4] * inv, o[8 * v + 5] * inv);
          q.w = pack_bf16x2(o[8 * v + 6] * inv, o[8 * v + 7] * inv);
          if (pad) q = make_uint4(0u, 0u, 0u, 0u);
          if (ok) dst[v] = q;
        }
      }
      ++uc;
    }
  }

  tc_fence_before();
  __syncthreads();
  // in a pair, neither CTA frees TMEM or exits while the other's MMAs,
  // commits or hand-offs may still reach it
  if constexpr (kPair) cluster_sync();
  tc_fence_after();
  if (warp == kMmaWarp) {
    if constexpr (kPair)
      tmem_dealloc_pair(tmem, 512);
    else
      tmem_dealloc(tmem, 512);
  }
}

template <bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ AttnParams p) {
  attn_body<kFp8, false>(&tmap, &tmap, p);
}

// bf16 attention on CTA pairs (clusters of two); tmapK reads 64-key halves of
// the K tiles.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    attn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap tmapK,
                         const __grid_constant__ AttnParams p) {
  attn_body<false, true>(&tmap, &tmapK, p);
}

// ---------------------------------------------------------------- host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static const EncodeTiledFn fn = [] {   // initialised once, thread-safe
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(ptr);
    cudaGetLastError();
    return static_cast<EncodeTiledFn>(nullptr);
  }();
  return fn;
}

// Largest number of CTA pairs resident at once (one pair per two SMs of a
// cluster-capable partition), cached per device.
int g_pair_clusters[256] = {0};

cudaError_t launch_pair_kernel(const CUtensorMap& tmap, const CUtensorMap& tmapK, const AttnParams& p, int grid,
                               int dev, cudaStream_t stream) {
  static PerDeviceOnce setup;
  cudaError_t e = setup.run(dev, [] {
    cudaFuncAttributes fa;
    cudaError_t r = cudaFuncGetAttributes(&fa, attn_fwd_pair_kernel);
    if (r != cudaSuccess) return r;
    if (fa.numRegs != static_cast<int>(kLaunchRegs)) return cudaErrorInvalidConfiguration;   // see register split
    return cudaFuncSetAttribute(attn_fwd_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Smem<false, true>::kBytes);
  });
  if (e != cudaSuccess) return e;
  attn_fwd_pair_kernel<<<grid, kThreads, Smem<false, true>::kBytes, stream>>>(tmap, tmapK, p);
  return cudaGetLastError();
}

int pair_clusters(int dev, int sms) {
  static PerDeviceOnce setup;
  if (dev < 0 || dev >= 256) return sms / 2;
  const cudaError_t e = setup.run(dev, [dev, sms] {
    cudaError_t r = cudaFuncSetAttribute(attn_fwd_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Smem<false, true>::kBytes);
    if (r != cudaSuccess) return r;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = Smem<false, true>::kBytes;
    int n = 0;
    r = cudaOccupancyMaxActiveClusters(&n, attn_fwd_pair_kernel, &cfg);
    if (r != cudaSuccess) return r;
    g_pair_clusters[dev] = n;
    return cudaSuccess;
  });
  if (e != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return g_pair_clusters[dev];
}

template <bool kFp8>
cudaError_t launch_kernel(const CUtensorMap& tmap, const AttnParams& p, int grid, int dev, cudaStream_t stream) {
  static PerDeviceOnce setup;
  cudaError_t e = setup.run(dev, [] {
    cudaFuncAttributes fa;
    cudaError_t r = cudaFuncGetAttributes(&fa, attn_fwd_kernel<kFp8>);
    if (r != cudaSuccess) return r;
    if (fa.numRegs != static_cast<int>(kLaunchRegs)) return cudaErrorInvalidConfiguration;   // see register split
    return cudaFuncSetAttribute(attn_fwd_kernel<kFp8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Smem<kFp8>::kBytes);
  });
  if (e != cudaSuccess) return e;
  attn_fwd_kernel<kFp8><<<grid, kThreads, Smem<kFp8>::kBytes, stream>>>(tmap, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn(const AttnLaunch& a, cudaStream_t stream) {
  const ulysses_plan_t* pl = a.plan;
  EncodeTiledFn encode = get_encode_fn();
  if (!encode) return cudaErrorNotSupported;

  if (a.fp8 && a.fused) return cudaErrorInvalidValue;   // the E4M3 variant reads head-sharded T8 only
  const cuuint64_t eb = a.fp8 ? 1 : 2;                  // bytes per element
  // 5-D view (d, head, token, plane, rank) of the Q/K/V source
  cuuint64_t dims[5], strides[4];
  dims[0] = HD;
  if (!a.fused) {
    dims[1] = a.Hl;
    dims[2] = a.Np;
    dims[3] = a.C;
    dims[4] = a.P;
    strides[0] = HD * eb;
    strides[1] = static_cast<cuuint64_t>(a.Hl) * HD * eb;
    strides[2] = static_cast<cuuint64_t>(a.Np) * a.Hl * HD * eb;
    strides[3] = static_cast<cuuint64_t>(a.C) * a.Np * a.Hl * HD * eb;
  } else {
    dims[1] = a.H;
    dims[2] = a.Np;
    dims[3] = a.C;
    dims[4] = 1;
    strides[0] = HD * 2;
    strides[1] = static_cast<cuuint64_t>(a.tok_stride) * 2;
    strides[2] = static_cast<cuuint64_t>(a.plane_stride) * 2;
    strides[3] = std::max<cuuint64_t>(strides[1] * a.Np, strides[2] * a.C);
  }
  // one box is 128 rows of 128 bytes: 64 bf16 or 128 E4M3 columns
  cuuint32_t box[5] = {a.fp8 ? 128u : 64u, 1, BM, 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUtensorMap tmap, tmapK;
  CUresult cr = encode(&tmap, a.fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5,
                       const_cast<void*>(a.base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                       CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
  // bf16 attention runs on CTA pairs when the plan asks for it; the pair
  // kernel also reads 64-key halves of the K tiles (boxes of 64 rows)
  const bool pair = !a.fp8 && pl->pair_cta;
  if (pair) {
    cuuint32_t boxK[5] = {64, 1, BM / 2, 1, 1};
    cr = encode(&tmapK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(a.base), dims, strides, boxK, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
  }
  const int unit_rows = pair ? kPairUnitRows : kUnitRows;

  AttnParams p;
  std::memset(&p, 0, sizeof(p));
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.lse_stride = a.lse_stride;
  p.err = pl->dev_err;
  p.o_stride_r = a.o_stride_r;
  p.o_stride_n = a.o_stride_n;
  p.o_stride_j = a.o_stride_j;
  p.N = static_cast<int32_t>(a.N);
  p.Np = static_cast<int32_t>(a.Np);
  p.Hl = a.Hl;
  p.P = a.P;
  p.fused = a.fused;
  p.causal = pl->causal;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  if (a.push_rows > 0) {
    // every output row n < Np must map to a table entry n / push_rows
    if (!a.push || a.push_ranks < 1 || a.push_ranks > ULYSSES_MAX_PUSH_RANKS || a.push_rows * a.push_ranks < a.Np)
      return cudaErrorInvalidValue;
    for (int q = 0; q < a.push_ranks; ++q)
      if (!a.push->p[q]) return cudaErrorInvalidValue;
    p.push_rows = a.push_rows;
    p.push_ranks = a.push_ranks;
    p.push = *a.push;
  }
  // extents of the output (per table entry when pushing) and of the lse rows
  p.out_ext = (a.push_rows > 0 ? (a.push_rows - 1) * a.o_stride_n
                               : (a.P - 1) * a.o_stride_r + (a.Np - 1) * a.o_stride_n) +
              (a.Hl - 1) * a.o_stride_j + HD;
  p.lse_ext = static_cast<int64_t>(a.P) * a.Hl * a.lse_stride;

  // Non-empty segments, longest first.  The segment that ends at N also
  // covers the pad query rows [N, Np), which are written as zeros.
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
    SegDesc& d = p.seg[k];
    d.start = sg.start;
    d.kv_end = sg.end;
    d.q_end = (sg.end == a.N) ? static_cast<int32_t>(a.Np) : sg.end;
    d.nqb = (d.q_end - d.start + unit_rows - 1) / unit_rows;
    d.unit_base = units;
    d.pair_base = pairs;
    units += d.nqb * a.P * a.Hl;
    pairs += (d.nqb + 1) / 2 * a.P * a.Hl;
  }
  p.nseg = nseg;
  p.num_units = units;
  p.num_pairs = pairs;
  if (units == 0) return cudaSuccess;

  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (pair) {
    const int clusters = pair_clusters(dev, sms);
    if (clusters < 1) return cudaErrorInvalidConfiguration;
    p.paired = (p.causal && units >= 2 * clusters) ? 1 : 0;
    return launch_pair_kernel(tmap, tmapK, p, 2 * std::min(units, clusters), dev, stream);
  }
  p.paired = (p.causal && units >= 2 * sms) ? 1 : 0;
  const int grid = std::min(units, sms);
  return a.fp8 ? launch_kernel<true>(tmap, p, grid, dev, stream) : launch_kernel<false>(tmap, p, grid, dev, stream);
}

}  // namespace ulysses
