/*
 * ulysses.h -- C ABI of the one-GPU Ulysses sequence-parallel attention layer
 * for NVIDIA B200 (sm_100a).
 *
 * The layer (DistributedAttention.forward_stacked, "hao-ai-lab FastVideo,
 * compare aryan/h3-nvfp4-stack-speedups...main", fastvideo/attention/layer.py)
 * has three steps, all run by kernels of this library:
 *
 *   1. repack_fwd  -- the Ulysses all-to-all in mode 0 (scatter heads, gather
 *      sequence): P sequence-sharded slabs become P head-sharded slabs.
 *      Shapes from the mode comment above ulysses_a2a_tuned ("hao-ai-lab
 *      FastVideo, compare main...perf/ulysses-h3-adaptive",
 *      csrc/comm/ulysses_all_to_all.cu):  [B, S_local, H, D] -> [B, S_global, H_local, D].
 *   2. attn_fwd    -- non-causal softmax attention per head-sharded slab
 *      (the FA4 backend of flash_attn_cute.py: softmax_scale, varlen through
 *      cu_seqlens).
 *   3. repack_bwd  -- mode 1, the inverse map, applied to the attention output.
 *
 * In the one-GPU calls all P "virtual ranks" are slabs of one GPU's memory
 * and there is no collective; the "multi-GPU push" section below runs the
 * same steps with one process per GPU.
 *
 * Notation: N real tokens, P virtual ranks, H heads, D = 128 head dim,
 * Hl = H / P, C planes (3 = Q,K,V; 4 = Q,K,V,G), Nl = ceil(N / P),
 * Np = P * Nl (padded token count).  All tensors are bf16, row-major.
 *
 *   sequence-sharded input  S : Np rows; element (n, c, h, d) at
 *                               n*token_stride + c*plane_stride + h*D + d
 *                               (default token_stride = C*H*D, plane_stride = H*D,
 *                               i.e. [Np, C, H, D]); rank q owns rows [q*Nl, (q+1)*Nl).
 *   head-sharded            T : [P, C, Np, Hl, D];  T[r,c,n,j,d] = S[n,c,r*Hl+j,d]
 *   head-sharded output   O_T : [P, Np, Hl, D]
 *   sequence output       O_S : [Np, H, D]
 *
 * Rows n in [N, Np) are padding: the repack moves them like any other row,
 * attention never uses them as keys and writes zero output rows for them.
 *
 * Conventions for every call:
 *   - pointers named dev_* or taking tensors are caller-owned DEVICE memory on
 *     the current device, 16-byte aligned; outputs must not overlap inputs;
 *   - `stream` is a cudaStream_t (CUstream) passed as void*; NULL is the
 *     legacy default stream;
 *   - calls are asynchronous on `stream`, allocate nothing and do not
 *     synchronise (except ulysses_last_device_error);
 *   - invalid arguments are reported through the return code, never abort.
 */
#ifndef ULYSSES_H_
#define ULYSSES_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
enum {
  ULYSSES_OK = 0,
  ULYSSES_ERR_ARG = 1,          /* null/overlapping pointer, bad size, bad cu_seqlens */
  ULYSSES_ERR_DIVISIBILITY = 2, /* H % P != 0 (heads must split evenly across ranks) */
  ULYSSES_ERR_ALIGN = 3,        /* pointer or stride not a multiple of 16 bytes */
  ULYSSES_ERR_WINDOW = 4,       /* one plane per rank exceeds the 1 GiB window */
  ULYSSES_ERR_WORKSPACE = 5,    /* workspace smaller than ulysses_workspace_bytes() */
  ULYSSES_ERR_CUDA = 6,         /* a CUDA runtime/driver call failed (or no device) */
  ULYSSES_ERR_DEVICE = 7,       /* a kernel reported an error (see ulysses_last_device_error) */
  ULYSSES_ERR_UNSUPPORTED = 8   /* D != 128, too many sequences, ... */
};

/* Per-rank window cap: at most 1 GiB moved per rank per repack launch
 * ("Ulysses performance on GB200": each rank keeps at most 1 GiB of window
 * storage and exchanges one plane at a time; MAX_WINDOW_BYTES in ulysses_a2a.py). */
#define ULYSSES_MAX_WINDOW_BYTES (1024LL * 1024LL * 1024LL)
/* Most packed sequences one plan accepts (cu_seqlens has num_seqs + 1 entries). */
#define ULYSSES_MAX_SEQS 64
/* ulysses_plan_ex flag: causal attention (query n sees keys m <= n of its
 * segment), as in the causal flash wrapper of the prime-rl Ulysses context
 * parallelism pull request. */
#define ULYSSES_PLAN_CAUSAL 1u
/* ulysses_plan_ex flag: run the bf16 attention forward on CTA pairs
 * (clusters of two SMs; one cta_group::2 MMA of 256 query rows per tile, each
 * SM loading half of every K and V tile) instead of the default one CTA per
 * SM.  Both give the same bits; on B200 the pair kernel measured 19-22%
 * slower (the cross-SM hand-offs lengthen the S -> softmax -> P V chain that
 * bounds the loop), so it is opt-in. */
#define ULYSSES_PLAN_PAIR_ATTENTION 2u
/* ulysses_plan_ex flag: run the attention backward in two passes without
 * atomics (keys, then queries; S and dP are computed in both), so its output
 * is the same bits on every run.  The default is one pass over the keys that
 * adds dQ into an fp32 accumulator in the workspace with reductions performed
 * in L2: faster, but the order of those additions varies between runs, and so
 * can the last bit of a dQ value. */
#define ULYSSES_PLAN_DETERMINISTIC 4u
/* Most ranks the multi-GPU push calls address (one NVLink domain). */
#define ULYSSES_MAX_PUSH_RANKS 64

typedef struct ulysses_plan_s ulysses_plan_t;

/*
 * Create a plan (host object owned by the library; free with
 * ulysses_plan_destroy).  The plan is immutable and may be shared by any
 * number of calls; backward reuses the forward plan, as _FusedUlyssesA2A does
 * ("Outputs own their storage, and backward uses the plan saved by its forward").
 *
 *   N            real tokens (>= 1)
 *   H, D, P      heads, head dim (must be 128), virtual ranks (1 <= P <= H, H % P == 0)
 *   planes       C: 3 (Q,K,V) or 4 (Q,K,V,G; G is moved but not attended); 1..8 accepted
 *   token_stride, plane_stride
 *                element strides of the sequence-sharded input; 0, 0 selects
 *                [Np, C, H, D].  Must be multiples of 8 elements (16 bytes).
 *   plane_chunk  planes per repack launch; 0 = the largest count whose bytes
 *                per rank fit in 1 GiB
 *   cu_seqlens_host, num_seqs
 *                host array of num_seqs+1 int32 prefix sums (first 0, last N,
 *                non-decreasing) for packed varlen sequences attended
 *                block-diagonally; NULL/0 = one sequence of length N.
 *
 * Errors: ARG, DIVISIBILITY, ALIGN, WINDOW (one plane per rank > 1 GiB, or a
 * plane_chunk whose bytes exceed it), UNSUPPORTED.  On success *out is set.
 * The plan holds a 16-byte device error word on the device current at
 * creation; without a CUDA device the plan is still created so its sizes can
 * be queried, and every launch returns ULYSSES_ERR_CUDA.
 */
int ulysses_plan(ulysses_plan_t** out, int64_t N, int32_t H, int32_t D, int32_t P, int32_t planes,
                 int64_t token_stride, int64_t plane_stride, int64_t plane_chunk,
                 const int32_t* cu_seqlens_host, int32_t num_seqs);

/* ulysses_plan with option flags (ULYSSES_PLAN_CAUSAL,
 * ULYSSES_PLAN_PAIR_ATTENTION, ULYSSES_PLAN_DETERMINISTIC); ulysses_plan is
 * ulysses_plan_ex with flags = 0.  Unknown flag bits -> ULYSSES_ERR_ARG. */
int ulysses_plan_ex(ulysses_plan_t** out, int64_t N, int32_t H, int32_t D, int32_t P, int32_t planes,
                    int64_t token_stride, int64_t plane_stride, int64_t plane_chunk,
                    const int32_t* cu_seqlens_host, int32_t num_seqs, uint32_t flags);

void ulysses_plan_destroy(ulysses_plan_t* plan);

/* Np = P * ceil(N / P): rows every buffer is sized for. */
int64_t ulysses_plan_padded_tokens(const ulysses_plan_t* plan);

/* Planes moved per repack launch (the window chunk the plan chose). */
int32_t ulysses_plan_plane_chunk(const ulysses_plan_t* plan);

/* Bytes one rank exchanges per plane: Nl * H * D * 2. */
int64_t ulysses_plan_window_bytes_per_plane(const ulysses_plan_t* plan);

/* Workspace for ulysses_layer_fwd with fused = 0: T (P*C*Np*Hl*D) plus
 * O_T (P*Np*Hl*D) bf16 elements, each region 256-byte aligned.  0 bytes are
 * needed with fused = 1. */
size_t ulysses_workspace_bytes(const ulysses_plan_t* plan);

/*
 * Step 1, Ulysses mode 0: src_seq (sequence-sharded, plan strides, C planes)
 * -> dst_heads T [P, C, Np, Hl, D].  One launch per plane chunk, each moving
 * at most 1 GiB per rank (the per-plane loop of run_armed in ulysses_a2a.py).
 * Bit-exact copy.  Errors: ARG, ALIGN, CUDA.
 */
int ulysses_repack_fwd(const ulysses_plan_t* plan, const void* src_seq, void* dst_heads, void* stream);

/*
 * Step 1 with the QKV prologue fused in: the mode-0 repack of
 * ulysses_repack_fwd, where planes 0 (Q) and 1 (K) first get per-head RMSNorm
 * and partial rotate-half RoPE, as mk/qkv_prologue.py does on the FastVideo
 * layer page ("per-head QK RMSNorm + partial RoPE + stacked QKV output"):
 *   y = x / sqrt(mean(x^2) + eps) * w                     (w: norm_q_weight / norm_k_weight)
 *   y[i] = y[i] cos[n,i] - y[i + rd/2] sin[n,i]          for i <  rd/2
 *   y[i] = y[i] cos[n,i] + y[i - rd/2] sin[n,i]          for rd/2 <= i < rd
 * channels >= rd unchanged; planes >= 2 copied verbatim.  fp32 arithmetic,
 * one bf16 rounding per output element.  It moves the same bytes as the plain
 * repack (the prologue's own read and write of Q and K disappear).
 *   norm_q_weight, norm_k_weight: device bf16 [D]
 *   cos_table, sin_table:         device bf16 [Np, rotary_dim] (row n = token n;
 *                                 may be NULL when rotary_dim = 0)
 *   rotary_dim:                   0 .. D, a multiple of 16 (96 in the pages)
 *   eps:                          > 0 (1e-5 in the pages)
 * Errors: ARG (C < 2, bad eps/rotary_dim, overlap), ALIGN (any pointer not
 * 16-byte aligned), UNSUPPORTED (rotary_dim % 16 != 0), CUDA.
 */
int ulysses_prologue_repack_fwd(const ulysses_plan_t* plan, const void* src_seq, void* dst_heads,
                                const void* norm_q_weight, const void* norm_k_weight, const void* cos_table,
                                const void* sin_table, int32_t rotary_dim, float eps, void* stream);

/*
 * Step 3, Ulysses mode 1 (the inverse map): src_heads [P, planes, Np, Hl, D]
 * -> dst_seq.  With planes == C, dst_seq uses the plan's input strides (a full
 * round trip restores the input bit for bit).  With planes < C, dst_seq is a
 * dense [Np, planes, H, D] buffer; planes == 1 gives the layer output
 * [Np, H, D].  Errors: ARG, ALIGN, CUDA.
 */
int ulysses_repack_bwd(const ulysses_plan_t* plan, const void* src_heads, void* dst_seq, int32_t planes,
                       void* stream);

/*
 * Step 2: out_heads O_T [P, Np, Hl, D] = softmax(softmax_scale * Q K^T) V for
 * every rank r and local head j, with Q, K, V the planes 0, 1, 2 of
 * qkv_heads T [P, C, Np, Hl, D].  Non-causal unless the plan was made with
 * ULYSSES_PLAN_CAUSAL; query row n attends to the keys of its cu_seqlens
 * segment (all keys < N without cu_seqlens), only those m <= n when causal.  fp32
 * accumulation and softmax, bf16 probabilities for the second product, bf16
 * output; pad rows [N, Np) are written as zeros.  Errors: ARG, ALIGN, CUDA.
 */
int ulysses_attn_fwd(const ulysses_plan_t* plan, const void* qkv_heads, void* out_heads, float softmax_scale,
                     void* stream);

/* ---------------------------------------------------------------- FP8 (E4M3) variant
 * The MiniMax-H3 recipe branch described on "Request FA4's 2-CTA kernel for
 * MiniMax-H3 on SM103 and SM107" (TensorRT-LLM pull request 21275) runs
 * cuDNN FP8 attention with Q and K cast to FP8 in a fused step, and the
 * layer page's FA4 wrappers have an FP8 P V path (FA4_FP8_PV_USE_FUSED_PACK).
 * The pages fix no scaling recipe; here the cast is a direct conversion of
 * each bf16 value of Q, K, V to the nearest E4M3 value (ties to even,
 * saturating at +-448, no scale factor), the probabilities P are stored as
 * E4M3 for the second product (they stay below 2^8), and accumulation,
 * softmax and the output are as in the bf16 path.  Plane 3 (the gate) is cast
 * and repacked with the others but not attended.
 */

/*
 * Mode 0 with the cast: dst_heads_fp8 [P, C, Np, Hl, D] of one-byte E4M3
 * codes, T8[r, c, n, j, d] = e4m3(S[n, c, r*Hl + j, d]).  Same window rule as
 * ulysses_repack_fwd.  Errors: ARG (null or overlapping pointers), ALIGN,
 * CUDA.
 */
int ulysses_repack_fwd_fp8(const ulysses_plan_t* plan, const void* src_seq, void* dst_heads_fp8, void* stream);

/*
 * Step 2 on E4M3 operands: out_heads O_T [P, Np, Hl, D] (bf16) from
 * qkv_heads_fp8 [P, C, Np, Hl, D] (planes 0, 1, 2 = Q, K, V as E4M3 codes).
 * Segments and the causal flag as ulysses_attn_fwd.  Errors: ARG, ALIGN,
 * CUDA.
 */
int ulysses_attn_fwd_fp8(const ulysses_plan_t* plan, const void* qkv_heads_fp8, void* out_heads,
                         float softmax_scale, void* stream);

/* Workspace of ulysses_layer_fwd_fp8: T8 (one byte per element) then O_T (bf16),
 * each 256-byte aligned. */
size_t ulysses_workspace_bytes_fp8(const ulysses_plan_t* plan);

/*
 * The FP8 layer with softmax_scale = 1/sqrt(D): ulysses_repack_fwd_fp8 ->
 * ulysses_attn_fwd_fp8 -> ulysses_repack_bwd(planes = 1), out_seq O_S
 * [Np, H, D] bf16 from qkv_seq (bf16, plan strides).  Errors: ARG, ALIGN,
 * WORKSPACE, CUDA.
 */
int ulysses_layer_fwd_fp8(const ulysses_plan_t* plan, const void* qkv_seq, void* out_seq, void* workspace,
                          size_t workspace_bytes, void* stream);

/*
 * ulysses_layer_fwd_fp8 from HOST buffers, streamed by head groups exactly as
 * ulysses_layer_fwd_host (same groups, streams, events and ordering against
 * `stream`); the workspace is ulysses_workspace_bytes_fp8() long and holds
 * the groups' E4M3 head slabs, then their outputs.  The result equals
 * ulysses_layer_fwd_fp8's bit for bit.  Errors: as ulysses_layer_fwd_host.
 */
int ulysses_layer_fwd_fp8_host(const ulysses_plan_t* plan, const void* host_qkv_seq, void* host_out_seq,
                               void* dev_qkv_seq, void* dev_out_seq, void* workspace, size_t workspace_bytes,
                               void* stream);

/* ---------------------------------------------------------------- multi-GPU push
 * Steps 1 and 3 across P real GPUs, one process per GPU: rank q owns the
 * sequence rows [q*Nl, (q+1)*Nl).  These are the all-to-all exchanges of
 * "Ulysses performance on GB200" (fine-grained remote stores into each peer's
 * window, one plane at a time, 1 GiB per rank), done as a push: each rank
 * writes its data straight into the other ranks' buffers with plain 16-byte
 * stores through peer pointers.  The pointers are device addresses valid on
 * the calling rank's device -- CUDA IPC (or VMM) mappings of the peers'
 * allocations over NVLink, or local buffers when the ranks are emulated on
 * one GPU.  No TMA and no multicast reads or writes peer memory.
 *
 * Every rank creates the plan with the same global arguments (N, H, P,
 * planes, cu_seqlens, flags); the shards use the default token-interleaved
 * layout (token_stride = C*H*D, plane_stride = H*D), otherwise
 * ULYSSES_ERR_UNSUPPORTED, as is P > ULYSSES_MAX_PUSH_RANKS.
 *
 *   shard       S_q : [Nl, planes, H, D] on rank q; row i is sequence row
 *                     q*Nl + i (rows at or past N are padding and must be zero)
 *   head slab   T_r : [planes, Np, Hl, D] on rank r (rank r's slab of T)
 *   out shard   O_q : [Nl, planes, H, D] on rank q ([Nl, H, D] for the layer)
 * (planes = C for the layer's input, 1 for its output, 3 for Q/K/V gradients).
 *
 * For training, a rank keeps its head-sharded output and log-sum-exp
 * (ulysses_attn_fwd_lse_slab, then ulysses_repack_bwd_push of the output),
 * pushes the output gradient into the dO slabs (ulysses_repack_fwd_push with
 * planes = 1), runs ulysses_attn_bwd_slab and pushes dQ, dK, dV back
 * (ulysses_repack_bwd_push with planes = 3).
 *
 * Pointer tables are HOST arrays of P device pointers indexed by rank; each
 * must be 16-byte aligned, non-null, and must not overlap the call's source
 * or another entry's buffer.
 * The calls only store: the caller orders the exchange, i.e. rank r reads T_r
 * (or O_r) only after every rank's push into it has completed, with a
 * stream-ordered barrier (an NCCL all-reduce of one word on the same stream,
 * or a symmetric-memory barrier).  Errors: ARG (rank out of range, null or
 * overlapping pointer), ALIGN, UNSUPPORTED, CUDA.
 */

/* Step 1 pushed by rank `rank`, on the first `planes` planes (1..C; C for
 * the layer's Q, K, V, 1 for an output gradient): src_shard [Nl, planes, H, D]
 * into head slabs [planes, Np, Hl, D],
 *   dst_heads[r][c, rank*Nl + i, j, :] = src_shard[i, c, r*Hl + j, :]
 * for every rank r, plane c and row i < Nl.  One launch per plane chunk (at
 * most 1 GiB per rank, as ulysses_repack_fwd). */
int ulysses_repack_fwd_push(const ulysses_plan_t* plan, int32_t rank, const void* src_shard,
                            void* const* dst_heads, int32_t planes, void* stream);

/* Steps 2 and 3 in one kernel on rank `rank`: attention over the rank's head
 * slab `heads` (T_r, all Np rows; segments, causal flag and pad rows as
 * ulysses_attn_fwd), each output row n stored by the epilogue straight into
 * its owning rank q = n / Nl:  dst_seq[q][n - q*Nl, rank*Hl + j, :] = O(n, j). */
int ulysses_attn_fwd_push(const ulysses_plan_t* plan, int32_t rank, const void* heads, void* const* dst_seq,
                          float softmax_scale, void* stream);

/* Step 3 alone, pushed by rank `rank` from its head rows src_heads
 * [planes, Np, Hl, D]: dst_seq[q][i, c, rank*Hl + j, :] =
 * src_heads[c, q*Nl + i, j, :] into [Nl, planes, H, D] shards (1 <= planes <= C). */
int ulysses_repack_bwd_push(const ulysses_plan_t* plan, int32_t rank, const void* src_heads,
                            void* const* dst_seq, int32_t planes, void* stream);

/* ---- all-to-all fallback (no peer access): the collective moves the bytes,
 * these kernels pack and unpack them.  Chunk r of each buffer is what rank r
 * receives (or sent), in rank order, as an all-to-all with equal splits
 * (ncclAllToAll, torch.distributed.all_to_all_single) expects. */

/* Plane `plane` of src_shard [Nl, planes, H, D] (planes = C for the layer's
 * input, 1 for an output gradient) -> send [P, Nl, Hl, D]:
 *   send[r, i, j, :] = src_shard[i, plane, r*Hl + j, :].
 * After the exchange, rank r's receive buffer [P, Nl, Hl, D] is that plane of
 * its head slab, rows in rank order.  Errors: ARG (planes outside 1..8, plane
 * outside 0..planes-1, null or overlapping pointers), ALIGN, UNSUPPORTED, CUDA. */
int ulysses_a2a_pack(const ulysses_plan_t* plan, const void* src_shard, int32_t planes, int32_t plane, void* send,
                     void* stream);

/* The output direction: a plane of a rank's head-sharded rows [Np, Hl, D] is
 * already [P, Nl, Hl, D] in destination order; after the exchange,
 * recv [P, Nl, Hl, D] (chunk r = rank r's heads of this rank's rows) goes to
 * plane `plane` of out_shard [Nl, planes, H, D]:
 *   out_shard[i, plane, r*Hl + j, :] = recv[r, i, j, :].
 * Errors: as ulysses_a2a_pack. */
int ulysses_a2a_unpack(const ulysses_plan_t* plan, const void* recv, void* out_shard, int32_t planes, int32_t plane,
                       void* stream);

/* Attention over ONE rank's head slab of the plan (steps 2 of the multi-GPU
 * layer for training): heads T_r [C, Np, Hl, D] -> out_heads [Np, Hl, D] and
 * lse [Hl][stride] (ulysses_lse_bytes(plan) / P bytes; the stride as
 * ulysses_attn_fwd_lse).  Segments, causal flag and pad rows as
 * ulysses_attn_fwd.  Errors: as ulysses_attn_fwd_lse. */
int ulysses_attn_fwd_lse_slab(const ulysses_plan_t* plan, const void* heads, void* out_heads, void* lse,
                              float softmax_scale, void* stream);

/* The attention backward of one rank's slab: (dQ, dK, dV) [3, Np, Hl, D] from
 * heads T_r, its out_heads and lse (ulysses_attn_fwd_lse_slab) and the output
 * gradient dout_heads [Np, Hl, D]; the workspace is
 * ulysses_attn_bwd_workspace_bytes(plan) / P bytes.  Errors: as
 * ulysses_attn_bwd. */
int ulysses_attn_bwd_slab(const ulysses_plan_t* plan, const void* heads, const void* out_heads,
                          const void* dout_heads, const void* lse, void* dqkv_heads, void* workspace,
                          size_t workspace_bytes, float softmax_scale, void* stream);

/* ---------------------------------------------------------------- training
 * The gradient of the layer.  The FastVideo transport carries gradients back
 * through the inverse map under the forward's plan (_FusedUlyssesA2A.backward
 * in ulysses_a2a.py); attention's own gradient is that of
 * O = softmax(s Q K^T) V:  dV = P^T dO,  dS = P o (dO V^T - rowsum(dO o O)),
 * dQ = s dS K,  dK = s dS^T Q.
 */

/* Bytes of the log-sum-exp buffer: P*Hl rows of lse_row_stride floats
 * (Np rounded up to 4, plus 128). */
size_t ulysses_lse_bytes(const ulysses_plan_t* plan);

/*
 * ulysses_attn_fwd that also writes, per (rank, local head, query row n),
 * lse[(r*Hl + j) * stride + n] = m + log2(l): the row's log-sum-exp of
 * s*log2(e)*Q K^T in base 2 (device fp32, ulysses_lse_bytes()).  Errors: as
 * ulysses_attn_fwd.
 */
int ulysses_attn_fwd_lse(const ulysses_plan_t* plan, const void* qkv_heads, void* out_heads, void* lse,
                         float softmax_scale, void* stream);

/* Workspace of ulysses_attn_bwd: the row terms -rowsum(dO o O) and a negated
 * copy of lse, each ulysses_lse_bytes() long, then (unless the plan has
 * ULYSSES_PLAN_DETERMINISTIC) the fp32 dQ accumulator, P*Hl*Np*D*4 bytes
 * from the next 256-byte boundary. */
size_t ulysses_attn_bwd_workspace_bytes(const ulysses_plan_t* plan);

/*
 * dqkv_heads [P, 3, Np, Hl, D] = (dQ, dK, dV) for the attention step, given
 * qkv_heads T [P, C, Np, Hl, D], its output out_heads O_T [P, Np, Hl, D], the
 * output gradient dout_heads [P, Np, Hl, D] and the forward's lse.  Honors the
 * plan's segments and causal flag; pad rows get zero gradients.  fp32
 * accumulation, bf16 output.  By default one pass over the keys: dK and dV
 * accumulate in TMEM, dQ in the workspace's fp32 accumulator through L2
 * reductions (run-to-run order varies; see ULYSSES_PLAN_DETERMINISTIC for the
 * two-pass, bit-reproducible form).  Errors: ARG, ALIGN, WORKSPACE, CUDA.
 */
int ulysses_attn_bwd(const ulysses_plan_t* plan, const void* qkv_heads, const void* out_heads,
                     const void* dout_heads, const void* lse, void* dqkv_heads, void* workspace,
                     size_t workspace_bytes, float softmax_scale, void* stream);

/* Workspace of ulysses_layer_bwd: dO_T, (dQ, dK, dV) head-sharded and the row terms. */
size_t ulysses_layer_bwd_workspace_bytes(const ulysses_plan_t* plan);

/*
 * Backward of the unfused layer (softmax_scale 1/sqrt(D)): mode 0 on
 * dout_seq [Np, H, D], ulysses_attn_bwd with the forward's saved qkv_heads,
 * out_heads and lse, then mode 1 on (dQ, dK, dV) into planes 0..2 of dqkv_seq
 * (the plan's input layout; planes >= 3 are not written -- attention does not
 * use the gate).  Errors: ARG, ALIGN, WORKSPACE, CUDA.
 */
int ulysses_layer_bwd(const ulysses_plan_t* plan, const void* qkv_heads, const void* out_heads, const void* lse,
                      const void* dout_seq, void* dqkv_seq, void* workspace, size_t workspace_bytes, void* stream);

/*
 * The whole layer with softmax_scale = 1/sqrt(D):  out_seq O_S [Np, H, D]
 * from qkv_seq (sequence-sharded, plan strides).
 *   fused = 0: repack_fwd -> attn_fwd -> repack_bwd(planes = 1) through the
 *              caller's workspace (>= ulysses_workspace_bytes()).
 *   fused = 1: one attention launch whose tensor maps read qkv_seq directly
 *              and whose epilogue writes O_S; the head-sharded copies never
 *              exist.  workspace may be NULL.  Same arithmetic, same tile
 *              order: the output equals the fused = 0 output bit for bit.
 * Errors: ARG, ALIGN, WORKSPACE, CUDA.
 */
int ulysses_layer_fwd(const ulysses_plan_t* plan, const void* qkv_seq, void* out_seq, void* workspace,
                      size_t workspace_bytes, int32_t fused, void* stream);

/*
 * ulysses_layer_fwd from HOST buffers: host_qkv_seq (the plan's input
 * layout) is copied into dev_qkv_seq, the layer runs into dev_out_seq, and
 * O_S [Np, H, D] is copied back to host_out_seq.  Device buffers and the
 * workspace are the caller's; the host buffers should be pinned (pageable
 * memory works but serialises the copies with the host).
 *
 * The work is streamed by groups of heads inside each virtual rank, which is
 * exact because a head's share of the layer (mode 0 into a head slab,
 * attention, mode 1 back into that head's columns of O_S) touches no other
 * head's data: the host->device copy of group g+1's head columns overlaps
 * group g's kernels on `stream`, which overlap the device->host copy of group
 * g-1's output columns.  A group is the smallest divisor of H/P heads whose
 * attention launch still fills every SM about three times over (at most one
 * rank); the last rank's groups shrink (that size, then about half of what
 * is left each time, down to one head), so that little work remains after
 * the last input copy.  With fused = 0 the workspace holds the groups' head slabs one after
 * another (its size is ulysses_workspace_bytes() as for the device layer; its
 * layout is internal).  The copies run on two streams owned by the plan
 * (created with their events by the plan's first call of this function,
 * destroyed with the plan) and are ordered against `stream` by events: they
 * start after the work already queued on `stream`, and `stream` completes
 * only after the last output copy, so synchronising `stream` is enough before
 * reading host_out_seq.  Concurrent calls with one plan are serialised on the
 * host while they enqueue.  The result equals ulysses_layer_fwd's bit for
 * bit.  Errors: as ulysses_layer_fwd; CUDA if a stream, event or copy could
 * not be created or queued (the device buffers may then hold partial
 * results).
 */
int ulysses_layer_fwd_host(const ulysses_plan_t* plan, const void* host_qkv_seq, void* host_out_seq,
                           void* dev_qkv_seq, void* dev_out_seq, void* workspace, size_t workspace_bytes,
                           int32_t fused, void* stream);

/*
 * Synchronise `stream`, then read and clear the plan's device error word.
 * Returns 0 when no kernel reported an error, otherwise the error bits
 * (1 = a pipeline wait timed out and the kernel gave up; 2 = a work unit
 * decoded outside the problem; 4 = in the bounds-checked build
 * libulysses_debug.so only, a computed global offset fell outside its
 * buffer and the access was skipped; 8 = the one-pass attention backward
 * found its dynamic shared memory not 1024-byte aligned and did nothing), or
 * -1 if the synchronisation itself failed.
 */
int ulysses_last_device_error(const ulysses_plan_t* plan, void* stream);

/*
 * The fused layer (as ulysses_layer_fwd with fused = 1) for callers that
 * cannot allocate device memory: code running inside an allocator or memory
 * pool callback, a process whose device memory is reserved up front, or a
 * runtime that forbids cudaMalloc after start-up.  ulysses_plan() allocates a
 * device error word, so those callers cannot make a plan; this entry point
 * takes the plan's arguments directly and allocates nothing (no cudaMalloc,
 * cudaFree or allocating library call).  The pages have no counterpart: it
 * exists for this library's users only.
 *
 * The attention kernel's only scratch memory, its 4-byte device error word,
 * lives in a file-scope device array of 256 bytes that every GPU loading the
 * library holds until the process exits.  Each call clears the word on
 * `stream` before launching.  All calls share that array, so calls that
 * overlap on the GPU (other streams, other threads) race on it.  The first
 * call in each CUDA context (a device's primary context, and again after a
 * cudaDeviceReset or with another driver-API context current) looks up the
 * array's device address in that context (and may trigger the library's
 * lazy module load): make that first call before any stream capture.  A call
 * never needs more than the 4 bytes, whatever N, H or P; a scratch
 * requirement above the 256-byte maximum would be refused with
 * ULYSSES_ERR_UNSUPPORTED.
 *
 * Arguments as ulysses_plan() (planes must be >= 3) and ulysses_layer_fwd():
 * qkv_seq / out_seq are device buffers ([Np, C, H, D] by default strides,
 * [Np, H, D] out).  host_status: NULL for a fully asynchronous call, which
 * then reports no device-side errors (a timed-out wait or a bad work unit
 * leaves a wrong output that nothing reports, and the next call clears the
 * word); otherwise the call synchronises `stream` after the launch and
 * stores the kernel's error bits there (0 = none; ULYSSES_ERR_DEVICE is
 * returned when they are non-zero).  Errors: ARG, DIVISIBILITY, ALIGN,
 * UNSUPPORTED, CUDA, DEVICE.
 */
int ulysses_layer_fwd_fused_noalloc(const void* qkv_seq, void* out_seq, int64_t N, int32_t H, int32_t D,
                                    int32_t P, int32_t planes, int64_t token_stride, int64_t plane_stride,
                                    const int32_t* cu_seqlens_host, int32_t num_seqs, int32_t* host_status,
                                    void* stream);

/* Static description of a return code. */
const char* ulysses_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* ULYSSES_H_ */
