// Host-side declarations shared by the C ABI (api.cpp) and the kernel files.
#pragma once

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>
#include <mutex>

#include "../../include/ulysses.h"

namespace ulysses {

struct Segment {
  int32_t start, end;   // key / query range [start, end) of one packed sequence
};

struct HostPipe;   // copy streams and events of the host-buffer layer (api.cpp)

// One-time setup per device (kernel attributes), safe to call from several
// host threads at once.  run(dev, f) calls f() until it has succeeded once
// for dev; devices past kMaxDevices run f() on every call.
class PerDeviceOnce {
 public:
  template <class F>
  cudaError_t run(int dev, F&& f) {
    const bool tracked = dev >= 0 && dev < kMaxDevices;
    if (tracked && done_[dev].load(std::memory_order_acquire)) return cudaSuccess;
    std::lock_guard<std::mutex> lock(mu_);
    if (tracked && done_[dev].load(std::memory_order_relaxed)) return cudaSuccess;
    const cudaError_t e = f();
    if (e == cudaSuccess && tracked) done_[dev].store(true, std::memory_order_release);
    return e;
  }

 private:
  static constexpr int kMaxDevices = 256;
  std::mutex mu_;
  std::atomic<bool> done_[kMaxDevices] = {};
};

}  // namespace ulysses

struct ulysses_plan_s {
  int64_t N, Np, Nl;
  int32_t H, D, P, Hl, C;
  int64_t token_stride, plane_stride;   // elements, sequence-sharded input
  int32_t plane_chunk;
  int32_t num_seqs;
  int32_t causal;                       // attention sees keys m <= n only
  int32_t pair_cta;                     // bf16 attention on CTA pairs (clusters of two) instead of one CTA per SM
  int32_t deterministic;                // backward in two passes without atomics (bit-reproducible)
  ulysses::Segment segs[ULYSSES_MAX_SEQS];
  int32_t device;                       // device the plan's scratch lives on (-1: none)
  unsigned int* dev_err;                // device error word (16 bytes allocated)
  ulysses::HostPipe* pipe;              // created by the first ulysses_layer_fwd_host call
};

namespace ulysses {

// One repack launch over planes [c0, c0 + cc).
//   dir = 0: seq -> heads (mode 0), dir = 1: heads -> seq (mode 1).
//   seq side: element (n, c, h, d) at n*tok_stride + c*plane_stride + h*D + d
//   head side: [P, Ctot, Np, Hl, D]
// err: device error word for the bounds-checked build (bounds.cuh); may be null.
cudaError_t launch_repack(int dir, const void* src, void* dst, int64_t Np, int32_t H, int32_t P, int32_t Ctot,
                          int32_t c0, int32_t cc, int64_t tok_stride, int64_t plane_stride, cudaStream_t stream,
                          unsigned int* err = nullptr);

// Mode 0 with the E4M3 cast (FP8 attention variant) over planes [c0, c0 + cc):
// head side [P, Ctot, Np, Hl, D] of one-byte codes.
cudaError_t launch_repack_fp8(const void* src, void* dst, int64_t Np, int32_t H, int32_t P, int32_t Ctot,
                              int32_t c0, int32_t cc, int64_t tok_stride, int64_t plane_stride,
                              cudaStream_t stream, unsigned int* err = nullptr);

// Prologue (per-head RMSNorm + partial RoPE on planes 0 and 1) fused with one
// mode-0 repack launch over planes [c0, c0 + cc).
cudaError_t launch_prologue_repack(const void* src, void* dst, const void* wq, const void* wk, const void* cos,
                                   const void* sin, int32_t rd, float eps, int64_t Np, int32_t H, int32_t P,
                                   int32_t Ctot, int32_t c0, int32_t cc, int64_t tok_stride, int64_t plane_stride,
                                   cudaStream_t stream, unsigned int* err = nullptr);

// Destination table of the multi-GPU push (a kernel parameter): entry r is
// rank r's buffer (a peer mapping, or a local buffer when ranks are emulated).
struct PushTable {
  void* p[ULYSSES_MAX_PUSH_RANKS];
};

// One push launch over planes [c0, c0 + cc) by rank `rank` (transport.cu).
//   dir = 0: shard [Nl, C, H, D] -> dst.p[r] = T_r [C, Np, Hl, D], rows rank*Nl + i
//   dir = 1: head rows [C, Np, Hl, D] -> dst.p[q] = [Nl, C, H, D], heads rank*Hl + j
cudaError_t launch_push(int dir, const void* src, const PushTable& dst, int64_t Nl, int64_t Np, int32_t H,
                        int32_t P, int32_t C, int32_t c0, int32_t cc, int32_t rank, cudaStream_t stream,
                        unsigned int* err = nullptr);

// Attention launch description (filled by api.cpp).
struct AttnLaunch {
  const void* base;        // Q/K/V source buffer
  int fused;               // 0: head-sharded T; 1: sequence-sharded S (plan strides)
  int64_t Np, N;
  int32_t H, P, Hl, C;
  int64_t tok_stride, plane_stride;     // for fused = 1
  void* out;
  int64_t o_stride_r, o_stride_n, o_stride_j;   // elements
  float scale;
  const ulysses_plan_t* plan;
  float* lse = nullptr;          // optional log2-domain LSE output [P*Hl][lse_stride]
  int64_t lse_stride = 0;
  int fp8 = 0;                   // 1: base holds E4M3 codes [P, C, Np, Hl, D] (fused must be 0)
  // multi-GPU push epilogue: when push_rows > 0, output row n goes to
  // push->p[n / push_rows] + (n % push_rows) * o_stride_n + j * o_stride_j
  const PushTable* push = nullptr;
  int64_t push_rows = 0;
  int32_t push_ranks = 0;        // entries of push in use (push_rows * push_ranks >= Np)
};

cudaError_t launch_attn(const AttnLaunch& a, cudaStream_t stream);

// Row stride (floats) of the LSE / D buffers of one (rank, local head): Np
// rounded up to 4 plus 144, so the 132-float bulk copy the backward makes for
// any 128-row block starting below Np (from the block start rounded down to
// a multiple of 4, keeping the copy 16-byte aligned) stays inside the buffer.
inline int64_t lse_row_stride(int64_t Np) { return (Np + 3) / 4 * 4 + 144; }

// Attention backward launch description (filled by api.cpp).
struct AttnBwdLaunch {
  const void* qkv;      // head-sharded T [P, C, Np, Hl, D]
  const void* out;      // O_T [P, Np, Hl, D]
  const void* dout;     // dO_T [P, Np, Hl, D]
  const float* lse;     // [P*Hl][lse_stride] from the forward
  float* delta;         // workspace: -rowsum(dO o O), then -lse, each [P*Hl][lse_stride]
  float* dq_acc;        // one-pass backward: fp32 [P*Hl][Np][D] dQ accumulator (workspace); null = two passes
  void* dqkv;           // [P, 3, Np, Hl, D]
  float scale;
  const ulysses_plan_t* plan;
};

cudaError_t launch_attn_bwd(const AttnBwdLaunch& a, cudaStream_t stream);

}  // namespace ulysses
