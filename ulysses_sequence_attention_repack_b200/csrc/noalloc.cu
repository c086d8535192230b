// Allocation-free entry point: the fused layer (one attention launch reading
// the sequence-sharded input, writing the sequence-sharded output) with its
// scratch memory in a file-scope device array instead of a plan.
//
// Who needs it: code that must not call cudaMalloc -- for example a caller
// running inside a custom allocator or memory-pool callback, a process whose
// device memory is fully reserved up front, or an embedding runtime that
// forbids allocation after start-up.  ulysses_plan() allocates a device error
// word, so such callers cannot create a plan; this entry point needs none.
//
// The only scratch the attention kernel uses is its 4-byte device error word
// (set when a bounded wait gives up).  Here it lives in g_noalloc_scratch,
// which every GPU that loads the library holds until the process exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "internal.h"

namespace {

constexpr size_t kScratchBytes = 256;         // stated maximum: 64 words
constexpr size_t kScratchNeededBytes = 4;     // one error word per call, any problem size
constexpr int kCacheSlots = 64;

// File-scope scratch.  Host code must not use this name as an address: in
// host code it is only a stand-in for the symbol; the device address comes
// from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned int g_noalloc_scratch[kScratchBytes / sizeof(unsigned int)];

// The array's device address is valid only in the CUDA context it was looked
// up in, so the lookups are cached per context: by the driver's context ID,
// which is never reused within a process.  A cudaDeviceReset, or a different
// driver-API context made current on the same device, gives a new ID and a
// fresh lookup instead of a stale address.
struct ScratchSlot {
  unsigned long long ctx_id;
  unsigned int* addr;
};
std::mutex g_setup_mutex;
ScratchSlot g_slots[kCacheSlots] = {};
int g_next_slot = 0;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_get_current = nullptr;
CtxGetIdFn g_get_id = nullptr;
bool g_api_looked_up = false;

// 1: *id is the current context's ID; 0: no context is current yet;
// -1: the driver offers no context IDs.  Called with g_setup_mutex held.
int current_context_id(unsigned long long* id) {
  if (!g_api_looked_up) {
    g_api_looked_up = true;
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
        qa == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
        qb == cudaDriverEntryPointSuccess) {
      g_get_current = reinterpret_cast<CtxGetCurrentFn>(a);
      g_get_id = reinterpret_cast<CtxGetIdFn>(b);
    }
    cudaGetLastError();
  }
  if (!g_get_current || !g_get_id) return -1;
  CUcontext ctx = nullptr;
  if (g_get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  return g_get_id(ctx, id) == CUDA_SUCCESS ? 1 : -1;
}

// Device address of g_noalloc_scratch in the current context, looked up once
// per context with its device current.  Without context IDs from the driver
// the address is looked up on every call (a lookup, no allocation).
int scratch_address(unsigned int** out) {
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  unsigned long long id = 0;
  int have = current_context_id(&id);
  if (have == 1) {
    for (const ScratchSlot& sl : g_slots)
      if (sl.addr && sl.ctx_id == id) {
        *out = sl.addr;
        return ULYSSES_OK;
      }
  }
  // with no context current yet, this first runtime call makes the device's
  // primary context current (and may load the library's device code)
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
    cudaGetLastError();
    return ULYSSES_ERR_CUDA;
  }
  if (have == 0) have = current_context_id(&id);
  if (have == 1) {
    g_slots[g_next_slot] = {id, static_cast<unsigned int*>(ptr)};
    g_next_slot = (g_next_slot + 1) % kCacheSlots;
  }
  *out = static_cast<unsigned int*>(ptr);
  return ULYSSES_OK;
}

}  // namespace

extern "C" int ulysses_layer_fwd_fused_noalloc(const void* qkv_seq, void* out_seq, int64_t N, int32_t H, int32_t D,
                                               int32_t P, int32_t planes, int64_t token_stride,
                                               int64_t plane_stride, const int32_t* cu_seqlens_host,
                                               int32_t num_seqs, int32_t* host_status, void* stream) {
  if (kScratchNeededBytes > kScratchBytes) return ULYSSES_ERR_UNSUPPORTED;
  if (!qkv_seq || !out_seq) return ULYSSES_ERR_ARG;
  if (D != 128) return ULYSSES_ERR_UNSUPPORTED;
  if (N < 1 || H < 1 || P < 1 || planes < 3 || planes > 8) return ULYSSES_ERR_ARG;
  if (H > 1024) return ULYSSES_ERR_UNSUPPORTED;
  if (P > H || H % P != 0) return ULYSSES_ERR_DIVISIBILITY;
  const int64_t Nl = (N + P - 1) / P;
  const int64_t Np = Nl * P;
  if (Np > (int64_t(1) << 31) - 4096) return ULYSSES_ERR_UNSUPPORTED;
  const int64_t row = static_cast<int64_t>(H) * D;
  if (token_stride == 0 && plane_stride == 0) {
    token_stride = planes * row;
    plane_stride = row;
  }
  if (token_stride <= 0 || plane_stride <= 0) return ULYSSES_ERR_ARG;
  if (token_stride % 8 || plane_stride % 8) return ULYSSES_ERR_ALIGN;
  const bool token_major = plane_stride >= row && token_stride >= (planes - 1) * plane_stride + row;
  const bool plane_major = token_stride >= row && plane_stride >= (Np - 1) * token_stride + row;
  if (!token_major && !plane_major) return ULYSSES_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(qkv_seq) & 15u) || (reinterpret_cast<uintptr_t>(out_seq) & 15u))
    return ULYSSES_ERR_ALIGN;
  const int64_t in_bytes = ((Np - 1) * token_stride + (planes - 1) * plane_stride + row) * 2;
  const int64_t out_bytes = Np * row * 2;
  const uintptr_t a = reinterpret_cast<uintptr_t>(qkv_seq), b = reinterpret_cast<uintptr_t>(out_seq);
  if (a < b + static_cast<uintptr_t>(out_bytes) && b < a + static_cast<uintptr_t>(in_bytes)) return ULYSSES_ERR_ARG;

  // host-side description of the call (a stack object: nothing is allocated)
  ulysses_plan_t plan;
  std::memset(&plan, 0, sizeof(plan));
  plan.N = N;
  plan.Np = Np;
  plan.Nl = Nl;
  plan.H = H;
  plan.D = D;
  plan.P = P;
  plan.Hl = H / P;
  plan.C = planes;
  plan.token_stride = token_stride;
  plan.plane_stride = plane_stride;
  plan.plane_chunk = 1;
  if (cu_seqlens_host == nullptr || num_seqs == 0) {
    if (cu_seqlens_host == nullptr && num_seqs != 0) return ULYSSES_ERR_ARG;
    plan.segs[0] = {0, static_cast<int32_t>(N)};
    plan.num_seqs = 1;
  } else {
    if (num_seqs < 0) return ULYSSES_ERR_ARG;
    if (num_seqs > ULYSSES_MAX_SEQS) return ULYSSES_ERR_UNSUPPORTED;
    if (cu_seqlens_host[0] != 0 || cu_seqlens_host[num_seqs] != N) return ULYSSES_ERR_ARG;
    for (int32_t s = 0; s < num_seqs; ++s) {
      if (cu_seqlens_host[s + 1] < cu_seqlens_host[s]) return ULYSSES_ERR_ARG;
      plan.segs[s] = {cu_seqlens_host[s], cu_seqlens_host[s + 1]};
    }
    plan.num_seqs = num_seqs;
  }

  unsigned int* scratch = nullptr;
  int st = scratch_address(&scratch);
  if (st != ULYSSES_OK) return st;
  plan.dev_err = scratch;   // word 0: the kernel's error word
  cudaGetDevice(&plan.device);

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the error word must start at zero; the array keeps the last call's contents
  if (cudaMemsetAsync(scratch, 0, kScratchNeededBytes, s) != cudaSuccess) {
    cudaGetLastError();
    return ULYSSES_ERR_CUDA;
  }
  ulysses::AttnLaunch l;
  l.base = qkv_seq;
  l.fused = 1;
  l.Np = Np;
  l.N = N;
  l.H = H;
  l.P = P;
  l.Hl = H / P;
  l.C = planes;
  l.tok_stride = token_stride;
  l.plane_stride = plane_stride;
  l.out = out_seq;
  l.o_stride_r = static_cast<int64_t>(plan.Hl) * D;
  l.o_stride_n = row;
  l.o_stride_j = D;
  l.scale = 1.0f / std::sqrt(static_cast<float>(D));
  l.plan = &plan;
  if (ulysses::launch_attn(l, s) != cudaSuccess) {
    cudaGetLastError();
    return ULYSSES_ERR_CUDA;
  }
  if (host_status) {
    unsigned int v = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess ||
        cudaMemcpy(&v, scratch, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) {
      cudaGetLastError();
      return ULYSSES_ERR_CUDA;
    }
    *host_status = static_cast<int32_t>(v);
    if (v != 0) return ULYSSES_ERR_DEVICE;
  }
  return ULYSSES_OK;
}
