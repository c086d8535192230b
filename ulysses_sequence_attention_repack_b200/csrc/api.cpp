// C ABI of the one-GPU Ulysses layer: plan validation, buffer checks and the
// launch sequence of the three steps.  Declarations and argument contracts
// are in include/ulysses.h.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>

#include "internal.h"

namespace {

// NVTX ranges (domain "ulysses") around every launching entry point and
// around the three steps inside the layer calls, so a timeline profiler
// shows repack -> attention -> inverse repack.  Without a profiler attached
// a range costs one function-pointer check.
nvtxDomainHandle_t nvtx_domain() {
  static const nvtxDomainHandle_t d = nvtxDomainCreateA("ulysses");
  return d;
}

class NvtxRange {
 public:
  explicit NvtxRange(const char* name) {
    nvtxEventAttributes_t a;
    std::memset(&a, 0, sizeof(a));
    a.version = NVTX_VERSION;
    a.size = NVTX_EVENT_ATTRIB_STRUCT_SIZE;
    a.messageType = NVTX_MESSAGE_TYPE_ASCII;
    a.message.ascii = name;
    nvtxDomainRangePushEx(nvtx_domain(), &a);
  }
  ~NvtxRange() { nvtxDomainRangePop(nvtx_domain()); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

constexpr int32_t kHeadDim = 128;
constexpr int32_t kMaxHeads = 1024;
constexpr int32_t kMaxPlanes = 8;
constexpr int64_t kMaxRows = (int64_t(1) << 31) - 4096;   // kernels index rows with int32

inline int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool overlap(const void* a, int64_t abytes, const void* b, int64_t bbytes) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + static_cast<uintptr_t>(bbytes) && y < x + static_cast<uintptr_t>(abytes);
}

// bytes spanned by the sequence-sharded buffer with the given strides
inline int64_t seq_extent_bytes(const ulysses_plan_t* p, int32_t planes, int64_t tok, int64_t pl) {
  return ((p->Np - 1) * tok + static_cast<int64_t>(planes - 1) * pl + static_cast<int64_t>(p->H) * p->D) * 2;
}
inline int64_t heads_bytes(const ulysses_plan_t* p, int32_t planes) {
  return static_cast<int64_t>(p->P) * planes * p->Np * p->Hl * p->D * 2;
}
inline int64_t out_seq_bytes(const ulysses_plan_t* p) { return p->Np * p->H * p->D * 2; }
inline int64_t heads_bytes_fp8(const ulysses_plan_t* p, int32_t planes) { return heads_bytes(p, planes) / 2; }

// Launch-time device check: the plan's error word lives on one device.
int device_ready(const ulysses_plan_t* p) {
  if (!p || !p->dev_err) return ULYSSES_ERR_CUDA;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return ULYSSES_ERR_CUDA;
  }
  return dev == p->device ? ULYSSES_OK : ULYSSES_ERR_ARG;
}

int status_of(cudaError_t e) {
  if (e == cudaSuccess) return ULYSSES_OK;
  cudaGetLastError();
  return ULYSSES_ERR_CUDA;
}

int repack_fwd_impl(const ulysses_plan_t* p, const void* src, void* dst, cudaStream_t st) {
  for (int32_t c0 = 0; c0 < p->C; c0 += p->plane_chunk) {
    const int32_t cc = std::min(p->plane_chunk, p->C - c0);
    int s = status_of(ulysses::launch_repack(0, src, dst, p->Np, p->H, p->P, p->C, c0, cc, p->token_stride,
                                             p->plane_stride, st, p->dev_err));
    if (s != ULYSSES_OK) return s;
  }
  return ULYSSES_OK;
}

// dst layout for mode 1 with `planes` planes (see ulysses_repack_bwd)
void bwd_dst_strides(const ulysses_plan_t* p, int32_t planes, int64_t* tok, int64_t* pl) {
  if (planes == p->C) {
    *tok = p->token_stride;
    *pl = p->plane_stride;
  } else {
    *tok = static_cast<int64_t>(planes) * p->H * p->D;
    *pl = static_cast<int64_t>(p->H) * p->D;
  }
}

int repack_bwd_impl(const ulysses_plan_t* p, const void* src, void* dst, int32_t planes, cudaStream_t st) {
  int64_t tok, pl;
  bwd_dst_strides(p, planes, &tok, &pl);
  // same window rule as the forward direction: at most plane_chunk planes per launch
  for (int32_t c0 = 0; c0 < planes; c0 += p->plane_chunk) {
    const int32_t cc = std::min(p->plane_chunk, planes - c0);
    int s = status_of(
        ulysses::launch_repack(1, src, dst, p->Np, p->H, p->P, planes, c0, cc, tok, pl, st, p->dev_err));
    if (s != ULYSSES_OK) return s;
  }
  return ULYSSES_OK;
}

inline int64_t lse_bytes(const ulysses_plan_t* p) {
  return static_cast<int64_t>(p->P) * p->Hl * ulysses::lse_row_stride(p->Np) * 4;
}

int attn_impl(const ulysses_plan_t* p, const void* base, int fused, void* out, float scale, cudaStream_t st,
              float* lse = nullptr, int fp8 = 0) {
  ulysses::AttnLaunch a;
  a.base = base;
  a.fused = fused;
  a.Np = p->Np;
  a.N = p->N;
  a.H = p->H;
  a.P = p->P;
  a.Hl = p->Hl;
  a.C = p->C;
  a.tok_stride = p->token_stride;
  a.plane_stride = p->plane_stride;
  a.out = out;
  if (fused) {   // O_S [Np, H, D], head h = r*Hl + j
    a.o_stride_r = static_cast<int64_t>(p->Hl) * p->D;
    a.o_stride_n = static_cast<int64_t>(p->H) * p->D;
  } else {       // O_T [P, Np, Hl, D]
    a.o_stride_r = p->Np * p->Hl * p->D;
    a.o_stride_n = static_cast<int64_t>(p->Hl) * p->D;
  }
  a.o_stride_j = p->D;
  a.scale = scale;
  a.plan = p;
  a.lse = lse;
  a.lse_stride = ulysses::lse_row_stride(p->Np);
  a.fp8 = fp8;
  return status_of(ulysses::launch_attn(a, st));
}

int repack_fwd_fp8_impl(const ulysses_plan_t* p, const void* src, void* dst, cudaStream_t st) {
  for (int32_t c0 = 0; c0 < p->C; c0 += p->plane_chunk) {
    const int32_t cc = std::min(p->plane_chunk, p->C - c0);
    int s = status_of(ulysses::launch_repack_fp8(src, dst, p->Np, p->H, p->P, p->C, c0, cc, p->token_stride,
                                                 p->plane_stride, st, p->dev_err));
    if (s != ULYSSES_OK) return s;
  }
  return ULYSSES_OK;
}

// ---------------------------------------------------------------- host-buffer layer, pipelined by head group
//
// Virtual rank r owns heads [r*Hl, (r+1)*Hl) after the all-to-all, and each
// head's share of the layer (mode 0 into a head slab, attention on it, mode 1
// back into that head's columns of O_S) reads and writes nothing of the other
// heads.  The host path therefore streams the layer by groups of heads inside
// each rank: the copy of group g+1's head columns to the device overlaps
// group g's kernels, which overlap the copy of group g-1's output columns
// back to the host.

}  // namespace

namespace ulysses {

// Two copy streams (host->device, device->host) and the events that order
// them against the caller's stream: start, one input and one output event per
// head group, done.  Owned by the plan, created by its first host-buffer call.
struct HostPipe {
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t* in = nullptr;
  cudaEvent_t* out = nullptr;
  int32_t n = 0;            // head groups (events per array)
  int32_t* h0 = nullptr;    // first head of each group
  int32_t* hg = nullptr;    // heads of each group (a group never spans two ranks)
};

}  // namespace ulysses

namespace {

std::mutex g_pipe_mutex;   // guards pipe creation and the enqueue of one host-buffer call

void destroy_pipe(ulysses::HostPipe* h) {
  if (!h) return;
  if (h->h2d) cudaStreamDestroy(h->h2d);
  if (h->d2h) cudaStreamDestroy(h->d2h);
  if (h->start) cudaEventDestroy(h->start);
  if (h->done) cudaEventDestroy(h->done);
  for (int32_t i = 0; i < h->n; ++i) {
    if (h->in && h->in[i]) cudaEventDestroy(h->in[i]);
    if (h->out && h->out[i]) cudaEventDestroy(h->out[i]);
  }
  delete[] h->in;
  delete[] h->out;
  delete[] h->h0;
  delete[] h->hg;
  delete h;
  cudaGetLastError();
}

// Heads per group: the smallest divisor of Hl whose attention launch still
// fills every SM about three times over (256-row work units per head, as the
// attention kernel tiles them), so the groups stay efficient while the
// pipeline's fill (one group's copy in) stays short.
int32_t host_group_heads(const ulysses_plan_t* p, int sms) {
  int64_t units_per_head = 0;
  for (int32_t s = 0; s < p->num_seqs; ++s) {
    const int64_t q_end = (p->segs[s].end == p->N) ? p->Np : p->segs[s].end;
    if (p->segs[s].end > p->segs[s].start) units_per_head += (q_end - p->segs[s].start + 255) / 256;
  }
  for (int32_t d = 1; d < p->Hl; ++d)
    if (p->Hl % d == 0 && d * units_per_head >= 3 * static_cast<int64_t>(sms)) return d;
  return p->Hl;
}

// The plan's pipe, created on first use (call with g_pipe_mutex held, on the plan's device).
ulysses::HostPipe* plan_pipe(const ulysses_plan_t* p) {
  if (p->pipe) return p->pipe;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  ulysses::HostPipe* h = new (std::nothrow) ulysses::HostPipe;
  if (!h) return nullptr;
  // Groups of hg heads, except that the last rank tapers (hg, then about
  // half of what is left each time, down to one head): after the last input
  // copy only the last, smallest group's kernels and output copy remain, the
  // pipeline's drain.  A smaller group fills fewer SMs, but the kernels are
  // waiting for the copies there anyway.
  const int32_t hg = host_group_heads(p, sms);
  int32_t groups = (p->P - 1) * (p->Hl / hg);
  for (int32_t left = p->Hl; left > 0; ++groups) left -= std::min(hg, left > 1 ? (left + 1) / 2 : 1);
  h->in = new (std::nothrow) cudaEvent_t[groups]();
  h->out = new (std::nothrow) cudaEvent_t[groups]();
  h->h0 = new (std::nothrow) int32_t[groups];
  h->hg = new (std::nothrow) int32_t[groups];
  bool ok = h->in && h->out && h->h0 && h->hg;
  if (ok) {
    h->n = groups;
    int32_t g = 0, head = 0;
    for (int32_t r = 0; r + 1 < p->P; ++r)
      for (int32_t k = 0; k < p->Hl / hg; ++k, ++g, head += hg) {
        h->h0[g] = head;
        h->hg[g] = hg;
      }
    for (int32_t left = p->Hl; left > 0; ++g) {
      const int32_t size = std::min(hg, left > 1 ? (left + 1) / 2 : 1);
      h->h0[g] = head;
      h->hg[g] = size;
      head += size;
      left -= size;
    }
  }
  ok = ok && cudaStreamCreateWithFlags(&h->h2d, cudaStreamNonBlocking) == cudaSuccess;
  ok = ok && cudaStreamCreateWithFlags(&h->d2h, cudaStreamNonBlocking) == cudaSuccess;
  ok = ok && cudaEventCreateWithFlags(&h->start, cudaEventDisableTiming) == cudaSuccess;
  ok = ok && cudaEventCreateWithFlags(&h->done, cudaEventDisableTiming) == cudaSuccess;
  for (int32_t i = 0; ok && i < groups; ++i) {
    ok = cudaEventCreateWithFlags(&h->in[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&h->out[i], cudaEventDisableTiming) == cudaSuccess;
  }
  if (!ok) {
    destroy_pipe(h);
    return nullptr;
  }
  const_cast<ulysses_plan_t*>(p)->pipe = h;   // a cache: the plan's geometry stays immutable
  return h;
}

// Copy the columns of heads [h0, h0 + hg) of the sequence-sharded input
// (every token and plane) from host to device; both sides use the plan's strides.
cudaError_t copy_heads_in(const ulysses_plan_t* p, int32_t h0, int32_t hg, const uint8_t* host, uint8_t* dev,
                          cudaStream_t s) {
  const size_t width = static_cast<size_t>(hg) * p->D * 2;
  const size_t off = static_cast<size_t>(h0) * p->D * 2;
  const size_t tok = static_cast<size_t>(p->token_stride) * 2, pl = static_cast<size_t>(p->plane_stride) * 2;
  if (p->C == 1 || p->token_stride == static_cast<int64_t>(p->C) * p->plane_stride)   // rows (n, c) at pitch pl
    return cudaMemcpy2DAsync(dev + off, pl, host + off, pl, width, static_cast<size_t>(p->Np) * p->C,
                             cudaMemcpyHostToDevice, s);
  if (p->plane_stride == p->Np * p->token_stride)   // rows (c, n) at pitch tok
    return cudaMemcpy2DAsync(dev + off, tok, host + off, tok, width, static_cast<size_t>(p->Np) * p->C,
                             cudaMemcpyHostToDevice, s);
  for (int32_t c = 0; c < p->C; ++c) {
    const size_t o = off + static_cast<size_t>(c) * pl;
    cudaError_t e = cudaMemcpy2DAsync(dev + o, tok, host + o, tok, width, static_cast<size_t>(p->Np),
                                      cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// The layer for heads [h0, h0 + hg) (inside one rank) on `st`: their columns
// of S in, their columns of O_S out.  The kernels see the group as a one-rank
// problem (P = 1, H = hg) at offset pointers; with fused = 0 its head slab and
// attention output live in the caller's workspace at Tg / OTg.
// mode: 0 = unfused bf16, 1 = fused bf16, 2 = unfused with the E4M3 cast
// (Tg then holds one byte per element)
int group_layer_impl(const ulysses_plan_t* p, int32_t h0, int32_t hg, const uint8_t* S, uint8_t* OS, uint8_t* Tg,
                     uint8_t* OTg, int32_t mode, float scale, cudaStream_t st) {
  const int32_t fused = mode == 1;
  const int32_t fp8 = mode == 2;
  const int64_t cols = static_cast<int64_t>(hg) * p->D;   // elements of the group's heads in a row
  const int64_t row = static_cast<int64_t>(p->H) * p->D;
  const uint8_t* Sg = S + static_cast<int64_t>(h0) * p->D * 2;
  uint8_t* OSg = OS + static_cast<int64_t>(h0) * p->D * 2;
  ulysses::AttnLaunch a;
  a.fused = fused;
  a.Np = p->Np;
  a.N = p->N;
  a.H = hg;
  a.P = 1;
  a.Hl = hg;
  a.C = p->C;
  a.tok_stride = p->token_stride;
  a.plane_stride = p->plane_stride;
  a.o_stride_j = p->D;
  a.scale = scale;
  a.plan = p;
  if (fused) {
    a.base = Sg;
    a.out = OSg;
    a.o_stride_r = cols;
    a.o_stride_n = row;
    return status_of(ulysses::launch_attn(a, st));
  }
  for (int32_t c0 = 0; c0 < p->C; c0 += p->plane_chunk) {
    const int32_t cc = std::min(p->plane_chunk, p->C - c0);
    int s = status_of(fp8 ? ulysses::launch_repack_fp8(Sg, Tg, p->Np, hg, 1, p->C, c0, cc, p->token_stride,
                                                       p->plane_stride, st, p->dev_err)
                          : ulysses::launch_repack(0, Sg, Tg, p->Np, hg, 1, p->C, c0, cc, p->token_stride,
                                                   p->plane_stride, st, p->dev_err));
    if (s != ULYSSES_OK) return s;
  }
  a.fp8 = fp8;
  a.base = Tg;
  a.out = OTg;
  a.o_stride_r = p->Np * cols;
  a.o_stride_n = cols;
  int s = status_of(ulysses::launch_attn(a, st));
  if (s != ULYSSES_OK) return s;
  return status_of(
      ulysses::launch_repack(1, OTg, OSg, p->Np, hg, 1, 1, 0, 1, row, row, st, p->dev_err));
}

// Multi-GPU push: the plan must describe the default token-interleaved
// layout, which is also the layout of every rank's shard.
bool push_layout_ok(const ulysses_plan_t* p) {
  return p->P <= ULYSSES_MAX_PUSH_RANKS && p->token_stride == static_cast<int64_t>(p->C) * p->H * p->D &&
         p->plane_stride == static_cast<int64_t>(p->H) * p->D;
}

// Copies the caller's P destination pointers into a kernel table.  Each must
// be non-null and 16-byte aligned, and none may overlap the source range or
// another destination.
int push_table(const ulysses_plan_t* p, void* const* ptrs, int64_t dst_bytes, const void* src, int64_t src_bytes,
               ulysses::PushTable* t) {
  if (!ptrs) return ULYSSES_ERR_ARG;
  std::memset(t, 0, sizeof(*t));
  for (int32_t r = 0; r < p->P; ++r) {
    if (!ptrs[r]) return ULYSSES_ERR_ARG;
    if (!aligned16(ptrs[r])) return ULYSSES_ERR_ALIGN;
    if (overlap(src, src_bytes, ptrs[r], dst_bytes)) return ULYSSES_ERR_ARG;
    for (int32_t q = 0; q < r; ++q)
      if (overlap(ptrs[q], dst_bytes, ptrs[r], dst_bytes)) return ULYSSES_ERR_ARG;
    t->p[r] = ptrs[r];
  }
  return ULYSSES_OK;
}

// One rank's view of a plan: the same sequence geometry (N, Np, segments,
// causal flag, device error word) over that rank's Hl heads, as a one-rank
// problem whose head-sharded buffers are the rank's slabs.
ulysses_plan_t slab_view(const ulysses_plan_t* p) {
  ulysses_plan_t v = *p;
  v.P = 1;
  v.H = p->Hl;
  v.Nl = p->Np;
  v.pipe = nullptr;
  return v;
}

}  // namespace

extern "C" {

int ulysses_plan(ulysses_plan_t** out, int64_t N, int32_t H, int32_t D, int32_t P, int32_t planes,
                 int64_t token_stride, int64_t plane_stride, int64_t plane_chunk, const int32_t* cu_seqlens_host,
                 int32_t num_seqs) {
  return ulysses_plan_ex(out, N, H, D, P, planes, token_stride, plane_stride, plane_chunk, cu_seqlens_host, num_seqs,
                         0u);
}

int ulysses_plan_ex(ulysses_plan_t** out, int64_t N, int32_t H, int32_t D, int32_t P, int32_t planes,
                    int64_t token_stride, int64_t plane_stride, int64_t plane_chunk, const int32_t* cu_seqlens_host,
                    int32_t num_seqs, uint32_t flags) {
  if (!out) return ULYSSES_ERR_ARG;
  *out = nullptr;
  if (flags & ~(ULYSSES_PLAN_CAUSAL | ULYSSES_PLAN_PAIR_ATTENTION | ULYSSES_PLAN_DETERMINISTIC))
    return ULYSSES_ERR_ARG;
  if (D != kHeadDim) return ULYSSES_ERR_UNSUPPORTED;
  if (N < 1 || H < 1 || P < 1 || planes < 1 || planes > kMaxPlanes) return ULYSSES_ERR_ARG;
  if (H > kMaxHeads) return ULYSSES_ERR_UNSUPPORTED;
  if (P > H || H % P != 0) return ULYSSES_ERR_DIVISIBILITY;
  const int64_t Nl = (N + P - 1) / P;
  const int64_t Np = Nl * P;
  if (Np > kMaxRows) return ULYSSES_ERR_UNSUPPORTED;

  // strides of the sequence-sharded input (elements)
  const int64_t row = static_cast<int64_t>(H) * D;
  if (token_stride == 0 && plane_stride == 0) {
    token_stride = planes * row;
    plane_stride = row;
  }
  if (token_stride <= 0 || plane_stride <= 0) return ULYSSES_ERR_ARG;
  if (token_stride % 8 || plane_stride % 8) return ULYSSES_ERR_ALIGN;
  const bool token_major = plane_stride >= row && token_stride >= (planes - 1) * plane_stride + row;
  const bool plane_major = token_stride >= row && plane_stride >= (Np - 1) * token_stride + row;
  if (!token_major && !plane_major && planes > 1) return ULYSSES_ERR_ARG;   // rows would overlap
  if (planes == 1 && token_stride < row) return ULYSSES_ERR_ARG;

  // window: bytes per rank per plane, and planes per launch
  const int64_t per_plane = Nl * row * 2;
  if (per_plane > ULYSSES_MAX_WINDOW_BYTES) return ULYSSES_ERR_WINDOW;
  int64_t chunk = plane_chunk;
  if (chunk == 0) chunk = std::min<int64_t>(planes, ULYSSES_MAX_WINDOW_BYTES / per_plane);
  if (chunk < 1 || chunk > planes) return ULYSSES_ERR_ARG;
  if (chunk * per_plane > ULYSSES_MAX_WINDOW_BYTES) return ULYSSES_ERR_WINDOW;

  // packed sequences
  ulysses::Segment segs[ULYSSES_MAX_SEQS];
  int32_t nseq = 0;
  if (cu_seqlens_host == nullptr || num_seqs == 0) {
    if (cu_seqlens_host == nullptr && num_seqs != 0) return ULYSSES_ERR_ARG;
    segs[0] = {0, static_cast<int32_t>(N)};
    nseq = 1;
  } else {
    if (num_seqs < 0) return ULYSSES_ERR_ARG;
    if (num_seqs > ULYSSES_MAX_SEQS) return ULYSSES_ERR_UNSUPPORTED;
    if (cu_seqlens_host[0] != 0 || cu_seqlens_host[num_seqs] != N) return ULYSSES_ERR_ARG;
    for (int32_t s = 0; s < num_seqs; ++s) {
      if (cu_seqlens_host[s + 1] < cu_seqlens_host[s]) return ULYSSES_ERR_ARG;
      segs[s] = {cu_seqlens_host[s], cu_seqlens_host[s + 1]};
    }
    nseq = num_seqs;
  }

  ulysses_plan_t* p = new (std::nothrow) ulysses_plan_t;
  if (!p) return ULYSSES_ERR_ARG;
  std::memset(p, 0, sizeof(*p));
  p->N = N;
  p->Np = Np;
  p->Nl = Nl;
  p->H = H;
  p->D = D;
  p->P = P;
  p->Hl = H / P;
  p->C = planes;
  p->token_stride = token_stride;
  p->plane_stride = plane_stride;
  p->plane_chunk = static_cast<int32_t>(chunk);
  p->num_seqs = nseq;
  p->causal = (flags & ULYSSES_PLAN_CAUSAL) ? 1 : 0;
  p->pair_cta = (flags & ULYSSES_PLAN_PAIR_ATTENTION) ? 1 : 0;
  p->deterministic = (flags & ULYSSES_PLAN_DETERMINISTIC) ? 1 : 0;
  std::memcpy(p->segs, segs, sizeof(ulysses::Segment) * nseq);
  p->device = -1;
  p->dev_err = nullptr;
  p->pipe = nullptr;

  // device error word (16 bytes) on the current device; absent without a GPU
  int dev = -1;
  if (cudaGetDevice(&dev) == cudaSuccess) {
    void* e = nullptr;
    if (cudaMalloc(&e, 16) == cudaSuccess) {
      if (cudaMemset(e, 0, 16) == cudaSuccess) {
        p->dev_err = static_cast<unsigned int*>(e);
        p->device = dev;
      } else {
        cudaFree(e);
      }
    }
  }
  cudaGetLastError();   // a missing device is not an error of plan creation
  *out = p;
  return ULYSSES_OK;
}

void ulysses_plan_destroy(ulysses_plan_t* plan) {
  if (!plan) return;
  if (plan->dev_err) {
    int cur = -1;
    cudaGetDevice(&cur);
    if (cur != plan->device) cudaSetDevice(plan->device);
    destroy_pipe(plan->pipe);
    cudaFree(plan->dev_err);
    if (cur >= 0 && cur != plan->device) cudaSetDevice(cur);
    cudaGetLastError();
  }
  delete plan;
}

int64_t ulysses_plan_padded_tokens(const ulysses_plan_t* plan) { return plan ? plan->Np : -1; }

int32_t ulysses_plan_plane_chunk(const ulysses_plan_t* plan) { return plan ? plan->plane_chunk : -1; }

int64_t ulysses_plan_window_bytes_per_plane(const ulysses_plan_t* plan) {
  return plan ? plan->Nl * plan->H * plan->D * 2 : -1;
}

size_t ulysses_workspace_bytes(const ulysses_plan_t* plan) {
  if (!plan) return 0;
  return static_cast<size_t>(align_up(heads_bytes(plan, plan->C), 256) + align_up(heads_bytes(plan, 1), 256));
}

int ulysses_repack_fwd(const ulysses_plan_t* plan, const void* src_seq, void* dst_heads, void* stream) {
  NvtxRange range("ulysses_repack_fwd");
  if (!plan || !src_seq || !dst_heads) return ULYSSES_ERR_ARG;
  if (!aligned16(src_seq) || !aligned16(dst_heads)) return ULYSSES_ERR_ALIGN;
  if (overlap(src_seq, seq_extent_bytes(plan, plan->C, plan->token_stride, plan->plane_stride), dst_heads,
              heads_bytes(plan, plan->C)))
    return ULYSSES_ERR_ARG;
  int s = device_ready(plan);
  if (s != ULYSSES_OK) return s;
  return repack_fwd_impl(plan, src_seq, dst_heads, static_cast<cudaStream_t>(stream));
}

int ulysses_repack_bwd(const ulysses_plan_t* plan, const void* src_heads, void* dst_seq, int32_t planes,
                       void* stream) {
  NvtxRange range("ulysses_repack_bwd");
  if (!plan || !src_heads || !dst_seq) return ULYSSES_ERR_ARG;
  if (planes < 1 || planes > plan->C) return ULYSSES_ERR_ARG;
  if (!aligned16(src_heads) || !aligned16(dst_seq)) return ULYSSES_ERR_ALIGN;
  int64_t tok, pl;
  bwd_dst_strides(plan, planes, &tok, &pl);
  if (overlap(src_heads, heads_bytes(plan, planes), dst_seq, seq_extent_bytes(plan, planes, tok, pl)))
    return ULYSSES_ERR_ARG;
  int s = device_ready(plan);
  if (s != ULYSSES_OK) return s;
  return repack_bwd_impl(plan, src_heads, dst_seq, planes, static_cast<cudaStream_t>(stream));
}

int ulysses_prologue_repack_fwd(const ulysses_plan_t* plan, const void* src_seq, void* dst_heads,
                                const void* norm_q_weight, const void* norm_k_weight, const void* cos_table,
                                const void* sin_table, int32_t rotary_dim, float eps, void* stream) {
  NvtxRange range("ulysses_prologue_repack_fwd");
  if (!plan || !src_seq || !dst_heads || !norm_q_weight || !norm_k_weight) return ULYSSES_ERR_ARG;
  if (plan->C < 2 || !(eps > 0.f) || !std::isfinite(eps)) return ULYSSES_ERR_ARG;
  if (rotary_dim < 0 || rotary_dim > plan->D) return ULYSSES_ERR_ARG;
  if (rotary_dim % 16) return ULYSSES_ERR_UNSUPPORTED;
  if (rotary_dim > 0 && (!cos_table || !sin_table)) return ULYSSES_ERR_ARG;
  const void* ptrs[] = {src_seq, dst_heads, norm_q_weight, norm_k_weight};
  for (const void* q : ptrs)
    if (!aligned16(q)) return ULYSSES_ERR_ALIGN;
  if (rotary_dim > 0 && (!aligned16(cos_table) || !aligned16(sin_table))) return ULYSSES_ERR_ALIGN;
  if (overlap(src_seq, seq_extent_bytes(plan, plan->C, plan->token_stride, plan->plane_stride), dst_heads,
              heads_bytes(plan, plan->C)))
    return ULYSSES_ERR_ARG;
  int s = device_ready(plan);
  if (s != ULYSSES_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int32_t c0 = 0; c0 < plan->C; c0 += plan->plane_chunk) {
    const int32_t cc = std::min(plan->plane_chunk, plan->C - c0);
    s = status_of(ulysses::launch_prologue_repack(src_seq, dst_heads, norm_q_weight, norm_k_weight, cos_table,
                                                  sin_table, rotary_dim, eps, plan->Np, plan->H, plan->P, plan->C,
                                                  c0, cc, plan->token_stride, plan->plane_stride, st, plan->dev_err));
    if (s != ULYSSES_OK) return s;
  }
  return ULYSSES_OK;
}

int ulysses_attn_fwd(const ulysses_plan_t* plan, const void* qkv_heads, void* out_heads, float softmax_scale,
                     void* stream) {
  NvtxRange range("ulysses_attn_fwd");
  if (!plan || !qkv_heads || !out_heads) return ULYSSES_ERR_ARG;
  if (plan->C < 3 || !(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return ULYSSES_ERR_ARG;
  if (!aligned16(qkv_heads) || !aligned16(out_heads)) return ULYSSES_ERR_ALIGN;
  if (overlap(qkv_heads, heads_bytes(plan, plan->C), out_heads, heads_bytes(plan, 1))) return ULYSSES_ERR_ARG;
  int s = device_ready(plan);
  if (s != ULYSSES_OK) return s;
  return attn_impl(plan, qkv_heads, 0, out_heads, softmax_scale, static_cast<cudaStream_t>(stream));
}

int ulysses_repack_fwd_fp8(const ulysses_plan_t* plan, const void* src_seq, void* dst_heads_fp8, void* stream) {
  NvtxRange range("ulysses_repack_fwd_fp8");
  if (!plan || !src_seq || !dst_heads_fp8) return ULYSSES_ERR_ARG;
  if (!aligned16(src_seq) || !aligned16(dst_heads_fp8)) return ULYSSES_ERR_ALIGN;
  if (overlap(src_seq, seq_extent_bytes(plan, plan->C, plan->token_stride, plan->plane_stride), dst_heads_fp8,
              heads_bytes_fp8(plan, plan->C)))
    return ULYSSES_ERR_ARG;
  int s = device_ready(plan);
  if (s != ULYSSES_OK) return s;
  return repack_fwd_fp8_impl(plan, src_seq, dst_heads_fp8, static_cast<cudaStream_t>(stream));
}

int ulysses_attn_fwd_fp8(const ulysses_plan_t* plan, const void* qkv_heads_fp8, void* out_heads, float softmax_scale,
                         void* stream) {
  NvtxRange range("ulysses_attn_fwd_fp8");
  if (!plan || !qkv_heads_fp8 || !out_heads) return ULYSSES_ERR_ARG;
  if (plan->C < 3 || !(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return ULYSSES_ERR_ARG;
  if (!aligned16(qkv_heads_fp8) || !aligned16(out_heads)) return ULYSSES_ERR_ALIGN;
  if (overlap(qkv_heads_fp8, heads_bytes_fp8(plan, plan->C), out_heads, heads_bytes(plan, 1))) return ULYSSES_ERR_ARG;
  int s = device_ready(plan);
  if (s != ULYSSES_OK) return s;
  return attn_impl(plan, qkv_heads_fp8, 0, out_heads, softmax_scale, static_cast<cudaStream_t>(stream), nullptr, 1);
}

size_t ulysses_workspace_bytes_fp8(const ulysses_plan_t* plan) {
  if (!plan) return 0;
  return static_cast<size_t>(align_up(heads_bytes_fp8(plan, plan->C), 256) + align_up(heads_bytes(plan, 1), 256));
}

int ulysses_layer_fwd_fp8(const ulysses_plan_t* plan, const void* qkv_seq, void* out_seq, void* workspace,
                          size_t workspace_bytes, void* stream) {
  NvtxRange range("ulysses_layer_fwd_fp8");
  if (!plan || !qkv_seq || !out_seq) return ULYSSES_ERR_ARG;
  if (plan->C < 3) return ULYSSES_ERR_ARG;
  if (!aligned16(qkv_seq) || !aligned16(out_seq)) return ULYSSES_ERR_ALIGN;
  const int64_t in_bytes = seq_extent_bytes(plan, plan->C, plan->token_stride, plan->plane_stride);
  if (overlap(qkv_seq, in_bytes, out_seq, out_seq_bytes(plan))) return ULYSSES_ERR_ARG;
  if (!workspace || workspace_bytes < ulysses_workspace_bytes_fp8(plan)) return ULYSSES_ERR_WORKSPACE;
  if (!aligned16(workspace)) return ULYSSES_ERR_ALIGN;
  const int64_t ws = static_cast<int64_t>(ulysses_workspace_bytes_fp8(plan));
  if (overlap(workspace, ws, qkv_seq, in_bytes) || overlap(workspace, ws, out_seq, out_seq_bytes(plan)))
    return ULYSSES_ERR_ARG;
  int s = device_ready(plan);
  if (s != ULYSSES_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* T8 = static_cast<uint8_t*>(workspace);
  uint8_t* OT = T8 + align_up(heads_bytes_fp8(plan, plan->C), 256);
  if ((s = repack_fwd_fp8_impl(plan, qkv_seq, T8, st)) != ULYSSES_OK) return s;
  if ((s = attn_impl(plan, T8, 0, OT, 1.0f / std::sqrt(static_cast<float>(plan->D)), st, nullptr, 1)) != ULYSSES_OK)
    return s;
  return repack_bwd_impl(plan, OT, out_seq, 1, st);
}

size_t ulysses_lse_bytes(const ulysses_plan_t* plan) { return plan ? static_cast<size_t>(lse_bytes(plan)) : 0; }

int ulysses_attn_fwd_lse(const ulysses_plan_t* plan, const void* qkv_heads, void* out_heads, void* lse,
                         float softmax_scale, void* stream) {
  NvtxRange range("ulysses_attn_fwd_lse");
  if (!plan || !qkv_heads || !out_heads || !lse) return ULYSSES_ERR_ARG;
  if (plan->C < 3 || !(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return ULYSSES_ERR_ARG;
  if (!aligned16(qkv_heads) || !aligned16(out_heads) || !aligned16(lse)) return ULYSSES_ERR_ALIGN;
  if (overlap(qkv_heads, heads_bytes(plan, plan->C), out_heads, heads_bytes(plan, 1)) ||
      overlap(lse, lse_bytes(plan), qkv_heads, heads_bytes(plan, plan->C)) ||
      overlap(lse, lse_bytes(plan), out_heads, heads_bytes(plan, 1)))
    return ULYSSES_ERR_ARG;
  int s = device_ready(plan);
  if (s != ULYSSES_OK) return s;
  return attn_impl(plan, qkv_heads, 0, out_heads, softmax_scale, static_cast<cudaStream_t>(stream),
                   static_cast<float*>(lse));
}

// The one-pass backward's fp32 dQ accumulator [P*Hl][Np][D] (none for a
// deterministic plan), placed after the row terms at a 256-byte boundary.
// The offset rounds to 256 * P bytes so that the workspace is exactly P times
// that of one rank's slab (ulysses_attn_bwd_slab takes 1/P of it).
static int64_t dq_acc_offset(const ulysses_plan_t* plan) { return align_up(2 * lse_bytes(plan), 256 * plan->P); }
static int64_t dq_acc_bytes(const ulysses_plan_t* plan) {
  return plan->deterministic ? 0 : static_cast<int64_t>(plan->P) * plan->Hl * plan->Np * plan->D * 4;
}

size_t ulysses_attn_bwd_workspace_bytes(const ulysses_plan_t* plan) {
  if (!plan) return 0;
  return static_cast<size_t>(plan->deterministic ? 2 * lse_bytes(plan) : dq_acc_offset(plan) + dq_acc_bytes(plan));
}

int ulysses_attn_bwd(const ulysses_plan_t* plan, const void* qkv_heads, const void* out_heads,
                     const void* dout_heads, const void* lse, void* dqkv_heads, void* workspace,
                     size_t workspace_bytes, float softmax_scale, void* stream) {
  NvtxRange range("ulysses_attn_bwd");
  if (!plan || !qkv_heads || !out_heads || !dout_heads || !lse || !dqkv_heads) return ULYSSES_ERR_ARG;
  if (plan->C < 3 || !(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return ULYSSES_ERR_ARG;
  if (!workspace || workspace_bytes < ulysses_attn_bwd_workspace_bytes(plan)) return ULYSSES_ERR_WORKSPACE;
  const void* ptrs[] = {qkv_heads, out_heads, dout_heads, lse, dqkv_heads, workspace};
  for (const void* q : ptrs)
    if (!aligned16(q)) return ULYSSES_ERR_ALIGN;
  const int64_t dq = heads_bytes(plan, 3), lb = lse_bytes(plan),
                ws = static_cast<int64_t>(ulysses_attn_bwd_workspace_bytes(plan));
  if (overlap(dqkv_heads, dq, qkv_heads, heads_bytes(plan, plan->C)) || overlap(dqkv_heads, dq, out_heads, heads_bytes(plan, 1)) ||
      overlap(dqkv_heads, dq, dout_heads, heads_bytes(plan, 1)) || overlap(dqkv_heads, dq, lse, lb) ||
      overlap(workspace, ws, dqkv_heads, dq) || overlap(workspace, ws, lse, lb) ||
      overlap(workspace, ws, qkv_heads, heads_bytes(plan, plan->C)) || overlap(workspace, ws, out_heads, heads_bytes(plan, 1)) ||
      overlap(workspace, ws, dout_heads, heads_bytes(plan, 1)))
    return ULYSSES_ERR_ARG;
  int s = device_ready(plan);
  if (s != ULYSSES_OK) return s;
  ulysses::AttnBwdLaunch a;
  a.qkv = qkv_heads;
  a.out = out_heads;
  a.dout = dout_heads;
  a.lse = static_cast<const float*>(lse);
  a.delta = static_cast<float*>(workspace);
  a.dq_acc = plan->deterministic
                 ? nullptr
                 : reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + dq_acc_offset(plan));
  a.dqkv = dqkv_heads;
  a.scale = softmax_scale;
  a.plan = plan;
  return status_of(ulysses::launch_attn_bwd(a, static_cast<cudaStream_t>(stream)));
}

size_t ulysses_layer_bwd_workspace_bytes(const ulysses_plan_t* plan) {
  if (!plan) return 0;
  return static_cast<size_t>(align_up(heads_bytes(plan, 1), 256) + align_up(heads_bytes(plan, 3), 256) +
                             align_up(static_cast<int64_t>(ulysses_attn_bwd_workspace_bytes(plan)), 256));
}

int ulysses_layer_bwd(const ulysses_plan_t* plan, const void* qkv_heads, const void* out_heads, const void* lse,
                      const void* dout_seq, void* dqkv_seq, void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange range("ulysses_layer_bwd");
  if (!plan || !qkv_heads || !out_heads || !lse || !dout_seq || !dqkv_seq) return ULYSSES_ERR_ARG;
  if (plan->C < 3) return ULYSSES_ERR_ARG;
  if (!workspace || workspace_bytes < ulysses_layer_bwd_workspace_bytes(plan)) return ULYSSES_ERR_WORKSPACE;
  const void* ptrs[] = {qkv_heads, out_heads, lse, dout_seq, dqkv_seq, workspace};
  for (const void* q : ptrs)
    if (!aligned16(q)) return ULYSSES_ERR_ALIGN;
  const int64_t ws = static_cast<int64_t>(ulysses_layer_bwd_workspace_bytes(plan));
  const int64_t dseq = seq_extent_bytes(plan, plan->C, plan->token_stride, plan->plane_stride);
  if (overlap(workspace, ws, qkv_heads, heads_bytes(plan, plan->C)) || overlap(workspace, ws, out_heads, heads_bytes(plan, 1)) ||
      overlap(workspace, ws, lse, lse_bytes(plan)) || overlap(workspace, ws, dout_seq, out_seq_bytes(plan)) ||
      overlap(workspace, ws, dqkv_seq, dseq) || overlap(dqkv_seq, dseq, dout_seq, out_seq_bytes(plan)) ||
      overlap(dqkv_seq, dseq, qkv_heads, heads_bytes(plan, plan->C)))
    return ULYSSES_ERR_ARG;
  int s = device_ready(plan);
  if (s != ULYSSES_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* dOT = static_cast<uint8_t*>(workspace);
  uint8_t* dT = dOT + align_up(heads_bytes(plan, 1), 256);
  float* delta = reinterpret_cast<float*>(dT + align_up(heads_bytes(plan, 3), 256));
  // mode 0 on the output gradient (one dense plane [Np, H, D])
  const int64_t row = static_cast<int64_t>(plan->H) * plan->D;
  s = status_of(
      ulysses::launch_repack(0, dout_seq, dOT, plan->Np, plan->H, plan->P, 1, 0, 1, row, row, st, plan->dev_err));
  if (s != ULYSSES_OK) return s;
  ulysses::AttnBwdLaunch a;
  a.qkv = qkv_heads;
  a.out = out_heads;
  a.dout = dOT;
  a.lse = static_cast<const float*>(lse);
  a.delta = delta;
  a.dq_acc = plan->deterministic ? nullptr
                                 : reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(delta) + dq_acc_offset(plan));
  a.dqkv = dT;
  a.scale = 1.0f / std::sqrt(static_cast<float>(plan->D));
  a.plan = plan;
  s = status_of(ulysses::launch_attn_bwd(a, st));
  if (s != ULYSSES_OK) return s;
  // mode 1 on dQ, dK, dV into planes 0..2 of the plan's input layout
  for (int32_t c0 = 0; c0 < 3; c0 += plan->plane_chunk) {
    const int32_t cc = std::min(plan->plane_chunk, 3 - c0);
    s = status_of(ulysses::launch_repack(1, dT, dqkv_seq, plan->Np, plan->H, plan->P, 3, c0, cc, plan->token_stride,
                                         plan->plane_stride, st, plan->dev_err));
    if (s != ULYSSES_OK) return s;
  }
  return ULYSSES_OK;
}

int ulysses_layer_fwd(const ulysses_plan_t* plan, const void* qkv_seq, void* out_seq, void* workspace,
                      size_t workspace_bytes, int32_t fused, void* stream) {
  NvtxRange range("ulysses_layer_fwd");
  if (!plan || !qkv_seq || !out_seq) return ULYSSES_ERR_ARG;
  if (plan->C < 3 || (fused != 0 && fused != 1)) return ULYSSES_ERR_ARG;
  if (!aligned16(qkv_seq) || !aligned16(out_seq)) return ULYSSES_ERR_ALIGN;
  const int64_t in_bytes = seq_extent_bytes(plan, plan->C, plan->token_stride, plan->plane_stride);
  if (overlap(qkv_seq, in_bytes, out_seq, out_seq_bytes(plan))) return ULYSSES_ERR_ARG;
  const float scale = 1.0f / std::sqrt(static_cast<float>(plan->D));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (fused) {
    int s = device_ready(plan);
    if (s != ULYSSES_OK) return s;
    NvtxRange step("fused attention");
    return attn_impl(plan, qkv_seq, 1, out_seq, scale, st);
  }
  if (!workspace) return ULYSSES_ERR_WORKSPACE;
  if (workspace_bytes < ulysses_workspace_bytes(plan)) return ULYSSES_ERR_WORKSPACE;
  if (!aligned16(workspace)) return ULYSSES_ERR_ALIGN;
  const int64_t ws = static_cast<int64_t>(ulysses_workspace_bytes(plan));
  if (overlap(workspace, ws, qkv_seq, in_bytes) || overlap(workspace, ws, out_seq, out_seq_bytes(plan)))
    return ULYSSES_ERR_ARG;
  int s = device_ready(plan);
  if (s != ULYSSES_OK) return s;
  uint8_t* T = static_cast<uint8_t*>(workspace);
  uint8_t* OT = T + align_up(heads_bytes(plan, plan->C), 256);
  {
    NvtxRange step("repack_fwd");
    if ((s = repack_fwd_impl(plan, qkv_seq, T, st)) != ULYSSES_OK) return s;
  }
  {
    NvtxRange step("attention");
    if ((s = attn_impl(plan, T, 0, OT, scale, st)) != ULYSSES_OK) return s;
  }
  NvtxRange step("repack_bwd");
  return repack_bwd_impl(plan, OT, out_seq, 1, st);
}

}  // extern "C"

namespace {

// The host-buffer layer for the three modes of group_layer_impl.
int layer_host_impl(const ulysses_plan_t* plan, const void* host_qkv_seq, void* host_out_seq, void* dev_qkv_seq,
                    void* dev_out_seq, void* workspace, size_t workspace_bytes, int32_t mode, void* stream) {
  if (!plan || !host_qkv_seq || !host_out_seq || !dev_qkv_seq || !dev_out_seq) return ULYSSES_ERR_ARG;
  const int32_t fused = mode == 1;
  if (plan->C < 3 || mode < 0 || mode > 2) return ULYSSES_ERR_ARG;
  if (!aligned16(dev_qkv_seq) || !aligned16(dev_out_seq)) return ULYSSES_ERR_ALIGN;
  const int64_t in_bytes = seq_extent_bytes(plan, plan->C, plan->token_stride, plan->plane_stride);
  if (overlap(dev_qkv_seq, in_bytes, dev_out_seq, out_seq_bytes(plan)) ||
      overlap(host_qkv_seq, in_bytes, host_out_seq, out_seq_bytes(plan)))
    return ULYSSES_ERR_ARG;
  uint8_t* T = nullptr;
  uint8_t* OT = nullptr;
  if (!fused) {
    const size_t need = mode == 2 ? ulysses_workspace_bytes_fp8(plan) : ulysses_workspace_bytes(plan);
    if (!workspace || workspace_bytes < need) return ULYSSES_ERR_WORKSPACE;
    if (!aligned16(workspace)) return ULYSSES_ERR_ALIGN;
    const int64_t ws = static_cast<int64_t>(need);
    if (overlap(workspace, ws, dev_qkv_seq, in_bytes) || overlap(workspace, ws, dev_out_seq, out_seq_bytes(plan)))
      return ULYSSES_ERR_ARG;
    T = static_cast<uint8_t*>(workspace);
    OT = T + align_up(mode == 2 ? heads_bytes_fp8(plan, plan->C) : heads_bytes(plan, plan->C), 256);
  }
  int s = device_ready(plan);
  if (s != ULYSSES_OK) return s;
  const float scale = 1.0f / std::sqrt(static_cast<float>(plan->D));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const uint8_t* hin = static_cast<const uint8_t*>(host_qkv_seq);
  uint8_t* hout = static_cast<uint8_t*>(host_out_seq);
  uint8_t* din = static_cast<uint8_t*>(dev_qkv_seq);
  uint8_t* dout = static_cast<uint8_t*>(dev_out_seq);

  std::lock_guard<std::mutex> lock(g_pipe_mutex);
  ulysses::HostPipe* h = plan_pipe(plan);
  if (!h) return ULYSSES_ERR_CUDA;
  const int32_t groups = h->n;
  const size_t head_bytes = static_cast<size_t>(plan->D) * 2, pitch = static_cast<size_t>(plan->H) * plan->D * 2;
  // the copies start after everything already queued on the caller's stream
  if (cudaEventRecord(h->start, st) != cudaSuccess || cudaStreamWaitEvent(h->h2d, h->start, 0) != cudaSuccess)
    return status_of(cudaErrorUnknown);
  for (int32_t g = 0; g < groups; ++g) {
    if (copy_heads_in(plan, h->h0[g], h->hg[g], hin, din, h->h2d) != cudaSuccess ||
        cudaEventRecord(h->in[g], h->h2d) != cudaSuccess)
      return status_of(cudaErrorUnknown);
  }
  // with fused = 0 the groups' head slabs and attention outputs sit one after
  // another in the workspace (they add up to the whole T and O_T)
  int64_t t_off = 0, o_off = 0;
  for (int32_t g = 0; g < groups; ++g) {
    const int32_t h0 = h->h0[g], hg = h->hg[g];
    const size_t off = h0 * head_bytes, width = hg * head_bytes;
    if (cudaStreamWaitEvent(st, h->in[g], 0) != cudaSuccess) return status_of(cudaErrorUnknown);
    uint8_t* Tg = fused ? nullptr : T + t_off;
    uint8_t* OTg = fused ? nullptr : OT + o_off;
    t_off += static_cast<int64_t>(plan->C) * plan->Np * static_cast<int64_t>(width) / (mode == 2 ? 2 : 1);
    o_off += plan->Np * static_cast<int64_t>(width);
    if ((s = group_layer_impl(plan, h0, hg, din, dout, Tg, OTg, mode, scale, st)) != ULYSSES_OK) return s;
    if (cudaEventRecord(h->out[g], st) != cudaSuccess || cudaStreamWaitEvent(h->d2h, h->out[g], 0) != cudaSuccess ||
        cudaMemcpy2DAsync(hout + off, pitch, dout + off, pitch, width, static_cast<size_t>(plan->Np),
                          cudaMemcpyDeviceToHost, h->d2h) != cudaSuccess)
      return status_of(cudaErrorUnknown);
  }
  // the caller's stream completes only after the last output copy
  if (cudaEventRecord(h->done, h->d2h) != cudaSuccess || cudaStreamWaitEvent(st, h->done, 0) != cudaSuccess)
    return status_of(cudaErrorUnknown);
  return ULYSSES_OK;
}

}  // namespace

extern "C" {

int ulysses_layer_fwd_host(const ulysses_plan_t* plan, const void* host_qkv_seq, void* host_out_seq,
                           void* dev_qkv_seq, void* dev_out_seq, void* workspace, size_t workspace_bytes,
                           int32_t fused, void* stream) {
  NvtxRange range("ulysses_layer_fwd_host");
  if (fused != 0 && fused != 1) return ULYSSES_ERR_ARG;
  return layer_host_impl(plan, host_qkv_seq, host_out_seq, dev_qkv_seq, dev_out_seq, workspace, workspace_bytes,
                         fused, stream);
}

int ulysses_layer_fwd_fp8_host(const ulysses_plan_t* plan, const void* host_qkv_seq, void* host_out_seq,
                               void* dev_qkv_seq, void* dev_out_seq, void* workspace, size_t workspace_bytes,
                               void* stream) {
  NvtxRange range("ulysses_layer_fwd_fp8_host");
  return layer_host_impl(plan, host_qkv_seq, host_out_seq, dev_qkv_seq, dev_out_seq, workspace, workspace_bytes, 2,
                         stream);
}

int ulysses_repack_fwd_push(const ulysses_plan_t* plan, int32_t rank, const void* src_shard,
                            void* const* dst_heads, int32_t planes, void* stream) {
  NvtxRange range("ulysses_repack_fwd_push");
  if (!plan || !src_shard || !dst_heads || rank < 0 || rank >= plan->P || planes < 1 || planes > plan->C)
    return ULYSSES_ERR_ARG;
  if (!push_layout_ok(plan)) return ULYSSES_ERR_UNSUPPORTED;
  if (!aligned16(src_shard)) return ULYSSES_ERR_ALIGN;
  const int64_t shard_bytes = plan->Nl * planes * plan->H * plan->D * 2;
  const int64_t slab_bytes = static_cast<int64_t>(planes) * plan->Np * plan->Hl * plan->D * 2;
  ulysses::PushTable t;
  int s = push_table(plan, dst_heads, slab_bytes, src_shard, shard_bytes, &t);
  if (s != ULYSSES_OK) return s;
  if ((s = device_ready(plan)) != ULYSSES_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int32_t c0 = 0; c0 < planes; c0 += plan->plane_chunk) {
    const int32_t cc = std::min(plan->plane_chunk, planes - c0);
    s = status_of(ulysses::launch_push(0, src_shard, t, plan->Nl, plan->Np, plan->H, plan->P, planes, c0, cc, rank,
                                       st, plan->dev_err));
    if (s != ULYSSES_OK) return s;
  }
  return ULYSSES_OK;
}

int ulysses_repack_bwd_push(const ulysses_plan_t* plan, int32_t rank, const void* src_heads, void* const* dst_seq,
                            int32_t planes, void* stream) {
  NvtxRange range("ulysses_repack_bwd_push");
  if (!plan || !src_heads || !dst_seq || rank < 0 || rank >= plan->P || planes < 1 || planes > plan->C)
    return ULYSSES_ERR_ARG;
  if (!push_layout_ok(plan)) return ULYSSES_ERR_UNSUPPORTED;
  if (!aligned16(src_heads)) return ULYSSES_ERR_ALIGN;
  const int64_t slab_bytes = static_cast<int64_t>(planes) * plan->Np * plan->Hl * plan->D * 2;
  const int64_t shard_bytes = plan->Nl * planes * plan->H * plan->D * 2;
  ulysses::PushTable t;
  int s = push_table(plan, dst_seq, shard_bytes, src_heads, slab_bytes, &t);
  if (s != ULYSSES_OK) return s;
  if ((s = device_ready(plan)) != ULYSSES_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int32_t c0 = 0; c0 < planes; c0 += plan->plane_chunk) {
    const int32_t cc = std::min(plan->plane_chunk, planes - c0);
    s = status_of(ulysses::launch_push(1, src_heads, t, plan->Nl, plan->Np, plan->H, plan->P, planes, c0, cc, rank,
                                       st, plan->dev_err));
    if (s != ULYSSES_OK) return s;
  }
  return ULYSSES_OK;
}

int ulysses_attn_fwd_push(const ulysses_plan_t* plan, int32_t rank, const void* heads, void* const* dst_seq,
                          float softmax_scale, void* stream) {
  NvtxRange range("ulysses_attn_fwd_push");
  if (!plan || !heads || !dst_seq || rank < 0 || rank >= plan->P) return ULYSSES_ERR_ARG;
  if (plan->C < 3 || !(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return ULYSSES_ERR_ARG;
  if (!push_layout_ok(plan)) return ULYSSES_ERR_UNSUPPORTED;
  if (!aligned16(heads)) return ULYSSES_ERR_ALIGN;
  const int64_t slab_bytes = static_cast<int64_t>(plan->C) * plan->Np * plan->Hl * plan->D * 2;
  const int64_t shard_bytes = plan->Nl * plan->H * plan->D * 2;
  ulysses::PushTable t;
  int s = push_table(plan, dst_seq, shard_bytes, heads, slab_bytes, &t);
  if (s != ULYSSES_OK) return s;
  if ((s = device_ready(plan)) != ULYSSES_OK) return s;
  // this rank's heads start at column rank*Hl of every destination row
  for (int32_t q = 0; q < plan->P; ++q)
    t.p[q] = static_cast<uint8_t*>(t.p[q]) + static_cast<int64_t>(rank) * plan->Hl * plan->D * 2;
  ulysses::AttnLaunch a;
  a.base = heads;
  a.fused = 0;
  a.Np = plan->Np;
  a.N = plan->N;
  a.H = plan->Hl;   // one rank's slab: a one-rank problem of Hl heads
  a.P = 1;
  a.Hl = plan->Hl;
  a.C = plan->C;
  a.tok_stride = plan->token_stride;
  a.plane_stride = plan->plane_stride;
  a.out = t.p[0];
  a.o_stride_r = 0;
  a.o_stride_n = static_cast<int64_t>(plan->H) * plan->D;
  a.o_stride_j = plan->D;
  a.scale = softmax_scale;
  a.plan = plan;
  a.push = &t;
  a.push_rows = plan->Nl;
  a.push_ranks = plan->P;
  return status_of(ulysses::launch_attn(a, static_cast<cudaStream_t>(stream)));
}

int ulysses_a2a_pack(const ulysses_plan_t* plan, const void* src_shard, int32_t planes, int32_t plane, void* send,
                     void* stream) {
  NvtxRange range("ulysses_a2a_pack");
  if (!plan || !src_shard || !send || planes < 1 || planes > kMaxPlanes || plane < 0 || plane >= planes)
    return ULYSSES_ERR_ARG;
  if (!push_layout_ok(plan)) return ULYSSES_ERR_UNSUPPORTED;
  if (!aligned16(src_shard) || !aligned16(send)) return ULYSSES_ERR_ALIGN;
  const int64_t row = static_cast<int64_t>(plan->H) * plan->D;
  const int64_t shard_bytes = plan->Nl * planes * row * 2;
  const int64_t send_bytes = plan->Nl * row * 2;
  if (overlap(src_shard, shard_bytes, send, send_bytes)) return ULYSSES_ERR_ARG;
  int s = device_ready(plan);
  if (s != ULYSSES_OK) return s;
  // mode 0 over the shard's Nl rows, one plane: send [P, 1, Nl, Hl, D]
  const uint8_t* src = static_cast<const uint8_t*>(src_shard) + static_cast<int64_t>(plane) * row * 2;
  return status_of(ulysses::launch_repack(0, src, send, plan->Nl, plan->H, plan->P, 1, 0, 1, planes * row, row,
                                          static_cast<cudaStream_t>(stream), plan->dev_err));
}

int ulysses_a2a_unpack(const ulysses_plan_t* plan, const void* recv, void* out_shard, int32_t planes, int32_t plane,
                       void* stream) {
  NvtxRange range("ulysses_a2a_unpack");
  if (!plan || !recv || !out_shard || planes < 1 || planes > kMaxPlanes || plane < 0 || plane >= planes)
    return ULYSSES_ERR_ARG;
  if (!push_layout_ok(plan)) return ULYSSES_ERR_UNSUPPORTED;
  if (!aligned16(recv) || !aligned16(out_shard)) return ULYSSES_ERR_ALIGN;
  const int64_t row = static_cast<int64_t>(plan->H) * plan->D;
  if (overlap(recv, plan->Nl * row * 2, out_shard, plan->Nl * planes * row * 2)) return ULYSSES_ERR_ARG;
  int s = device_ready(plan);
  if (s != ULYSSES_OK) return s;
  // mode 1 over Nl rows, one plane: recv [P, 1, Nl, Hl, D] -> plane `plane` of [Nl, planes, H, D]
  uint8_t* dst = static_cast<uint8_t*>(out_shard) + static_cast<int64_t>(plane) * row * 2;
  return status_of(ulysses::launch_repack(1, recv, dst, plan->Nl, plan->H, plan->P, 1, 0, 1, planes * row, row,
                                          static_cast<cudaStream_t>(stream), plan->dev_err));
}

int ulysses_attn_fwd_lse_slab(const ulysses_plan_t* plan, const void* heads, void* out_heads, void* lse,
                              float softmax_scale, void* stream) {
  NvtxRange range("ulysses_attn_fwd_lse_slab");
  if (!plan) return ULYSSES_ERR_ARG;
  const ulysses_plan_t v = slab_view(plan);
  return ulysses_attn_fwd_lse(&v, heads, out_heads, lse, softmax_scale, stream);
}

int ulysses_attn_bwd_slab(const ulysses_plan_t* plan, const void* heads, const void* out_heads,
                          const void* dout_heads, const void* lse, void* dqkv_heads, void* workspace,
                          size_t workspace_bytes, float softmax_scale, void* stream) {
  NvtxRange range("ulysses_attn_bwd_slab");
  if (!plan) return ULYSSES_ERR_ARG;
  const ulysses_plan_t v = slab_view(plan);
  return ulysses_attn_bwd(&v, heads, out_heads, dout_heads, lse, dqkv_heads, workspace, workspace_bytes,
                          softmax_scale, stream);
}

int ulysses_last_device_error(const ulysses_plan_t* plan, void* stream) {
  if (!plan || !plan->dev_err) return -1;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  unsigned int v = 0;
  if (cudaMemcpy(&v, plan->dev_err, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  if (v != 0 && cudaMemset(plan->dev_err, 0, sizeof(v)) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  return static_cast<int>(v);
}

const char* ulysses_strerror(int code) {
  switch (code) {
    case ULYSSES_OK: return "ok";
    case ULYSSES_ERR_ARG: return "invalid argument (null or overlapping pointer, bad size or cu_seqlens)";
    case ULYSSES_ERR_DIVISIBILITY: return "heads are not divisible by the number of ranks";
    case ULYSSES_ERR_ALIGN: return "pointer or stride is not 16-byte aligned";
    case ULYSSES_ERR_WINDOW: return "one plane per rank exceeds the 1 GiB window";
    case ULYSSES_ERR_WORKSPACE: return "workspace missing or too small";
    case ULYSSES_ERR_CUDA: return "CUDA call failed or no CUDA device";
    case ULYSSES_ERR_DEVICE: return "a kernel reported an error";
    case ULYSSES_ERR_UNSUPPORTED: return "unsupported configuration";
    default: return "unknown error code";
  }
}

}  // extern "C"
