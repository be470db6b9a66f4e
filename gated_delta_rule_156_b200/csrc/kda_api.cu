// C-ABI boundary of libkda.so: argument validation, workspace, dispatch.
// Every argument error is found here, on the host, before anything launches.
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "../../include/kda.h"
#include "kda_internal.h"

namespace {

thread_local int g_last_cuda_error = 0;

kda_status cuda_fail(cudaError_t e) {
  g_last_cuda_error = (int)e;
  return KDA_ERR_CUDA;
}

bool supported_dim(int d) { return d == 32 || d == 64 || d == 128; }
bool supported_chunk(int c) { return c == 16 || c == 32 || c == 64; }
bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
bool aligned4(const void* p) { return ((uintptr_t)p & 3u) == 0; }

struct Range {
  uintptr_t lo, hi;
};
Range span(const void* p, size_t bytes) {
  return Range{(uintptr_t)p, (uintptr_t)p + bytes};
}
bool overlap(Range a, Range b) {
  return a.lo != 0 && b.lo != 0 && a.lo < b.hi && b.lo < a.hi && a.hi > a.lo &&
         b.hi > b.lo;
}

// Keep freed stream-ordered workspace in the device's pool instead of handing
// it back to the driver at every synchronisation.
void keep_pool_memory() {
  static std::atomic<uint64_t> done_mask{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return;
  const uint64_t bit = 1ull << dev;
  if (done_mask.load() & bit) return;
  cudaMemPool_t pool;
  if (cudaDeviceGetDefaultMemPool(&pool, dev) == cudaSuccess) {
    uint64_t thr = UINT64_MAX;
    cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &thr);
  }
  done_mask.fetch_or(bit);
}

// Stream-ordered workspace for one call.  With KDA_WORKSPACE_FILL set to a
// byte value (0-255) the workspace is first filled with that byte: a test
// aid, since with 127 every fp32 word reads 3.4e38 and a kernel that read a
// place before writing it would turn its results non-finite or far off.
cudaError_t take_workspace(size_t bytes, cudaStream_t stream, void** ws) {
  *ws = nullptr;
  if (!bytes) return cudaSuccess;
  keep_pool_memory();
  cudaError_t e = cudaMallocAsync(ws, bytes, stream);
  if (e != cudaSuccess) {
    *ws = nullptr;
    return e;
  }
  const char* fill = getenv("KDA_WORKSPACE_FILL");
  if (fill && *fill) e = cudaMemsetAsync(*ws, atoi(fill) & 255, bytes, stream);
  return e;
}

// Shape-only checks shared by the launch entry points and the planner.
kda_status validate_chunk_shape(const kda_shape* s, bool packed, int* n_seqs) {
  if (!s) return KDA_ERR_INVALID_ARG;
  if (s->B < 0 || s->T < 0 || s->H < 1) return KDA_ERR_INVALID_ARG;
  if (s->io_dtype != KDA_BF16 && s->io_dtype != KDA_F32)
    return KDA_ERR_INVALID_ARG;
  if (!supported_dim(s->dk) || !supported_dim(s->dv)) return KDA_ERR_UNSUPPORTED;
  if (!supported_chunk(s->chunk)) return KDA_ERR_UNSUPPORTED;
  *n_seqs = s->B;
  if (packed) {
    if (s->B != 1 || s->n_seqs < 1) return KDA_ERR_INVALID_ARG;
    *n_seqs = s->n_seqs;
  }
  if ((size_t)s->B * (size_t)s->T > (size_t)INT32_MAX ||
      (size_t)*n_seqs * (size_t)s->H > (size_t)INT32_MAX || s->H > 65535)
    return KDA_ERR_UNSUPPORTED;
  return KDA_OK;
}

void fill_args(const kda_shape* s, int n_seqs, kda::ChunkArgs* a) {
  a->n_seqs = n_seqs;
  a->T = s->T;
  a->H = s->H;
  a->dk = s->dk;
  a->dv = s->dv;
  a->chunk = s->chunk;
  a->bf16 = s->io_dtype == KDA_BF16;
}

kda_status validate_chunk(const kda_shape* s, const void* q, const void* k,
                          const void* v, const float* la, const float* beta,
                          const float* s_init, const int32_t* cu, void* out,
                          float* s_final, kda::ChunkArgs* a,
                          int gate = kda::kGateChannel) {
  int n_seqs = 0;
  const kda_status st = validate_chunk_shape(s, cu != nullptr, &n_seqs);
  if (st != KDA_OK) return st;
  if (gate != kda::kGateChannel && gate != kda::kGateHead &&
      gate != kda::kGateNone)
    return KDA_ERR_INVALID_ARG;
  const size_t esz = s->io_dtype == KDA_BF16 ? 2 : 4;
  const size_t tokens = (size_t)s->B * (size_t)s->T;
  const size_t H = s->H;
  const bool any_tokens = tokens > 0;
  const bool any_state = n_seqs > 0;
  if (gate == kda::kGateNone) la = nullptr;  // alpha = 1: no gate tensor
  if (any_tokens && (!q || !k || !v || !beta || !out)) return KDA_ERR_INVALID_ARG;
  if (any_tokens && gate != kda::kGateNone && !la) return KDA_ERR_INVALID_ARG;
  if (any_state && !s_final) return KDA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, s_init, out, s_final};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
  if (la && !(gate == kda::kGateChannel ? aligned16(la) : aligned4(la)))
    return KDA_ERR_MISALIGNED;
  if ((beta && !aligned4(beta)) || (cu && !aligned4(cu)))
    return KDA_ERR_MISALIGNED;
  // The output may alias no input; the final state may only coincide exactly
  // with the initial state (in-place update).
  const Range rq = span(q, tokens * H * s->dk * esz),
              rk = span(k, tokens * H * s->dk * esz),
              rv = span(v, tokens * H * s->dv * esz),
              rl = span(la, tokens * H * (gate == kda::kGateChannel ? s->dk : 1) * 4),
              rb = span(beta, tokens * H * 4),
              ro = span(out, tokens * H * s->dv * esz),
              rsi = span(s_init, (size_t)n_seqs * H * s->dk * s->dv * 4),
              rsf = span(s_final, (size_t)n_seqs * H * s->dk * s->dv * 4),
              rc = span(cu, cu ? 4 * ((size_t)n_seqs + 1) : 0);
  for (Range r : {rq, rk, rv, rl, rb, rsi, rsf, rc})
    if (any_tokens && overlap(ro, r)) return KDA_ERR_INVALID_ARG;
  for (Range r : {rq, rk, rv, rl, rb, rc})
    if (any_state && overlap(rsf, r)) return KDA_ERR_INVALID_ARG;
  if (s_init && overlap(rsf, rsi) && s_init != s_final) return KDA_ERR_INVALID_ARG;

  a->q = q;
  a->k = k;
  a->v = v;
  a->log_alpha = la;
  a->beta = beta;
  a->initial_state = s_init;
  a->cu_seqlens = cu;
  a->out = out;
  a->final_state = s_final;
  fill_args(s, n_seqs, a);
  a->gate = gate;
  return KDA_OK;
}

enum class Path { kStaged, kFused, kTwoPass };

kda_status run_with_workspace(size_t bytes, cudaStream_t stream, Path path,
                              const kda::ChunkArgs& a) {
  void* ws = nullptr;
  cudaError_t e;
  if ((e = take_workspace(bytes, stream, &ws)) != cudaSuccess) {
    if (ws) cudaFreeAsync(ws, stream);
    return cuda_fail(e);
  }
  e = path == Path::kFused     ? kda::launch_fused(a, ws, stream)
      : path == Path::kTwoPass ? kda::launch_twopass(a, ws, stream)
                               : kda::launch_staged(a, ws, stream);
  if (ws) {
    const cudaError_t f = cudaFreeAsync(ws, stream);
    if (e == cudaSuccess) e = f;
  }
  return e == cudaSuccess ? KDA_OK : cuda_fail(e);
}

// ---- fixed scratch for kda_chunk_fwd_staged_noalloc ----------------------
// The four-stage pipeline's workspace for callers that cannot allocate device
// memory.  Every GPU that loads this library holds the array until the
// process exits.  Host code must not pass `g_noalloc_scratch` itself to a
// kernel: on the host that name is only a stand-in, so its device address is
// looked up once per device below.
static __device__ __align__(256) unsigned char
    g_noalloc_scratch[KDA_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device, looked up (with
// that device current) the first time each device asks, then cached.
void* noalloc_scratch(cudaError_t* err) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    *err = e;
    return nullptr;
  }
  if (dev < 0 || dev >= 64) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) {
      *err = e;
      return nullptr;
    }
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace

extern "C" {

kda_status kda_chunk_fwd(const kda_shape* shape, const void* q, const void* k,
                         const void* v, const float* log_alpha,
                         const float* beta, const float* initial_state,
                         const int32_t* cu_seqlens, void* out,
                         float* final_state, cudaStream_t stream) {
  kda::ChunkArgs a{};
  const kda_status st = validate_chunk(shape, q, k, v, log_alpha, beta,
                                       initial_state, cu_seqlens, out,
                                       final_state, &a);
  if (st != KDA_OK) return st;
  if (kda::fused_supported(a))
    return run_with_workspace(kda::twopass_workspace_bytes(a), stream, Path::kTwoPass, a);
  return run_with_workspace(kda::staged_workspace_bytes(a), stream, Path::kStaged, a);
}

kda_status kda_chunk_fwd_split(const kda_shape* shape, int gate, const void* q,
                               const void* k, const void* v,
                               const float* gate_tensor, const float* beta,
                               const float* initial_state, void* out,
                               float* final_state, int n_segments,
                               cudaStream_t stream) {
  if (!shape || shape->B != 1 || n_segments < 0 || n_segments > 64)
    return KDA_ERR_INVALID_ARG;
  kda::ChunkArgs a{};
  const kda_status st = validate_chunk(shape, q, k, v, gate_tensor, beta,
                                       initial_state, nullptr, out,
                                       final_state, &a, gate);
  if (st != KDA_OK) return st;
  if (n_segments == 0) {
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
      e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    n_segments = kda::split_auto_segments(a, sms);
  }
  const kda::SplitGeom g = kda::split_geometry(a, n_segments);
  const size_t bytes = kda::split_workspace_bytes(a, g);
  void* ws = nullptr;
  cudaError_t e;
  if ((e = take_workspace(bytes, stream, &ws)) != cudaSuccess) {
    if (ws) cudaFreeAsync(ws, stream);
    return cuda_fail(e);
  }
  e = kda::launch_split(a, g, ws, stream);
  if (ws) {
    const cudaError_t f = cudaFreeAsync(ws, stream);
    if (e == cudaSuccess) e = f;
  }
  return e == cudaSuccess ? KDA_OK : cuda_fail(e);
}

kda_status kda_chunk_fwd_split_plan(const kda_shape* shape, int gate,
                                    int n_segments, int num_sms, int* segments,
                                    int* kernels, size_t* workspace_bytes) {
  if (!shape || shape->B != 1 || n_segments < 0 || n_segments > 64)
    return KDA_ERR_INVALID_ARG;
  if (n_segments == 0 && num_sms < 1) return KDA_ERR_INVALID_ARG;
  if (gate != kda::kGateChannel && gate != kda::kGateHead &&
      gate != kda::kGateNone)
    return KDA_ERR_INVALID_ARG;
  int n_seqs = 0;
  const kda_status st = validate_chunk_shape(shape, false, &n_seqs);
  if (st != KDA_OK) return st;
  kda::ChunkArgs a{};
  fill_args(shape, n_seqs, &a);
  a.gate = gate;
  if (n_segments == 0) n_segments = kda::split_auto_segments(a, num_sms);
  const kda::SplitGeom g = kda::split_geometry(a, n_segments);
  if (segments) *segments = g.k;
  if (kernels) *kernels = kda::split_kernel_count(a, g);
  if (workspace_bytes) *workspace_bytes = kda::split_workspace_bytes(a, g);
  return KDA_OK;
}

kda_status kda_chunk_fwd_staged(const kda_shape* shape, const void* q,
                                const void* k, const void* v,
                                const float* log_alpha, const float* beta,
                                const float* initial_state,
                                const int32_t* cu_seqlens, void* out,
                                float* final_state, cudaStream_t stream) {
  kda::ChunkArgs a{};
  const kda_status st = validate_chunk(shape, q, k, v, log_alpha, beta,
                                       initial_state, cu_seqlens, out,
                                       final_state, &a);
  if (st != KDA_OK) return st;
  return run_with_workspace(kda::staged_workspace_bytes(a), stream, Path::kStaged, a);
}

kda_status kda_chunk_bwd(const kda_shape* shape, const void* q, const void* k,
                         const void* v, const float* log_alpha,
                         const float* beta, const float* initial_state,
                         const int32_t* cu_seqlens, const void* d_out,
                         const float* d_final_state, void* dq, void* dk,
                         void* dv, float* d_log_alpha, float* d_beta,
                         float* d_initial_state, cudaStream_t stream) {
  int n_seqs = 0;
  kda_status st = validate_chunk_shape(shape, cu_seqlens != nullptr, &n_seqs);
  if (st != KDA_OK) return st;
  const size_t esz = shape->io_dtype == KDA_BF16 ? 2 : 4;
  const size_t tokens = (size_t)shape->B * (size_t)shape->T;
  const size_t H = shape->H, dkk = shape->dk, dvv = shape->dv;
  if (tokens > 0 && (!q || !k || !v || !log_alpha || !beta || !d_out || !dq ||
                     !dk || !dv || !d_log_alpha || !d_beta))
    return KDA_ERR_INVALID_ARG;
  const void* p16[] = {q, k, v, initial_state, d_out, d_final_state, dq, dk,
                       dv, d_initial_state};
  for (const void* p : p16)
    if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
  const void* p4[] = {log_alpha, beta, cu_seqlens, d_log_alpha, d_beta};
  for (const void* p : p4)
    if (p && !aligned4(p)) return KDA_ERR_MISALIGNED;
  // No output may overlap an input or another output.
  const size_t sbytes = (size_t)n_seqs * H * dkk * dvv * 4;
  const Range ins[] = {span(q, tokens * H * dkk * esz),
                       span(k, tokens * H * dkk * esz),
                       span(v, tokens * H * dvv * esz),
                       span(log_alpha, tokens * H * dkk * 4),
                       span(beta, tokens * H * 4),
                       span(initial_state, sbytes),
                       span(cu_seqlens, cu_seqlens ? 4 * ((size_t)n_seqs + 1) : 0),
                       span(d_out, tokens * H * dvv * esz),
                       span(d_final_state, sbytes)};
  const Range outs[] = {span(dq, tokens * H * dkk * esz),
                        span(dk, tokens * H * dkk * esz),
                        span(dv, tokens * H * dvv * esz),
                        span(d_log_alpha, tokens * H * dkk * 4),
                        span(d_beta, tokens * H * 4),
                        span(d_initial_state, sbytes)};
  for (size_t i = 0; i < 6; ++i) {
    for (const Range& r : ins)
      if (overlap(outs[i], r)) return KDA_ERR_INVALID_ARG;
    for (size_t j = i + 1; j < 6; ++j)
      if (overlap(outs[i], outs[j])) return KDA_ERR_INVALID_ARG;
  }
  kda::BwdArgs b{};
  b.f.q = q;
  b.f.k = k;
  b.f.v = v;
  b.f.log_alpha = log_alpha;
  b.f.beta = beta;
  b.f.initial_state = initial_state;
  b.f.cu_seqlens = cu_seqlens;
  fill_args(shape, n_seqs, &b.f);
  b.d_out = d_out;
  b.d_final_state = d_final_state;
  b.dq = dq;
  b.dk = dk;
  b.dv = dv;
  b.d_log_alpha = d_log_alpha;
  b.d_beta = d_beta;
  b.d_initial_state = d_initial_state;
  void* ws = nullptr;
  cudaError_t e;
  const size_t bytes = kda::bwd_workspace_bytes(b);
  if ((e = take_workspace(bytes, stream, &ws)) != cudaSuccess) {
    if (ws) cudaFreeAsync(ws, stream);
    return cuda_fail(e);
  }
  e = kda::launch_bwd(b, ws, stream);
  if (ws) {
    const cudaError_t f = cudaFreeAsync(ws, stream);
    if (e == cudaSuccess) e = f;
  }
  return e == cudaSuccess ? KDA_OK : cuda_fail(e);
}

kda_status kda_chunk_bwd_plan(const kda_shape* shape, int packed, int* kernels,
                              size_t* workspace_bytes) {
  int n_seqs = 0;
  const kda_status st = validate_chunk_shape(shape, packed != 0, &n_seqs);
  if (st != KDA_OK) return st;
  kda::BwdArgs b{};
  fill_args(shape, n_seqs, &b.f);
  static const int32_t kTag = 0;  // only tells the planner the layout
  b.f.cu_seqlens = packed ? &kTag : nullptr;
  if (kernels) *kernels = kda::bwd_kernel_count(b);
  if (workspace_bytes) *workspace_bytes = kda::bwd_workspace_bytes(b);
  return KDA_OK;
}

kda_status kda_chunk_bwd_layout(const kda_shape* shape, int packed, int cap,
                                size_t* offsets, size_t* sizes,
                                int* first_launch, int* last_launch,
                                int* count) {
  if (!count || cap < 0) return KDA_ERR_INVALID_ARG;
  if (cap > 0 && (!offsets || !sizes || !first_launch || !last_launch))
    return KDA_ERR_INVALID_ARG;
  int n_seqs = 0;
  const kda_status st = validate_chunk_shape(shape, packed != 0, &n_seqs);
  if (st != KDA_OK) return st;
  kda::BwdArgs b{};
  fill_args(shape, n_seqs, &b.f);
  static const int32_t kTag = 0;  // only tells the planner the layout
  b.f.cu_seqlens = packed ? &kTag : nullptr;
  kda::BwdArray arr[64];
  const int n = kda::bwd_workspace_layout(b, arr, 64);
  for (int i = 0; i < n && i < cap && i < 64; ++i) {
    offsets[i] = arr[i].offset;
    sizes[i] = arr[i].bytes;
    first_launch[i] = arr[i].first;
    last_launch[i] = arr[i].last;
  }
  *count = n;
  return KDA_OK;
}

kda_status kda_chunk_fwd_gated(const kda_shape* shape, int gate, const void* q,
                               const void* k, const void* v,
                               const float* log_gate, const float* beta,
                               const float* initial_state,
                               const int32_t* cu_seqlens, void* out,
                               float* final_state, int staged,
                               cudaStream_t stream) {
  kda::ChunkArgs a{};
  const kda_status st = validate_chunk(shape, q, k, v, log_gate, beta,
                                       initial_state, cu_seqlens, out,
                                       final_state, &a, gate);
  if (st != KDA_OK) return st;
  if (!staged && kda::fused_supported(a))
    return run_with_workspace(kda::twopass_workspace_bytes(a), stream, Path::kTwoPass, a);
  return run_with_workspace(kda::staged_workspace_bytes(a), stream, Path::kStaged, a);
}

}  // extern "C"

namespace {
bool set_prologue(const kda_prologue* p, kda::Prologue* out) {
  if (!p) return true;
  if (!(p->q_scale == p->q_scale) || !(p->gate_scale == p->gate_scale))
    return false;  // NaN scales
  out->norm_qk = p->normalize_qk != 0;
  out->q_scale = p->q_scale;
  out->gate_logits = p->gate_logits != 0;
  out->gate_scale = p->gate_scale;
  return true;
}
}  // namespace

extern "C" {

kda_status kda_chunk_fwd_ex(const kda_shape* shape, int gate,
                            const kda_prologue* prologue, const void* q,
                            const void* k, const void* v,
                            const float* gate_tensor, const float* beta,
                            const float* initial_state,
                            const int32_t* cu_seqlens, void* out,
                            float* final_state, int staged,
                            cudaStream_t stream) {
  kda::ChunkArgs a{};
  const kda_status st = validate_chunk(shape, q, k, v, gate_tensor, beta,
                                       initial_state, cu_seqlens, out,
                                       final_state, &a, gate);
  if (st != KDA_OK) return st;
  if (!set_prologue(prologue, &a.pro)) return KDA_ERR_INVALID_ARG;
  if (!staged && kda::fused_supported(a))
    return run_with_workspace(kda::twopass_workspace_bytes(a), stream, Path::kTwoPass, a);
  return run_with_workspace(kda::staged_workspace_bytes(a), stream, Path::kStaged, a);
}

kda_status kda_chunk_fwd_twopass(const kda_shape* shape, int gate,
                                 const kda_prologue* prologue, const void* q,
                                 const void* k, const void* v,
                                 const float* gate_tensor, const float* beta,
                                 const float* initial_state,
                                 const int32_t* cu_seqlens, void* out,
                                 float* final_state, cudaStream_t stream) {
  kda::ChunkArgs a{};
  const kda_status st = validate_chunk(shape, q, k, v, gate_tensor, beta,
                                       initial_state, cu_seqlens, out,
                                       final_state, &a, gate);
  if (st != KDA_OK) return st;
  if (!set_prologue(prologue, &a.pro)) return KDA_ERR_INVALID_ARG;
  if (!kda::fused_supported(a)) {
    // nothing to do for an empty request; other shapes are unsupported here
    if (a.bf16 && a.chunk == 64 && (a.dk == 64 || a.dk == 128) &&
        (a.dv == 64 || a.dv == 128))
      return run_with_workspace(kda::staged_workspace_bytes(a), stream,
                                Path::kStaged, a);
    return KDA_ERR_UNSUPPORTED;
  }
  return run_with_workspace(kda::twopass_workspace_bytes(a), stream,
                            Path::kTwoPass, a);
}

kda_status kda_chunk_fwd_paired(const kda_shape* shape, int gate,
                                const kda_prologue* prologue, const void* q,
                                const void* k, const void* v,
                                const float* gate_tensor, const float* beta,
                                const float* initial_state,
                                const int32_t* cu_seqlens, void* out,
                                float* final_state, cudaStream_t stream) {
  kda::ChunkArgs a{};
  const kda_status st = validate_chunk(shape, q, k, v, gate_tensor, beta,
                                       initial_state, cu_seqlens, out,
                                       final_state, &a, gate);
  if (st != KDA_OK) return st;
  if (!set_prologue(prologue, &a.pro)) return KDA_ERR_INVALID_ARG;
  if (!kda::fused_supported(a)) {
    if (a.bf16 && a.chunk == 64 && (a.dk == 64 || a.dk == 128) &&
        (a.dv == 64 || a.dv == 128))
      return run_with_workspace(kda::staged_workspace_bytes(a), stream,
                                Path::kStaged, a);
    return KDA_ERR_UNSUPPORTED;
  }
  return run_with_workspace(kda::fused_workspace_bytes(a), stream,
                            Path::kFused, a);
}

kda_status kda_chunk_fwd_staged_noalloc(
    const kda_shape* shape, const void* q, const void* k, const void* v,
    const float* log_alpha, const float* beta, const float* initial_state,
    const int32_t* cu_seqlens, void* out, float* final_state,
    cudaStream_t stream) {
  kda::ChunkArgs a{};
  const kda_status st = validate_chunk(shape, q, k, v, log_alpha, beta,
                                       initial_state, cu_seqlens, out,
                                       final_state, &a);
  if (st != KDA_OK) return st;
  // Too large for the fixed array: refuse before touching the device.
  if (kda::staged_workspace_bytes(a) > (size_t)KDA_NOALLOC_SCRATCH_BYTES)
    return KDA_ERR_UNSUPPORTED;
  cudaError_t e = cudaSuccess;
  void* ws = noalloc_scratch(&e);
  if (!ws) return cuda_fail(e);
  e = kda::launch_staged(a, ws, stream);
  return e == cudaSuccess ? KDA_OK : cuda_fail(e);
}

kda_status kda_recurrent_step(const kda_shape* s, const void* q, const void* k,
                              const void* v, const float* log_alpha,
                              const float* beta, float* state_inout, void* out,
                              cudaStream_t stream) {
  return kda_recurrent_step_gated(s, KDA_GATE_CHANNEL, q, k, v, log_alpha,
                                  beta, state_inout, out, stream);
}

kda_status kda_recurrent_step_gated(const kda_shape* s, int gate, const void* q,
                                    const void* k, const void* v,
                                    const float* log_alpha, const float* beta,
                                    float* state_inout, void* out,
                                    cudaStream_t stream) {
  return kda_recurrent_step_ex(s, gate, nullptr, q, k, v, log_alpha, beta,
                               state_inout, out, stream);
}

kda_status kda_recurrent_step_ex(const kda_shape* s, int gate,
                                 const kda_prologue* prologue, const void* q,
                                 const void* k, const void* v,
                                 const float* log_alpha, const float* beta,
                                 float* state_inout, void* out,
                                 cudaStream_t stream) {
  if (!s) return KDA_ERR_INVALID_ARG;
  kda::Prologue pro;
  if (!set_prologue(prologue, &pro)) return KDA_ERR_INVALID_ARG;
  if (gate != KDA_GATE_CHANNEL && gate != KDA_GATE_HEAD && gate != KDA_GATE_NONE)
    return KDA_ERR_INVALID_ARG;
  if (gate == KDA_GATE_NONE) log_alpha = nullptr;
  if (s->B < 0 || s->T < 0 || s->H < 1) return KDA_ERR_INVALID_ARG;
  if (s->io_dtype != KDA_BF16 && s->io_dtype != KDA_F32)
    return KDA_ERR_INVALID_ARG;
  if (!supported_dim(s->dk) || !supported_dim(s->dv)) return KDA_ERR_UNSUPPORTED;
  const size_t esz = s->io_dtype == KDA_BF16 ? 2 : 4;
  const size_t tokens = (size_t)s->B * (size_t)s->T, H = s->H;
  if ((size_t)s->B * H > (size_t)INT32_MAX) return KDA_ERR_UNSUPPORTED;
  if (s->B > 0 && !state_inout) return KDA_ERR_INVALID_ARG;
  if (tokens > 0 && (!q || !k || !v || !beta || !out)) return KDA_ERR_INVALID_ARG;
  if (tokens > 0 && gate != KDA_GATE_NONE && !log_alpha)
    return KDA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, state_inout, out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return KDA_ERR_MISALIGNED;
  if (log_alpha && !(gate == KDA_GATE_CHANNEL ? aligned16(log_alpha)
                                               : aligned4(log_alpha)))
    return KDA_ERR_MISALIGNED;
  if (beta && !aligned4(beta)) return KDA_ERR_MISALIGNED;
  const Range rq = span(q, tokens * H * s->dk * esz),
              rk = span(k, tokens * H * s->dk * esz),
              rv = span(v, tokens * H * s->dv * esz),
              rl = span(log_alpha,
                        tokens * H * (gate == KDA_GATE_CHANNEL ? s->dk : 1) * 4),
              rb = span(beta, tokens * H * 4),
              ro = span(out, tokens * H * s->dv * esz),
              rs = span(state_inout, (size_t)s->B * H * s->dk * s->dv * 4);
  for (Range r : {rq, rk, rv, rl, rb, rs})
    if (tokens > 0 && overlap(ro, r)) return KDA_ERR_INVALID_ARG;
  for (Range r : {rq, rk, rv, rl, rb})
    if (s->B > 0 && overlap(rs, r)) return KDA_ERR_INVALID_ARG;

  kda::RecurrentArgs a{q, k, v, log_alpha, beta, state_inout, out,
                       s->B, s->T, s->H, s->dk, s->dv,
                       s->io_dtype == KDA_BF16, gate, pro};
  const cudaError_t e = kda::launch_recurrent(a, stream);
  return e == cudaSuccess ? KDA_OK : cuda_fail(e);
}

kda_status kda_chunk_fwd_plan(const kda_shape* shape, int packed, int staged,
                              int* path, int* kernels,
                              size_t* workspace_bytes) {
  int n_seqs = 0;
  const kda_status st = validate_chunk_shape(shape, packed != 0, &n_seqs);
  if (st != KDA_OK) return st;
  kda::ChunkArgs a{};
  fill_args(shape, n_seqs, &a);
  a.cu_seqlens = packed ? reinterpret_cast<const int32_t*>(16) : nullptr;
  const bool tc = !staged && kda::fused_supported(a);
  if (path) *path = tc ? 2 : 0;
  if (kernels) *kernels = tc ? kda::twopass_kernel_count(a)
                             : kda::staged_kernel_count(a);
  if (workspace_bytes)
    *workspace_bytes = tc ? kda::twopass_workspace_bytes(a)
                          : kda::staged_workspace_bytes(a);
  return KDA_OK;
}

const char* kda_status_string(kda_status status) {
  switch (status) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG: invalid argument";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: unsupported size";
    case KDA_ERR_MISALIGNED: return "KDA_ERR_MISALIGNED: pointer not 16-byte aligned";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA: a CUDA call failed";
    case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: a bounded device wait gave up";
    case KDA_ERR_RANGE:
      return "KDA_ERR_RANGE: a chunk's decay exceeded the supported range";
  }
  return "unknown kda_status";
}

kda_status kda_device_status(cudaStream_t stream) {
  int flag = 0, split_flag = 0, range_fused = 0, range_staged = 0,
      range_bwd = 0, bwd_flag = 0;
  cudaError_t e = kda::fused_take_timeout(stream, &flag);
  if (e == cudaSuccess) e = kda::split_take_timeout(stream, &split_flag);
  if (e == cudaSuccess) e = kda::fused_take_range(stream, &range_fused);
  if (e == cudaSuccess) e = kda::staged_take_range(stream, &range_staged);
  if (e == cudaSuccess) e = kda::bwd_take_range(stream, &range_bwd);
  if (e == cudaSuccess) e = kda::bwd_take_timeout(stream, &bwd_flag);
  if (e != cudaSuccess) return cuda_fail(e);
  if (flag || split_flag || bwd_flag) return KDA_ERR_TIMEOUT;
  return range_fused || range_staged || range_bwd ? KDA_ERR_RANGE : KDA_OK;
}

kda_status kda_selftest_timeout(int limit_us, cudaStream_t stream) {
  if (limit_us < 1 || limit_us > 100000) return KDA_ERR_INVALID_ARG;
  const cudaError_t e = kda::launch_timeout_probe(limit_us, stream);
  return e == cudaSuccess ? KDA_OK : cuda_fail(e);
}

kda_status kda_workspace_pool(size_t* reserved_bytes, size_t* used_bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  keep_pool_memory();
  cudaMemPool_t pool;
  if ((e = cudaDeviceGetDefaultMemPool(&pool, dev)) != cudaSuccess)
    return cuda_fail(e);
  uint64_t v = 0;
  if (reserved_bytes) {
    if ((e = cudaMemPoolGetAttribute(pool, cudaMemPoolAttrReservedMemCurrent,
                                     &v)) != cudaSuccess)
      return cuda_fail(e);
    *reserved_bytes = (size_t)v;
  }
  if (used_bytes) {
    if ((e = cudaMemPoolGetAttribute(pool, cudaMemPoolAttrUsedMemCurrent, &v)) !=
        cudaSuccess)
      return cuda_fail(e);
    *used_bytes = (size_t)v;
  }
  return KDA_OK;
}

kda_status kda_profile_pass_event(void* event) {
  kda::set_pass_event(static_cast<cudaEvent_t>(event));
  return KDA_OK;
}

int kda_last_cuda_error(void) { return g_last_cuda_error; }

int kda_version(void) { return 100; }

}  // extern "C"
