// Internal launch interface between the C-ABI layer (kda_api.cu) and the
// kernel files.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace kda {

// Forget-gate layouts: one log(alpha) per key channel (KDA), one per head
// (Gated DeltaNet), or none (alpha = 1, DeltaNet).
enum GateMode { kGateChannel = 0, kGateHead = 1, kGateNone = 2 };

// Optional input prologue applied inside the kernels: per-token L2
// normalisation of q and k over d_k, a scale on q, and log(alpha) formed as
// gate_scale * logsigmoid(x) from raw gate logits x.
struct Prologue {
  bool norm_qk = false;
  float q_scale = 1.f;
  bool gate_logits = false;
  float gate_scale = 1.f;
};

struct RecurrentArgs {
  const void* q;
  const void* k;
  const void* v;
  const float* log_alpha;
  const float* beta;
  float* state;
  void* out;
  int B, T, H, dk, dv;
  bool bf16;
  int gate = kGateChannel;
  Prologue pro;
};

struct ChunkArgs {
  const void* q;
  const void* k;
  const void* v;
  const float* log_alpha;
  const float* beta;
  const float* initial_state;  // may be null
  const int32_t* cu_seqlens;   // may be null (dense layout)
  void* out;
  float* final_state;
  int n_seqs;  // B for the dense layout
  int T;       // tokens per sequence (dense) or total tokens (packed)
  int H, dk, dv, chunk;
  bool bf16;
  int gate = kGateChannel;
  Prologue pro;
};

// Token-by-token evaluation (kda_decode.cu).
cudaError_t launch_recurrent(const RecurrentArgs& a, cudaStream_t stream);

// Four-stage fp32 pipeline (kda_staged.cu).  `workspace` must hold
// staged_workspace_bytes(a) bytes, 256-byte aligned.
size_t staged_workspace_bytes(const ChunkArgs& a);
int staged_kernel_count(const ChunkArgs& a);
cudaError_t launch_staged(const ChunkArgs& a, void* workspace,
                          cudaStream_t stream);
// The staged pipeline's pieces the backward pass wraps around its own
// per-chunk preparation.  With state_pass false: the packed-layout chunk
// offsets and g = cumulative log-decay [tokens, H, dk].  The caller then
// writes W [tokens, H, dk] into view->w, U [tokens, H, dv] into view->d and
// Kh = k exp(g_C - g) [tokens, H, dk] (g_C: g at the chunk's last token)
// into view->kh.
// With state_pass true: the serial state pass, which turns U into
// Delta = U - W S_0 in place, stores every chunk-start state
// [max_chunks, H, dk, dv] in view->s and the final state in a.final_state.
// All fp32; channel gate, no prologue.  With state_pass false only the first
// staged_prefix_bytes(a) bytes of the workspace are touched (the chunk
// offsets and g); view->w, d, kh and s then point past them.
struct StagedView {
  const int32_t* chunk_off;
  const float* g;
  float* w;
  float* d;
  float* kh;
  const float* s;
};
cudaError_t launch_staged_part(const ChunkArgs& a, void* workspace,
                               StagedView* view, bool state_pass,
                               cudaStream_t stream);
size_t staged_prefix_bytes(const ChunkArgs& a);

// Sequence-split prefill of one long sequence (kda_split.cu): k segments of
// Ls tokens (a multiple of the chunk; the last one takes the rest) evaluated
// side by side and joined by a scan of their state transitions.  k = 1 is
// the plain chunkwise forward.  `a` is a dense single-sequence request
// (n_seqs = 1, no cu_seqlens).
struct SplitGeom {
  int Ls;
  int k;
};
SplitGeom split_geometry(const ChunkArgs& a, int n_segments);
// The segment count the call picks when asked for none: the largest k whose
// 2k - 1 concurrent chains (k value, k - 1 transition) fit on num_sms SMs.
int split_auto_segments(const ChunkArgs& a, int num_sms);
size_t split_workspace_bytes(const ChunkArgs& a, const SplitGeom& g);
int split_kernel_count(const ChunkArgs& a, const SplitGeom& g);
cudaError_t launch_split(const ChunkArgs& a, const SplitGeom& g, void* workspace,
                         cudaStream_t stream);

// The backward pass's reverse state-gradient chain on the tensor cores
// (kda_bwd_chain_tc.cuh, tf32 products): 64-token chunks, d_k and d_v in
// {64, 128}.  Inputs and outputs are the backward workspace's fp32 arrays;
// wt is W transposed per chunk, [chunks, H, d_k, 64] with zero columns past
// each chunk's last token.
struct RevChainArgs {
  const float* kb;       // Kb [tokens, H, dk]
  const float* wt;       // W^T [chunks, H, dk, 64]
  const float* qdo;      // Qt^T dO [chunks, H, dk, dv]
  const float* pdo;      // P^T dO [tokens, H, dv]
  const float* s;        // chunk-start states [chunks, H, dk, dv]
  const float* fin;      // final states [n_seqs, H, dk, dv]
  const float* gam;      // exp(g_C) [chunks, H, dk]
  const float* d_final;  // or null
  float* gst;            // G out [chunks, H, dk, dv]
  float* dd;             // dDelta out [tokens, H, dv]
  float* dgam;           // gam * d gam partials [chunks, H, dv / 32, dk]
  float* ddT;            // -dDelta^T per chunk [chunks, H, dv, 64], or null
  float* d_init;         // or null
  const int32_t* cu;
  const int32_t* chunk_off;
  int n_seqs, T, H, dk, dv;
  int64_t n_chunks;
};
cudaError_t launch_rev_chain_tc(const RevChainArgs& a, cudaStream_t stream);

// The backward pass's copy of the forward's state pass on the tensor cores
// (kda_bwd_chain_tc.cuh): Delta = U - W S over u in place, every chunk-start
// state into s, the final state into s_final; W and Kh^T rounded to tf32 by
// prep, S and Delta split into tf32 high part and remainder.
struct StateChainArgs {
  const float* w;        // W [tokens, H, dk]
  float* u;              // U in, Delta out [tokens, H, dv]
  const float* khT;      // Kh^T per chunk [chunks, H, dk, 64]
  const float* gam;      // exp(g_C) [chunks, H, dk]
  float* s;              // chunk-start states [chunks, H, dk, dv]
  const float* s_init;   // [n_seqs, H, dk, dv] or null
  float* s_final;        // [n_seqs, H, dk, dv]
  const int32_t* cu;
  const int32_t* chunk_off;
  int n_seqs, T, H, dk, dv;
  int64_t n_chunks;
};
cudaError_t launch_state_chain_tc(const StateChainArgs& a, cudaStream_t stream);

// Chunkwise backward pass (kda_backward.cu): the gradients of
// L = <d_out, out> + <d_final_state, final_state> with respect to q, k, v,
// log(alpha), beta and the initial state, in fp32 arithmetic (with bf16
// inputs in 64-token chunks every product runs on the tensor cores in tf32).
struct BwdArgs {
  ChunkArgs f;                  // forward arguments; f.out, f.final_state unused
  const void* d_out;            // [tokens, H, dv], io dtype
  const float* d_final_state;   // [n_seqs, H, dk, dv] or null (zero)
  void* dq;                     // [tokens, H, dk], io dtype
  void* dk;                     // [tokens, H, dk], io dtype
  void* dv;                     // [tokens, H, dv], io dtype
  float* d_log_alpha;           // [tokens, H, dk]
  float* d_beta;                // [tokens, H]
  float* d_initial_state;       // [n_seqs, H, dk, dv] or null (not wanted)
};
size_t bwd_workspace_bytes(const BwdArgs& a);
int bwd_kernel_count(const BwdArgs& a);
// One array of the backward's workspace: its byte offset and size, and the
// first and last launch of the call (in launch order) that touch it.
struct BwdArray {
  size_t offset, bytes;
  int first, last;
};
// The arrays of a backward call's workspace, the first `cap` of them into
// `out`; returns how many there are: 0 on the fp32 path, whose arrays never
// share memory.
int bwd_workspace_layout(const BwdArgs& a, BwdArray* out, int cap);
cudaError_t launch_bwd(const BwdArgs& a, void* workspace, cudaStream_t stream);

// Fused tensor-core prefill (kda_fused_sm100.cu): bf16 io, dk, dv in
// {64, 128}, chunk 64.  `workspace` must hold fused_workspace_bytes(a).
bool fused_supported(const ChunkArgs& a);
size_t fused_workspace_bytes(const ChunkArgs& a);
int fused_kernel_count(const ChunkArgs& a);
// Synchronises `stream`, then reads and clears the flag a fused kernel sets
// when one of its bounded waits gave up.
cudaError_t fused_take_timeout(cudaStream_t stream, int* flag);
// The same for the sequence split's tensor-core correction (kda_split.cu).
cudaError_t split_take_timeout(cudaStream_t stream, int* flag);
// Synchronises `stream`, then reads and clears the flag a chunkwise kernel
// sets when a chunk's total log-decay on some channel exceeds
// kDecayRangeMax (the fused kernels, the four-stage pipeline and the
// backward pass each keep their own).
cudaError_t fused_take_range(cudaStream_t stream, int* flag);
cudaError_t staged_take_range(cudaStream_t stream, int* flag);
cudaError_t bwd_take_range(cudaStream_t stream, int* flag);
cudaError_t bwd_take_timeout(cudaStream_t stream, int* flag);
// Diagnostic: one CTA whose bounded wait runs out after limit_us.
cudaError_t launch_timeout_probe(int limit_us, cudaStream_t stream);
cudaError_t launch_fused(const ChunkArgs& a, void* workspace,
                         cudaStream_t stream);
// Two-pass tensor-core prefill (kda_twopass_sm100.cuh, in the fused
// translation unit): a parallel factorisation pass writing one package per
// (chunk, head) into `workspace`, then the chain kernel.  Same shapes as the
// fused kernel.
size_t twopass_workspace_bytes(const ChunkArgs& a);
int twopass_kernel_count(const ChunkArgs& a);
cudaError_t launch_twopass(const ChunkArgs& a, void* workspace,
                           cudaStream_t stream,
                           cudaEvent_t factor_done = nullptr);
// The chain kernel alone, over packages another call's factorisation pass
// wrote (the layouts must agree chunk for chunk from `packages` on): for a
// run whose q, k, log alpha and beta are a shifted copy of that call's.  Its
// workspace holds only the packed layout's order and offsets.
size_t twopass_chain_workspace_bytes(const ChunkArgs& a);
int twopass_chain_kernel_count(const ChunkArgs& a);
cudaError_t launch_twopass_chain(const ChunkArgs& a, void* workspace,
                                 const void* packages, cudaStream_t stream);
// Where the package of chunk `first_chunk` (of a's layout) starts in a
// two-pass workspace.
const void* twopass_packages(const ChunkArgs& a, const void* workspace,
                             int64_t first_chunk);
// Profiling aid: an event the calling thread's two-pass launches record on
// their stream between the factorisation pass and the chain kernel (null:
// none).
void set_pass_event(cudaEvent_t e);
cudaEvent_t pass_event();

// Upper bound on the number of chunks of a request (packed sequences may each
// add one partial chunk).
inline int64_t max_chunks(const ChunkArgs& a) {
  const int64_t C = a.chunk;
  if (a.cu_seqlens == nullptr)
    return (int64_t)a.n_seqs * ((a.T + C - 1) / C);
  return (a.T + C - 1) / C + a.n_seqs;
}

}  // namespace kda
