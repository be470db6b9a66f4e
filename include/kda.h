/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention forward library.
 *
 * The operation (stated in this header's own words):
 *   Per (sequence, head) a state S in R^{d_k x d_v} is carried across tokens.
 *   For token t with query q_t, key k_t (in R^{d_k}), value v_t (in R^{d_v}),
 *   write rate beta_t and per-key-channel forget vector alpha_t = exp(l_t):
 *       S'  = Diag(alpha_t) S_{t-1}             decay each key channel (row)
 *       S_t = S' + beta_t k_t (v_t - S'^T k_t)^T delta-rule write of the error
 *       o_t = S_t^T q_t                          read with the query
 *   i.e. S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T.
 *   Sources: "Kimi Delta Attention" (akshathtiwari.co.in), the delta-rule and
 *   channel-wise gating passages; "The fourth layer remembers"
 *   (praveentn.live), section "What each kind of layer keeps"; "Teacher guide -
 *   Kimi Delta Attention", section 12.1 and the Misconceptions table.
 *   kda_chunk_fwd evaluates it chunkwise (the recurrence reorganised into
 *   matrix products, "You Could Have Come Up with Kimi Delta Attention",
 *   daily.dev, Summary); kda_recurrent_step evaluates it token by token with
 *   constant memory and work per token ("The fourth layer remembers", the
 *   paragraph after the forget gate).  Both give the same result up to
 *   floating-point rounding.
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE memory owned by the caller; the library
 *     never frees or retains them.  Calls are asynchronous on `stream` and never
 *     synchronise the host.  Temporary workspace, when a path needs it, is
 *     stream-ordered (cudaMallocAsync / cudaFreeAsync on `stream`).
 *   - Layouts are dense row-major:
 *       q, k       [B, T, H, d_k]   io dtype (bf16 or fp32)
 *       v, out     [B, T, H, d_v]   io dtype
 *       log_alpha  [B, T, H, d_k]   fp32, l = log(alpha) <= 0 (no lower bound
 *                                   is applied; the caller forms the gate)
 *       beta       [B, T, H]        fp32
 *       states     [N, H, d_k, d_v] fp32, N = B (or n_seqs with cu_seqlens)
 *     q and k are used as given: any scaling or L2 normalisation is the
 *     caller's.
 *   - q, k, v, log_alpha, out and the states must be 16-byte aligned; beta
 *     and cu_seqlens 4-byte aligned (KDA_ERR_MISALIGNED otherwise).
 *   - `out` must not alias an input.  Argument errors are detected on the host
 *     before anything is launched; no exception crosses the ABI.
 *   - Supported sizes: d_k, d_v in {32, 64, 128}; chunk in {16, 32, 64}.
 *     Others return KDA_ERR_UNSUPPORTED.
 *   - Numerical range: the chunkwise path factorises the decay inside a
 *     chunk as exp(g_r - g_i) = exp(g_r - rho) exp(rho - g_i), with g the
 *     running sum of l inside the chunk.  Per key channel, rho is the chunk
 *     start while |g_C| (the channel's total log-decay over the chunk) is at
 *     most 60, and g_C / 2 above that, so no factor exceeds exp(|g_C| / 2).
 *     Results are exact up to rounding for |g_C| <= 160 on every channel of
 *     every chunk: for chunk 64, any gate with alpha >= 0.082 on every token
 *     qualifies (the pages' worked gate of 0.2 included).  A chunk beyond
 *     that makes the call's outputs unspecified and sets a device flag that
 *     kda_device_status reports as KDA_ERR_RANGE.  kda_recurrent_step has no
 *     such limit.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KDA_OK = 0,
  KDA_ERR_INVALID_ARG = 1, /* null pointer, bad size, aliasing            */
  KDA_ERR_UNSUPPORTED = 2, /* valid request outside the supported sizes    */
  KDA_ERR_MISALIGNED = 3,  /* a pointer is not 16-byte aligned             */
  KDA_ERR_CUDA = 4,        /* a CUDA call failed; see kda_last_cuda_error  */
  KDA_ERR_TIMEOUT = 5,     /* a bounded device-side wait gave up           */
  KDA_ERR_RANGE = 6        /* a chunk's decay exceeded the supported range
                              (reported by kda_device_status)              */
} kda_status;

typedef enum { KDA_BF16 = 0, KDA_F32 = 1 } kda_dtype;

/* Layout of the forget gate's log(alpha) for the *_gated entry points. */
typedef enum {
  KDA_GATE_CHANNEL = 0, /* [B, T, H, d_k]: one per key channel (KDA)          */
  KDA_GATE_HEAD = 1,    /* [B, T, H]: one per head, all channels alike
                           (Gated DeltaNet)                                   */
  KDA_GATE_NONE = 2     /* no tensor, alpha = 1 (DeltaNet); pass NULL          */
} kda_gate;

typedef struct {
  int B;      /* batch (number of sequences when cu_seqlens is NULL; 1 with it) */
  int T;      /* tokens per sequence, or total packed tokens with cu_seqlens  */
  int H;      /* heads                                                          */
  int dk;     /* key / query head dimension                                     */
  int dv;     /* value head dimension                                           */
  int chunk;  /* chunk length C of the chunkwise evaluation (16, 32 or 64)      */
  int n_seqs; /* number of packed sequences (used only with cu_seqlens)         */
  kda_dtype io_dtype; /* dtype of q, k, v and out                               */
} kda_shape;

/*
 * kda_chunk_fwd -- chunkwise prefill over whole sequences.
 *
 *   q, k, v, log_alpha, beta : inputs, layouts above.
 *   initial_state : [N, H, d_k, d_v] fp32 start state, or NULL for zeros.
 *   cu_seqlens    : NULL for the dense [B, T, ...] layout.  Otherwise int32
 *                   device array of n_seqs + 1 token offsets into the packed
 *                   token axis (B must be 1, T the total): sequence s owns tokens
 *                   cu_seqlens[s] .. cu_seqlens[s+1]-1.  It must start at 0, be
 *                   non-decreasing and end at T; it is device memory, so it is
 *                   not checked on the host: the kernels clamp every offset into
 *                   [0, T] (they stay in bounds), but results for a malformed
 *                   array are unspecified.  Chunks never straddle sequences;
 *                   a sequence's last chunk may be partial; empty sequences are
 *                   allowed (their final state is their initial state).
 *   out           : [B, T, H, d_v] io dtype, written.
 *   final_state   : [N, H, d_k, d_v] fp32, written (may equal initial_state).
 *
 * bf16 inputs with d_k, d_v in {64, 128} and chunk = 64 run the two-pass
 * tensor-core evaluation of kda_chunk_fwd_twopass (a factorisation pass over
 * every (chunk, head), then the serial chain; stream-ordered workspace of
 * one package per (chunk, head), see kda_chunk_fwd_plan); every other
 * supported request runs the four-stage kernel pipeline of
 * kda_chunk_fwd_staged.  fp32 state throughout.
 */
KDA_API kda_status kda_chunk_fwd(const kda_shape* shape, const void* q, const void* k,
                         const void* v, const float* log_alpha,
                         const float* beta, const float* initial_state,
                         const int32_t* cu_seqlens, void* out,
                         float* final_state, cudaStream_t stream);

/*
 * kda_chunk_fwd_staged -- same contract as kda_chunk_fwd, always evaluated as
 * four kernels with an intermediate workspace in HBM:
 *   (1) per-chunk cumulative log-decay g;  (2) intra-chunk factors: the
 *   decay-scaled strictly-lower matrix A, T = (I + A)^-1 by forward
 *   substitution, W = T Diag(beta) K~ and U = T Diag(beta) V;  (3) the
 *   inter-chunk state pass, sequential over chunks, parallel over
 *   (sequence, head, d_v tile);  (4) the output, q.S plus the masked
 *   intra-chunk q.k^T term.  All arithmetic is fp32 (the all-fp32 mode).
 * Workspace: about (2 d_k + d_v) * 4 bytes per token and head plus
 * d_k * d_v * 4 bytes per chunk and head, allocated stream-ordered.
 */
KDA_API kda_status kda_chunk_fwd_staged(const kda_shape* shape, const void* q,
                                const void* k, const void* v,
                                const float* log_alpha, const float* beta,
                                const float* initial_state,
                                const int32_t* cu_seqlens, void* out,
                                float* final_state, cudaStream_t stream);

/*
 * kda_chunk_fwd_gated -- kda_chunk_fwd with the forget gate in one of the
 * three layouts of kda_gate.  A channel-uniform gate is Gated DeltaNet, no
 * gate is DeltaNet; both are special cases of the same recurrence ("Kimi
 * Delta Attention", akshathtiwari.co.in: Gated DeltaNet's single per-head
 * gate, sharpened by KDA into one gate per channel; "The fourth layer
 * remembers": the earlier design's one decay number per head per token).
 * With KDA_GATE_HEAD / KDA_GATE_NONE the kernels read 4 bytes / nothing per
 * token and head instead of 4 d_k bytes and form one decay per row.
 *   gate     : a kda_gate value.
 *   log_gate : [B, T, H, d_k] (channel, 16-byte aligned), [B, T, H] (head,
 *              4-byte aligned) or NULL (none).
 *   staged   : nonzero forces the four-stage fp32 pipeline
 *              (kda_chunk_fwd_staged); zero picks as kda_chunk_fwd does.
 * Everything else as kda_chunk_fwd.
 */
KDA_API kda_status kda_chunk_fwd_gated(const kda_shape* shape, int gate,
                                       const void* q, const void* k,
                                       const void* v, const float* log_gate,
                                       const float* beta,
                                       const float* initial_state,
                                       const int32_t* cu_seqlens, void* out,
                                       float* final_state, int staged,
                                       cudaStream_t stream);

/* kda_recurrent_step with the forget gate in one of the kda_gate layouts
 * (see kda_chunk_fwd_gated); everything else as kda_recurrent_step. */
KDA_API kda_status kda_recurrent_step_gated(const kda_shape* shape, int gate,
                                            const void* q, const void* k,
                                            const void* v,
                                            const float* log_gate,
                                            const float* beta,
                                            float* state_inout, void* out,
                                            cudaStream_t stream);

/*
 * Optional input prologue for the *_ex entry points, applied inside the
 * kernels so the caller needs no separate pass over q, k and the gate:
 *   normalize_qk : nonzero -> q and k are L2-normalised per token and head
 *                  over d_k (in fp32) before use.
 *   q_scale      : q is multiplied by q_scale after normalisation (1 = none).
 *   gate_logits  : nonzero -> the gate tensor holds raw logits x and
 *                  log(alpha) = gate_scale * logsigmoid(x); zero -> it holds
 *                  log(alpha) itself (gate_scale ignored).
 * The pages leave the gate's parameterisation open ("The fourth layer
 * remembers": a forget-gate module without a lower bound); logsigmoid of a
 * logit is the plainest reading of such a gate.  A NULL prologue means none.
 */
typedef struct {
  int normalize_qk;
  float q_scale;
  int gate_logits;
  float gate_scale;
} kda_prologue;

/* kda_chunk_fwd_gated with an optional input prologue (see kda_prologue). */
KDA_API kda_status kda_chunk_fwd_ex(const kda_shape* shape, int gate,
                                    const kda_prologue* prologue,
                                    const void* q, const void* k,
                                    const void* v, const float* gate_tensor,
                                    const float* beta,
                                    const float* initial_state,
                                    const int32_t* cu_seqlens, void* out,
                                    float* final_state, int staged,
                                    cudaStream_t stream);

/* kda_recurrent_step_gated with an optional input prologue. */
KDA_API kda_status kda_recurrent_step_ex(const kda_shape* shape, int gate,
                                         const kda_prologue* prologue,
                                         const void* q, const void* k,
                                         const void* v,
                                         const float* gate_tensor,
                                         const float* beta,
                                         float* state_inout, void* out,
                                         cudaStream_t stream);

/*
 * kda_chunk_fwd_twopass -- the chunkwise prefill of kda_chunk_fwd_ex
 * evaluated in two tensor-core passes instead of one fused kernel:
 *   (1) a factorisation pass over every (chunk, head) side by side (each CTA
 *       takes up to four of them in turn): the decay-scaled operands, A and
 *       P, T' = (I + A)^-1 Diag(beta) and W = T' K~ of every chunk, written
 *       to a workspace as one package per (chunk, head) (66,576 bytes at
 *       d_k = 128);
 *   (2) a chain kernel per (sequence, head, 64-column d_v tile) that reads
 *       the packages in order and runs only the serial state and output
 *       products, with the fp32 state in tensor memory.
 * Same arguments, layouts and results (up to rounding order) as
 * kda_chunk_fwd_ex without the `staged` flag.  bf16 io with d_k, d_v in
 * {64, 128} and chunk 64 only (KDA_ERR_UNSUPPORTED otherwise).  Workspace:
 * stream-ordered, max_chunks * H * 67,584 bytes at d_k = 128 (50,176 at
 * d_k = 64), plus the packed layout's order and chunk offsets.
 */
KDA_API kda_status kda_chunk_fwd_twopass(const kda_shape* shape, int gate,
                                         const kda_prologue* prologue,
                                         const void* q, const void* k,
                                         const void* v,
                                         const float* gate_tensor,
                                         const float* beta,
                                         const float* initial_state,
                                         const int32_t* cu_seqlens, void* out,
                                         float* final_state,
                                         cudaStream_t stream);

/*
 * kda_chunk_fwd_paired -- the same chunkwise prefill as kda_chunk_fwd_ex
 * (without its `staged` flag) in ONE tensor-core kernel and no workspace
 * (the packed layout needs 4 bytes per sequence for its longest-first
 * order): per (sequence, head) a cluster of two CTAs, one per 64-column
 * tile of d_v, that factorise alternate chunks and hand each chunk's
 * package to the other over distributed shared memory while each runs the
 * state chain of its own tile.  Slower than the two-pass default on every
 * measured shape (for example 0.67 ms against 0.52 ms for a B=2, T=8192,
 * H=32, d=128 layer on a B200); kept for callers that must not hold the
 * two-pass workspace.  bf16 io with d_k, d_v in {64, 128} and chunk
 * 64 (d_v = 64: one CTA per head); KDA_ERR_UNSUPPORTED otherwise.
 */
KDA_API kda_status kda_chunk_fwd_paired(const kda_shape* shape, int gate,
                                        const kda_prologue* prologue,
                                        const void* q, const void* k,
                                        const void* v,
                                        const float* gate_tensor,
                                        const float* beta,
                                        const float* initial_state,
                                        const int32_t* cu_seqlens, void* out,
                                        float* final_state,
                                        cudaStream_t stream);

/* Size in bytes of the fixed device scratch array behind
 * kda_chunk_fwd_staged_noalloc (16 MiB). */
#define KDA_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * kda_chunk_fwd_staged_noalloc -- kda_chunk_fwd_staged for callers that must
 * not allocate device memory.  (The pages have no counterpart of this entry
 * point: it is a deployment convenience of this library.)
 *
 * Who needs it: code whose device memory is owned and planned by someone
 * else.  Examples are a plugin run inside an inference engine that hands it
 * pre-planned buffers and forbids allocation in its execute path, a serving
 * loop that must never stall or fail on an allocator under memory pressure,
 * and a process whose HBM is already claimed by another caching allocator.
 * kda_chunk_fwd_staged allocates its workspace stream-ordered on every call,
 * which such callers cannot allow.
 *
 * What it does: exactly the kda_chunk_fwd_staged computation (same
 * arguments, layouts and results), with the workspace taken from one static
 * device array of KDA_NOALLOC_SCRATCH_BYTES that every GPU loading this library
 * holds until the process exits.  It calls no cudaMalloc, cudaFree or other
 * allocating routine.
 *   - Size limit: requests whose workspace (kda_chunk_fwd_plan with staged = 1
 *     reports it) exceeds KDA_NOALLOC_SCRATCH_BYTES return KDA_ERR_UNSUPPORTED
 *     before anything is launched.
 *   - First call on a device: it looks up the array's device address on the
 *     current device (cudaGetSymbolAddress) and caches it until the process
 *     exits.  Make that first call before any stream capture.  Resetting the
 *     device (cudaDeviceReset, or any teardown of its primary context)
 *     between calls is not supported: the cached address would be stale.
 *   - Sharing: every call on a device uses the same array, which keeps the
 *     last call's contents.  Nothing in it has to start at zero (each call
 *     writes every scratch byte before reading it).  Calls whose executions
 *     overlap on the GPU (different streams, or without ordering between
 *     them) race on the array and give wrong results: serialise them.
 */
KDA_API kda_status kda_chunk_fwd_staged_noalloc(
    const kda_shape* shape, const void* q, const void* k, const void* v,
    const float* log_alpha, const float* beta, const float* initial_state,
    const int32_t* cu_seqlens, void* out, float* final_state,
    cudaStream_t stream);

/*
 * kda_recurrent_step -- token-by-token evaluation (decode).
 *
 *   shape->B  : number of independent sequences; shape->T : tokens per
 *               sequence in this call (1 for one decode step; T > 1 runs T
 *               steps with the state kept on chip); shape->chunk and n_seqs
 *               are ignored; cu_seqlens is not supported here.
 *   q, k, v, log_alpha, beta : [B, T, H, ...] as above.
 *   state_inout : [B, H, d_k, d_v] fp32, read and overwritten in place.
 *   out         : [B, T, H, d_v] io dtype.
 * Streams each head's fp32 state through the SMs once per call.
 */
KDA_API kda_status kda_recurrent_step(const kda_shape* shape, const void* q,
                              const void* k, const void* v,
                              const float* log_alpha, const float* beta,
                              float* state_inout, void* out,
                              cudaStream_t stream);

/*
 * kda_chunk_fwd_plan -- how kda_chunk_fwd (staged = 0) or kda_chunk_fwd_staged
 * (staged = 1) would evaluate a request of this shape; launches nothing and
 * touches no device memory.
 *   packed          : nonzero when cu_seqlens will be passed.
 *   path            : out, 2 = two-pass tensor-core evaluation
 *                     (kda_chunk_fwd_twopass), 0 = four-stage fp32 pipeline
 *                     (may be NULL).
 *   kernels         : out, kernel launches one call makes (may be NULL).
 *   workspace_bytes : out, stream-ordered workspace one call allocates (may be
 *                     NULL).
 * Returns KDA_OK, or the status the call itself would return for this shape.
 */
KDA_API kda_status kda_chunk_fwd_plan(const kda_shape* shape, int packed,
                                      int staged, int* path, int* kernels,
                                      size_t* workspace_bytes);

/*
 * kda_selftest_umma -- diagnostic, not part of the forward pass: one
 * D[128 x N] = A[128 x K] * B[K x N] product (bf16 in, fp32 out) on the
 * tensor cores through the same shared-memory layouts (128-byte swizzle),
 * operand descriptors and TMEM read-back as the fused prefill kernel.
 *   a_mn = 0: A is [128, K] row-major (K-major); 1: A is [K, 128] (M-major).
 *   b_mn = 0: B is [N, K] row-major (K-major); 1: B is [K, N] (N-major).
 *   N, K in {64, 128}; panel_rows (>= K, multiple of 8, <= 256) is the row
 *   count of each M-/N-major shared-memory panel.  D is [128, N] row-major.
 * One CTA, asynchronous on `stream`; device pointers owned by the caller.
 */
KDA_API kda_status kda_selftest_umma(int a_mn, int b_mn, int N, int K,
                                     int panel_rows, const void* A,
                                     const void* B, float* D,
                                     cudaStream_t stream);

/* Human-readable name of a status code (static string, never NULL). */
KDA_API const char* kda_status_string(kda_status status);

/* Synchronises `stream` and reports whether any kernel of this library on
 * this device gave up a bounded device-side wait since the last call
 * (KDA_ERR_TIMEOUT), else whether a chunkwise call met a chunk whose decay
 * exceeded the supported range (KDA_ERR_RANGE, see "Numerical range"
 * above), else KDA_OK.  The flags are cleared.  The kernels never wait
 * without a time limit; a wait that runs out abandons the rest of that CTA's
 * work and leaves its outputs unspecified. */
KDA_API kda_status kda_device_status(cudaStream_t stream);

/* kda_chunk_bwd -- the backward pass of kda_chunk_fwd (per-key-channel gate,
 * no input prologue): for the scalar
 *     L = sum(d_out * out) + sum(d_final_state * final_state)
 * it writes dL/dq, dL/dk, dL/dv, dL/dlog_alpha, dL/dbeta and (when
 * d_initial_state is not NULL) dL/dinitial_state.  The gradient follows the
 * chunkwise factorisation of the forward ("You Could Have Come Up with Kimi
 * Delta Attention", daily.dev, Summary); the pages print no gradient, so it
 * is the chain rule applied to that factorisation, checked against an fp64
 * reverse-mode evaluation of the token recurrence.
 *
 * Arguments: shape, q, k, v, log_alpha, beta, initial_state (may be NULL =
 * zeros), cu_seqlens (may be NULL) exactly as for kda_chunk_fwd (shape's
 * chunk in {16, 32, 64}, dims in {32, 64, 128});
 *   d_out          [tokens, H, d_v]    io dtype, the gradient of out
 *   d_final_state  [n_seqs, H, d_k, d_v] fp32 or NULL (zero)
 *   dq, dk         [tokens, H, d_k]    io dtype (written)
 *   dv             [tokens, H, d_v]    io dtype (written)
 *   d_log_alpha    [tokens, H, d_k]    fp32 (written)
 *   d_beta         [tokens, H]         fp32 (written)
 *   d_initial_state [n_seqs, H, d_k, d_v] fp32 (written) or NULL.
 * All pointers are device pointers owned by the caller; io-dtype tensors and
 * states 16-byte aligned, the other fp32 tensors and cu_seqlens 4-byte
 * aligned (KDA_ERR_MISALIGNED otherwise).  No output may overlap an input or
 * another output (KDA_ERR_INVALID_ARG).  All arithmetic is fp32 except for
 * bf16 inputs with chunk 64 (d_k, d_v in {64, 128}): there every product
 * runs on the tensor cores in tf32 (10-bit mantissa, fp32 accumulation; the
 * forward's state pass with high and low tf32 parts of its state and Delta),
 * within the bf16 tolerance of 1e-2 relative L2 (a bounded wait that gives up is reported by kda_device_status as
 * KDA_ERR_TIMEOUT); the call
 * re-runs the forward's chunk stages and allocates its fp32 workspace from
 * the stream-ordered pool (kda_chunk_bwd_plan reports its size; on the
 * tensor-core path intermediates whose lifetimes do not overlap share
 * memory, about 5.3 GB at B=2, T=8192, H=32, d=128).  Stream
 * ordered: returns after queueing the kernels.
 * Numerical range: the backward keeps the chunk-start factorisation of the
 * decay, exact while |g_C| <= 80 on every channel of every chunk (g_C as
 * under "Numerical range" above); beyond that its outputs are unspecified
 * and kda_device_status reports KDA_ERR_RANGE. */
KDA_API kda_status kda_chunk_bwd(const kda_shape* shape, const void* q,
                                 const void* k, const void* v,
                                 const float* log_alpha, const float* beta,
                                 const float* initial_state,
                                 const int32_t* cu_seqlens, const void* d_out,
                                 const float* d_final_state, void* dq, void* dk,
                                 void* dv, float* d_log_alpha, float* d_beta,
                                 float* d_initial_state, cudaStream_t stream);

/* kda_chunk_bwd_plan -- kernels a kda_chunk_bwd call of this shape launches
 * and the workspace bytes it allocates; no device work.  `packed` selects the
 * cu_seqlens layout (then shape->n_seqs sequences). */
KDA_API kda_status kda_chunk_bwd_plan(const kda_shape* shape, int packed,
                                      int* kernels, size_t* workspace_bytes);

/* kda_chunk_bwd_layout -- how a kda_chunk_bwd call of this shape lays out its
 * workspace; no device work.  On the tensor-core path (bf16, chunk 64, d_k
 * and d_v in {64, 128}) the call's intermediate arrays share memory where
 * their lifetimes do not overlap.  For each array i < min(*count, cap) it
 * writes its byte offset in the workspace, its size in bytes, and the first
 * and last launch of the call (numbered in launch order) that touch it; two
 * arrays whose launch ranges overlap never share a byte.  *count receives
 * the number of arrays (0 on the fp32 path, whose arrays are all apart).
 *   shape, packed : as kda_chunk_bwd_plan.
 *   cap           : room in each output array (0: count only).
 *   offsets, sizes, first_launch, last_launch : host arrays of cap entries
 *                   (may be NULL when cap is 0).
 * KDA_ERR_INVALID_ARG for a NULL count, a negative cap, or NULL arrays with
 * cap > 0; shape errors as kda_chunk_bwd_plan. */
KDA_API kda_status kda_chunk_bwd_layout(const kda_shape* shape, int packed,
                                        int cap, size_t* offsets,
                                        size_t* sizes, int* first_launch,
                                        int* last_launch, int* count);

/*
 * kda_chunk_fwd_split -- the chunkwise prefill of ONE long sequence (dense
 * layout, shape->B == 1, no cu_seqlens), evaluated as n_segments segments
 * side by side instead of one serial chain of chunks, then joined by a scan
 * over the segments.
 *
 * Why it is exact: the state update is affine in the state ("Kimi Delta
 * Attention", akshathtiwari.co.in, the delta-rule passage).  Inside a segment
 * entered with state S_in, and with M_t the product of the token transitions
 * (I - beta k k^T) Diag(alpha) from the segment start to token t,
 *     S_t = M_t S_in + S_t|0,      o_t = o_t|0 + S_in^T (M_t^T q_t),
 * where |0 is the evaluation from a zero state.  M_t is the state of the same
 * recurrence run with v = 0 from the identity, and M_t^T q_t is its output.
 * The call:
 *   1. evaluates all segments at once as a packed batch: segment 0 from
 *      initial_state, the others from zero (outputs go to `out`);
 *   2. concurrently, on a second stream it joins before returning, evaluates
 *      segments 1..n-1 with v = 0, d_v = d_k and the identity as start state;
 *   3. scans: S_in(1) = S_end(0), S_in(j+1) = M_end(j) S_in(j) + S_end|0(j);
 *      the last step writes final_state;
 *   4. adds S_in(j)^T (M_t^T q_t) to the outputs of segments 1..n-1.
 * Steps 1 and 2 run the path kda_chunk_fwd picks for their shapes; on the
 * two-pass path step 2 runs only its chain kernel, over the packages step 1
 * wrote (a package does not depend on v).  Step 3
 * is fp32.  Step 4 runs on the tensor cores (bf16 operands, fp32
 * accumulation) for bf16 io with d_k, d_v in {64, 128}, and in fp32
 * otherwise.  Segments are ceil(chunks / n_segments) chunks long, rounded
 * up to a multiple of 128 tokens when step 4 runs on the tensor cores; the
 * last takes the rest, and fewer segments result when the rounding or the
 * chunk count leaves fewer.
 * With bf16 io, step 1's outputs, step 2's M_t^T q_t and step 4's S_in pass
 * through bf16: the result agrees with kda_chunk_fwd to the bf16 tolerance,
 * not bit for bit.
 *
 * When it pays: steps 1 and 2 run 2n - 1 chains of T/n tokens side by side,
 * so the call shortens the serial chain when one sequence leaves most SMs
 * idle (few heads).  When the GPU is already full, the extra work of step 2
 * makes it slower than kda_chunk_fwd.
 *
 * Arguments: as kda_chunk_fwd_gated with B = 1 and cu_seqlens = NULL, plus
 * n_segments in 0 .. 64.  1 runs kda_chunk_fwd_gated's evaluation.  0 picks
 * the count: the largest k whose 2k - 1 concurrent chains fit on the
 * device's SMs, each chain taking one CTA per head and 64 columns of the
 * wider of d_k and d_v (so H = 32, d = 128 is not split at all on a B200).
 * Errors: as kda_chunk_fwd_gated; B != 1 or n_segments out of range ->
 * KDA_ERR_INVALID_ARG.  Workspace: stream-ordered (kda_chunk_fwd_split_plan
 * reports it).  The call queues work on `stream` and on a library-owned
 * stream and makes `stream` wait for all of it.
 */
KDA_API kda_status kda_chunk_fwd_split(const kda_shape* shape, int gate,
                                       const void* q, const void* k,
                                       const void* v, const float* gate_tensor,
                                       const float* beta,
                                       const float* initial_state, void* out,
                                       float* final_state, int n_segments,
                                       cudaStream_t stream);

/* kda_chunk_fwd_split_plan -- the segments (after the reduction above), kernel
 * launches and workspace bytes of a kda_chunk_fwd_split call; no device
 * work.  num_sms stands in for the device's SM count when n_segments is 0
 * (it must then be >= 1; otherwise it is ignored).  Any out pointer may be
 * NULL. */
KDA_API kda_status kda_chunk_fwd_split_plan(const kda_shape* shape, int gate,
                                            int n_segments, int num_sms,
                                            int* segments, int* kernels,
                                            size_t* workspace_bytes);

/* kda_selftest_timeout -- diagnostic of the failure reporting, not part of
 * the forward pass: launches one CTA that waits on a device barrier nothing
 * completes, using the library's bounded wait with a limit of limit_us
 * microseconds (1 .. 100000).  The wait gives up, the CTA sets the device
 * status flag and exits normally (no fault, no hang), so the next
 * kda_device_status on this stream returns KDA_ERR_TIMEOUT. */
KDA_API kda_status kda_selftest_timeout(int limit_us, cudaStream_t stream);

/*
 * kda_workspace_pool -- where the stream-ordered workspace lives.  The
 * paths that need workspace (the four-stage pipeline, the packed layout's
 * longest-first order, the sequence split and the backward pass) take it
 * with cudaMallocAsync from the current device's default memory pool and
 * give it back with cudaFreeAsync on the same stream.  The library sets that
 * pool's release threshold to the maximum on first use, so freed workspace
 * stays cached in the pool: after the first call of a given size, repeated
 * calls reuse the pool's memory and reserve nothing new from the device.
 * Calls on different streams never share a workspace.  With the
 * environment variable KDA_WORKSPACE_FILL set to a byte value (0-255), each
 * call first fills its workspace with that byte (a test aid: no kernel may
 * read a place of it before writing it, so the results must not change).
 *   reserved_bytes : out, memory the pool currently holds (may be NULL).
 *   used_bytes     : out, memory of the pool in use right now (may be NULL).
 * Reads the current device's pool; launches nothing.
 */
KDA_API kda_status kda_workspace_pool(size_t* reserved_bytes,
                                      size_t* used_bytes);

/*
 * kda_profile_pass_event -- profiling aid for the two-pass prefill.  While
 * `event` (a cudaEvent_t created by the caller, passed as void*) is set, every
 * call made on this thread that runs the two-pass path (kda_chunk_fwd,
 * kda_chunk_fwd_gated, kda_chunk_fwd_ex and kda_chunk_fwd_twopass on the
 * bf16 shapes of the fused kernels, and the segment runs of
 * kda_chunk_fwd_split) records it on its stream between the factorisation
 * pass and the chain kernel, so that events recorded before and after the
 * call time the two passes apart.  NULL clears it.  The event stays owned by
 * the caller and must outlive the calls that record it.  Other paths ignore
 * it.  Always returns KDA_OK; a failed record surfaces as the call's
 * KDA_ERR_CUDA.
 */
KDA_API kda_status kda_profile_pass_event(void* event);

/* The cudaError_t value behind the most recent KDA_ERR_CUDA on this thread
 * (0 if none). */
KDA_API int kda_last_cuda_error(void);

/* Library version as major * 10000 + minor * 100 + patch. */
KDA_API int kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
