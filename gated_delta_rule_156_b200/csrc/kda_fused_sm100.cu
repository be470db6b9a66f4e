// Fused chunkwise KDA prefill for sm_100a: host side (tensor maps, the
// longest-first order of packed sequences, dispatch) and the device-side
// timeout flag.  The kernel itself is in kda_fused_ws_sm100.cuh, included
// below so that it shares this translation unit's flag and helpers.
//
// Per chunk of C = 64 tokens with chunk-start state S (rows = key channels):
//   g      = running sum of log(alpha) inside the chunk, per key channel
//   Kt     = k exp(g)   Qt = q exp(g)   Kb = k exp(-g)
//   MMA1   [Kt; Qt] . Kb^T                 -> A_raw (rows 0-63), QK (64-127)
//   A      = strictly_lower(Diag(beta) A_raw);  P = lower_incl(QK)
//   Tm     = (I + A)^-1  (recursive doubling on 16 x 16 blocks, fp32)
//   T'     = Tm Diag(beta)
//   MMA2   T' . [Kt | V]                    -> W = T' Kt, U = T' V
//   MMA3   [W; Qt] . S                      -> W S (rows 0-63), Qt S (64-127)
//   Delta  = U - W S
//   MMA4   S += Kb^T . Delta ; then S <- Diag(exp(g_C)) S
//   MMA5   P . Delta accumulated onto Qt S  -> O
// This is the recurrence S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1}
// + b_t k_t v_t^T, o_t = S_t^T q_t regrouped over chunks (the chunkwise,
// Diagonal-Plus-Low-Rank form: "Kimi Delta Attention", akshathtiwari.co.in;
// "You Could Have Come Up with Kimi Delta Attention", daily.dev, Summary).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_tmap.h"
#include "sm100_ptx.cuh"

namespace kda {

// Set by a kernel whose bounded wait gave up (read and cleared on the host).
__device__ int g_fused_timeout = 0;
// Set when a chunk's decay exceeds the factorisation's range (read and
// cleared on the host).
__device__ int g_fused_range = 0;

namespace {

constexpr int kC = 64;  // chunk length of the fused kernel

// Packed layout: order the sequences longest first so the long serial chains
// start in the first wave.  rank(i) = #{j : len_j > len_i or (len_j == len_i
// and j < i)}.  Identity order beyond 8192 sequences.
__global__ void order_kernel(const int32_t* __restrict__ cu, int n_seqs, int T,
                             int32_t* __restrict__ order) {
  for (int i = threadIdx.x; i < n_seqs; i += blockDim.x) {
    if (n_seqs > 8192) {
      order[i] = i;
      continue;
    }
    int a, b;
    seq_range(cu, i, T, &a, &b);
    const int li = b - a;
    int rank = 0;
    for (int j = 0; j < n_seqs; ++j) {
      int c, d;
      seq_range(cu, j, T, &c, &d);
      const int lj = d - c;
      rank += (lj > li) || (lj == li && j < i);
    }
    order[rank] = i;
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr,
                                cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 3-D map over a [tokens, H, d] tensor with box {inner, 1, 64 tokens}.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt,
              int esize, int d, int H, int tokens, int inner,
              CUtensorMapSwizzle sw) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)tokens};
  cuuint64_t strides[2] = {(cuuint64_t)d * esize, (cuuint64_t)H * d * esize};
  cuuint32_t box[3] = {(cuuint32_t)inner, 1, (cuuint32_t)kC};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// bf16 [tokens, H, d] tensor, box of 64 channels x 64 tokens, 128-byte swizzle.
bool make_tile_map(CUtensorMap* m, const void* base, int d, int H, int tokens) {
  return make_map(m, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, H, tokens, 64,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace kda

#include "kda_fused_ws_sm100.cuh"
#include "kda_fused_pair_sm100.cuh"
#include "kda_twopass_sm100.cuh"
#include "kda_bwd_chain_tc.cuh"

namespace kda {
namespace {

int64_t total_tokens(const ChunkArgs& a) {
  return a.cu_seqlens ? (int64_t)a.T : (int64_t)a.n_seqs * a.T;
}

}  // namespace

bool fused_supported(const ChunkArgs& a) {
  return a.bf16 && a.chunk == kC && (a.dk == 64 || a.dk == 128) &&
         (a.dv == 64 || a.dv == 128) && a.n_seqs > 0 && total_tokens(a) > 0;
}

size_t fused_workspace_bytes(const ChunkArgs& a) {
  return a.cu_seqlens ? (((size_t)a.n_seqs * 4 + 255) & ~size_t(255)) : 0;
}

int fused_kernel_count(const ChunkArgs& a) { return a.cu_seqlens ? 2 : 1; }

namespace {
// Waits on an mbarrier that nothing completes, with the same bounded wait the
// fused kernel uses; when the limit runs out it sets the device status flag
// and returns.  Exercises the timeout reporting without a fault or a hang.
__global__ void timeout_probe_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    sm100::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !sm100::mbar_wait(&bar, 0, limit_ns))
    atomicExch(&g_fused_timeout, 1);
  __syncthreads();
}
}  // namespace

cudaError_t launch_timeout_probe(int limit_us, cudaStream_t stream) {
  timeout_probe_kernel<<<1, 32, 0, stream>>>((uint64_t)limit_us * 1000ull);
  return cudaGetLastError();
}

cudaError_t fused_take_timeout(cudaStream_t stream, int* flag) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  int zero = 0;
  if ((e = cudaMemcpyFromSymbol(flag, g_fused_timeout, sizeof(int))) !=
      cudaSuccess)
    return e;
  return cudaMemcpyToSymbol(g_fused_timeout, &zero, sizeof(int));
}

cudaError_t fused_take_range(cudaStream_t stream, int* flag) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  int zero = 0;
  if ((e = cudaMemcpyFromSymbol(flag, g_fused_range, sizeof(int))) !=
      cudaSuccess)
    return e;
  return cudaMemcpyToSymbol(g_fused_range, &zero, sizeof(int));
}

size_t twopass_workspace_bytes(const ChunkArgs& a) {
  return twopass::workspace_bytes(a);
}

size_t twopass_chain_workspace_bytes(const ChunkArgs& a) {
  return twopass::workspace_bytes(a, true);
}

int twopass_chain_kernel_count(const ChunkArgs& a) {
  return a.cu_seqlens ? 3 : 1;
}

const void* twopass_packages(const ChunkArgs& a, const void* workspace,
                             int64_t first_chunk) {
  return twopass::packages_in(a, const_cast<void*>(workspace)) +
         (size_t)first_chunk * a.H * twopass::package_slot(a.dk);
}

int twopass_kernel_count(const ChunkArgs& a) { return a.cu_seqlens ? 4 : 2; }

namespace {
thread_local cudaEvent_t t_pass_event = nullptr;
}  // namespace
void set_pass_event(cudaEvent_t e) { t_pass_event = e; }
cudaEvent_t pass_event() { return t_pass_event; }

cudaError_t launch_twopass(const ChunkArgs& a, void* workspace,
                           cudaStream_t stream, cudaEvent_t factor_done) {
  return twopass::launch(a, workspace, stream, nullptr, factor_done);
}

cudaError_t launch_twopass_chain(const ChunkArgs& a, void* workspace,
                                 const void* packages, cudaStream_t stream) {
  return twopass::launch(a, workspace, stream,
                         static_cast<const uint8_t*>(packages), nullptr);
}

cudaError_t launch_fused(const ChunkArgs& a, void* workspace,
                         cudaStream_t stream) {
  const int32_t* order = nullptr;
  if (a.cu_seqlens) {
    int32_t* o = static_cast<int32_t*>(workspace);
    order_kernel<<<1, 1024, 0, stream>>>(a.cu_seqlens, a.n_seqs, a.T, o);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    order = o;
  }
  // d_v = 128: the two 64-column tiles of a head share the per-chunk
  // factorisation as a cluster pair; d_v = 64: one CTA per head.
  if (a.dv == 2 * ws::kDvt) return pair::launch_fused_pair(a, order, stream);
  return ws::launch_fused_ws(a, order, stream);
}

namespace {
// 2-D fp32 map over `rows` rows of `cols` floats, box of 32 columns x
// `box_rows` rows, 128-byte swizzle.
bool make_rows_map(CUtensorMap* m, const float* base, int64_t rows, int cols,
                   int box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 4};
  cuuint32_t box[2] = {32, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base),
             dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DK>
cudaError_t run_rev_chain_tc(const RevChainArgs& a, cudaStream_t stream) {
  using Lay = bwdtc::Layout<DK>;
  const int tokens = a.cu ? a.T : a.n_seqs * a.T;
  const int64_t crows = a.n_chunks * a.H * DK;
  const auto F32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
  bwdtc::Maps m;
  if (!make_map(&m.kb, a.kb, F32, 4, DK, a.H, tokens, 32, SW) ||
      !make_map(&m.pdo, a.pdo, F32, 4, a.dv, a.H, tokens, 32, SW) ||
      !make_map(&m.dd, a.dd, F32, 4, a.dv, a.H, tokens, 32, SW) ||
      !make_rows_map(&m.wt, a.wt, crows, 64, DK) ||
      !make_rows_map(&m.qdo, a.qdo, crows, a.dv, DK) ||
      !make_rows_map(&m.s, a.s, crows, a.dv, DK) ||
      !make_rows_map(&m.gst, a.gst, crows, a.dv, DK) ||
      !make_rows_map(&m.fin, a.fin, (int64_t)a.n_seqs * a.H * DK, a.dv, DK) ||
      (a.ddT && !make_rows_map(&m.ddt, a.ddT, a.n_chunks * a.H * a.dv, 64, 64)))
    return cudaErrorInvalidValue;
  bwdtc::Params p{a.gam, a.d_final, a.dd, a.dgam, a.d_init, a.cu,
                  a.chunk_off, a.n_seqs, a.T, a.H, a.dv, a.ddT ? 1 : 0};
  const size_t smem = Lay::bytes + 1024;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(bwdtc::rev_chain_kernel<DK>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem)) != cudaSuccess)
    return e;
  const unsigned grid = (unsigned)a.n_seqs * a.H * (a.dv / bwdtc::kTile);
  bwdtc::rev_chain_kernel<DK><<<grid, bwdtc::kThreads, smem, stream>>>(m, p);
  return cudaGetLastError();
}
}  // namespace

template <int DK>
cudaError_t run_state_chain_tc(const StateChainArgs& a, cudaStream_t stream) {
  using Lay = bwdtc::StateLayout<DK>;
  const int tokens = a.cu ? a.T : a.n_seqs * a.T;
  const int64_t crows = a.n_chunks * a.H * DK;
  const auto F32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
  bwdtc::StateMaps m;
  if (!make_map(&m.w, a.w, F32, 4, DK, a.H, tokens, 32, SW) ||
      !make_map(&m.u, a.u, F32, 4, a.dv, a.H, tokens, 32, SW) ||
      !make_rows_map(&m.kht, a.khT, crows, 64, DK) ||
      !make_rows_map(&m.s, a.s, crows, a.dv, DK))
    return cudaErrorInvalidValue;
  bwdtc::StateParams p{a.gam, a.s_init, a.s_final, a.u, a.cu, a.chunk_off,
                       a.n_seqs, a.T, a.H, a.dv};
  const size_t smem = Lay::bytes + 1024;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(bwdtc::state_chain_kernel<DK>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem)) != cudaSuccess)
    return e;
  const unsigned grid = (unsigned)a.n_seqs * a.H * (a.dv / bwdtc::kTile);
  bwdtc::state_chain_kernel<DK><<<grid, bwdtc::kThreads, smem, stream>>>(m, p);
  return cudaGetLastError();
}

cudaError_t launch_state_chain_tc(const StateChainArgs& a,
                                  cudaStream_t stream) {
  if (a.dk == 128) return run_state_chain_tc<128>(a, stream);
  if (a.dk == 64) return run_state_chain_tc<64>(a, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_rev_chain_tc(const RevChainArgs& a, cudaStream_t stream) {
  if (a.dk == 128) return run_rev_chain_tc<128>(a, stream);
  if (a.dk == 64) return run_rev_chain_tc<64>(a, stream);
  return cudaErrorInvalidValue;
}

bool make_f32_tok_map(CUtensorMap* m, const float* base, int cols, int H,
                      int tokens) {
  return make_map(m, base, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, cols, H, tokens,
                  32, CU_TENSOR_MAP_SWIZZLE_128B);
}

bool make_f32_rows_map(CUtensorMap* m, const float* base, int64_t rows,
                       int cols, int box_rows) {
  return make_rows_map(m, base, rows, cols, box_rows);
}

}  // namespace kda
