// Sequence-split prefill: one long sequence evaluated as n segments side by
// side, joined by a scan of the segments' state transitions.
//
// The recurrence's state update is affine in the state ("Kimi Delta
// Attention", akshathtiwari.co.in, the delta-rule passage: S_t = (I - beta_t
// k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T).  Inside a segment that
// starts from S_in, with M_t the product of the token transitions from the
// segment start to token t and |0 marking the evaluation from a zero state:
//     S_t = M_t S_in + S_t|0,        o_t = o_t|0 + S_in^T (M_t^T q_t).
// M_t is itself the state of the same recurrence run with v = 0 from the
// identity, and M_t^T q_t that run's output.  So:
//   (1) value run: every segment at once as a packed batch, segment 0 from the
//       true initial state, the others from zero;
//   (2) transition run (on a second stream, concurrently): segments 1..n-1
//       with v = 0, d_v = d_k and the identity as start state, giving
//       X_t = M_t^T q_t and each segment's transition M_end;
//   (3) scan: S_in(1) = S_end(0); S_in(j+1) = M_end(j) S_in(j) + S_end|0(j);
//       the last step gives the final state;
//   (4) correction: o_t += S_in(j)^T X_t for the tokens of segments 1..n-1.
// Steps (1) and (2) run the library's own prefill kernels (two-pass or
// four-stage, as kda_chunk_fwd would pick for their shapes).  On the two-pass
// path step (2) runs only its chain kernel, over the packages step (1)'s
// factorisation pass wrote: the transition run's q, k, log alpha and beta are
// step (1)'s from segment 1 on, and a package does not depend on v.  (3) is
// an fp32 kernel below, and (4) a tcgen05 product for bf16 io with d in
// {64, 128} (an fp32 register-blocked product otherwise).
#include <mutex>
#include <type_traits>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "sm100_ptx.cuh"

namespace kda {

// Set by the tensor-core correction when its bounded MMA wait gives up; read
// and cleared by kda_device_status.
__device__ int g_split_timeout = 0;

namespace {

constexpr int kThreads = 256;

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// The output correction runs on the tensor cores for bf16 io with d_k, d_v in
// {64, 128}, in tiles of kFixTile tokens (the MMA's M).
constexpr int kFixTile = 128;
bool fix_on_tensor_cores(const ChunkArgs& a) {
  return a.bf16 && (a.dk == 64 || a.dk == 128) && (a.dv == 64 || a.dv == 128);
}

struct SplitWs {
  int32_t* cu_val;   // [k + 1] segment offsets of the value run
  int32_t* cu_tr;    // [k] offsets of the transition run (segments 1..k-1)
  float* init_val;   // [k, H, dk, dv] start states of the value run
  float* end_val;    // [k, H, dk, dv] its end states
  float* ident;      // [k - 1, H, dk, dk] identity start states
  float* trans;      // [k - 1, H, dk, dk] segment transitions M_end
  float* s_in;       // [k - 1, H, dk, dv] entry states of segments 1..k-1
  __nv_bfloat16* s_in_bf;  // the same in bf16, as the tensor-core correction's
                           // MN-major operand: [k - 1, H, dv / 64, dk, 64],
                           // each [dk, 64] panel 128-byte swizzled
  void* vzero;       // [T - Ls, H, dk] io dtype, zeros
  void* x;           // [T - Ls, H, dk] io dtype, M_t^T q_t
  void* ws_val;      // the value run's own workspace
  void* ws_tr;       // the transition run's own workspace
};

ChunkArgs value_args(const ChunkArgs& a, const SplitGeom& g, const SplitWs& w) {
  ChunkArgs v = a;
  v.cu_seqlens = w.cu_val;
  v.n_seqs = g.k;
  v.initial_state = w.init_val;
  v.final_state = w.end_val;
  return v;
}

ChunkArgs trans_args(const ChunkArgs& a, const SplitGeom& g, const SplitWs& w) {
  ChunkArgs t = a;
  const size_t esz = a.bf16 ? 2 : 4;
  const size_t off = (size_t)g.Ls * a.H;  // token-heads before segment 1
  const char* q = static_cast<const char*>(a.q);
  const char* k = static_cast<const char*>(a.k);
  t.q = q ? q + off * a.dk * esz : nullptr;
  t.k = k ? k + off * a.dk * esz : nullptr;
  t.v = w.vzero;
  t.log_alpha = a.log_alpha
                    ? a.log_alpha + off * (a.gate == kGateChannel ? a.dk : 1)
                    : nullptr;
  t.beta = a.beta ? a.beta + off : nullptr;
  t.cu_seqlens = w.cu_tr;
  t.n_seqs = g.k - 1;
  t.T = a.T - g.Ls;
  t.dv = a.dk;
  t.initial_state = w.ident;
  t.out = w.x;
  t.final_state = w.trans;
  return t;
}

// The value and transition runs take kda_chunk_fwd's own evaluation: the
// two-pass tensor-core path where it applies, else the four-stage pipeline.
size_t run_workspace(const ChunkArgs& a) {
  return fused_supported(a) ? twopass_workspace_bytes(a)
                            : staged_workspace_bytes(a);
}

int run_kernels(const ChunkArgs& a) {
  return fused_supported(a) ? twopass_kernel_count(a) : staged_kernel_count(a);
}

cudaError_t run_forward(const ChunkArgs& a, void* ws, cudaStream_t s) {
  return fused_supported(a) ? launch_twopass(a, ws, s) : launch_staged(a, ws, s);
}

// On the two-pass path the transition run reads the value run's packages:
// its q, k, log alpha and beta are the value run's from segment 1 on, and a
// package does not depend on v, so only its chain kernel runs.
bool shares_packages(const ChunkArgs& value) { return fused_supported(value); }
size_t trans_workspace(const ChunkArgs& value, const ChunkArgs& trans) {
  return shares_packages(value) ? twopass_chain_workspace_bytes(trans)
                                : run_workspace(trans);
}
int trans_kernels(const ChunkArgs& value, const ChunkArgs& trans) {
  return shares_packages(value) ? twopass_chain_kernel_count(trans)
                                : run_kernels(trans);
}

// Sizes and kernel counts depend on whether cu_seqlens is present, not on its
// contents: while planning (no workspace yet) the offsets point at a tag.
const int32_t kPlanTag = 0;
SplitWs tagged(SplitWs w) {
  if (!w.cu_val) w.cu_val = const_cast<int32_t*>(&kPlanTag);
  if (!w.cu_tr) w.cu_tr = const_cast<int32_t*>(&kPlanTag);
  return w;
}

SplitWs carve_split(const ChunkArgs& a, const SplitGeom& g, void* base,
                    size_t* total) {
  const size_t esz = a.bf16 ? 2 : 4;
  const size_t H = a.H, dk = a.dk, dv = a.dv, k = g.k;
  const size_t rest = (size_t)(a.T - g.Ls) * H * dk;  // token-head-channels
  size_t off = 0;
  char* p = static_cast<char*>(base);
  auto take = [&](size_t bytes) {
    char* r = p ? p + off : nullptr;
    off = align256(off + bytes);
    return static_cast<void*>(r);
  };
  SplitWs w{};
  w.cu_val = static_cast<int32_t*>(take(4 * (k + 1)));
  w.cu_tr = static_cast<int32_t*>(take(4 * k));
  w.init_val = static_cast<float*>(take(4 * k * H * dk * dv));
  w.end_val = static_cast<float*>(take(4 * k * H * dk * dv));
  w.ident = static_cast<float*>(take(4 * (k - 1) * H * dk * dk));
  w.trans = static_cast<float*>(take(4 * (k - 1) * H * dk * dk));
  w.s_in = static_cast<float*>(take(4 * (k - 1) * H * dk * dv));
  w.s_in_bf = static_cast<__nv_bfloat16*>(take(2 * (k - 1) * H * dk * dv));
  w.vzero = take(esz * rest);
  w.x = take(esz * rest);
  // the two runs' own workspaces: sized for the packed layout they run in
  const SplitWs probe = tagged(w);
  w.ws_val = take(run_workspace(value_args(a, g, probe)));
  w.ws_tr = take(trans_workspace(value_args(a, g, probe), trans_args(a, g, probe)));
  if (total) *total = off;
  return w;
}

// Offsets, start states and the zero values of both runs, in one grid-stride
// pass: cu_val = {0, Ls, 2 Ls, .., T}; cu_tr the same shifted by Ls;
// init_val = {S_0 or 0, 0, ..}; ident = identity per (segment, head); vzero
// = 0.
__global__ void __launch_bounds__(kThreads)
    split_setup_kernel(SplitWs w, const float* __restrict__ s0, int T, int Ls,
                       int k, int H, int dk, int dv, size_t vzero_words) {
  const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  if (tid <= (size_t)k) w.cu_val[tid] = min((int)tid * Ls, T);
  if (tid < (size_t)k) w.cu_tr[tid] = min((int)tid * Ls, T - Ls);
  const size_t nstate = (size_t)H * dk * dv;
  for (size_t i = tid; i < (size_t)k * nstate; i += stride)
    w.init_val[i] = (i < nstate && s0) ? s0[i] : 0.f;
  const size_t nid = (size_t)(k - 1) * H * dk * dk;
  for (size_t i = tid; i < nid; i += stride) {
    const size_t rc = i % ((size_t)dk * dk);
    w.ident[i] = (rc / dk == rc % dk) ? 1.f : 0.f;
  }
  uint4* z = static_cast<uint4*>(w.vzero);
  for (size_t i = tid; i < vzero_words; i += stride) z[i] = make_uint4(0, 0, 0, 0);
}

// (3) Per (head, 32-column tile of d_v): S = S_end(0); for j = 1 .. k-1:
// S_in(j) = S, S <- M_end(j) S + S_end|0(j); the final S is the final state.
// M_end(j) is staged whole in shared memory (rows padded to d_k + 1), the
// tile of S beside it; thread (g8, j8) owns rows g8 + 32 a, columns j8 + 8 b.
constexpr int kScanTile = 32, kScanTp = kScanTile + 1;

__global__ void __launch_bounds__(kThreads)
    split_scan_kernel(SplitWs w, float* __restrict__ final_state, int k, int H,
                      int dk, int dv, int bf_panels) {
  const int h = blockIdx.x, j0 = blockIdx.y * kScanTile, tid = threadIdx.x;
  const int dkp = dk + 1, NA = dk / 32, g8 = tid >> 3, j8 = tid & 7;
  extern __shared__ float sm[];
  float* S = sm;              // [dk][kScanTp]
  float* M = S + dk * kScanTp;  // [dk][dkp]
  const size_t nst = (size_t)H * dk * dv;
  for (int idx = tid; idx < dk * kScanTile; idx += kThreads) {
    const int c = idx / kScanTile, jj = idx % kScanTile;
    S[c * kScanTp + jj] = w.end_val[(size_t)h * dk * dv + (size_t)c * dv + j0 + jj];
  }
  for (int j = 1; j < k; ++j) {
    const float* Mj = w.trans + ((size_t)(j - 1) * H + h) * dk * dk;
    const float* Ej = w.end_val + (size_t)j * nst + (size_t)h * dk * dv;
    float* Sin = w.s_in + (size_t)(j - 1) * nst + (size_t)h * dk * dv;
    for (int idx = tid; idx < dk * dk; idx += kThreads)
      M[(idx / dk) * dkp + idx % dk] = Mj[idx];
    __syncthreads();
    uint8_t* Sbf = reinterpret_cast<uint8_t*>(w.s_in_bf) +
                   2 * ((size_t)(j - 1) * H + h) * dk * dv;
    for (int idx = tid; idx < dk * kScanTile; idx += kThreads) {
      const int c = idx / kScanTile, jj = idx % kScanTile;
      const float sv = S[c * kScanTp + jj];
      Sin[(size_t)c * dv + j0 + jj] = sv;
      if (bf_panels) {  // element (c, n) of panel n / 64, swizzled
        const int n = j0 + jj, nn = n & 63;
        *reinterpret_cast<__nv_bfloat16*>(
            Sbf + (size_t)(n >> 6) * dk * 128 + c * 128 +
            ((((nn >> 3) ^ (c & 7)) << 4) | ((nn & 7) << 1))) =
            __float2bfloat16_rn(sv);
      }
    }
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
#pragma unroll 4
    for (int c = 0; c < dk; ++c) {
      float sv[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) sv[b] = S[c * kScanTp + j8 + 8 * b];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        if (a < NA) {
          const float m = M[(g8 + 32 * a) * dkp + c];
#pragma unroll
          for (int b = 0; b < 4; ++b) acc[a][b] += m * sv[b];
        }
      }
    }
    __syncthreads();  // every read of S and M is done
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      if (a < NA) {
        const int r = g8 + 32 * a;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int jj = j8 + 8 * b;
          S[r * kScanTp + jj] = acc[a][b] + Ej[(size_t)r * dv + j0 + jj];
        }
      }
    }
    __syncthreads();
  }
  for (int idx = tid; idx < dk * kScanTile; idx += kThreads) {
    const int c = idx / kScanTile, jj = idx % kScanTile;
    final_state[(size_t)h * dk * dv + (size_t)c * dv + j0 + jj] =
        S[c * kScanTp + jj];
  }
}

// (4) Per (chunk of segments 1..k-1, head): out[t] += S_in(j)^T X[t] for its
// C tokens (a chunk never straddles segments, whose length is a multiple of
// C).  X is staged transposed (XT[c][r], lanes walking down the rows so the
// scattered stores hit distinct banks) and S_in(j) as is, both with rows
// padded by four floats; thread (ti, tj) of a 16 x 16 grid owns the RM x RN
// block at rows RM ti.., columns RN tj.. (RM = C / 16, RN = d_v / 16), so
// each step of the contraction is a few 16-byte shared loads for RM x RN
// FMAs.
template <int N>
__device__ __forceinline__ void lds_run(const float* p, float* v) {
  if constexpr (N >= 4) {
#pragma unroll
    for (int q = 0; q < N / 4; ++q) {
      const float4 x = *reinterpret_cast<const float4*>(p + 4 * q);
      v[4 * q] = x.x;
      v[4 * q + 1] = x.y;
      v[4 * q + 2] = x.z;
      v[4 * q + 3] = x.w;
    }
  } else if constexpr (N == 2) {
    const float2 x = *reinterpret_cast<const float2*>(p);
    v[0] = x.x;
    v[1] = x.y;
  } else {
    v[0] = p[0];
  }
}

// Eight consecutive io-dtype elements as fp32 (one 16-byte load for bf16,
// two for fp32), and back.
__device__ __forceinline__ void ld8(const __nv_bfloat16* p, float* v) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __bfloat1622float2(h[e]);
    v[2 * e] = f.x;
    v[2 * e + 1] = f.y;
  }
}
__device__ __forceinline__ void ld8(const float* p, float* v) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void st8(__nv_bfloat16* p, const float* v) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void st8(float* p, const float* v) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}

template <typename IO, int RM, int RN>
__global__ void __launch_bounds__(kThreads)
    split_fix_kernel(SplitWs w, IO* __restrict__ out, int T, int Ls, int k,
                     int H, int dk, int dv) {
  constexpr int C = 16 * RM, DV = 16 * RN, LX = C + 4, LS = DV + 4;
  const int t0 = Ls + blockIdx.x * C, h = blockIdx.y, tid = threadIdx.x;
  const int L = min(C, T - t0);
  const int j = min(t0 / Ls, k - 1);
  extern __shared__ __align__(16) float sm[];
  float* XT = sm;              // [dk][LX]
  float* S = XT + dk * LX;     // [dk][LS]
  const IO* x = static_cast<const IO*>(w.x);
  // XT[c][r] = X[r][c]: thread (r, 8-column group), rows past L zero; all
  // of a thread's loads are issued before its stores
  {
    constexpr int NX = 64 * 128 / 8 / kThreads;  // C * dk / 8 <= NX * kThreads
    float v[NX][8];
#pragma unroll
    for (int u = 0; u < NX; ++u) {
      const int idx = u * kThreads + tid;
      const int r = idx % C, c = (idx / C) * 8;
#pragma unroll
      for (int e = 0; e < 8; ++e) v[u][e] = 0.f;
      if (idx < C * (dk / 8) && r < L)
        ld8(x + ((size_t)(t0 - Ls + r) * H + h) * dk + c, v[u]);
    }
#pragma unroll
    for (int u = 0; u < NX; ++u) {
      const int idx = u * kThreads + tid;
      if (idx < C * (dk / 8)) {
        const int r = idx % C, c = (idx / C) * 8;
#pragma unroll
        for (int e = 0; e < 8; ++e) XT[(c + e) * LX + r] = v[u][e];
      }
    }
  }
  // S_in(j), sixteen 16-byte loads in flight per thread at a time
  {
    const float* Sin = w.s_in + ((size_t)(j - 1) * H + h) * dk * dv;
    const int units = dk * (DV / 4);
    for (int base = 0; base < units; base += 16 * kThreads) {
      float4 v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int idx = base + u * kThreads + tid;
        if (idx < units) {
          const int c = idx / (DV / 4), q = idx % (DV / 4);
          v[u] = *reinterpret_cast<const float4*>(Sin + (size_t)c * dv + 4 * q);
        }
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int idx = base + u * kThreads + tid;
        if (idx < units) {
          const int c = idx / (DV / 4), q = idx % (DV / 4);
          *reinterpret_cast<float4*>(S + c * LS + 4 * q) = v[u];
        }
      }
    }
  }
  __syncthreads();
  const int ti = tid >> 4, tj = tid & 15;
  float acc[RM][RN];
#pragma unroll
  for (int a = 0; a < RM; ++a)
#pragma unroll
    for (int b = 0; b < RN; ++b) acc[a][b] = 0.f;
  const float* ap = XT + RM * ti;
  const float* bp = S + RN * tj;
#pragma unroll 4
  for (int c = 0; c < dk; ++c) {
    float av[RM], bv[RN];
    lds_run<RM>(ap + c * LX, av);
    lds_run<RN>(bp + c * LS, bv);
#pragma unroll
    for (int a = 0; a < RM; ++a)
#pragma unroll
      for (int b = 0; b < RN; ++b) acc[a][b] += av[a] * bv[b];
  }
#pragma unroll
  for (int a = 0; a < RM; ++a) {
    const int r = RM * ti + a;
    if (r < L) {
      IO* o = out + ((size_t)(t0 + r) * H + h) * dv + RN * tj;
      if constexpr (RN == 8) {  // one 16-byte read and write per row (bf16)
        float y[8];
        ld8(o, y);
#pragma unroll
        for (int b = 0; b < 8; ++b) y[b] += acc[a][b];
        st8(o, y);
      } else {
#pragma unroll
        for (int b = 0; b < RN; ++b)
          o[b] = from_f32<IO>(to_f32(o[b]) + acc[a][b]);
      }
    }
  }
}

// (4') The correction on the tensor cores, for bf16 io with d_k, d_v in
// {64, 128}: per (128-token tile, head) one M = 128, N = d_v, K = d_k product
// of the tile's X rows (K-major, 128-byte-swizzled panels; rows past the
// sequence are zero) and S_in(j) rounded to bf16 (MN-major panels of d_k
// rows), accumulated in TMEM.  Segments are whole tiles on this path, so a
// tile never straddles two.  Each thread owns one TMEM lane, i.e. one token,
// and adds its row into the output 16 bytes at a time.  The MMA wait is
// bounded; if it gives up the block writes nothing and raises the library's
// timeout flag.
template <int DK, int DV>
__global__ void __launch_bounds__(128)
    split_fix_tc_kernel(SplitWs w, __nv_bfloat16* __restrict__ out, int T,
                        int Ls, int k, int H, int C, int* timeout_flag) {
  using namespace sm100;
  constexpr uint32_t kApanel = 128 * 128;  // 128 rows of 64 bf16
  constexpr uint32_t kBpanel = DK * 128;   // DK K-rows of 64 bf16
  extern __shared__ __align__(1024) uint8_t sm_raw[];
  uint8_t* sA = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = sA + (DK / 64) * kApanel;
  constexpr uint32_t kBbytes = (DV / 64) * kBpanel;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sB + kBbytes);  // [0] B, [1] MMA
  uint32_t* tbase = reinterpret_cast<uint32_t*>(bar + 2);
  const int t0 = Ls + blockIdx.x * kFixTile, h = blockIdx.y, tid = threadIdx.x;
  const int L = min(kFixTile, T - t0);
  const int j = min(t0 / Ls, k - 1);
  // B = S_in(j) in bf16, already in its swizzled N-major panels: one bulk
  // single-destination copy completing on bar[0], while the threads stage A
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(bar + 1, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(bar, kBbytes);
    const uint8_t* src = reinterpret_cast<const uint8_t*>(w.s_in_bf) +
                         2 * ((size_t)(j - 1) * H + h) * DK * DV;
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1], %2, [%3];" ::"r"(smem_u32(sB)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(kBbytes), "r"(smem_u32(bar))
        : "memory");
  }
  // A[r][c] = X[r][c]: every load of the thread in flight before its stores
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(w.x);
  {
    constexpr int NA = kFixTile * (DK / 8) / 128;
    uint4 v[NA];
#pragma unroll
    for (int u = 0; u < NA; ++u) {
      const int idx = u * 128 + tid;
      const int r = idx / (DK / 8), pc = idx % (DK / 8);
      v[u] = make_uint4(0u, 0u, 0u, 0u);
      if (r < L)
        v[u] = *reinterpret_cast<const uint4*>(
            x + ((size_t)(t0 - Ls + r) * H + h) * DK + pc * 8);
    }
#pragma unroll
    for (int u = 0; u < NA; ++u) {
      const int idx = u * 128 + tid;
      const int r = idx / (DK / 8), pc = idx % (DK / 8);
      *reinterpret_cast<uint4*>(sA + (pc / 8) * kApanel + r * 128 +
                                (((pc % 8) ^ (r & 7)) << 4)) = v[u];
    }
  }
  if (tid < 32) {
    tmem_alloc(tbase, 128);
    tmem_relinquish();
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tbase;
  bool ok = true;
  if (tid == 0) {
    ok = mbar_wait(bar, 0);  // B has landed
    if (ok) {
      const uint32_t idesc = idesc_bf16(128, DV, false, true);
      const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
#pragma unroll
      for (int ks = 0; ks < DK / 16; ++ks)
        mma_bf16(tmem,
                 desc_sw128(a0 + (ks / 4) * kApanel + (ks % 4) * 32, 16, 1024),
                 desc_sw128(b0 + ks * 2048, kBpanel, 1024), idesc,
                 ks > 0 ? 1u : 0u);
      mma_commit(bar + 1);
    } else {
      mbar_wait(bar, 0, 100000000ull);  // the copy, before the block leaves
    }
  }
  ok = __syncthreads_and(ok) != 0;
  if (ok) ok = mbar_wait(bar + 1, 0);
  tc_fence_after();
  const int warp = tid >> 5;
  {  // TMEM lane = row of the tile
    const int r = tid;
#pragma unroll
    for (int c = 0; c < DV; c += 32) {
      float v[32];
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c, v);
      if (ok && r < L) {
        __nv_bfloat16* o = out + ((size_t)(t0 + r) * H + h) * DV + c;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float y[8];
          ld8(o + 8 * q, y);
#pragma unroll
          for (int e = 0; e < 8; ++e) y[e] += v[8 * q + e];
          st8(o + 8 * q, y);
        }
      }
    }
  }
  if (!ok && tid == 0) atomicExch(timeout_flag, 1);
  tc_fence_before();
  __syncthreads();
  if (tid < 32) tmem_dealloc(tmem, 128);
}

template <int DK, int DV>
cudaError_t launch_fix_tc_t(const SplitWs& w, __nv_bfloat16* out,
                            const ChunkArgs& a, const SplitGeom& g, dim3 grid,
                            int* flag, cudaStream_t stream) {
  const size_t smem = 1024 + (DK / 64) * 128 * 128 + (DV / 64) * DK * 128 + 64;
  static_assert(((DV / 64) * DK * 128) % 16 == 0, "bulk copy size");
  cudaError_t e = cudaFuncSetAttribute(split_fix_tc_kernel<DK, DV>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  split_fix_tc_kernel<DK, DV><<<grid, 128, smem, stream>>>(
      w, out, a.T, g.Ls, g.k, a.H, a.chunk, flag);
  return cudaGetLastError();
}


cudaError_t launch_fix_tc(const SplitWs& w, __nv_bfloat16* out,
                          const ChunkArgs& a, const SplitGeom& g, dim3 grid,
                          cudaStream_t stream) {
  int* flag = nullptr;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&flag),
                                       g_split_timeout);
  if (e != cudaSuccess) return e;
  if (a.dk == 64)
    return a.dv == 64 ? launch_fix_tc_t<64, 64>(w, out, a, g, grid, flag, stream)
                      : launch_fix_tc_t<64, 128>(w, out, a, g, grid, flag, stream);
  return a.dv == 64 ? launch_fix_tc_t<128, 64>(w, out, a, g, grid, flag, stream)
                    : launch_fix_tc_t<128, 128>(w, out, a, g, grid, flag, stream);
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)bytes);
}

// A non-blocking stream per device for the transition run, created on first
// use and kept for the life of the process.
cudaError_t side_stream(cudaStream_t* out) {
  static std::mutex mu;
  static cudaStream_t streams[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!streams[dev]) {
    e = cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking);
    if (e != cudaSuccess) {
      streams[dev] = nullptr;
      return e;
    }
  }
  *out = streams[dev];
  return cudaSuccess;
}

template <typename IO, int RM, int RN>
cudaError_t launch_fix_t(const SplitWs& w, IO* out, const ChunkArgs& a,
                         const SplitGeom& g, dim3 grid, cudaStream_t stream) {
  const size_t smem = 4 * (size_t)a.dk * ((16 * RM + 4) + (16 * RN + 4));
  cudaError_t e = set_smem(split_fix_kernel<IO, RM, RN>, smem);
  if (e != cudaSuccess) return e;
  split_fix_kernel<IO, RM, RN><<<grid, kThreads, smem, stream>>>(
      w, out, a.T, g.Ls, g.k, a.H, a.dk, a.dv);
  return cudaGetLastError();
}

template <typename IO, int RM>
cudaError_t launch_fix_n(const SplitWs& w, IO* out, const ChunkArgs& a,
                         const SplitGeom& g, dim3 grid, cudaStream_t stream) {
  switch (a.dv) {
    case 32: return launch_fix_t<IO, RM, 2>(w, out, a, g, grid, stream);
    case 64: return launch_fix_t<IO, RM, 4>(w, out, a, g, grid, stream);
    case 128: return launch_fix_t<IO, RM, 8>(w, out, a, g, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

// The correction with the register blocking its chunk length and d_v ask for.
template <typename IO>
cudaError_t launch_fix(const SplitWs& w, IO* out, const ChunkArgs& a,
                       const SplitGeom& g, dim3 grid, cudaStream_t stream) {
  switch (a.chunk) {
    case 16: return launch_fix_n<IO, 1>(w, out, a, g, grid, stream);
    case 32: return launch_fix_n<IO, 2>(w, out, a, g, grid, stream);
    case 64: return launch_fix_n<IO, 4>(w, out, a, g, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <typename IO>
cudaError_t run_split(const ChunkArgs& a, const SplitGeom& g, void* workspace,
                      cudaStream_t stream) {
  SplitWs w = carve_split(a, g, workspace, nullptr);
  const size_t esz = a.bf16 ? 2 : 4;
  const size_t vz_words = esz * (size_t)(a.T - g.Ls) * a.H * a.dk / 16;
  cudaError_t e;
  split_setup_kernel<<<4 * 148, kThreads, 0, stream>>>(
      w, a.initial_state, a.T, g.Ls, g.k, a.H, a.dk, a.dv, vz_words);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  // (1) on `stream`, (2) on the side stream, joined by events
  cudaStream_t side = nullptr;
  if ((e = side_stream(&side)) != cudaSuccess) return e;
  cudaEvent_t fork = nullptr, join = nullptr;
  if ((e = cudaEventCreateWithFlags(&fork, cudaEventDisableTiming)) != cudaSuccess)
    return e;
  if ((e = cudaEventCreateWithFlags(&join, cudaEventDisableTiming)) != cudaSuccess) {
    cudaEventDestroy(fork);
    return e;
  }
  auto done = [&](cudaError_t r) {
    cudaEventDestroy(fork);
    cudaEventDestroy(join);
    return r;
  };
  if ((e = cudaEventRecord(fork, stream)) != cudaSuccess) return done(e);
  if ((e = cudaStreamWaitEvent(side, fork, 0)) != cudaSuccess) return done(e);
  const ChunkArgs va = value_args(a, g, w), ta = trans_args(a, g, w);
  if (shares_packages(va)) {
    // the value run on `stream`; once its factorisation pass is done, the
    // transition run's chain on the side stream over the same packages from
    // segment 1 on (segment 0 holds Ls / C chunks)
    cudaEvent_t factored = nullptr;
    if ((e = cudaEventCreateWithFlags(&factored, cudaEventDisableTiming)) !=
        cudaSuccess)
      return done(e);
    const cudaError_t e_val = launch_twopass(va, w.ws_val, stream, factored);
    const cudaError_t e_dep =
        e_val == cudaSuccess ? cudaStreamWaitEvent(side, factored, 0) : e_val;
    const cudaError_t e_tr =
        e_dep == cudaSuccess
            ? launch_twopass_chain(
                  ta, w.ws_tr,
                  twopass_packages(va, w.ws_val, (int64_t)(g.Ls / a.chunk)),
                  side)
            : cudaSuccess;
    // whatever failed, `stream` waits for the side stream before the
    // caller can release the workspace
    const cudaError_t e_rec = cudaEventRecord(join, side);
    const cudaError_t e_wait =
        e_rec == cudaSuccess ? cudaStreamWaitEvent(stream, join, 0) : e_rec;
    cudaEventDestroy(factored);
    for (cudaError_t r : {e_val, e_dep, e_tr, e_rec, e_wait})
      if (r != cudaSuccess) return done(r);
  } else {
    // whatever fails below, `stream` waits for the side stream before the
    // caller can release the workspace
    const cudaError_t e_tr = run_forward(ta, w.ws_tr, side);
    const cudaError_t e_rec = cudaEventRecord(join, side);
    const cudaError_t e_val =
        e_tr == cudaSuccess ? run_forward(va, w.ws_val, stream) : cudaSuccess;
    const cudaError_t e_wait =
        e_rec == cudaSuccess ? cudaStreamWaitEvent(stream, join, 0) : e_rec;
    for (cudaError_t r : {e_tr, e_rec, e_val, e_wait})
      if (r != cudaSuccess) return done(r);
  }
  done(cudaSuccess);

  // (3) scan, (4) correction
  const int dk = a.dk, dv = a.dv, H = a.H, C = a.chunk;
  const size_t sms = 4 * ((size_t)dk * kScanTp + (size_t)dk * (dk + 1));
  if ((e = set_smem(split_scan_kernel, sms)) != cudaSuccess) return e;
  split_scan_kernel<<<dim3(H, dv / kScanTile), kThreads, sms, stream>>>(
      w, a.final_state, g.k, H, dk, dv, fix_on_tensor_cores(a) ? 1 : 0);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const unsigned nblk = (unsigned)((a.T - g.Ls + C - 1) / C);
  if constexpr (std::is_same<IO, __nv_bfloat16>::value) {
    if (fix_on_tensor_cores(a)) {
      const unsigned ntile = (unsigned)((a.T - g.Ls + kFixTile - 1) / kFixTile);
      return launch_fix_tc(w, static_cast<IO*>(a.out), a, g, dim3(ntile, H),
                           stream);
    }
  }
  return launch_fix<IO>(w, static_cast<IO*>(a.out), a, g, dim3(nblk, H),
                        stream);
}

}  // namespace

int split_auto_segments(const ChunkArgs& a, int num_sms) {
  // CTAs one segment's chain occupies: one per head and 64-wide value tile
  // (the chain kernel's two CTAs at d_v = 128); the transition run has
  // d_v = d_k, so take the wider of the two
  const int wide = a.dv > a.dk ? a.dv : a.dk;
  const int per_seg = a.H * (wide > 64 ? wide / 64 : 1);
  int k = 1;
  while (k < 64 && (2 * (k + 1) - 1) * per_seg <= num_sms) ++k;
  return k;
}

cudaError_t split_take_timeout(cudaStream_t stream, int* flag) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  int zero = 0;
  if ((e = cudaMemcpyFromSymbol(flag, g_split_timeout, sizeof(int))) !=
      cudaSuccess)
    return e;
  return cudaMemcpyToSymbol(g_split_timeout, &zero, sizeof(int));
}

SplitGeom split_geometry(const ChunkArgs& a, int n_segments) {
  SplitGeom g{};
  const int C = a.chunk;
  const int nch = (a.T + C - 1) / C;
  const int n = n_segments < nch ? n_segments : nch;
  if (n <= 1) {
    g.k = 1;
    g.Ls = a.T;
    return g;
  }
  g.Ls = ((nch + n - 1) / n) * C;
  if (fix_on_tensor_cores(a))  // whole 128-token correction tiles per segment
    g.Ls = (g.Ls + kFixTile - 1) / kFixTile * kFixTile;
  g.k = (a.T + g.Ls - 1) / g.Ls;
  if (g.k <= 1) {
    g.k = 1;
    g.Ls = a.T;
  }
  return g;
}

size_t split_workspace_bytes(const ChunkArgs& a, const SplitGeom& g) {
  if (g.k <= 1) return run_workspace(a);
  size_t total = 0;
  carve_split(a, g, nullptr, &total);
  return total;
}

int split_kernel_count(const ChunkArgs& a, const SplitGeom& g) {
  if (g.k <= 1) return run_kernels(a);
  const SplitWs w = tagged(SplitWs{});
  // setup, the two runs, scan, correction
  return 1 + run_kernels(value_args(a, g, w)) +
         trans_kernels(value_args(a, g, w), trans_args(a, g, w)) + 2;
}

cudaError_t launch_split(const ChunkArgs& a, const SplitGeom& g, void* workspace,
                         cudaStream_t stream) {
  if (g.k <= 1) return run_forward(a, workspace, stream);
  return a.bf16 ? run_split<__nv_bfloat16>(a, g, workspace, stream)
                : run_split<float>(a, g, workspace, stream);
}

}  // namespace kda
