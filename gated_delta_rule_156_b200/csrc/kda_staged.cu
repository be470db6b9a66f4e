// Four-stage chunkwise KDA forward, all arithmetic in fp32 (SIMT).
//
// The recurrence S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T,
// o_t = S_t^T q_t, regrouped over chunks of C tokens (the chunkwise form that
// turns the recurrence into matrix products, "You Could Have Come Up with Kimi
// Delta Attention", daily.dev, Summary; the Diagonal-Plus-Low-Rank transition
// of "Kimi Delta Attention", akshathtiwari.co.in).  Inside a chunk with start
// state S_0 and positions r = 1..C:
//   g_r  = sum_{i<=r} l_i                          (1) cumulative log-decay
//   Kt   = k * exp(g), Kb = k * exp(-g), Qt = q * exp(g), Kh = k * exp(g_C - g)
//   A    = strictly_lower(Diag(b) Kt Kb^T)         (2) intra-chunk factors
// (A and lower_incl(Qt Kb^T) only need exp(g_r - g_i) for i <= r; they are
// formed from k exp(g - rho) and k exp(rho - g) with the per-channel
// reference rho of decay_ref, so strong gates stay inside the fp32 range.)
//   Tm   = (I + A)^-1    blocked: 16 x 16 diagonal blocks by forward
//                        substitution, the blocks below by recursive doubling
//   W    = Tm Diag(b) Kt,  U = Tm Diag(b) V
//   D    = U - W S_0                               (3) state pass (serial)
//   S_C  = Diag(exp(g_C)) S_0 + Kh^T D
//   O    = Qt S_0 + lower_incl(Qt Kb^T) D           (4) output
// Each stage is its own kernel with its inputs and outputs in an HBM
// workspace; stages (1), (2), (4) are parallel over (chunk, head), stage (3)
// over (sequence, head, 64-column tile of d_v; 32 when d_v = 32), and stage
// (4) over 32-column tiles.  This is the all-fp32 mode and the reference
// decomposition the fused tensor-core kernel is built from.
#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_inverse.cuh"

namespace kda {

// Set when a chunk's decay exceeds the factorisation's range (read and
// cleared on the host).
__device__ int g_staged_range = 0;

namespace {

constexpr int kThreads = 256;
constexpr int kDvTile = 32;

bool has_prologue(const ChunkArgs& a) {
  return a.pro.norm_qk || a.pro.q_scale != 1.f ||
         (a.pro.gate_logits && a.gate != kGateNone);
}

struct Ws {
  void* qn;            // prologue outputs (only with an input prologue):
  void* kn;            //   normalised q, k [tokens, H, dk] in the io dtype,
  float* lan;          //   log(alpha) [tokens, H, dk or 1]
  int32_t* chunk_off;  // [n_seqs + 1] (packed layout only)
  float* g;            // [tokens, H, dk]   cumulative log-decay within chunk
  float* w;            // [tokens, H, dk]   W rows
  float* u;            // [tokens, H, dv]   U rows, overwritten by D
  float* kh;           // [tokens, H, dk]   Kh = k exp(g_C - g)
  float* s;            // [max_chunks, H, dk, dv]  chunk-start states
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

Ws carve(const ChunkArgs& a, void* base, size_t* total,
         size_t* prefix = nullptr) {
  const size_t tokens =
      a.cu_seqlens ? (size_t)a.T : (size_t)a.n_seqs * (size_t)a.T;
  const size_t H = a.H;
  size_t off = 0;
  Ws w{};
  char* p = static_cast<char*>(base);
  auto take = [&](size_t bytes) {
    char* r = p ? p + off : nullptr;
    off = align256(off + bytes);
    return r;
  };
  if (has_prologue(a)) {
    const size_t esz = a.bf16 ? 2 : 4;
    w.qn = take(esz * tokens * H * a.dk);
    w.kn = take(esz * tokens * H * a.dk);
    w.lan = reinterpret_cast<float*>(
        take(4 * tokens * H * (a.gate == kGateChannel ? a.dk : 1)));
  }
  w.chunk_off = reinterpret_cast<int32_t*>(take(4 * (size_t)(a.n_seqs + 1)));
  w.g = reinterpret_cast<float*>(take(4 * tokens * H * a.dk));
  if (prefix) *prefix = off;
  w.w = reinterpret_cast<float*>(take(4 * tokens * H * a.dk));
  w.u = reinterpret_cast<float*>(take(4 * tokens * H * a.dv));
  w.kh = reinterpret_cast<float*>(take(4 * tokens * H * a.dk));
  w.s = reinterpret_cast<float*>(
      take(4 * (size_t)max_chunks(a) * H * a.dk * a.dv));
  if (total) *total = off;
  return w;
}

// Optional input prologue, one warp per (token, head): q and k L2-normalised
// over d_k (q also scaled), and raw gate logits turned into
// log(alpha) = scale * logsigmoid(x); results go to the workspace.
template <typename IO>
__global__ void prologue_kernel(const IO* __restrict__ q, const IO* __restrict__ k,
                                const float* __restrict__ la, IO* __restrict__ qn,
                                IO* __restrict__ kn, float* __restrict__ lan,
                                int H, int dk, int gate, Prologue pro) {
  const size_t th = blockIdx.x;  // token * H + head
  const int lane = threadIdx.x;
  float sk = 0.f, sq = 0.f;
  for (int c = lane; c < dk; c += 32) {
    const float kc = to_f32(k[th * dk + c]), qc = to_f32(q[th * dk + c]);
    sk += kc * kc;
    sq += qc * qc;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sk += __shfl_xor_sync(0xffffffffu, sk, o);
    sq += __shfl_xor_sync(0xffffffffu, sq, o);
  }
  const float ik = pro.norm_qk ? rsqrtf(sk) : 1.f;
  const float iq = (pro.norm_qk ? rsqrtf(sq) : 1.f) * pro.q_scale;
  for (int c = lane; c < dk; c += 32) {
    kn[th * dk + c] = from_f32<IO>(to_f32(k[th * dk + c]) * ik);
    qn[th * dk + c] = from_f32<IO>(to_f32(q[th * dk + c]) * iq);
  }
  if (gate == kGateNone) return;
  const int nl = gate == kGateChannel ? dk : 1;
  for (int c = lane; c < nl; c += 32) {
    float x = la[th * nl + c];
    if (pro.gate_logits)
      x = pro.gate_scale * (fminf(x, 0.f) - log1pf(__expf(-fabsf(x))));
    lan[th * nl + c] = x;
  }
}

// Packed layout: exclusive prefix sum of ceil(len_s / C) per sequence.
__global__ void plan_kernel(const int32_t* __restrict__ cu, int n_seqs, int T,
                            int C, int32_t* __restrict__ chunk_off) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int acc = 0;
  chunk_off[0] = 0;
  for (int s = 0; s < n_seqs; ++s) {
    int a, b;
    seq_range(cu, s, T, &a, &b);
    acc += (b - a + C - 1) / C;
    chunk_off[s + 1] = acc;
  }
}

// (1) g_r = sum_{i<=r} l_i within the chunk; one thread per key channel.
// With a per-head gate every channel reads the head's log(alpha); with no
// gate (alpha = 1) g stays zero.
__global__ void cumsum_kernel(const float* __restrict__ la, float* __restrict__ g,
                              const int32_t* cu, const int32_t* chunk_off,
                              int n_seqs, int T, int H, int dk, int C, int gate) {
  int seq, tok0, L;
  if (!locate_chunk(blockIdx.x, cu, chunk_off, n_seqs, T, C, &seq, &tok0, &L))
    return;
  const int h = blockIdx.y;
  for (int c = threadIdx.x; c < dk; c += blockDim.x) {
    float acc = 0.f;
    for (int r = 0; r < L; ++r) {
      const size_t idx = ((size_t)(tok0 + r) * H + h) * dk + c;
      acc += gate == kGateChannel ? la[idx]
             : gate == kGateHead  ? la[(size_t)(tok0 + r) * H + h]
                                  : 0.f;
      g[idx] = acc;
    }
  }
}

// (2) A, Tm = (I + A)^-1, W = Tm Diag(b) Kt, U = Tm Diag(b) V, and the
// state pass's Kh = k exp(g_C - g).
template <typename IO>
__global__ void __launch_bounds__(kThreads)
    intra_kernel(const IO* __restrict__ k, const IO* __restrict__ v,
                 const float* __restrict__ beta, const float* __restrict__ g,
                 float* __restrict__ w_out, float* __restrict__ u_out,
                 float* __restrict__ kh_out,
                 const int32_t* cu, const int32_t* chunk_off, int n_seqs, int T,
                 int H, int dk, int dv, int C) {
  int seq, tok0, L;
  if (!locate_chunk(blockIdx.x, cu, chunk_off, n_seqs, T, C, &seq, &tok0, &L))
    return;
  const int h = blockIdx.y, tid = threadIdx.x;
  extern __shared__ float sm[];
  const int ldk = dk + 1;          // padded rows: no bank conflicts
  float* Kt = sm;                  // [C][ldk]
  float* Kb = Kt + C * ldk;        // [C][ldk]
  float* V = Kb + C * ldk;         // [C][dv]
  float* A = V + C * dv;           // [64][kFS], zero-padded past C
  float* Tm = A + 64 * ws::kFS;    // [64][kFS], (I + A)^-1
  float* Msc = Tm + 64 * ws::kFS;  // [1024] scratch of the inverse
  float* bs = Msc + 1024;          // [C]
  float* gl = bs + C;              // [dk] g at the chunk's last row
  float* rho = gl + dk;            // [dk] reference of the A factorisation

  for (int c = tid; c < dk; c += kThreads) {
    gl[c] = g[((size_t)(tok0 + L - 1) * H + h) * dk + c];
    rho[c] = decay_ref(gl[c]);
    if (fabsf(gl[c]) > kDecayRangeMax) atomicExch(&g_staged_range, 1);
  }
  __syncthreads();
  // Kt holds k exp(g - rho) and Kb k exp(rho - g): their products are the
  // exact exp(g_r - g_i) factors of A; W is rescaled by exp(rho) below to the
  // chunk-start Kt = k exp(g).
  for (int idx = tid; idx < C * dk; idx += kThreads) {
    const int r = idx / dk, c = idx % dk;
    float kt = 0.f, kb = 0.f;
    if (r < L) {
      const size_t gi = ((size_t)(tok0 + r) * H + h) * dk + c;
      const float kv = to_f32(k[gi]), gv = g[gi];
      kt = kv * __expf(gv - rho[c]);
      kb = kv * __expf(rho[c] - gv);
      kh_out[gi] = kv * __expf(gl[c] - gv);
    }
    Kt[r * ldk + c] = kt;
    Kb[r * ldk + c] = kb;
  }
  for (int idx = tid; idx < C * dv; idx += kThreads) {
    const int r = idx / dv, j = idx % dv;
    V[idx] = r < L ? to_f32(v[((size_t)(tok0 + r) * H + h) * dv + j]) : 0.f;
  }
  for (int r = tid; r < C; r += kThreads)
    bs[r] = r < L ? beta[(size_t)(tok0 + r) * H + h] : 0.f;
  __syncthreads();

  for (int idx = tid; idx < 64 * ws::kFS; idx += kThreads) {
    A[idx] = 0.f;
    Tm[idx] = 0.f;
  }
  __syncthreads();
  // Thread (ti, tj) owns rows ti + 16 a and columns tj + 16 b of each
  // product: with the padded rows every shared load is conflict-free or a
  // broadcast, and a step of the contraction feeds a block of FMAs.
  const int ti = tid >> 4, tj = tid & 15, nr = C / 16;
  {
    float m[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) m[a][b] = 0.f;
#pragma unroll 2
    for (int c = 0; c < dk; ++c) {
      float kt[4], kb[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        kt[a] = a < nr ? Kt[(ti + 16 * a) * ldk + c] : 0.f;
        kb[a] = a < nr ? Kb[(tj + 16 * a) * ldk + c] : 0.f;
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) m[a][b] += kt[a] * kb[b];
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int r = ti + 16 * a, i = tj + 16 * b;
        if (a < nr && b < nr && i < r) A[r * ws::kFS + i] = m[a][b] * bs[r];
      }
  }
  __syncthreads();
  // Tm = (I + A)^-1 by recursive doubling on 16 x 16 blocks (the rows and
  // columns past C are zero in A, so they stay identity in Tm)
  ws::invert_unit_lower(A, Tm, Msc, tid);
  __syncthreads();
  // Tm Diag(b), in place (Tm is lower triangular, zero above the diagonal)
  for (int idx = tid; idx < C * C; idx += kThreads) {
    const int r = idx / C, i = idx % C;
    Tm[r * ws::kFS + i] *= bs[i];
  }
  __syncthreads();
  // W = (Tm Diag(b)) Kt and U = (Tm Diag(b)) V over i = 0 .. C - 1 (the
  // terms above the diagonal are exact zeros)
  {
    const int nw = dk / 16, nu = dv / 16;
    float aw[4][8], au[4][8];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 8; ++b) aw[a][b] = au[a][b] = 0.f;
#pragma unroll 2
    for (int i = 0; i < C; ++i) {
      float t[4], kt[8], vv[8];
#pragma unroll
      for (int a = 0; a < 4; ++a) t[a] = a < nr ? Tm[(ti + 16 * a) * ws::kFS + i] : 0.f;
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        kt[b] = b < nw ? Kt[i * ldk + tj + 16 * b] : 0.f;
        vv[b] = b < nu ? V[i * dv + tj + 16 * b] : 0.f;
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          aw[a][b] += t[a] * kt[b];
          au[a][b] += t[a] * vv[b];
        }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int r = ti + 16 * a;
      if (a < nr && r < L) {
        const size_t rw = ((size_t)(tok0 + r) * H + h) * dk;
        const size_t ru = ((size_t)(tok0 + r) * H + h) * dv;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          if (b < nw) w_out[rw + tj + 16 * b] = aw[a][b] * __expf(rho[tj + 16 * b]);
          if (b < nu) u_out[ru + tj + 16 * b] = au[a][b];
        }
      }
    }
  }
}

// (3) Sequential over the chunks of one sequence; one TILE-wide column tile
// of S (64, or 32 when d_v = 32, so that a d = 128 layer is one wave of CTAs).
//   D = U - W S ;  S <- Diag(exp(g_C)) S + Kh^T D,  Kh = k exp(g_C - g) from
// stage (2).  Stores every chunk-start state (for stage 4), D (over U), and
// the final state.  The next chunk's W, Kh, U tile and decay are loaded into
// registers while the current chunk computes, so the serial loop does not
// wait on memory.  Shared rows are padded (TILE + 1 floats for the tiles,
// dk + 1 for the token rows) so the products are free of bank conflicts; each
// thread owns a block of outputs (rows strided by 32, columns by 8) whose sums
// run as independent chains.
template <int TILE>
__global__ void __launch_bounds__(kThreads)
    state_kernel(const float* __restrict__ g, const float* __restrict__ w,
                 const float* __restrict__ kh, float* __restrict__ u,
                 float* __restrict__ s_chunks,
                 const float* __restrict__ s_init, float* __restrict__ s_final,
                 const int32_t* cu, const int32_t* chunk_off, int n_seqs, int T,
                 int H, int dk, int dv, int C) {
  constexpr int TP = TILE + 1, NB = TILE / 8;
  constexpr int NP = 64 * 128 / kThreads;   // C * dk <= NP * kThreads
  constexpr int NU = 64 * TILE / kThreads;  // C * TILE <= NU * kThreads
  const int seq = blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * TILE;
  const int tid = threadIdx.x;
  const int dkp = dk + 1, NA = dk / 32;
  const int g8 = tid >> 3, j8 = tid & 7;
  extern __shared__ float sm[];
  float* S = sm;                  // [dk][TP]
  float* Wc = S + dk * TP;        // [C][dkp]
  float* Kh = Wc + C * dkp;       // [C][dkp]
  float* D = Kh + C * dkp;        // [C][TP]
  float* gam = D + C * TP;        // [dk] exp(g_C)

  const size_t sbase = ((size_t)seq * H + h) * dk * dv;
  for (int idx = tid; idx < dk * TILE; idx += kThreads) {
    const int c = idx / TILE, jj = idx % TILE;
    S[c * TP + jj] = s_init ? s_init[sbase + (size_t)c * dv + j0 + jj] : 0.f;
  }
  int start, end;
  seq_range(cu, seq, T, &start, &end);
  const int nch = (end - start + C - 1) / C;
  const int cid0 = cu ? chunk_off[seq] : seq * ((T + C - 1) / C);

  float pw[NP], pk[NP], pu[NU], pg = 0.f;
  auto fetch = [&](int ch) {
    const int tok0 = start + ch * C, L = min(C, end - tok0);
#pragma unroll
    for (int q = 0; q < NP; ++q) {
      const int idx = q * kThreads + tid, r = idx / dk;
      const bool in = idx < C * dk && r < L;
      const size_t gi = ((size_t)(tok0 + r) * H + h) * dk + idx % dk;
      pw[q] = in ? w[gi] : 0.f;
      pk[q] = in ? kh[gi] : 0.f;
    }
#pragma unroll
    for (int q = 0; q < NU; ++q) {
      const int idx = q * kThreads + tid, r = idx / TILE;
      const bool in = idx < C * TILE && r < L;
      pu[q] = in ? u[((size_t)(tok0 + r) * H + h) * dv + j0 + idx % TILE] : 0.f;
    }
    pg = tid < dk ? g[((size_t)(tok0 + L - 1) * H + h) * dk + tid] : 0.f;
  };
  if (nch > 0) fetch(0);
  __syncthreads();

  for (int ch = 0; ch < nch; ++ch) {
    const int tok0 = start + ch * C, L = min(C, end - tok0);
    const size_t cbase = ((size_t)(cid0 + ch) * H + h) * dk * dv;
    for (int idx = tid; idx < dk * TILE; idx += kThreads) {
      const int c = idx / TILE, jj = idx % TILE;
      s_chunks[cbase + (size_t)c * dv + j0 + jj] = S[c * TP + jj];
    }
#pragma unroll
    for (int q = 0; q < NP; ++q) {
      const int idx = q * kThreads + tid;
      if (idx < C * dk) {
        const int r = idx / dk, c = idx % dk;
        Wc[r * dkp + c] = pw[q];
        Kh[r * dkp + c] = pk[q];
      }
    }
#pragma unroll
    for (int q = 0; q < NU; ++q) {
      const int idx = q * kThreads + tid;
      if (idx < C * TILE) D[(idx / TILE) * TP + idx % TILE] = pu[q];
    }
    if (tid < dk) gam[tid] = __expf(pg);
    __syncthreads();
    if (ch + 1 < nch) fetch(ch + 1);
    {  // D = U - W S   (rows g8, g8 + 32; columns j8 + 8 b)
      float acc[2][NB];
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < NB; ++b) acc[a][b] = 0.f;
      #pragma unroll 4
      for (int c = 0; c < dk; ++c) {
        float sv[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) sv[b] = S[c * TP + j8 + 8 * b];
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          const int r = g8 + 32 * a;
          const float wv = r < C ? Wc[r * dkp + c] : 0.f;
#pragma unroll
          for (int b = 0; b < NB; ++b) acc[a][b] += wv * sv[b];
        }
      }
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        const int r = g8 + 32 * a;
        if (r < L) {
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            const int jj = j8 + 8 * b;
            const float dvl = D[r * TP + jj] - acc[a][b];
            D[r * TP + jj] = dvl;
            u[((size_t)(tok0 + r) * H + h) * dv + j0 + jj] = dvl;
          }
        }
      }
    }
    __syncthreads();
    {  // S <- Diag(exp(g_C)) S + Kh^T D   (rows g8 + 32 a; columns j8 + 8 b)
      float acc[4][NB];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < NB; ++b) acc[a][b] = 0.f;
      #pragma unroll 4
      for (int r = 0; r < L; ++r) {
        float dvv[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) dvv[b] = D[r * TP + j8 + 8 * b];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          if (a < NA) {
            const float khv = Kh[r * dkp + g8 + 32 * a];
#pragma unroll
            for (int b = 0; b < NB; ++b) acc[a][b] += khv * dvv[b];
          }
        }
      }
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        if (a < NA) {
          const int c = g8 + 32 * a;
          const float ga = gam[c];
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            const int i = c * TP + j8 + 8 * b;
            S[i] = ga * S[i] + acc[a][b];
          }
        }
      }
    }
    __syncthreads();
  }
  for (int idx = tid; idx < dk * TILE; idx += kThreads) {
    const int c = idx / TILE, jj = idx % TILE;
    s_final[sbase + (size_t)c * dv + j0 + jj] = S[c * TP + jj];
  }
}

// (4) O = Qt S_0 + lower_incl(Qt Kb^T) D, per chunk and 32-column tile.
template <typename IO>
__global__ void __launch_bounds__(kThreads)
    output_kernel(const IO* __restrict__ q, const IO* __restrict__ k,
                  const float* __restrict__ g, const float* __restrict__ d,
                  const float* __restrict__ s_chunks, IO* __restrict__ out,
                  const int32_t* cu, const int32_t* chunk_off, int n_seqs,
                  int T, int H, int dk, int dv, int C) {
  const int cid = blockIdx.x;
  int seq, tok0, L;
  if (!locate_chunk(cid, cu, chunk_off, n_seqs, T, C, &seq, &tok0, &L)) return;
  const int h = blockIdx.y, j0 = blockIdx.z * kDvTile, tid = threadIdx.x;
  extern __shared__ float sm[];
  const int ldk = dk + 1;         // padded rows: no bank conflicts
  float* Qt = sm;                 // [C][ldk]
  float* Kb = Qt + C * ldk;       // [C][ldk]
  float* P = Kb + C * ldk;        // [C][C]
  float* S = P + C * C;           // [dk][kDvTile]
  float* D = S + dk * kDvTile;    // [C][kDvTile]
  float* rho = D + C * kDvTile;   // [dk] reference of the P factorisation

  for (int c = tid; c < dk; c += kThreads)
    rho[c] = decay_ref(g[((size_t)(tok0 + L - 1) * H + h) * dk + c]);
  __syncthreads();
  // Qt holds q exp(g - rho), Kb k exp(rho - g); the state rows are scaled by
  // exp(rho) so that Qt S is the chunk-start q exp(g) S.
  for (int idx = tid; idx < C * dk; idx += kThreads) {
    const int r = idx / dk, c = idx % dk;
    float qt = 0.f, kb = 0.f;
    if (r < L) {
      const size_t gi = ((size_t)(tok0 + r) * H + h) * dk + c;
      const float gv = g[gi];
      qt = to_f32(q[gi]) * __expf(gv - rho[c]);
      kb = to_f32(k[gi]) * __expf(rho[c] - gv);
    }
    Qt[r * ldk + c] = qt;
    Kb[r * ldk + c] = kb;
  }
  const size_t cbase = ((size_t)cid * H + h) * dk * dv;
  for (int idx = tid; idx < dk * kDvTile; idx += kThreads) {
    const int c = idx / kDvTile, jj = idx % kDvTile;
    S[idx] = s_chunks[cbase + (size_t)c * dv + j0 + jj] * __expf(rho[c]);
  }
  for (int idx = tid; idx < C * kDvTile; idx += kThreads) {
    const int r = idx / kDvTile, jj = idx % kDvTile;
    D[idx] = r < L ? d[((size_t)(tok0 + r) * H + h) * dv + j0 + jj] : 0.f;
  }
  __syncthreads();
  for (int idx = tid; idx < C * C; idx += kThreads) {
    const int r = idx / C, i = idx % C;
    float acc = 0.f;
    if (i <= r)
      for (int c = 0; c < dk; ++c) acc += Qt[r * ldk + c] * Kb[i * ldk + c];
    P[idx] = acc;
  }
  __syncthreads();
  for (int idx = tid; idx < L * kDvTile; idx += kThreads) {
    const int r = idx / kDvTile, jj = idx % kDvTile;
    float acc = 0.f;
    for (int c = 0; c < dk; ++c) acc += Qt[r * ldk + c] * S[c * kDvTile + jj];
    for (int i = 0; i <= r; ++i) acc += P[r * C + i] * D[i * kDvTile + jj];
    out[((size_t)(tok0 + r) * H + h) * dv + j0 + jj] = from_f32<IO>(acc);
  }
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)bytes);
}

// Which stages run: all four (the forward), or the pieces the backward pass
// wraps around its own per-chunk preparation (the plan and the cumulative
// log-decay first, the state pass after W and U are in place).
enum class Part { kAll, kPrefix, kStatePass };

template <typename IO>
cudaError_t run(const ChunkArgs& a, void* workspace, cudaStream_t stream,
                Part part = Part::kAll) {
  Ws w = carve(a, workspace, nullptr);
  const int C = a.chunk, H = a.H, dk = a.dk, dv = a.dv;
  const int64_t nch = max_chunks(a);
  const int32_t* cu = a.cu_seqlens;
  const IO* q = static_cast<const IO*>(a.q);
  const IO* k = static_cast<const IO*>(a.k);
  const IO* v = static_cast<const IO*>(a.v);
  IO* out = static_cast<IO*>(a.out);
  cudaError_t e;

  if (part != Part::kStatePass) {
    if (cu) {
      plan_kernel<<<1, 32, 0, stream>>>(cu, a.n_seqs, a.T, C, w.chunk_off);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (nch > 0) {
      cumsum_kernel<<<dim3((unsigned)nch, H), dk, 0, stream>>>(
          a.log_alpha, w.g, cu, w.chunk_off, a.n_seqs, a.T, H, dk, C, a.gate);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (part == Part::kPrefix) return cudaSuccess;
  }
  if (part == Part::kAll && nch > 0) {
    const dim3 grid((unsigned)nch, H);

    const size_t sm2 = 4 * ((size_t)2 * C * (dk + 1) + (size_t)C * dv +
                            2 * 64 * ws::kFS + 1024 + C + 2 * dk);
    if ((e = set_smem(intra_kernel<IO>, sm2)) != cudaSuccess) return e;
    intra_kernel<IO><<<grid, kThreads, sm2, stream>>>(
        k, v, a.beta, w.g, w.w, w.u, w.kh, cu, w.chunk_off, a.n_seqs, a.T, H,
        dk, dv, C);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    const int tile = dv >= 64 ? 64 : 32, tp = tile + 1;
    const size_t sm3 = 4 * ((size_t)dk * tp + 2 * (size_t)C * (dk + 1) +
                            (size_t)C * tp + dk);
    const dim3 sgrid(a.n_seqs, H, dv / tile);
    if (tile == 64) {
      if ((e = set_smem(state_kernel<64>, sm3)) != cudaSuccess) return e;
      state_kernel<64><<<sgrid, kThreads, sm3, stream>>>(
          w.g, w.w, w.kh, w.u, w.s, a.initial_state, a.final_state, cu,
          w.chunk_off, a.n_seqs, a.T, H, dk, dv, C);
    } else {
      if ((e = set_smem(state_kernel<32>, sm3)) != cudaSuccess) return e;
      state_kernel<32><<<sgrid, kThreads, sm3, stream>>>(
          w.g, w.w, w.kh, w.u, w.s, a.initial_state, a.final_state, cu,
          w.chunk_off, a.n_seqs, a.T, H, dk, dv, C);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }

  if (nch > 0 && part == Part::kAll) {
    const size_t sm4 = 4 * (2 * (size_t)C * (dk + 1) + (size_t)C * C +
                            (size_t)dk * kDvTile + (size_t)C * kDvTile + dk);
    if ((e = set_smem(output_kernel<IO>, sm4)) != cudaSuccess) return e;
    output_kernel<IO><<<dim3((unsigned)nch, H, dv / kDvTile), kThreads, sm4,
                        stream>>>(q, k, w.g, w.u, w.s, out, cu, w.chunk_off,
                                  a.n_seqs, a.T, H, dk, dv, C);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

size_t staged_workspace_bytes(const ChunkArgs& a) {
  size_t total = 0;
  carve(a, nullptr, &total);
  return total;
}

size_t staged_prefix_bytes(const ChunkArgs& a) {
  size_t total = 0, prefix = 0;
  carve(a, nullptr, &total, &prefix);
  return prefix;
}

int staged_kernel_count(const ChunkArgs& a) {
  if (a.n_seqs == 0) return 0;
  const bool any_chunks = max_chunks(a) > 0;
  return (a.cu_seqlens ? 1 : 0) + 1 + (any_chunks ? 3 : 0) +
         (has_prologue(a) && any_chunks ? 1 : 0);
}

cudaError_t launch_staged_part(const ChunkArgs& a, void* workspace,
                               StagedView* view, bool state_pass,
                               cudaStream_t stream) {
  Ws w = carve(a, workspace, nullptr);
  view->chunk_off = w.chunk_off;
  view->g = w.g;
  view->w = w.w;
  view->d = w.u;
  view->kh = w.kh;
  view->s = w.s;
  if (a.n_seqs == 0 || a.H == 0) return cudaSuccess;
  const Part part = state_pass ? Part::kStatePass : Part::kPrefix;
  return a.bf16 ? run<__nv_bfloat16>(a, workspace, stream, part)
                : run<float>(a, workspace, stream, part);
}

cudaError_t staged_take_range(cudaStream_t stream, int* flag) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  if ((e = cudaMemcpyFromSymbol(flag, g_staged_range, sizeof(int))) !=
      cudaSuccess)
    return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_staged_range, &zero, sizeof(int));
}

cudaError_t launch_staged(const ChunkArgs& a, void* workspace,
                          cudaStream_t stream) {
  if (a.n_seqs == 0 || a.H == 0) return cudaSuccess;
  if (!has_prologue(a))
    return a.bf16 ? run<__nv_bfloat16>(a, workspace, stream)
                  : run<float>(a, workspace, stream);
  // Input prologue first, into the workspace; then the four stages read the
  // prepared q, k and log(alpha).
  Ws w = carve(a, workspace, nullptr);
  const size_t tokens =
      a.cu_seqlens ? (size_t)a.T : (size_t)a.n_seqs * (size_t)a.T;
  if (tokens > 0) {
    const unsigned grid = (unsigned)(tokens * a.H);
    if (a.bf16)
      prologue_kernel<__nv_bfloat16><<<grid, 32, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(a.q),
          static_cast<const __nv_bfloat16*>(a.k), a.log_alpha,
          static_cast<__nv_bfloat16*>(w.qn), static_cast<__nv_bfloat16*>(w.kn),
          w.lan, a.H, a.dk, a.gate, a.pro);
    else
      prologue_kernel<float><<<grid, 32, 0, stream>>>(
          static_cast<const float*>(a.q), static_cast<const float*>(a.k),
          a.log_alpha, static_cast<float*>(w.qn), static_cast<float*>(w.kn),
          w.lan, a.H, a.dk, a.gate, a.pro);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  ChunkArgs b = a;
  b.q = w.qn;
  b.k = w.kn;
  b.log_alpha = a.gate == kGateNone ? nullptr : w.lan;
  b.pro = Prologue{};
  // b's workspace is the part of ours after the prologue outputs
  size_t pre = 0;
  {
    ChunkArgs c = a;
    c.pro = Prologue{};
    size_t whole = 0, rest = 0;
    carve(a, nullptr, &whole);
    carve(c, nullptr, &rest);
    pre = whole - rest;
  }
  void* rest_ws = static_cast<char*>(workspace) + pre;
  return a.bf16 ? run<__nv_bfloat16>(b, rest_ws, stream)
                : run<float>(b, rest_ws, stream);
}

}  // namespace kda
