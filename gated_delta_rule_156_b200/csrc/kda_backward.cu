// Chunkwise backward pass of the KDA forward, all arithmetic in fp32 (SIMT).
//
// The gradients of L = <dO, O> + <dS_T, S_T> follow from the chain rule
// applied to each line of the chunkwise forward (the forward's own chunk
// factorisation, "You Could Have Come Up with Kimi Delta Attention",
// daily.dev, Summary; the pages motivate the chunkwise form for training but
// print no gradient).  Per chunk, with S_0 the chunk-start state, dS_C the
// gradient of the state leaving the chunk and g the cumulative log-decay:
//   Kt = k e^g, Kb = k e^-g, Qt = q e^g, gam = e^{g_C}, M = Kt Kb^T,
//   Tm = (I + strictly_lower(Diag(b) M))^-1, W = Tm Diag(b) Kt,
//   Delta = Tm Diag(b) V - W S_0, P = lower_incl(Qt Kb^T)
//   G      = Diag(gam) dS_C
//   dDelta = Kb G + P^T dO
//   dS_0   = G + Qt^T dO - W^T dDelta            (the serial chain, in reverse)
//   d gam  = rowsum((S_0 + Kb^T Delta) * dS_C)
//   dP  = lower_incl(dO Delta^T)
//   dQt = dO S_0^T + dP Kb
//   dKb = Delta G^T + dP^T Qt + dA^T Diag(b) Kt
//   dW  = -dDelta S_0^T
//   dTm = dW (b Kt)^T + dDelta (b V)^T
//   dA  = strictly_lower(-Tm^T dTm Tm^T)
//   dKt = b (Tm^T dW + dA Kb),  dV = b Tm^T dDelta
//   db  = rowsum(Tm^T dW * Kt) + rowsum(Tm^T dDelta * V) + rowsum(dA * M)
//   dk  = dKt e^g + dKb e^-g,  dq = dQt e^g
//   dg  = dKt * Kt + dQt * Qt - dKb * Kb  (+ gam * d gam on the last row)
//   dlog_alpha = reverse cumulative sum of dg within the chunk
// The forward quantities come from stages (1)-(3) of the four-stage forward
// (g, W, Delta, chunk-start states).  A prep kernel forms Kt, Kb, Qt, M, P and
// Tm per chunk; the reverse chain runs per (sequence, head, 32-column d_v
// tile); the remaining products are batched small matrix products over every
// (chunk, head) with all operands staged in shared memory; a last kernel
// combines them into the input gradients.  Channel gate, no input prologue.
#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_inverse.cuh"

namespace kda {

namespace {

constexpr int kThreads = 256;
constexpr int kDvTile = 32;

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct BwdWs {
  StagedView fv;
  void* staged;                   // the forward's workspace
  float* fin;                     // scratch final state of the forward
  float *kt, *kb, *qt, *bkt;      // [tokens, H, dk]
  float *v32, *bv, *do32, *dd;    // [tokens, H, dv]
  float *tm, *mm, *pp;            // [chunks, H, C, C]
  float *gam;                     // [chunks, H, dk]
  float *gst;                     // G = Diag(gam) dS_C, [chunks, H, dk, dv]
  float *dgam;                    // [chunks, H, dv / 32, dk] partial sums
  float *dp, *dtm, *tmp, *da;     // [chunks, H, C, C]
  float *dqt, *dkb, *dw, *dbk, *y1;  // [tokens, H, dk]
  float *dbv;                     // [tokens, H, dv]
};

ChunkArgs forward_args(const BwdArgs& a, float* fin) {
  ChunkArgs f = a.f;
  f.out = nullptr;
  f.final_state = fin;
  f.gate = kGateChannel;
  f.pro = Prologue{};
  return f;
}

BwdWs carve_bwd(const BwdArgs& a, void* base, size_t* total) {
  const ChunkArgs& f = a.f;
  const size_t tokens =
      f.cu_seqlens ? (size_t)f.T : (size_t)f.n_seqs * (size_t)f.T;
  const size_t H = f.H, dk = f.dk, dv = f.dv, C = f.chunk;
  const size_t nch = (size_t)max_chunks(f);
  size_t off = 0;
  char* p = static_cast<char*>(base);
  auto take = [&](size_t bytes) {
    char* r = p ? p + off : nullptr;
    off = align256(off + bytes);
    return reinterpret_cast<float*>(r);
  };
  BwdWs w{};
  w.fin = take(4 * (size_t)f.n_seqs * H * dk * dv);
  const ChunkArgs fa = forward_args(a, nullptr);
  w.staged = take(staged_workspace_bytes(fa));
  const size_t tdk = 4 * tokens * H * dk, tdv = 4 * tokens * H * dv;
  const size_t sq = 4 * nch * H * C * C, st = 4 * nch * H * dk * dv;
  w.kt = take(tdk); w.kb = take(tdk); w.qt = take(tdk); w.bkt = take(tdk);
  w.v32 = take(tdv); w.bv = take(tdv); w.do32 = take(tdv); w.dd = take(tdv);
  w.tm = take(sq); w.mm = take(sq); w.pp = take(sq);
  w.gam = take(4 * nch * H * dk);
  w.gst = take(st);
  w.dgam = take(4 * nch * H * (dv / kDvTile) * dk);
  w.dp = take(sq); w.dtm = take(sq); w.tmp = take(sq); w.da = take(sq);
  w.dqt = take(tdk); w.dkb = take(tdk); w.dw = take(tdk); w.dbk = take(tdk);
  w.y1 = take(tdk);
  w.dbv = take(tdv);
  if (total) *total = off;
  return w;
}

// Per (chunk, head): Kt, Kb, Qt, b Kt and fp32 copies of V, b V, dO; gam;
// M = Kt Kb^T (strictly lower), P = lower_incl(Qt Kb^T) and
// Tm = (I + Diag(b) M)^-1 by forward substitution (one column per thread).
template <typename IO>
__global__ void __launch_bounds__(kThreads)
    prep_kernel(const IO* __restrict__ q, const IO* __restrict__ k,
                const IO* __restrict__ v, const float* __restrict__ beta,
                const IO* __restrict__ dout, const float* __restrict__ g,
                BwdWs w, const int32_t* cu, const int32_t* chunk_off, int n_seqs,
                int T, int H, int dk, int dv, int C) {
  const int cid = blockIdx.x;
  int seq, tok0, L;
  if (!locate_chunk(cid, cu, chunk_off, n_seqs, T, C, &seq, &tok0, &L)) return;
  const int h = blockIdx.y, tid = threadIdx.x;
  extern __shared__ float sm[];
  const int ldk = dk + 1;          // padded rows: no bank conflicts
  float* Kt = sm;                  // [C][ldk]
  float* Kb = Kt + C * ldk;        // [C][ldk]
  float* Qt = Kb + C * ldk;        // [C][ldk]
  float* A = Qt + C * ldk;         // [64][kFS] b M, zero-padded past C
  float* Tm = A + 64 * ws::kFS;    // [64][kFS]
  float* Msc = Tm + 64 * ws::kFS;  // [1024] scratch of the inverse
  float* bs = Msc + 1024;          // [C]

  for (int r = tid; r < C; r += kThreads)
    bs[r] = r < L ? beta[(size_t)(tok0 + r) * H + h] : 0.f;
  __syncthreads();
  for (int idx = tid; idx < C * dk; idx += kThreads) {
    const int r = idx / dk, c = idx % dk;
    float kt = 0.f, kb = 0.f, qt = 0.f;
    if (r < L) {
      const size_t gi = ((size_t)(tok0 + r) * H + h) * dk + c;
      const float kv = to_f32(k[gi]), qv = to_f32(q[gi]), gv = g[gi];
      const float e = __expf(gv), ie = __expf(-gv);
      kt = kv * e;
      kb = kv * ie;
      qt = qv * e;
      w.kt[gi] = kt;
      w.kb[gi] = kb;
      w.qt[gi] = qt;
      w.bkt[gi] = bs[r] * kt;
    }
    Kt[r * ldk + c] = kt;
    Kb[r * ldk + c] = kb;
    Qt[r * ldk + c] = qt;
  }
  for (int idx = tid; idx < L * dv; idx += kThreads) {
    const int r = idx / dv, j = idx % dv;
    const size_t gi = ((size_t)(tok0 + r) * H + h) * dv + j;
    const float vv = to_f32(v[gi]);
    w.v32[gi] = vv;
    w.bv[gi] = bs[r] * vv;
    w.do32[gi] = to_f32(dout[gi]);
  }
  for (int c = tid; c < dk; c += kThreads)
    w.gam[((size_t)cid * H + h) * dk + c] =
        __expf(g[((size_t)(tok0 + L - 1) * H + h) * dk + c]);
  __syncthreads();
  const size_t sqb = ((size_t)cid * H + h) * C * C;
  for (int idx = tid; idx < 64 * ws::kFS; idx += kThreads) {
    A[idx] = 0.f;
    Tm[idx] = 0.f;
  }
  __syncthreads();
  for (int idx = tid; idx < C * C; idx += kThreads) {
    const int r = idx / C, i = idx % C;
    float m = 0.f, pv = 0.f;
    if (r < L && i <= r) {
      for (int c = 0; c < dk; ++c) pv += Qt[r * ldk + c] * Kb[i * ldk + c];
      if (i < r)
        for (int c = 0; c < dk; ++c) m += Kt[r * ldk + c] * Kb[i * ldk + c];
    }
    A[r * ws::kFS + i] = bs[r] * m;
    w.mm[sqb + idx] = m;
    w.pp[sqb + idx] = i <= r ? pv : 0.f;
  }
  __syncthreads();
  // Tm = (I + Diag(b) M)^-1 by recursive doubling (identity past C)
  ws::invert_unit_lower(A, Tm, Msc, tid);
  __syncthreads();
  for (int idx = tid; idx < C * C; idx += kThreads)
    w.tm[sqb + idx] = Tm[(idx / C) * ws::kFS + idx % C];
}

// The reverse chain over one sequence's chunks for one head and one 32-column
// tile of d_v.  Per chunk (last first), with dS the gradient of the state
// leaving it: partial d gam, G = Diag(gam) dS (stored), dDelta = Kb G + P^T dO
// (stored), then dS <- G + Qt^T dO - W^T dDelta.  Each product gives every
// thread a block of outputs (rows strided by 32, columns by 8) so that the
// sums over the contraction index run as independent chains; the shared rows
// are padded (33 floats for the 32-wide tiles, d_k + 1 for the token rows)
// so both access directions are free of bank conflicts.
constexpr int kTp = kDvTile + 1;

__global__ void __launch_bounds__(kThreads)
    chain_kernel(BwdWs w, const float* __restrict__ d_final,
                 float* __restrict__ d_init, const int32_t* cu, int n_seqs,
                 int T, int H, int dk, int dv, int C) {
  const int seq = blockIdx.x, h = blockIdx.y, tile = blockIdx.z;
  const int j0 = tile * kDvTile, tid = threadIdx.x, ntile = dv / kDvTile;
  const int dkp = dk + 1, NA = dk / 32;
  const int g8 = tid >> 3, j8 = tid & 7;  // row group, column group
  extern __shared__ float sm[];
  float* dS = sm;                    // [dk][kTp]
  float* S0 = dS + dk * kTp;         // [dk][kTp]
  float* Kb = S0 + dk * kTp;         // [C][dkp]
  float* Qt = Kb + C * dkp;          // [C][dkp]
  float* Wc = Qt + C * dkp;          // [C][dkp]
  float* P = Wc + C * dkp;           // [C][C]
  float* dO = P + C * C;             // [C][kTp]
  float* De = dO + C * kTp;          // [C][kTp] Delta
  float* dD = De + C * kTp;          // [C][kTp] dDelta
  float* gC = dD + C * kTp;          // [dk]

  const size_t sbase = ((size_t)seq * H + h) * dk * dv;
  for (int idx = tid; idx < dk * kDvTile; idx += kThreads) {
    const int c = idx / kDvTile, jj = idx % kDvTile;
    dS[c * kTp + jj] = d_final ? d_final[sbase + (size_t)c * dv + j0 + jj] : 0.f;
  }
  int start, end;
  seq_range(cu, seq, T, &start, &end);
  const int nch = (end - start + C - 1) / C;
  const int cid0 = cu ? w.fv.chunk_off[seq] : seq * ((T + C - 1) / C);
  __syncthreads();

  for (int ch = nch - 1; ch >= 0; --ch) {
    const int cid = cid0 + ch, tok0 = start + ch * C, L = min(C, end - tok0);
    const size_t cbase = ((size_t)cid * H + h) * dk * dv;
    // staging loads batched eight deep so their latencies overlap
    for (int base = 0; base < C * dk; base += 8 * kThreads) {
      float kb[8], qt[8], wv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int idx = base + u * kThreads + tid;
        const int r = idx / dk, c = idx % dk;
        kb[u] = qt[u] = wv[u] = 0.f;
        if (idx < C * dk && r < L) {
          const size_t gi = ((size_t)(tok0 + r) * H + h) * dk + c;
          kb[u] = w.kb[gi];
          qt[u] = w.qt[gi];
          wv[u] = w.fv.w[gi];
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int idx = base + u * kThreads + tid;
        if (idx < C * dk) {
          const int r = idx / dk, c = idx % dk;
          Kb[r * dkp + c] = kb[u];
          Qt[r * dkp + c] = qt[u];
          Wc[r * dkp + c] = wv[u];
        }
      }
    }
    for (int idx = tid; idx < C * C; idx += kThreads)
      P[idx] = w.pp[((size_t)cid * H + h) * C * C + idx];
    {
      float o[8], de[8], s0[16];
#pragma unroll
      for (int u = 0; u < 8; ++u) {  // C * 32 <= 8 * kThreads
        const int idx = u * kThreads + tid;
        const int r = idx / kDvTile, jj = idx % kDvTile;
        o[u] = de[u] = 0.f;
        if (idx < C * kDvTile && r < L) {
          const size_t gi = ((size_t)(tok0 + r) * H + h) * dv + j0 + jj;
          o[u] = w.do32[gi];
          de[u] = w.fv.d[gi];
        }
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {  // dk * 32 <= 16 * kThreads
        const int idx = u * kThreads + tid;
        const int c = idx / kDvTile, jj = idx % kDvTile;
        s0[u] = idx < dk * kDvTile ? w.fv.s[cbase + (size_t)c * dv + j0 + jj] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int idx = u * kThreads + tid;
        if (idx < C * kDvTile) {
          const int r = idx / kDvTile, jj = idx % kDvTile;
          dO[r * kTp + jj] = o[u];
          De[r * kTp + jj] = de[u];
        }
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int idx = u * kThreads + tid;
        if (idx < dk * kDvTile) S0[(idx / kDvTile) * kTp + idx % kDvTile] = s0[u];
      }
    }
    for (int c = tid; c < dk; c += kThreads)
      gC[c] = w.gam[((size_t)cid * H + h) * dk + c];
    __syncthreads();

    // partial d gam over this tile: rowsum((S_0 + Kb^T Delta) * dS)
    {
      float x[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) x[a][b] = 0.f;
      for (int r = 0; r < L; ++r) {
        float de[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) de[b] = De[r * kTp + j8 + 8 * b];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          if (a < NA) {
            const float kb = Kb[r * dkp + g8 + 32 * a];
#pragma unroll
            for (int b = 0; b < 4; ++b) x[a][b] += kb * de[b];
          }
        }
      }
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        if (a < NA) {
          const int c = g8 + 32 * a;
          float part = 0.f;
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int jj = j8 + 8 * b;
            part += (S0[c * kTp + jj] + x[a][b]) * dS[c * kTp + jj];
          }
          part += __shfl_xor_sync(0xffffffffu, part, 1);
          part += __shfl_xor_sync(0xffffffffu, part, 2);
          part += __shfl_xor_sync(0xffffffffu, part, 4);
          if (j8 == 0)
            w.dgam[(((size_t)cid * H + h) * ntile + tile) * dk + c] = part;
        }
      }
    }
    __syncthreads();
    for (int idx = tid; idx < dk * kDvTile; idx += kThreads) {
      const int c = idx / kDvTile, jj = idx % kDvTile;
      const float gv = gC[c] * dS[c * kTp + jj];
      dS[c * kTp + jj] = gv;
      w.gst[cbase + (size_t)c * dv + j0 + jj] = gv;
    }
    __syncthreads();
    // dDelta = Kb G + P^T dO  (rows g8, g8 + 32)
    {
      float acc[2][4];
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
      for (int c = 0; c < dk; ++c) {
        float gv[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) gv[b] = dS[c * kTp + j8 + 8 * b];
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          const int r = g8 + 32 * a;  // Kb rows past L are zero, past C absent
          const float kb = r < C ? Kb[r * dkp + c] : 0.f;
#pragma unroll
          for (int b = 0; b < 4; ++b) acc[a][b] += kb * gv[b];
        }
      }
      for (int i = 0; i < L; ++i) {
        float o[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) o[b] = dO[i * kTp + j8 + 8 * b];
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          const int r = g8 + 32 * a;
          const float pv = r < C ? P[i * C + r] : 0.f;
#pragma unroll
          for (int b = 0; b < 4; ++b) acc[a][b] += pv * o[b];
        }
      }
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        const int r = g8 + 32 * a;
        if (r < C) {
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int jj = j8 + 8 * b;
            const float v = r < L ? acc[a][b] : 0.f;
            dD[r * kTp + jj] = v;
            if (r < L) w.dd[((size_t)(tok0 + r) * H + h) * dv + j0 + jj] = v;
          }
        }
      }
    }
    __syncthreads();
    // dS <- G + Qt^T dO - W^T dDelta
    {
      float acc[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
      for (int r = 0; r < L; ++r) {
        float o[4], dd[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          o[b] = dO[r * kTp + j8 + 8 * b];
          dd[b] = dD[r * kTp + j8 + 8 * b];
        }
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          if (a < NA) {
            const float qt = Qt[r * dkp + g8 + 32 * a];
            const float wv = Wc[r * dkp + g8 + 32 * a];
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[a][b] += qt * o[b] - wv * dd[b];
          }
        }
      }
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        if (a < NA) {
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int i = (g8 + 32 * a) * kTp + j8 + 8 * b;
            dS[i] += acc[a][b];
          }
        }
      }
    }
    __syncthreads();
  }
  if (d_init) {
    for (int idx = tid; idx < dk * kDvTile; idx += kThreads) {
      const int c = idx / kDvTile, jj = idx % kDvTile;
      d_init[sbase + (size_t)c * dv + j0 + jj] = dS[c * kTp + jj];
    }
  }
}

// ---------------------------------------------------------------------------
// Batched small products over every (chunk, head): Out (m x n) = alpha op(A)
// op(B) (+ Out), with op = transpose or not and an optional lower-triangular
// mask on Out.  An operand is one of: token rows [tokens, H, cols] (rows are
// the chunk's tokens, zero past its length), a per-chunk square [chunks, H,
// C, C], or a per-chunk state [chunks, H, dk, dv].  Both operands are staged
// whole in shared memory (m, n, k <= 128); each thread owns an up to 8 x 8
// block of Out strided by 16 in both directions.
enum MatKind { kTok = 0, kSq = 1, kState = 2 };
enum Dim { kDimL = 0, kDimDk = 1, kDimDv = 2 };
enum Mask { kMaskNone = 0, kMaskLowerIncl = 1, kMaskStrictLower = 2 };

struct MatRef {
  float* p;
  int kind;
  int cols;    // kTok: row width; kSq: C; kState: dv
  int trans;
};

struct BmmOp {
  MatRef out, a, b;
  int m, n, k;     // Dim codes
  int mask;
  float alpha;
  int accumulate;
  int md, nd, kd;  // the largest m, n, k can be (row widths of the staging)
};

__device__ __forceinline__ int dim_of(int code, int L, int dk, int dv) {
  return code == kDimL ? L : code == kDimDk ? dk : dv;
}

__device__ __forceinline__ size_t elem_off(const MatRef& x, int r, int c,
                                           int cid, int h, int tok0, int H,
                                           int C, int dk) {
  if (x.kind == kTok) return ((size_t)(tok0 + r) * H + h) * x.cols + c;
  if (x.kind == kSq) return (((size_t)cid * H + h) * C + r) * C + c;
  return (((size_t)cid * H + h) * dk + r) * x.cols + c;
}

// op(A) is staged transposed (AT[t][i]) and op(B) as is (Bs[t][j]), both in
// the order the source is laid out in memory, with rows padded to a multiple
// of four floats; each thread then owns the 8 x 8 block of Out at rows
// 8 ti .. 8 ti + 7 and columns 8 tj .. 8 tj + 7, and every step of the
// contraction is four 16-byte shared loads for 64 FMAs.
__global__ void __launch_bounds__(kThreads)
    bmm_kernel(BmmOp op, const int32_t* cu, const int32_t* chunk_off, int n_seqs,
               int T, int H, int dk, int dv, int C) {
  const int cid = blockIdx.x;
  int seq, tok0, L;
  if (!locate_chunk(cid, cu, chunk_off, n_seqs, T, C, &seq, &tok0, &L)) return;
  const int h = blockIdx.y, tid = threadIdx.x;
  const int m = dim_of(op.m, L, dk, dv), n = dim_of(op.n, L, dk, dv);
  const int kk = dim_of(op.k, L, dk, dv);
  const int la = op.md + 4, lb = op.nd + 4;
  extern __shared__ __align__(16) float sm[];
  float* AT = sm;                 // [kd][la]
  float* Bs = sm + op.kd * la;    // [kd][lb]
  {
    // op(A)(i, t) = A(i, t) or A(t, i); walk the source row by row
    const int rows = op.a.trans ? kk : m, cols = op.a.trans ? m : kk;
    for (int idx = tid; idx < rows * cols; idx += kThreads) {
      const int r = idx / cols, c = idx % cols;
      const float x = op.a.p[elem_off(op.a, r, c, cid, h, tok0, H, C, dk)];
      if (op.a.trans) AT[r * la + c] = x;   // r = t, c = i
      else AT[c * la + r] = x;              // r = i, c = t
    }
  }
  {
    const int rows = op.b.trans ? n : kk, cols = op.b.trans ? kk : n;
    for (int idx = tid; idx < rows * cols; idx += kThreads) {
      const int r = idx / cols, c = idx % cols;
      const float x = op.b.p[elem_off(op.b, r, c, cid, h, tok0, H, C, dk)];
      if (op.b.trans) Bs[c * lb + r] = x;   // r = j, c = t
      else Bs[r * lb + c] = x;              // r = t, c = j
    }
  }
  __syncthreads();
  const int ti = tid >> 4, tj = tid & 15;
  if (8 * ti >= m || 8 * tj >= n) return;
  float acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
  const float* ap = AT + 8 * ti;
  const float* bp = Bs + 8 * tj;
  for (int t = 0; t < kk; ++t) {
    const float4 a0 = *reinterpret_cast<const float4*>(ap + t * la);
    const float4 a1 = *reinterpret_cast<const float4*>(ap + t * la + 4);
    const float4 b0 = *reinterpret_cast<const float4*>(bp + t * lb);
    const float4 b1 = *reinterpret_cast<const float4*>(bp + t * lb + 4);
    const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
      for (int b = 0; b < 8; ++b) acc[a][b] += av[a] * bv[b];
  }
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int i = 8 * ti + a;
    if (i >= m) continue;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      const int j = 8 * tj + b;
      if (j >= n) continue;
      float x = op.alpha * acc[a][b];
      if ((op.mask == kMaskLowerIncl && j > i) ||
          (op.mask == kMaskStrictLower && j >= i))
        x = 0.f;
      float* o = op.out.p + elem_off(op.out, i, j, cid, h, tok0, H, C, dk);
      *o = op.accumulate ? *o + x : x;
    }
  }
}

// Per (chunk, head): the input gradients from the products above.
template <typename IO>
__global__ void __launch_bounds__(kThreads)
    final_kernel(BwdWs w, const float* __restrict__ beta,
                 const float* __restrict__ g, IO* __restrict__ dq,
                 IO* __restrict__ dk_out, IO* __restrict__ dv_out,
                 float* __restrict__ dla, float* __restrict__ dbeta,
                 const int32_t* cu, const int32_t* chunk_off, int n_seqs, int T,
                 int H, int dk, int dv, int C) {
  const int cid = blockIdx.x;
  int seq, tok0, L;
  if (!locate_chunk(cid, cu, chunk_off, n_seqs, T, C, &seq, &tok0, &L)) return;
  const int h = blockIdx.y, tid = threadIdx.x, ntile = dv / kDvTile;
  extern __shared__ float sm[];
  float* dg = sm;  // [C][dk]
  for (int idx = tid; idx < L * dk; idx += kThreads) {
    const int r = idx / dk;
    const size_t gi = ((size_t)(tok0 + r) * H + h) * dk + idx % dk;
    const float b = beta[(size_t)(tok0 + r) * H + h];
    const float dKt = b * (w.dbk[gi] + w.y1[gi]);
    const float dKb = w.dkb[gi], dQt = w.dqt[gi];
    const float gv = g[gi], e = __expf(gv), ie = __expf(-gv);
    dk_out[gi] = from_f32<IO>(dKt * e + dKb * ie);
    dq[gi] = from_f32<IO>(dQt * e);
    dg[idx] = dKt * w.kt[gi] + dQt * w.qt[gi] - dKb * w.kb[gi];
  }
  for (int idx = tid; idx < L * dv; idx += kThreads) {
    const int r = idx / dv;
    const size_t gi = ((size_t)(tok0 + r) * H + h) * dv + idx % dv;
    dv_out[gi] = from_f32<IO>(beta[(size_t)(tok0 + r) * H + h] * w.dbv[gi]);
  }
  __syncthreads();
  for (int c = tid; c < dk; c += kThreads) {
    float dgm = 0.f;
    for (int t = 0; t < ntile; ++t)
      dgm += w.dgam[(((size_t)cid * H + h) * ntile + t) * dk + c];
    dg[(L - 1) * dk + c] += w.gam[((size_t)cid * H + h) * dk + c] * dgm;
    float acc = 0.f;
    for (int r = L - 1; r >= 0; --r) {
      acc += dg[r * dk + c];
      dla[((size_t)(tok0 + r) * H + h) * dk + c] = acc;
    }
  }
  const size_t sqb = ((size_t)cid * H + h) * C * C;
  for (int r = tid; r < L; r += kThreads) {
    const size_t rk = ((size_t)(tok0 + r) * H + h) * dk;
    const size_t rv = ((size_t)(tok0 + r) * H + h) * dv;
    float acc = 0.f;
    for (int c = 0; c < dk; ++c) acc += w.dbk[rk + c] * w.kt[rk + c];
    for (int j = 0; j < dv; ++j) acc += w.dbv[rv + j] * w.v32[rv + j];
    for (int i = 0; i < r; ++i) acc += w.da[sqb + r * C + i] * w.mm[sqb + r * C + i];
    dbeta[(size_t)(tok0 + r) * H + h] = acc;
  }
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)bytes);
}

template <typename IO>
cudaError_t run_bwd(const BwdArgs& a, void* workspace, cudaStream_t stream) {
  BwdWs w = carve_bwd(a, workspace, nullptr);
  const ChunkArgs f = forward_args(a, w.fin);
  cudaError_t e = launch_staged_state(f, w.staged, &w.fv, stream);
  if (e != cudaSuccess) return e;
  const int C = f.chunk, H = f.H, dk = f.dk, dv = f.dv;
  const int64_t nch = max_chunks(f);
  const int32_t* cu = f.cu_seqlens;
  const int32_t* co = w.fv.chunk_off;
  const dim3 grid((unsigned)(nch > 0 ? nch : 1), H);

  if (nch > 0) {
    const size_t smp = 4 * (3 * (size_t)C * (dk + 1) + 2 * 64 * ws::kFS + 1024 + C);
    if ((e = set_smem(prep_kernel<IO>, smp)) != cudaSuccess) return e;
    prep_kernel<IO><<<grid, kThreads, smp, stream>>>(
        static_cast<const IO*>(f.q), static_cast<const IO*>(f.k),
        static_cast<const IO*>(f.v), f.beta, static_cast<const IO*>(a.d_out),
        w.fv.g, w, cu, co, f.n_seqs, f.T, H, dk, dv, C);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const size_t smc = 4 * (2 * (size_t)dk * kTp + 3 * (size_t)C * (dk + 1) +
                          (size_t)C * C + 3 * (size_t)C * kTp + dk);
  if ((e = set_smem(chain_kernel, smc)) != cudaSuccess) return e;
  chain_kernel<<<dim3(f.n_seqs, H, dv / kDvTile), kThreads, smc, stream>>>(
      w, a.d_final_state, a.d_initial_state, cu, f.n_seqs, f.T, H, dk, dv, C);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (nch == 0) return cudaSuccess;

  if ((e = set_smem(bmm_kernel, 4 * 2 * 128 * 132)) != cudaSuccess) return e;
  auto tok = [](float* p, int cols, int t = 0) { return MatRef{p, kTok, cols, t}; };
  auto sq = [&](float* p, int t = 0) { return MatRef{p, kSq, C, t}; };
  auto stt = [&](const float* p, int t = 0) {
    return MatRef{const_cast<float*>(p), kState, dv, t};
  };
  auto dmax = [&](int code) { return code == kDimL ? C : code == kDimDk ? dk : dv; };
  auto bmm = [&](MatRef o, MatRef x, MatRef y, int m, int n, int k, int mask,
                 float alpha, int accumulate) {
    const BmmOp op{o,     x,    y,          m,       n,       k,
                   mask,  alpha, accumulate, dmax(m), dmax(n), dmax(k)};
    const size_t smem =
        4 * (size_t)(dmax(k) * (dmax(m) + 4) + dmax(k) * (dmax(n) + 4));
    bmm_kernel<<<grid, kThreads, smem, stream>>>(op, cu, co, f.n_seqs, f.T, H,
                                                 dk, dv, C);
    return cudaGetLastError();
  };
  float* De = const_cast<float*>(w.fv.d);  // Delta
  const float* S0 = w.fv.s;
#define KDA_BMM(...) \
  if ((e = bmm(__VA_ARGS__)) != cudaSuccess) return e;
  // dP = lower_incl(dO Delta^T)
  KDA_BMM(sq(w.dp), tok(w.do32, dv), tok(De, dv, 1), kDimL, kDimL, kDimDv,
          kMaskLowerIncl, 1.f, 0)
  // dQt = dO S_0^T + dP Kb
  KDA_BMM(tok(w.dqt, dk), tok(w.do32, dv), stt(S0, 1), kDimL, kDimDk, kDimDv,
          kMaskNone, 1.f, 0)
  KDA_BMM(tok(w.dqt, dk), sq(w.dp), tok(w.kb, dk), kDimL, kDimDk, kDimL,
          kMaskNone, 1.f, 1)
  // dKb = Delta G^T + dP^T Qt  (+ dA^T b Kt below)
  KDA_BMM(tok(w.dkb, dk), tok(De, dv), stt(w.gst, 1), kDimL, kDimDk, kDimDv,
          kMaskNone, 1.f, 0)
  KDA_BMM(tok(w.dkb, dk), sq(w.dp, 1), tok(w.qt, dk), kDimL, kDimDk, kDimL,
          kMaskNone, 1.f, 1)
  // dW = -dDelta S_0^T
  KDA_BMM(tok(w.dw, dk), tok(w.dd, dv), stt(S0, 1), kDimL, kDimDk, kDimDv,
          kMaskNone, -1.f, 0)
  // dTm = dW (b Kt)^T + dDelta (b V)^T
  KDA_BMM(sq(w.dtm), tok(w.dw, dk), tok(w.bkt, dk, 1), kDimL, kDimL, kDimDk,
          kMaskNone, 1.f, 0)
  KDA_BMM(sq(w.dtm), tok(w.dd, dv), tok(w.bv, dv, 1), kDimL, kDimL, kDimDv,
          kMaskNone, 1.f, 1)
  // Tm^T dW, Tm^T dDelta, Tm^T dTm
  KDA_BMM(tok(w.dbk, dk), sq(w.tm, 1), tok(w.dw, dk), kDimL, kDimDk, kDimL,
          kMaskNone, 1.f, 0)
  KDA_BMM(tok(w.dbv, dv), sq(w.tm, 1), tok(w.dd, dv), kDimL, kDimDv, kDimL,
          kMaskNone, 1.f, 0)
  KDA_BMM(sq(w.tmp), sq(w.tm, 1), sq(w.dtm), kDimL, kDimL, kDimL, kMaskNone,
          1.f, 0)
  // dA = strictly_lower(-(Tm^T dTm) Tm^T)
  KDA_BMM(sq(w.da), sq(w.tmp), sq(w.tm, 1), kDimL, kDimL, kDimL,
          kMaskStrictLower, -1.f, 0)
  // dA Kb, and dKb += dA^T (b Kt)
  KDA_BMM(tok(w.y1, dk), sq(w.da), tok(w.kb, dk), kDimL, kDimDk, kDimL,
          kMaskNone, 1.f, 0)
  KDA_BMM(tok(w.dkb, dk), sq(w.da, 1), tok(w.bkt, dk), kDimL, kDimDk, kDimL,
          kMaskNone, 1.f, 1)
#undef KDA_BMM
  const size_t smf = 4 * (size_t)C * dk;
  if ((e = set_smem(final_kernel<IO>, smf)) != cudaSuccess) return e;
  final_kernel<IO><<<grid, kThreads, smf, stream>>>(
      w, f.beta, w.fv.g, static_cast<IO*>(a.dq), static_cast<IO*>(a.dk),
      static_cast<IO*>(a.dv), a.d_log_alpha, a.d_beta, cu, co, f.n_seqs, f.T,
      H, dk, dv, C);
  return cudaGetLastError();
}

constexpr int kBmmOps = 14;

}  // namespace

size_t bwd_workspace_bytes(const BwdArgs& a) {
  size_t total = 0;
  carve_bwd(a, nullptr, &total);
  return total;
}

int bwd_kernel_count(const BwdArgs& a) {
  const ChunkArgs f = forward_args(a, nullptr);
  if (f.n_seqs == 0 || f.H == 0) return 0;
  const bool any = max_chunks(f) > 0;
  // the forward's stages (1)-(3), the reverse chain, then prep, the batched
  // products and the final combination
  return staged_kernel_count(f) - (any ? 1 : 0) + 1 +
         (any ? 1 + kBmmOps + 1 : 0);
}

cudaError_t launch_bwd(const BwdArgs& a, void* workspace, cudaStream_t stream) {
  if (a.f.n_seqs == 0 || a.f.H == 0) return cudaSuccess;
  return a.f.bf16 ? run_bwd<__nv_bfloat16>(a, workspace, stream)
                  : run_bwd<float>(a, workspace, stream);
}

}  // namespace kda
