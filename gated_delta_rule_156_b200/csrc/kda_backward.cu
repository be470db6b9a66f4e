// Chunkwise backward pass of the KDA forward, in fp32 SIMT arithmetic except
// with bf16 inputs in 64-token chunks: there every product runs on the
// tensor cores in tf32 (prep and the batched products here, the forward's
// state pass and the reverse chain in kda_bwd_chain_tc.cuh; the state pass
// with high and low tf32 parts of its state and Delta).
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
//   db  = rowsum(Tm^T dW * Kt) + rowsum(Tm^T dDelta * V) + rowsum(dA * M),
//         where rowsum(dA * M) = rowsum((dA Kb) * Kt) since M = Kt Kb^T
//   dk  = dKt e^g + dKb e^-g,  dq = dQt e^g
//   dg  = dKt * Kt + dQt * Qt - dKb * Kb  (+ gam * d gam on the last row)
//   dlog_alpha = reverse cumulative sum of dg within the chunk
// Launch order:
//   - stage (1) of the four-stage forward (g);
//   - a prep kernel per (chunk, head): Kt, Kb, Qt, b Kt, P and Tm, plus the
//     forward's own W, U and Kh, so the forward's stage (2) is not run;
//   - the forward's state pass: Delta and every chunk-start state (stage 3
//     of the four-stage forward, or its tensor-core form);
//   - the two products that do not depend on dS, Qt^T dO and P^T dO;
//   - the reverse chain per (sequence, head, 32-column d_v tile; 64 columns
//     on the tensor cores), which
//     keeps only dDelta and the dS update in its serial loop and takes
//     gam * d gam = rowsum(S_next * dS_C) from the next chunk's start state
//     (S_next = Diag(gam)(S_0 + Kb^T Delta));
//   - the remaining products, batched over every (chunk, head) with their
//     operands staged in shared memory and merged into multi-term launches;
//   - a last kernel that combines them into the input gradients.
// Channel gate, no input prologue.
#include <algorithm>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "kda_inverse.cuh"
#include "kda_tmap.h"
#include "sm100_ptx.cuh"

namespace kda {

// Set when a chunk's decay exceeds the backward's range (read and cleared on
// the host).  The backward keeps the chunk-start factorisation (k e^g and
// k e^-g), which stays inside the fp32 range while |g_C| <= kBwdDecayMax.
__device__ int g_bwd_range = 0;
// Set when a bounded wait of the backward's tensor-core products gave up.
__device__ int g_bwd_timeout = 0;
constexpr float kBwdDecayMax = 80.f;

namespace {

constexpr int kThreads = 256;

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct BwdWs {
  StagedView fv;
  void* staged;                   // the forward's workspace
  float* fin;                     // scratch final state of the forward
  float* wt;                      // W^T per chunk [chunks, H, dk, C], or null
  // transposed per-chunk copies for the tensor-core products (or null):
  // [chunks, H, d, C], zero past each chunk's last token; ddT holds -dDelta^T
  float *qtT, *kbT, *bktT, *doT, *ddT;
  float* khT;  // Kh^T per chunk [chunks, H, dk, C] for the state pass, tf32
  float *kb, *qt, *bkt;           // [tokens, H, dk]; qt on the SIMT path only
  float *bv, *do32, *dd;          // [tokens, H, dv]
  float *tm, *pp;                 // [chunks, H, C, C]
  float *gam;                     // [chunks, H, dk]
  float *gst;                     // G = Diag(gam) dS_C, [chunks, H, dk, dv]
  float *dgam;                    // [chunks, H, dv / 32, dk] partials of gam * d gam
  float *dp, *dtm, *tmp, *da;     // [chunks, H, C, C]
  float *dqt, *dkb, *dw, *dbk;    // [tokens, H, dk]; dbk = Tm^T dW + dA Kb
  float *dbv;                     // [tokens, H, dv]
  float *qdo;                     // Qt^T dO, [chunks, H, dk, dv]
  float *pdo;                     // P^T dO, [tokens, H, dv]
};

ChunkArgs forward_args(const BwdArgs& a, float* fin) {
  ChunkArgs f = a.f;
  f.out = nullptr;
  f.final_state = fin;
  f.gate = kGateChannel;
  f.pro = Prologue{};
  return f;
}

// The tensor-core path (every product in tf32) where the shape allows it:
// bf16 inputs, 64-token chunks, d_k and d_v in {64, 128}, and rows of the
// per-chunk copies within a tensor map's signed 32-bit coordinates.  The
// state pass there keeps fp32-grade operands (high and low tf32 parts):
// with bf16 operands in the state (the two-pass forward's chain, tried)
// dlog_alpha missed the 1e-2 bar under strong gates (1.9e-2 for the
// undivided logsigmoid gate), where its reverse sum of differences amplifies
// the state's rounding.
bool tensor_chain(const ChunkArgs& f) {
  return fused_supported(f) && max_chunks(f) > 0 &&
         max_chunks(f) * f.H * (f.dk > f.dv ? f.dk : f.dv) < ((int64_t)1 << 31);
}

BwdWs carve_bwd(const BwdArgs& a, void* base, size_t* total,
                BwdArray* info = nullptr, int cap = 0, int* count = nullptr) {
  const ChunkArgs& f = a.f;
  const size_t tokens =
      f.cu_seqlens ? (size_t)f.T : (size_t)f.n_seqs * (size_t)f.T;
  const size_t H = f.H, dk = f.dk, dv = f.dv, C = f.chunk;
  const size_t nch = (size_t)max_chunks(f);
  const ChunkArgs fa = forward_args(a, nullptr);
  const size_t tdk = 4 * tokens * H * dk, tdv = 4 * tokens * H * dv;
  const size_t sq = 4 * nch * H * C * C, st = 4 * nch * H * dk * dv;
  const size_t fin = 4 * (size_t)f.n_seqs * H * dk * dv;
  const size_t gam = 4 * nch * H * dk, dgam = 4 * nch * H * (dv / 32) * dk;
  char* p = static_cast<char*>(base);
  BwdWs w{};
  if (!tensor_chain(fa)) {  // fp32 SIMT path: every array apart
    size_t off = 0;
    auto take = [&](size_t bytes) {
      char* r = p ? p + off : nullptr;
      off = align256(off + bytes);
      return reinterpret_cast<float*>(r);
    };
    w.fin = take(fin);
    w.staged = take(staged_workspace_bytes(fa));
    w.kb = take(tdk); w.qt = take(tdk); w.bkt = take(tdk);
    w.bv = take(tdv); w.do32 = take(tdv); w.dd = take(tdv);
    w.tm = take(sq); w.pp = take(sq);
    w.gam = take(gam);
    w.gst = take(st);
    w.dgam = take(dgam);
    w.dp = take(sq); w.dtm = take(sq); w.tmp = take(sq); w.da = take(sq);
    w.dqt = take(tdk); w.dkb = take(tdk); w.dw = take(tdk); w.dbk = take(tdk);
    w.dbv = take(tdv);
    w.qdo = take(st);
    w.pdo = take(tdv);
    if (total) *total = off;
    if (count) *count = 0;
    return w;
  }
  // Tensor-core path: arrays share memory where their lifetimes (from the
  // launch that first writes one to the last launch that reads it, both
  // included) do not overlap.  The launches, in order:
  enum {
    kPrefix,  // chunk offsets (packed layout), g
    kPrep,    // prep_tc_kernel
    kState,   // the forward's state pass
    kQdo, kPdo,
    kRev,     // reverse chain
    kDp, kDqt, kDw, kDtm, kDbv, kTmp, kDa, kDbk, kDkb,  // batched products
    kFinal
  };
  const size_t tk = 4 * nch * H * dk * C, tv = 4 * nch * H * dv * C;
  struct Arr {
    float** ptr;
    size_t bytes;
    int first, last;
  };
  float *staged = nullptr, *sw = nullptr, *su = nullptr, *ss = nullptr;
  const Arr arr[] = {
      {&staged, staged_prefix_bytes(fa), kPrefix, kFinal},
      {&w.fin, fin, kState, kRev},
      {&sw, tdk, kPrep, kState},  // W, row-major
      {&su, tdv, kPrep, kDkb},    // U, then Delta in place
      {&ss, st, kState, kDw},     // chunk-start states
      {&w.wt, tk, kPrep, kRev},
      {&w.qtT, tk, kPrep, kDkb},
      {&w.kbT, tk, kPrep, kDbk},
      {&w.bktT, tk, kPrep, kDkb},
      {&w.doT, tv, kPrep, kPdo},
      {&w.ddT, tv, kRev, kDbv},
      {&w.khT, tk, kPrep, kState},
      {&w.kb, tdk, kPrep, kRev},
      {&w.bkt, tdk, kPrep, kDtm},
      {&w.bv, tdv, kPrep, kDtm},
      {&w.do32, tdv, kPrep, kDqt},
      {&w.dd, tdv, kRev, kDtm},
      {&w.tm, sq, kPrep, kDbk},
      {&w.pp, sq, kPrep, kPdo},
      {&w.gam, gam, kPrep, kRev},
      {&w.gst, st, kRev, kDkb},
      {&w.dgam, dgam, kRev, kFinal},
      {&w.dp, sq, kDp, kDkb},
      {&w.dtm, sq, kDtm, kTmp},
      {&w.tmp, sq, kTmp, kDa},
      {&w.da, sq, kDa, kDkb},
      {&w.dqt, tdk, kDqt, kFinal},
      {&w.dkb, tdk, kDkb, kFinal},
      {&w.dw, tdk, kDw, kDbk},
      {&w.dbk, tdk, kDbk, kFinal},
      {&w.dbv, tdv, kDbv, kFinal},
      {&w.qdo, st, kQdo, kRev},
      {&w.pdo, tdv, kPdo, kRev},
  };
  constexpr int n = sizeof(arr) / sizeof(arr[0]);
  // first fit, largest arrays first: each goes to the lowest offset free of
  // every array placed before it whose lifetime it shares
  int order[n], live[n];
  size_t offs[n];
  for (int i = 0; i < n; ++i) order[i] = i;
  std::stable_sort(order, order + n, [&](int x, int y) {
    return arr[x].bytes > arr[y].bytes;
  });
  size_t top = 0;
  for (int r = 0; r < n; ++r) {
    const Arr& x = arr[order[r]];
    int nl = 0;
    for (int s = 0; s < r; ++s) {
      const Arr& y = arr[order[s]];
      if (y.first <= x.last && x.first <= y.last) live[nl++] = order[s];
    }
    std::sort(live, live + nl, [&](int i, int j) { return offs[i] < offs[j]; });
    size_t off = 0;
    for (int s = 0; s < nl; ++s) {
      if (off + x.bytes <= offs[live[s]]) break;
      off = std::max(off, align256(offs[live[s]] + arr[live[s]].bytes));
    }
    offs[order[r]] = off;
    top = std::max(top, align256(off + x.bytes));
  }
  for (int i = 0; i < n; ++i)
    *arr[i].ptr = p ? reinterpret_cast<float*>(p + offs[i]) : nullptr;
  for (int i = 0; i < n && i < cap; ++i)
    info[i] = BwdArray{offs[i], arr[i].bytes, arr[i].first, arr[i].last};
  if (count) *count = n;
  w.staged = staged;
  w.fv.w = sw;
  w.fv.d = su;
  w.fv.s = ss;
  if (total) *total = top;
  return w;
}

// Floats in each of prep's three shared regions: a [C][d_k + 1] or [C][d_v]
// token tile, or the inverse's 64 x kFS tile (plus its scratch).
__host__ __device__ constexpr int prep_region(int C, int dk, int dv) {
  return C * (dk + 1 > dv ? dk + 1 : dv) > 64 * ws::kFS + 1024
             ? C * (dk + 1 > dv ? dk + 1 : dv)
             : 64 * ws::kFS + 1024;
}

// Per (chunk, head): Kt, Kb, Qt, b Kt and fp32 copies of V, b V, dO; gam;
// M = Kt Kb^T (strictly lower, kept only on chip), P = lower_incl(Qt Kb^T),
// Tm = (I + Diag(b) M)^-1 by recursive doubling, and the forward's
// W = Tm Diag(b) Kt: row-major for the SIMT chain (w_out, else null), and
// W^T per chunk for the tensor-core chain (wt_out, else null); for the SIMT
// state pass also U = Tm Diag(b) V and Kh = k exp(g_C - g) (u_out, kh_out
// null otherwise).
template <typename IO>
__global__ void __launch_bounds__(kThreads, 2)  // two CTAs per SM
    prep_kernel(const IO* __restrict__ q, const IO* __restrict__ k,
                const IO* __restrict__ v, const float* __restrict__ beta,
                const IO* __restrict__ dout, const float* __restrict__ g,
                BwdWs w, float* __restrict__ w_out, float* __restrict__ u_out,
                float* __restrict__ kh_out, float* __restrict__ wt_out,
                const int32_t* cu, const int32_t* chunk_off, int n_seqs,
                int T, int H, int dk, int dv, int C) {
  const int cid = blockIdx.x;
  int seq, tok0, L;
  if (!locate_chunk(cid, cu, chunk_off, n_seqs, T, C, &seq, &tok0, &L)) return;
  const int h = blockIdx.y, tid = threadIdx.x;
  extern __shared__ float sm[];
  // Three [C][ldk] regions, reused as the chunk moves on so that two CTAs
  // fit on an SM: Kt, then V (once W is formed); Kb, then A and the
  // inverse's scratch (once M and P are formed); Qt, then Tm.
  const int ldk = dk + 1;          // padded rows: no bank conflicts
  const int reg = prep_region(C, dk, dv);
  float* Kt = sm;                  // [C][ldk]
  float* V = Kt;                   // [C][dv]
  float* Kb = Kt + reg;            // [C][ldk]
  float* A = Kb;                   // [64][kFS] b M, zero-padded past C
  float* Msc = A + 64 * ws::kFS;   // [1024] scratch of the inverse
  float* Qt = Kb + reg;            // [C][ldk]
  float* Tm = Qt;                  // [64][kFS]
  float* bs = Qt + reg;            // [C]
  float* gl = bs + C;              // [dk] g at the chunk's last row

  for (int r = tid; r < C; r += kThreads)
    bs[r] = r < L ? beta[(size_t)(tok0 + r) * H + h] : 0.f;
  for (int c = tid; c < dk; c += kThreads) {
    gl[c] = g[((size_t)(tok0 + L - 1) * H + h) * dk + c];
    if (fabsf(gl[c]) > kBwdDecayMax) atomicExch(&g_bwd_range, 1);
  }
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
      w.kb[gi] = kb;
      w.qt[gi] = qt;
      w.bkt[gi] = bs[r] * kt;
      if (kh_out) kh_out[gi] = kv * __expf(gl[c] - gv);
    }
    Kt[r * ldk + c] = kt;
    Kb[r * ldk + c] = kb;
    Qt[r * ldk + c] = qt;
  }
  // V and dO: fp32 copies out now, V held in registers until W is formed
  constexpr int kVU = 64 * 128 / kThreads;  // C * dv <= kVU * kThreads
  float vr[kVU];
#pragma unroll
  for (int u = 0; u < kVU; ++u) {
    const int idx = u * kThreads + tid;
    const int r = idx / dv;
    vr[u] = 0.f;
    if (idx < C * dv && r < L) {
      const size_t gi = ((size_t)(tok0 + r) * H + h) * dv + idx % dv;
      vr[u] = to_f32(v[gi]);
      w.bv[gi] = bs[r] * vr[u];
      w.do32[gi] = to_f32(dout[gi]);
    }
  }
  for (int c = tid; c < dk; c += kThreads)
    w.gam[((size_t)cid * H + h) * dk + c] = __expf(gl[c]);
  __syncthreads();
  if (w.qtT) {  // transposed per-chunk copies for the tensor-core products
    const size_t tb = ((size_t)cid * H + h) * dk * C;
    for (int idx = tid; idx < dk * C; idx += kThreads) {
      const int c = idx / C, r = idx % C;  // a warp reads one padded column
      const bool in = r < L;
      w.qtT[tb + idx] = in ? Qt[r * ldk + c] : 0.f;
      w.kbT[tb + idx] = in ? Kb[r * ldk + c] : 0.f;
      w.bktT[tb + idx] = in ? bs[r] * Kt[r * ldk + c] : 0.f;
    }
  }
  const size_t sqb = ((size_t)cid * H + h) * C * C;
  // Thread (ti, tj) owns rows ti + 16 a and columns tj + 16 b of each
  // product, so the padded rows give conflict-free loads.
  const int ti = tid >> 4, tj = tid & 15, nr = C / 16;
  float m[4][4];
  {
    float pv[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) m[a][b] = pv[a][b] = 0.f;
#pragma unroll 2
    for (int c = 0; c < dk; ++c) {
      float kt[4], qt[4], kb[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const bool in = a < nr;
        kt[a] = in ? Kt[(ti + 16 * a) * ldk + c] : 0.f;
        qt[a] = in ? Qt[(ti + 16 * a) * ldk + c] : 0.f;
        kb[a] = in ? Kb[(tj + 16 * a) * ldk + c] : 0.f;
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          m[a][b] += kt[a] * kb[b];
          pv[a][b] += qt[a] * kb[b];
        }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        if (a < nr && b < nr) {
          const int r = ti + 16 * a, i = tj + 16 * b;
          m[a][b] = (r < L && i < r) ? m[a][b] : 0.f;
          w.pp[sqb + r * C + i] = (r < L && i <= r) ? pv[a][b] : 0.f;
        }
      }
  }
  __syncthreads();  // Kb and Qt are dead: A and Tm take their places
  for (int idx = tid; idx < 64 * ws::kFS; idx += kThreads) {
    A[idx] = 0.f;
    Tm[idx] = 0.f;
  }
  __syncthreads();
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int r = ti + 16 * a, i = tj + 16 * b;
      if (a < nr && b < nr) A[r * ws::kFS + i] = bs[r] * m[a][b];
    }
  __syncthreads();
  // Tm = (I + Diag(b) M)^-1 by recursive doubling (identity past C)
  ws::invert_unit_lower(A, Tm, Msc, tid);
  __syncthreads();
  for (int idx = tid; idx < C * C; idx += kThreads) {
    const int r = idx / C, i = idx % C;
    w.tm[sqb + idx] = Tm[r * ws::kFS + i];
  }
  __syncthreads();
  // Tm Diag(b), in place (Tm is lower triangular, zero above the diagonal)
  for (int idx = tid; idx < C * C; idx += kThreads) {
    const int r = idx / C, i = idx % C;
    Tm[r * ws::kFS + i] *= bs[i];
  }
  __syncthreads();
  // W = (Tm Diag(b)) Kt, then U = (Tm Diag(b)) V with V over Kt, each over
  // i = 0 .. C - 1 (the terms above the diagonal are exact zeros)
  // (U only for the SIMT state pass; the two-pass forward forms its own)
  for (int pass = 0; pass < (u_out ? 2 : 1); ++pass) {
    const float* X = pass == 0 ? Kt : V;
    const int ldx = pass == 0 ? ldk : dv;
    const int nx = (pass == 0 ? dk : dv) / 16, cols = pass == 0 ? dk : dv;
    float* out = pass == 0 ? w_out : u_out;
    if (pass == 1) {
      __syncthreads();  // every read of Kt is done
#pragma unroll
      for (int u = 0; u < kVU; ++u) {
        const int idx = u * kThreads + tid;
        if (idx < C * dv) V[idx] = vr[u];
      }
      __syncthreads();
    }
    float acc[4][8];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
#pragma unroll 2
    for (int i = 0; i < C; ++i) {
      float t[4], xv[8];
#pragma unroll
      for (int a = 0; a < 4; ++a) t[a] = a < nr ? Tm[(ti + 16 * a) * ws::kFS + i] : 0.f;
#pragma unroll
      for (int b = 0; b < 8; ++b) xv[b] = b < nx ? X[i * ldx + tj + 16 * b] : 0.f;
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] += t[a] * xv[b];
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int r = ti + 16 * a;
      if (out && a < nr && r < L) {
        const size_t ro = ((size_t)(tok0 + r) * H + h) * cols;
#pragma unroll
        for (int b = 0; b < 8; ++b)
          if (b < nx) out[ro + tj + 16 * b] = acc[a][b];
      }
    }
    if (pass == 0 && wt_out) {
      // W^T for the tensor-core chain, staged transposed in the dead A
      // region (column index XOR the row's low bits against bank
      // conflicts) and written out coalesced at the end
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b)
          if (a < nr && b < nx) {
            const int r = ti + 16 * a, col = tj + 16 * b;
            A[col * C + (r ^ (col & 31))] = acc[a][b];
          }
    }
  }
  if (wt_out) {  // W^T [dk][C] of this chunk from the A region, zero past L
    __syncthreads();  // every thread's part of W^T is staged
    const size_t tb = ((size_t)cid * H + h) * dk * C;
    for (int idx = tid; idx < dk * C; idx += kThreads) {
      const int col = idx / C, r = idx % C;
      wt_out[tb + idx] = r < L ? A[col * C + (r ^ (col & 31))] : 0.f;
    }
  }
  if (w.doT) {
    // dO^T per chunk: dO staged row-wise (column index XOR the row's low
    // bits) in the Kt region, which nothing reads after W is formed
    __syncthreads();
    for (int idx = tid; idx < C * dv; idx += kThreads) {
      const int r = idx / dv, c = idx % dv;
      Kt[r * dv + (c ^ (r & 31))] =
          r < L ? to_f32(dout[((size_t)(tok0 + r) * H + h) * dv + c]) : 0.f;
    }
    __syncthreads();
    const size_t tb = ((size_t)cid * H + h) * dv * C;
    for (int idx = tid; idx < dv * C; idx += kThreads) {
      const int c = idx / C, r = idx % C;
      w.doT[tb + idx] = Kt[r * dv + (c ^ (r & 31))];
    }
  }
}

// prep on the tensor cores, for bf16 inputs in 64-token chunks (the
// tensor-core backward): the same outputs as prep_kernel in that mode, with
// its four products as tcgen05 kind::tf32 MMAs on 128-byte-swizzled
// K-major fp32 panels: M = Kt Kb^T and P = Qt Kb^T (M = 64 shape, K = d_k),
// then W = T' Kt and U = T' V (K = the 64 tokens, Kt and V transposed in
// shared memory).  The inverse stays the SIMT recursive doubling.  W goes
// out row-major (for the state pass) and as W^T per chunk.  Shared memory:
// the Kt panels, then one region that holds the Qt and Kb panels, later the
// inverse's tiles, then T' and Kt^T, then V^T, then dO for its transposed
// copy.
template <int DK>
struct PrepTcLayout {
  static constexpr uint32_t kt = 0;                   // DK / 32 panels, 8 KB
  static constexpr uint32_t r2 = DK * 256;            // Qt | Kb panels ...
  static constexpr uint32_t qt = r2, kb = r2 + DK * 256;
  static constexpr uint32_t am = r2;                  // [64][kFS] fp32
  static constexpr uint32_t msc = r2 + 64 * ws::kFS * 4;
  static constexpr uint32_t tm = msc + 4096;          // [64][kFS] fp32
  static constexpr uint32_t tp = r2 + 40960;          // T': two 8 KB panels
  static constexpr uint32_t ktt = r2;                 // Kt^T: two DK-row panels
  static constexpr uint32_t r2_bytes =
      2 * DK * 256 > 57344 ? 2 * DK * 256 : 57344;
  static constexpr uint32_t misc = r2 + r2_bytes;     // barrier, TMEM slot
  static constexpr uint32_t bs = misc + 64;           // [64] beta
  static constexpr uint32_t gl = bs + 256;            // [DK] g at the last row
  static constexpr uint32_t bytes = gl + DK * 4;
  static_assert(tm + 64 * ws::kFS * 4 <= tp, "inverse tiles below T'");
  static_assert(ktt + 2 * DK * 128 <= tp, "Kt^T below T'");
  static_assert(tp + 16384 <= r2 + r2_bytes, "T' inside the region");
};

template <int DK>
__global__ void __launch_bounds__(kThreads, 2)
    prep_tc_kernel(const __nv_bfloat16* __restrict__ q,
                   const __nv_bfloat16* __restrict__ k,
                   const __nv_bfloat16* __restrict__ v,
                   const float* __restrict__ beta,
                   const __nv_bfloat16* __restrict__ dout,
                   const float* __restrict__ g, BwdWs w,
                   const int32_t* cu, const int32_t* chunk_off, int n_seqs,
                   int T, int H, int dv) {
  using namespace sm100;
  using Lay = PrepTcLayout<DK>;
  constexpr int C = 64;
  const int cid = blockIdx.x;
  int seq, tok0, L;
  if (!locate_chunk(cid, cu, chunk_off, n_seqs, T, C, &seq, &tok0, &L)) return;
  const int h = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* KT = sm + Lay::kt;
  uint8_t* QT = sm + Lay::qt;
  uint8_t* KB = sm + Lay::kb;
  float* Am = reinterpret_cast<float*>(sm + Lay::am);
  float* Msc = reinterpret_cast<float*>(sm + Lay::msc);
  float* Tm = reinterpret_cast<float*>(sm + Lay::tm);
  uint8_t* TP = sm + Lay::tp;
  uint8_t* KTT = sm + Lay::ktt;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + Lay::misc);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 1);
  float* bs = reinterpret_cast<float*>(sm + Lay::bs);
  float* gl = reinterpret_cast<float*>(sm + Lay::gl);
  auto pel = [](uint8_t* panels, int r, int c) {  // (row r, column c)
    return reinterpret_cast<float*>(panels + (c >> 5) * 8192 +
                                    swz32(r, c & 31));
  };

  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tslot, 256);
    tmem_relinquish();
  }
  for (int r = tid; r < C; r += kThreads)
    bs[r] = r < L ? beta[(size_t)(tok0 + r) * H + h] : 0.f;
  for (int c = tid; c < DK; c += kThreads) {
    gl[c] = g[((size_t)(tok0 + L - 1) * H + h) * DK + c];
    if (fabsf(gl[c]) > kBwdDecayMax) atomicExch(&g_bwd_range, 1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  // ---- Kt, Kb, Qt: the workspace rows and the operand panels, four
  // channels per thread and step (8-byte bf16 and 16-byte fp32 accesses)
  auto ld_bf4 = [](const __nv_bfloat16* p, float* x) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
    x[0] = __low2float(a); x[1] = __high2float(a);
    x[2] = __low2float(b); x[3] = __high2float(b);
  };
  auto st4 = [](float* p, const float* x) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  };
  for (int idx = tid; idx < C * DK / 4; idx += kThreads) {
    const int r = idx / (DK / 4), c = (idx % (DK / 4)) * 4;
    float kt[4] = {0.f, 0.f, 0.f, 0.f}, kb[4] = {0.f, 0.f, 0.f, 0.f},
          qt[4] = {0.f, 0.f, 0.f, 0.f};
    if (r < L) {
      const size_t gi = ((size_t)(tok0 + r) * H + h) * DK + c;
      float kv[4], qv[4];
      ld_bf4(k + gi, kv);
      ld_bf4(q + gi, qv);
      const float4 g4 = *reinterpret_cast<const float4*>(g + gi);
      const float gv[4] = {g4.x, g4.y, g4.z, g4.w};
      float bk[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float e = __expf(gv[u]), ie = __expf(-gv[u]);
        kt[u] = kv[u] * e;
        kb[u] = kv[u] * ie;
        qt[u] = qv[u] * e;
        bk[u] = bs[r] * kt[u];
      }
      st4(w.kb + gi, kb);  // (Kt and Qt rows: the final kernel recomputes them)
      st4(w.bkt + gi, bk);
    }
    st4(pel(KT, r, c), kt);
    st4(pel(KB, r, c), kb);
    st4(pel(QT, r, c), qt);
  }
  for (int idx = tid; idx < L * dv / 4; idx += kThreads) {
    const int r = idx / (dv / 4);
    const size_t gi = ((size_t)(tok0 + r) * H + h) * dv + (idx % (dv / 4)) * 4;
    float vv[4], dd[4], bvv[4];
    ld_bf4(v + gi, vv);
    ld_bf4(dout + gi, dd);
#pragma unroll
    for (int u = 0; u < 4; ++u) bvv[u] = bs[r] * vv[u];
    st4(w.bv + gi, bvv);
    st4(w.do32 + gi, dd);
  }
  for (int c = tid; c < DK; c += kThreads)
    w.gam[((size_t)cid * H + h) * DK + c] = __expf(gl[c]);
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();

  // ---- M = Kt Kb^T (TMEM columns 0-63), P = Qt Kb^T (64-127)
  if (tid == 0) {
    tc_fence_after();
    constexpr uint32_t id = idesc_tf32(64, 64);
#pragma unroll
    for (int ks = 0; ks < DK / 8; ++ks) {
      const uint32_t o = (ks >> 2) * 8192 + (ks & 3) * 32;
      const uint64_t bd = desc_sw128(smem_u32(KB) + o, 16, 1024);
      mma_tf32(tmem, desc_sw128(smem_u32(KT) + o, 16, 1024), bd, id, ks > 0);
      mma_tf32(tmem + 64, desc_sw128(smem_u32(QT) + o, 16, 1024), bd, id,
               ks > 0);
    }
    mma_commit(bar);
  }
  // the transposed copies meanwhile (reads only)
  {
    const size_t tb = ((size_t)cid * H + h) * DK * C;
    // a thread reads four consecutive channels of one token row (16-byte
    // shared loads) and writes them to four transposed rows; a warp covers
    // 32 consecutive tokens, so each global store is one 128-byte segment
    for (int idx = tid; idx < DK / 4 * C; idx += kThreads) {
      const int r = idx % C, c = (idx / C) * 4;
      const float4 q4 = *reinterpret_cast<const float4*>(pel(QT, r, c));
      const float4 b4 = *reinterpret_cast<const float4*>(pel(KB, r, c));
      const float4 t4 = *reinterpret_cast<const float4*>(pel(KT, r, c));
      const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
      const float kbv[4] = {b4.x, b4.y, b4.z, b4.w};
      const float ktv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const size_t o = tb + (size_t)(c + u) * C + r;
        w.qtT[o] = qv[u];
        w.kbT[o] = kbv[u];
        w.bktT[o] = bs[r] * ktv[u];
        // Kh = k exp(g_C - g) = Kb exp(g_C), rounded to the nearest tf32
        w.khT[o] = sm100::tf32_rna(kbv[u] * __expf(gl[c + u]));
      }
    }
  }
  bool ok = __syncthreads_and(mbar_wait(bar, 0, 2000000000ull));
  tc_fence_after();
  if (ok) {
    // ---- A = Diag(b) strictly_lower(M) for the inverse; P out
    for (int idx = tid; idx < 64 * ws::kFS; idx += kThreads) {
      Am[idx] = 0.f;
      Tm[idx] = 0.f;
    }
    __syncthreads();
    const int qd = warp & 3, half = warp >> 2, r = 16 * qd + lane;
    float mv[32], pv[32];
    tmem_ld32(tmem + ((uint32_t)(32 * qd) << 16) + 32 * half, mv);
    tmem_ld32(tmem + ((uint32_t)(32 * qd) << 16) + 64 + 32 * half, pv);
    if (lane < 16) {  // M = 64 accumulator rows 16 qd .. 16 qd + 15
      const size_t sqb = ((size_t)cid * H + h) * C * C;
      float* pr = w.pp + sqb + r * C + 32 * half;
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const int i = 32 * half + u;
        Am[r * ws::kFS + i] = (r < L && i < r) ? bs[r] * mv[u] : 0.f;
        pv[u] = (r < L && i <= r) ? pv[u] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        reinterpret_cast<float4*>(pr)[u] =
            make_float4(pv[4 * u], pv[4 * u + 1], pv[4 * u + 2], pv[4 * u + 3]);
    }
    tc_fence_before();
    __syncthreads();
    // ---- Tm = (I + A)^-1; T' = Tm Diag(b) as the A panels of W = T' Kt
    ws::invert_unit_lower(Am, Tm, Msc, tid);
    __syncthreads();
    {
      const size_t sqb = ((size_t)cid * H + h) * C * C;
      for (int idx = tid; idx < C * C; idx += kThreads) {
        const int rr = idx / C, i = idx % C;
        const float t = Tm[rr * ws::kFS + i];
        w.tm[sqb + idx] = t;
        *pel(TP, rr, i) = t * bs[i];
      }
    }
    __syncthreads();
    // Kt^T as the K-major B panels of W (rows = channels, K = tokens)
    for (int idx = tid; idx < C * DK; idx += kThreads) {
      const int c = idx / C, i = idx % C;
      *reinterpret_cast<float*>(KTT + (i >> 5) * (DK * 128) + swz32(c, i & 31)) =
          *pel(KT, i, c);
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id = idesc_tf32(64, DK);
#pragma unroll
      for (int ks = 0; ks < C / 8; ++ks)
        mma_tf32(tmem,
                 desc_sw128(smem_u32(TP) + (ks >> 2) * 8192 + (ks & 3) * 32,
                            16, 1024),
                 desc_sw128(smem_u32(KTT) + (ks >> 2) * (DK * 128) +
                                (ks & 3) * 32,
                            16, 1024),
                 id, ks > 0);
      mma_commit(bar);
    }
    ok = __syncthreads_and(mbar_wait(bar, 1, 2000000000ull));
    tc_fence_after();
  }
  if (ok) {
    // ---- V^T as the K-major B panels of U = T' V (Kt^T is read), then U
    uint8_t* VT = sm + Lay::r2;
    for (int idx = tid; idx < C * dv / 4; idx += kThreads) {
      const int s = idx / (dv / 4), j = (idx % (dv / 4)) * 4;
      float x[4] = {0.f, 0.f, 0.f, 0.f};
      if (s < L) ld_bf4(v + ((size_t)(tok0 + s) * H + h) * dv + j, x);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        *reinterpret_cast<float*>(VT + (s >> 5) * (dv * 128) +
                                  swz32(j + u, s & 31)) = x[u];
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t id = idesc_tf32(64, dv);
#pragma unroll
      for (int ks = 0; ks < C / 8; ++ks)
        mma_tf32(tmem + DK,
                 desc_sw128(smem_u32(TP) + (ks >> 2) * 8192 + (ks & 3) * 32,
                            16, 1024),
                 desc_sw128(smem_u32(VT) + (ks >> 2) * (dv * 128) +
                                (ks & 3) * 32,
                            16, 1024),
                 id, ks > 0);
      mma_commit(bar);
    }
    // ---- W out, row-major and as W^T: thread row r holds W[r][columns]
    const int qd = warp & 3, half = warp >> 2, r = 16 * qd + lane;
    const size_t tb = ((size_t)cid * H + h) * DK * C;
#pragma unroll
    for (int cc = 0; cc < DK / 64; ++cc) {
      const int j0 = half * (DK / 2) + 32 * cc;
      float wv[32];
      tmem_ld32(tmem + ((uint32_t)(32 * qd) << 16) + j0, wv);
      if (lane < 16) {
#pragma unroll
        for (int u = 0; u < 32; ++u)
          w.wt[tb + (size_t)(j0 + u) * C + r] = r < L ? wv[u] : 0.f;
        if (r < L) {  // rounded to the nearest tf32 for the state pass
          float4* wr = reinterpret_cast<float4*>(
              w.fv.w + ((size_t)(tok0 + r) * H + h) * DK + j0);
#pragma unroll
          for (int u = 0; u < 8; ++u)
            wr[u] = make_float4(
                sm100::tf32_rna(wv[4 * u]), sm100::tf32_rna(wv[4 * u + 1]),
                sm100::tf32_rna(wv[4 * u + 2]), sm100::tf32_rna(wv[4 * u + 3]));
        }
      }
    }
    ok = __syncthreads_and(mbar_wait(bar, 0, 2000000000ull));
    tc_fence_after();
  }
  if (ok) {
    const int qd = warp & 3, half = warp >> 2, r = 16 * qd + lane;
    // ---- U out (row-major, the state pass turns it into Delta)
    for (int cc = 0; cc < dv / 64; ++cc) {
      const int j0 = half * (dv / 2) + 32 * cc;
      float uv[32];
      tmem_ld32(tmem + ((uint32_t)(32 * qd) << 16) + DK + j0, uv);
      if (lane < 16 && r < L) {
        float4* ur = reinterpret_cast<float4*>(
            w.fv.d + ((size_t)(tok0 + r) * H + h) * dv + j0);
#pragma unroll
        for (int u = 0; u < 8; ++u)
          ur[u] = make_float4(uv[4 * u], uv[4 * u + 1], uv[4 * u + 2],
                              uv[4 * u + 3]);
      }
    }
    // ---- dO^T per chunk, staged row-wise (XOR-swizzled) in the region
    float* Ds = reinterpret_cast<float*>(sm + Lay::r2);
    for (int idx = tid; idx < C * dv / 4; idx += kThreads) {
      const int rr = idx / (dv / 4), c = (idx % (dv / 4)) * 4;
      float x[4] = {0.f, 0.f, 0.f, 0.f};
      if (rr < L) ld_bf4(dout + ((size_t)(tok0 + rr) * H + h) * dv + c, x);
#pragma unroll
      for (int u = 0; u < 4; ++u) Ds[rr * dv + ((c + u) ^ (rr & 31))] = x[u];
    }
    __syncthreads();
    const size_t tv = ((size_t)cid * H + h) * dv * C;
    for (int idx = tid; idx < dv * C; idx += kThreads) {
      const int c = idx / C, rr = idx % C;
      w.doT[tv + idx] = Ds[rr * dv + (c ^ (rr & 31))];
    }
  } else if (tid == 0) {
    atomicExch(&g_bwd_timeout, 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

// The reverse chain over one sequence's chunks for one head and one 32-wide
// column tile of d_v (92 KB of shared memory at d = 128, so two CTAs share an
// SM and a B=2, H=32 layer's 256 CTAs run as one wave).  Per chunk (last first), with dS the gradient of the
// state leaving it:
//   gam * d gam (partial over the tile) = rowsum(S_next * dS), S_next being
//     the state leaving the chunk (= gam (S_0 + Kb^T Delta)): the next
//     chunk's stored start state, or the final state;
//   G = Diag(gam) dS (stored);
//   dDelta = Kb G + P^T dO (stored), P^T dO precomputed;
//   dS <- G + Qt^T dO - W^T dDelta, Qt^T dO precomputed.
// Only the two products with dS on their path are left in the serial loop.
// Each gives every thread a block of outputs (rows strided by 32, columns by
// 8) whose sums over the contraction index run as independent chains; the
// shared rows are padded (TILE + 1 floats for the tiles, d_k + 1 for the
// token rows) so both access directions are free of bank conflicts.
constexpr int kChainTile = 32;

template <int TILE>
__global__ void __launch_bounds__(kThreads)
    chain_kernel(BwdWs w, const float* __restrict__ d_final,
                 float* __restrict__ d_init, const int32_t* cu, int n_seqs,
                 int T, int H, int dk, int dv, int C) {
  constexpr int TP = TILE + 1, NB = TILE / 8;
  const int seq = blockIdx.x, h = blockIdx.y, tile = blockIdx.z;
  const int j0 = tile * TILE, tid = threadIdx.x, ntile = dv / TILE;
  const int dkp = dk + 1, NA = dk / 32;
  const int g8 = tid >> 3, j8 = tid & 7;  // row group, column group
  extern __shared__ float sm[];
  float* dS = sm;                    // [dk][TP]
  float* Kb = dS + dk * TP;          // [C][dkp]
  float* Wc = Kb + C * dkp;          // [C][dkp]
  float* dD = Wc + C * dkp;          // [C][TP] dDelta
  float* gC = dD + C * TP;           // [dk]

  const size_t sbase = ((size_t)seq * H + h) * dk * dv;
  for (int idx = tid; idx < dk * TILE; idx += kThreads) {
    const int c = idx / TILE, jj = idx % TILE;
    dS[c * TP + jj] = d_final ? d_final[sbase + (size_t)c * dv + j0 + jj] : 0.f;
  }
  int start, end;
  seq_range(cu, seq, T, &start, &end);
  const int nch = (end - start + C - 1) / C;
  const int cid0 = cu ? w.fv.chunk_off[seq] : seq * ((T + C - 1) / C);
  __syncthreads();

  for (int ch = nch - 1; ch >= 0; --ch) {
    const int cid = cid0 + ch, tok0 = start + ch * C, L = min(C, end - tok0);
    const size_t cbase = ((size_t)cid * H + h) * dk * dv;
    // per-thread operands straight to registers: S_next, P^T dO, Qt^T dO
    const float* snx = ch + 1 < nch ? w.fv.s + cbase + (size_t)H * dk * dv
                                    : w.fin + sbase;
    float sn[4][NB], dacc[2][NB], sacc[4][NB];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const size_t o = (size_t)(g8 + 32 * a) * dv + j0 + j8 + 8 * b;
        sn[a][b] = a < NA ? snx[o] : 0.f;
        sacc[a][b] = a < NA ? w.qdo[cbase + o] : 0.f;
      }
#pragma unroll
    for (int a = 0; a < 2; ++a) {
      const int r = g8 + 32 * a;
#pragma unroll
      for (int b = 0; b < NB; ++b)
        dacc[a][b] = r < L ? w.pdo[((size_t)(tok0 + r) * H + h) * dv + j0 +
                                   j8 + 8 * b]
                           : 0.f;
    }
    // staging loads batched eight deep so their latencies overlap
    for (int base = 0; base < C * dk; base += 8 * kThreads) {
      float kb[8], wv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int idx = base + u * kThreads + tid;
        const int r = idx / dk, c = idx % dk;
        kb[u] = wv[u] = 0.f;
        if (idx < C * dk && r < L) {
          const size_t gi = ((size_t)(tok0 + r) * H + h) * dk + c;
          kb[u] = w.kb[gi];
          wv[u] = w.fv.w[gi];
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int idx = base + u * kThreads + tid;
        if (idx < C * dk) {
          const int r = idx / dk, c = idx % dk;
          Kb[r * dkp + c] = kb[u];
          Wc[r * dkp + c] = wv[u];
        }
      }
    }
    for (int c = tid; c < dk; c += kThreads)
      gC[c] = w.gam[((size_t)cid * H + h) * dk + c];
    // gam * d gam over this tile (dS is only read here)
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      if (a < NA) {
        const int c = g8 + 32 * a;
        float part = 0.f;
#pragma unroll
        for (int b = 0; b < NB; ++b) part += sn[a][b] * dS[c * TP + j8 + 8 * b];
        part += __shfl_xor_sync(0xffffffffu, part, 1);
        part += __shfl_xor_sync(0xffffffffu, part, 2);
        part += __shfl_xor_sync(0xffffffffu, part, 4);
        if (j8 == 0)
          w.dgam[(((size_t)cid * H + h) * ntile + tile) * dk + c] = part;
      }
    }
    __syncthreads();
    for (int idx = tid; idx < dk * TILE; idx += kThreads) {
      const int c = idx / TILE, jj = idx % TILE;
      const float gv = gC[c] * dS[c * TP + jj];
      dS[c * TP + jj] = gv;
      w.gst[cbase + (size_t)c * dv + j0 + jj] = gv;
    }
    __syncthreads();
    // dDelta = P^T dO + Kb G  (rows g8, g8 + 32)
    #pragma unroll 4
    for (int c = 0; c < dk; ++c) {
      float gv[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) gv[b] = dS[c * TP + j8 + 8 * b];
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        const int r = g8 + 32 * a;  // Kb rows past L are zero, past C absent
        const float kb = r < C ? Kb[r * dkp + c] : 0.f;
#pragma unroll
        for (int b = 0; b < NB; ++b) dacc[a][b] += kb * gv[b];
      }
    }
#pragma unroll
    for (int a = 0; a < 2; ++a) {
      const int r = g8 + 32 * a;
      if (r < C) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const int jj = j8 + 8 * b;
          const float v = r < L ? dacc[a][b] : 0.f;
          dD[r * TP + jj] = v;
          if (r < L) w.dd[((size_t)(tok0 + r) * H + h) * dv + j0 + jj] = v;
        }
      }
    }
    __syncthreads();
    // dS <- G + Qt^T dO - W^T dDelta
    #pragma unroll 4
    for (int r = 0; r < L; ++r) {
      float dd[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) dd[b] = dD[r * TP + j8 + 8 * b];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        if (a < NA) {
          const float wv = Wc[r * dkp + g8 + 32 * a];
#pragma unroll
          for (int b = 0; b < NB; ++b) sacc[a][b] -= wv * dd[b];
        }
      }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      if (a < NA) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const int i = (g8 + 32 * a) * TP + j8 + 8 * b;
          dS[i] += sacc[a][b];
        }
      }
    }
    __syncthreads();
  }
  if (d_init) {
    for (int idx = tid; idx < dk * TILE; idx += kThreads) {
      const int c = idx / TILE, jj = idx % TILE;
      d_init[sbase + (size_t)c * dv + j0 + jj] = dS[c * TP + jj];
    }
  }
}

// ---------------------------------------------------------------------------
// Batched small products over every (chunk, head): Out (m x n) = alpha sum of
// op(A) op(B) over one to three terms (+ Out), with op = transpose or not and an
// optional lower-triangular mask on Out.  An operand is one of: token rows
// [tokens, H, cols] (rows are the chunk's tokens), a per-chunk square
// [chunks, H, C, C], or a per-chunk state [chunks, H, dk, dv].  m, n and the
// contraction length are each L, d_k or d_v.
// kTokT: a per-chunk transposed copy of token rows, [chunks, H, cols, C]
// (rows = the channels, C token columns).
enum MatKind { kTok = 0, kSq = 1, kState = 2, kTokT = 3 };
enum Dim { kDimL = 0, kDimDk = 1, kDimDv = 2 };
enum Mask { kMaskNone = 0, kMaskLowerIncl = 1, kMaskStrictLower = 2 };

struct MatRef {
  float* p;
  int kind;
  int cols;    // kTok: row width; kSq: C; kState: dv
  int trans;
};

struct BmmTerm {
  MatRef a, b;
  int kd;      // the padded contraction length (C, d_k or d_v)
};

struct BmmOp {
  MatRef out;
  BmmTerm term[3];
  int nterms;
  int m, n;    // Dim codes
  int md, nd;  // padded m and n
  int mask;
  float alpha;
  int accumulate;
};

__device__ __forceinline__ int dim_of(int code, int L, int dk, int dv) {
  return code == kDimL ? L : code == kDimDk ? dk : dv;
}

// One operand source as a row-major matrix: row 0 and the row stride, plus
// the valid extent (token rows and square entries past L read as zero).
struct Src {
  float* p;
  size_t stride;
  int vrows, vcols;
};

__device__ __forceinline__ Src src_of(const MatRef& x, int cid, int h,
                                      int tok0, int L, int H, int C, int dk) {
  if (x.kind == kTok)
    return Src{x.p + ((size_t)tok0 * H + h) * x.cols, (size_t)H * x.cols, L,
               x.cols};
  if (x.kind == kSq)
    return Src{x.p + ((size_t)cid * H + h) * C * C, (size_t)C, L, L};
  if (x.kind == kTokT)
    return Src{x.p + ((size_t)cid * H + h) * x.cols * C, (size_t)C, x.cols, L};
  return Src{x.p + ((size_t)cid * H + h) * dk * x.cols, (size_t)x.cols, dk,
             x.cols};
}

// Four consecutive entries (r, c .. c + 3), c a multiple of four.  A square's
// last valid vector can be partial; its tail lies inside the C x C
// allocation and is zeroed.
__device__ __forceinline__ float4 ld_src4(const Src& s, int r, int c) {
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (r < s.vrows && c < s.vcols) {
    v = *reinterpret_cast<const float4*>(s.p + (size_t)r * s.stride + c);
    if (c + 1 >= s.vcols) v.y = 0.f;
    if (c + 2 >= s.vcols) v.z = 0.f;
    if (c + 3 >= s.vcols) v.w = 0.f;
  }
  return v;
}

// dst[r * ld + c] = src(r, c) over the padded rows x cols (multiples of 16):
// consecutive threads take consecutive 16-byte vectors of a row.
__device__ __forceinline__ void stage_direct(const Src& s, int rows, int cols,
                                             float* dst, int ld, int tid) {
  const int cv = cols >> 2, units = rows * cv;
  for (int base = 0; base < units; base += 4 * kThreads) {
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int idx = base + u * kThreads + tid;
      v[u] = idx < units ? ld_src4(s, idx / cv, (idx % cv) * 4)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int idx = base + u * kThreads + tid;
      if (idx < units)
        *reinterpret_cast<float4*>(dst + (idx / cv) * ld + (idx % cv) * 4) = v[u];
    }
  }
}

// dst[c * ld + r] = src(r, c): consecutive threads take consecutive rows, each
// reading 32 contiguous bytes, so the scattered shared stores of a warp fall
// in distinct banks.
__device__ __forceinline__ void stage_transposed(const Src& s, int rows,
                                                 int cols, float* dst, int ld,
                                                 int tid) {
  const int units = rows * (cols >> 3);
  for (int base = 0; base < units; base += 2 * kThreads) {
    float4 v[2][2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int idx = base + u * kThreads + tid;
      const int r = idx % rows, c = (idx / rows) * 8;
      const bool in = idx < units;
      v[u][0] = in ? ld_src4(s, r, c) : make_float4(0.f, 0.f, 0.f, 0.f);
      v[u][1] = in ? ld_src4(s, r, c + 4) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int idx = base + u * kThreads + tid;
      if (idx < units) {
        const int r = idx % rows, c = (idx / rows) * 8;
        float* d = dst + c * ld + r;
        d[0 * ld] = v[u][0].x;
        d[1 * ld] = v[u][0].y;
        d[2 * ld] = v[u][0].z;
        d[3 * ld] = v[u][0].w;
        d[4 * ld] = v[u][1].x;
        d[5 * ld] = v[u][1].y;
        d[6 * ld] = v[u][1].z;
        d[7 * ld] = v[u][1].w;
      }
    }
  }
}

template <int N>
__device__ __forceinline__ void lds_vec(const float* p, float* v) {
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

// op(A) is staged transposed (AT[t][i]) and op(B) as is (Bs[t][j]), zero past
// the valid extent, rows padded by four floats.  The 256 threads form a
// 16 x 16 grid over the padded md x nd output; thread (ti, tj) owns the
// RM x RN block at rows RM ti.., columns RN tj.. (RM = md / 16, RN = nd / 16),
// so every thread works and each step of the contraction is a few vector
// shared loads for RM x RN FMAs.  Up to 4 x 8 blocks the registers are capped
// so that three CTAs share an SM and hide each other's staging.
template <int RM, int RN>
__global__ void __launch_bounds__(kThreads, RM * RN >= 64 ? 1 : 3)
    bmm_kernel(BmmOp op, const int32_t* cu, const int32_t* chunk_off, int n_seqs,
               int T, int H, int dk, int dv, int C) {
  const int cid = blockIdx.x;
  int seq, tok0, L;
  if (!locate_chunk(cid, cu, chunk_off, n_seqs, T, C, &seq, &tok0, &L)) return;
  const int h = blockIdx.y, tid = threadIdx.x;
  const int md = 16 * RM, nd = 16 * RN;
  const int la = md + 4, lb = nd + 4;
  extern __shared__ __align__(16) float sm[];
  const int ti = tid >> 4, tj = tid & 15;
  float acc[RM][RN];
#pragma unroll
  for (int a = 0; a < RM; ++a)
#pragma unroll
    for (int b = 0; b < RN; ++b) acc[a][b] = 0.f;
  for (int term = 0; term < op.nterms; ++term) {
    const BmmTerm tm = term == 0 ? op.term[0]
                       : term == 1 ? op.term[1] : op.term[2];
    const int kd = tm.kd;
    float* AT = sm;            // [kd][la]
    float* Bs = sm + kd * la;  // [kd][lb]
    if (term > 0) __syncthreads();  // the previous term's reads are done
    const Src sa = src_of(tm.a, cid, h, tok0, L, H, C, dk);
    const Src sb = src_of(tm.b, cid, h, tok0, L, H, C, dk);
    if (tm.a.trans) stage_direct(sa, kd, md, AT, la, tid);  // source A[t][i]
    else stage_transposed(sa, md, kd, AT, la, tid);         // source A[i][t]
    if (tm.b.trans) stage_transposed(sb, nd, kd, Bs, lb, tid);  // B[j][t]
    else stage_direct(sb, kd, nd, Bs, lb, tid);                 // B[t][j]
    __syncthreads();
    const float* ap = AT + RM * ti;
    const float* bp = Bs + RN * tj;
#pragma unroll 4
    for (int t = 0; t < kd; ++t) {
      float av[RM], bv[RN];
      lds_vec<RM>(ap + t * la, av);
      lds_vec<RN>(bp + t * lb, bv);
#pragma unroll
      for (int a = 0; a < RM; ++a)
#pragma unroll
        for (int b = 0; b < RN; ++b) acc[a][b] += av[a] * bv[b];
    }
  }
  const int m = dim_of(op.m, L, dk, dv), n = dim_of(op.n, L, dk, dv);
  const Src so = src_of(op.out, cid, h, tok0, L, H, C, dk);
  const int j0 = RN * tj;
#pragma unroll
  for (int a = 0; a < RM; ++a) {
    const int i = RM * ti + a;
    if (i >= m || j0 >= n) continue;
    float x[RN];
#pragma unroll
    for (int b = 0; b < RN; ++b) {
      const int j = j0 + b;
      x[b] = op.alpha * acc[a][b];
      if ((op.mask == kMaskLowerIncl && j > i) ||
          (op.mask == kMaskStrictLower && j >= i))
        x[b] = 0.f;
    }
    float* o = so.p + (size_t)i * so.stride + j0;
    if (RN >= 4 && j0 + RN <= n) {
#pragma unroll
      for (int q = 0; q < RN / 4; ++q) {
        float4* o4 = reinterpret_cast<float4*>(o + 4 * q);
        float4 y = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
        if (op.accumulate) {
          const float4 z = *o4;
          y.x += z.x;
          y.y += z.y;
          y.z += z.z;
          y.w += z.w;
        }
        *o4 = y;
      }
    } else {
#pragma unroll
      for (int b = 0; b < RN; ++b)
        if (j0 + b < n) o[b] = op.accumulate ? o[b] + x[b] : x[b];
    }
  }
}

// Per (chunk, head): the input gradients from the products above.
template <typename IO>
__global__ void __launch_bounds__(kThreads)
    final_kernel(BwdWs w, const IO* __restrict__ q, const IO* __restrict__ k,
                 const IO* __restrict__ v, const float* __restrict__ beta,
                 const float* __restrict__ g, IO* __restrict__ dq,
                 IO* __restrict__ dk_out, IO* __restrict__ dv_out,
                 float* __restrict__ dla, float* __restrict__ dbeta,
                 const int32_t* cu, const int32_t* chunk_off, int n_seqs, int T,
                 int H, int dk, int dv, int C) {
  const int cid = blockIdx.x;
  int seq, tok0, L;
  if (!locate_chunk(cid, cu, chunk_off, n_seqs, T, C, &seq, &tok0, &L)) return;
  const int h = blockIdx.y, tid = threadIdx.x, ntile = dv / kChainTile;
  extern __shared__ float sm[];
  float* dg = sm;          // [C][dk]
  float* pb = sm + C * dk; // [C][dk / 4] partials of rowsum(dKt/b * Kt)
  // four consecutive channels per thread and step (d_k, d_v multiples of 4);
  // Kt, Kb and Qt are recomputed from k, q and g exactly as prep forms them
  auto ld4 = [](const float* p) { return *reinterpret_cast<const float4*>(p); };
  // four consecutive io values as one 8-byte (bf16) or 16-byte (fp32) access
  auto ld4io = [](const IO* p, float* x) {
    if constexpr (sizeof(IO) == 2) {
      const uint2 u = *reinterpret_cast<const uint2*>(p);
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
      const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
      x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    } else {
      const float4 f = *reinterpret_cast<const float4*>(p);
      x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
    }
  };
  auto st4io = [](IO* p, const float* x) {
    if constexpr (sizeof(IO) == 2) {
      const __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]);
      const __nv_bfloat162 b = __floats2bfloat162_rn(x[2], x[3]);
      uint2 u;
      u.x = *reinterpret_cast<const uint32_t*>(&a);
      u.y = *reinterpret_cast<const uint32_t*>(&b);
      *reinterpret_cast<uint2*>(p) = u;
    } else {
      *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
    }
  };
  const int dk4 = dk / 4, dv4 = dv / 4;
  for (int idx = tid; idx < L * dk4; idx += kThreads) {
    const int r = idx / dk4, c = (idx % dk4) * 4;
    const size_t gi = ((size_t)(tok0 + r) * H + h) * dk + c;
    const float b = beta[(size_t)(tok0 + r) * H + h];
    const float4 bk = ld4(w.dbk + gi), kb4 = ld4(w.dkb + gi),
                 qt4 = ld4(w.dqt + gi), g4 = ld4(g + gi);
    float kv[4], qv[4];
    ld4io(k + gi, kv);
    ld4io(q + gi, qv);
    const float dbk[4] = {bk.x, bk.y, bk.z, bk.w};
    const float dKb[4] = {kb4.x, kb4.y, kb4.z, kb4.w};
    const float dQt[4] = {qt4.x, qt4.y, qt4.z, qt4.w};
    const float gv[4] = {g4.x, g4.y, g4.z, g4.w};
    float o[4], gk[4], gq[4], part = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float e = __expf(gv[u]), ie = __expf(-gv[u]);
      const float kt = kv[u] * e, kb = kv[u] * ie, qt = qv[u] * e;
      const float dKt = b * dbk[u];
      gk[u] = dKt * e + dKb[u] * ie;
      gq[u] = dQt[u] * e;
      o[u] = dKt * kt + dQt[u] * qt - dKb[u] * kb;
      part += dbk[u] * kt;
    }
    st4io(dk_out + gi, gk);
    st4io(dq + gi, gq);
    *reinterpret_cast<float4*>(dg + r * dk + c) = make_float4(o[0], o[1], o[2], o[3]);
    pb[r * dk4 + c / 4] = part;
  }
  for (int idx = tid; idx < L * dv4; idx += kThreads) {
    const int r = idx / dv4, c = (idx % dv4) * 4;
    const size_t gi = ((size_t)(tok0 + r) * H + h) * dv + c;
    const float b = beta[(size_t)(tok0 + r) * H + h];
    const float4 x = ld4(w.dbv + gi);
    const float y[4] = {b * x.x, b * x.y, b * x.z, b * x.w};
    st4io(dv_out + gi, y);
  }
  __syncthreads();
  for (int c = tid; c < dk; c += kThreads) {
    float dgm = 0.f;
    for (int t = 0; t < ntile; ++t)
      dgm += w.dgam[(((size_t)cid * H + h) * ntile + t) * dk + c];
    dg[(L - 1) * dk + c] += dgm;  // the partials already carry gam
    float acc = 0.f;
    for (int r = L - 1; r >= 0; --r) {
      acc += dg[r * dk + c];
      dla[((size_t)(tok0 + r) * H + h) * dk + c] = acc;
    }
  }
  // d beta: one warp per row, lanes across the row, then a shuffle sum
  const int warp = tid >> 5, lane = tid & 31;
  for (int r = warp; r < L; r += kThreads / 32) {
    const size_t rv = ((size_t)(tok0 + r) * H + h) * dv;
    float acc = 0.f;
    for (int c = lane; c < dk4; c += 32) acc += pb[r * dk4 + c];
    for (int j = lane; j < dv; j += 32) acc += w.dbv[rv + j] * to_f32(v[rv + j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) dbeta[(size_t)(tok0 + r) * H + h] = acc;
  }
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)bytes);
}

// 16-byte loads each thread keeps in flight while staging a tensor-core
// operand (the staging is bound by their latency; eight and four measured
// slower than four and two).
constexpr int kDirectBatch = 4, kTransBatch = 2;

// op(A) (rows i, contraction t) as a K-major tf32 operand: 128-byte-swizzled
// panels of 32 t each, `rows` x 128 B per panel.  Source A[i][t]: each thread
// moves one 16-byte vector of a source row.
__device__ __forceinline__ void stage_km_direct(const Src& s, int rows, int cols,
                                                uint8_t* dst, int panel,
                                                int tid) {
  const int cv = cols >> 2, units = rows * cv;
  for (int base = 0; base < units; base += kDirectBatch * kThreads) {
    float4 v[kDirectBatch];
#pragma unroll
    for (int u = 0; u < kDirectBatch; ++u) {
      const int idx = base + u * kThreads + tid;
      v[u] = idx < units ? ld_src4(s, idx / cv, (idx % cv) * 4)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kDirectBatch; ++u) {
      const int idx = base + u * kThreads + tid;
      if (idx < units) {
        const int r = idx / cv, c = (idx % cv) * 4;
        *reinterpret_cast<float4*>(dst + (c >> 5) * panel +
                                   sm100::swz32(r, c & 31)) = v[u];
      }
    }
  }
}
// The same operand from a source stored the other way round, S[t][i]
// (source rows = t): consecutive threads take consecutive source rows, each
// reading 32 contiguous bytes, so the scalar shared stores of a warp fill one
// 128-byte panel row.
__device__ __forceinline__ void stage_km_transposed(const Src& s, int rows,
                                                    int cols, uint8_t* dst,
                                                    int panel, int tid) {
  const int units = rows * (cols >> 3);
  for (int base = 0; base < units; base += kTransBatch * kThreads) {
    float4 v[kTransBatch][2];
#pragma unroll
    for (int u = 0; u < kTransBatch; ++u) {
      const int idx = base + u * kThreads + tid;
      const int r = idx % rows, c = (idx / rows) * 8;
      const bool in = idx < units;
      v[u][0] = in ? ld_src4(s, r, c) : make_float4(0.f, 0.f, 0.f, 0.f);
      v[u][1] = in ? ld_src4(s, r, c + 4) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kTransBatch; ++u) {
      const int idx = base + u * kThreads + tid;
      if (idx < units) {
        const int r = idx % rows, c = (idx / rows) * 8;
        uint8_t* d = dst + (r >> 5) * panel;
        const float x[8] = {v[u][0].x, v[u][0].y, v[u][0].z, v[u][0].w,
                            v[u][1].x, v[u][1].y, v[u][1].z, v[u][1].w};
#pragma unroll
        for (int q = 0; q < 8; ++q)
          *reinterpret_cast<float*>(d + sm100::swz32(c + q, r & 31)) = x[q];
      }
    }
  }
}

// Tensor maps of the operands that TMA stages: [term][0 = A, 1 = B].
struct BmmMaps {
  CUtensorMap m[3][2];
};

// Tensor-core form of bmm_kernel for bf16 inputs in 64-token chunks (every
// dimension 64 or 128): per (chunk, head), each term's op(A) and op(B) are
// staged as K-major tf32 operands and multiplied by tcgen05 kind::tf32 into
// one TMEM accumulator of MD x ND; the epilogue applies alpha, the mask and
// the accumulation as bmm_kernel does.  MD = 64 uses the M = 64 shape, whose
// rows 16 q .. 16 q + 15 land in TMEM lanes 32 q .. 32 q + 15.
// Operands already K-major in memory (token rows or states whose rows are
// M or N) arrive by TMA, one 32-column box per panel (bit 2 term + side of
// tma_mask); the threads stage the others meanwhile.  A token box's rows
// past the chunk are other tokens (or zero past the tensor): they only
// reach output rows or columns past m or n, which are not stored.
// A CTA takes `per_cta` consecutive (chunk, head) items, heads fastest, and
// pays its set-up (barriers, TMEM allocation) once for all of them.
template <int MD, int ND>
__global__ void __launch_bounds__(kThreads, 3)
    bmm_tc_kernel(BmmOp op, const __grid_constant__ BmmMaps maps,
                  int tma_mask, const int32_t* cu, const int32_t* chunk_off,
                  int n_seqs, int T, int H, int dk, int dv, int C,
                  int64_t n_items, int per_cta) {
  using namespace sm100;
  const int tid = threadIdx.x, warp = tid >> 5;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int kPanA = MD * 128, kPanB = ND * 128;
  // panels per operand: the longest contraction of the op's terms / 32
  int npan = 1;
  for (int t = 0; t < op.nterms; ++t)
    npan = max(npan, (t == 0 ? op.term[0].kd : t == 1 ? op.term[1].kd
                                                       : op.term[2].kd) / 32);
  uint8_t* As = sm;                  // npan panels
  uint8_t* Bs = sm + npan * kPanA;   // npan panels
  uint64_t* bar = reinterpret_cast<uint64_t*>(Bs + npan * kPanB);
  uint64_t* tbar = bar + 1;  // TMA operand copies
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 2);
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(tbar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tslot, ND);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  bool ok = true;
  uint32_t tphase = 0, mphase = 0;  // completions of tbar and bar so far
  const int64_t item0 = (int64_t)blockIdx.x * per_cta;
  const int64_t item_end = min(item0 + per_cta, n_items);
  for (int64_t item = item0; item < item_end && ok; ++item) {
    const int cid = (int)(item / H), h = (int)(item % H);
    int seq, tok0, L;
    if (!locate_chunk(cid, cu, chunk_off, n_seqs, T, C, &seq, &tok0, &L))
      continue;
    for (int term = 0; term < op.nterms && ok; ++term) {
      const BmmTerm tm = term == 0 ? op.term[0]
                         : term == 1 ? op.term[1] : op.term[2];
      const int kd = tm.kd;
      const bool ta = (tma_mask >> (2 * term)) & 1;
      const bool tb = (tma_mask >> (2 * term + 1)) & 1;
      if (tid == 0 && (ta || tb)) {
        mbar_arrive_expect_tx(
            tbar, (ta ? (kd / 32) * kPanA : 0) + (tb ? (kd / 32) * kPanB : 0));
        for (int side = 0; side < 2; ++side) {
          if (!(side == 0 ? ta : tb)) continue;
          const MatRef& x = side == 0 ? tm.a : tm.b;
          uint8_t* dst = side == 0 ? As : Bs;
          const int pan = side == 0 ? kPanA : kPanB;
          for (int q = 0; q < kd / 32; ++q) {
            if (x.kind == kTok)
              tma_load_3d(dst + q * pan, &maps.m[term][side], tbar, 32 * q, h,
                          tok0);
            else  // states: d_k rows; transposed copies: x.cols rows
              tma_load_2d(dst + q * pan, &maps.m[term][side], tbar, 32 * q,
                          (int)(((size_t)cid * H + h) *
                                (x.kind == kState ? dk : x.cols)));
          }
        }
      }
      const Src sa = src_of(tm.a, cid, h, tok0, L, H, C, dk);
      const Src sb = src_of(tm.b, cid, h, tok0, L, H, C, dk);
      if (!ta) {
        if (tm.a.trans)  // A[t][i]
          stage_km_transposed(sa, kd, MD, As, kPanA, tid);
        else  // A[i][t]
          stage_km_direct(sa, MD, kd, As, kPanA, tid);
      }
      if (!tb) {
        if (tm.b.trans)  // B[j][t]
          stage_km_direct(sb, ND, kd, Bs, kPanB, tid);
        else  // B[t][j]
          stage_km_transposed(sb, kd, ND, Bs, kPanB, tid);
      }
      if (ta || tb) {
        ok = __syncthreads_and(mbar_wait(tbar, tphase & 1u, 2000000000ull));
        ++tphase;
        if (!ok) break;
      }
      fence_proxy_async();
      tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        constexpr uint32_t id = idesc_tf32(MD, ND);
        for (int ks = 0; ks < kd / 8; ++ks)
          mma_tf32(tmem,
                   desc_sw128(smem_u32(As) + (ks >> 2) * kPanA + (ks & 3) * 32,
                              16, 1024),
                   desc_sw128(smem_u32(Bs) + (ks >> 2) * kPanB + (ks & 3) * 32,
                              16, 1024),
                   id, (term > 0 || ks > 0) ? 1u : 0u);
        mma_commit(bar);
      }
      // the operands are read once the products complete: the next term may
      // then restage them
      ok = __syncthreads_and(mbar_wait(bar, mphase & 1u, 2000000000ull));
      ++mphase;
      tc_fence_after();
    }
    if (!ok) {
      if (tid == 0) atomicExch(&g_bwd_timeout, 1);
    } else {
      const int m = dim_of(op.m, L, dk, dv), n = dim_of(op.n, L, dk, dv);
      const Src so = src_of(op.out, cid, h, tok0, L, H, C, dk);
      const int lane = tid & 31, q = warp & 3, chalf = tid >> 7;
      const int i =
          MD == 128 ? 32 * q + lane : (lane < 16 ? 16 * q + lane : MD);
      const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16);
  #pragma unroll
      for (int cc = 0; cc < ND / 64; ++cc) {
        const int j0 = chalf * (ND / 2) + 32 * cc;
        float x[32];
        tmem_ld32(taddr + j0, x);
        if (i < m && j0 < n) {
  #pragma unroll
          for (int b = 0; b < 32; ++b) {
            const int j = j0 + b;
            x[b] *= op.alpha;
            if ((op.mask == kMaskLowerIncl && j > i) ||
                (op.mask == kMaskStrictLower && j >= i))
              x[b] = 0.f;
          }
          float* o = so.p + (size_t)i * so.stride + j0;
          if (j0 + 32 <= n) {
  #pragma unroll
            for (int v = 0; v < 8; ++v) {
              float4* o4 = reinterpret_cast<float4*>(o + 4 * v);
              float4 y = make_float4(x[4 * v], x[4 * v + 1], x[4 * v + 2],
                                     x[4 * v + 3]);
              if (op.accumulate) {
                const float4 z = *o4;
                y.x += z.x;
                y.y += z.y;
                y.z += z.z;
                y.w += z.w;
              }
              *o4 = y;
            }
          } else {
  #pragma unroll
            for (int b = 0; b < 32; ++b)
              if (j0 + b < n) o[b] = op.accumulate ? o[b] + x[b] : x[b];
          }
        }
      }
    }
    // this item's TMEM reads end before the next item's products start
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }  // items
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, ND);
}

// Items (chunk, head) one tensor-core product CTA takes in turn at most (the
// A/B on B = 2, T = 8192, H = 32, d = 128: 1 item 5.86 ms, 2 5.69, 4 5.66,
// 8 5.87 ms for the whole backward).
constexpr int kBmmItems = 4;

template <int MD, int ND>
cudaError_t launch_bmm_tc_t(const BmmOp& op, const BmmMaps& maps, int mask,
                            dim3 grid, cudaStream_t stream, const int32_t* cu,
                            const int32_t* co, int n_seqs, int T, int H,
                            int dk, int dv, int C) {
  // shared memory for the longest contraction of the op's terms: ops that
  // contract over 64 only fit twice as many CTAs on an SM
  int kdmax = 32;
  for (int t = 0; t < op.nterms; ++t)
    kdmax = op.term[t].kd > kdmax ? op.term[t].kd : kdmax;
  const size_t smem = (size_t)(kdmax / 32) * (MD + ND) * 128 + 1024 + 64;
  cudaError_t e = set_smem(bmm_tc_kernel<MD, ND>, smem);
  if (e != cudaSuccess) return e;
  // items per CTA: 4, 2 or 1, whichever still leaves two resident waves
  const int64_t items = (int64_t)grid.x * grid.y;
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) !=
          cudaSuccess ||
      (e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
           &per_sm, bmm_tc_kernel<MD, ND>, kThreads, smem)) != cudaSuccess)
    return e;
  const int64_t wave = (int64_t)sms * (per_sm > 0 ? per_sm : 1);
  const int per = items >= 2 * kBmmItems * wave ? kBmmItems
                  : items >= kBmmItems * wave   ? kBmmItems / 2
                                                : 1;
  const unsigned ctas = (unsigned)((items + per - 1) / per);
  bmm_tc_kernel<MD, ND><<<ctas, kThreads, smem, stream>>>(
      op, maps, mask, cu, co, n_seqs, T, H, dk, dv, C, items, per);
  return cudaGetLastError();
}

// The maps of the operands stored K-major with M or N as their rows: token
// rows (their rows are the chunk's tokens, M or N = 64), states whose rows
// are d_k, and the transposed per-chunk copies (rows = channels, K = the 64
// tokens, zero past the chunk).  Square per-chunk operands stay with the
// threads, which zero their entries past the chunk's length.
int bmm_tc_maps(const BmmOp& op, BmmMaps* maps, int tokens, int64_t nch,
                int H, int dk) {
  int mask = 0;
  for (int t = 0; t < op.nterms; ++t)
    for (int side = 0; side < 2; ++side) {
      const MatRef& x = side == 0 ? op.term[t].a : op.term[t].b;
      const bool direct = side == 0 ? !x.trans : x.trans;
      const int rows = side == 0 ? op.md : op.nd;  // the box's rows
      if (!direct) continue;
      bool ok = false;
      if (x.kind == kTok && rows == 64 && op.term[t].kd == x.cols)
        ok = make_f32_tok_map(&maps->m[t][side], x.p, x.cols, H, tokens);
      else if (x.kind == kState && rows == dk && op.term[t].kd == x.cols)
        ok = make_f32_rows_map(&maps->m[t][side], x.p, nch * H * dk, x.cols,
                               dk);
      else if (x.kind == kTokT && rows == x.cols && op.term[t].kd == 64)
        ok = make_f32_rows_map(&maps->m[t][side], x.p, nch * H * x.cols, 64,
                               x.cols);
      if (ok) mask |= 1 << (2 * t + side);
    }
  return mask;
}

cudaError_t launch_bmm_tc(const BmmOp& op, int C, dim3 grid,
                          cudaStream_t stream, const int32_t* cu,
                          const int32_t* co, int n_seqs, int T, int H, int dk,
                          int dv, int64_t nch) {
  BmmMaps maps;
  const int mask =
      bmm_tc_maps(op, &maps, cu ? T : n_seqs * T, nch, H, dk);
#define KDA_TC(M_, N_)                                                    \
  if (op.md == M_ && op.nd == N_)                                         \
    return launch_bmm_tc_t<M_, N_>(op, maps, mask, grid, stream, cu, co,  \
                                   n_seqs, T, H, dk, dv, C);
  KDA_TC(64, 64)
  KDA_TC(64, 128)
  KDA_TC(128, 64)
  KDA_TC(128, 128)
#undef KDA_TC
  return cudaErrorInvalidValue;
}

// Launch one batched product with the thread blocking its padded shape asks
// for: RM = md / 16 rows and RN = nd / 16 columns per thread.
template <int RM, int RN>
cudaError_t launch_bmm_t(const BmmOp& op, size_t smem, dim3 grid,
                         cudaStream_t stream, const int32_t* cu,
                         const int32_t* co, int n_seqs, int T, int H, int dk,
                         int dv, int C) {
  cudaError_t e = set_smem(bmm_kernel<RM, RN>, smem);
  if (e != cudaSuccess) return e;
  bmm_kernel<RM, RN><<<grid, kThreads, smem, stream>>>(op, cu, co, n_seqs, T, H,
                                                       dk, dv, C);
  return cudaGetLastError();
}

template <int RM>
cudaError_t launch_bmm_n(const BmmOp& op, int C, size_t smem, dim3 grid,
                         cudaStream_t stream, const int32_t* cu,
                         const int32_t* co, int n_seqs, int T, int H, int dk,
                         int dv) {
  switch (op.nd) {
    case 16: return launch_bmm_t<RM, 1>(op, smem, grid, stream, cu, co, n_seqs, T, H, dk, dv, C);
    case 32: return launch_bmm_t<RM, 2>(op, smem, grid, stream, cu, co, n_seqs, T, H, dk, dv, C);
    case 64: return launch_bmm_t<RM, 4>(op, smem, grid, stream, cu, co, n_seqs, T, H, dk, dv, C);
    case 128: return launch_bmm_t<RM, 8>(op, smem, grid, stream, cu, co, n_seqs, T, H, dk, dv, C);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_bmm(const BmmOp& op, int C, size_t smem, dim3 grid,
                       cudaStream_t stream, const int32_t* cu,
                       const int32_t* co, int n_seqs, int T, int H, int dk,
                       int dv) {
  switch (op.md) {
    case 16: return launch_bmm_n<1>(op, C, smem, grid, stream, cu, co, n_seqs, T, H, dk, dv);
    case 32: return launch_bmm_n<2>(op, C, smem, grid, stream, cu, co, n_seqs, T, H, dk, dv);
    case 64: return launch_bmm_n<4>(op, C, smem, grid, stream, cu, co, n_seqs, T, H, dk, dv);
    case 128: return launch_bmm_n<8>(op, C, smem, grid, stream, cu, co, n_seqs, T, H, dk, dv);
    default: return cudaErrorInvalidValue;
  }
}

template <typename IO>
cudaError_t run_bwd(const BwdArgs& a, void* workspace, cudaStream_t stream) {
  BwdWs w = carve_bwd(a, workspace, nullptr);
  const ChunkArgs f = forward_args(a, w.fin);
  // the forward's plan and cumulative log-decay (on the tensor-core path W,
  // U and the states have their own places in the shared workspace)
  const StagedView packed = w.fv;
  cudaError_t e = launch_staged_part(f, w.staged, &w.fv, false, stream);
  if (e != cudaSuccess) return e;
  if (packed.s) {
    w.fv.w = packed.w;
    w.fv.d = packed.d;
    w.fv.kh = nullptr;
    w.fv.s = packed.s;
  }
  const int C = f.chunk, H = f.H, dk = f.dk, dv = f.dv;
  const int64_t nch = max_chunks(f);
  const int32_t* cu = f.cu_seqlens;
  const int32_t* co = w.fv.chunk_off;
  const dim3 grid((unsigned)(nch > 0 ? nch : 1), H);

  if (nch > 0) {
    const bool tc = w.wt && sizeof(IO) == 2;
    const size_t smp = 4 * (3 * (size_t)prep_region(C, dk, dv) + C + dk);
    if (tc) {  // bf16 inputs in 64-token chunks: prep on the tensor cores
      const __nv_bfloat16* b16[4] = {
          reinterpret_cast<const __nv_bfloat16*>(f.q),
          reinterpret_cast<const __nv_bfloat16*>(f.k),
          reinterpret_cast<const __nv_bfloat16*>(f.v),
          reinterpret_cast<const __nv_bfloat16*>(a.d_out)};
      if (dk == 128) {
        const size_t sz = PrepTcLayout<128>::bytes + 1024;
        if ((e = set_smem(prep_tc_kernel<128>, sz)) != cudaSuccess) return e;
        prep_tc_kernel<128><<<grid, kThreads, sz, stream>>>(
            b16[0], b16[1], b16[2], f.beta, b16[3], w.fv.g, w, cu, co,
            f.n_seqs, f.T, H, dv);
      } else {
        const size_t sz = PrepTcLayout<64>::bytes + 1024;
        if ((e = set_smem(prep_tc_kernel<64>, sz)) != cudaSuccess) return e;
        prep_tc_kernel<64><<<grid, kThreads, sz, stream>>>(
            b16[0], b16[1], b16[2], f.beta, b16[3], w.fv.g, w, cu, co,
            f.n_seqs, f.T, H, dv);
      }
    } else if ((e = set_smem(prep_kernel<IO>, smp)) != cudaSuccess) {
      return e;
    } else {
    prep_kernel<IO><<<grid, kThreads, smp, stream>>>(
        static_cast<const IO*>(f.q), static_cast<const IO*>(f.k),
        static_cast<const IO*>(f.v), f.beta, static_cast<const IO*>(a.d_out),
        w.fv.g, w, w.fv.w, w.fv.d, w.fv.kh, w.wt, cu, co, f.n_seqs, f.T, H, dk,
        dv, C);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // the forward's serial state pass: chunk-start states, Delta over U, and
  // the final state (fp32 SIMT, or on the tensor cores with fp32-grade
  // operands: hi + lo tf32 parts of S and Delta)
  if (w.khT) {
    StateChainArgs sa{};
    sa.w = w.fv.w;
    sa.u = w.fv.d;
    sa.khT = w.khT;
    sa.gam = w.gam;
    sa.s = const_cast<float*>(w.fv.s);
    sa.s_init = f.initial_state;
    sa.s_final = w.fin;
    sa.cu = cu;
    sa.chunk_off = w.fv.chunk_off;
    sa.n_seqs = f.n_seqs;
    sa.T = f.T;
    sa.H = f.H;
    sa.dk = f.dk;
    sa.dv = f.dv;
    sa.n_chunks = max_chunks(f);
    e = launch_state_chain_tc(sa, stream);
  } else {
    e = launch_staged_part(f, w.staged, &w.fv, true, stream);
  }
  if (e != cudaSuccess) return e;

  auto tok = [](float* p, int cols, int t = 0) { return MatRef{p, kTok, cols, t}; };
  // token rows contracted over the tokens: the transposed per-chunk copy on
  // the tensor-core path (op = its transpose, K-major there), else the rows
  auto tokc = [&](float* rows, float* copy, int cols) {
    return copy ? MatRef{copy, kTokT, cols, 1} : MatRef{rows, kTok, cols, 0};
  };
  auto sq = [&](float* p, int t = 0) { return MatRef{p, kSq, C, t}; };
  auto stt = [&](const float* p, int t = 0) {
    return MatRef{const_cast<float*>(p), kState, dv, t};
  };
  auto dmax = [&](int code) { return code == kDimL ? C : code == kDimDk ? dk : dv; };
  auto term = [&](MatRef x, MatRef y, int k) { return BmmTerm{x, y, dmax(k)}; };
  auto bmm3 = [&](MatRef o, BmmTerm t0, BmmTerm t1, BmmTerm t2, int nterms,
                  int m, int n, int mask, float alpha, int accumulate) {
    BmmOp op{};
    op.out = o;
    op.term[0] = t0;
    op.term[1] = t1;
    op.term[2] = t2;
    op.nterms = nterms;
    op.m = m;
    op.n = n;
    op.md = dmax(m);
    op.nd = dmax(n);
    op.mask = mask;
    op.alpha = alpha;
    op.accumulate = accumulate;
    const int kd = max(t0.kd, max(nterms > 1 ? t1.kd : 0, nterms > 2 ? t2.kd : 0));
    if (w.wt)  // bf16 inputs in 64-token chunks: on the tensor cores (tf32)
      return launch_bmm_tc(op, C, grid, stream, cu, co, f.n_seqs, f.T, H, dk,
                           dv, nch);
    const size_t smem = 4 * (size_t)kd * ((op.md + 4) + (op.nd + 4));
    return launch_bmm(op, C, smem, grid, stream, cu, co, f.n_seqs, f.T, H, dk,
                      dv);
  };
  auto bmm2 = [&](MatRef o, BmmTerm t0, BmmTerm t1, int nterms, int m, int n,
                  int mask, float alpha, int accumulate) {
    return bmm3(o, t0, t1, t1, nterms, m, n, mask, alpha, accumulate);
  };
  auto bmm = [&](MatRef o, MatRef x, MatRef y, int n, int k, int mask,
                 float alpha, int accumulate) {
    const BmmTerm t = term(x, y, k);
    return bmm2(o, t, t, 1, kDimL, n, mask, alpha, accumulate);
  };
  float* De = w.fv.d;  // Delta
  const float* S0 = w.fv.s;
#define KDA_BMM(...) \
  if ((e = __VA_ARGS__) != cudaSuccess) return e;
  if (nch > 0) {
    // the chain's terms that do not depend on dS: Qt^T dO and P^T dO
    const BmmTerm tq =
        term(w.qtT ? MatRef{w.qtT, kTokT, dk, 0} : tok(w.qt, dk, 1),
             tokc(w.do32, w.doT, dv), kDimL);
    KDA_BMM(bmm2(stt(w.qdo), tq, tq, 1, kDimDk, kDimDv, kMaskNone, 1.f, 0))
    KDA_BMM(bmm(tok(w.pdo, dv), sq(w.pp, 1), tokc(w.do32, w.doT, dv), kDimDv,
                kDimL, kMaskNone, 1.f, 0))
  }
  if (w.wt) {  // on the tensor cores (tf32), one CTA per 64 d_v columns
    RevChainArgs r{};
    r.kb = w.kb;
    r.wt = w.wt;
    r.qdo = w.qdo;
    r.pdo = w.pdo;
    r.s = w.fv.s;
    r.fin = w.fin;
    r.gam = w.gam;
    r.d_final = a.d_final_state;
    r.gst = w.gst;
    r.dd = w.dd;
    r.dgam = w.dgam;
    r.ddT = w.ddT;
    r.d_init = a.d_initial_state;
    r.cu = cu;
    r.chunk_off = co;
    r.n_seqs = f.n_seqs;
    r.T = f.T;
    r.H = H;
    r.dk = dk;
    r.dv = dv;
    r.n_chunks = nch;
    if ((e = launch_rev_chain_tc(r, stream)) != cudaSuccess) return e;
  } else {
    constexpr int tp = kChainTile + 1;
    const size_t smc = 4 * ((size_t)dk * tp + 2 * (size_t)C * (dk + 1) +
                            (size_t)C * tp + dk);
    if ((e = set_smem(chain_kernel<kChainTile>, smc)) != cudaSuccess) return e;
    chain_kernel<kChainTile><<<dim3(f.n_seqs, H, dv / kChainTile), kThreads,
                               smc, stream>>>(w, a.d_final_state,
                                              a.d_initial_state, cu, f.n_seqs,
                                              f.T, H, dk, dv, C);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (nch == 0) return cudaSuccess;

  // dP = lower_incl(dO Delta^T)
  KDA_BMM(bmm(sq(w.dp), tok(w.do32, dv), tok(De, dv, 1), kDimL, kDimDv,
              kMaskLowerIncl, 1.f, 0))
  // dQt = dO S_0^T + dP Kb
  KDA_BMM(bmm2(tok(w.dqt, dk), term(tok(w.do32, dv), stt(S0, 1), kDimDv),
               term(sq(w.dp), tokc(w.kb, w.kbT, dk), kDimL), 2, kDimL, kDimDk,
               kMaskNone, 1.f, 0))
  // dW = -dDelta S_0^T
  KDA_BMM(bmm(tok(w.dw, dk), tok(w.dd, dv), stt(S0, 1), kDimDk, kDimDv,
              kMaskNone, -1.f, 0))
  // dTm = dW (b Kt)^T + dDelta (b V)^T
  KDA_BMM(bmm2(sq(w.dtm), term(tok(w.dw, dk), tok(w.bkt, dk, 1), kDimDk),
               term(tok(w.dd, dv), tok(w.bv, dv, 1), kDimDv), 2, kDimL, kDimL,
               kMaskNone, 1.f, 0))
  // Tm^T dDelta and Tm^T dTm
  // (the transposed copy of dDelta is negated)
  KDA_BMM(bmm(tok(w.dbv, dv), sq(w.tm, 1), tokc(w.dd, w.ddT, dv), kDimDv,
              kDimL, kMaskNone, w.ddT ? -1.f : 1.f, 0))
  KDA_BMM(bmm(sq(w.tmp), sq(w.tm, 1), sq(w.dtm), kDimL, kDimL, kMaskNone, 1.f,
              0))
  // dA = strictly_lower(-(Tm^T dTm) Tm^T)
  KDA_BMM(bmm(sq(w.da), sq(w.tmp), sq(w.tm, 1), kDimL, kDimL, kMaskStrictLower,
              -1.f, 0))
  // dKt / b = Tm^T dW + dA Kb
  KDA_BMM(bmm2(tok(w.dbk, dk), term(sq(w.tm, 1), tok(w.dw, dk), kDimL),
               term(sq(w.da), tokc(w.kb, w.kbT, dk), kDimL), 2, kDimL, kDimDk,
               kMaskNone, 1.f, 0))
  // dKb = Delta G^T + dP^T Qt + dA^T (b Kt)
  KDA_BMM(bmm3(tok(w.dkb, dk), term(tok(De, dv), stt(w.gst, 1), kDimDv),
               term(sq(w.dp, 1), tokc(w.qt, w.qtT, dk), kDimL),
               term(sq(w.da, 1), tokc(w.bkt, w.bktT, dk), kDimL), 3, kDimL,
               kDimDk,
               kMaskNone, 1.f, 0))
#undef KDA_BMM
  const size_t smf = 4 * (size_t)C * dk + (size_t)C * dk;
  if ((e = set_smem(final_kernel<IO>, smf)) != cudaSuccess) return e;
  final_kernel<IO><<<grid, kThreads, smf, stream>>>(
      w, static_cast<const IO*>(f.q), static_cast<const IO*>(f.k),
      static_cast<const IO*>(f.v), f.beta,
      w.fv.g, static_cast<IO*>(a.dq), static_cast<IO*>(a.dk),
      static_cast<IO*>(a.dv), a.d_log_alpha, a.d_beta, cu, co, f.n_seqs, f.T,
      H, dk, dv, C);
  return cudaGetLastError();
}

constexpr int kBmmOps = 11;

}  // namespace

cudaError_t bwd_take_range(cudaStream_t stream, int* flag) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  if ((e = cudaMemcpyFromSymbol(flag, g_bwd_range, sizeof(int))) != cudaSuccess)
    return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_bwd_range, &zero, sizeof(int));
}

cudaError_t bwd_take_timeout(cudaStream_t stream, int* flag) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  if ((e = cudaMemcpyFromSymbol(flag, g_bwd_timeout, sizeof(int))) !=
      cudaSuccess)
    return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_bwd_timeout, &zero, sizeof(int));
}

size_t bwd_workspace_bytes(const BwdArgs& a) {
  size_t total = 0;
  carve_bwd(a, nullptr, &total);
  return total;
}

int bwd_workspace_layout(const BwdArgs& a, BwdArray* out, int cap) {
  size_t total = 0;
  int count = 0;
  carve_bwd(a, nullptr, &total, out, out ? cap : 0, &count);
  return count;
}

int bwd_kernel_count(const BwdArgs& a) {
  const ChunkArgs f = forward_args(a, nullptr);
  if (f.n_seqs == 0 || f.H == 0) return 0;
  const bool any = max_chunks(f) > 0;
  // the plan (packed layout), the forward's state pass and the reverse chain
  // always; with any chunk also the cumulative log-decay, prep, the batched
  // products and the final combination
  return (f.cu_seqlens ? 1 : 0) + 2 + (any ? 1 + 1 + kBmmOps + 1 : 0);
}

cudaError_t launch_bwd(const BwdArgs& a, void* workspace, cudaStream_t stream) {
  if (a.f.n_seqs == 0 || a.f.H == 0) return cudaSuccess;
  return a.f.bf16 ? run_bwd<__nv_bfloat16>(a, workspace, stream)
                  : run_bwd<float>(a, workspace, stream);
}

}  // namespace kda
