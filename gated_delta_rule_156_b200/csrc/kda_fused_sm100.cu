// Fused chunkwise KDA prefill for sm_100a: one CTA walks all chunks of one
// (sequence, head, 64-column tile of d_v) with the fp32 state in registers,
// bf16 operands staged by TMA into 128-byte-swizzled shared memory and every
// dense chunk contraction on the 5th-generation tensor cores (tcgen05.mma,
// fp32 accumulators in TMEM).
//
// Per chunk of C = 64 tokens with chunk-start state S (rows = key channels):
//   g      = running sum of log(alpha) inside the chunk, per key channel
//   Kt     = k exp(g)   Qt = q exp(g)   Kb = k exp(-g)   Kh = k exp(g_C - g)
//   MMA1   [Kt; Qt] . Kb^T                 -> A_raw (rows 0-63), QK (64-127)
//   A      = strictly_lower(Diag(beta) A_raw);  P = lower_incl(QK)
//   Tm     = (I + A)^-1  (blocked forward substitution, fp32, 16x16 blocks)
//   T'     = Tm Diag(beta)
//   MMA2   [T'; P] . [Kt | V]               -> W = T' Kt, U = T' V (rows 0-63)
//   MMA3   [W; Qt] . S                      -> W S (rows 0-63), Qt S (64-127)
//   Delta  = U - W S
//   MMA4   Kh^T . Delta                     -> the state increment
//   MMA5   [T'; P] . Delta (accumulated)    -> rows 64-127: O = Qt S + P Delta
//   S      <- Diag(exp(g_C)) S + Kh^T Delta
// This is the recurrence S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1}
// + b_t k_t v_t^T, o_t = S_t^T q_t regrouped over chunks (the chunkwise,
// Diagonal-Plus-Low-Rank form: "Kimi Delta Attention", akshathtiwari.co.in;
// "You Could Have Come Up with Kimi Delta Attention", daily.dev, Summary).
//
// Layout notes: stacking the 64-row operands pairwise ([Kt; Qt], [W; Qt],
// [T'; P]) makes every MMA an M = 128 instruction whose accumulator row r is
// TMEM lane r, so each thread reads exactly the rows it owns: threads 0-63
// the W/U/Delta rows, threads 64-127 the P and output rows, thread c the
// state row of key channel c.  The same token-major 128-byte-swizzled tiles
// serve as K-major and MN-major operands, so no transposes are staged.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "kda_common.cuh"
#include "kda_internal.h"
#include "sm100_ptx.cuh"

namespace kda {

// Set by a kernel whose bounded wait gave up (read and cleared on the host).
__device__ int g_fused_timeout = 0;

namespace {

using namespace sm100;

constexpr int kC = 64;        // chunk length
constexpr int kDvt = 64;      // d_v columns per CTA
constexpr int kThreads = 256;
constexpr int kFS = 68;       // fp32 row stride (floats) of the A / Tm tiles

template <int DK>
struct Layout {
  static constexpr uint32_t NP = DK / 64;  // 64-channel panels
  static constexpr uint32_t stage_q = 0;                       // NP x 8 KB
  static constexpr uint32_t stage_k = stage_q + NP * 8192;     // NP x 8 KB
  static constexpr uint32_t stage_la = stage_k + NP * 8192;    // DK/32 x 8 KB
  static constexpr uint32_t vbuf = stage_la + (DK / 32) * 8192;  // 8 KB
  static constexpr uint32_t kq = vbuf + 8192;       // NP x 16 KB, 128 rows
  static constexpr uint32_t kb = kq + NP * 16384;   // NP x 8 KB
  static constexpr uint32_t kh = kb + NP * 8192;    // 2 x 8 KB (M = 128)
  static constexpr uint32_t tpp = kh + 2 * 8192;    // 16 KB, 128 rows x 64
  static constexpr uint32_t sop = tpp + 16384;      // DK rows x 128 B
  static constexpr uint32_t dop = sop + DK * 128;   // 64 rows x 128 B
  static constexpr uint32_t afp = dop + 8192;       // 64 x kFS fp32
  static constexpr uint32_t tfp = afp + 18432;      // 64 x kFS fp32
  static constexpr uint32_t msc = tfp + 18432;      // 1024 fp32 scratch
  static constexpr uint32_t misc = msc + 4096;      // beta, exp(g_C), barriers
  static constexpr uint32_t bytes = misc + 1024;
  static constexpr uint32_t tx_in = 2 * NP * 8192 + (DK / 32) * 8192;
  // TMEM columns
  static constexpr uint32_t t_d1 = 0;
  static constexpr uint32_t t_w = 64;
  static constexpr uint32_t t_u = 64 + DK;
  static constexpr uint32_t t_d3 = 128 + DK;
  static constexpr uint32_t t_d4 = 192 + DK;
};

struct FusedParams {
  const float* beta;
  const float* s_init;
  float* s_final;
  __nv_bfloat16* out;
  const int32_t* cu;
  const int32_t* order;  // sequence index by rank (packed layout), or null
  int n_seqs, T, H, dv, n_tiles;
};

// (I + A)^-1 for the strictly-lower 64 x 64 A in `A` (row stride kFS) into
// `X` (row stride kFS), by recursive doubling on unit-lower blocks:
//   [L11 0; L21 L22]^-1 = [X11 0; -X22 L21 X11  X22].
// Phase 0 inverts the four 16 x 16 diagonal blocks by forward substitution
// (one column per thread).  Phases 1-2 form the two 16 x 16 blocks (1,0) and
// (3,2) that complete the 32 x 32 diagonal halves; phases 3-4 form the
// 32 x 32 block coupling the halves.  Every product phase uses all threads
// with float4 operand loads.  `M` holds 1024 floats of scratch.  The
// strictly-upper part of X outside the diagonal 16-blocks is never written:
// the caller zeroes it once.
__device__ __forceinline__ void invert_unit_lower(const float* A, float* X,
                                                  float* M, int tid) {
  if (tid < 64) {
    const int o = (tid >> 4) * 16, j = tid & 15;
    float x[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float a[16];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        if (4 * q4 < r) {
          const float4 t =
              *reinterpret_cast<const float4*>(A + (o + r) * kFS + o + 4 * q4);
          a[4 * q4] = t.x; a[4 * q4 + 1] = t.y; a[4 * q4 + 2] = t.z;
          a[4 * q4 + 3] = t.w;
        }
      }
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int i = 0; i < r; ++i) {
        if (i & 1) s1 -= a[i] * x[i];
        else s0 -= a[i] * x[i];
      }
      x[r] = r < j ? 0.f : (r == j ? 1.f : s0 + s1);
    }
#pragma unroll
    for (int r = 0; r < 16; ++r) X[(o + r) * kFS + o + j] = x[r];
  }
  __syncthreads();
  {  // blocks (1,0) and (3,2): thread = (block b, row r, column pair c)
    const int b = tid >> 7, r = (tid >> 3) & 15, c = (tid & 7) * 2;
    const int bi = 2 * b + 1, bj = 2 * b;  // rows of block bi, cols of bj
    float m0 = 0.f, m1 = 0.f;
#pragma unroll
    for (int k = 0; k < 16; k += 4) {  // M = A_{bi,bj} X_{bj,bj}
      const float4 a4 =
          *reinterpret_cast<const float4*>(A + (16 * bi + r) * kFS + 16 * bj + k);
      const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 x2 = *reinterpret_cast<const float2*>(
            X + (16 * bj + k + u) * kFS + 16 * bj + c);
        m0 += av[u] * x2.x;
        m1 += av[u] * x2.y;
      }
    }
    *reinterpret_cast<float2*>(M + b * 256 + r * 16 + c) = make_float2(m0, m1);
    __syncthreads();
    float y0 = 0.f, y1 = 0.f;
#pragma unroll
    for (int k = 0; k < 16; k += 4) {  // X_{bi,bj} = -X_{bi,bi} M
      const float4 x4 =
          *reinterpret_cast<const float4*>(X + (16 * bi + r) * kFS + 16 * bi + k);
      const float xv[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 m2 =
            *reinterpret_cast<const float2*>(M + b * 256 + (k + u) * 16 + c);
        y0 -= xv[u] * m2.x;
        y1 -= xv[u] * m2.y;
      }
    }
    *reinterpret_cast<float2*>(X + (16 * bi + r) * kFS + 16 * bj + c) =
        make_float2(y0, y1);
  }
  __syncthreads();
  {  // the 32 x 32 block (rows 32-63, cols 0-31): thread = (row r, 4 cols)
    const int r = tid >> 3, c = (tid & 7) * 4;
    float m[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k = 0; k < 32; k += 4) {  // M = A_{21} X_{11}
      const float4 a4 =
          *reinterpret_cast<const float4*>(A + (32 + r) * kFS + k);
      const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float4 x4 =
            *reinterpret_cast<const float4*>(X + (k + u) * kFS + c);
        m[0] += av[u] * x4.x; m[1] += av[u] * x4.y;
        m[2] += av[u] * x4.z; m[3] += av[u] * x4.w;
      }
    }
    *reinterpret_cast<float4*>(M + r * 32 + c) = make_float4(m[0], m[1], m[2], m[3]);
    __syncthreads();
    float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k = 0; k < 32; k += 4) {  // X_{21} = -X_{22} M
      const float4 x4 =
          *reinterpret_cast<const float4*>(X + (32 + r) * kFS + 32 + k);
      const float xv[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float4 m4 = *reinterpret_cast<const float4*>(M + (k + u) * 32 + c);
        y[0] -= xv[u] * m4.x; y[1] -= xv[u] * m4.y;
        y[2] -= xv[u] * m4.z; y[3] -= xv[u] * m4.w;
      }
    }
    *reinterpret_cast<float4*>(X + (32 + r) * kFS + c) =
        make_float4(y[0], y[1], y[2], y[3]);
  }
  __syncthreads();
}

// Store `n` consecutive 16-byte chunks (8 bf16 each, starting at chunk
// `c0`) of one row of a 128-byte-swizzled panel.
template <int N>
__device__ __forceinline__ void st_chunks_sw128(uint8_t* panel, int row, int c0,
                                                const float* v) {
#pragma unroll
  for (int c = 0; c < N; ++c) {
    uint4 w;
    w.x = pack_bf16x2(v[8 * c + 0], v[8 * c + 1]);
    w.y = pack_bf16x2(v[8 * c + 2], v[8 * c + 3]);
    w.z = pack_bf16x2(v[8 * c + 4], v[8 * c + 5]);
    w.w = pack_bf16x2(v[8 * c + 6], v[8 * c + 7]);
    *reinterpret_cast<uint4*>(panel + row * 128 + (((c0 + c) ^ (row & 7)) << 4)) =
        w;
  }
}

template <int DK>
__global__ void __launch_bounds__(kThreads, 1)
    fused_kernel(const __grid_constant__ CUtensorMap tm_q,
                 const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v,
                 const __grid_constant__ CUtensorMap tm_la,
                 const FusedParams p) {
  using Lay = Layout<DK>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* st_q = sm + Lay::stage_q;
  uint8_t* st_k = sm + Lay::stage_k;
  const float* st_la = reinterpret_cast<const float*>(sm + Lay::stage_la);
  uint8_t* vbuf = sm + Lay::vbuf;
  uint8_t* kq = sm + Lay::kq;
  uint8_t* kb = sm + Lay::kb;
  uint8_t* kh = sm + Lay::kh;
  uint8_t* tpp = sm + Lay::tpp;
  uint8_t* sop = sm + Lay::sop;
  uint8_t* dop = sm + Lay::dop;
  float* afp = reinterpret_cast<float*>(sm + Lay::afp);
  float* tfp = reinterpret_cast<float*>(sm + Lay::tfp);
  float* msc = reinterpret_cast<float*>(sm + Lay::msc);
  float* red = afp;  // the prologue's partial sums (afp is free then)
  float* beta_s = reinterpret_cast<float*>(sm + Lay::misc);        // [64]
  float* gexp_s = reinterpret_cast<float*>(sm + Lay::misc + 256);  // [DK]
  uint64_t* bar_in = reinterpret_cast<uint64_t*>(sm + Lay::misc + 768);
  uint64_t* bar_v = bar_in + 1;
  uint64_t* bar_mma = bar_in + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_in + 3);

  const int tid = threadIdx.x, warp = tid >> 5;
  // TMEM access: warp w reads lanes 32 (w % 4) .. +31; warps 0-3 take the
  // first 32 columns of a 64-column accumulator, warps 4-7 the second.
  const int row_t = tid & 127;  // this thread's TMEM lane / accumulator row
  const int colh = warp >> 2;   // which 32-column half
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;

  const int u = blockIdx.x;
  const int tile = u % p.n_tiles;
  const int h = (u / p.n_tiles) % p.H;
  const int rank = u / (p.n_tiles * p.H);
  const int seq = p.order ? p.order[rank] : rank;
  const int j0 = tile * kDvt;
  int start, end;
  seq_range(p.cu, seq, p.T, &start, &end);
  const int nch = (end - start + kC - 1) / kC;

  if (tid == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_la);
    mbar_init(bar_in, 1);
    mbar_init(bar_v, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  for (int i = tid; i < 64 * kFS; i += kThreads) tfp[i] = 0.f;
  if (DK == 64) {  // channels 64-127 of the M = 128 Kh^T operand stay zero
    uint4* z = reinterpret_cast<uint4*>(kh + 8192);
    for (int i = tid; i < 512; i += kThreads) z[i] = make_uint4(0, 0, 0, 0);
  }

  // The state tile: thread t owns row row_t (key channel), columns
  // 32 colh .. 32 colh + 31 of this CTA's 64-column tile, in fp32 registers.
  const bool owns_state = row_t < DK;
  float s[32];
  const size_t sbase = (((size_t)seq * p.H + h) * DK) * p.dv + j0;
  if (owns_state) {
    if (p.s_init) {
      const float4* src = reinterpret_cast<const float4*>(
          p.s_init + sbase + (size_t)row_t * p.dv + 32 * colh);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 x = src[i];
        s[4 * i] = x.x; s[4 * i + 1] = x.y; s[4 * i + 2] = x.z; s[4 * i + 3] = x.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) s[i] = 0.f;
    }
    st_chunks_sw128<4>(sop, row_t, 4 * colh, s);
  }

  auto issue_inputs = [&](int tok) {
    mbar_arrive_expect_tx(bar_in, Lay::tx_in);
#pragma unroll
    for (int pnl = 0; pnl < (int)Lay::NP; ++pnl) {
      tma_load_3d(st_q + pnl * 8192, &tm_q, bar_in, pnl * 64, h, tok);
      tma_load_3d(st_k + pnl * 8192, &tm_k, bar_in, pnl * 64, h, tok);
    }
#pragma unroll
    for (int b = 0; b < DK / 32; ++b)
      tma_load_3d(sm + Lay::stage_la + b * 8192, &tm_la, bar_in, b * 32, h, tok);
  };
  auto issue_v = [&](int tok) {
    mbar_arrive_expect_tx(bar_v, 8192);
    tma_load_3d(vbuf, &tm_v, bar_v, j0, h, tok);
  };

  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (tid == 0 && nch > 0) {
    issue_inputs(start);
    issue_v(start);
  }
  float beta_next = 0.f;
  if (tid < kC && nch > 0 && tid < end - start)
    beta_next = p.beta[(size_t)(start + tid) * p.H + h];

  uint32_t ph_in = 0, ph_v = 0, ph_mma = 0;
  bool failed = false;
  bool in_flight = false;    // an input TMA was issued and not waited for
  bool v_pending = nch > 0;  // (thread 0) a V TMA was issued, not waited for

  for (int n = 0; n < nch; ++n) {
    const int tok0 = start + n * kC;
    const int L = min(kC, end - tok0);
    const bool has_next = n + 1 < nch;
    if (tid < kC) {
      beta_s[tid] = beta_next;
      beta_next = 0.f;
      if (has_next && tid < end - (tok0 + kC))
        beta_next = p.beta[(size_t)(tok0 + kC + tid) * p.H + h];
    }

    // ---- inputs of this chunk have landed
    bool ok = mbar_wait(bar_in, ph_in);
    ph_in ^= 1;
    in_flight = false;
    if (__syncthreads_or(!ok)) { failed = true; break; }

    // ---- prologue: decay prefix sums and the four scaled copies of k, q.
    // Thread = (4-channel group cg, block of RPT consecutive rows).  The
    // products are formed in packed bf16 (the operands are bf16 anyway).
    {
      constexpr int NCG = DK / 4;                 // channel groups
      constexpr int NRB = kThreads / NCG;         // row blocks
      constexpr int RPT = kC / NRB;               // rows per thread
      const int cg = tid % NCG, rb = tid / NCG;
      const int pnl = cg >> 4;                    // 64-channel panel
      const int ck = (cg >> 1) & 7;               // 16-byte chunk in the row
      const int cb = (cg & 1) * 8;                // byte offset in the chunk
      const float* la_base = st_la + (cg >> 3) * (64 * 32) + (cg & 7) * 4;
      float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
        const int r = rb * RPT + i;
        if (r < L) {
          const float4 x = *reinterpret_cast<const float4*>(la_base + r * 32);
          part[0] += x.x; part[1] += x.y; part[2] += x.z; part[3] += x.w;
        }
      }
      *reinterpret_cast<float4*>(red + rb * DK + 4 * cg) =
          make_float4(part[0], part[1], part[2], part[3]);
      __syncthreads();
      float g[4] = {0.f, 0.f, 0.f, 0.f}, tot[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int b2 = 0; b2 < NRB; ++b2) {
        const float4 y = *reinterpret_cast<const float4*>(red + b2 * DK + 4 * cg);
        if (b2 < rb) { g[0] += y.x; g[1] += y.y; g[2] += y.z; g[3] += y.w; }
        tot[0] += y.x; tot[1] += y.y; tot[2] += y.z; tot[3] += y.w;
      }
      constexpr float kLog2e = 1.4426950408889634f;
      float gct[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) gct[c] = ex2_approx(tot[c] * kLog2e);
      if (rb == 0)
        *reinterpret_cast<float4*>(gexp_s + 4 * cg) =
            make_float4(gct[0], gct[1], gct[2], gct[3]);
      const __nv_bfloat162 gc01 = __floats2bfloat162_rn(gct[0], gct[1]);
      const __nv_bfloat162 gc23 = __floats2bfloat162_rn(gct[2], gct[3]);
      const uint8_t* pq = st_q + pnl * 8192;
      const uint8_t* pk = st_k + pnl * 8192;
      uint8_t* pkq = kq + pnl * 16384;
      uint8_t* pkb = kb + pnl * 8192;
      uint8_t* pkh = kh + pnl * 8192;
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
        const int r = rb * RPT + i;
        const uint32_t off = r * 128 + ((ck ^ (r & 7)) << 4) + cb;
        const bool valid = r < L;
        const uint2 kr = *reinterpret_cast<const uint2*>(pk + off);
        const uint2 qr = *reinterpret_cast<const uint2*>(pq + off);
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (valid) x = *reinterpret_cast<const float4*>(la_base + r * 32);
        g[0] += x.x; g[1] += x.y; g[2] += x.z; g[3] += x.w;
        float e[4], ie[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float t = g[c] * kLog2e;
          e[c] = valid ? ex2_approx(t) : 0.f;
          ie[c] = valid ? ex2_approx(-t) : 0.f;
        }
        const __nv_bfloat162 e01 = __floats2bfloat162_rn(e[0], e[1]);
        const __nv_bfloat162 e23 = __floats2bfloat162_rn(e[2], e[3]);
        const __nv_bfloat162 i01 = __floats2bfloat162_rn(ie[0], ie[1]);
        const __nv_bfloat162 i23 = __floats2bfloat162_rn(ie[2], ie[3]);
        const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kr);
        const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(&qr);
        const __nv_bfloat162 kb01 = __hmul2(k2[0], i01), kb23 = __hmul2(k2[1], i23);
        uint2 wt, wq, wb, wh;
        *reinterpret_cast<__nv_bfloat162*>(&wt.x) = __hmul2(k2[0], e01);
        *reinterpret_cast<__nv_bfloat162*>(&wt.y) = __hmul2(k2[1], e23);
        *reinterpret_cast<__nv_bfloat162*>(&wq.x) = __hmul2(q2[0], e01);
        *reinterpret_cast<__nv_bfloat162*>(&wq.y) = __hmul2(q2[1], e23);
        *reinterpret_cast<__nv_bfloat162*>(&wb.x) = kb01;
        *reinterpret_cast<__nv_bfloat162*>(&wb.y) = kb23;
        *reinterpret_cast<__nv_bfloat162*>(&wh.x) = __hmul2(kb01, gc01);
        *reinterpret_cast<__nv_bfloat162*>(&wh.y) = __hmul2(kb23, gc23);
        *reinterpret_cast<uint2*>(pkq + off) = wt;
        *reinterpret_cast<uint2*>(pkq + 64 * 128 + off) = wq;
        *reinterpret_cast<uint2*>(pkb + off) = wb;
        *reinterpret_cast<uint2*>(pkh + off) = wh;
      }
    }
    fence_proxy_async();
    __syncthreads();
    const float gexp_c = owns_state ? gexp_s[row_t] : 1.f;

    // ---- MMA1: [Kt; Qt] . Kb^T ; then prefetch the next chunk's inputs
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16(128, 64, false, false);
#pragma unroll
      for (int ks = 0; ks < DK / 16; ++ks) {
        const uint32_t off = (ks & 3) * 32;
        mma_bf16(tmem + Lay::t_d1,
                 desc_sw128(smem_u32(kq) + (ks >> 2) * 16384 + off, 16, 1024),
                 desc_sw128(smem_u32(kb) + (ks >> 2) * 8192 + off, 16, 1024),
                 idesc, ks > 0);
      }
      mma_commit(bar_mma);
      if (has_next) issue_inputs(tok0 + kC);
    }
    in_flight = has_next;
    ok = mbar_wait(bar_mma, ph_mma);
    ph_mma ^= 1;
    if (__syncthreads_or(!ok)) { failed = true; break; }
    tc_fence_after();

    // ---- A (rows 0-63, fp32) and P (rows 64-127, bf16 into [T'; P])
    {
      float v[32];
      tmem_ld32(tmem + lane_base + Lay::t_d1 + 32 * colh, v);
      if (row_t < 64) {
        const float b = beta_s[row_t];
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const int c = 32 * colh + i;
          float4 w;
          w.x = c + 0 < row_t ? b * v[i + 0] : 0.f;
          w.y = c + 1 < row_t ? b * v[i + 1] : 0.f;
          w.z = c + 2 < row_t ? b * v[i + 2] : 0.f;
          w.w = c + 3 < row_t ? b * v[i + 3] : 0.f;
          *reinterpret_cast<float4*>(afp + row_t * kFS + c) = w;
        }
      } else {
        const int r = row_t - 64;
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 32 * colh + i <= r ? v[i] : 0.f;
        st_chunks_sw128<4>(tpp, row_t, 4 * colh, v);
      }
    }
    tc_fence_before();
    __syncthreads();

    invert_unit_lower(afp, tfp, msc, tid);

    {  // T' = Tm Diag(beta): row tid % 64, 16 columns per thread
      const int r = tid & 63, qc = tid >> 6;
      float v[16];
#pragma unroll
      for (int i = 0; i < 16; i += 4) {
        const float4 t =
            *reinterpret_cast<const float4*>(tfp + r * kFS + 16 * qc + i);
        const float4 b = *reinterpret_cast<const float4*>(beta_s + 16 * qc + i);
        v[i] = t.x * b.x; v[i + 1] = t.y * b.y; v[i + 2] = t.z * b.z;
        v[i + 3] = t.w * b.w;
      }
      st_chunks_sw128<2>(tpp, r, 2 * qc, v);
    }
    fence_proxy_async();
    __syncthreads();

    // ---- MMA2: W = T' Kt (N = DK), U = T' V (N = 64)
    if (tid == 0) {
      tc_fence_after();
      ok = mbar_wait(bar_v, ph_v);
      ph_v ^= 1;
      v_pending = !ok;
      if (ok) {
        const uint32_t iw = idesc_bf16(128, DK, false, true);
        const uint32_t iu = idesc_bf16(128, 64, false, true);
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks) {
          const uint64_t a = desc_sw128(smem_u32(tpp) + ks * 32, 16, 1024);
          mma_bf16(tmem + Lay::t_w, a,
                   desc_sw128(smem_u32(kq) + ks * 2048, 16384, 1024), iw, ks > 0);
          mma_bf16(tmem + Lay::t_u, a,
                   desc_sw128(smem_u32(vbuf) + ks * 2048, 8192, 1024), iu, ks > 0);
        }
        mma_commit(bar_mma);
      }
    }
    if (__syncthreads_or(!ok)) { failed = true; break; }
    ok = mbar_wait(bar_mma, ph_mma);
    ph_mma ^= 1;
    if (__syncthreads_or(!ok)) { failed = true; break; }
    tc_fence_after();

    // ---- W rows (bf16) over the Kt rows of [Kt; Qt] -> [W; Qt]
    if (row_t < 64) {
#pragma unroll
      for (int j = 0; j < DK / 64; ++j) {
        const int hh = colh * (DK / 64) + j;  // 32-column piece of the row
        float v[32];
        tmem_ld32(tmem + lane_base + Lay::t_w + 32 * hh, v);
        st_chunks_sw128<4>(kq + (hh >> 1) * 16384, row_t, 4 * (hh & 1), v);
      }
    }
    tc_fence_before();
    fence_proxy_async();
    __syncthreads();

    // ---- MMA3: [W; Qt] . S ; V buffer is free for the next chunk
    if (tid == 0) {
      tc_fence_after();
      if (has_next) {
        issue_v(tok0 + kC);
        v_pending = true;
      }
      const uint32_t idesc = idesc_bf16(128, 64, false, true);
#pragma unroll
      for (int ks = 0; ks < DK / 16; ++ks)
        mma_bf16(tmem + Lay::t_d3,
                 desc_sw128(smem_u32(kq) + (ks >> 2) * 16384 + (ks & 3) * 32,
                            16, 1024),
                 desc_sw128(smem_u32(sop) + ks * 2048, 8192, 1024), idesc,
                 ks > 0);
      mma_commit(bar_mma);
    }
    ok = mbar_wait(bar_mma, ph_mma);
    ph_mma ^= 1;
    if (__syncthreads_or(!ok)) { failed = true; break; }
    tc_fence_after();

    // ---- Delta = U - W S  (rows 0-63), bf16 into the MN-major Delta tile
    if (row_t < 64) {
      float uu[32], ws[32];
      tmem_ld32(tmem + lane_base + Lay::t_u + 32 * colh, uu);
      tmem_ld32(tmem + lane_base + Lay::t_d3 + 32 * colh, ws);
#pragma unroll
      for (int i = 0; i < 32; ++i) uu[i] -= ws[i];
      st_chunks_sw128<4>(dop, row_t, 4 * colh, uu);
    }
    tc_fence_before();
    fence_proxy_async();
    __syncthreads();

    // ---- MMA4: Kh^T . Delta ; MMA5: [T'; P] . Delta accumulated onto Qt S
    if (tid == 0) {
      tc_fence_after();
      const uint32_t i4 = idesc_bf16(128, 64, true, true);
      const uint32_t i5 = idesc_bf16(128, 64, false, true);
#pragma unroll
      for (int ks = 0; ks < kC / 16; ++ks) {
        const uint64_t bd = desc_sw128(smem_u32(dop) + ks * 2048, 8192, 1024);
        mma_bf16(tmem + Lay::t_d4,
                 desc_sw128(smem_u32(kh) + ks * 2048, 8192, 1024), bd, i4,
                 ks > 0);
        mma_bf16(tmem + Lay::t_d3,
                 desc_sw128(smem_u32(tpp) + ks * 32, 16, 1024), bd, i5, 1u);
      }
      mma_commit(bar_mma);
    }
    ok = mbar_wait(bar_mma, ph_mma);
    ph_mma ^= 1;
    if (__syncthreads_or(!ok)) { failed = true; break; }
    tc_fence_after();

    // ---- outputs (rows 64-127) and the state update (row per channel)
    if (row_t >= 64) {
      const int r = row_t - 64;
      float o[32];
      tmem_ld32(tmem + lane_base + Lay::t_d3 + 32 * colh, o);
      if (r < L) {
        uint4* dst = reinterpret_cast<uint4*>(
            p.out + ((size_t)(tok0 + r) * p.H + h) * p.dv + j0 + 32 * colh);
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint4 w;
          w.x = pack_bf16x2(o[8 * ch + 0], o[8 * ch + 1]);
          w.y = pack_bf16x2(o[8 * ch + 2], o[8 * ch + 3]);
          w.z = pack_bf16x2(o[8 * ch + 4], o[8 * ch + 5]);
          w.w = pack_bf16x2(o[8 * ch + 6], o[8 * ch + 7]);
          dst[ch] = w;
        }
      }
    }
    {
      float d4[32];
      tmem_ld32(tmem + lane_base + Lay::t_d4 + 32 * colh, d4);
      if (owns_state) {
#pragma unroll
        for (int i = 0; i < 32; ++i) s[i] = gexp_c * s[i] + d4[i];
        st_chunks_sw128<4>(sop, row_t, 4 * colh, s);
      }
    }
    tc_fence_before();
    fence_proxy_async();
    __syncthreads();
  }

  if (failed) {
    if (tid == 0) {
      atomicExch(&g_fused_timeout, 1);
      if (in_flight) mbar_wait(bar_in, ph_in, 100000000ull);
      if (v_pending) mbar_wait(bar_v, ph_v, 100000000ull);
    }
  } else if (owns_state) {
    float4* dst = reinterpret_cast<float4*>(p.s_final + sbase +
                                            (size_t)row_t * p.dv + 32 * colh);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      dst[i] = make_float4(s[4 * i], s[4 * i + 1], s[4 * i + 2], s[4 * i + 3]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

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

namespace kda {
namespace {

int64_t total_tokens(const ChunkArgs& a) {
  return a.cu_seqlens ? (int64_t)a.T : (int64_t)a.n_seqs * a.T;
}

template <int DK>
cudaError_t run(const ChunkArgs& a, void* workspace, cudaStream_t stream) {
  using Lay = Layout<DK>;
  const int tokens = (int)total_tokens(a);
  CUtensorMap tq, tk, tv, tl;
  if (!make_map(&tq, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DK, a.H, tokens,
                64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tk, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DK, a.H, tokens,
                64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tv, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.dv, a.H,
                tokens, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tl, a.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, DK, a.H,
                tokens, 32, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  FusedParams p{};
  p.beta = a.beta;
  p.s_init = a.initial_state;
  p.s_final = a.final_state;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.cu = a.cu_seqlens;
  p.order = nullptr;
  p.n_seqs = a.n_seqs;
  p.T = a.T;
  p.H = a.H;
  p.dv = a.dv;
  p.n_tiles = a.dv / kDvt;
  cudaError_t e;
  if (a.cu_seqlens) {
    int32_t* order = static_cast<int32_t*>(workspace);
    order_kernel<<<1, 1024, 0, stream>>>(a.cu_seqlens, a.n_seqs, a.T, order);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    p.order = order;
  }
  const size_t smem = Lay::bytes + 1024;
  if ((e = cudaFuncSetAttribute(fused_kernel<DK>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem)) != cudaSuccess)
    return e;
  const unsigned grid = (unsigned)a.n_seqs * a.H * p.n_tiles;
  fused_kernel<DK><<<grid, kThreads, smem, stream>>>(tq, tk, tv, tl, p);
  return cudaGetLastError();
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

cudaError_t fused_take_timeout(cudaStream_t stream, int* flag) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  int zero = 0;
  if ((e = cudaMemcpyFromSymbol(flag, g_fused_timeout, sizeof(int))) !=
      cudaSuccess)
    return e;
  return cudaMemcpyToSymbol(g_fused_timeout, &zero, sizeof(int));
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
  return ws::launch_fused_ws(a, order, stream);
}

}  // namespace kda
