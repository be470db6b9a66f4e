// The two serial chains of the chunkwise backward pass on the tensor cores
// (tcgen05 kind::tf32, fp32 operands in 128-byte-swizzled shared memory,
// fp32 accumulators in TMEM): the reverse state-gradient chain
// (rev_chain_kernel, below) and the backward's copy of the forward's state
// pass (state_chain_kernel, at the end of the file).  Included by
// kda_fused_sm100.cu, whose tensor-map encoder and device timeout flag they
// share.
//
// The reverse chain:
// Per chunk, walking each sequence's chunks from last to first, with dS the
// gradient of the state leaving the chunk (the chain rule applied to the
// chunkwise form S_C = Diag(gam)(S_0 + Kb^T Delta), Delta = U - W S_0; "You
// Could Have Come Up with Kimi Delta Attention", daily.dev, Summary):
//   gam * d gam = rowsum(S_next * dS)      (S_next = Diag(gam)(S_0 + Kb^T
//                                           Delta), the next start state)
//   G      = Diag(gam) dS
//   dDelta = Kb G + P^T dO                 (MMA 1: M = 64 tokens, K = d_k)
//   dS    <- G + Qt^T dO - W^T dDelta      (MMA 2: M = d_k, K = 64 tokens)
// G, dDelta (and -dDelta^T per chunk) and the gam * d gam partials go to the
// workspace for the batched products that follow; the last dS is the
// initial-state gradient.
//
// One CTA of 256 threads per (sequence, head, 64-column d_v tile); thread c
// owns TMEM lane c % 128 and 32 columns 32 (c / 128) .. + 31.  dS stays in
// TMEM from the first step to the last.  Every tile moves by TMA, so global
// traffic is coalesced although each thread owns one row: Kb and W^T
// (written transposed by the backward's prep kernel) for the products,
// Qt^T dO, the next start state and P^T dO for the epilogues, each fetched
// for the next chunk as soon as its buffer is free; G and dDelta are written
// in place of Qt^T dO and P^T dO and stored by TMA.  The epilogues also write
// G and -dDelta straight into the K-major B operands of the two products.
// tf32 operands need K-major layouts on both sides, hence the transposed
// copy of W.
namespace kda {
namespace bwdtc {

using sm100::idesc_tf32;
using sm100::tf32_rna;
using sm100::tma_load_2d;
using sm100::mma_tf32;
using sm100::swz32;
using ws::named_sync_or;
using ws::tmem_st32;
using ws::tmem_wait_st;
using ws::wait_or_abort;

constexpr int kC = 64;        // chunk length
constexpr int kTile = 64;     // d_v columns per CTA
constexpr int kThreads = 256;
constexpr int kBarAll = 1;

struct Params {
  const float* gam;      // exp(g_C)     [chunks, H, dk]
  const float* d_final;  // [n_seqs, H, dk, dv] or null (zero)
  float* dd;             // dDelta [tokens, H, dv] (ragged chunks' rows)
  float* dgam;           // partials     [chunks, H, dv / 32, dk]
  float* d_init;         // [n_seqs, H, dk, dv] or null
  const int32_t* cu;
  const int32_t* chunk_off;
  int n_seqs, T, H, dv;
  int store_ddt;         // also store -dDelta^T per chunk (map ddt)
};

// The fp32 tensor maps (128-byte swizzle, boxes 32 columns wide): Kb and
// P^T dO / dDelta over [tokens, H, d] (64-token boxes); W^T over
// [chunks * H * dk, 64]; Qt^T dO, the start states, G over
// [chunks * H * dk, dv] and the final states over [n_seqs * H * dk, dv]
// (d_k-row boxes); -dDelta^T over [chunks * H * dv, 64] (64-row boxes).
struct Maps {
  CUtensorMap kb, wt, qdo, s, fin, pdo, gst, dd, ddt;
};

template <int DK>
struct Layout {
  // Kb: DK / 32 panels of 64 token rows x 128 B, plus one more panel of
  // padding, since the M = 128 product reads 128 rows from each panel start
  static constexpr uint32_t kb_bytes = (DK / 32 + 1) * 8192;
  static constexpr uint32_t kb = 0;
  // W^T: two panels (tokens 0-31, 32-63) of 128 rows (d_k, padded) x 128 B
  static constexpr uint32_t wt = kb + kb_bytes;
  static constexpr uint32_t gop = wt + 2 * 16384;        // G: 64 rows (j) x DK
  static constexpr uint32_t dop = gop + (DK / 32) * 8192; // -dDelta: 64 x 64
  // Qt^T dO (then G) and the next start state: two panels (32 columns
  // each) of DK rows x 128 B; P^T dO (then dDelta): two of 64 rows
  static constexpr uint32_t qt = dop + 2 * 8192;
  static constexpr uint32_t st = qt + 2 * DK * 128;
  static constexpr uint32_t pt = st + 2 * DK * 128;
  static constexpr uint32_t misc = pt + 2 * 8192;
  static constexpr uint32_t bytes = misc + 256;
  static constexpr uint32_t kb_tx = (DK / 32) * 8192;
  static constexpr uint32_t wt_tx = 2 * DK * 128;
  static constexpr uint32_t qt_tx = 2 * DK * 128;
  static constexpr uint32_t pt_tx = 2 * 8192;
  static constexpr uint32_t t_ds = 0, t_dd = 64;  // TMEM columns
  static_assert(bytes + 1024 <= 232448, "shared memory");
};

__device__ __forceinline__ void tma_store_2d(const void* tmap, const void* src,
                                             int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], "
      "[%1];" ::"l"(reinterpret_cast<uint64_t>(tmap)),
      "r"(sm100::smem_u32(src)), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_store_3d(const void* tmap, const void* src,
                                             int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, "
      "%4}], [%1];" ::"l"(reinterpret_cast<uint64_t>(tmap)),
      "r"(sm100::smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Until every bulk store committed so far has read its shared-memory source.
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

template <int DK>
__global__ void __launch_bounds__(kThreads, 1)
    rev_chain_kernel(const __grid_constant__ Maps m, const Params p) {
  using namespace sm100;
  using Lay = Layout<DK>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* kb = sm + Lay::kb;
  uint8_t* wt = sm + Lay::wt;
  uint8_t* gop = sm + Lay::gop;
  uint8_t* dop = sm + Lay::dop;
  uint8_t* qt = sm + Lay::qt;
  uint8_t* st = sm + Lay::st;
  uint8_t* pt = sm + Lay::pt;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::misc);
  // one barrier per operand buffer, each completing once per step
  enum { kKb, kWt, kQt, kSt, kPt, kNbuf };
  uint64_t* bar_mma = bars + kNbuf;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNbuf + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + kNbuf + 2);

  const int c = threadIdx.x, warp = c >> 5;
  const int row = c & 127, half = c >> 7;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  const int n_tiles = p.dv / kTile;
  const int tile = blockIdx.x % n_tiles;
  const int h = (blockIdx.x / n_tiles) % p.H;
  const int seq = blockIdx.x / (n_tiles * p.H);
  const int jt = tile * kTile;              // the tile's first column
  const int j0 = jt + 32 * half;            // this thread's first column
  int start, end;
  seq_range(p.cu, seq, p.T, &start, &end);
  const int nch = (end - start + kC - 1) / kC;
  const int cid0 = p.cu ? p.chunk_off[seq] : seq * ((p.T + kC - 1) / kC);
  const bool owns_state = row < DK;
  const size_t sbase = ((size_t)seq * p.H + h) * DK * p.dv;
  // rows of the d_k-row maps
  auto crow = [&](int n) { return (int)(((size_t)(cid0 + n) * p.H + h) * DK); };

  if (c == 0) {
    prefetch_tmap(&m.kb);
    prefetch_tmap(&m.wt);
    prefetch_tmap(&m.qdo);
    prefetch_tmap(&m.s);
    prefetch_tmap(&m.pdo);
    for (int i = 0; i < kNbuf + 1; ++i) mbar_init(bars + i, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Loads of step s (chunk nch - 1 - s), issued by thread 0 only; `issued`
  // counts the loads of each buffer (one outstanding at most).
  int issued[kNbuf] = {0, 0, 0, 0, 0};
  auto load_kb = [&](int s) {
    mbar_arrive_expect_tx(bars + kKb, Lay::kb_tx);
    for (int q = 0; q < DK / 32; ++q)
      tma_load_3d(kb + q * 8192, &m.kb, bars + kKb, 32 * q, h,
                  start + (nch - 1 - s) * kC);
    ++issued[kKb];
  };
  auto load_wt = [&](int s) {
    mbar_arrive_expect_tx(bars + kWt, Lay::wt_tx);
    for (int q = 0; q < 2; ++q)
      tma_load_2d(wt + q * 16384, &m.wt, bars + kWt, 32 * q, crow(nch - 1 - s));
    ++issued[kWt];
  };
  auto load_qt = [&](int s) {
    mbar_arrive_expect_tx(bars + kQt, Lay::qt_tx);
    for (int q = 0; q < 2; ++q)
      tma_load_2d(qt + q * DK * 128, &m.qdo, bars + kQt, jt + 32 * q,
                  crow(nch - 1 - s));
    ++issued[kQt];
  };
  auto load_st = [&](int s) {  // the start state of chunk nch - s (or final)
    mbar_arrive_expect_tx(bars + kSt, Lay::qt_tx);
    for (int q = 0; q < 2; ++q) {
      if (s == 0)
        tma_load_2d(st + q * DK * 128, &m.fin, bars + kSt, jt + 32 * q,
                    (int)(((size_t)seq * p.H + h) * DK));
      else
        tma_load_2d(st + q * DK * 128, &m.s, bars + kSt, jt + 32 * q,
                    crow(nch - s));
    }
    ++issued[kSt];
  };
  auto load_pt = [&](int s) {
    mbar_arrive_expect_tx(bars + kPt, Lay::pt_tx);
    for (int q = 0; q < 2; ++q)
      tma_load_3d(pt + q * 8192, &m.pdo, bars + kPt, jt + 32 * q, h,
                  start + (nch - 1 - s) * kC);
    ++issued[kPt];
  };
  if (c == 0 && nch > 0) {
    load_st(0);
    load_qt(0);
    load_kb(0);
    load_pt(0);
    load_wt(0);
  }

  if (owns_state) {  // dS of the last chunk: the final-state gradient
    float v[32];
    if (p.d_final) {
      const float4* src = reinterpret_cast<const float4*>(
          p.d_final + sbase + (size_t)row * p.dv + j0);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 x = src[i];
        v[4 * i] = x.x; v[4 * i + 1] = x.y; v[4 * i + 2] = x.z;
        v[4 * i + 3] = x.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = 0.f;
    }
    tmem_st32(tmem + lane_base + Lay::t_ds + 32 * half, v);
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // this thread's 128-byte row inside a swizzled operand panel
  auto ld_row = [](const uint8_t* panel, int r, float* v) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float4 x = *reinterpret_cast<const float4*>(
          panel + r * 128 + ((k ^ (r & 7)) << 4));
      v[4 * k] = x.x; v[4 * k + 1] = x.y; v[4 * k + 2] = x.z;
      v[4 * k + 3] = x.w;
    }
  };
  auto st_row = [](uint8_t* panel, int r, const float* v) {
#pragma unroll
    for (int k = 0; k < 8; ++k)
      *reinterpret_cast<float4*>(panel + r * 128 + ((k ^ (r & 7)) << 4)) =
          make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
  };

  float gmv = (owns_state && nch > 0)
                  ? p.gam[((size_t)(cid0 + nch - 1) * p.H + h) * DK + row]
                  : 0.f;
  uint32_t ph_mma = 0;
  bool failed = false;
  int s = 0;
  for (; s < nch; ++s) {
    const int n = nch - 1 - s;
    const int cid = cid0 + n, tok0 = start + n * kC;
    const int L = min(kC, end - tok0);
    const uint32_t par = (uint32_t)s & 1u;
    bool ok = true;

    // ---- G = Diag(gam) dS, gam * d gam; TMEM dS <- G + Qt^T dO
    if (owns_state) {
      ok = wait_or_abort<false>(bars + kSt, par, abort_flag) &&
           wait_or_abort<false>(bars + kQt, par, abort_flag);
      if (ok) {
        float v[32], x[32];
        tmem_ld32(tmem + lane_base + Lay::t_ds + 32 * half, v);
        ld_row(st + half * DK * 128, row, x);
        float part = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) part += x[i] * v[i];
        p.dgam[(((size_t)cid * p.H + h) * (p.dv / 32) + j0 / 32) * DK + row] =
            part;
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= gmv;
        // B operand of product 1: element (k = row, n = column), K-major
        // panels of 32 rows (d_k) each
        uint8_t* panel = gop + (row >> 5) * 8192;
#pragma unroll
        for (int i = 0; i < 32; ++i)
          *reinterpret_cast<float*>(panel + swz32(32 * half + i, row & 31)) =
              v[i];
        uint8_t* qp = qt + half * DK * 128;
        ld_row(qp, row, x);
        st_row(qp, row, v);  // G, stored by TMA below
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] += x[i];
        tmem_st32(tmem + lane_base + Lay::t_ds + 32 * half, v);
        tmem_wait_st();
      } else {
        *abort_flag = 1;
      }
      if (n > 0) gmv = p.gam[((size_t)(cid - 1) * p.H + h) * DK + row];
    }
    fence_proxy_async();
    tc_fence_before();
    if (named_sync_or(kBarAll, kThreads, !ok)) {
      failed = true;
      break;
    }

    // ---- product 1: D = Kb G (rows 0-63 meaningful); G out; next loads
    if (c == 0) {
      tc_fence_after();
      for (int q = 0; q < 2; ++q)
        tma_store_2d(&m.gst, qt + q * DK * 128, jt + 32 * q, crow(n));
      bulk_commit();
      if (s + 1 < nch) load_st(s + 1);
      ok = wait_or_abort<false>(bars + kKb, par, abort_flag);
      if (ok) {
        constexpr uint32_t id = idesc_tf32(128, kTile);
#pragma unroll
        for (int ks = 0; ks < DK / 8; ++ks)
          mma_tf32(tmem + Lay::t_dd,
                   desc_sw128(smem_u32(kb) + (ks >> 2) * 8192 + (ks & 3) * 32,
                              16, 1024),
                   desc_sw128(smem_u32(gop) + (ks >> 2) * 8192 + (ks & 3) * 32,
                              16, 1024),
                   id, ks > 0);
        mma_commit(bar_mma);
        bulk_wait_read();  // G has left the Qt^T dO buffer
        if (s + 1 < nch) load_qt(s + 1);
      } else {
        *abort_flag = 1;
      }
    }
    ok = ok && wait_or_abort<false>(bar_mma, ph_mma, abort_flag);
    ph_mma ^= 1;
    if (named_sync_or(kBarAll, kThreads, !ok)) {
      failed = true;
      break;
    }
    tc_fence_after();
    if (c == 0 && s + 1 < nch) load_kb(s + 1);

    // ---- dDelta = Kb G + P^T dO (token rows 0-63; zero past the chunk)
    if (row < kC) {
      ok = wait_or_abort<false>(bars + kPt, par, abort_flag);
      if (ok) {
        float d[32], x[32];
        const bool in = row < L;
        uint8_t* pp = pt + half * 8192;
        ld_row(pp, row, x);
        tmem_ld32(tmem + lane_base + Lay::t_dd + 32 * half, d);
#pragma unroll
        for (int i = 0; i < 32; ++i) d[i] = in ? d[i] + x[i] : 0.f;
        if (L < kC && in) {  // a ragged chunk: the rows past it belong to
                             // the next sequence, so no box store
          float4* d4 = reinterpret_cast<float4*>(
              p.dd + ((size_t)(tok0 + row) * p.H + h) * p.dv + j0);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            d4[i] =
                make_float4(d[4 * i], d[4 * i + 1], d[4 * i + 2], d[4 * i + 3]);
        }
        st_row(pp, row, d);
        // B operand of product 2, negated: element (k = token, n = column)
        uint8_t* panel = dop + (row >> 5) * 8192;
#pragma unroll
        for (int i = 0; i < 32; ++i)
          *reinterpret_cast<float*>(panel + swz32(32 * half + i, row & 31)) =
              -d[i];
      } else {
        *abort_flag = 1;
      }
    }
    fence_proxy_async();
    tc_fence_before();
    if (named_sync_or(kBarAll, kThreads, !ok)) {
      failed = true;
      break;
    }

    // ---- product 2: dS += W^T (-dDelta); dDelta out; next loads
    if (c == 0) {
      tc_fence_after();
      if (L == kC) {
        for (int q = 0; q < 2; ++q)
          tma_store_3d(&m.dd, pt + q * 8192, jt + 32 * q, h, tok0);
        bulk_commit();
      }
      if (p.store_ddt) {  // the B panels: -dDelta^T, zero past the chunk
        for (int q = 0; q < 2; ++q)
          tma_store_2d(&m.ddt, dop + q * 8192, 32 * q,
                       (int)(((size_t)cid * p.H + h) * p.dv + jt));
        bulk_commit();
      }
      ok = wait_or_abort<false>(bars + kWt, par, abort_flag);
      if (ok) {
        constexpr uint32_t id = idesc_tf32(128, kTile);
#pragma unroll
        for (int ks = 0; ks < kC / 8; ++ks)
          mma_tf32(tmem + Lay::t_ds,
                   desc_sw128(smem_u32(wt) + (ks >> 2) * 16384 + (ks & 3) * 32,
                              16, 1024),
                   desc_sw128(smem_u32(dop) + (ks >> 2) * 8192 + (ks & 3) * 32,
                              16, 1024),
                   id, 1u);
        mma_commit(bar_mma);
        bulk_wait_read();  // dDelta has left the P^T dO buffer
        if (s + 1 < nch) load_pt(s + 1);
      } else {
        *abort_flag = 1;
      }
    }
    ok = ok && wait_or_abort<false>(bar_mma, ph_mma, abort_flag);
    ph_mma ^= 1;
    if (named_sync_or(kBarAll, kThreads, !ok)) {
      failed = true;
      break;
    }
    tc_fence_after();
    if (c == 0 && s + 1 < nch) load_wt(s + 1);
  }
  if (failed) {
    if (c == 0) {
      atomicExch(&g_fused_timeout, 1);
#pragma unroll
      for (int b = 0; b < kNbuf; ++b)  // the copy still in flight, if any
        if (issued[b] > 0)
          mbar_wait(bars + b, (uint32_t)(issued[b] - 1) & 1u, 100000000ull);
    }
  } else if (owns_state && p.d_init) {
    float v[32];
    tmem_ld32(tmem + lane_base + Lay::t_ds + 32 * half, v);
    float4* dst = reinterpret_cast<float4*>(p.d_init + sbase +
                                            (size_t)row * p.dv + j0);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
  if (c == 0) bulk_wait_all();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

// ---------------------------------------------------------------------------
// The forward's state pass for the backward, on the tensor cores: per chunk,
// walking each sequence forward (the chunkwise form "You Could Have Come Up
// with Kimi Delta Attention", daily.dev, Summary):
//   Delta = U - W S           (product A: M = 64 tokens, N = 64, K = d_k)
//   S    <- Diag(gam) S + Kh^T Delta, Kh = k exp(g_C - g)
//                             (product B: M = d_k, N = 64, K = 64 tokens)
// storing every chunk-start state, Delta over U, and the final state.  The
// state's rounding is amplified in dlog_alpha under strong gates (its reverse
// sum of differences of terms that grow like exp|g|), so this pass keeps
// fp32-grade operands: S and Delta, formed here, enter their products as a
// tf32 high part plus the tf32 remainder (product A takes both parts of S
// as one N = 128 operand, product B two MMAs per step), and W and Kh^T
// arrive from prep already rounded to the nearest tf32.  One CTA of 256
// threads per (sequence, head, 64-column d_v tile), S in TMEM throughout;
// W, U and Kh^T by TMA into one buffer each, refilled as soon as it is free;
// Delta stored by TMA in place of U (thread stores for a ragged last chunk),
// each chunk-start state by TMA from a staging tile.

struct StateParams {
  const float* gam;      // exp(g_C) [chunks, H, dk]
  const float* s_init;   // [n_seqs, H, dk, dv] or null (zero)
  float* s_final;        // [n_seqs, H, dk, dv]
  float* dd;             // Delta over U [tokens, H, dv] (ragged chunks' rows)
  const int32_t* cu;
  const int32_t* chunk_off;
  int n_seqs, T, H, dv;
};

// W and U / Delta over [tokens, H, d] (64-token boxes); Kh^T over
// [chunks * H * dk, 64] and the chunk-start states over [chunks * H * dk, dv]
// (d_k-row boxes).
struct StateMaps {
  CUtensorMap w, u, kht, s;
};

template <int DK>
struct StateLayout {
  static constexpr uint32_t wb = 0;                          // W + pad panel
  static constexpr uint32_t ub = wb + (DK / 32 + 1) * 8192;  // U / Delta
  static constexpr uint32_t kb = ub + 2 * 8192;              // Kh^T, 128 rows
  // S as the B operand of product A: per 32-row K panel, 64 N-rows of the
  // tf32 high part then 64 of the remainder (one N = 128 operand)
  static constexpr uint32_t sop = kb + 2 * 16384;
  static constexpr uint32_t dhi = sop + (DK / 32) * 16384;   // Delta, B operand
  static constexpr uint32_t dlo = dhi + 2 * 8192;
  static constexpr uint32_t sst = dlo + 2 * 8192;            // S staging
  static constexpr uint32_t misc = sst + 2 * DK * 128;
  static constexpr uint32_t bytes = misc + 256;
  static constexpr uint32_t w_tx = (DK / 32) * 8192;
  static constexpr uint32_t u_tx = 2 * 8192;
  static constexpr uint32_t k_tx = 2 * DK * 128;
  // TMEM columns: S; W S_hi and W S_lo side by side
  static constexpr uint32_t t_s = 0, t_d = 64;
  static_assert(bytes + 1024 <= 232448, "shared memory");
};

template <int DK>
__global__ void __launch_bounds__(kThreads, 1)
    state_chain_kernel(const __grid_constant__ StateMaps m,
                       const StateParams p) {
  using namespace sm100;
  using Lay = StateLayout<DK>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* wb = sm + Lay::wb;
  uint8_t* ub = sm + Lay::ub;
  uint8_t* kb = sm + Lay::kb;
  uint8_t* sop = sm + Lay::sop;
  uint8_t* dhi = sm + Lay::dhi;
  uint8_t* dlo = sm + Lay::dlo;
  uint8_t* sst = sm + Lay::sst;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::misc);
  enum { kW, kU, kK, kNbuf };
  uint64_t* bar_mma = bars + kNbuf;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNbuf + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + kNbuf + 2);

  const int c = threadIdx.x, warp = c >> 5;
  const int row = c & 127, half = c >> 7;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  const int n_tiles = p.dv / kTile;
  const int tile = blockIdx.x % n_tiles;
  const int h = (blockIdx.x / n_tiles) % p.H;
  const int seq = blockIdx.x / (n_tiles * p.H);
  const int jt = tile * kTile, j0 = jt + 32 * half;
  int start, end;
  seq_range(p.cu, seq, p.T, &start, &end);
  const int nch = (end - start + kC - 1) / kC;
  const int cid0 = p.cu ? p.chunk_off[seq] : seq * ((p.T + kC - 1) / kC);
  const bool owns_state = row < DK;
  const size_t sbase = ((size_t)seq * p.H + h) * DK * p.dv;
  auto crow = [&](int n) { return (int)(((size_t)(cid0 + n) * p.H + h) * DK); };

  if (c == 0) {
    prefetch_tmap(&m.w);
    prefetch_tmap(&m.u);
    prefetch_tmap(&m.kht);
    prefetch_tmap(&m.s);
    for (int i = 0; i < kNbuf + 1; ++i) mbar_init(bars + i, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  int issued[kNbuf] = {0, 0, 0};
  auto load_w = [&](int n) {
    mbar_arrive_expect_tx(bars + kW, Lay::w_tx);
    for (int q = 0; q < DK / 32; ++q)
      tma_load_3d(wb + q * 8192, &m.w, bars + kW, 32 * q, h, start + n * kC);
    ++issued[kW];
  };
  auto load_u = [&](int n) {
    mbar_arrive_expect_tx(bars + kU, Lay::u_tx);
    for (int q = 0; q < 2; ++q)
      tma_load_3d(ub + q * 8192, &m.u, bars + kU, jt + 32 * q, h,
                  start + n * kC);
    ++issued[kU];
  };
  auto load_k = [&](int n) {
    mbar_arrive_expect_tx(bars + kK, Lay::k_tx);
    for (int q = 0; q < 2; ++q)
      tma_load_2d(kb + q * 16384, &m.kht, bars + kK, 32 * q, crow(n));
    ++issued[kK];
  };
  if (c == 0 && nch > 0) {
    load_w(0);
    load_u(0);
    load_k(0);
  }
  auto ld_row = [](const uint8_t* panel, int r, float* v) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float4 x = *reinterpret_cast<const float4*>(
          panel + r * 128 + ((k ^ (r & 7)) << 4));
      v[4 * k] = x.x; v[4 * k + 1] = x.y; v[4 * k + 2] = x.z;
      v[4 * k + 3] = x.w;
    }
  };
  auto st_row = [](uint8_t* panel, int r, const float* v) {
#pragma unroll
    for (int k = 0; k < 8; ++k)
      *reinterpret_cast<float4*>(panel + r * 128 + ((k ^ (r & 7)) << 4)) =
          make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
  };
  // S (this thread's row, 32 columns) into the K-major B panels of product A
  // as tf32 high part and remainder, and into the staging tile
  auto put_state = [&](const float* v, bool stage) {
    uint8_t* ph = sop + (row >> 5) * 16384;
    uint8_t* pl = ph + 8192;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float hi = tf32_rna(v[i]);
      *reinterpret_cast<float*>(ph + swz32(32 * half + i, row & 31)) = hi;
      *reinterpret_cast<float*>(pl + swz32(32 * half + i, row & 31)) =
          v[i] - hi;
    }
    if (stage) st_row(sst + half * DK * 128, row, v);
  };

  // ---- the start state
  if (owns_state) {
    float v[32];
    if (p.s_init) {
      const float4* src = reinterpret_cast<const float4*>(
          p.s_init + sbase + (size_t)row * p.dv + j0);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 x = src[i];
        v[4 * i] = x.x; v[4 * i + 1] = x.y; v[4 * i + 2] = x.z;
        v[4 * i + 3] = x.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = 0.f;
    }
    tmem_st32(tmem + lane_base + Lay::t_s + 32 * half, v);
    put_state(v, nch > 0);
    if (nch == 0) {  // an empty sequence: the final state is the start state
      float4* dst = reinterpret_cast<float4*>(p.s_final + sbase +
                                              (size_t)row * p.dv + j0);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
    tmem_wait_st();
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  if (c == 0 && nch > 0) {
    tc_fence_after();
    for (int q = 0; q < 2; ++q)
      tma_store_2d(&m.s, sst + q * DK * 128, jt + 32 * q, crow(0));
    bulk_commit();
  }

  uint32_t ph_mma = 0;
  bool failed = false;
  int n = 0;
  for (; n < nch; ++n) {
    const int cid = cid0 + n, tok0 = start + n * kC;
    const int L = min(kC, end - tok0);
    const uint32_t par = (uint32_t)n & 1u;
    bool ok = true;

    // ---- product A: D = W S (rows 0-63 meaningful)
    if (c == 0) {
      tc_fence_after();
      ok = wait_or_abort<false>(bars + kW, par, abort_flag);
      if (ok) {
        // one N = 128 MMA per K step: W S_hi in columns 0-63 of the
        // accumulator, W S_lo in 64-127 (an MMA below N = 128 costs about
        // as much as one at N = 128)
        constexpr uint32_t id = idesc_tf32(128, 2 * kTile);
#pragma unroll
        for (int ks = 0; ks < DK / 8; ++ks) {
          const uint64_t ad = desc_sw128(
              smem_u32(wb) + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024);
          mma_tf32(tmem + Lay::t_d, ad,
                   desc_sw128(smem_u32(sop) + (ks >> 2) * 16384 + (ks & 3) * 32,
                              16, 1024),
                   id, ks > 0);
        }
        mma_commit(bar_mma);
      } else {
        *abort_flag = 1;
      }
    }
    const float gmv =
        owns_state ? p.gam[((size_t)cid * p.H + h) * DK + row] : 0.f;
    ok = ok && wait_or_abort<false>(bar_mma, ph_mma, abort_flag);
    ph_mma ^= 1;
    if (named_sync_or(kBarAll, kThreads, !ok)) {
      failed = true;
      break;
    }
    tc_fence_after();
    if (c == 0 && n + 1 < nch) load_w(n + 1);

    // ---- Delta = U - W S (token rows; zero past the chunk); S <- gam S
    if (row < kC) {
      ok = wait_or_abort<false>(bars + kU, par, abort_flag);
      if (ok) {
        float d[32], dl[32], u[32];
        const bool in = row < L;
        uint8_t* up = ub + half * 8192;
        ld_row(up, row, u);
        tmem_ld32(tmem + lane_base + Lay::t_d + 32 * half, d);
        tmem_ld32(tmem + lane_base + Lay::t_d + 64 + 32 * half, dl);
#pragma unroll
        for (int i = 0; i < 32; ++i) d[i] = in ? u[i] - (d[i] + dl[i]) : 0.f;
        if (L < kC && in) {  // a ragged chunk: no box store past it
          float4* d4 = reinterpret_cast<float4*>(
              p.dd + ((size_t)(tok0 + row) * p.H + h) * p.dv + j0);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            d4[i] =
                make_float4(d[4 * i], d[4 * i + 1], d[4 * i + 2], d[4 * i + 3]);
        }
        st_row(up, row, d);
        uint8_t* ph = dhi + (row >> 5) * 8192;
        uint8_t* pl = dlo + (row >> 5) * 8192;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float hi = tf32_rna(d[i]);
          *reinterpret_cast<float*>(ph + swz32(32 * half + i, row & 31)) = hi;
          *reinterpret_cast<float*>(pl + swz32(32 * half + i, row & 31)) =
              d[i] - hi;
        }
      } else {
        *abort_flag = 1;
      }
    }
    if (owns_state) {
      float v[32];
      tmem_ld32(tmem + lane_base + Lay::t_s + 32 * half, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= gmv;
      tmem_st32(tmem + lane_base + Lay::t_s + 32 * half, v);
      tmem_wait_st();
    }
    fence_proxy_async();
    tc_fence_before();
    if (named_sync_or(kBarAll, kThreads, !ok)) {
      failed = true;
      break;
    }

    // ---- product B: S += Kh^T Delta; Delta out; next U
    if (c == 0) {
      tc_fence_after();
      if (L == kC) {
        for (int q = 0; q < 2; ++q)
          tma_store_3d(&m.u, ub + q * 8192, jt + 32 * q, h, tok0);
        bulk_commit();
      }
      ok = wait_or_abort<false>(bars + kK, par, abort_flag);
      if (ok) {
        constexpr uint32_t id = idesc_tf32(128, kTile);
#pragma unroll
        for (int ks = 0; ks < kC / 8; ++ks) {
          const uint64_t ad = desc_sw128(
              smem_u32(kb) + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
          const uint32_t o = (ks >> 2) * 8192 + (ks & 3) * 32;
          mma_tf32(tmem + Lay::t_s, ad, desc_sw128(smem_u32(dhi) + o, 16, 1024),
                   id, 1u);
          mma_tf32(tmem + Lay::t_s, ad, desc_sw128(smem_u32(dlo) + o, 16, 1024),
                   id, 1u);
        }
        mma_commit(bar_mma);
        bulk_wait_read();  // Delta and the last state have left shared memory
        if (n + 1 < nch) load_u(n + 1);
      } else {
        *abort_flag = 1;
      }
    }
    ok = ok && wait_or_abort<false>(bar_mma, ph_mma, abort_flag);
    ph_mma ^= 1;
    if (named_sync_or(kBarAll, kThreads, !ok)) {
      failed = true;
      break;
    }
    tc_fence_after();
    if (c == 0 && n + 1 < nch) load_k(n + 1);

    // ---- the next chunk's start state (or the final state)
    if (owns_state) {
      float v[32];
      tmem_ld32(tmem + lane_base + Lay::t_s + 32 * half, v);
      if (n + 1 < nch) {
        put_state(v, true);
      } else {
        float4* dst = reinterpret_cast<float4*>(p.s_final + sbase +
                                                (size_t)row * p.dv + j0);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          dst[i] =
              make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    if (c == 0 && n + 1 < nch) {
      tc_fence_after();
      for (int q = 0; q < 2; ++q)
        tma_store_2d(&m.s, sst + q * DK * 128, jt + 32 * q, crow(n + 1));
      bulk_commit();
    }
  }
  if (failed && c == 0) {
    atomicExch(&g_fused_timeout, 1);
#pragma unroll
    for (int b = 0; b < kNbuf; ++b)  // the copy still in flight, if any
      if (issued[b] > 0)
        mbar_wait(bars + b, (uint32_t)(issued[b] - 1) & 1u, 100000000ull);
  }
  if (c == 0) bulk_wait_all();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

}  // namespace bwdtc
}  // namespace kda
