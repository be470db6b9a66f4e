// Two-pass chunkwise KDA prefill for sm_100a: the per-chunk factorisation of
// every (chunk, head) as one fully parallel pass, then the serial state chain
// as a second kernel that only runs the state and output products.
//
// Pass 1, factor_kernel: CTAs of 256 threads, two per SM, each taking up to
// four consecutive (chunk, head) items in turn.  Per item it forms the same
// chunk package the paired kernel hands from its producer to its consumers
// (kda_fused_pair_sm100.cuh): [W; Qt] (W over Kt), Kb, P, T' and the package
// vector (exp(g_C - rho), exp(rho), the rho flag), in the same shared-memory
// layout, and writes it to an HBM workspace with bulk copies.  No CTA waits
// for another, so the factorisation of all chunks runs side by side on every
// SM instead of along each sequence.
//
// Pass 2, chain_kernel: one CTA of 256 threads per (sequence, head,
// 64-column d_v tile), two threads per TMEM lane (32 columns each).  Per chunk it bulk-loads the package (two ahead,
// double-buffered) and V, and runs the paired kernel's consumer steps:
// U = T' V and [W; Qt] S (MMA3), Delta = U - W S, S += Kb^T Delta (MMA4) and
// the outputs P Delta + Qt S (MMA5), then S <- exp(g_C - rho) S.  The fp32
// state stays in TMEM across the chunks.
//
// The mathematics and its sources are those of the fused kernels
// (kda_fused_sm100.cu): the recurrence regrouped over chunks ("You Could Have
// Come Up with Kimi Delta Attention", daily.dev, Summary; the
// Diagonal-Plus-Low-Rank chunkwise form, "Kimi Delta Attention",
// akshathtiwari.co.in).
#pragma once

namespace kda {
namespace twopass {

using namespace sm100;
using pair::PairLayout;
using ws::invert_unit_lower_tc;
using ws::kC;
using ws::kDvt;
using ws::kFS;
using ws::kGcFloats;
using ws::ldg_f1_if;
using ws::ldg_f4_if;
using ws::mbar_arrive;
using ws::named_sync;
using ws::named_sync_or;
using ws::prologue_rows;
using ws::rescale_qt;
using ws::st_chunks;
using ws::tmem_st32;
using ws::tmem_wait_st;
using ws::wait_or_abort;

constexpr int kFactorThreads = 256;
constexpr int kChainThreads = 256;
constexpr int kBarAll = 3;  // named barrier id of a whole CTA

__device__ __forceinline__ void bulk_store(void* gdst, const void* src,
                                           uint32_t bytes) {
  asm volatile(
      "cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
      "r"(smem_u32(src)), "r"(bytes)
      : "memory");
}
__device__ __forceinline__ void bulk_load(void* dst, const void* gsrc,
                                          uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], "
      "[%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// Until the bulk stores committed so far have read their shared-memory
// source (the global writes complete on their own before the grid ends).
__device__ __forceinline__ void bulk_commit_wait_read() {
  asm volatile(
      "cp.async.bulk.commit_group;\n\t"
      "cp.async.bulk.wait_group.read 0;" ::
          : "memory");
}
__device__ __forceinline__ void bulk_commit_wait_all() {
  asm volatile(
      "cp.async.bulk.commit_group;\n\t"
      "cp.async.bulk.wait_group 0;" ::
          : "memory");
}

struct TwoPassParams {
  Prologue pro;
  const float* beta;
  const float* log_alpha;
  const float* s_init;
  float* s_final;
  __nv_bfloat16* out;
  const int32_t* cu;
  const int32_t* chunk_off;  // packed layout: chunks before each sequence
  const int32_t* order;      // packed layout: longest sequence first
  uint8_t* packages;         // [max_chunks][H] packages of Lay::slot bytes
  int n_seqs, T, H, dv;
  int n_items;        // (chunk, head) factorisations: max_chunks * H
  int items_per_cta;  // consecutive items one factorisation CTA takes
};

template <int DK>
struct FactorLayout {
  using P = PairLayout<DK>;
  static constexpr uint32_t slot = 0;  // the package, P::slot bytes
  static constexpr uint32_t afp = P::slot;
  static constexpr uint32_t tfp = afp + 64 * kFS * 4;
  static constexpr uint32_t msc = tfp + 64 * kFS * 4;  // 512 floats
  static constexpr uint32_t misc = msc + 2048;          // betas, barriers
  static constexpr uint32_t bytes = misc + 512;
  static_assert(bytes + 1024 <= 116 * 1024, "two CTAs per SM");
};

// ------------------------------------------------------------ pass 1
template <int DK, int GATE>
__global__ void __launch_bounds__(kFactorThreads, 2)
    factor_kernel(const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_k,
                  const TwoPassParams p) {
  using Lay = FactorLayout<DK>;
  using PL = PairLayout<DK>;
  constexpr int NCG = DK / 4;
  constexpr int NRB = kFactorThreads / NCG;
  constexpr int RPT = kC / NRB;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* slot = sm + Lay::slot;
  uint8_t* kq = slot + PL::s_kq;
  uint8_t* kb = slot + PL::s_kb;
  uint8_t* pp = slot + PL::s_pp;
  uint8_t* tp = slot + PL::s_tp;
  float* gc = reinterpret_cast<float*>(slot + PL::s_gc);
  float* afp = reinterpret_cast<float*>(sm + Lay::afp);
  float* tfp = reinterpret_cast<float*>(sm + Lay::tfp);
  float* msc = reinterpret_cast<float*>(sm + Lay::msc);
  float* betas = reinterpret_cast<float*>(sm + Lay::misc);  // [64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::misc + 256);
  uint64_t* bar_in = bars + 0;
  uint64_t* bar_m1 = bars + 1;
  uint64_t* bar_m2 = bars + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 4);
  uint64_t* bar_fin = bars + 5;  // failure path: MMAs in flight drained

  const int t = threadIdx.x, warp = t >> 5;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  const int colh = warp >> 2, row_t = t & 127;
  const int cg = t % NCG, rb = t / NCG;
  const int pnl = cg >> 4;

  if (t == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    mbar_init(bar_in, 1);
    mbar_init(bar_m1, 1);
    mbar_init(bar_m2, 1);
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  for (int i = t; i < 64 * kFS; i += kFactorThreads) tfp[i] = 0.f;
  if (DK == 64) {  // the second M-panel of Kb stays zero
    uint4* z = reinterpret_cast<uint4*>(kb + 8192);
    for (int i = t; i < 512; i += kFactorThreads) z[i] = make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // The CTA takes items_per_cta consecutive items (chunk, head), heads
  // fastest, so that neighbouring CTAs read adjacent columns of the same
  // token rows; its set-up is paid once for all of them.  Each barrier
  // completes once per item, so its parity alternates with the items done.
  uint32_t ph = 0;
  const int item0 = (int)blockIdx.x * p.items_per_cta;
  const int item_end = min(item0 + p.items_per_cta, p.n_items);
  for (int item = item0; item < item_end; ++item) {
    const int h = item % p.H;
    const int cid = item / p.H;
    uint8_t* gpk = p.packages + ((size_t)cid * p.H + h) * PL::slot;
    int seq = 0, tok0 = 0, L = 0;
    if (!locate_chunk(cid, p.cu, p.chunk_off, p.n_seqs, p.T, kC, &seq, &tok0,
                      &L))
      continue;
    if (t == 0) {  // raw q and k: k over the Kt rows, q over the Qt rows
      mbar_arrive_expect_tx(bar_in, PL::tx_qk);
#pragma unroll
      for (int q = 0; q < (int)PL::NP; ++q) {
        tma_load_3d(kq + q * 16384 + 8192, &tm_q, bar_in, q * 64, h, tok0);
        tma_load_3d(kq + q * 16384, &tm_k, bar_in, q * 64, h, tok0);
      }
    }
    float4 la_reg[RPT];
    {
      const float* la_g = GATE == kGateChannel
                              ? p.log_alpha + (size_t)h * DK + 4 * cg
                              : p.log_alpha + h;
      const size_t la_stride =
          GATE == kGateChannel ? (size_t)p.H * DK : (size_t)p.H;
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
        const int rr = rb * RPT + i;
        la_reg[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (GATE == kGateChannel)
          ldg_f4_if(la_reg[i], la_g + (size_t)(tok0 + rr) * la_stride, rr < L);
        else if (GATE == kGateHead)
          ldg_f1_if(la_reg[i].x, la_g + (size_t)(tok0 + rr) * la_stride,
                    rr < L);
      }
    }
    if (t < kC) {
      float b = 0.f;
      ldg_f1_if(b, p.beta + (size_t)(tok0 + t) * p.H + h, t < L);
      betas[t] = b;
    }
    bool ok = wait_or_abort<true>(bar_in, ph, abort_flag);
    bool failed = named_sync_or(kBarAll, kFactorThreads, !ok);
    if (!failed) {
      // ---- prologue, in place over the raw q and k
      prologue_rows<DK, GATE>(la_reg, afp, gc, kq + pnl * 16384 + 8192,
                              kq + pnl * 16384, kq + pnl * 16384,
                              kb + pnl * 8192, L, p.pro, t);
      fence_proxy_async();
      named_sync(kBarAll, kFactorThreads);
      if (t == 0) {  // MMA1: [Kt; Qt] . Kb^T
        tc_fence_after();
        const uint32_t idesc = idesc_bf16(128, 64, false, false);
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
          const uint32_t off = (ks & 3) * 32;
          mma_bf16(tmem,
                   desc_sw128(smem_u32(kq) + (ks >> 2) * 16384 + off, 16, 1024),
                   desc_sw128(smem_u32(kb) + (ks >> 2) * 8192 + off, 16, 1024),
                   idesc, ks > 0);
        }
        mma_commit(bar_m1);
      }
      ok = wait_or_abort<false>(bar_m1, ph, abort_flag);
      failed = named_sync_or(kBarAll, kFactorThreads, !ok);
    }
    if (!failed) {
      tc_fence_after();
      {  // A (fp32) and P (bf16 into the package)
        float v[32];
        tmem_ld32(tmem + lane_base + 32 * colh, v);
        if (row_t < 64) {
          const float b = betas[row_t];
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
          const int rr = row_t - 64;
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 32 * colh + i <= rr ? v[i] : 0.f;
          st_chunks<4>(pp, rr, 4 * colh, v);
        }
      }
      // MMA1 has read Qt: back to the chunk-start q e^g where rho != 0
      if (gc[2 * DK] != 0.f) rescale_qt<PL::NP>(kq, gc + DK, t);
      tc_fence_before();
      fence_proxy_async();
      named_sync(kBarAll, kFactorThreads);
      if (t == 0) {  // Qt, Kb, P and the package vector are final: store them
        // now, under the inverse (W and T' follow at the end)
#pragma unroll
        for (int q = 0; q < (int)PL::NP; ++q)
          bulk_store(gpk + q * 16384 + 8192, kq + q * 16384 + 8192, 8192);
        bulk_store(gpk + PL::s_kb, kb, 16384);  // (d_k = 64: its zero panel too)
        bulk_store(gpk + PL::s_pp, pp, 8192);
        bulk_store(gpk + PL::s_gc, gc, PL::gc_bytes);
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      }

      invert_unit_lower_tc(afp, tfp, msc, t);

      {  // T' = Tm Diag(beta), rows masked to the lower triangle
        const int rr = t & 63, qc = t >> 6;
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
          const int c = 16 * qc + i;
          const float4 x = *reinterpret_cast<const float4*>(tfp + rr * kFS + c);
          const float4 b = *reinterpret_cast<const float4*>(betas + c);
          v[i] = c + 0 <= rr ? x.x * b.x : 0.f;
          v[i + 1] = c + 1 <= rr ? x.y * b.y : 0.f;
          v[i + 2] = c + 2 <= rr ? x.z * b.z : 0.f;
          v[i + 3] = c + 3 <= rr ? x.w * b.w : 0.f;
        }
        st_chunks<2>(tp, rr, 2 * qc, v);
      }
      fence_proxy_async();
      named_sync(kBarAll, kFactorThreads);
      if (t == 0) {  // MMA2: W = T' Kt (N = DK)
        tc_fence_after();
        const uint32_t iw = idesc_bf16(128, DK, false, true);
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks)
          mma_bf16(tmem + 64, desc_sw128(smem_u32(tp) + ks * 32, 16, 1024),
                   desc_sw128(smem_u32(kq) + ks * 2048, 16384, 1024), iw,
                   ks > 0);
        mma_commit(bar_m2);
      }
      ok = wait_or_abort<false>(bar_m2, ph, abort_flag);
      failed = named_sync_or(kBarAll, kFactorThreads, !ok);
    }
    if (!failed) {
      tc_fence_after();
      if (row_t < 64) {  // W rows (bf16) over the Kt rows:
        // T' (k e^(g-rho)) scaled by exp(rho) per column = T' (k e^g)
#pragma unroll
        for (int jj = 0; jj < DK / 64; ++jj) {
          const int hh = colh * (DK / 64) + jj;
          float v[32];
          tmem_ld32(tmem + lane_base + 64 + 32 * hh, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= gc[DK + 32 * hh + i];
          st_chunks<4>(kq + (hh >> 1) * 16384, row_t, 4 * (hh & 1), v);
        }
      }
      tc_fence_before();
      fence_proxy_async();
      named_sync(kBarAll, kFactorThreads);
      if (t == 0) {  // W and T' to HBM; the next item's loads (or the
        // exit) wait until every store has read shared memory
#pragma unroll
        for (int q = 0; q < (int)PL::NP; ++q)
          bulk_store(gpk + q * 16384, kq + q * 16384, 8192);
        bulk_store(gpk + PL::s_tp, tp, 8192);
        bulk_commit_wait_read();
      }
      ph ^= 1;
    } else {
      if (t == 0) {
        atomicExch(&g_fused_timeout, 1);
        mbar_wait(bar_in, ph, 100000000ull);  // the q/k load, if in flight
        mma_commit(bar_fin);                  // and the MMAs
        mbar_wait(bar_fin, 0, 100000000ull);
        bulk_commit_wait_all();  // the early package stores read shared memory
      }
      break;  // failed is the same in every thread
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

// ------------------------------------------------------------ pass 2
template <int DK>
struct ChainLayout {
  using P = PairLayout<DK>;
  static constexpr uint32_t slots = 0;               // two packages
  static constexpr uint32_t sop = 2 * P::slot;       // S, DK rows
  static constexpr uint32_t dop = sop + DK * 128;    // Delta, 64 rows
  static constexpr uint32_t vbuf = dop + 8192;       // two V tiles
  static constexpr uint32_t misc = vbuf + 16384;     // barriers
  static constexpr uint32_t bytes = misc + 512;
  // TMEM columns
  static constexpr uint32_t t_u = 0;
  static constexpr uint32_t t_d3 = 64;
  static constexpr uint32_t t_d3b = 128;
  static constexpr uint32_t t_s = 192;
  static_assert(sop % 1024 == 0 && dop % 1024 == 0 && vbuf % 1024 == 0,
                "swizzle atoms");
  static_assert(bytes + 1024 <= 232448, "shared memory");
};

template <int DK>
__global__ void __launch_bounds__(kChainThreads, 1)
    chain_kernel(const __grid_constant__ CUtensorMap tm_v,
                 const TwoPassParams p) {
  using Lay = ChainLayout<DK>;
  using PL = PairLayout<DK>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sop = sm + Lay::sop;
  uint8_t* dop = sm + Lay::dop;
  uint8_t* vbuf = sm + Lay::vbuf;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::misc);
  uint64_t* pk_full = bars + 0;  // [2] a package landed in slot s
  uint64_t* bar_v = bars + 2;    // [2]
  uint64_t* bar_cm = bars + 4;
  uint64_t* bar_sop = bars + 5;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 6);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 7);

  // eight warps: thread c owns TMEM lane (row) c % 128 and the 32 columns
  // 32 (c / 128) .. + 31 of the 64-column tile
  const int c = threadIdx.x, warp = c >> 5;
  const int row = c & 127, half = c >> 7;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  const int n_tiles = p.dv / kDvt;
  const int tile = blockIdx.x % n_tiles;
  const int h = (blockIdx.x / n_tiles) % p.H;
  const int rank = blockIdx.x / (n_tiles * p.H);
  const int seq = p.order ? p.order[rank] : rank;
  const int j0 = tile * kDvt;
  int start, end;
  seq_range(p.cu, seq, p.T, &start, &end);
  const int nch = (end - start + kC - 1) / kC;
  const int cid0 = p.cu ? p.chunk_off[seq] : seq * ((p.T + kC - 1) / kC);
  auto slot_of = [&](int s) { return sm + Lay::slots + s * PL::slot; };
  const bool owns_state = row < DK;

  if (c == 0) {
    prefetch_tmap(&tm_v);
    for (int s = 0; s < 2; ++s) {
      mbar_init(pk_full + s, 1);
      mbar_init(bar_v + s, 1);
    }
    mbar_init(bar_cm, 1);
    mbar_init(bar_sop, kChainThreads / 32);
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

  auto issue_pk = [&](int n) {  // the package of chunk n into slot n & 1
    uint64_t* b = pk_full + (n & 1);
    mbar_arrive_expect_tx(b, PL::copy_bytes);
    bulk_load(slot_of(n & 1),
              p.packages + ((size_t)(cid0 + n) * p.H + h) * PL::slot,
              PL::copy_bytes, b);
  };
  auto issue_v = [&](int n) {
    uint64_t* b = bar_v + (n & 1);
    mbar_arrive_expect_tx(b, 8192);
    tma_load_3d(vbuf + (n & 1) * 8192, &tm_v, b, j0, h, start + n * kC);
  };
  int pk_issued = 0, v_issued = 0;
  if (c == 0) {
    for (int n = 0; n < 2 && n < nch; ++n) issue_pk(n);
    if (nch > 0) issue_v(0);
  }
  pk_issued = nch < 2 ? nch : 2;
  v_issued = nch > 0 ? 1 : 0;

  const size_t sbase = (((size_t)seq * p.H + h) * DK) * p.dv + j0;
  if (owns_state) {  // initial state into TMEM (fp32) and the bf16 operand
    float v[32];
    if (p.s_init) {
      const float4* src = reinterpret_cast<const float4*>(
          p.s_init + sbase + (size_t)row * p.dv + 32 * half);
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
    st_chunks<4>(sop, row, 4 * half, v);
    tmem_wait_st();
  }
  tc_fence_before();
  fence_proxy_async();
  __syncthreads();

  uint32_t ph_cm = 0;
  bool failed = false;
  int n = 0;
  for (; n < nch; ++n) {
    const int s = n & 1;
    const int tok0 = start + n * kC;
    const int L = min(kC, end - tok0);
    uint8_t* slot = slot_of(s);
    uint8_t* kq = slot + PL::s_kq;
    uint8_t* kb = slot + PL::s_kb;
    uint8_t* pp = slot + PL::s_pp;
    uint8_t* tp = slot + PL::s_tp;
    const float* gc = reinterpret_cast<const float*>(slot + PL::s_gc);
    uint8_t* vb = vbuf + (n & 1) * 8192;
    const uint32_t d3 = (n & 1) ? Lay::t_d3b : Lay::t_d3;
    if (n + 1 < nch) {  // V of the next chunk (its buffer was freed by n - 1)
      if (c == 0) issue_v(n + 1);
      v_issued = n + 2;
    }
    bool ok = true;
    if (c == 0) {  // ---- U = T' V ; [W; Qt] . S
      ok = wait_or_abort<true>(pk_full + s, (uint32_t)(n >> 1) & 1u,
                               abort_flag);
      ok = ok && wait_or_abort<false>(bar_v + (n & 1), (uint32_t)(n >> 1) & 1u,
                                      abort_flag);
      if (n > 0)
        ok = ok && wait_or_abort<false>(bar_sop, (uint32_t)(n - 1) & 1u,
                                        abort_flag);
      if (ok) {
        tc_fence_after();
        fence_proxy_async();
        const uint32_t idesc = idesc_bf16(128, 64, false, true);
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks)
          mma_bf16(tmem + Lay::t_u, desc_sw128(smem_u32(tp) + ks * 32, 16, 1024),
                   desc_sw128(smem_u32(vb) + ks * 2048, 8192, 1024), idesc,
                   ks > 0);
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks)
          mma_bf16(tmem + d3,
                   desc_sw128(smem_u32(kq) + (ks >> 2) * 16384 + (ks & 3) * 32,
                              16, 1024),
                   desc_sw128(smem_u32(sop) + ks * 2048, 8192, 1024), idesc,
                   ks > 0);
        mma_commit(bar_cm);
      } else {
        *abort_flag = 1;  // the other threads leave their wait below
      }
    }
    ok = ok && wait_or_abort<false>(bar_cm, ph_cm, abort_flag);
    ph_cm ^= 1;
    if (named_sync_or(kBarAll, kChainThreads, !ok)) {
      failed = true;
      break;
    }
    tc_fence_after();

    // ---- Delta = U - W S (rows 0-63)
    if (row < 64) {
      float uu[32], wsv[32];
      tmem_ld32(tmem + lane_base + Lay::t_u + 32 * half, uu);
      tmem_ld32(tmem + lane_base + d3 + 32 * half, wsv);
#pragma unroll
      for (int i = 0; i < 32; ++i) uu[i] -= wsv[i];
      st_chunks<4>(dop, row, 4 * half, uu);
    }
    const float gamma = owns_state ? gc[row] : 1.f;
    if (owns_state && gc[2 * DK] != 0.f) {
      // S_C = e^(g_C - rho) (e^rho S_0 + Kb^T Delta): pre-scale the state
      const float er = gc[DK + row];
      float v[32];
      tmem_ld32(tmem + lane_base + Lay::t_s + 32 * half, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= er;
      tmem_st32(tmem + lane_base + Lay::t_s + 32 * half, v);
      tmem_wait_st();
    }
    tc_fence_before();
    fence_proxy_async();
    named_sync(kBarAll, kChainThreads);

    // ---- MMA4: S += Kb^T Delta ; MMA5: rows 64-127 += P Delta
    if (c == 0) {
      tc_fence_after();
      const uint32_t i4 = idesc_bf16(128, 64, true, true);
      const uint32_t i5 = idesc_bf16(128, 64, false, true);
#pragma unroll
      for (int ks = 0; ks < kC / 16; ++ks) {
        const uint64_t bd = desc_sw128(smem_u32(dop) + ks * 2048, 8192, 1024);
        mma_bf16(tmem + Lay::t_s,
                 desc_sw128(smem_u32(kb) + ks * 2048, 8192, 1024), bd, i4, 1u);
        mma_bf16(tmem + d3, desc_sw128(smem_u32(pp) - 8192 + ks * 32, 16, 1024),
                 bd, i5, 1u);
      }
      mma_commit(bar_cm);
    }
    ok = wait_or_abort<false>(bar_cm, ph_cm, abort_flag);
    ph_cm ^= 1;
    if (named_sync_or(kBarAll, kChainThreads, !ok)) {
      failed = true;
      break;
    }
    tc_fence_after();
    if (c == 0 && n + 2 < nch) {  // slot s is used up: the package after next
      issue_pk(n + 2);
      pk_issued = n + 3;
    } else if (n + 2 < nch) {
      pk_issued = n + 3;
    }

    // ---- S <- exp(g_C - rho) S: the bf16 operand of the next MMA3 first,
    // then TMEM (the store completes before the next MMA4 is issued)
    if (owns_state) {
      float v[32];
      tmem_ld32(tmem + lane_base + Lay::t_s + 32 * half, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= gamma;
      st_chunks<4>(sop, row, 4 * half, v);
      tmem_st32(tmem + lane_base + Lay::t_s + 32 * half, v);
    }
    fence_proxy_async();
    tc_fence_before();
    __syncwarp();
    if ((c & 31) == 0) mbar_arrive(bar_sop);

    // ---- outputs (rows 64-127 of this chunk's buffer), overlapping the next
    // chunk's MMA3
    if (row >= 64) {
      const int rr = row - 64;
      float o[32];
      tmem_ld32(tmem + lane_base + d3 + 32 * half, o);
      if (rr < L) {
        uint4* dst = reinterpret_cast<uint4*>(
            p.out + ((size_t)(tok0 + rr) * p.H + h) * p.dv + j0 + 32 * half);
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
    if (owns_state) tmem_wait_st();
    tc_fence_before();
  }
  if (failed) {
    if (c == 0) {
      atomicExch(&g_fused_timeout, 1);
      // loads still in flight: packages n .. pk_issued - 1, V n .. v_issued - 1
      for (int m = n; m < pk_issued; ++m)
        mbar_wait(pk_full + (m & 1), (uint32_t)(m >> 1) & 1u, 100000000ull);
      for (int m = n; m < v_issued; ++m)
        mbar_wait(bar_v + (m & 1), (uint32_t)(m >> 1) & 1u, 100000000ull);
    }
  } else if (owns_state) {
    tc_fence_after();
    float v[32];
    tmem_ld32(tmem + lane_base + Lay::t_s + 32 * half, v);
    float4* dst = reinterpret_cast<float4*>(p.s_final + sbase +
                                            (size_t)row * p.dv + 32 * half);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

// Packed layout: exclusive prefix sum of the per-sequence chunk counts.
__global__ void chunk_offsets_kernel(const int32_t* __restrict__ cu, int n_seqs,
                                     int T, int32_t* __restrict__ chunk_off) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int acc = 0;
  chunk_off[0] = 0;
  for (int s = 0; s < n_seqs; ++s) {
    int a, b;
    seq_range(cu, s, T, &a, &b);
    acc += (b - a + kC - 1) / kC;
    chunk_off[s + 1] = acc;
  }
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace: the longest-first order and the chunk offsets (packed layout),
// then one package per (chunk, head) unless the chain reads packages kept
// elsewhere (chain_only).
inline size_t package_slot(int dk) {
  return dk == 128 ? PairLayout<128>::slot : PairLayout<64>::slot;
}
inline size_t index_bytes(const ChunkArgs& a) {
  return a.cu_seqlens
             ? align256((size_t)a.n_seqs * 4) + align256(((size_t)a.n_seqs + 1) * 4)
             : 0;
}
inline size_t workspace_bytes(const ChunkArgs& a, bool chain_only = false) {
  return index_bytes(a) +
         (chain_only ? 0 : (size_t)max_chunks(a) * a.H * package_slot(a.dk));
}
inline uint8_t* packages_in(const ChunkArgs& a, void* workspace) {
  return static_cast<uint8_t*>(workspace) + index_bytes(a);
}

// One call: the packed layout's order and chunk offsets, then (unless
// `packages` is given) the factorisation pass into the workspace, an event
// (factor_done, if given) and the chain kernel.  With `packages` given only
// the chain runs, reading the packages there: chunk c of this call's layout,
// head h, at packages + (c * H + h) * slot.
template <int DK, int GATE>
cudaError_t run(const ChunkArgs& a, void* workspace, cudaStream_t stream,
                const uint8_t* packages, cudaEvent_t factor_done) {
  const int tokens = a.cu_seqlens ? a.T : a.n_seqs * a.T;
  CUtensorMap tq, tk, tv;
  if (!make_tile_map(&tv, a.v, a.dv, a.H, tokens)) return cudaErrorInvalidValue;
  if (!packages && (!make_tile_map(&tq, a.q, DK, a.H, tokens) ||
                    !make_tile_map(&tk, a.k, DK, a.H, tokens)))
    return cudaErrorInvalidValue;
  TwoPassParams p{};
  p.pro = a.pro;
  p.beta = a.beta;
  p.log_alpha = a.log_alpha;
  p.s_init = a.initial_state;
  p.s_final = a.final_state;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.cu = a.cu_seqlens;
  p.n_seqs = a.n_seqs;
  p.T = a.T;
  p.H = a.H;
  p.dv = a.dv;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaError_t e;
  if (a.cu_seqlens) {
    int32_t* order = reinterpret_cast<int32_t*>(ws);
    int32_t* coff =
        reinterpret_cast<int32_t*>(ws + align256((size_t)a.n_seqs * 4));
    order_kernel<<<1, 1024, 0, stream>>>(a.cu_seqlens, a.n_seqs, a.T, order);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    chunk_offsets_kernel<<<1, 32, 0, stream>>>(a.cu_seqlens, a.n_seqs, a.T,
                                               coff);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    p.order = order;
    p.chunk_off = coff;
  }
  if (packages) {
    p.packages = const_cast<uint8_t*>(packages);
  } else {
    p.packages = packages_in(a, workspace);
    const int64_t nchunks = max_chunks(a);
    const size_t smem1 = FactorLayout<DK>::bytes + 1024;
    if ((e = cudaFuncSetAttribute(factor_kernel<DK, GATE>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem1)) != cudaSuccess)
      return e;
    p.n_items = (int)(nchunks * a.H);
    {  // items per CTA: 4, 2 or 1, whichever still leaves two resident waves
      int dev = 0, sms = 0, per_sm = 0;
      if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
          (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount,
                                      dev)) != cudaSuccess ||
          (e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
               &per_sm, factor_kernel<DK, GATE>, kFactorThreads, smem1)) !=
              cudaSuccess)
        return e;
      const int64_t wave = (int64_t)sms * (per_sm > 0 ? per_sm : 1);
      p.items_per_cta =
          p.n_items >= 8 * wave ? 4 : p.n_items >= 4 * wave ? 2 : 1;
    }
    const unsigned grid1 =
        (unsigned)((p.n_items + p.items_per_cta - 1) / p.items_per_cta);
    factor_kernel<DK, GATE><<<grid1, kFactorThreads, smem1, stream>>>(tq, tk,
                                                                      p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (cudaEvent_t ev = pass_event())
      if ((e = cudaEventRecord(ev, stream)) != cudaSuccess) return e;
    if (factor_done)
      if ((e = cudaEventRecord(factor_done, stream)) != cudaSuccess) return e;
  }
  const size_t smem2 = ChainLayout<DK>::bytes + 1024;
  if ((e = cudaFuncSetAttribute(chain_kernel<DK>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem2)) != cudaSuccess)
    return e;
  const unsigned grid2 = (unsigned)a.n_seqs * a.H * (a.dv / kDvt);
  chain_kernel<DK><<<grid2, kChainThreads, smem2, stream>>>(tv, p);
  return cudaGetLastError();
}

inline cudaError_t launch(const ChunkArgs& a, void* workspace,
                          cudaStream_t stream, const uint8_t* packages = nullptr,
                          cudaEvent_t factor_done = nullptr) {
  if (a.gate == kGateHead)
    return a.dk == 128
               ? run<128, kGateHead>(a, workspace, stream, packages, factor_done)
               : run<64, kGateHead>(a, workspace, stream, packages, factor_done);
  if (a.gate == kGateNone)
    return a.dk == 128
               ? run<128, kGateNone>(a, workspace, stream, packages, factor_done)
               : run<64, kGateNone>(a, workspace, stream, packages, factor_done);
  return a.dk == 128
             ? run<128, kGateChannel>(a, workspace, stream, packages, factor_done)
             : run<64, kGateChannel>(a, workspace, stream, packages, factor_done);
}

}  // namespace twopass
}  // namespace kda
