// Paired fused chunkwise KDA prefill for sm_100a: the two CTAs of a cluster
// split the per-chunk factorisation of one (sequence, head) between them.
//
// The mathematics is the warp-specialised kernel's (kda_fused_ws_sm100.cuh):
// per chunk the producer forms the decay-scaled operands, A and P (MMA1), the
// inverse T' = (I + A)^-1 Diag(beta) and W = T' Kt (MMA2); the consumer runs
// the serial state chain for its 64-column d_v tile.  In that kernel the two
// CTAs of the d_v = 128 tiles of a head each factorise every chunk, and the
// factorisation sets the pace.  Here CTA r of the pair factorises only the
// chunks n = r, r + 2, r + 4, ... and hands the result to both consumers: to
// its own through shared memory, to its peer by one bulk shared-to-shared
// copy over the cluster (distributed shared memory).  Each CTA then carries
// half of the factorisation work and all of its own tile's chain.
//
// A chunk's package in a slot is [W; Qt] (W over Kt once MMA2 is done), Kb,
// P, T' and exp(g_C).  The consumer forms U = T' V for its own tile itself
// (one more small MMA), so the package does not depend on the tile.  Each CTA
// has two slots; in CTA r chunk n sits in slot ((n + r) >> 1) & 1, so every
// slot alternates one own chunk with the peer chunk that follows it in the
// consumer's order.  The raw q and k of an own chunk are loaded by TMA
// straight into its slot and transformed in place, and that load is issued
// by the consumer as soon as it has used the peer chunk before it in the same
// slot.  The package crosses to the peer as bulk shared-to-shared copies
// (distributed shared memory runs at about 35 GB/s between the two SMs of a
// pair, so 64.5 KB take about 2 us): Qt, Kb, P and exp(g_C) as soon as the
// peer's slot is free, T' after the inverse, W at the hand-over.
//
// Barriers per CTA: bar_in[s] (q, k of an own chunk landed in slot s),
// full[s] (an own chunk is ready in slot s: local arrive), pfull[s] (a peer
// chunk has fully arrived in slot s: the peer's expect-tx arrive plus the
// copies' byte counts), send_ok[s] (this CTA's consumer is done with its own
// chunk in slot s, so the peer may send the next chunk there).  The peer's
// slot is free for a send once the peer's consumer has released its own
// chunk there (send_ok, signalled remotely) and the peer's copy of that chunk
// to this CTA has been read out, which its complete arrival here (pfull)
// proves.  Every wait is bounded; a failed CTA also raises its peer's abort
// flag, and both CTAs meet at a final cluster barrier only after all their
// outgoing copies have completed.
#pragma once

namespace kda {
namespace pair {

using namespace sm100;
using ws::invert_unit_lower_tc;
using ws::kGcFloats;
using ws::rescale_qt;
using ws::kBarCons;
using ws::kBarProd;
using ws::kC;
using ws::kCons;
using ws::kDvt;
using ws::kFS;
using ws::kProd;
using ws::kThreads;
using ws::ldg_f1_if;
using ws::ldg_f4_if;
using ws::mbar_arrive;
using ws::named_sync;
using ws::named_sync_or;
using ws::prologue_rows;
using ws::st_chunks;
using ws::tmem_st32;
using ws::tmem_wait_st;
using ws::wait_or_abort;
using ws::WsParams;

// ------------------------------------------------------------ cluster PTX
__device__ __forceinline__ uint32_t cta_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// The address of the same shared-memory location in CTA `rank` of the
// cluster.
__device__ __forceinline__ uint32_t peer_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
               : "=r"(r)
               : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void remote_arrive(uint32_t bar) {
  asm volatile(
      "mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar)
      : "memory");
}
__device__ __forceinline__ void remote_arrive_tx(uint32_t bar, uint32_t bytes) {
  asm volatile(
      "mbarrier.arrive.expect_tx.release.cluster.shared::cluster.b64 _, [%0], "
      "%1;" ::"r"(bar),
      "r"(bytes)
      : "memory");
}
// Bulk copy of `bytes` from this CTA's shared memory to a peer's, completing
// on the peer's mbarrier `bar` (both cluster addresses).
__device__ __forceinline__ void copy_to_peer(uint32_t dst, const void* src,
                                             uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes "
      "[%0], [%1], %2, [%3];" ::"r"(dst),
      "r"(smem_u32(src)), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// Non-blocking test of a phase (cluster-scope acquire).
__device__ __forceinline__ bool test_wait_cluster(uint64_t* bar,
                                                  uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Pull one TMA box into L2 ahead of its load.
__device__ __forceinline__ void prefetch_box_l2(const void* tmap, int c0, int c1,
                                                int c2) {
  asm volatile(
      "cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
          reinterpret_cast<uint64_t>(tmap)),
      "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::
          : "memory");
}
__device__ __forceinline__ void remote_store(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v)
               : "memory");
}
// Bounded wait with cluster-scope acquire (the phase may be completed by the
// peer CTA), sleeping in the barrier unit; abandoned on the abort flag.
__device__ __forceinline__ bool try_wait_cluster(uint64_t* bar,
                                                 uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, "
      "%3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(500000u)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool wait_cluster(uint64_t* bar, uint32_t parity,
                                             volatile int* abort_flag) {
  if (try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (try_wait_cluster(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > 2000000000ull) return false;
  }
}

template <int DK>
struct PairLayout {
  static constexpr uint32_t NP = DK / 64;
  // one slot (the copied package), offsets inside it
  static constexpr uint32_t s_kq = 0;               // [Kt/W; Qt], NP panels
  static constexpr uint32_t s_kb = NP * 16384;      // Kb, two 8 KB panels
  static constexpr uint32_t s_pp = s_kb + 16384;    // P
  static constexpr uint32_t s_tp = s_pp + 8192;     // T'
  static constexpr uint32_t s_gc = s_tp + 8192;     // package vector
  static constexpr uint32_t gc_bytes = kGcFloats<DK> * 4;
  static constexpr uint32_t copy_bytes = s_gc + gc_bytes;
  static constexpr uint32_t slot = (copy_bytes + 1023) & ~1023u;
  // The package goes to the peer in three parts, each as soon as it exists
  // and the peer's slot is free: Qt, Kb, P and exp(g_C) (early), T' (after
  // the inverse), W (last).  Kb's second panel is all zero when DK = 64 and
  // stays out (zero in every slot from the start).
  static constexpr uint32_t kb_bytes = DK == 64 ? 8192 : 16384;
  static constexpr uint32_t push_bytes =
      NP * 8192 /* Qt */ + kb_bytes + 8192 /* P */ + gc_bytes + 8192 /* T' */ +
      NP * 8192 /* W */;
  // producer-private
  static constexpr uint32_t afp = 2 * slot;         // 64 x kFS fp32
  static constexpr uint32_t tfp = afp + 64 * kFS * 4;
  static constexpr uint32_t msc = tfp + 64 * kFS * 4;
  // consumer-private
  static constexpr uint32_t sop = msc + 4096;       // S, DK rows
  static constexpr uint32_t dop = sop + DK * 128;   // Delta, 64 rows
  static constexpr uint32_t vbuf = dop + 8192;      // two V tiles
  static constexpr uint32_t misc = vbuf + 16384;    // betas, barriers
  static constexpr uint32_t bytes = misc + 1024;
  static constexpr uint32_t tx_qk = 2 * NP * 8192;
  // TMEM columns
  static constexpr uint32_t t_d1 = 0;
  static constexpr uint32_t t_w = 64;
  static constexpr uint32_t t_u = 64 + DK;
  static constexpr uint32_t t_d3 = 128 + DK;
  static constexpr uint32_t t_s = 192 + DK;
  static constexpr uint32_t t_d3b = 256 + DK;  // MMA3/MMA5 of odd chunks
  static_assert(t_d3b + 64 <= 512, "TMEM columns");
  static_assert(slot % 1024 == 0 && sop % 1024 == 0 && dop % 1024 == 0 &&
                    vbuf % 1024 == 0,
                "swizzle atoms");
  static_assert(copy_bytes % 16 == 0 && push_bytes < (1u << 20), "push size");
  static_assert(gc_bytes % 16 == 0, "package vector copy size");
  static_assert(bytes + 1024 <= 232448, "shared memory");
};

template <int DK, int GATE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    fused_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const WsParams p) {
  using Lay = PairLayout<DK>;
  constexpr int NCG = DK / 4;
  constexpr int NRB = kProd / NCG;
  constexpr int RPT = kC / NRB;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* afp = reinterpret_cast<float*>(sm + Lay::afp);
  float* tfp = reinterpret_cast<float*>(sm + Lay::tfp);
  uint8_t* sop = sm + Lay::sop;
  uint8_t* dop = sm + Lay::dop;
  uint8_t* vbuf = sm + Lay::vbuf;
  float* betas = reinterpret_cast<float*>(sm + Lay::misc);  // [64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::misc + 256);
  uint64_t* bar_in = bars + 0;   // [2]
  uint64_t* full = bars + 2;     // [2] own chunk ready (local arrive)
  uint64_t* pfull = bars + 4;    // [2] peer chunk arrived (peer's pushes)
  uint64_t* send_ok = bars + 6;  // [2]
  uint64_t* bar_v = bars + 8;    // [2]
  uint64_t* bar_m1 = bars + 10;
  uint64_t* bar_m2 = bars + 11;
  uint64_t* bar_cm = bars + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 14);
  // q/k loads issued per slot: [0..1] by the producer, [2..3] by the consumer
  int* issued = reinterpret_cast<int*>(bars + 15);
  // the consumer's four warps have written the next chunk's bf16 state
  uint64_t* bar_sop = bars + 17;

  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t r = cta_rank(), peer = r ^ 1u;
  const int unit = blockIdx.x >> 1;
  const int h = unit % p.H;
  const int rank = unit / p.H;
  const int seq = p.order ? p.order[rank] : rank;
  const int j0 = (int)r * kDvt;
  int start, end;
  seq_range(p.cu, seq, p.T, &start, &end);
  const int nch = (end - start + kC - 1) / kC;
  auto slot_of = [&](int s) { return sm + s * Lay::slot; };

  if (tid == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_in + s, 1);
      mbar_init(full + s, 1);
      mbar_init(pfull + s, 1);
      mbar_init(send_ok + s, 1);
      mbar_init(bar_v + s, 1);
    }
    mbar_init(bar_m1, 1);
    mbar_init(bar_m2, 1);
    mbar_init(bar_cm, 1);
    mbar_init(bar_sop, 4);
    *abort_flag = 0;
    for (int i = 0; i < 4; ++i) issued[i] = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  for (int i = tid; i < 64 * kFS; i += kThreads) tfp[i] = 0.f;
  if (DK == 64) {  // the second M-panel of each Kb stays zero
    for (int i = tid; i < 2 * 512; i += kThreads) {
      uint4* z = reinterpret_cast<uint4*>(slot_of(i >> 9) + Lay::s_kb + 8192);
      z[i & 511] = make_uint4(0, 0, 0, 0);
    }
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync_all();  // both CTAs' barriers exist before any remote access
  const uint32_t tmem = *tmem_slot;
  const uint32_t peer_pfull = peer_addr(pfull, peer);
  const uint32_t peer_ok = peer_addr(send_ok, peer);
  const uint32_t peer_slots = peer_addr(sm, peer);
  const uint32_t peer_abort = peer_addr((const void*)abort_flag, peer);
  bool failed = false;

  // raw q and k of chunk starting at token tok into slot s (kq panels: k
  // over the Kt rows, q over the Qt rows)
  auto issue_qk = [&](int s, int tok) {
    uint8_t* kq = slot_of(s) + Lay::s_kq;
    mbar_arrive_expect_tx(bar_in + s, Lay::tx_qk);
#pragma unroll
    for (int q = 0; q < (int)Lay::NP; ++q) {
      tma_load_3d(kq + q * 16384 + 8192, &tm_q, bar_in + s, q * 64, h, tok);
      tma_load_3d(kq + q * 16384, &tm_k, bar_in + s, q * 64, h, tok);
    }
  };
  auto raise_abort = [&]() {
    *abort_flag = 1;
    remote_store(peer_abort, 1u);
    atomicExch(&g_fused_timeout, 1);
  };

  uint32_t waited0 = 0u, waited1 = 0u;  // bar_in phases consumed (producer)
  if (tid < kProd) {
    // =================================================== producer role
    const int t = tid;
    const int colh = warp >> 2;
    const int row_t = t & 127;
    const int cg = t % NCG, rb = t / NCG;
    const int pnl = cg >> 4;
    const float* la_g = GATE == kGateChannel ? p.log_alpha + (size_t)h * DK + 4 * cg
                                             : p.log_alpha + h;
    const size_t la_stride = GATE == kGateChannel ? (size_t)p.H * DK : (size_t)p.H;
    const int n_own = nch > (int)r ? (nch - (int)r + 1) / 2 : 0;

    float4 la_reg[RPT];
    auto load_la = [&](int tok0, int L) {
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
        const int rr = rb * RPT + i;
        la_reg[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (GATE == kGateChannel)
          ldg_f4_if(la_reg[i], la_g + (size_t)(tok0 + rr) * la_stride, rr < L);
        else if (GATE == kGateHead)
          ldg_f1_if(la_reg[i].x, la_g + (size_t)(tok0 + rr) * la_stride, rr < L);
      }
    };
    if (t == 0) {  // own chunks whose slot has no earlier occupant
      for (int j = 0; j < n_own && (int)r + 2 * j < 3; ++j) {
        issue_qk((j + (int)r) & 1, start + ((int)r + 2 * j) * kC);
        issued[(j + (int)r) & 1] += 1;
      }
    }
    float beta_next = 0.f;
    if (n_own > 0) {
      const int tok0 = start + (int)r * kC;
      load_la(tok0, min(kC, end - tok0));
      ldg_f1_if(beta_next, p.beta + (size_t)(tok0 + t) * p.H + h,
                t < kC && t < end - tok0);
    }
    uint32_t ph_m1 = 0, ph_m2 = 0;
    // Thread 32 (the copier) sends the package to the peer, so that the
    // copies' issue never holds up thread 0's MMAs; its state per chunk:
    const bool copier = t == 32;
    bool send_fail = false;  // a wait for the peer's slot gave up
    bool slot_ok = false, sent_early = false, sent_tp = false;

    for (int j = 0; j < n_own; ++j) {
      const int n = (int)r + 2 * j;
      const int s = (j + (int)r) & 1;
      const int tok0 = start + n * kC;
      const int L = min(kC, end - tok0);
      const bool has_next = j + 1 < n_own;
      uint8_t* slot = slot_of(s);
      uint8_t* kq = slot + Lay::s_kq;
      uint8_t* kb = slot + Lay::s_kb;
      uint8_t* pp = slot + Lay::s_pp;
      uint8_t* tp = slot + Lay::s_tp;
      float* gc = reinterpret_cast<float*>(slot + Lay::s_gc);
      if (t < kC) betas[t] = beta_next;
      beta_next = 0.f;
      ldg_f1_if(beta_next, p.beta + (size_t)(tok0 + 2 * kC + t) * p.H + h,
                t < kC && has_next && t < end - (tok0 + 2 * kC));
      if (t == 0 && has_next) {  // the next own chunk's q and k into L2
#pragma unroll
        for (int q = 0; q < (int)Lay::NP; ++q) {
          prefetch_box_l2(&tm_q, q * 64, h, tok0 + 2 * kC);
          prefetch_box_l2(&tm_k, q * 64, h, tok0 + 2 * kC);
        }
      }
      const uint32_t wn = s ? waited1 : waited0;
      bool ok = wait_or_abort<true>(bar_in + s, wn & 1u, abort_flag);
      if (ok) {
        if (s) ++waited1;
        else ++waited0;
      }
      if (named_sync_or(kBarProd, kProd, !ok || send_fail)) {
        failed = true;
        break;
      }
      const uint32_t ps = (uint32_t)j & 1u;  // the peer's slot for this chunk
      const uint32_t pdst = peer_slots + ps * Lay::slot;
      const uint32_t pbar = peer_pfull + 8u * ps;
      // The peer's slot ps is free once the peer's consumer has used the
      // peer's own chunk before this one there (send_ok) and the peer's copy
      // of that chunk to this CTA has been read out, which the arrival of
      // all its bytes here (pfull) proves.  The first chunks find it free.
      auto peer_slot_free = [&](bool block) {
        const int ip = j + (int)r - 1;  // that chunk, as this CTA's peer chunk
        if (ip < 0) return true;
        const uint32_t par = (uint32_t)(ip >> 1) & 1u;
        uint64_t* pf = pfull + (ip & 1);
        return block ? wait_cluster(send_ok + ps, par, abort_flag) &&
                           wait_cluster(pf, par, abort_flag)
                     : test_wait_cluster(send_ok + ps, par) &&
                           test_wait_cluster(pf, par);
      };
      auto push_early = [&]() {  // Qt, Kb, P, exp(g_C)
        remote_arrive_tx(pbar, Lay::push_bytes);
#pragma unroll
        for (int q = 0; q < (int)Lay::NP; ++q)
          copy_to_peer(pdst + q * 16384 + 8192, slot + q * 16384 + 8192, 8192,
                       pbar);
        copy_to_peer(pdst + Lay::s_kb, slot + Lay::s_kb, Lay::kb_bytes, pbar);
        copy_to_peer(pdst + Lay::s_pp, slot + Lay::s_pp, 8192, pbar);
        copy_to_peer(pdst + Lay::s_gc, slot + Lay::s_gc, Lay::gc_bytes, pbar);
        sent_early = true;
      };
      if (copier) slot_ok = sent_early = sent_tp = false;

      // ---- prologue, in place over the raw q and k in the slot
      prologue_rows<DK, GATE>(la_reg, afp, gc, kq + pnl * 16384 + 8192,
                              kq + pnl * 16384, kq + pnl * 16384,
                              kb + pnl * 8192, L, p.pro, t);
      if (has_next) load_la(tok0 + 2 * kC, min(kC, end - (tok0 + 2 * kC)));
      fence_proxy_async();
      named_sync(kBarProd, kProd);
      if (t == 0) {  // MMA1: [Kt; Qt] . Kb^T
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
        mma_commit(bar_m1);
      }

      // ---- A (fp32) and P (bf16 into the slot)
      ok = wait_or_abort<false>(bar_m1, ph_m1, abort_flag);
      ph_m1 ^= 1;
      if (named_sync_or(kBarProd, kProd, !ok)) {
        failed = true;
        break;
      }
      tc_fence_after();
      {
        float v[32];
        tmem_ld32(tmem + lane_base + Lay::t_d1 + 32 * colh, v);
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
      if (gc[2 * DK] != 0.f) rescale_qt<Lay::NP>(kq, gc + DK, t);
      tc_fence_before();
      fence_proxy_async();  // P and Qt, to the copy engine
      named_sync(kBarProd, kProd);

      invert_unit_lower_tc(afp, tfp, reinterpret_cast<float*>(sm + Lay::msc), t);

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
      named_sync(kBarProd, kProd);
      if (copier) {  // early parts to the peer while MMA2 runs
        slot_ok = peer_slot_free(false);
        if (slot_ok) {
          push_early();
          copy_to_peer(pdst + Lay::s_tp, tp, 8192, pbar);
          sent_tp = true;
        }
      }
      if (t == 0) {  // MMA2: W = T' Kt (N = DK)
        tc_fence_after();
        const uint32_t iw = idesc_bf16(128, DK, false, true);
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks)
          mma_bf16(tmem + Lay::t_w,
                   desc_sw128(smem_u32(tp) + ks * 32, 16, 1024),
                   desc_sw128(smem_u32(kq) + ks * 2048, 16384, 1024), iw,
                   ks > 0);
        mma_commit(bar_m2);
      }
      ok = wait_or_abort<false>(bar_m2, ph_m2, abort_flag);
      ph_m2 ^= 1;
      if (named_sync_or(kBarProd, kProd, !ok)) {
        failed = true;
        break;
      }
      tc_fence_after();
      if (row_t < 64) {  // W rows (bf16) over the Kt rows of the slot:
        // T' (k e^(g-rho)) scaled by exp(rho) per column = T' (k e^g)
#pragma unroll
        for (int jj = 0; jj < DK / 64; ++jj) {
          const int hh = colh * (DK / 64) + jj;
          float v[32];
          tmem_ld32(tmem + lane_base + Lay::t_w + 32 * hh, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= gc[DK + 32 * hh + i];
          st_chunks<4>(kq + (hh >> 1) * 16384, row_t, 4 * (hh & 1), v);
        }
      }
      tc_fence_before();
      fence_proxy_async();
      named_sync(kBarProd, kProd);
      if (t == 0) mbar_arrive(full + s);  // to this CTA's consumer
      if (copier) {
        if (!slot_ok) slot_ok = peer_slot_free(true);
        if (slot_ok) {  // the rest of the package: (Qt, Kb, P, T') and W
          if (!sent_early) push_early();
          if (!sent_tp) copy_to_peer(pdst + Lay::s_tp, tp, 8192, pbar);
#pragma unroll
          for (int q = 0; q < (int)Lay::NP; ++q)
            copy_to_peer(pdst + q * 16384, slot + q * 16384, 8192, pbar);
          bulk_commit();
        } else {
          send_fail = true;
        }
      }
    }
    failed = named_sync_or(kBarProd, kProd, failed || send_fail);
    if (t == 0 && failed) raise_abort();
    if (copier) {
      bulk_commit();  // copies issued before a failure cut the chunk short
      bulk_wait_all();  // outgoing copies complete before the peer may leave
    }
  } else {
    // =================================================== consumer role
    const int c = tid - kProd;  // TMEM lane = accumulator row
    const bool owns_state = c < DK;
    const size_t sbase = (((size_t)seq * p.H + h) * DK) * p.dv + j0;
    if (owns_state) {  // initial state into TMEM (fp32) and the bf16 operand
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float v[32];
        if (p.s_init) {
          const float4* src = reinterpret_cast<const float4*>(
              p.s_init + sbase + (size_t)c * p.dv + 32 * hf);
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
        tmem_st32(tmem + lane_base + Lay::t_s + 32 * hf, v);
        st_chunks<4>(sop, c, 4 * hf, v);
      }
      tmem_wait_st();
    }
    tc_fence_before();
    fence_proxy_async();
    named_sync(kBarCons, kCons);
    auto issue_v = [&](int n) {
      uint64_t* b = bar_v + (n & 1);
      mbar_arrive_expect_tx(b, 8192);
      tma_load_3d(vbuf + (n & 1) * 8192, &tm_v, b, j0, h, start + n * kC);
    };
    int v_issued = 0;
    if (c == 0 && nch > 0) issue_v(0);
    v_issued = nch > 0 ? 1 : 0;
    uint32_t ph_cm = 0;
    int n = 0;
    // Per chunk n: thread 0 issues U = T' V and MMA3 as soon as the package,
    // V and the bf16 state S_n are in place; Delta; MMA4 and MMA5; then the
    // state S_(n+1) = exp(g_C) S is written as the bf16 operand first (the
    // four warps announce it on bar_sop, which releases the next MMA3) and
    // back to TMEM after, and the outputs of chunk n are stored from their
    // TMEM buffer (two buffers, alternating by chunk) while the next MMA3
    // runs.
    for (; n < nch; ++n) {
      const int s = ((n + (int)r) >> 1) & 1;
      const bool own = (n & 1) == (int)r;
      const int tok0 = start + n * kC;
      const int L = min(kC, end - tok0);
      uint8_t* slot = slot_of(s);
      uint8_t* kq = slot + Lay::s_kq;
      uint8_t* kb = slot + Lay::s_kb;
      uint8_t* pp = slot + Lay::s_pp;
      uint8_t* tp = slot + Lay::s_tp;
      const float* gc = reinterpret_cast<const float*>(slot + Lay::s_gc);
      uint8_t* vb = vbuf + (n & 1) * 8192;
      const uint32_t d3 = (n & 1) ? Lay::t_d3b : Lay::t_d3;
      if (n + 1 < nch) {  // V of the next chunk (its buffer was freed by n - 1)
        if (c == 0) issue_v(n + 1);
        v_issued = n + 2;
      }
      // own chunk j = n >> 1 is the (j >> 1)-th own use of its slot; peer
      // chunk i = n >> 1 the (i >> 1)-th peer use
      const uint32_t par = (uint32_t)(n >> 2) & 1u;
      bool ok = true;
      if (c == 0) {  // ---- U = T' V ; [W; Qt] . S
        ok = wait_cluster((own ? full : pfull) + s, par, abort_flag);
        ok = ok && wait_or_abort<false>(bar_v + (n & 1),
                                        (uint32_t)(n >> 1) & 1u, abort_flag);
        if (n > 0)
          ok = ok && wait_or_abort<false>(bar_sop, (uint32_t)(n - 1) & 1u,
                                          abort_flag);
        if (ok) {
          tc_fence_after();
          if (!own) fence_proxy_async();  // the peer's stores, to the MMA reads
          const uint32_t idesc = idesc_bf16(128, 64, false, true);
#pragma unroll
          for (int ks = 0; ks < kC / 16; ++ks)
            mma_bf16(tmem + Lay::t_u,
                     desc_sw128(smem_u32(tp) + ks * 32, 16, 1024),
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
          raise_abort();  // the other threads leave their wait below
        }
      }
      ok = ok && wait_or_abort<false>(bar_cm, ph_cm, abort_flag);
      ph_cm ^= 1;
      if (named_sync_or(kBarCons, kCons, !ok)) {
        failed = true;
        break;
      }
      tc_fence_after();

      // ---- Delta = U - W S (rows 0-63)
      if (c < 64) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          float uu[32], wsv[32];
          tmem_ld32(tmem + lane_base + Lay::t_u + 32 * hf, uu);
          tmem_ld32(tmem + lane_base + d3 + 32 * hf, wsv);
#pragma unroll
          for (int i = 0; i < 32; ++i) uu[i] -= wsv[i];
          st_chunks<4>(dop, c, 4 * hf, uu);
        }
      }
      const float gamma = owns_state ? gc[c] : 1.f;
      if (owns_state && gc[2 * DK] != 0.f) {
        // S_C = e^(g_C - rho) (e^rho S_0 + Kb^T Delta): pre-scale the state
        const float er = gc[DK + c];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          float v[32];
          tmem_ld32(tmem + lane_base + Lay::t_s + 32 * hf, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= er;
          tmem_st32(tmem + lane_base + Lay::t_s + 32 * hf, v);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      fence_proxy_async();
      named_sync(kBarCons, kCons);

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
          mma_bf16(tmem + d3,
                   desc_sw128(smem_u32(pp) - 8192 + ks * 32, 16, 1024), bd, i5,
                   1u);
        }
        mma_commit(bar_cm);
      }
      ok = wait_or_abort<false>(bar_cm, ph_cm, abort_flag);
      ph_cm ^= 1;
      if (named_sync_or(kBarCons, kCons, !ok)) {
        failed = true;
        break;
      }
      tc_fence_after();
      if (c == 0) {  // slot s is used up
        if (own) {
          remote_arrive(peer_ok + 8u * (uint32_t)s);
        } else if (n + 3 < nch) {  // the own chunk that follows in slot s
          issue_qk(s, start + (n + 3) * kC);
          issued[2 + s] += 1;
        }
      }

      // ---- S <- exp(g_C) S: the bf16 operand of the next MMA3 first, then
      // TMEM (the store completes before the next MMA4 is issued)
      if (owns_state) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          float v[32];
          tmem_ld32(tmem + lane_base + Lay::t_s + 32 * hf, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= gamma;
          st_chunks<4>(sop, c, 4 * hf, v);
          tmem_st32(tmem + lane_base + Lay::t_s + 32 * hf, v);
        }
      }
      fence_proxy_async();
      tc_fence_before();
      __syncwarp();
      if ((c & 31) == 0) mbar_arrive(bar_sop);

      // ---- outputs (rows 64-127 of this chunk's buffer), overlapping the
      // next chunk's MMA3
      if (c >= 64) {
        const int rr = c - 64;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          float o[32];
          tmem_ld32(tmem + lane_base + d3 + 32 * hf, o);
          if (rr < L) {
            uint4* dst = reinterpret_cast<uint4*>(
                p.out + ((size_t)(tok0 + rr) * p.H + h) * p.dv + j0 + 32 * hf);
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
      }
      if (owns_state) tmem_wait_st();
      tc_fence_before();
    }
    if (failed) {
      if (c == 0) {
        raise_abort();
        // V loads still in flight: chunks n .. v_issued - 1 (n's was not
        // consumed when the wait gave up before it)
        for (int m = n; m < v_issued; ++m)
          mbar_wait(bar_v + (m & 1), (uint32_t)(m >> 1) & 1u, 100000000ull);
      }
    } else if (owns_state) {
      tc_fence_after();
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float v[32];
        tmem_ld32(tmem + lane_base + Lay::t_s + 32 * hf, v);
        float4* dst = reinterpret_cast<float4*>(p.s_final + sbase +
                                                (size_t)c * p.dv + 32 * hf);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    // q/k loads issued into a slot but never waited for (after a failure)
    for (int s = 0; s < 2; ++s) {
      const uint32_t done = s ? waited1 : waited0;
      for (uint32_t m = done; m < (uint32_t)(issued[s] + issued[2 + s]); ++m)
        mbar_wait(bar_in + s, m & 1u, 100000000ull);
    }
  }
  cluster_sync_all();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// Host side: one cluster of two CTAs per (sequence, head), CTA r on the d_v
// columns 64 r .. 64 r + 63 (d_v = 128 only).
template <int DK, int GATE>
cudaError_t run_pair(const ChunkArgs& a, const int32_t* order,
                     cudaStream_t stream) {
  using Lay = PairLayout<DK>;
  const int tokens = a.cu_seqlens ? a.T : a.n_seqs * a.T;
  CUtensorMap tq, tk, tv;
  if (!make_tile_map(&tq, a.q, DK, a.H, tokens) ||
      !make_tile_map(&tk, a.k, DK, a.H, tokens) ||
      !make_tile_map(&tv, a.v, a.dv, a.H, tokens))
    return cudaErrorInvalidValue;
  WsParams p{};
  p.pro = a.pro;
  p.beta = a.beta;
  p.log_alpha = a.log_alpha;
  p.s_init = a.initial_state;
  p.s_final = a.final_state;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.cu = a.cu_seqlens;
  p.order = order;
  p.n_seqs = a.n_seqs;
  p.T = a.T;
  p.H = a.H;
  p.dv = a.dv;
  p.n_tiles = 2;
  const size_t smem = Lay::bytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(
      fused_pair_kernel<DK, GATE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
      (int)smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = 2u * (unsigned)a.n_seqs * (unsigned)a.H;
  fused_pair_kernel<DK, GATE><<<grid, kThreads, smem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

inline cudaError_t launch_fused_pair(const ChunkArgs& a, const int32_t* order,
                                     cudaStream_t stream) {
  if (a.gate == kGateHead)
    return a.dk == 128 ? run_pair<128, kGateHead>(a, order, stream)
                       : run_pair<64, kGateHead>(a, order, stream);
  if (a.gate == kGateNone)
    return a.dk == 128 ? run_pair<128, kGateNone>(a, order, stream)
                       : run_pair<64, kGateNone>(a, order, stream);
  return a.dk == 128 ? run_pair<128, kGateChannel>(a, order, stream)
                     : run_pair<64, kGateChannel>(a, order, stream);
}

}  // namespace pair
}  // namespace kda
