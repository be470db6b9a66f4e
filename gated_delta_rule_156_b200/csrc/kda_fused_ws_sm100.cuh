// Warp-specialised fused chunkwise KDA prefill for sm_100a.
//
// Same mathematics as the single-role kernel (see kda_fused_sm100.cu), split
// into two roles that work on different chunks at the same time:
//   producer (warps 0-7, 256 threads): for chunk n it forms the decay-scaled
//     operands (prologue), A and P (MMA1), T' = (I + A)^-1 Diag(beta) (blocked
//     inverse), W = T' Kt and U = T' V (MMA2), and hands them over in operand
//     slot n mod 2;
//   consumer (warps 8-11, 128 threads): for chunk n it forms W S and Qt S
//     (MMA3), Delta = U - W S, the state update and the output (MMA4, MMA5).
// While the consumer runs the serial state chain of chunk n the producer
// works on chunk n + 1.  The slots are handed over by full/empty mbarriers.
//
// The state stays in TMEM in fp32.  The consumer uses the identity
//   S_C = Diag(exp(g_C)) S_0 + Kh^T Delta = Diag(exp(g_C)) (S_0 + Kb^T Delta),
// since Kh = Kb Diag(exp(g_C)) row-wise.  MMA4 therefore accumulates
// Kb^T Delta straight onto the state, and the epilogue rescales each state row
// by exp(g_C) (tcgen05.ld / tcgen05.st).  The separate Kh operand is not
// needed.  log(alpha) is prefetched into the producer's registers with plain
// global loads one chunk ahead; q, k and V arrive by TMA.
// Included by kda_fused_sm100.cu (same translation unit: it shares the
// device-side timeout flag and the tensor-map helper).
#pragma once

#include "kda_inverse_tc.cuh"

namespace kda {
namespace ws {

using namespace sm100;

constexpr int kC = 64;
constexpr int kDvt = 64;
constexpr int kProd = 256;  // producer threads (warps 0-7)
constexpr int kCons = 128;  // consumer threads (warps 8-11)
constexpr int kThreads = kProd + kCons;
constexpr int kBarProd = kBarInv, kBarCons = 2;  // named barrier ids
static_assert(kProd == kInvThreads, "the inverse runs on the producer");

// Floats of a chunk's package vector: exp(g_C - rho) and exp(rho) per
// channel, the "some rho != 0" word, padding to 16 bytes.
template <int DK>
constexpr int kGcFloats = 2 * DK + 4;

template <int DK>
struct WsLayout {
  static constexpr uint32_t NP = DK / 64;
  // producer-private
  static constexpr uint32_t stage_q = 0;                    // NP x 8 KB
  static constexpr uint32_t stage_k = stage_q + NP * 8192;  // NP x 8 KB
  static constexpr uint32_t vbuf = stage_k + NP * 8192;     // 8 KB
  static constexpr uint32_t afp = vbuf + 8192;              // 64 x kFS fp32
  static constexpr uint32_t tfp = afp + 64 * kFS * 4;       // 64 x kFS fp32
  static constexpr uint32_t msc = tfp + 64 * kFS * 4;       // 1024 fp32
  static constexpr uint32_t tp = msc + 4096;                // T', 64 rows
  // slots (two of each)
  static constexpr uint32_t kq = tp + 8192;                 // [Kt/W; Qt]
  static constexpr uint32_t kq_stride = NP * 16384;
  static constexpr uint32_t kb = kq + 2 * kq_stride;        // Kb, 2 panels
  static constexpr uint32_t pp = kb + 2 * 16384;            // P, 64 rows
  // consumer-private
  static constexpr uint32_t sop = pp + 2 * 8192;            // S, DK rows
  static constexpr uint32_t dop = sop + DK * 128;           // Delta, 64 rows
  static constexpr uint32_t misc = dop + 8192;
  // betas [2][64], package vectors [2][kGcFloats], barriers
  static constexpr uint32_t gcs = 512;
  static constexpr uint32_t bars = gcs + 2 * kGcFloats<DK> * 4;
  static constexpr uint32_t bytes = misc + 3072;
  static_assert(bars + 128 <= 3072, "misc area");
  static_assert(bytes + 1024 <= 232448, "shared memory");
  static constexpr uint32_t tx_qk = 2 * NP * 8192;
  // TMEM columns: D1 (two buffers), W, U (two slots), D3, S
  static constexpr uint32_t t_d1 = 0;
  static constexpr uint32_t t_w = 128;
  static constexpr uint32_t t_u0 = 128 + DK;
  static constexpr uint32_t t_d3 = 256 + DK;
  static constexpr uint32_t t_s = 320 + DK;
  static_assert(t_s + 64 <= 512, "TMEM columns");
  static_assert(tp % 1024 == 0 && kq % 1024 == 0, "swizzle atoms");
};

struct WsParams {
  Prologue pro;
  const float* beta;
  const float* log_alpha;
  const float* s_init;
  float* s_final;
  __nv_bfloat16* out;
  const int32_t* cu;
  const int32_t* order;
  int n_seqs, T, H, dv, n_tiles;
};

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// Barrier over `n` threads that also returns whether any thread's `pred`
// was set.
__device__ __forceinline__ bool named_sync_or(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// Bounded wait that also gives up when the other role has failed.  The
// try_wait carries a suspend-time hint, so a waiting warp sleeps in the
// barrier unit (issuing nothing) until the phase completes or 0.5 ms pass.
__device__ __forceinline__ bool try_wait_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(500000u)
      : "memory");
  return ok != 0;
}
// Bounded wait, also abandoned when the other role has failed.  Waits on
// the other role (slot full / empty) sleep in the barrier unit; waits on this
// role's own MMAs and TMA copies, which end within microseconds, poll.
template <bool kSleep>
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag) {
  auto once = [&]() {
    return kSleep ? try_wait_sleep(bar, parity) : mbar_try_wait(bar, parity);
  };
  if (once()) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (once()) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > 2000000000ull) return false;
  }
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, "
      "%31, %32};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]),
      "f"(v[6]), "f"(v[7]), "f"(v[8]), "f"(v[9]), "f"(v[10]), "f"(v[11]),
      "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]), "f"(v[16]), "f"(v[17]),
      "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]),
      "f"(v[24]), "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]), "f"(v[29]),
      "f"(v[30]), "f"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Predicated loads into registers that keep their old value when `pred` is
// false: no select follows the load, so nothing waits for it until the value
// is used (the prefetches below are used one chunk later).
__device__ __forceinline__ void ldg_f4_if(float4& v, const float* p, bool pred) {
  asm volatile(
      "{\n\t.reg .pred q;\n\t"
      "setp.ne.u32 q, %4, 0;\n\t"
      "@q ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%5];\n\t}"
      : "+f"(v.x), "+f"(v.y), "+f"(v.z), "+f"(v.w)
      : "r"((uint32_t)pred), "l"(p));
}
__device__ __forceinline__ void ldg_f1_if(float& v, const float* p, bool pred) {
  asm volatile(
      "{\n\t.reg .pred q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "@q ld.global.nc.f32 %0, [%2];\n\t}"
      : "+f"(v)
      : "r"((uint32_t)pred), "l"(p));
}

// Rows 64-127 (Qt) of the NP 64-column panels of a [Kt; Qt] operand, scaled
// in place by exp(rho) per column (gr): Qt = q e^(g - rho) becomes the
// chunk-start q e^g.  256 threads, 16 bytes at a time.
template <int NP>
__device__ __forceinline__ void rescale_qt(uint8_t* kq, const float* gr, int t) {
#pragma unroll
  for (int i = 0; i < 2 * NP; ++i) {
    const int x = t + 256 * i;
    const int pnl = x >> 9, rr = 64 + ((x & 511) >> 3), ch = x & 7;
    uint4* p = reinterpret_cast<uint4*>(kq + pnl * 16384 + rr * 128 +
                                        ((ch ^ (rr & 7)) << 4));
    uint4 w = *p;
    __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&w);
    const float* f = gr + pnl * 64 + ch * 8;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 v = __bfloat1622float2(h2[j]);
      h2[j] = __floats2bfloat162_rn(v.x * f[2 * j], v.y * f[2 * j + 1]);
    }
    *p = w;
  }
}

template <int N>
__device__ __forceinline__ void st_chunks(uint8_t* panel, int row, int c0,
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

// The producer prologue of one chunk, over all 256 producer threads: turns
// the log(alpha) rows held in registers (raw gate logits with the prologue)
// into the running decay g and, with the per-channel reference rho =
// decay_ref(g_C), writes the decay-scaled bf16 operands Kt = k e^(g-rho) and
// Qt = q e^(g-rho) (rows 0-63 and 64-127 of the [Kt; Qt] panel pkq) and
// Kb = k e^(rho-g) (panel pkb) from the raw q and k rows at pq and pk.  The
// package vector gc (kGcFloats floats) receives exp(g_C - rho) per channel,
// then exp(rho) per channel, then a nonzero word when some channel of the
// chunk has rho != 0 (its Qt rows and W columns are then rescaled by exp(rho)
// to the chunk-start operands, and its state pre-scaled, see rescale_qt and
// the consumers).  A chunk whose decay leaves the supported range raises
// g_fused_range.  Thread t owns channels 4 cg .. 4 cg + 3 of rows
// rb RPT .. rb RPT + RPT - 1; rows at or past L are written as zeros.  pq and
// pk may be the same bytes as the destination rows (in-place transform): each
// element is read and rewritten by the same thread.  `red` is DK * NRB
// floats of scratch.
template <int DK, int GATE>
__device__ __forceinline__ void prologue_rows(float4* la_reg, float* red,
                                              float* gc, const uint8_t* pq,
                                              const uint8_t* pk, uint8_t* pkq,
                                              uint8_t* pkb, int L,
                                              const Prologue& pro, int t) {
  constexpr int NCG = DK / 4;
  constexpr int NRB = kProd / NCG;
  constexpr int RPT = kC / NRB;
  const int cg = t % NCG, rb = t / NCG;
  const int ck = (cg >> 1) & 7, cb = (cg & 1) * 8;
  if (GATE != kGateNone && pro.gate_logits) {
    // raw logits x -> log(alpha) = scale * logsigmoid(x), valid rows only
    const float sc = pro.gate_scale;
    auto ls = [&](float x) {
      // log1p(e) as log(1 + e): e = exp(-|x|) <= 1, so the two differ by
      // less than 6e-8 in absolute terms, far below bf16 resolution
      return sc * (fminf(x, 0.f) - __logf(1.f + __expf(-fabsf(x))));
    };
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      if (rb * RPT + i < L) {
        la_reg[i].x = ls(la_reg[i].x);
        if (GATE == kGateChannel) {
          la_reg[i].y = ls(la_reg[i].y);
          la_reg[i].z = ls(la_reg[i].z);
          la_reg[i].w = ls(la_reg[i].w);
        }
      }
    }
  }
  if (GATE == kGateHead) {
#pragma unroll
    for (int i = 0; i < RPT; ++i)
      la_reg[i].y = la_reg[i].z = la_reg[i].w = la_reg[i].x;
  }
  float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    part[0] += la_reg[i].x; part[1] += la_reg[i].y;
    part[2] += la_reg[i].z; part[3] += la_reg[i].w;
  }
  *reinterpret_cast<float4*>(red + rb * DK + 4 * cg) =
      make_float4(part[0], part[1], part[2], part[3]);
  named_sync(kBarProd, kProd);
  float g[4] = {0.f, 0.f, 0.f, 0.f}, tot[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int b2 = 0; b2 < NRB; ++b2) {
    const float4 y = *reinterpret_cast<const float4*>(red + b2 * DK + 4 * cg);
    if (b2 < rb) { g[0] += y.x; g[1] += y.y; g[2] += y.z; g[3] += y.w; }
    tot[0] += y.x; tot[1] += y.y; tot[2] += y.z; tot[3] += y.w;
  }
  constexpr float kLog2e = 1.4426950408889634f;
  float rho[4];
  bool shifted = false, out_of_range = false;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    rho[c] = decay_ref(tot[c]);
    shifted |= rho[c] != 0.f;
    out_of_range |= fabsf(tot[c]) > kDecayRangeMax;
  }
  if (t < 32) {  // warp 0 holds every channel (rb 0, and rb 1 when DK = 64)
    const bool any = __any_sync(0xffffffffu, shifted);
    if (rb == 0) {
      *reinterpret_cast<float4*>(gc + 4 * cg) = make_float4(
          ex2_approx((tot[0] - rho[0]) * kLog2e), ex2_approx((tot[1] - rho[1]) * kLog2e),
          ex2_approx((tot[2] - rho[2]) * kLog2e), ex2_approx((tot[3] - rho[3]) * kLog2e));
      *reinterpret_cast<float4*>(gc + DK + 4 * cg) = make_float4(
          ex2_approx(rho[0] * kLog2e), ex2_approx(rho[1] * kLog2e),
          ex2_approx(rho[2] * kLog2e), ex2_approx(rho[3] * kLog2e));
      if (out_of_range) atomicExch(&g_fused_range, 1);
    }
    if (t == 0) gc[2 * DK] = any ? 1.f : 0.f;
  }
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const int r = rb * RPT + i;
    const uint32_t off = r * 128 + ((ck ^ (r & 7)) << 4) + cb;
    const bool valid = r < L;
    const uint2 kr = *reinterpret_cast<const uint2*>(pk + off);
    const uint2 qr = *reinterpret_cast<const uint2*>(pq + off);
    g[0] += la_reg[i].x; g[1] += la_reg[i].y;
    g[2] += la_reg[i].z; g[3] += la_reg[i].w;
    float e[4], ie[4];
    if (GATE == kGateChannel) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float x = (g[c] - rho[c]) * kLog2e;
        e[c] = valid ? ex2_approx(x) : 0.f;
        ie[c] = valid ? ex2_approx(-x) : 0.f;
      }
    } else {  // one decay for the whole row: two exponentials per row
      const float x = (g[0] - rho[0]) * kLog2e;
      const float e0 = !valid ? 0.f : GATE == kGateHead ? ex2_approx(x) : 1.f;
      const float i0 = !valid ? 0.f : GATE == kGateHead ? ex2_approx(-x) : 1.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        e[c] = e0;
        ie[c] = i0;
      }
    }
    const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kr);
    const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(&qr);
    uint2 wt, wq, wb;
    if (pro.norm_qk || pro.q_scale != 1.f) {
      // optional prologue: L2-normalise the rows of q and k (the row's NCG
      // threads reduce by shuffles) and scale q, in fp32
      const float2 k01 = __bfloat1622float2(k2[0]), k23 = __bfloat1622float2(k2[1]);
      const float2 q01 = __bfloat1622float2(q2[0]), q23 = __bfloat1622float2(q2[1]);
      float kf[4] = {k01.x, k01.y, k23.x, k23.y};
      float qf[4] = {q01.x, q01.y, q23.x, q23.y};
      float ik = 1.f, iq = pro.q_scale;
      if (pro.norm_qk) {
        float sk = kf[0] * kf[0] + kf[1] * kf[1] + kf[2] * kf[2] + kf[3] * kf[3];
        float sq = qf[0] * qf[0] + qf[1] * qf[1] + qf[2] * qf[2] + qf[3] * qf[3];
#pragma unroll
        for (int o = NCG / 2; o > 0; o >>= 1) {
          sk += __shfl_xor_sync(0xffffffffu, sk, o);
          sq += __shfl_xor_sync(0xffffffffu, sq, o);
        }
        ik = valid ? rsqrtf(sk) : 0.f;
        iq = valid ? rsqrtf(sq) * pro.q_scale : 0.f;
      }
      wt.x = pack_bf16x2(kf[0] * ik * e[0], kf[1] * ik * e[1]);
      wt.y = pack_bf16x2(kf[2] * ik * e[2], kf[3] * ik * e[3]);
      wq.x = pack_bf16x2(qf[0] * iq * e[0], qf[1] * iq * e[1]);
      wq.y = pack_bf16x2(qf[2] * iq * e[2], qf[3] * iq * e[3]);
      wb.x = pack_bf16x2(kf[0] * ik * ie[0], kf[1] * ik * ie[1]);
      wb.y = pack_bf16x2(kf[2] * ik * ie[2], kf[3] * ik * ie[3]);
    } else {
      const __nv_bfloat162 e01 = __floats2bfloat162_rn(e[0], e[1]);
      const __nv_bfloat162 e23 = __floats2bfloat162_rn(e[2], e[3]);
      const __nv_bfloat162 i01 = __floats2bfloat162_rn(ie[0], ie[1]);
      const __nv_bfloat162 i23 = __floats2bfloat162_rn(ie[2], ie[3]);
      *reinterpret_cast<__nv_bfloat162*>(&wt.x) = __hmul2(k2[0], e01);
      *reinterpret_cast<__nv_bfloat162*>(&wt.y) = __hmul2(k2[1], e23);
      *reinterpret_cast<__nv_bfloat162*>(&wq.x) = __hmul2(q2[0], e01);
      *reinterpret_cast<__nv_bfloat162*>(&wq.y) = __hmul2(q2[1], e23);
      *reinterpret_cast<__nv_bfloat162*>(&wb.x) = __hmul2(k2[0], i01);
      *reinterpret_cast<__nv_bfloat162*>(&wb.y) = __hmul2(k2[1], i23);
    }
    *reinterpret_cast<uint2*>(pkq + off) = wt;
    *reinterpret_cast<uint2*>(pkq + 64 * 128 + off) = wq;
    *reinterpret_cast<uint2*>(pkb + off) = wb;
  }
}

template <int DK, int GATE>
__global__ void __launch_bounds__(kThreads, 1)
    fused_ws_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const WsParams p) {
  using Lay = WsLayout<DK>;
  constexpr int NCG = DK / 4;        // producer prologue: 4-channel groups
  constexpr int NRB = kProd / NCG;   // row blocks
  constexpr int RPT = kC / NRB;      // rows per producer thread
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* st_q = sm + Lay::stage_q;
  uint8_t* st_k = sm + Lay::stage_k;
  uint8_t* vbuf = sm + Lay::vbuf;
  float* afp = reinterpret_cast<float*>(sm + Lay::afp);
  float* tfp = reinterpret_cast<float*>(sm + Lay::tfp);
  uint8_t* tp = sm + Lay::tp;
  uint8_t* sop = sm + Lay::sop;
  uint8_t* dop = sm + Lay::dop;
  float* betas = reinterpret_cast<float*>(sm + Lay::misc);          // [2][64]
  float* gcs = reinterpret_cast<float*>(sm + Lay::misc + Lay::gcs);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::misc + Lay::bars);
  constexpr int GCF = kGcFloats<DK>;
  uint64_t* bar_in = bars + 0;
  uint64_t* bar_v = bars + 1;
  uint64_t* bar_m1 = bars + 2;  // [2] MMA1 into D1 buffer b
  uint64_t* bar_m2 = bars + 4;  // MMA2
  uint64_t* bar_cm = bars + 5;
  uint64_t* full = bars + 6;    // [2]
  uint64_t* empty = bars + 8;   // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 10);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 11);

  const int tid = threadIdx.x, warp = tid >> 5;
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
    mbar_init(bar_in, 1);
    mbar_init(bar_v, 1);
    mbar_init(bar_m1 + 0, 1);
    mbar_init(bar_m1 + 1, 1);
    mbar_init(bar_m2, 1);
    mbar_init(bar_cm, 1);
    mbar_init(full + 0, 1);
    mbar_init(full + 1, 1);
    mbar_init(empty + 0, 1);
    mbar_init(empty + 1, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  for (int i = tid; i < 64 * kFS; i += kThreads) tfp[i] = 0.f;
  if (DK == 64) {  // the second M-panel of each Kb slot stays zero
    for (int i = tid; i < 2 * 512; i += kThreads) {
      uint4* z = reinterpret_cast<uint4*>(sm + Lay::kb + (i >> 9) * 16384 + 8192);
      z[i & 511] = make_uint4(0, 0, 0, 0);
    }
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool failed = false;

  if (tid < kProd) {
    // =================================================== producer role
    const int t = tid;
    const int colh = warp >> 2;  // 32-column half of a 64-column accumulator
    const int row_t = t & 127;
    const int cg = t % NCG, rb = t / NCG;
    const int pnl = cg >> 4;
    // log(alpha): one value per key channel (four per thread), one per head
    // (broadcast over the channels), or none (alpha = 1).
    const float* la_g = GATE == kGateChannel ? p.log_alpha + (size_t)h * DK + 4 * cg
                                             : p.log_alpha + h;
    const size_t la_stride = GATE == kGateChannel ? (size_t)p.H * DK : (size_t)p.H;

    auto issue_qk = [&](int tok) {
      mbar_arrive_expect_tx(bar_in, Lay::tx_qk);
#pragma unroll
      for (int q = 0; q < (int)Lay::NP; ++q) {
        tma_load_3d(st_q + q * 8192, &tm_q, bar_in, q * 64, h, tok);
        tma_load_3d(st_k + q * 8192, &tm_k, bar_in, q * 64, h, tok);
      }
    };
    auto issue_v = [&](int tok) {
      mbar_arrive_expect_tx(bar_v, 8192);
      tma_load_3d(vbuf, &tm_v, bar_v, j0, h, tok);
    };
    float4 la_reg[RPT];
    auto load_la = [&](int tok0, int L) {
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
        const int r = rb * RPT + i;
        la_reg[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (GATE == kGateChannel)
          ldg_f4_if(la_reg[i], la_g + (size_t)(tok0 + r) * la_stride, r < L);
        else if (GATE == kGateHead)
          ldg_f1_if(la_reg[i].x, la_g + (size_t)(tok0 + r) * la_stride, r < L);
      }
    };

    uint32_t ph_in = 0, ph_v = 0, ph_m2 = 0;
    bool in_flight = nch > 0, v_pending = nch > 0;
    float beta_next = 0.f;  // beta of the chunk whose prologue runs next
    if (t == 0 && nch > 0) {
      issue_qk(start);
      issue_v(start);
    }
    if (nch > 0) {
      load_la(start, min(kC, end - start));
      ldg_f1_if(beta_next, p.beta + (size_t)(start + t) * p.H + h,
                t < kC && t < end - start);
    }

    // front(m): wait for slot m % 2 and the q, k of chunk m; prologue into
    // the slot; issue MMA1(m) into D1 buffer m % 2 and the TMA of chunk m+1.
    // It runs between back1 and back2 of the previous chunk, so MMA2's
    // latency is spent on this prologue.
    auto front = [&](int m) -> bool {
      const int s = m & 1, use = m >> 1;
      const int tok0 = start + m * kC;
      const int L = min(kC, end - tok0);
      const bool has_next = m + 1 < nch;
      uint8_t* kq = sm + Lay::kq + s * Lay::kq_stride;
      uint8_t* kb = sm + Lay::kb + s * 16384;
      float* gc = gcs + s * GCF;
      if (t < kC) betas[s * 64 + t] = beta_next;
      beta_next = 0.f;
      ldg_f1_if(beta_next, p.beta + (size_t)(tok0 + kC + t) * p.H + h,
                t < kC && has_next && t < end - (tok0 + kC));
      bool ok = true;
      if (use >= 1) ok = wait_or_abort<true>(empty + s, (use - 1) & 1, abort_flag);
      ok = ok && wait_or_abort<false>(bar_in, ph_in, abort_flag);
      ph_in ^= 1;
      in_flight = false;
      if (named_sync_or(kBarProd, kProd, !ok)) return false;

      prologue_rows<DK, GATE>(la_reg, afp, gc,
                              st_q + pnl * 8192, st_k + pnl * 8192,
                              kq + pnl * 16384, kb + pnl * 8192, L, p.pro, t);
      if (has_next) load_la(tok0 + kC, min(kC, end - (tok0 + kC)));
      fence_proxy_async();
      named_sync(kBarProd, kProd);
      if (t == 0) {  // MMA1: [Kt; Qt] . Kb^T ; then q, k of the next chunk
        tc_fence_after();
        const uint32_t idesc = idesc_bf16(128, 64, false, false);
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
          const uint32_t off = (ks & 3) * 32;
          mma_bf16(tmem + Lay::t_d1 + 64 * s,
                   desc_sw128(smem_u32(kq) + (ks >> 2) * 16384 + off, 16, 1024),
                   desc_sw128(smem_u32(kb) + (ks >> 2) * 8192 + off, 16, 1024),
                   idesc, ks > 0);
        }
        mma_commit(bar_m1 + s);
        if (has_next) issue_qk(tok0 + kC);
      }
      in_flight = has_next;
      return true;
    };

    // back1(n): A and P from D1, the inverse, T', then issue MMA2 (W, U)
    // without waiting for it.
    auto back1 = [&](int n) -> bool {
      const int s = n & 1;
      uint8_t* kq = sm + Lay::kq + s * Lay::kq_stride;
      uint8_t* pp = sm + Lay::pp + s * 8192;
      const float* beta_s = betas + s * 64;
      bool ok = wait_or_abort<false>(bar_m1 + s, (n >> 1) & 1, abort_flag);
      if (named_sync_or(kBarProd, kProd, !ok)) return false;
      tc_fence_after();
      {  // A (fp32) and P (bf16 into the slot)
        float v[32];
        tmem_ld32(tmem + lane_base + Lay::t_d1 + 64 * s + 32 * colh, v);
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
          st_chunks<4>(pp, r, 4 * colh, v);
        }
      }
      // MMA1 has read Qt: back to the chunk-start q e^g where rho != 0
      if (gcs[s * GCF + 2 * DK] != 0.f) rescale_qt<Lay::NP>(kq, gcs + s * GCF + DK, t);
      tc_fence_before();
      named_sync(kBarProd, kProd);

      invert_unit_lower_tc(afp, tfp, reinterpret_cast<float*>(sm + Lay::msc), t);

      {  // T' = Tm Diag(beta), rows masked to the lower triangle
        const int r = t & 63, qc = t >> 6;
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
          const int c = 16 * qc + i;
          const float4 x = *reinterpret_cast<const float4*>(tfp + r * kFS + c);
          const float4 b = *reinterpret_cast<const float4*>(beta_s + c);
          v[i] = c + 0 <= r ? x.x * b.x : 0.f;
          v[i + 1] = c + 1 <= r ? x.y * b.y : 0.f;
          v[i + 2] = c + 2 <= r ? x.z * b.z : 0.f;
          v[i + 3] = c + 3 <= r ? x.w * b.w : 0.f;
        }
        st_chunks<2>(tp, r, 2 * qc, v);
      }
      fence_proxy_async();
      named_sync(kBarProd, kProd);

      if (t == 0) {  // MMA2: W = T' Kt (N = DK), U = T' V (N = 64) into U slot s
        tc_fence_after();
        ok = wait_or_abort<false>(bar_v, ph_v, abort_flag);
        ph_v ^= 1;
        v_pending = !ok;
        if (ok) {
          const uint32_t iw = idesc_bf16(128, DK, false, true);
          const uint32_t iu = idesc_bf16(128, 64, false, true);
#pragma unroll
          for (int ks = 0; ks < kC / 16; ++ks) {
            const uint64_t a = desc_sw128(smem_u32(tp) + ks * 32, 16, 1024);
            mma_bf16(tmem + Lay::t_w, a,
                     desc_sw128(smem_u32(kq) + ks * 2048, 16384, 1024), iw,
                     ks > 0);
            mma_bf16(tmem + Lay::t_u0 + 64 * s, a,
                     desc_sw128(smem_u32(vbuf) + ks * 2048, 8192, 1024), iu,
                     ks > 0);
          }
          mma_commit(bar_m2);
        }
      }
      return !named_sync_or(kBarProd, kProd, !ok);
    };

    // back2(n): wait for MMA2, W into the slot, hand slot n % 2 over.
    auto back2 = [&](int n) -> bool {
      const int s = n & 1;
      const int tok0 = start + n * kC;
      uint8_t* kq = sm + Lay::kq + s * Lay::kq_stride;
      bool ok = wait_or_abort<false>(bar_m2, ph_m2, abort_flag);
      ph_m2 ^= 1;
      if (named_sync_or(kBarProd, kProd, !ok)) return false;
      tc_fence_after();
      if (t == 0 && n + 1 < nch) {  // V is free once MMA2 has completed
        issue_v(tok0 + kC);
        v_pending = true;
      }
      if (row_t < 64) {  // W rows (bf16) over the Kt rows of the slot:
        // T' (k e^(g-rho)) scaled by exp(rho) per column = T' (k e^g)
        const float* gr = gcs + s * GCF + DK;
#pragma unroll
        for (int j = 0; j < DK / 64; ++j) {
          const int hh = colh * (DK / 64) + j;
          float v[32];
          tmem_ld32(tmem + lane_base + Lay::t_w + 32 * hh, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= gr[32 * hh + i];
          st_chunks<4>(kq + (hh >> 1) * 16384, row_t, 4 * (hh & 1), v);
        }
      }
      tc_fence_before();
      fence_proxy_async();
      named_sync(kBarProd, kProd);
      if (t == 0) mbar_arrive(full + s);
      return true;
    };

    // Per chunk n: back1(n), then the next chunk's prologue and MMA1 while
    // MMA2(n) runs, then back2(n).
    if (nch > 0 && !front(0)) failed = true;
    for (int n = 0; n < nch && !failed; ++n) {
      if (!back1(n) || (n + 1 < nch && !front(n + 1)) || !back2(n))
        failed = true;
    }
    if (failed && t == 0) {
      *abort_flag = 1;
      atomicExch(&g_fused_timeout, 1);
      if (in_flight) mbar_wait(bar_in, ph_in, 100000000ull);
      if (v_pending) mbar_wait(bar_v, ph_v, 100000000ull);
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
    uint32_t ph_cm = 0;

    for (int n = 0; n < nch; ++n) {
      const int s = n & 1, use = n >> 1;
      const int tok0 = start + n * kC;
      const int L = min(kC, end - tok0);
      uint8_t* kq = sm + Lay::kq + s * Lay::kq_stride;
      uint8_t* kb = sm + Lay::kb + s * 16384;
      uint8_t* pp = sm + Lay::pp + s * 8192;
      bool ok = wait_or_abort<true>(full + s, use & 1, abort_flag);
      if (named_sync_or(kBarCons, kCons, !ok)) { failed = true; break; }
      tc_fence_after();

      // ---- MMA3: [W; Qt] . S
      if (c == 0) {
        const uint32_t idesc = idesc_bf16(128, 64, false, true);
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks)
          mma_bf16(tmem + Lay::t_d3,
                   desc_sw128(smem_u32(kq) + (ks >> 2) * 16384 + (ks & 3) * 32,
                              16, 1024),
                   desc_sw128(smem_u32(sop) + ks * 2048, 8192, 1024), idesc,
                   ks > 0);
        mma_commit(bar_cm);
      }
      ok = wait_or_abort<false>(bar_cm, ph_cm, abort_flag);
      ph_cm ^= 1;
      if (named_sync_or(kBarCons, kCons, !ok)) { failed = true; break; }
      tc_fence_after();

      // ---- Delta = U - W S (rows 0-63)
      if (c < 64) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          float uu[32], ws[32];
          tmem_ld32(tmem + lane_base + Lay::t_u0 + 64 * s + 32 * hf, uu);
          tmem_ld32(tmem + lane_base + Lay::t_d3 + 32 * hf, ws);
#pragma unroll
          for (int i = 0; i < 32; ++i) uu[i] -= ws[i];
          st_chunks<4>(dop, c, 4 * hf, uu);
        }
      }
      const float gamma = owns_state ? gcs[s * GCF + c] : 1.f;
      if (owns_state && gcs[s * GCF + 2 * DK] != 0.f) {
        // S_C = e^(g_C - rho) (e^rho S_0 + Kb^T Delta): pre-scale the state
        const float er = gcs[s * GCF + DK + c];
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
          mma_bf16(tmem + Lay::t_d3,
                   desc_sw128(smem_u32(pp) - 8192 + ks * 32, 16, 1024), bd, i5,
                   1u);
        }
        mma_commit(bar_cm);
      }
      ok = wait_or_abort<false>(bar_cm, ph_cm, abort_flag);
      ph_cm ^= 1;
      if (named_sync_or(kBarCons, kCons, !ok)) { failed = true; break; }
      tc_fence_after();
      if (c == 0) mbar_arrive(empty + s);  // slot s (and U slot s) consumed

      // ---- outputs (rows 64-127) and the state rescale by exp(g_C)
      if (c >= 64) {
        const int r = c - 64;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          float o[32];
          tmem_ld32(tmem + lane_base + Lay::t_d3 + 32 * hf, o);
          if (r < L) {
            uint4* dst = reinterpret_cast<uint4*>(
                p.out + ((size_t)(tok0 + r) * p.H + h) * p.dv + j0 + 32 * hf);
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
      if (owns_state) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          float v[32];
          tmem_ld32(tmem + lane_base + Lay::t_s + 32 * hf, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= gamma;
          tmem_st32(tmem + lane_base + Lay::t_s + 32 * hf, v);
          st_chunks<4>(sop, c, 4 * hf, v);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      fence_proxy_async();
      named_sync(kBarCons, kCons);
    }
    if (failed) {
      *abort_flag = 1;
      if (c == 0) atomicExch(&g_fused_timeout, 1);
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
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// Host side: tensor maps for q, k, v and the launch, one CTA per (sequence,
// head, 64-column d_v tile).
template <int DK, int GATE>
cudaError_t run_ws(const ChunkArgs& a, const int32_t* order,
                   cudaStream_t stream) {
  using Lay = WsLayout<DK>;
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
  p.n_tiles = a.dv / kDvt;
  const size_t smem = Lay::bytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(
      fused_ws_kernel<DK, GATE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
      (int)smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)a.n_seqs * a.H * p.n_tiles;
  fused_ws_kernel<DK, GATE><<<grid, kThreads, smem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

inline cudaError_t launch_fused_ws(const ChunkArgs& a, const int32_t* order,
                                   cudaStream_t stream) {
  if (a.gate == kGateHead)
    return a.dk == 128 ? run_ws<128, kGateHead>(a, order, stream)
                       : run_ws<64, kGateHead>(a, order, stream);
  if (a.gate == kGateNone)
    return a.dk == 128 ? run_ws<128, kGateNone>(a, order, stream)
                       : run_ws<64, kGateNone>(a, order, stream);
  return a.dk == 128 ? run_ws<128, kGateChannel>(a, order, stream)
                     : run_ws<64, kGateChannel>(a, order, stream);
}

}  // namespace ws
}  // namespace kda
