// Reverse state-gradient chain of the chunkwise backward pass on the tensor
// cores (tcgen05 kind::tf32, fp32 operands in 128-byte-swizzled shared
// memory, fp32 accumulators in TMEM).  Included by kda_fused_sm100.cu, whose
// tensor-map encoder and device timeout flag it shares.
//
// Per chunk, walking each sequence's chunks from last to first, with dS the
// gradient of the state leaving the chunk (the chain rule applied to the
// chunkwise form S_C = Diag(gam)(S_0 + Kb^T Delta), Delta = U - W S_0; "You
// Could Have Come Up with Kimi Delta Attention", daily.dev, Summary):
//   gam * d gam = rowsum(S_next * dS)      (S_next = Diag(gam)(S_0 + Kb^T
//                                           Delta), the next start state)
//   G      = Diag(gam) dS
//   dDelta = Kb G + P^T dO                 (MMA 1: M = 64 tokens, K = d_k)
//   dS    <- G + Qt^T dO - W^T dDelta      (MMA 2: M = d_k, K = 64 tokens)
// G, dDelta and the gam * d gam partials go to the workspace for the batched
// products that follow; the last dS is the initial-state gradient.
//
// One CTA of 256 threads per (sequence, head, 64-column d_v tile); thread c
// owns TMEM lane c % 128 and 32 columns 32 (c / 128) .. + 31.  dS stays in
// TMEM from the first step to the last.  Kb and W^T (written transposed by
// the backward's prep kernel) arrive by TMA one chunk ahead into two
// buffers; G and -dDelta are written by the epilogues straight into the
// K-major B operands of the two MMAs.  tf32 operands need K-major layouts on
// both sides, hence the transposed copy of W.
namespace kda {
namespace bwdtc {

using ws::named_sync_or;
using ws::tmem_st32;
using ws::tmem_wait_st;
using ws::wait_or_abort;

constexpr int kC = 64;        // chunk length
constexpr int kTile = 64;     // d_v columns per CTA
constexpr int kThreads = 256;
constexpr int kBarAll = 1;

__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// fp32 element (row, c) of a 128-byte-swizzled panel whose rows hold 32 fp32
// (K-major: rows along M or N, 32 consecutive k per row).
__device__ __forceinline__ uint32_t swz32(int row, int c) {
  return (uint32_t)(row * 128 + (((c >> 2) ^ (row & 7)) << 4) + ((c & 3) << 2));
}

__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap,
                                            uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::"
      "bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(sm100::smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1),
      "r"(sm100::smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t adesc,
                                         uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

struct Params {
  const float* qdo;      // Qt^T dO      [chunks, H, dk, dv]
  const float* pdo;      // P^T dO       [tokens, H, dv]
  const float* s;        // start states [chunks, H, dk, dv]
  const float* fin;      // final states [n_seqs, H, dk, dv]
  const float* gam;      // exp(g_C)     [chunks, H, dk]
  const float* d_final;  // [n_seqs, H, dk, dv] or null (zero)
  float* gst;            // G            [chunks, H, dk, dv]
  float* dd;             // dDelta       [tokens, H, dv]
  float* dgam;           // partials     [chunks, H, dv / 32, dk]
  float* d_init;         // [n_seqs, H, dk, dv] or null
  const int32_t* cu;
  const int32_t* chunk_off;
  int n_seqs, T, H, dv;
};

template <int DK>
struct Layout {
  // Kb: DK / 32 panels of 64 token rows x 128 B, plus one more panel of
  // padding, since the M = 128 product reads 128 rows from each panel start
  static constexpr uint32_t kb_bytes = (DK / 32 + 1) * 8192;
  // W^T: two panels (tokens 0-31, 32-63) of 128 rows (d_k, padded) x 128 B
  static constexpr uint32_t wt_bytes = 2 * 16384;
  static constexpr uint32_t kb = 0;                       // two buffers
  static constexpr uint32_t wt = kb + 2 * kb_bytes;       // two buffers
  static constexpr uint32_t gop = wt + 2 * wt_bytes;      // G: 64 rows (j) x DK
  static constexpr uint32_t dop = gop + (DK / 32) * 8192; // -dDelta: 64 x 64
  static constexpr uint32_t misc = dop + 2 * 8192;
  static constexpr uint32_t bytes = misc + 256;
  static constexpr uint32_t kb_tx = (DK / 32) * 8192;
  static constexpr uint32_t wt_tx = 2 * DK * 128;
  static constexpr uint32_t t_ds = 0, t_dd = 64;  // TMEM columns
  static_assert(bytes + 1024 <= 232448, "shared memory");
};

template <int DK>
__global__ void __launch_bounds__(kThreads, 1)
    rev_chain_kernel(const __grid_constant__ CUtensorMap tm_kb,
                     const __grid_constant__ CUtensorMap tm_wt,
                     const Params p) {
  using namespace sm100;
  using Lay = Layout<DK>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* gop = sm + Lay::gop;
  uint8_t* dop = sm + Lay::dop;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::misc);
  uint64_t* kb_full = bars;      // two
  uint64_t* wt_full = bars + 2;  // two
  uint64_t* bar_mma = bars + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 6);

  const int c = threadIdx.x, warp = c >> 5;
  const int row = c & 127, half = c >> 7;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  const int n_tiles = p.dv / kTile;
  const int tile = blockIdx.x % n_tiles;
  const int h = (blockIdx.x / n_tiles) % p.H;
  const int seq = blockIdx.x / (n_tiles * p.H);
  const int j0 = tile * kTile + 32 * half;  // this thread's first column
  int start, end;
  seq_range(p.cu, seq, p.T, &start, &end);
  const int nch = (end - start + kC - 1) / kC;
  const int cid0 = p.cu ? p.chunk_off[seq] : seq * ((p.T + kC - 1) / kC);
  const bool owns_state = row < DK;
  const size_t sbase = ((size_t)seq * p.H + h) * DK * p.dv;

  if (c == 0) {
    prefetch_tmap(&tm_kb);
    prefetch_tmap(&tm_wt);
    for (int b = 0; b < 2; ++b) {
      mbar_init(kb_full + b, 1);
      mbar_init(wt_full + b, 1);
    }
    mbar_init(bar_mma, 1);
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

  // step s handles chunk nch - 1 - s; its operands sit in buffer s & 1
  auto issue = [&](int s) {
    const int n = nch - 1 - s;
    const int b = s & 1;
    uint8_t* kb = sm + Lay::kb + b * Lay::kb_bytes;
    uint8_t* wt = sm + Lay::wt + b * Lay::wt_bytes;
    mbar_arrive_expect_tx(kb_full + b, Lay::kb_tx);
    for (int q = 0; q < DK / 32; ++q)
      tma_load_3d(kb + q * 8192, &tm_kb, kb_full + b, 32 * q, h,
                  start + n * kC);
    mbar_arrive_expect_tx(wt_full + b, Lay::wt_tx);
    const int wrow = (int)(((size_t)(cid0 + n) * p.H + h) * DK);
    for (int q = 0; q < 2; ++q)
      tma_load_2d(wt + q * 16384, &tm_wt, wt_full + b, 32 * q, wrow);
  };
  int issued = 0;
  if (c == 0) {
    for (int s = 0; s < 2 && s < nch; ++s) issue(s);
  }
  issued = nch < 2 ? nch : 2;

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

  // Per-thread operands of one step's epilogues, loaded a phase ahead of
  // their use: Qt^T dO, the next start state and gam for G (step s + 1's
  // are fetched during step s's second product), P^T dO for dDelta (fetched
  // while the first product runs).
  float qd[32], sn[32], gmv = 0.f;
  auto load_state_operands = [&](int s_) {
    const int n = nch - 1 - s_, cid = cid0 + n;
    const size_t cbase = ((size_t)cid * p.H + h) * DK * p.dv;
    const float4* q4 = reinterpret_cast<const float4*>(
        p.qdo + cbase + (size_t)row * p.dv + j0);
    const float* snx = n + 1 < nch ? p.s + cbase + (size_t)p.H * DK * p.dv
                                   : p.fin + sbase;
    const float4* s4 =
        reinterpret_cast<const float4*>(snx + (size_t)row * p.dv + j0);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 x = q4[i], y = s4[i];
      qd[4 * i] = x.x; qd[4 * i + 1] = x.y; qd[4 * i + 2] = x.z;
      qd[4 * i + 3] = x.w;
      sn[4 * i] = y.x; sn[4 * i + 1] = y.y; sn[4 * i + 2] = y.z;
      sn[4 * i + 3] = y.w;
    }
    gmv = p.gam[((size_t)cid * p.H + h) * DK + row];
  };
  if (owns_state && nch > 0) load_state_operands(0);

  uint32_t ph_mma = 0;
  bool failed = false;
  int s = 0;
  for (; s < nch; ++s) {
    const int n = nch - 1 - s, b = s & 1;
    const int cid = cid0 + n, tok0 = start + n * kC;
    const int L = min(kC, end - tok0);
    const size_t cbase = ((size_t)cid * p.H + h) * DK * p.dv;

    // ---- G = Diag(gam) dS, gam * d gam; TMEM dS <- G + Qt^T dO
    if (owns_state) {
      float v[32];
      tmem_ld32(tmem + lane_base + Lay::t_ds + 32 * half, v);
      float part = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) part += sn[i] * v[i];
      p.dgam[(((size_t)cid * p.H + h) * (p.dv / 32) + j0 / 32) * DK + row] =
          part;
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= gmv;
      float4* g4 = reinterpret_cast<float4*>(p.gst + cbase +
                                             (size_t)row * p.dv + j0);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        g4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      // B operand of product 1: element (k = row, n = column), K-major
      // panels of 32 rows (d_k) each
      uint8_t* panel = gop + (row >> 5) * 8192;
#pragma unroll
      for (int i = 0; i < 32; ++i)
        *reinterpret_cast<float*>(panel + swz32(32 * half + i, row & 31)) = v[i];
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] += qd[i];
      tmem_st32(tmem + lane_base + Lay::t_ds + 32 * half, v);
      tmem_wait_st();
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();

    // ---- product 1: D = Kb G (rows 0-63 meaningful)
    bool ok = true;
    if (c == 0) {
      tc_fence_after();
      ok = wait_or_abort<false>(kb_full + b, (uint32_t)(s >> 1) & 1u,
                                abort_flag);
      if (ok) {
        const uint8_t* kb = sm + Lay::kb + b * Lay::kb_bytes;
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
      } else {
        *abort_flag = 1;
      }
    }
    float pd[32];
    const bool in = row < L;
    if (row < kC) {
      const float4* p4 = reinterpret_cast<const float4*>(
          p.pdo + ((size_t)(tok0 + (in ? row : 0)) * p.H + h) * p.dv + j0);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 x = in ? p4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        pd[4 * i] = x.x; pd[4 * i + 1] = x.y; pd[4 * i + 2] = x.z;
        pd[4 * i + 3] = x.w;
      }
    }
    ok = ok && wait_or_abort<false>(bar_mma, ph_mma, abort_flag);
    ph_mma ^= 1;
    if (named_sync_or(kBarAll, kThreads, !ok)) {
      failed = true;
      break;
    }
    tc_fence_after();

    // ---- dDelta = Kb G + P^T dO (token rows 0-63; zero past the chunk)
    if (row < kC) {
      float d[32];
      tmem_ld32(tmem + lane_base + Lay::t_dd + 32 * half, d);
#pragma unroll
      for (int i = 0; i < 32; ++i) d[i] = in ? d[i] + pd[i] : 0.f;
      if (in) {
        float4* d4 = reinterpret_cast<float4*>(
            p.dd + ((size_t)(tok0 + row) * p.H + h) * p.dv + j0);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          d4[i] = make_float4(d[4 * i], d[4 * i + 1], d[4 * i + 2], d[4 * i + 3]);
      }
      // B operand of product 2, negated: element (k = token, n = column)
      uint8_t* panel = dop + (row >> 5) * 8192;
#pragma unroll
      for (int i = 0; i < 32; ++i)
        *reinterpret_cast<float*>(panel + swz32(32 * half + i, row & 31)) = -d[i];
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();

    // ---- product 2: dS += W^T (-dDelta)
    if (c == 0) {
      tc_fence_after();
      ok = wait_or_abort<false>(wt_full + b, (uint32_t)(s >> 1) & 1u,
                                abort_flag);
      if (ok) {
        const uint8_t* wt = sm + Lay::wt + b * Lay::wt_bytes;
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
      } else {
        *abort_flag = 1;
      }
    }
    if (owns_state && s + 1 < nch) load_state_operands(s + 1);
    ok = ok && wait_or_abort<false>(bar_mma, ph_mma, abort_flag);
    ph_mma ^= 1;
    if (named_sync_or(kBarAll, kThreads, !ok)) {
      failed = true;
      break;
    }
    tc_fence_after();
    // both buffers b are free again: the operands of step s + 2
    if (s + 2 < nch) {
      if (c == 0) issue(s + 2);
      issued = s + 3;
    }
  }
  if (failed) {
    if (c == 0) {
      atomicExch(&g_fused_timeout, 1);
      for (int m = s; m < issued; ++m) {  // copies still in flight
        mbar_wait(kb_full + (m & 1), (uint32_t)(m >> 1) & 1u, 100000000ull);
        mbar_wait(wt_full + (m & 1), (uint32_t)(m >> 1) & 1u, 100000000ull);
      }
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
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

}  // namespace bwdtc
}  // namespace kda
