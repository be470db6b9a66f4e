// Token-by-token KDA step (decode): streams each head's fp32 state once.
//
// Per (sequence, head) and token t (state S is d_k x d_v, rows = key channels):
//   S' = Diag(exp(l_t)) S ;  e = S'^T k_t ;  delta = beta_t (v_t - e)
//   S  = S' + k_t delta^T ;  o_t = S^T q_t = S'^T q_t + delta (k_t . q_t)
// ("The fourth layer remembers", section "What each kind of layer keeps": a
// fixed d_k x d_v matrix per head and constant work per decoded token; the
// update itself is the delta rule with a per-key-channel decay, "Kimi Delta
// Attention", akshathtiwari.co.in.)
//
// Work split: one CTA per (sequence, head).  The state is HBM-bound (two
// passes of 4 * d_k * d_v bytes per head per call against 7 d_k d_v flops), so
// the kernel is laid out for bandwidth: thread (row group rg, column group cg)
// keeps rows rg*R .. rg*R+R-1, columns 4cg .. 4cg+3 of S in registers, a warp
// covers whole 512-byte rows (fully coalesced 128-bit loads and stores), and
// every thread issues all of its state loads before it touches them.  The
// column sums over d_k are a register partial per thread, then one pass over
// the 8 row groups in shared memory.  With T > 1 the state stays in registers
// across tokens and is written once at the end.  The gate may also be one
// value per head (Gated DeltaNet) or absent (alpha = 1, DeltaNet), and an
// optional prologue normalises q and k and turns gate logits into
// log(alpha) = scale * logsigmoid(x) on the fly.
#include "kda_common.cuh"
#include "kda_internal.h"

namespace kda {

namespace {

constexpr int kRowGroups = 8;

// PLAIN: per-channel gate and no prologue (the common case, kept free of the
// per-token selects and extra reductions of the general path).
template <int DK, int DV, typename IO, bool PLAIN>
__global__ void __launch_bounds__((DV / 4) * kRowGroups)
    recurrent_kernel(const IO* __restrict__ q, const IO* __restrict__ k,
                     const IO* __restrict__ v,
                     const float* __restrict__ log_alpha,
                     const float* __restrict__ beta, float* __restrict__ state,
                     IO* __restrict__ out, int T, int H, int gate,
                     Prologue pro) {
  constexpr int CG = DV / 4;          // float4 column groups
  constexpr int R = DK / kRowGroups;  // rows per thread
  constexpr int NT = CG * kRowGroups;
  const int tid = threadIdx.x;
  const int cg = tid % CG, rg = tid / CG;
  const int bh = blockIdx.x;  // sequence * H + head
  const int b = bh / H, h = bh % H;

  __shared__ float s_k[DK], s_q[DK], s_a[DK], s_v[DV];
  __shared__ float4 s_e[kRowGroups][CG], s_p[kRowGroups][CG];
  __shared__ float s_kq, s_beta, s_invk, s_invq;

  float4* st = reinterpret_cast<float4*>(state + (size_t)bh * DK * DV);
  float4 s[R];
#pragma unroll
  for (int i = 0; i < R; ++i) s[i] = __ldcs(st + (rg * R + i) * CG + cg);

  for (int t = 0; t < T; ++t) {
    const size_t tok = (size_t)b * T + t;
    const size_t ok = (tok * H + h) * DK, ov = (tok * H + h) * DV;
    for (int c = tid; c < DK; c += NT) {
      s_k[c] = to_f32(k[ok + c]);
      s_q[c] = to_f32(q[ok + c]);
      if (PLAIN) {
        s_a[c] = __expf(log_alpha[ok + c]);
      } else {
        float l = gate == kGateChannel ? log_alpha[ok + c]
                  : gate == kGateHead  ? log_alpha[tok * H + h]
                                       : 0.f;
        if (pro.gate_logits && gate != kGateNone)  // scale * logsigmoid(l)
          // log1p(e) as log(1 + e), e <= 1: under 6e-8 apart
          l = pro.gate_scale * (fminf(l, 0.f) - __logf(1.f + __expf(-fabsf(l))));
        s_a[c] = __expf(l);
      }
    }
    for (int j = tid; j < DV; j += NT) s_v[j] = to_f32(v[ov + j]);
    if (tid < 32) {  // k . q (and, with the prologue, the norms), one warp
      float kq = 0.f, kk = 0.f, qq = 0.f;
      for (int c = tid; c < DK; c += 32) {
        const float kc = to_f32(k[ok + c]), qc = to_f32(q[ok + c]);
        kq += kc * qc;
        if (!PLAIN) {
          kk += kc * kc;
          qq += qc * qc;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        kq += __shfl_xor_sync(0xffffffffu, kq, o);
        if (!PLAIN) {
          kk += __shfl_xor_sync(0xffffffffu, kk, o);
          qq += __shfl_xor_sync(0xffffffffu, qq, o);
        }
      }
      if (tid == 0) {
        const float ik = !PLAIN && pro.norm_qk ? rsqrtf(kk) : 1.f;
        const float iq =
            (!PLAIN && pro.norm_qk ? rsqrtf(qq) : 1.f) * (PLAIN ? 1.f : pro.q_scale);
        s_invk = ik;
        s_invq = iq;
        s_kq = kq * ik * iq;
        s_beta = beta[tok * H + h];
      }
    }
    __syncthreads();
    const float invk = PLAIN ? 1.f : s_invk, invq = PLAIN ? 1.f : s_invq;

    float4 e = make_float4(0.f, 0.f, 0.f, 0.f), p = e;
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const int r = rg * R + i;
      const float a = s_a[r], kr = s_k[r] * invk, qr = s_q[r] * invq;
      s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
      e.x += s[i].x * kr; e.y += s[i].y * kr; e.z += s[i].z * kr; e.w += s[i].w * kr;
      p.x += s[i].x * qr; p.y += s[i].y * qr; p.z += s[i].z * qr; p.w += s[i].w * qr;
    }
    s_e[rg][cg] = e;
    s_p[rg][cg] = p;
    __syncthreads();
    float4 et = s_e[0][cg], pt = s_p[0][cg];
#pragma unroll
    for (int g = 1; g < kRowGroups; ++g) {
      const float4 a = s_e[g][cg], c = s_p[g][cg];
      et.x += a.x; et.y += a.y; et.z += a.z; et.w += a.w;
      pt.x += c.x; pt.y += c.y; pt.z += c.z; pt.w += c.w;
    }
    const float bt = s_beta, kq = s_kq;
    float4 d;
    d.x = bt * (s_v[4 * cg + 0] - et.x);
    d.y = bt * (s_v[4 * cg + 1] - et.y);
    d.z = bt * (s_v[4 * cg + 2] - et.z);
    d.w = bt * (s_v[4 * cg + 3] - et.w);
    if (rg == 0) {
      IO* o = out + ov + 4 * cg;
      o[0] = from_f32<IO>(pt.x + d.x * kq);
      o[1] = from_f32<IO>(pt.y + d.y * kq);
      o[2] = from_f32<IO>(pt.z + d.z * kq);
      o[3] = from_f32<IO>(pt.w + d.w * kq);
    }
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const float kr = s_k[rg * R + i] * invk;
      s[i].x += kr * d.x; s[i].y += kr * d.y; s[i].z += kr * d.z; s[i].w += kr * d.w;
    }
    __syncthreads();  // shared vectors are rewritten by the next token
  }
#pragma unroll
  for (int i = 0; i < R; ++i) __stcs(st + (rg * R + i) * CG + cg, s[i]);
}

template <int DK, int DV, typename IO>
cudaError_t launch_dkdv(const RecurrentArgs& a, cudaStream_t stream) {
  constexpr int NT = (DV / 4) * kRowGroups;
  const unsigned grid = (unsigned)a.B * (unsigned)a.H;
  const bool plain = a.gate == kGateChannel && !a.pro.norm_qk &&
                     a.pro.q_scale == 1.f && !a.pro.gate_logits;
  if (plain)
    recurrent_kernel<DK, DV, IO, true><<<grid, NT, 0, stream>>>(
        static_cast<const IO*>(a.q), static_cast<const IO*>(a.k),
        static_cast<const IO*>(a.v), a.log_alpha, a.beta, a.state,
        static_cast<IO*>(a.out), a.T, a.H, a.gate, a.pro);
  else
    recurrent_kernel<DK, DV, IO, false><<<grid, NT, 0, stream>>>(
        static_cast<const IO*>(a.q), static_cast<const IO*>(a.k),
        static_cast<const IO*>(a.v), a.log_alpha, a.beta, a.state,
        static_cast<IO*>(a.out), a.T, a.H, a.gate, a.pro);
  return cudaGetLastError();
}

template <typename IO>
cudaError_t launch_io(const RecurrentArgs& a, cudaStream_t stream) {
#define KDA_DEC_CASE(DK_, DV_) \
  if (a.dk == DK_ && a.dv == DV_) return launch_dkdv<DK_, DV_, IO>(a, stream);
  KDA_DEC_CASE(32, 32) KDA_DEC_CASE(32, 64) KDA_DEC_CASE(32, 128)
  KDA_DEC_CASE(64, 32) KDA_DEC_CASE(64, 64) KDA_DEC_CASE(64, 128)
  KDA_DEC_CASE(128, 32) KDA_DEC_CASE(128, 64) KDA_DEC_CASE(128, 128)
#undef KDA_DEC_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_recurrent(const RecurrentArgs& a, cudaStream_t stream) {
  if (a.B == 0 || a.H == 0) return cudaSuccess;
  return a.bf16 ? launch_io<__nv_bfloat16>(a, stream)
                : launch_io<float>(a, stream);
}

}  // namespace kda
