// Diagnostic: one 128 x N x K bf16 tensor-core product through the same
// shared-memory layouts, descriptors and TMEM read-back the fused prefill
// kernel uses, so the operand encodings can be checked in isolation against a
// library matmul.
#include "../../include/kda.h"
#include "sm100_ptx.cuh"

namespace kda {
namespace {

using namespace sm100;

__global__ void __launch_bounds__(128)
    umma_probe_kernel(int a_mn, int b_mn, int N, int K, int panel_rows,
                      const __nv_bfloat16* __restrict__ A,
                      const __nv_bfloat16* __restrict__ B,
                      float* __restrict__ D) {
  extern __shared__ __align__(1024) uint8_t sm_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int M = 128;
  // A: K-major -> K/64 panels of 128 rows; MN-major -> 2 panels of
  // panel_rows K-rows.  B likewise with N.
  const uint32_t a_panel = a_mn ? panel_rows * 128 : M * 128;
  const uint32_t b_panel = b_mn ? panel_rows * 128 : N * 128;
  const uint32_t a_bytes = a_mn ? 2 * a_panel : (K / 64) * a_panel;
  uint8_t* sA = base;
  uint8_t* sB = base + ((a_bytes + 1023) & ~1023u);
  uint8_t* tail = sB + (b_mn ? (N / 64) * b_panel : (K / 64) * b_panel);
  uint64_t* bar = reinterpret_cast<uint64_t*>(tail);
  uint32_t* tbase = reinterpret_cast<uint32_t*>(tail + 8);

  for (int i = tid; i < M * K; i += 128) {  // logical A[m][k]
    const int m = i / K, kk = i % K;
    const __nv_bfloat16 x = A[a_mn ? (size_t)kk * M + m : (size_t)m * K + kk];
    uint8_t* p = a_mn ? sA + (m / 64) * a_panel + sw128_off(kk, m % 64)
                      : sA + (kk / 64) * a_panel + sw128_off(m, kk % 64);
    *reinterpret_cast<__nv_bfloat16*>(p) = x;
  }
  for (int i = tid; i < N * K; i += 128) {  // logical B[k][n]
    const int kk = i / N, n = i % N;
    const __nv_bfloat16 x = B[b_mn ? (size_t)kk * N + n : (size_t)n * K + kk];
    uint8_t* p = b_mn ? sB + (n / 64) * b_panel + sw128_off(kk, n % 64)
                      : sB + (kk / 64) * b_panel + sw128_off(n, kk % 64);
    *reinterpret_cast<__nv_bfloat16*>(p) = x;
  }
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (tid < 32) {
    tmem_alloc(tbase, 256);
    tmem_relinquish();
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tbase;
  if (tid == 0) {
    const uint32_t idesc = idesc_bf16(M, N, a_mn != 0, b_mn != 0);
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
    for (int ks = 0; ks < K / 16; ++ks) {
      const uint64_t ad =
          a_mn ? desc_sw128(a0 + ks * 2048, a_panel, 1024)
               : desc_sw128(a0 + (ks / 4) * a_panel + (ks % 4) * 32, 16, 1024);
      const uint64_t bd =
          b_mn ? desc_sw128(b0 + ks * 2048, b_panel, 1024)
               : desc_sw128(b0 + (ks / 4) * b_panel + (ks % 4) * 32, 16, 1024);
      mma_bf16(tmem, ad, bd, idesc, ks > 0 ? 1u : 0u);
    }
    mma_commit(bar);
  }
  const bool ok = mbar_wait(bar, 0);
  tc_fence_after();
  const int warp = tid / 32;
  for (int c = 0; c < N; c += 32) {
    float v[32];
    tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c, v);
    for (int j = 0; j < 32; ++j)
      D[(size_t)tid * N + c + j] = ok ? v[j] : __int_as_float(0x7fc00000);
  }
  tc_fence_before();
  __syncthreads();
  if (tid < 32) tmem_dealloc(tmem, 256);
}

}  // namespace
}  // namespace kda

extern "C" KDA_API kda_status kda_selftest_umma(int a_mn, int b_mn, int N,
                                                int K, int panel_rows,
                                                const void* A, const void* B,
                                                float* D, cudaStream_t stream) {
  if (!A || !B || !D) return KDA_ERR_INVALID_ARG;
  if ((N != 64 && N != 128) || (K != 64 && K != 128)) return KDA_ERR_UNSUPPORTED;
  if (panel_rows < K || panel_rows % 8 != 0 || panel_rows > 256)
    return KDA_ERR_INVALID_ARG;
  const size_t a_bytes = a_mn ? 2 * panel_rows * 128 : (K / 64) * 128 * 128;
  const size_t b_bytes = b_mn ? (N / 64) * panel_rows * 128 : (K / 64) * N * 128;
  const size_t smem = 1024 + ((a_bytes + 1023) & ~size_t(1023)) + b_bytes + 64;
  cudaError_t e = cudaFuncSetAttribute(
      kda::umma_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
      (int)smem);
  if (e == cudaSuccess) {
    kda::umma_probe_kernel<<<1, 128, smem, stream>>>(
        a_mn, b_mn, N, K, panel_rows, static_cast<const __nv_bfloat16*>(A),
        static_cast<const __nv_bfloat16*>(B), D);
    e = cudaGetLastError();
  }
  return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}
