// (I + A)^-1 of a strictly-lower 64 x 64 fp32 matrix in shared memory on 256
// threads, with the block couplings on the tensor cores: warp-level tf32
// products (mma.sync m16n8k8, fp32 accumulate).  Used by the fused bf16
// prefill producers, whose T' is rounded to bf16 afterwards; the fp32 paths
// keep the all-fp32 version in kda_inverse.cuh.
//
// Blocks of 16: with L = I + A split into 16 x 16 blocks L_ij and X = L^-1,
//   X_ii = L_ii^-1                 forward substitution, one column a thread;
//   X_10 = -X_11 A_10 X_00, X_32 = -X_33 A_32 X_22    (the 32 x 32 diagonal
//                                                       blocks are complete);
//   X_(32..63, 0..31) = -X_(32..63, 32..63) A_(32..63, 0..31) X_(0..31, 0..31).
// This is the block form of [L11 0; L21 L22]^-1 = [X11 0; -X22 L21 X11 X22]
// applied at 16 and then at 32.
#pragma once

#include <stdint.h>

#include "kda_inverse.cuh"

namespace kda {
namespace ws {

__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

// d (16 x 8 accumulator fragment) += A (16 x 8 KS, row stride lda) *
// B (8 KS x 8, row stride ldb), one warp.  Fragment layouts of
// mma.m16n8k8.tf32: with g = lane / 4 and q = lane % 4, A holds (g, q),
// (g + 8, q), (g, q + 4), (g + 8, q + 4); B holds (q, g), (q + 4, g); the
// accumulator holds (g, 2q), (g, 2q + 1), (g + 8, 2q), (g + 8, 2q + 1).
template <int KS>
__device__ __forceinline__ void warp_mm_tf32(const float* A, int lda,
                                             const float* B, int ldb, float* d,
                                             int lane) {
  const int g = lane >> 2, q = lane & 3;
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const float* a = A + 8 * ks;
    const float* b = B + 8 * ks * ldb;
    const uint32_t a0 = to_tf32(a[g * lda + q]);
    const uint32_t a1 = to_tf32(a[(g + 8) * lda + q]);
    const uint32_t a2 = to_tf32(a[g * lda + q + 4]);
    const uint32_t a3 = to_tf32(a[(g + 8) * lda + q + 4]);
    const uint32_t b0 = to_tf32(b[q * ldb + g]);
    const uint32_t b1 = to_tf32(b[(q + 4) * ldb + g]);
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}

// Store a 16 x 8 accumulator fragment, times sgn, at C (row stride ldc).
__device__ __forceinline__ void warp_st_frag(float* C, int ldc, const float* d,
                                             int lane, float sgn) {
  const int g = lane >> 2, q = lane & 3;
  *reinterpret_cast<float2*>(C + g * ldc + 2 * q) =
      make_float2(sgn * d[0], sgn * d[1]);
  *reinterpret_cast<float2*>(C + (g + 8) * ldc + 2 * q) =
      make_float2(sgn * d[2], sgn * d[3]);
}

// X = (I + A)^-1 for the strictly-lower A (row stride kFS; its upper 32 x 32
// block, rows 0-31 and columns 32-63, is used as scratch and left
// unspecified).  X's entries above the 16 x 16 diagonal blocks must be zero
// on entry and stay zero.  `M` is 512 floats of scratch.  256 threads.
__device__ __forceinline__ void invert_unit_lower_tc(float* A, float* X,
                                                     float* M, int t) {
  const int warp = t >> 5, lane = t & 31;
  if (t < 64) {  // X_bb: column j of block b, right-looking substitution
    const int o = (t >> 4) * 16, j = t & 15;
    float s[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) s[r] = r == j ? 1.f : 0.f;
#pragma unroll
    for (int i = 0; i < 15; ++i) {
      const float xi = s[i];  // final: every row above i has been applied
#pragma unroll
      for (int r = i + 1; r < 16; ++r)
        s[r] -= A[(o + r) * kFS + o + i] * xi;
    }
#pragma unroll
    for (int r = 0; r < 16; ++r) X[(o + r) * kFS + o + j] = s[r];
  }
  inv_sync();
  if (warp < 4) {  // X_10 and X_32, eight columns a warp
    const int b = warp >> 1, nt = warp & 1;
    const int bi = 2 * b + 1, bj = 2 * b;
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    warp_mm_tf32<2>(A + 16 * bi * kFS + 16 * bj, kFS,
                    X + 16 * bj * kFS + 16 * bj + 8 * nt, kFS, d, lane);
    float* Mw = M + warp * 128;  // 16 x 8, row stride 8
    warp_st_frag(Mw, 8, d, lane, 1.f);
    __syncwarp();
    float e[4] = {0.f, 0.f, 0.f, 0.f};
    warp_mm_tf32<2>(X + 16 * bi * kFS + 16 * bi, kFS, Mw, 8, e, lane);
    warp_st_frag(X + 16 * bi * kFS + 16 * bj + 8 * nt, kFS, e, lane, -1.f);
  }
  inv_sync();
  // the 32 x 32 coupling: P = A_(32.., 0..31) X_(0..31, 0..31) into the
  // unused upper block of A, then X_(32.., 0..31) = -X_(32.., 32..) P
  const int mt = warp >> 2, nt = warp & 3;
  float* P = A + 32;  // rows 0-31, columns 32-63 of A
  {
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    warp_mm_tf32<4>(A + (32 + 16 * mt) * kFS, kFS, X + 8 * nt, kFS, d, lane);
    warp_st_frag(P + 16 * mt * kFS + 8 * nt, kFS, d, lane, 1.f);
  }
  inv_sync();
  {
    float e[4] = {0.f, 0.f, 0.f, 0.f};
    warp_mm_tf32<4>(X + (32 + 16 * mt) * kFS + 32, kFS, P + 8 * nt, kFS, e,
                    lane);
    warp_st_frag(X + (32 + 16 * mt) * kFS + 8 * nt, kFS, e, lane, -1.f);
  }
  inv_sync();
}

}  // namespace ws
}  // namespace kda
