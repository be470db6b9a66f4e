// (I + A)^-1 of a strictly-lower 64 x 64 fp32 matrix in shared memory, by
// recursive doubling on 256 threads; shared by the fused prefill producers,
// the four-stage forward and the backward pass.
#pragma once

namespace kda {
namespace ws {

constexpr int kFS = 68;  // fp32 row stride of the A / X tiles
constexpr int kBarInv = 1;    // named barrier used inside the inverse
constexpr int kInvThreads = 256;

__device__ __forceinline__ void inv_sync() {
  asm volatile("bar.sync %0, %1;" ::"r"(kBarInv), "r"(kInvThreads) : "memory");
}

// C = A B (or -A B) for 32 x 32 fp32 tiles in shared memory (leading
// dimensions in floats), on 256 threads: each thread accumulates a 4 x 4
// block of C over a quarter of K, the four quarters sit on lanes l, l ^ 8,
// l ^ 16, l ^ 24 and are summed with shuffles, and each of the four lanes
// then stores one row of the block.  Four 128-bit loads of A and four of B
// feed 64 FMAs, which keeps the shared-memory load bytes per FMA low.
template <bool NEG>
__device__ __forceinline__ void mm32_tiles(const float* Ab, int lda,
                                           const float* Bb, int ldb, float* Cb,
                                           int ldc, int t) {
  const int q = (t >> 3) & 3;
  const int tile = (t >> 5) * 8 + (t & 7);
  const int tr = tile >> 3, tc = tile & 7;
  float m[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) m[i][j] = 0.f;
#pragma unroll
  for (int kk = 0; kk < 8; kk += 4) {
    const int k4 = q * 8 + kk;
    float4 a[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      a[i] = *reinterpret_cast<const float4*>(Ab + (4 * tr + i) * lda + k4);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float4 x = *reinterpret_cast<const float4*>(Bb + (k4 + u) * ldb + 4 * tc);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float av = u == 0 ? a[i].x : u == 1 ? a[i].y : u == 2 ? a[i].z : a[i].w;
        m[i][0] += av * x.x; m[i][1] += av * x.y;
        m[i][2] += av * x.z; m[i][3] += av * x.w;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      m[i][j] += __shfl_xor_sync(0xffffffffu, m[i][j], 8);
      m[i][j] += __shfl_xor_sync(0xffffffffu, m[i][j], 16);
    }
  float4 w;
  w.x = q == 0 ? m[0][0] : q == 1 ? m[1][0] : q == 2 ? m[2][0] : m[3][0];
  w.y = q == 0 ? m[0][1] : q == 1 ? m[1][1] : q == 2 ? m[2][1] : m[3][1];
  w.z = q == 0 ? m[0][2] : q == 1 ? m[1][2] : q == 2 ? m[2][2] : m[3][2];
  w.w = q == 0 ? m[0][3] : q == 1 ? m[1][3] : q == 2 ? m[2][3] : m[3][3];
  if (NEG) {
    w.x = -w.x; w.y = -w.y; w.z = -w.z; w.w = -w.w;
  }
  *reinterpret_cast<float4*>(Cb + (4 * tr + q) * ldc + 4 * tc) = w;
}

// (I + A)^-1 of the strictly-lower 64 x 64 A (row stride kFS) into X by
// recursive doubling on unit-lower blocks,
//   [L11 0; L21 L22]^-1 = [X11 0; -X22 L21 X11  X22]:
// the four 16 x 16 diagonal blocks by forward substitution, then blocks
// (1,0) and (3,2), then the 32 x 32 coupling block (register-tiled products,
// mm32_tiles).  256 producer threads;
// X's strictly-upper part outside the diagonal blocks must be zero.
__device__ __forceinline__ void invert_unit_lower(const float* A, float* X,
                                                  float* M, int t) {
  if (t < 64) {
    const int o = (t >> 4) * 16, j = t & 15;
    float x[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float a[16];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        if (4 * q4 < r) {
          const float4 v =
              *reinterpret_cast<const float4*>(A + (o + r) * kFS + o + 4 * q4);
          a[4 * q4] = v.x; a[4 * q4 + 1] = v.y; a[4 * q4 + 2] = v.z;
          a[4 * q4 + 3] = v.w;
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
  inv_sync();
  {
    const int b = t >> 7, r = (t >> 3) & 15, c = (t & 7) * 2;
    const int bi = 2 * b + 1, bj = 2 * b;
    float m0 = 0.f, m1 = 0.f;
#pragma unroll
    for (int k = 0; k < 16; k += 4) {
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
    inv_sync();
    float y0 = 0.f, y1 = 0.f;
#pragma unroll
    for (int k = 0; k < 16; k += 4) {
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
  inv_sync();
  mm32_tiles<false>(A + 32 * kFS, kFS, X, kFS, M, 32, t);  // M = L21 X11
  inv_sync();
  mm32_tiles<true>(X + 32 * kFS + 32, kFS, M, 32, X + 32 * kFS, kFS, t);
  inv_sync();
}

}  // namespace ws
}  // namespace kda
