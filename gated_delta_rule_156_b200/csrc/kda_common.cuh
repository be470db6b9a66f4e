// Device helpers shared by the KDA kernels: io-dtype conversion and the
// mapping from a chunk id to its sequence and token range.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ int clampi(int x, int lo, int hi) {
  return x < lo ? lo : (x > hi ? hi : x);
}

// Token range [start, end) of sequence s.  Dense layout: s * T .. s * T + T.
// Packed layout: cu_seqlens[s] .. cu_seqlens[s + 1], clamped into [0, T] and
// forced non-decreasing so a malformed offset array can never send a kernel
// out of bounds.
__device__ __forceinline__ void seq_range(const int32_t* __restrict__ cu, int s,
                                          int T, int* start, int* end) {
  if (cu == nullptr) {
    *start = s * T;
    *end = s * T + T;
  } else {
    int a = clampi(cu[s], 0, T);
    int b = clampi(cu[s + 1], 0, T);
    *start = a;
    *end = b < a ? a : b;
  }
}

// Chunk `cid` -> (sequence, first token, valid length).  Dense layout: every
// sequence has ceil(T / C) chunks.  Packed layout: `chunk_off` holds the
// exclusive prefix sum of the per-sequence chunk counts (n_seqs + 1 entries).
// Returns false for ids past the last chunk (grids are sized by an upper
// bound).
__device__ __forceinline__ bool locate_chunk(int cid, const int32_t* cu,
                                             const int32_t* chunk_off,
                                             int n_seqs, int T, int C, int* seq,
                                             int* tok0, int* len) {
  if (cu == nullptr) {
    const int nc = (T + C - 1) / C;
    if (nc == 0) return false;
    const int s = cid / nc, c = cid % nc;
    if (s >= n_seqs) return false;
    *seq = s;
    *tok0 = s * T + c * C;
    *len = min(C, T - c * C);
    return true;
  }
  if (cid >= chunk_off[n_seqs]) return false;
  int lo = 0, hi = n_seqs;  // find s with chunk_off[s] <= cid < chunk_off[s+1]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (chunk_off[mid] <= cid)
      lo = mid;
    else
      hi = mid;
  }
  int a, b;
  seq_range(cu, lo, T, &a, &b);
  *seq = lo;
  *tok0 = a + (cid - chunk_off[lo]) * C;
  *len = min(C, b - *tok0);
  return *len > 0;
}

// Reference point of the decay factorisation inside a chunk.  The products
// A and P need exp(g_r - g_i) for i <= r, formed as exp(g_r - rho) *
// exp(rho - g_i) from one operand per row and one per column.  With rho = 0
// (the chunk start) the column factor exp(-g_i) grows like exp(|g_C|); with
// rho = g_C / 2 both factors stay within exp(|g_C| / 2).  A channel whose
// decay over the chunk is moderate keeps rho = 0 (its operands are then
// exactly the chunk-start ones); a strong one moves to the middle.  Past
// kDecayRangeMax even the middle reference overflows fp32, and the kernels
// report the call through the device range flag.
constexpr float kDecayRefMin = 60.f;
constexpr float kDecayRangeMax = 160.f;
__device__ __forceinline__ float decay_ref(float g_last) {
  return fabsf(g_last) > kDecayRefMin ? 0.5f * g_last : 0.f;
}

}  // namespace kda
