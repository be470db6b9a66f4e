// fp32 tensor maps (128-byte swizzle, boxes 32 columns wide) shared by the
// backward pass's tensor-core kernels; encoded through the driver entry
// point in kda_fused_sm100.cu.
#pragma once
#include <cuda.h>
#include <stdint.h>

namespace kda {
// [tokens, H, cols] fp32, box of 32 columns x one head x 64 tokens.
bool make_f32_tok_map(CUtensorMap* m, const float* base, int cols, int H,
                      int tokens);
// [rows, cols] fp32, box of 32 columns x box_rows rows.
bool make_f32_rows_map(CUtensorMap* m, const float* base, int64_t rows,
                       int cols, int box_rows);
}  // namespace kda
