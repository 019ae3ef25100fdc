// Definitions shared by the block-32 MXFP8 casts (the kernel is in
// mx_cast_warp.cuh): cast modes, the scale rule of a mode, and the argument
// block of a launch.
//
// The casts of the pages: rowwise 1x32 "dim0", columnwise 32x1 "dim1", the
// fused rowwise+columnwise cast, and 32x32 weight blocks (torchtitan PR
// #5334, description; ao "[moe training] Add backward_override to the MXFP8
// grouped GEMM", Design notes), plain and over the group pad path (same ao
// page, Known follow-ups, "pad_token_groups_for_grouped_mm"; ao PR #4705
// stack list, "pad/unpad" and "M-groups scale rearrange" kernels). Every
// cast writes its scales straight into the blocked layout, with no
// rearrangement pass.
#pragma once

#include "mx_common.cuh"

namespace mx {

constexpr int kCastTile = 128;   // a cast CTA's tile: one 512-byte tile of each blocked scale output

enum CastMode : int { kModeRow = 1, kModeCol = 2, kModeRowCol = 3, kModeSquare = 4, kModeFloor = 8 };

// Scale byte of a block from its amax bits under the mode's rule (RCEIL by
// default, FLOOR when the mode carries kModeFloor).
template <int kMode>
__device__ __forceinline__ uint32_t scale_b(uint32_t amax_bits) {
  return (kMode & kModeFloor) ? floor_b(amax_bits) : rceil_b(amax_bits);
}

struct CastArgs {
  const uint16_t* x;   // bf16 source rows [rows_src, C] (per expert in a stack)
  int64_t rows_src;    // source rows
  int64_t C;           // columns (multiple of 32)
  int64_t rows_out;    // rows of the padded / row-major outputs (rows_src or m_cap)
  const int32_t* offs; // grouped only: cumulative group ends
  int G;               // grouped only: number of groups
  uint8_t* q;          // rowwise codes [rows_out, C] (square: forward codes)
  uint8_t* s;          // rowwise scales blocked(rows_out, C/32) (square: S_fwd)
  uint8_t* qt;         // columnwise codes [C, rows_out] (square: transposed codes), may be null
  uint8_t* st;         // columnwise scales blocked(C, rows_out/32) (square: S_dgrad), may be null
  int64_t x_stride, q_stride, s_stride, qt_stride, st_stride;   // per-expert strides (square)
};

}  // namespace mx
