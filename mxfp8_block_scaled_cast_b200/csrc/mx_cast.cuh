// Block-32 MXFP8 cast kernels for sm_100a.
//
// One templated kernel covers the four casts of the pages (rowwise 1x32
// "dim0", columnwise 32x1 "dim1", the fused rowwise+columnwise cast, and
// 32x32 weight blocks; torchtitan PR #5334, description; ao
// "[moe training] Add backward_override to the MXFP8 grouped GEMM", Design
// notes) and the group pad path (same ao page, Known follow-ups,
// "pad_token_groups_for_grouped_mm"; ao PR #4705 stack list, "pad/unpad" and
// "M-groups scale rearrange" kernels).
//
// Each CTA owns a 128x128 bf16 tile. That tile maps onto exactly one
// 512-byte 128x4 tile of every blocked scale output, so scales are staged in
// shared memory and written with one coalesced 512-byte store per output --
// the blocked layout is produced directly, with no rearrangement pass.
//
// Data movement: 256 threads each issue eight independent 16-byte streaming
// loads (a warp reads 2 x 256 contiguous bytes per load), so 32 KB per CTA
// are in flight. The rowwise path reduces amax over the 4 lanes that share a
// 32-element block with two xor-shuffles and writes 8 contiguous E4M3 bytes
// per thread. The columnwise path stages the bf16 tile in shared memory
// (row-major, 256-byte rows: a warp reading one row of 64 column pairs is
// bank-conflict free), each thread reduces and converts two columns of one
// 32-row block, and the transposed codes go through a second shared tile
// whose 16-byte chunks are XOR-swizzled by (row/2)%8 so that both the scatter
// into it and the coalesced 128-byte row stores out of it are conflict free.
#pragma once

#include "mx_common.cuh"

namespace mx {

constexpr int kCastTile = 128;
constexpr int kCastThreads = 256;
constexpr int kCastPasses = kCastTile * kCastTile / 8 / kCastThreads;   // 8
constexpr int kXsBytes = kCastTile * kCastTile * 2;                      // bf16 tile
constexpr int kQsBytes = kCastTile * kCastTile;                          // transposed codes

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

template <int kMode, bool kGrouped>
__global__ void __launch_bounds__(kCastThreads)
cast_tile_kernel(const CastArgs a) {
  extern __shared__ __align__(128) uint8_t dyn_smem[];
  __shared__ GroupSlot slot;
  __shared__ uint32_t s_amax[16];                 // square: per 32x32 tile amax bits
  __shared__ __align__(16) uint8_t s_row[512];    // rowwise scale tile
  __shared__ __align__(16) uint8_t s_col[512];    // columnwise scale tile

  constexpr bool kRow = (kMode & kModeRow) != 0;
  constexpr bool kCol = (kMode & kModeCol) != 0;
  constexpr bool kSq = (kMode & kModeSquare) != 0;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t c0 = (int64_t)blockIdx.x * kCastTile;
  const int64_t r0 = (int64_t)blockIdx.y * kCastTile;
  const int64_t z = blockIdx.z;
  const uint16_t* __restrict__ x = a.x + z * a.x_stride;
  const bool do_colpass = kCol || (kSq && a.qt != nullptr);

  long long src0 = r0;
  long long live = a.rows_src - r0;
  if (kSq && tid < 16) s_amax[tid] = 0u;
  if constexpr (kGrouped) {
    if (warp == 0) find_group_of_row(a.offs, a.G, a.rows_src, a.rows_out, r0, &slot);
    __syncthreads();
    src0 = slot.src0;
    live = slot.live;
  } else if (kSq) {
    __syncthreads();
  }

  // ---- load: pass p covers rows p*16 .. p*16+15, 16 threads per row ----
  const int cl = (tid & 15) * 8;
  const bool col_ok = c0 + cl < a.C;
  uint4 v[kCastPasses];
#pragma unroll
  for (int p = 0; p < kCastPasses; ++p) {
    const int rl = p * 16 + (tid >> 4);
    if (col_ok && rl < live) v[p] = ld_stream16(x + (src0 + rl) * a.C + c0 + cl);
    else v[p] = make_uint4(0u, 0u, 0u, 0u);
  }

  uint8_t* xs = dyn_smem;
  uint8_t* qs = dyn_smem + kXsBytes;
  if (do_colpass) {
#pragma unroll
    for (int p = 0; p < kCastPasses; ++p) {
      const int rl = p * 16 + (tid >> 4);
      *reinterpret_cast<uint4*>(xs + rl * 256 + cl * 2) = v[p];
    }
  }

  // ---- rowwise amax of each 1x32 block (4 lanes per block) ----
  uint32_t bamax[kCastPasses];
#pragma unroll
  for (int p = 0; p < kCastPasses; ++p) {
    uint32_t m = absmax_bf16x2(0u, v[p].x);
    m = absmax_bf16x2(m, v[p].y);
    m = absmax_bf16x2(m, v[p].z);
    m = absmax_bf16x2(m, v[p].w);
    m = max(m & 0xFFFFu, m >> 16);
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
    bamax[p] = m;
  }

  if constexpr (kSq) {
    // rows 2*warp and 2*warp+1 of each pass sit in lanes l and l^16
#pragma unroll
    for (int p = 0; p < kCastPasses; ++p) {
      uint32_t m = max(bamax[p], __shfl_xor_sync(0xFFFFFFFFu, bamax[p], 16));
      if (lane < 16 && (lane & 3) == 0) atomicMax(&s_amax[(p >> 1) * 4 + (cl >> 5)], m);
    }
    __syncthreads();
  }

  // ---- rowwise (or square forward) codes ----
  if constexpr (kRow || kSq) {
    uint8_t* __restrict__ q = a.q + z * a.q_stride;
#pragma unroll
    for (int p = 0; p < kCastPasses; ++p) {
      const int rl = p * 16 + (tid >> 4);
      const uint32_t b = kSq ? scale_b<kMode>(s_amax[(p >> 1) * 4 + (cl >> 5)]) : scale_b<kMode>(bamax[p]);
      const float inv = inv_scale(b);
      uint2 o;
      o.x = quant4(v[p].x, v[p].y, inv);
      o.y = quant4(v[p].z, v[p].w, inv);
      const int64_t row = r0 + rl;
      if (col_ok && row < a.rows_out) *reinterpret_cast<uint2*>(q + row * a.C + c0 + cl) = o;
      if (kRow && (tid & 3) == 0) s_row[in_tile(rl, cl >> 5)] = uint8_t(b);
    }
  }

  // ---- columnwise (or square transposed) codes through shared memory ----
  if (do_colpass) {
    __syncthreads();
    const int rb = warp >> 1;                 // 32-row block of the tile
    const int cp = (warp & 1) * 32 + lane;    // column pair: columns 2cp, 2cp+1
    uint32_t w[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) w[i] = *reinterpret_cast<const uint32_t*>(xs + (rb * 32 + i) * 256 + cp * 4);
    uint32_t b_lo, b_hi;
    if (kCol) {
      uint32_t acc = 0u;
#pragma unroll
      for (int i = 0; i < 32; ++i) acc = absmax_bf16x2(acc, w[i]);
      b_lo = scale_b<kMode>(acc & 0xFFFFu);
      b_hi = scale_b<kMode>(acc >> 16);
    } else {
      b_lo = b_hi = scale_b<kMode>(s_amax[rb * 4 + (cp >> 4)]);
    }
    const float inv_lo = inv_scale(b_lo), inv_hi = inv_scale(b_hi);
    const int c = 2 * cp;
    const int sw = (c >> 1) & 7;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint4 lo4, hi4;
      uint32_t* lo = reinterpret_cast<uint32_t*>(&lo4);
      uint32_t* hi = reinterpret_cast<uint32_t*>(&hi4);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = h * 16 + j * 4;
        lo[j] = cvt_e4m3x2(bf16_lo(w[i]) * inv_lo, bf16_lo(w[i + 1]) * inv_lo) |
                (cvt_e4m3x2(bf16_lo(w[i + 2]) * inv_lo, bf16_lo(w[i + 3]) * inv_lo) << 16);
        hi[j] = cvt_e4m3x2(bf16_hi(w[i]) * inv_hi, bf16_hi(w[i + 1]) * inv_hi) |
                (cvt_e4m3x2(bf16_hi(w[i + 2]) * inv_hi, bf16_hi(w[i + 3]) * inv_hi) << 16);
      }
      const int phys = (rb * 2 + h) ^ sw;
      *reinterpret_cast<uint4*>(qs + c * 128 + phys * 16) = lo4;
      *reinterpret_cast<uint4*>(qs + (c + 1) * 128 + phys * 16) = hi4;
    }
    if (kCol) {
      s_col[in_tile(c, rb)] = uint8_t(b_lo);
      s_col[in_tile(c + 1, rb)] = uint8_t(b_hi);
    }
  }

  __syncthreads();

  // ---- stores of the staged outputs ----
  if (do_colpass) {
    uint8_t* __restrict__ qt = a.qt + z * a.qt_stride;
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
      const int row = pass * 32 + (tid >> 3);
      const int ch = tid & 7;
      if (c0 + row < a.C && r0 + ch * 16 < a.rows_out) {
        const uint4 val = *reinterpret_cast<const uint4*>(qs + row * 128 + ((ch ^ ((row >> 1) & 7)) * 16));
        *reinterpret_cast<uint4*>(qt + (c0 + row) * a.rows_out + r0 + ch * 16) = val;
      }
    }
  }
  const int64_t col_tiles_row = ceil_div(ceil_div(a.C, kBlock), 4);          // of blocked(rows_out, C/32)
  const int64_t col_tiles_col = ceil_div(ceil_div(a.rows_out, kBlock), 4);   // of blocked(C, rows_out/32)
  const int64_t chunk_row = blockIdx.y * col_tiles_row + blockIdx.x;
  const int64_t chunk_col = blockIdx.x * col_tiles_col + blockIdx.y;
  if constexpr (kRow) {
    if (tid < 32)
      *reinterpret_cast<uint4*>(a.s + chunk_row * 512 + tid * 16) = *reinterpret_cast<const uint4*>(s_row + tid * 16);
  }
  if constexpr (kCol) {
    if (tid >= 32 && tid < 64)
      *reinterpret_cast<uint4*>(a.st + chunk_col * 512 + (tid - 32) * 16) =
          *reinterpret_cast<const uint4*>(s_col + (tid - 32) * 16);
  }
  if constexpr (kSq) {
    // S_fwd[n, kb] = S[n/32, kb] in blocked(rows_out, C/32); S_dgrad[k, nb] = S[nb, k/32]
    // in blocked(C, rows_out/32). Each thread writes the 4 scale bytes of one row.
    if (tid < 128) {
      const int n = tid;
      uint32_t word = 0u;
#pragma unroll
      for (int kb = 0; kb < 4; ++kb) word |= scale_b<kMode>(s_amax[(n >> 5) * 4 + kb]) << (8 * kb);
      *reinterpret_cast<uint32_t*>(a.s + z * a.s_stride + chunk_row * 512 + (n & 31) * 16 + (n >> 5) * 4) = word;
    } else if (a.st != nullptr) {
      const int k = tid - 128;
      uint32_t word = 0u;
#pragma unroll
      for (int nb = 0; nb < 4; ++nb) word |= scale_b<kMode>(s_amax[nb * 4 + (k >> 5)]) << (8 * nb);
      *reinterpret_cast<uint32_t*>(a.st + z * a.st_stride + chunk_col * 512 + (k & 31) * 16 + (k >> 5) * 4) = word;
    }
  }
}

}  // namespace mx
