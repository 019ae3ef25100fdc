// Warp-sliced fused rowwise + columnwise cast (torchtitan PR #5334,
// description: one read of the input gives both the rowwise 1x32 and the
// columnwise 32x1 casts), plain and over the group pad path.
//
// A CTA of four warps owns a 128x128 bf16 tile -- exactly one 512-byte tile
// of each blocked scale output -- and each warp owns 32 rows of it. A 32-row
// slice holds whole blocks in both directions: four 1x32 blocks per row and
// one 32x1 block per column. So every warp works alone (one CTA barrier, at
// the end, before the two 512-byte scale tiles are stored):
//   load     the slice (32 rows x 256 bytes) into the warp's 8 KB of shared
//            memory with 16-byte cp.async copies (zero fill past the tensor
//            or the group); 16-byte chunk ch of row i is stored at chunk
//            ch ^ (i % 8) of that row, so that both passes below read
//            without bank conflicts;
//   rows     lane i converts row i: four blocks, each 32 codes written as one
//            32-byte sector, and the row's four scale bytes staged as one
//            word of the shared scale tile;
//   columns  lane l converts column pairs l and l + 32: 32 rows each, the two
//            columns' 32 codes written as two 32-byte sectors of the
//            transposed output, and their scale bytes staged likewise.
// Every code is written from registers as whole 32-byte sectors (one 256-bit
// store per sector); the only shared-memory traffic is the staged input.
#pragma once

#include "mx_cast.cuh"

namespace mx {

constexpr int kWarpCastWarps = 4;
constexpr int kWarpCastThreads = 32 * kWarpCastWarps;
constexpr int kWarpSliceBytes = 32 * kCastTile * 2;                    // 8 KB
constexpr int kWarpCastSmem = kWarpCastWarps * kWarpSliceBytes;       // 32 KB

// 16-byte global -> shared copy; src_bytes = 0 writes 16 zero bytes.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// 32 bytes (one sector) from one thread: a 256-bit store when `p` is 32-byte
// aligned, two 128-bit stores otherwise.
__device__ __forceinline__ void st_sector(void* p, bool aligned32, uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3,
                                          uint32_t w4, uint32_t w5, uint32_t w6, uint32_t w7) {
  if (aligned32) {
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(w0), "r"(w1), "r"(w2), "r"(w3),
                 "r"(w4), "r"(w5), "r"(w6), "r"(w7)
                 : "memory");
  } else {
    reinterpret_cast<uint4*>(p)[0] = make_uint4(w0, w1, w2, w3);
    reinterpret_cast<uint4*>(p)[1] = make_uint4(w4, w5, w6, w7);
  }
}

// Eight bf16 (four words) scaled by `inv` -> eight E4M3 codes in two words.
__device__ __forceinline__ uint2 quant8(uint4 w, float inv) {
  uint2 r;
  r.x = quant4(w.x, w.y, inv);
  r.y = quant4(w.z, w.w, inv);
  return r;
}

template <int kMode, bool kGrouped>
__global__ void __launch_bounds__(kWarpCastThreads)
cast_warp_kernel(const CastArgs a) {
  static_assert((kMode & kModeRowCol) == kModeRowCol && !(kMode & kModeSquare), "fused rowwise + columnwise only");
  extern __shared__ __align__(128) uint8_t wsmem[];
  __shared__ GroupSlot slots[kWarpCastWarps];
  __shared__ __align__(16) uint8_t s_row[512];    // the tile's rowwise scale tile
  __shared__ __align__(16) uint8_t s_col[512];    // the tile's columnwise scale tile
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t c0 = int64_t(blockIdx.x) * kCastTile;
  const int64_t r0 = int64_t(blockIdx.y) * kCastTile;
  const uint16_t* __restrict__ x = a.x;

  // rows of this tile that hold data, and their first source row
  long long src0 = r0, live = a.rows_src - r0;
  if constexpr (kGrouped) {
    find_group_of_row(a.offs, a.G, a.rows_src, a.rows_out, r0, &slots[warp]);
    __syncwarp();
    src0 = slots[warp].src0;
    live = slots[warp].live;
  }
  const int rw = warp * 32;                           // first tile row of this warp
  uint8_t* slice = wsmem + warp * kWarpSliceBytes;
  const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(slice));

  // ---- load the 32 x 128 slice: per instruction two rows of 16 chunks ----
  const int ch = lane & 15;
  const bool col_ok = c0 + ch * 8 < a.C;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int i = 2 * j + (lane >> 4);
    const bool ok = col_ok && rw + i < live;
    const uint16_t* src = ok ? x + (src0 + rw + i) * a.C + c0 + ch * 8 : x;
    cp_async16(sbase + i * 256 + ((ch ^ (i & 7)) << 4), src, ok ? 16u : 0u);
  }
  cp_async_wait_all();
  __syncwarp();

  const int64_t col_tiles_row = ceil_div(ceil_div(a.C, kBlock), 4);          // of blocked(rows_out, C/32)
  const int64_t col_tiles_col = ceil_div(ceil_div(a.rows_out, kBlock), 4);   // of blocked(C, rows_out/32)
  const int64_t chunk_row = int64_t(blockIdx.y) * col_tiles_row + blockIdx.x;
  const int64_t chunk_col = int64_t(blockIdx.x) * col_tiles_col + blockIdx.y;
  const bool rows_out_ok = r0 + rw < a.rows_out;       // the warp's 32 output rows exist
  // row and column code offsets are multiples of 32 bytes, so 256-bit stores
  // only need 32-byte aligned base pointers (the ABI promises 16)
  const bool q_al = (reinterpret_cast<uintptr_t>(a.q) & 31u) == 0;
  const bool qt_al = (reinterpret_cast<uintptr_t>(a.qt) & 31u) == 0;

  // ---- rows: lane i converts row rw + i ----
  {
    const int i = lane;
    const uint8_t* rowp = slice + i * 256;
    const int64_t row = r0 + rw + i;
    uint32_t bytes = 0u;
#pragma unroll
    for (int kb = 0; kb < 4; ++kb) {
      uint4 v[4];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) v[cc] = *reinterpret_cast<const uint4*>(rowp + (((kb * 4 + cc) ^ (i & 7)) << 4));
      uint32_t m = 0u;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        m = absmax_bf16x2(m, v[cc].x);
        m = absmax_bf16x2(m, v[cc].y);
        m = absmax_bf16x2(m, v[cc].z);
        m = absmax_bf16x2(m, v[cc].w);
      }
      m = max(m & 0xFFFFu, m >> 16);
      const uint32_t b = scale_b<kMode>(m);
      bytes |= b << (8 * kb);
      const float inv = inv_scale(b);
      const uint2 q0 = quant8(v[0], inv), q1 = quant8(v[1], inv), q2 = quant8(v[2], inv), q3 = quant8(v[3], inv);
      if (row < a.rows_out && c0 + kb * 32 < a.C)
        st_sector(a.q + row * a.C + c0 + kb * 32, q_al, q0.x, q0.y, q1.x, q1.y, q2.x, q2.y, q3.x, q3.y);
    }
    // S[row, c0/32 + kb] for kb = 0..3: four consecutive bytes of the tile
    *reinterpret_cast<uint32_t*>(s_row + i * 16 + warp * 4) = bytes;
  }

  // ---- columns: lane l converts column pairs l and l + 32 ----
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int cp = h * 32 + lane;                      // columns 2cp, 2cp + 1 of the tile
    const int chunk = cp >> 2, word = cp & 3;
    uint32_t w[32];
#pragma unroll
    for (int i = 0; i < 32; ++i)
      w[i] = *reinterpret_cast<const uint32_t*>(slice + i * 256 + ((chunk ^ (i & 7)) << 4) + word * 4);
    uint32_t acc = 0u;
#pragma unroll
    for (int i = 0; i < 32; ++i) acc = absmax_bf16x2(acc, w[i]);
    const uint32_t b_lo = scale_b<kMode>(acc & 0xFFFFu), b_hi = scale_b<kMode>(acc >> 16);
    const float inv_lo = inv_scale(b_lo), inv_hi = inv_scale(b_hi);
    uint32_t lo[8], hi[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = 4 * j;
      lo[j] = cvt_e4m3x2(bf16_lo(w[i]) * inv_lo, bf16_lo(w[i + 1]) * inv_lo) |
              (cvt_e4m3x2(bf16_lo(w[i + 2]) * inv_lo, bf16_lo(w[i + 3]) * inv_lo) << 16);
      hi[j] = cvt_e4m3x2(bf16_hi(w[i]) * inv_hi, bf16_hi(w[i + 1]) * inv_hi) |
              (cvt_e4m3x2(bf16_hi(w[i + 2]) * inv_hi, bf16_hi(w[i + 3]) * inv_hi) << 16);
    }
    const int64_t c = c0 + 2 * cp;
    if (rows_out_ok && c < a.C) {
      st_sector(a.qt + c * a.rows_out + r0 + rw, qt_al, lo[0], lo[1], lo[2], lo[3], lo[4], lo[5], lo[6], lo[7]);
      st_sector(a.qt + (c + 1) * a.rows_out + r0 + rw, qt_al, hi[0], hi[1], hi[2], hi[3], hi[4], hi[5], hi[6], hi[7]);
    }
    // S_col[c, r/32]: row c of blocked(C, rows_out/32), column block r0/32 + warp
    s_col[in_tile(uint32_t(2 * cp), uint32_t(warp))] = uint8_t(b_lo);
    s_col[in_tile(uint32_t(2 * cp + 1), uint32_t(warp))] = uint8_t(b_hi);
  }

  // ---- both scale tiles leave as whole 512-byte stores ----
  __syncthreads();
  if (threadIdx.x < 32)
    *reinterpret_cast<uint4*>(a.s + chunk_row * 512 + threadIdx.x * 16) =
        *reinterpret_cast<const uint4*>(s_row + threadIdx.x * 16);
  else if (threadIdx.x < 64)
    *reinterpret_cast<uint4*>(a.st + chunk_col * 512 + (threadIdx.x - 32) * 16) =
        *reinterpret_cast<const uint4*>(s_col + (threadIdx.x - 32) * 16);
}

}  // namespace mx
