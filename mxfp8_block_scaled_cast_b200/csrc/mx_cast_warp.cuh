// Warp-sliced block-32 casts: rowwise 1x32 ("dim0"), columnwise 32x1
// ("dim1"), both from one read (torchtitan PR #5334, description: the fused
// rowwise/columnwise cast), and 32x32 weight blocks (same page, "32x32 RCEIL
// weight-scale policy"), plain and over the group pad path.
//
// A CTA of four warps owns a 128x128 bf16 tile -- exactly one 512-byte tile
// of each blocked scale output -- and each warp owns 32 rows of it. A 32-row
// slice holds whole blocks of every geometry: four 1x32 blocks per row, one
// 32x1 block per column, four 32x32 blocks. So every warp works alone (one
// CTA barrier, at the end, before the 512-byte scale tiles are stored):
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
//            transposed output, and their scale bytes staged likewise;
//   32x32    the four block maxima are reduced over the warp's lanes first;
//            rows then use the block scale (codes and the forward scale
//            view), columns the same scale (optional transposed codes and
//            the dgrad scale view).
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
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Waits until at most `n` of this thread's committed copy groups are still in flight.
template <int n>
__device__ __forceinline__ void cp_async_wait_group() { asm volatile("cp.async.wait_group %0;" ::"n"(n) : "memory"); }

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

// Largest of each 16-bit half over the 32 lanes of a warp.
__device__ __forceinline__ uint32_t warp_max_u16x2(uint32_t v) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) v = __vmaxu2(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// One 128x128 tile (column tile bx, row tile by, expert bz of a stack) of one
// cast; every thread of the CTA calls it. `wsmem` holds the four warps'
// slices, `s_row` / `s_col` the tile's two 512-byte scale tiles.
// Destinations of the scatter cast: group g's padded rows (codes) start at
// q[g], its 128-row scale bands at s[g]. A destination may be another GPU's
// memory (a peer mapping): the scatter cast writes it with plain stores.
struct ScatterDests {
  uint8_t* q[kMaxGroups];
  uint8_t* s[kMaxGroups];
};
// Destinations of the fused rowwise + columnwise scatter cast: q and s as
// above, and the group's columnwise outputs in the destination's transposed
// buffers: qt[g] its first padded token column of codes [C, cap[g]] (row
// stride cap[g], the destination's padded capacity), st[g] its first 512-byte
// tile of blocked(C, cap[g]/32) scales (cap[g]/128 tiles per 128-row band).
constexpr int kScatter2dMaxGroups = 512;     // the table is a kernel parameter (18 KB)
struct ScatterDests2d {
  uint8_t* q[kScatter2dMaxGroups];
  uint8_t* s[kScatter2dMaxGroups];
  uint8_t* qt[kScatter2dMaxGroups];
  uint8_t* st[kScatter2dMaxGroups];
  int32_t cap[kScatter2dMaxGroups];
};

template <int kMode, bool kGrouped, bool kScatter = false, class Dests = ScatterDests,
          bool kSplitLoad = (kMode & kModeCol) != 0>
__device__ __forceinline__ void cast_tile(const CastArgs& a, uint32_t bx, uint32_t by, uint32_t bz, uint8_t* wsmem,
                                          GroupSlot* slots, uint8_t* s_row, uint8_t* s_col,
                                          const Dests* dests = nullptr) {
  static_assert(!kScatter || (kGrouped && (kMode == kModeRow || kMode == kModeRowCol)),
                "the scatter casts are the grouped rowwise and fused casts");
  constexpr bool kRow = (kMode & kModeRow) != 0;
  constexpr bool kCol = (kMode & kModeCol) != 0;
  constexpr bool kSq = (kMode & kModeSquare) != 0;
  static_assert(!(kSq && (kRow || kCol || kGrouped)), "the 32x32 cast is its own mode");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t c0 = int64_t(bx) * kCastTile;
  const int64_t r0 = int64_t(by) * kCastTile;
  const int64_t z = bz;                               // expert of a 32x32 stack
  const uint16_t* __restrict__ x = a.x + z * a.x_stride;
  uint8_t* q = a.q ? a.q + z * a.q_stride : nullptr;
  uint8_t* s = a.s ? a.s + z * a.s_stride : nullptr;
  uint8_t* qt = a.qt ? a.qt + z * a.qt_stride : nullptr;
  uint8_t* st = a.st ? a.st + z * a.st_stride : nullptr;
  int64_t qt_rows = a.rows_out;                                               // row stride of qt
  int64_t col_tiles_col = ceil_div(ceil_div(a.rows_out, kBlock), 4);         // of blocked(C, rows_out/32)

  // rows of this tile that hold data, and their first source row
  long long src0 = r0, live = a.rows_src - r0;
  if constexpr (kGrouped) {
    find_group_of_row(a.offs, a.G, a.rows_src, a.rows_out, r0, &slots[warp]);
    __syncwarp();
    src0 = slots[warp].src0;
    live = slots[warp].live;
  }
  if constexpr (kScatter) {
    // the tile is rows r0 - pstart .. of its group's destination; a tile past
    // every group has none and writes nothing (the same for the whole CTA,
    // decided before any copy is issued)
    const int g = slots[warp].group;
    if (g < 0) return;
    const long long pstart = slots[warp].pstart;
    const int64_t bands = ceil_div(ceil_div(a.C, kBlock), 4) * 512;   // bytes of one 128-row scale band
    q = reinterpret_cast<uint8_t*>(reinterpret_cast<uintptr_t>(dests->q[g]) - uintptr_t(pstart * a.C));
    s = reinterpret_cast<uint8_t*>(reinterpret_cast<uintptr_t>(dests->s[g]) - uintptr_t((pstart / kCastTile) * bands));
    if constexpr (kCol) {
      // token column r of the source's padded layout is column r - pstart of
      // the group in the destination, whose row stride is its own capacity
      const int64_t cap = dests->cap[g];
      qt = reinterpret_cast<uint8_t*>(reinterpret_cast<uintptr_t>(dests->qt[g]) - uintptr_t(pstart));
      st = reinterpret_cast<uint8_t*>(reinterpret_cast<uintptr_t>(dests->st[g]) - uintptr_t((pstart / kCastTile) * 512));
      qt_rows = cap;
      col_tiles_col = cap / kCastTile;
    }
  }
  const int rw = warp * 32;                           // first tile row of this warp
  uint8_t* slice = wsmem + warp * kWarpSliceBytes;
  const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(slice));

  // ---- load the 32 x 128 slice ----
  // In two halves of 64 columns (two copy groups, per instruction four rows
  // of eight 16-byte chunks), so that the first half is converted while the
  // second is still arriving, or in one group of two rows of sixteen chunks
  // per instruction. A column pass (dim1, fused) always splits (measured:
  // +4-6% at 8192^2); rowwise and 32x32 split when the launch is at most a
  // few waves of tiles, where loads and stores otherwise run in lockstep
  // (+5% in-stream for 32x32 at 4096^2 and 8192^2 and rowwise at 16384x576),
  // and load whole slices on larger ones (the split cost them ~1% there).
  constexpr bool kTwoPhase = kSplitLoad;
  if constexpr (kTwoPhase) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int ch = half * 8 + (lane & 7);
      const bool col_ok = c0 + ch * 8 < a.C;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = 4 * j + (lane >> 3);
        const bool ok = col_ok && rw + i < live;
        const uint16_t* src = ok ? x + (src0 + rw + i) * a.C + c0 + ch * 8 : x;
        cp_async16(sbase + i * 256 + ((ch ^ (i & 7)) << 4), src, ok ? 16u : 0u);
      }
      cp_async_commit();
    }
  } else {
    const int ch = lane & 15;
    const bool col_ok = c0 + ch * 8 < a.C;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int i = 2 * j + (lane >> 4);
      const bool ok = col_ok && rw + i < live;
      const uint16_t* src = ok ? x + (src0 + rw + i) * a.C + c0 + ch * 8 : x;
      cp_async16(sbase + i * 256 + ((ch ^ (i & 7)) << 4), src, ok ? 16u : 0u);
    }
    cp_async_commit();
  }

  const int64_t col_tiles_row = ceil_div(ceil_div(a.C, kBlock), 4);          // of blocked(rows_out, C/32)
  const int64_t chunk_row = int64_t(by) * col_tiles_row + bx;
  const int64_t chunk_col = int64_t(bx) * col_tiles_col + by;
  const bool rows_out_ok = r0 + rw < a.rows_out;       // the warp's 32 output rows exist
  // row and column code offsets are multiples of 32 bytes, so 256-bit stores
  // only need 32-byte aligned base pointers (the ABI promises 16)
  const bool q_al = (reinterpret_cast<uintptr_t>(q) & 31u) == 0;
  const bool qt_al = (reinterpret_cast<uintptr_t>(qt) & 31u) == 0;
  const uint8_t* rowp = slice + lane * 256;            // lane i works on row rw + i
  auto chunk_of_row = [&](int c) {                     // 16-byte chunk c of row `lane`
    return *reinterpret_cast<const uint4*>(rowp + ((c ^ (lane & 7)) << 4));
  };

  // Each half (64 columns) is converted on its own: its two 32-column blocks
  // of every row, its 32 column pairs, and (32x32) its two block scales.
  uint32_t row_bytes = 0u;                             // the row's four scale bytes (rows / square)
  const bool col_codes = kCol || (kSq && qt != nullptr);
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    if (half == 0) {
      if constexpr (kTwoPhase) cp_async_wait_group<1>(); else cp_async_wait_group<0>();
    } else if constexpr (kTwoPhase) {
      cp_async_wait_group<0>();
    }
    __syncwarp();

    // ---- square: one scale per 32x32 block, the max over the warp's rows ----
    uint32_t bsq[2] = {0u, 0u};                          // the half's blocks 2*half, 2*half + 1
    if constexpr (kSq) {
      uint32_t m01 = 0u;                                 // the two blocks in the 16-bit halves
#pragma unroll
      for (int b2 = 0; b2 < 2; ++b2) {
        uint32_t m = 0u;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const uint4 v = chunk_of_row((2 * half + b2) * 4 + cc);
          m = absmax_bf16x2(m, v.x);
          m = absmax_bf16x2(m, v.y);
          m = absmax_bf16x2(m, v.z);
          m = absmax_bf16x2(m, v.w);
        }
        m = max(m & 0xFFFFu, m >> 16);
        m01 |= b2 ? (m << 16) : m;
      }
      m01 = warp_max_u16x2(m01);
      bsq[0] = scale_b<kMode>(m01 & 0xFFFFu);
      bsq[1] = scale_b<kMode>(m01 >> 16);
    }

    // ---- rows: lane i converts row rw + i (rowwise blocks, or square blocks) ----
    if constexpr (kRow || kSq) {
      const int64_t row = r0 + rw + lane;
#pragma unroll
      for (int b2 = 0; b2 < 2; ++b2) {
        const int kb = 2 * half + b2;
        uint4 v[4];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) v[cc] = chunk_of_row(kb * 4 + cc);
        uint32_t b;
        if constexpr (kSq) {
          b = bsq[b2];
        } else {
          uint32_t m = 0u;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            m = absmax_bf16x2(m, v[cc].x);
            m = absmax_bf16x2(m, v[cc].y);
            m = absmax_bf16x2(m, v[cc].z);
            m = absmax_bf16x2(m, v[cc].w);
          }
          b = scale_b<kMode>(max(m & 0xFFFFu, m >> 16));
        }
        row_bytes |= b << (8 * kb);
        const float inv = inv_scale(b);
        const uint2 q0 = quant8(v[0], inv), q1 = quant8(v[1], inv), q2 = quant8(v[2], inv), q3 = quant8(v[3], inv);
        if (row < a.rows_out && c0 + kb * 32 < a.C)
          st_sector(q + row * a.C + c0 + kb * 32, q_al, q0.x, q0.y, q1.x, q1.y, q2.x, q2.y, q3.x, q3.y);
      }
    }

    // ---- columns: lane l converts column pair l of the half (columns 64 half + 2l, + 1) ----
    if (kCol || (kSq && (qt != nullptr || st != nullptr))) {
      const int cp = half * 32 + lane;                 // columns 2cp, 2cp + 1 of the tile
      const int chunk = cp >> 2, word = cp & 3;
      const int blk = cp >> 4;                         // 32-column block of these columns
      uint32_t b_lo = 0u;
      if constexpr (kSq) b_lo = (blk & 1) ? bsq[1] : bsq[0];
      uint32_t b_hi = b_lo;
      if (col_codes) {
        uint32_t w[32];
#pragma unroll
        for (int i = 0; i < 32; ++i)
          w[i] = *reinterpret_cast<const uint32_t*>(slice + i * 256 + ((chunk ^ (i & 7)) << 4) + word * 4);
        if constexpr (kCol) {
          uint32_t acc = 0u;
#pragma unroll
          for (int i = 0; i < 32; ++i) acc = absmax_bf16x2(acc, w[i]);
          b_lo = scale_b<kMode>(acc & 0xFFFFu);
          b_hi = scale_b<kMode>(acc >> 16);
        }
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
          st_sector(qt + c * qt_rows + r0 + rw, qt_al, lo[0], lo[1], lo[2], lo[3], lo[4], lo[5], lo[6], lo[7]);
          st_sector(qt + (c + 1) * qt_rows + r0 + rw, qt_al, hi[0], hi[1], hi[2], hi[3], hi[4], hi[5], hi[6],
                    hi[7]);
        }
      }
      // S_col[c, r/32] (square: S_dgrad[k, n/32]): row c of blocked(C, rows_out/32),
      // column block r0/32 + warp
      s_col[in_tile(uint32_t(2 * cp), uint32_t(warp))] = uint8_t(b_lo);
      s_col[in_tile(uint32_t(2 * cp + 1), uint32_t(warp))] = uint8_t(b_hi);
    }
  }

  // S[row, c0/32 + kb] for kb = 0..3: four consecutive bytes of the row scale tile
  if constexpr (kRow || kSq) *reinterpret_cast<uint32_t*>(s_row + lane * 16 + warp * 4) = row_bytes;

  // ---- the scale tiles leave as whole 512-byte stores ----
  __syncthreads();
  if (threadIdx.x < 32) {
    if ((kRow || kSq) && s != nullptr)
      *reinterpret_cast<uint4*>(s + chunk_row * 512 + threadIdx.x * 16) =
          *reinterpret_cast<const uint4*>(s_row + threadIdx.x * 16);
  } else if (threadIdx.x < 64) {
    if ((kCol || kSq) && st != nullptr)
      *reinterpret_cast<uint4*>(st + chunk_col * 512 + (threadIdx.x - 32) * 16) =
          *reinterpret_cast<const uint4*>(s_col + (threadIdx.x - 32) * 16);
  }
}

template <int kMode, bool kGrouped, bool kSplitLoad = (kMode & kModeCol) != 0>
__global__ void __launch_bounds__(kWarpCastThreads)
cast_warp_kernel(const CastArgs a) {
  extern __shared__ __align__(128) uint8_t wsmem[];
  __shared__ GroupSlot slots[kWarpCastWarps];
  __shared__ __align__(16) uint8_t s_row[512];    // the tile's rowwise (square: forward) scale tile
  __shared__ __align__(16) uint8_t s_col[512];    // the tile's columnwise (square: dgrad) scale tile
  cast_tile<kMode, kGrouped, false, ScatterDests, kSplitLoad>(a, blockIdx.x, blockIdx.y, blockIdx.z, wsmem, slots,
                                                             s_row, s_col);
}

// The grouped rowwise cast with each group's padded rows written to its own
// destination (prime-rl PR #3388, Overview: enable_a2a, the MXFP8 dispatch of
// expert parallelism): the cast and the token exchange in one kernel, each
// tile stored straight into the receiving rank's buffer. The host follows it
// with system_fence_kernel on the same stream, so that the stores to peer
// memory are visible to the other GPUs once that launch is seen complete.
__global__ void __launch_bounds__(kWarpCastThreads)
cast_scatter_kernel(const __grid_constant__ CastArgs a, const __grid_constant__ ScatterDests d) {
  extern __shared__ __align__(128) uint8_t wsmem[];
  __shared__ GroupSlot slots[kWarpCastWarps];
  __shared__ __align__(16) uint8_t s_row[512];
  __shared__ __align__(16) uint8_t s_col[512];
  cast_tile<kModeRow, true, true>(a, blockIdx.x, blockIdx.y, blockIdx.z, wsmem, slots, s_row, s_col, &d);
}

// The fused rowwise + columnwise cast into per-group destinations: the
// backward dispatch of expert parallelism (dY of each token group cast both
// ways, straight into the expert's buffers, in the layout the expert's own
// fused grouped cast would write). Followed by system_fence_kernel, as above.
__global__ void __launch_bounds__(kWarpCastThreads)
cast_scatter2d_kernel(const __grid_constant__ CastArgs a, const __grid_constant__ ScatterDests2d d) {
  extern __shared__ __align__(128) uint8_t wsmem[];
  __shared__ GroupSlot slots[kWarpCastWarps];
  __shared__ __align__(16) uint8_t s_row[512];
  __shared__ __align__(16) uint8_t s_col[512];
  cast_tile<kModeRowCol, true, true, ScatterDests2d>(a, blockIdx.x, blockIdx.y, blockIdx.z, wsmem, slots, s_row,
                                                     s_col, &d);
}

// One system-scope fence issued after a kernel that stored to other GPUs'
// memory, on the same stream: every store of that kernel precedes it in stream
// order, so one fence for the whole launch replaces a fence in every CTA (which
// holds each CTA until its own stores are visible system-wide: measured 0.49x
// the throughput of the same cast into one local buffer, against 0.86x with
// this launch after it).
__global__ void system_fence_kernel() { __threadfence_system(); }

// Up to three independent dense casts in one launch (the linear's weight and
// activation casts): CTAs [0, n0) take cast 0's tiles, the next n1 cast 1's,
// then cast 2's, each in its own launch order (column tile fastest, then row
// tile, then expert). One launch instead of several lets the casts' partial
// last waves share the SMs and drops the gaps between launches; every tile is
// computed exactly as its own launch would, so the output bits are the same.
// A mode of -1 marks an unused slot.
struct CastJobs {
  CastArgs a[3];
  uint32_t gx[3], gy[3], gz[3];   // each cast's tile grid (column, row, expert)
};

template <int kM0, int kM1, int kM2>
__global__ void __launch_bounds__(kWarpCastThreads)
cast_multi_kernel(const __grid_constant__ CastJobs j) {
  extern __shared__ __align__(128) uint8_t wsmem[];
  __shared__ GroupSlot slots[kWarpCastWarps];
  __shared__ __align__(16) uint8_t s_row[512];
  __shared__ __align__(16) uint8_t s_col[512];
  uint32_t id = blockIdx.x;
  const uint32_t n0 = j.gx[0] * j.gy[0] * j.gz[0];
  const uint32_t n1 = kM1 < 0 ? 0u : j.gx[1] * j.gy[1] * j.gz[1];
  int k = 0;
  if (id >= n0) {
    id -= n0;
    k = 1;
    if (id >= n1) {
      id -= n1;
      k = 2;
    }
  }
  const uint32_t gx = j.gx[k], gy = j.gy[k];
  const uint32_t bx = id % gx, by = (id / gx) % gy, bz = id / (gx * gy);
  if (k == 0) {
    cast_tile<kM0, false>(j.a[0], bx, by, bz, wsmem, slots, s_row, s_col);
  } else if (k == 1) {
    if constexpr (kM1 >= 0) cast_tile<kM1, false>(j.a[1], bx, by, bz, wsmem, slots, s_row, s_col);
  } else {
    if constexpr (kM2 >= 0) cast_tile<kM2, false>(j.a[2], bx, by, bz, wsmem, slots, s_row, s_col);
  }
}

}  // namespace mx
