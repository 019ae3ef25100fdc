// Pipelined columnwise MXFP8 casts for sm_100a: dim1 (32x1) and the 32x32
// weight cast with transposed codes (the kernel also implements the fused
// rowwise+columnwise cast, which the library routes to the tile kernel)
// (torchtitan PR #5334, description; ao "[moe training] Add backward_override
// to the MXFP8 grouped GEMM", Summary and Design notes), with and without the
// group pad path. The arithmetic is the one of mx_cast.cuh (integer RCEIL on
// the bf16 bit fields, exact power-of-two scaling, cvt.rn.satfinite to E4M3)
// and the outputs are bitwise identical to it; only the data movement differs.
//
// Persistent CTAs of 256 threads walk the 128x128 tiles. Each tile arrives in
// shared memory through one 2D TMA load (32 KB, zero fill outside the tensor)
// into a two-deep ring, so the next tile streams in while this one is cast.
// The columnwise pass reads 16-byte vectors: a thread owns 8 columns x 8 rows
// and the four lanes holding the rest of the same 32-row block sit in the
// same warp (shfl.xor 8, 16), i.e. four times fewer shared-memory loads than
// one column pair per thread. Transposed codes go through a staging tile whose 16-byte
// pieces are XOR-swizzled by the destination row so both its writes and the
// coalesced 128-byte row stores out of it are bank-conflict free. In the 32x32
// mode the tile amax is reduced with shuffles (rows by xor 8 and 16, the four
// 8-column groups of a 32-column block by xor 1 and 2). Rowwise codes (the
// fused cast, and the forward codes of the 32x32 cast) are produced from the
// same registers, so each tile is read from shared memory once.
#pragma once

#include "mx_cast.cuh"
#include "mx_sm100.cuh"

namespace mx {

constexpr int kPipeThreads = 256;
constexpr int kPipeBufs = 2;
constexpr uint32_t kPipeTileBytes = kCastTile * kCastTile * 2;            // 32 KB bf16 tile
constexpr uint32_t kPipeOffQs = kPipeBufs * kPipeTileBytes;               // staging of transposed codes
constexpr uint32_t kPipeOffSrow = kPipeOffQs + kCastTile * kCastTile;     // 512 B rowwise scale tile
constexpr uint32_t kPipeOffScol = kPipeOffSrow + 512;                     // 512 B columnwise scale tile
constexpr uint32_t kPipeOffStile = kPipeOffScol + 512;                    // 16 words: 32x32 tile amax
constexpr uint32_t kPipeOffInfo = kPipeOffStile + 64;                     // per-buffer tile info
constexpr uint32_t kPipeOffBar = kPipeOffInfo + 64 * kPipeBufs;           // per-buffer mbarriers
constexpr uint32_t kPipeOffAbort = kPipeOffBar + 8 * kPipeBufs;
constexpr uint32_t kPipeSmem = kPipeOffAbort + 16 + 128;                  // + alignment slack

struct PipeTile {
  GroupSlot g;        // g.src0: first source row (TMA y); g.live: real rows (<= 0: all padding)
  long long r0, c0;   // output row and column of the tile
  long long z;        // expert (32x32 stacks)
};
static_assert(sizeof(PipeTile) <= 64, "tile info slot");

template <int kMode, bool kGrouped>
__global__ void __launch_bounds__(kPipeThreads, 2)
cast_pipe_kernel(const __grid_constant__ CUtensorMap xmap, const CastArgs a, int64_t tiles_c, int64_t tiles_r,
                 int64_t tiles_total) {
  extern __shared__ uint8_t pipe_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pipe_raw) + 127) & ~uintptr_t(127));
  constexpr bool kRow = (kMode & kModeRow) != 0;
  constexpr bool kCol = (kMode & kModeCol) != 0;
  constexpr bool kSq = (kMode & kModeSquare) != 0;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint8_t* qs = smem + kPipeOffQs;
  uint8_t* s_row = smem + kPipeOffSrow;
  uint8_t* s_col = smem + kPipeOffScol;
  uint32_t* s_tile = reinterpret_cast<uint32_t*>(smem + kPipeOffStile);
  PipeTile* info = reinterpret_cast<PipeTile*>(smem + kPipeOffInfo);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kPipeOffAbort);
  const uint32_t bar0 = smem_u32(smem + kPipeOffBar);
  const int64_t per_z = tiles_c * tiles_r;

  if (tid == 0) {
    for (int b = 0; b < kPipeBufs; ++b) mbar_init(bar0 + 8u * b, 1);
    fence_barrier_init();
    *abort_flag = 0;
    tma_prefetch_desc(&xmap);
  }
  __syncthreads();

  // Warp 0: resolve tile `tile` (its group for the pad path) and start its TMA
  // load into buffer b; a tile that is all padding completes the barrier
  // without a copy (the cast then reads zeros).
  auto prepare = [&](int64_t tile, int b) {
    PipeTile* ti = info + b;
    const int64_t z = tile / per_z, rem = tile % per_z;
    const int64_t r0 = (rem / tiles_c) * kCastTile, c0 = (rem % tiles_c) * kCastTile;
    if constexpr (kGrouped) {
      find_group_of_row(a.offs, a.G, a.rows_src, a.rows_out, r0, &ti->g);
    } else if (lane == 0) {
      ti->g.src0 = z * a.rows_src + r0;     // stacks are viewed as [G * rows, C]
      ti->g.live = a.rows_src - r0;
      ti->g.group = 0;
    }
    __syncwarp();
    if (lane == 0) {
      ti->r0 = r0;
      ti->c0 = c0;
      ti->z = z;
      const uint32_t bar = bar0 + 8u * b;
      if (ti->g.live > 0) {
        mbar_arrive_expect_tx(bar, kPipeTileBytes);
        tma_load_2d(smem_u32(smem + b * kPipeTileBytes), &xmap, int32_t(c0), int32_t(ti->g.src0), bar);
      } else {
        mbar_arrive(bar);
      }
    }
    __syncwarp();
  };

  const int64_t first = blockIdx.x, step = gridDim.x;
  int64_t prepared = 0;           // tiles whose copy was started (tracked by warp 0)
  if (warp == 0)
    for (int j = 0; j < kPipeBufs - 1; ++j)
      if (first + j * step < tiles_total) {
        prepare(first + j * step, j);
        ++prepared;
      }

  int64_t k = 0;
  for (int64_t tile = first; tile < tiles_total; tile += step, ++k) {
    const int b = int(k % kPipeBufs);
    if (warp == 0) {
      const int64_t ahead = tile + (kPipeBufs - 1) * step;
      if (ahead < tiles_total) {
        prepare(ahead, int((k + kPipeBufs - 1) % kPipeBufs));
        ++prepared;
      }
    }
    const bool ok = mbar_wait(bar0 + 8u * b, uint32_t((k / kPipeBufs) & 1), abort_flag);
    if (!__syncthreads_and(ok)) break;          // one decision for the whole CTA
    const PipeTile ti = info[b];
    const uint8_t* xs = smem + b * kPipeTileBytes;
    const long long live = ti.g.live > 0 ? ti.g.live : 0;
    const int64_t r0 = ti.r0, c0 = ti.c0, z = ti.z;

    // ---------------- columnwise pass: 8 columns x 8 rows per thread ----------------
    // warp w: 32-row block rb = w/2, columns 64*(w%2)..+63; lane: 8-column
    // group cg (8 per warp) and 8-row quarter qq of the block.
    const int rb = warp >> 1;
    const int cg = (lane & 7) + 8 * (warp & 1);
    const int qq = lane >> 3;
    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int row = rb * 32 + qq * 8 + i;
      v[i] = row < live ? *reinterpret_cast<const uint4*>(xs + row * 256 + cg * 16) : make_uint4(0u, 0u, 0u, 0u);
    }
    uint32_t am2[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t acc = 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i) acc = absmax_bf16x2(acc, reinterpret_cast<const uint32_t*>(&v[i])[q]);
      acc = __vmaxu2(acc, __shfl_xor_sync(0xFFFFFFFFu, acc, 8));    // the four quarters of the block
      am2[q] = __vmaxu2(acc, __shfl_xor_sync(0xFFFFFFFFu, acc, 16));
    }
    if constexpr (kSq) {
      uint32_t m = 0u;
#pragma unroll
      for (int q = 0; q < 4; ++q) m = max(m, max(am2[q] & 0xFFFFu, am2[q] >> 16));
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));             // four 8-column groups
      m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
      if (qq == 0 && (cg & 3) == 0) s_tile[rb * 4 + (cg >> 2)] = m;
      __syncthreads();
    }
    if (kCol || (kSq && a.qt != nullptr)) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t bj;
        if (kSq) bj = rceil_b(s_tile[rb * 4 + (cg >> 2)]);
        else bj = rceil_b((j & 1) ? (am2[j >> 1] >> 16) : (am2[j >> 1] & 0xFFFFu));
        const float inv = inv_scale(bj);
        uint2 o;
        uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          float f[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint32_t word = reinterpret_cast<const uint32_t*>(&v[4 * w + u])[j >> 1];
            f[u] = ((j & 1) ? bf16_hi(word) : bf16_lo(word)) * inv;
          }
          ow[w] = cvt_e4m3x2(f[0], f[1]) | (cvt_e4m3x2(f[2], f[3]) << 16);
        }
        // transposed tile row qrow, bytes rb*32 + qq*8 .. +7: 16-byte piece
        // rb*2 + qq/2 (XOR-swizzled by the row), 8-byte half qq%2
        const int qrow = cg * 8 + j;
        const int phys = (rb * 2 + (qq >> 1)) ^ ((qrow >> 3) & 7);
        *reinterpret_cast<uint2*>(qs + qrow * 128 + phys * 16 + (qq & 1) * 8) = o;
        if (kCol && qq == 0) s_col[in_tile(qrow, rb)] = uint8_t(bj);
      }
    }

    // ---------------- rowwise codes from the same registers ----------------
    // The four lanes holding one row's 32-column block are the lanes with
    // cg = 4m..4m+3 of the same warp, so the rowwise amax is two xor-shuffles.
    if constexpr (kRow || kSq) {
      uint8_t* __restrict__ q = a.q + z * a.q_stride;
      const bool col_ok = c0 + cg * 8 < a.C;
      const uint32_t b_tile = kSq ? rceil_b(s_tile[rb * 4 + (cg >> 2)]) : 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int row = rb * 32 + qq * 8 + i;
        uint32_t b;
        if constexpr (kSq) {
          b = b_tile;
        } else {
          uint32_t m = absmax_bf16x2(0u, v[i].x);
          m = absmax_bf16x2(m, v[i].y);
          m = absmax_bf16x2(m, v[i].z);
          m = absmax_bf16x2(m, v[i].w);
          m = max(m & 0xFFFFu, m >> 16);
          m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
          m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
          b = rceil_b(m);
          if ((cg & 3) == 0) s_row[in_tile(row, cg >> 2)] = uint8_t(b);
        }
        const float inv = inv_scale(b);
        uint2 o;
        o.x = quant4(v[i].x, v[i].y, inv);
        o.y = quant4(v[i].z, v[i].w, inv);
        if (col_ok && r0 + row < a.rows_out) *reinterpret_cast<uint2*>(q + (r0 + row) * a.C + c0 + cg * 8) = o;
      }
    }
    __syncthreads();

    // ---------------- staged stores ----------------
    const int64_t col_tiles_row = ceil_div(ceil_div(a.C, kBlock), 4);
    const int64_t col_tiles_col = ceil_div(ceil_div(a.rows_out, kBlock), 4);
    const int64_t bx = c0 / kCastTile, by = r0 / kCastTile;
    if (kCol || (kSq && a.qt != nullptr)) {
      uint8_t* __restrict__ qt = a.qt + z * a.qt_stride;
#pragma unroll
      for (int pass = 0; pass < 4; ++pass) {
        const int row = pass * 32 + (tid >> 3);
        const int ch = tid & 7;
        if (c0 + row < a.C && r0 + ch * 16 < a.rows_out) {
          const uint4 val = *reinterpret_cast<const uint4*>(qs + row * 128 + ((ch ^ ((row >> 3) & 7)) * 16));
          *reinterpret_cast<uint4*>(qt + (c0 + row) * a.rows_out + r0 + ch * 16) = val;
        }
      }
    }
    if constexpr (kRow) {
      if (tid < 32)
        *reinterpret_cast<uint4*>(a.s + (by * col_tiles_row + bx) * 512 + tid * 16) =
            *reinterpret_cast<const uint4*>(s_row + tid * 16);
    }
    if constexpr (kCol) {
      if (tid >= 32 && tid < 64)
        *reinterpret_cast<uint4*>(a.st + (bx * col_tiles_col + by) * 512 + (tid - 32) * 16) =
            *reinterpret_cast<const uint4*>(s_col + (tid - 32) * 16);
    }
    if constexpr (kSq) {
      // S_fwd[n, kb] = S[n/32, kb] and S_dgrad[k, nb] = S[nb, k/32]: one word per row
      const int n = tid & 127;
      uint32_t w = 0u;
      if (tid < 128) {
#pragma unroll
        for (int j = 0; j < 4; ++j) w |= rceil_b(s_tile[(n >> 5) * 4 + j]) << (8 * j);
        *reinterpret_cast<uint32_t*>(a.s + z * a.s_stride + (by * col_tiles_row + bx) * 512 + (n & 31) * 16 +
                                     (n >> 5) * 4) = w;
      } else if (a.st != nullptr) {
#pragma unroll
        for (int j = 0; j < 4; ++j) w |= rceil_b(s_tile[j * 4 + (n >> 5)]) << (8 * j);
        *reinterpret_cast<uint32_t*>(a.st + z * a.st_stride + (bx * col_tiles_col + by) * 512 + (n & 31) * 16 +
                                     (n >> 5) * 4) = w;
      }
    }
    __syncthreads();
  }
  // every started copy lands before the CTA's shared memory is released
  // (only an aborted loop leaves copies unconsumed)
  if (tid == 0)
    for (int64_t kk = k; kk < prepared; ++kk) mbar_drain(bar0 + 8u * int(kk % kPipeBufs), uint32_t((kk / kPipeBufs) & 1));
}

}  // namespace mx
