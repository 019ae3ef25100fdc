// MXFP8 scaled grouped GEMM on sm_100a tensor cores (tcgen05, TMEM, TMA).
//
// Computes, in fp32 with a bf16 result, the grouped products of the MXFP8
// grouped GEMM over an offsets array (ao "[moe training] Add
// backward_override to the MXFP8 grouped GEMM", Summary: forward, dgrad and
// wgrad of _MXFP8GroupedMM; ao PR #4705, "MXFP8 MoE grouped-mm"):
//
//   M-groups (forward, dgrad): out[rows of g, :] = A[padded rows of g, :] * B[g]^T
//     A codes [rows_a, K] (padded token rows), B codes [G, N, K], out [M, N].
//   K-groups (wgrad):          out[g] = A[:, tokens of g] * B[:, tokens of g]^T
//     A codes [N, m_cap], B codes [K, m_cap] (padded token columns), out [G, N, K].
//
// Both operands are K-major E4M3 with blocked E8M0 scales; each token group
// starts on a 128-row boundary of the padded layout (the pad path), so every
// 128-row scale tile and every 128-wide K tile belongs to one group.
//
// Design (one persistent CTA per SM, 192 threads, warp-specialised):
//   warp 4      TMA producer: per 128-deep K step, two tiled TMA loads
//               (A 128x128 B, B 256x128 B, 128-byte swizzle) and three
//               512-byte bulk copies of blocked scale tiles into a 4-stage
//               shared-memory ring, completing on a per-stage mbarrier.
//   warp 5      MMA issuer: copies the stage's scale tiles into TMEM
//               (tcgen05.cp 32x128b.warpx4) and issues four
//               tcgen05.mma.kind::mxf8f6f4.block_scale (M=128, N=256, K=32)
//               into a 128x256 fp32 TMEM accumulator; tcgen05.commit frees
//               the stage and, after the last K step, signals the epilogue.
//   warps 0-3   epilogue: tcgen05.ld of the accumulator (one row per thread),
//               fp32 -> bf16 (round to nearest even), row stores with the
//               padded->unpadded row map of the group (the unpad step is
//               fused here).
// The tile scheduler is static round robin over (group, m tile, n tile);
// group boundaries come from a per-CTA scan of the device offsets, so no
// host synchronisation is needed. An empty group in K-groups mode writes
// exact zeros (no MMA). There is no split-K and no atomic: results are
// deterministic.
#pragma once

#include "mx_sm100.cuh"

namespace mx {

constexpr int kBM = 128, kBN = 256, kBK = 128;
constexpr int kStages = 4;
constexpr int kGemmThreads = 192;
constexpr uint32_t kABytes = kBM * kBK;                   // 16 KB
constexpr uint32_t kBBytes = kBN * kBK;                   // 32 KB
constexpr uint32_t kSfaBytes = 512, kSfbBytes = 1024;
constexpr uint32_t kTxBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0;
constexpr uint32_t kSfaCol = 256;
constexpr uint32_t kSfbCol = kSfaCol + 4 * kStages;

// shared-memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + kStages * kABytes;
constexpr uint32_t kOffSfa = kOffB + kStages * kBBytes;
constexpr uint32_t kOffSfb = kOffSfa + kStages * kSfaBytes;
constexpr uint32_t kOffBar = kOffSfb + kStages * kSfbBytes;
constexpr uint32_t kNumBars = 2 * kStages + 3;            // full, empty, acc_full, acc_empty, done
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;     // tmem slot, abort, info words
constexpr uint32_t kOffEnds = kOffMisc + 64;
constexpr uint32_t kOffPstart = kOffEnds + 4 * kMaxGroups;
constexpr uint32_t kGemmSmem = kOffPstart + 4 * (kMaxGroups + 1) + 1024;   // + alignment slack

// Instruction descriptor of kind::mxf8f6f4 with block scaling: E4M3 A and B
// (format 0), both K-major, N>>3 in bits [17,23), E8M0 scales (bit 23),
// M>>4 in bits [24,29); the scale-factor byte ids (bits [4,6) for B and
// [29,31) for A) select which of the four K blocks packed in each TMEM
// scale column this MMA uses.
constexpr uint32_t kIdescBase = (uint32_t(kBN >> 3) << 17) | (1u << 23) | (uint32_t(kBM >> 4) << 24);

enum GemmMode : int { kGroupsM = 0, kGroupsK = 1 };

struct GemmArgs {
  const uint8_t* a_s;          // A blocked scales
  const uint8_t* b_s;          // B blocked scales (M-groups: G concatenated per-expert buffers)
  const int32_t* offs;         // cumulative group ends, or null for one dense group
  __nv_bfloat16* out;
  int G;
  int64_t M, N, K;             // see the mode description above
  int64_t m_cap;               // padded capacity (rows of A in M mode, token columns in K mode)
  int64_t a_sc_tiles;          // 4-column scale tiles per 128-row band of A's blocked scales
  int64_t b_sc_tiles;          // same for B
  int64_t b_sc_group_stride;   // bytes between experts' B scale buffers (M mode)
};

struct TileInfo {
  int g;
  int nk;              // number of 128-deep K steps (0: empty K group)
  int kt0;             // first K step (in units of 128)
  int64_t a_row0;      // first row of A
  int64_t b_row0;      // first row of B (global row of the TMA map)
  int64_t b_loc0;      // first row of B inside its scale buffer
  int64_t n0;          // first output column
  int64_t m_row0;      // M mode: first padded row; K mode: first output row
};

template <int kMode>
__device__ __forceinline__ TileInfo decode_tile(int64_t tile, const GemmArgs& a, const int32_t* ends,
                                                const int32_t* pstart) {
  TileInfo t;
  if (kMode == kGroupsM) {
    const int64_t nt = a.N / kBN;
    const int64_t mt = tile / nt;
    t.n0 = (tile % nt) * kBN;
    t.m_row0 = mt * kBM;
    int lo = 0, hi = a.G;   // largest g with pstart[g] <= row
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pstart[mid] <= t.m_row0) lo = mid; else hi = mid;
    }
    t.g = lo;
    t.nk = int(a.K / kBK);
    t.kt0 = 0;
    t.a_row0 = t.m_row0;
    t.b_loc0 = t.n0;
    t.b_row0 = int64_t(t.g) * a.N + t.n0;
  } else {
    const int64_t nt = a.K / kBN, mt = a.N / kBM;
    const int64_t per_g = nt * mt;
    t.g = int(tile / per_g);
    const int64_t rem = tile % per_g;
    t.m_row0 = (rem / nt) * kBM;
    t.n0 = (rem % nt) * kBN;
    const int64_t start = t.g ? ends[t.g - 1] : 0;
    const int64_t size = ends[t.g] - start;
    t.kt0 = int(pstart[t.g] / kBK);
    t.nk = int((size + kBK - 1) / kBK);
    t.a_row0 = t.m_row0;
    t.b_loc0 = t.n0;
    t.b_row0 = t.n0;
  }
  return t;
}

// Waits, bounded by time only (used to drain copies and MMAs before exit).
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > kWaitLimitNs) {
      flag_error(kErrTimeout);
      return;
    }
  }
}

template <int kMode>
__global__ void __launch_bounds__(kGemmThreads, 1)
mx_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
               const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kOffBar;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
  const uint32_t acc_full = bar0 + 8u * (2 * kStages);
  const uint32_t acc_empty = acc_full + 8u;
  const uint32_t done_bar = acc_full + 16u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  int64_t* info = reinterpret_cast<int64_t*>(smem + kOffMisc + 8);        // [0] total tiles
  int32_t* ends = reinterpret_cast<int32_t*>(smem + kOffEnds);
  int32_t* pstart = reinterpret_cast<int32_t*>(smem + kOffPstart);

  // ---------------------------------------------------------------- setup --
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_b);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4);
    mbar_init(done_bar, 1);
    fence_barrier_init();
    *abort_flag = 0;
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0) {
    // group table: ends[g] and padded starts pstart[0..G]
    bool bad = false;
    if (args.offs == nullptr) {
      if (lane == 0) {
        const int64_t len = args.M;
        ends[0] = int32_t(len);
        pstart[0] = 0;
        pstart[1] = int32_t(ceil_to(len, kBM));
      }
    } else {
      const unsigned full = 0xFFFFFFFFu;
      int64_t carry = 0, prev_end = 0;
      if (lane == 0) pstart[0] = 0;
      for (int base = 0; base < args.G; base += 32) {
        const int g = base + lane;
        const bool in = g < args.G;
        const int64_t e = in ? int64_t(__ldg(args.offs + g)) : 0;
        int64_t s = __shfl_up_sync(full, e, 1);
        if (lane == 0) s = prev_end;
        const int64_t size = in ? e - s : 0;
        if (in && size < 0) bad = true;
        const int64_t pad = size > 0 ? ceil_to(size, kBM) : 0;
        int64_t incl = pad;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int64_t t = __shfl_up_sync(full, incl, o);
          if (lane >= o) incl += t;
        }
        if (in) {
          ends[g] = int32_t(e);
          pstart[g + 1] = int32_t(carry + incl);
        }
        carry = __shfl_sync(full, carry + incl, 31);
        prev_end = __shfl_sync(full, e, min(31, args.G - 1 - base));
      }
      bad = __any_sync(full, bad);
      if (prev_end != args.M || carry > args.m_cap) bad = true;
    }
    if (lane == 0) {
      const int G = args.offs ? args.G : 1;
      int64_t total;
      if (kMode == kGroupsM) total = bad ? 0 : int64_t(pstart[G] / kBM) * (args.N / kBN);
      else total = bad ? 0 : int64_t(G) * (args.N / kBM) * (args.K / kBN);
      if (bad) flag_error(kErrOffsets);
      info[0] = total;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int64_t total_tiles = info[0];
  GemmArgs a = args;
  if (a.offs == nullptr) a.G = 1;

  // ----------------------------------------------------------- producer ---
  if (warp == 4) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;   // bit s: stage s has a load in flight or landed
      uint32_t last_par = 0; // bit s: parity of the last phase issued on stage s
      for (int64_t tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
        const TileInfo t = decode_tile<kMode>(tile, a, ends, pstart);
        const uint8_t* sfa = a.a_s + (t.a_row0 / kBM) * a.a_sc_tiles * 512;
        const uint8_t* sfb = a.b_s + int64_t(kMode == kGroupsM ? t.g : 0) * a.b_sc_group_stride +
                             (t.b_loc0 / kBM) * a.b_sc_tiles * 512;
        bool ok = true;
        for (int kt = 0; kt < t.nk; ++kt) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) { ok = false; break; }
          const int kk = t.kt0 + kt;
          const uint32_t fb = full_bar(stage);
          mbar_arrive_expect_tx(fb, kTxBytes);
          tma_load_2d(sbase + kOffA + stage * kABytes, &map_a, kk * kBK, int32_t(t.a_row0), fb);
          tma_load_2d(sbase + kOffB + stage * kBBytes, &map_b, kk * kBK, int32_t(t.b_row0), fb);
          bulk_load(sbase + kOffSfa + stage * kSfaBytes, sfa + int64_t(kk) * 512, 512, fb);
          bulk_load(sbase + kOffSfb + stage * kSfbBytes, sfb + int64_t(kk) * 512, 512, fb);
          bulk_load(sbase + kOffSfb + stage * kSfbBytes + 512, sfb + (a.b_sc_tiles + kk) * 512, 512, fb);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      // every issued copy must land before this CTA's shared memory is released
      for (int s = 0; s < kStages; ++s)
        if (issued & (1u << s)) mbar_drain(full_bar(s), (last_par >> s) & 1u);
    }
    __syncwarp();
  }
  // ---------------------------------------------------------------- MMA ---
  else if (warp == 5) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      const uint32_t d_tmem = tmem + kAccCol;
      for (int64_t tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
        const TileInfo t = decode_tile<kMode>(tile, a, ends, pstart);
        if (t.nk == 0) continue;
        if (!mbar_wait(acc_empty, acc_phase ^ 1u, abort_flag)) break;
        tc_fence_after();
        bool ok = true;
        for (int kt = 0; kt < t.nk; ++kt) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sfa_t = tmem + kSfaCol + 4u * stage;
          const uint32_t sfb_t = tmem + kSfbCol + 8u * stage;
          const uint32_t sfa_s = sbase + kOffSfa + stage * kSfaBytes;
          const uint32_t sfb_s = sbase + kOffSfb + stage * kSfbBytes;
          tmem_cp_32x128b_x4(sfa_t, smem_desc(sfa_s, 0, 128, 0));
          tmem_cp_32x128b_x4(sfb_t, smem_desc(sfb_s, 0, 128, 0));
          tmem_cp_32x128b_x4(sfb_t + 4, smem_desc(sfb_s + 512, 0, 128, 0));
          const uint32_t a_s = sbase + kOffA + stage * kABytes;
          const uint32_t b_s = sbase + kOffB + stage * kBBytes;
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k) {
            const uint64_t ad = smem_desc(a_s + 32u * k, 16, 1024, 2);
            const uint64_t bd = smem_desc(b_s + 32u * k, 16, 1024, 2);
            const uint32_t idesc = kIdescBase | (uint32_t(k) << 4) | (uint32_t(k) << 29);
            mma_mxf8(d_tmem, ad, bd, idesc, sfa_t, sfb_t, (kt | k) != 0 ? 1u : 0u);
          }
          tc_commit(empty_bar(stage));
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(acc_full);
        acc_phase ^= 1u;
      }
      // all MMAs of this thread complete before TMEM is released
      tc_commit(done_bar);
      mbar_drain(done_bar, 0);
    }
    __syncwarp();
  }
  // ----------------------------------------------------------- epilogue ---
  else {
    uint32_t acc_phase = 0;
    const int r = warp * 32 + lane;
    const uint32_t t_lane = tmem + (uint32_t(warp * 32) << 16) + kAccCol;
    for (int64_t tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      const TileInfo t = decode_tile<kMode>(tile, a, ends, pstart);
      __nv_bfloat16* dst = nullptr;
      if (kMode == kGroupsM) {
        const int64_t start = t.g ? ends[t.g - 1] : 0;
        const int64_t local = t.m_row0 + r - pstart[t.g];
        if (local < ends[t.g] - start) dst = a.out + (start + local) * a.N + t.n0;
      } else {
        dst = a.out + (int64_t(t.g) * a.N + t.m_row0 + r) * a.K + t.n0;
      }
      if (t.nk == 0) {
        if (dst) {
          const uint4 z = make_uint4(0u, 0u, 0u, 0u);
          for (int c = 0; c < kBN; c += 8) *reinterpret_cast<uint4*>(dst + c) = z;
        }
        continue;
      }
      if (!mbar_wait(acc_full, acc_phase, abort_flag)) break;
      tc_fence_after();
#pragma unroll 1
      for (int chunk = 0; chunk < kBN / 32; ++chunk) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(t_lane + uint32_t(chunk * 32), v);
        tmem_ld_wait();
        if (dst) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + chunk * 32);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint4 o;
            o.x = pack_bf16x2(__uint_as_float(v[8 * j + 0]), __uint_as_float(v[8 * j + 1]));
            o.y = pack_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3]));
            o.z = pack_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5]));
            o.w = pack_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7]));
            d4[j] = o;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      acc_phase ^= 1u;
    }
  }

  // ------------------------------------------------------------ teardown ---
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace mx
