// MXFP8 scaled grouped GEMM on sm_100a tensor cores (tcgen05 CTA pairs, TMEM, TMA).
//
// Computes, in fp32 with a bf16 result, the grouped products of the MXFP8
// grouped GEMM over an offsets array (ao "[moe training] Add
// backward_override to the MXFP8 grouped GEMM", Summary: forward, dgrad and
// wgrad of _MXFP8GroupedMM; ao PR #4705, "MXFP8 MoE grouped-mm"):
//
//   M-groups (forward, dgrad): out[rows of g, :] = A[padded rows of g, :] * B[g]^T
//     A codes [rows_a, K] (padded token rows), B codes [G, N, K], out [M, N];
//     or B codes [G, K, N] read MN-major (the dgrad from the forward's weight
//     codes, no transposed copy).
//   K-groups (wgrad):          out[g] = A[:, tokens of g] * B[:, tokens of g]^T
//     A codes [N, m_cap], B codes [K, m_cap] (padded token columns), out [G, N, K].
//
// Operands are E4M3 with blocked E8M0 scales along K (K-major, except B in
// the MN-major M-groups form); each token group
// starts on a 128-row boundary of the padded layout (the pad path), so every
// 128-row scale tile and every 128-wide K tile belongs to one group.
//
// Design: clusters of two CTAs (one per SM) compute 256x256 output tiles
// with the pair form of the block-scaled MMA. Per 128-deep K step each CTA
// loads, by TMA into its own shared memory, its 128 rows of A, its 128-row
// half of B, the 512-byte scale tile of its A rows and both scale tiles of
// the pair's 256 B rows; all loads count on the leader CTA's stage barrier.
// Per MMA this moves half the shared-memory and L2 bytes of a one-CTA 128x256
// tile; under the 1 kW power cap that buys clock (measured: 1989 against
// 1830 TFLOP/s sustained on 8192^3).
//   warp 4 (both CTAs)   TMA producer over a 6-stage ring.
//   warp 5 (leader only) MMA issuer: tcgen05.cp.cta_group::2 of the scale
//                        tiles into each CTA's TMEM, four
//                        tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale
//                        (M=256, N=256, K=32) into a 128x256 fp32 accumulator
//                        per CTA, and tcgen05.commit multicast to both CTAs
//                        to free the stage / signal the epilogue.
//   warps 0-3 (both)     epilogue: tcgen05.ld of the CTA's 128 accumulator
//                        rows into registers (bf16, round to nearest even),
//                        TMEM released to the leader, then stores with the
//                        padded->unpadded row map (the unpad step is fused
//                        here), staged through shared memory so each store
//                        instruction writes whole 64-byte row segments, while
//                        the next tile's MMAs already run.
// Two accumulator slots overlap in one 32-column subtile of TMEM; the
// epilogue drains that subtile first, so the next tile's MMAs start almost
// as soon as the previous tile ends.
// 256-row tiles are enumerated per group; a group's last tile may extend past
// the group, and those rows are computed but never stored. Static round robin
// over tiles; group boundaries come from a per-CTA scan of the device offsets,
// so there is no host synchronisation. An empty group in K-groups mode
// writes exact zeros. No split-K and no atomics: results are deterministic.
// No TMA multicast is used.
#pragma once

#include <type_traits>

#include "mx_sm100.cuh"

namespace mx {

constexpr int kPairM = 256, kCtaM = 128, kBN = 256, kBK = 128;
constexpr int kBM = kCtaM;
constexpr int kStages = 6;
constexpr int kGemmThreads = 192;
constexpr uint32_t kABytes = kCtaM * kBK;                 // 16 KB per CTA
constexpr uint32_t kBBytes = (kBN / 2) * kBK;             // 16 KB per CTA (half of B)
constexpr uint32_t kSfaBytes = 512, kSfbBytes = 1024;
constexpr uint32_t kTxBytes = 2 * (kABytes + kBBytes + kSfaBytes + kSfbBytes);   // both CTAs
// TMEM: two accumulator slots that overlap in one 32-column subtile
// (slot 0 = columns 0..255, slot 1 = columns 224..479) so the next tile's
// MMAs can start as soon as the epilogue has drained that subtile of the
// previous tile; scale factors use a two-slot ring at columns 480..503.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccSlot1 = 224;
constexpr uint32_t kOverlapCol = 224;                     // shared subtile [224, 256)
constexpr uint32_t kSfCol = 480;                          // slot k: SFA at +12k (4), SFB at +12k+4 (8)
static_assert(kSfCol + 24 <= kTmemCols, "TMEM budget");

// shared-memory map (offsets from a 1024-byte aligned base; identical in both CTAs)
constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + kStages * kABytes;
constexpr uint32_t kOffSfa = kOffB + kStages * kBBytes;
constexpr uint32_t kOffSfb = kOffSfa + kStages * kSfaBytes;
constexpr uint32_t kOffBar = kOffSfb + kStages * kSfbBytes;
constexpr uint32_t kNumBars = 2 * kStages + 6;            // full, empty, acc_full[2], acc_free[2], ovl_free, done
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;     // tmem slot, abort, info words
constexpr uint32_t kOffEnds = kOffMisc + 64;
constexpr uint32_t kOffPstart = kOffEnds + 4 * kMaxGroups;
constexpr uint32_t kOffTstart = kOffPstart + 4 * (kMaxGroups + 1);
constexpr uint32_t kOffStage = (kOffTstart + 4 * (kMaxGroups + 1) + 127) & ~127u;   // epilogue staging
constexpr uint32_t kStageWarpBytes = 32 * 64;            // 32 rows x 32 bf16 per epilogue warp
constexpr uint32_t kGemmSmem = kOffStage + 4 * kStageWarpBytes + 1024;   // + alignment slack
static_assert(kGemmSmem <= 227 * 1024, "shared memory budget");

// Instruction descriptor of kind::mxf8f6f4 with block scaling: E4M3 A and B
// (format 0), both K-major, N>>3 in bits [17,23), E8M0 scales (bit 23),
// M>>4 in bits [24,29) (M = 256 for the pair); the scale-factor byte ids
// (bits [4,6) for B and [29,31) for A) select which of the four K blocks
// packed in each TMEM scale column this MMA uses.
constexpr uint32_t kIdescBase = (uint32_t(kBN >> 3) << 17) | (1u << 23) | (uint32_t(kPairM >> 4) << 24);

// kGroupsMKn: M groups with B stored [G, K, N] (N contiguous), read as an
// MN-major operand -- the dgrad straight from the forward's weight codes.
enum GemmMode : int { kGroupsM = 0, kGroupsK = 1, kGroupsMKn = 2 };

struct GemmArgs {
  const int32_t* offs;         // cumulative group ends, or null for one dense group
  __nv_bfloat16* out;
  int G;
  int E;                       // experts: group g uses expert g % E (E == G: one expert per group)
  int64_t M, N, K;             // see the mode description above
  int64_t m_cap;               // padded capacity (rows of A in M mode, token columns in K mode)
  int64_t a_sc_tiles;          // 4-column scale tiles (512-byte chunks) per 128-row band of A
  int64_t b_sc_tiles;          // same for B
  int64_t b_sc_group_chunks;   // chunks between experts' B scale buffers (M mode)
};

struct TileInfo {
  int g;               // M modes: the group; K mode: the expert (output matrix)
  int nk;              // number of 128-deep K steps (0: every K group of the expert is empty)
  int kt0;             // M modes: first K step (in units of 128)
  int64_t m0;          // first row of A for the pair (M mode: padded row)
  int64_t b_row0;      // first row of B for the pair (global row of the TMA map)
  int64_t b_chunk0;    // scale chunk of B's first 128 rows at K step 0
  int64_t n0;          // first output column
};

template <int kMode>
__device__ __forceinline__ TileInfo decode_tile(int64_t tile, const GemmArgs& a, const int32_t* ends,
                                                const int32_t* pstart, const int32_t* tstart) {
  TileInfo t;
  if (kMode != kGroupsK) {
    const int64_t nt = ceil_div(a.N, kBN);
    const int64_t mt = tile / nt;
    t.n0 = (tile % nt) * kBN;
    int lo = 0, hi = a.G;   // largest g with tstart[g] <= mt
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (tstart[mid] <= mt) lo = mid; else hi = mid;
    }
    t.g = lo;
    t.m0 = pstart[t.g] + (mt - tstart[t.g]) * kPairM;
    t.nk = int(ceil_div(a.K, kBK));
    t.kt0 = 0;
    const int64_t we = t.g % a.E;     // the group's expert
    t.b_row0 = kMode == kGroupsMKn ? we * a.K : we * a.N + t.n0;
    t.b_chunk0 = we * a.b_sc_group_chunks + (t.n0 / kCtaM) * a.b_sc_tiles;
  } else {
    // output matrix e sums the token steps of groups e, e + E, e + 2E, ...
    const int64_t nt = ceil_div(a.K, kBN), mt = ceil_div(a.N, kPairM);
    const int64_t per_e = nt * mt;
    t.g = int(tile / per_e);
    const int64_t rem = tile % per_e;
    t.m0 = (rem / nt) * kPairM;
    t.n0 = (rem % nt) * kBN;
    t.kt0 = 0;
    int64_t nk = 0;
    for (int g = t.g; g < a.G; g += a.E) {
      const int64_t start = g ? ends[g - 1] : 0;
      nk += ceil_div(ends[g] - start, kBK);
    }
    t.nk = int(nk);
    t.b_row0 = t.n0;
    t.b_chunk0 = (t.n0 / kCtaM) * a.b_sc_tiles;
  }
  return t;
}

// The 128-deep K steps of a tile in order: in M modes steps kt0, kt0 + 1, ...;
// in K mode the padded token steps of groups e, e + E, e + 2E, ... (the groups
// of expert e, empty ones skipped).
struct KWalk {
  int g;          // current group (K mode)
  int left;       // steps left in it
  int64_t kk;     // current step
};

template <int kMode>
__device__ __forceinline__ KWalk kwalk_begin(const TileInfo& t, const GemmArgs& a) {
  KWalk w;
  w.g = kMode == kGroupsK ? t.g - a.E : t.g;
  w.left = kMode == kGroupsK ? 0 : t.nk;
  w.kk = t.kt0;
  return w;
}

// The step to load now; call only while steps of the tile remain.
template <int kMode>
__device__ __forceinline__ int64_t kwalk_step(KWalk& w, const GemmArgs& a, const int32_t* ends,
                                              const int32_t* pstart) {
  if (kMode == kGroupsK) {
    while (w.left == 0) {
      w.g += a.E;
      const int64_t start = w.g ? ends[w.g - 1] : 0;
      w.left = int(ceil_div(ends[w.g] - start, kBK));
      w.kk = pstart[w.g] / kBK;
    }
  }
  const int64_t kk = w.kk;
  ++w.kk;
  --w.left;
  return kk;
}

// ------------------------------------------------------------ epilogue ---
// One warp's part of a 256-column output tile: its 32 accumulator rows in
// TMEM slot `slot` (lane i of the warp owns row i; `dst` is that row's first
// output element, or null for a row that is not stored).
// The whole accumulator row is converted into registers (256 bf16 in 128
// words, round to nearest even) so that TMEM is released before the global
// stores, which then overlap the next tile's main loop. The 32-column subtile
// shared with the other slot is drained first and released at once
// (`leader_ovl`), then the rest of the slot (`leader_free`), both barriers of
// the pair's leader CTA, with relaxed arrives (the columns are read out, no
// data is handed over).
// Stores are coalesced: per 32-column chunk the warp's 32 rows go through a
// 2 KB shared buffer (16-byte pieces XOR-swizzled by row so both sides are
// bank-conflict free), then each instruction writes 8 rows x 64 contiguous
// bytes -- whole sectors instead of half-filled ones.
__device__ __forceinline__ void epilogue_tile(uint32_t lane_base, uint32_t slot, __nv_bfloat16* dst,
                                              uint32_t leader_ovl, uint32_t leader_free, uint8_t* stage_buf,
                                              int lane, int64_t cols_valid) {
  const uint32_t t_acc = lane_base + (slot ? kAccSlot1 : 0u);
  uint32_t rowv[kBN / 2];
  auto drain = [&](int chunk) {
    uint32_t v[32];
    tmem_ld_32x32b_x32(t_acc + uint32_t(chunk * 32), v);
    tmem_ld_wait();
#pragma unroll
    for (int jj = 0; jj < 16; ++jj)
      rowv[chunk * 16 + jj] = pack_bf16x2(__uint_as_float(v[2 * jj]), __uint_as_float(v[2 * jj + 1]));
  };
  auto release_shared_subtile = [&]() {
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster_relaxed(leader_ovl);
  };
  if (slot) {              // shared subtile = chunk 0 of slot 1
    drain(0);
    release_shared_subtile();
#pragma unroll
    for (int c = 1; c < kBN / 32; ++c) drain(c);
  } else {                 // shared subtile = chunk 7 of slot 0
    drain(kBN / 32 - 1);
    release_shared_subtile();
#pragma unroll
    for (int c = 0; c < kBN / 32 - 1; ++c) drain(c);
  }
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive_cluster_relaxed(leader_free);
  // the rows this lane stores from, gathered once: row i * 8 + lane / 4, i < 4
  const uint64_t mine = reinterpret_cast<uintptr_t>(dst);
  uint64_t rows[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) rows[i] = __shfl_sync(0xFFFFFFFFu, mine, i * 8 + (lane >> 2));
#pragma unroll
  for (int chunk = 0; chunk < kBN / 32; ++chunk) {
    if (chunk * 32 >= cols_valid) break;     // columns past the output (N or K not a multiple of 256)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t phys = uint32_t(k) ^ ((uint32_t(lane) >> 1) & 3u);
      *reinterpret_cast<uint4*>(stage_buf + lane * 64 + phys * 16) =
          make_uint4(rowv[chunk * 16 + 4 * k], rowv[chunk * 16 + 4 * k + 1], rowv[chunk * 16 + 4 * k + 2],
                     rowv[chunk * 16 + 4 * k + 3]);
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int rr = i * 8 + (lane >> 2);       // row within the warp's 32
      const int k = lane & 3;                   // 16-byte piece within the 64-byte segment
      const uint4 val = *reinterpret_cast<const uint4*>(stage_buf + rr * 64 + ((uint32_t(k) ^ ((uint32_t(rr) >> 1) & 3u)) * 16));
      if (rows[i]) {
        __nv_bfloat16* d = reinterpret_cast<__nv_bfloat16*>(rows[i]);
        *reinterpret_cast<uint4*>(d + chunk * 32 + k * 8) = val;
      }
    }
    __syncwarp();
  }
}

// Exact zeros for one output row of a 256-column tile (an empty K group), if stored.
__device__ __forceinline__ void store_zero_row(__nv_bfloat16* dst, int64_t cols_valid) {
  if (dst) {
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    const int n = cols_valid < kBN ? int(cols_valid) : kBN;
    for (int c = 0; c < n; c += 8) *reinterpret_cast<uint4*>(dst + c) = z;
  }
}

// Per-group output rows (M-group modes): row i of group g is written at
// base[g] + i * N instead of out + (start_g + i) * N. A base may be another
// GPU's memory (the expert-parallel combine: each group's outputs stored
// straight into the rank that sent its tokens, tile by tile as the GEMM
// runs). The kernels without it take an empty parameter.
struct RowDests {
  __nv_bfloat16* base[kMaxGroups];
};
struct NoRowDests {};
template <bool kRowDests>
using RowDestsT = typename std::conditional<kRowDests, RowDests, NoRowDests>::type;

template <int kMode, bool kRowDests = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
mx_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
               const __grid_constant__ CUtensorMap map_sfa, const __grid_constant__ CUtensorMap map_sfb,
               const GemmArgs args, const __grid_constant__ RowDestsT<kRowDests> rdests) {
  static_assert(!kRowDests || kMode != kGroupsK, "per-group output rows are for the M-group modes");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();      // 0 = leader of the pair
  const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kOffBar;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
  const uint32_t acc_full0 = bar0 + 8u * (2 * kStages);   // + 8 * slot
  const uint32_t acc_free0 = acc_full0 + 16u;              // + 8 * slot
  const uint32_t ovl_free = acc_full0 + 32u;
  const uint32_t done_bar = acc_full0 + 40u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  int64_t* info = reinterpret_cast<int64_t*>(smem + kOffMisc + 8);        // [0] total tiles
  int32_t* ends = reinterpret_cast<int32_t*>(smem + kOffEnds);
  int32_t* pstart = reinterpret_cast<int32_t*>(smem + kOffPstart);
  int32_t* tstart = reinterpret_cast<int32_t*>(smem + kOffTstart);

  // ---------------------------------------------------------------- setup --
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_b);
    tma_prefetch_desc(&map_sfa);
    tma_prefetch_desc(&map_sfb);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(acc_full0, 1);
    mbar_init(acc_full0 + 8, 1);
    mbar_init(acc_free0, 8);      // four epilogue warps in each CTA of the pair
    mbar_init(acc_free0 + 8, 8);
    mbar_init(ovl_free, 8);
    mbar_init(done_bar, 1);
    fence_barrier_init();
    *abort_flag = 0;
  }
  if (warp == 5) {
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == 0) {
    // group table: ends[g], padded starts pstart[0..G], 256-row tile starts tstart[0..G]
    bool bad = false;
    const int G = args.offs ? args.G : 1;
    if (args.offs == nullptr) {
      if (lane == 0) {
        ends[0] = int32_t(args.M);
        pstart[0] = 0;
        pstart[1] = int32_t(ceil_to(args.M, kCtaM));
        tstart[0] = 0;
        tstart[1] = int32_t(ceil_div(args.M, kPairM));
      }
    } else {
      const unsigned full = 0xFFFFFFFFu;
      int64_t carry = 0, tcarry = 0, prev_end = 0;
      if (lane == 0) {
        pstart[0] = 0;
        tstart[0] = 0;
      }
      for (int base = 0; base < G; base += 32) {
        const int g = base + lane;
        const bool in = g < G;
        const int64_t e = in ? int64_t(__ldg(args.offs + g)) : 0;
        int64_t s = __shfl_up_sync(full, e, 1);
        if (lane == 0) s = prev_end;
        const int64_t size = in ? e - s : 0;
        if (in && size < 0) bad = true;
        const int64_t pad = size > 0 ? ceil_to(size, kCtaM) : 0;
        const int64_t ntl = ceil_div(pad, kPairM);
        int64_t incl = pad, tincl = ntl;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int64_t t = __shfl_up_sync(full, incl, o);
          const int64_t u = __shfl_up_sync(full, tincl, o);
          if (lane >= o) {
            incl += t;
            tincl += u;
          }
        }
        if (in) {
          ends[g] = int32_t(e);
          pstart[g + 1] = int32_t(carry + incl);
          tstart[g + 1] = int32_t(tcarry + tincl);
        }
        carry = __shfl_sync(full, carry + incl, 31);
        tcarry = __shfl_sync(full, tcarry + tincl, 31);
        prev_end = __shfl_sync(full, e, min(31, G - 1 - base));
      }
      bad = __any_sync(full, bad);
      if (prev_end != args.M || carry > args.m_cap) bad = true;
    }
    if (lane == 0) {
      int64_t total;
      if (kMode != kGroupsK) total = bad ? 0 : int64_t(tstart[G]) * ceil_div(args.N, kBN);
      else total = bad ? 0 : int64_t(args.offs ? args.E : 1) * ceil_div(args.N, kPairM) * ceil_div(args.K, kBN);
      if (bad && rank == 0) flag_error(kErrOffsets);
      info[0] = total;
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();          // the pair's barriers are initialised before any remote use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int64_t total_tiles = info[0];
  GemmArgs a = args;
  if (a.offs == nullptr) a.G = a.E = 1;

  // ----------------------------------------------------------- producer ---
  if (warp == 4) {
    {
      // The whole warp runs the loop (warp-uniform state); one elected lane
      // issues the copies.
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_par = 0;
      for (int64_t tile = pair; tile < total_tiles; tile += npairs) {
        const TileInfo t = decode_tile<kMode>(tile, a, ends, pstart, tstart);
        const int32_t a_row = int32_t(t.m0 + kCtaM * rank);
        const int32_t b_row = int32_t(t.b_row0 + (kBN / 2) * rank);
        const int64_t sfa_chunk0 = ((t.m0 + kCtaM * rank) / kCtaM) * a.a_sc_tiles;
        bool ok = true;
        KWalk walk = kwalk_begin<kMode>(t, a);
        for (int kt = 0; kt < t.nk; ++kt) {
          if (!mbar_wait_warp(empty_bar(stage), phase ^ 1u, abort_flag)) { ok = false; break; }
          const int kk = int(kwalk_step<kMode>(walk, a, ends, pstart));
          const uint32_t fb = full_bar(stage);
          if (elect_one()) {
            if (rank == 0) mbar_arrive_expect_tx(fb, kTxBytes);
            const uint32_t lb = mapa_shared(fb, 0);
            tma_load_2d_pair(sbase + kOffA + stage * kABytes, &map_a, kk * kBK, a_row, lb);
            if (kMode == kGroupsMKn)     // 128 K rows x this CTA's 128 N columns
              tma_load_2d_pair(sbase + kOffB + stage * kBBytes, &map_b, int32_t(t.n0 + (kBN / 2) * rank),
                               int32_t(t.b_row0 + int64_t(kk) * kBK), lb);
            else
              tma_load_2d_pair(sbase + kOffB + stage * kBBytes, &map_b, kk * kBK, b_row, lb);
            tma_load_2d_pair(sbase + kOffSfa + stage * kSfaBytes, &map_sfa, 0, int32_t(sfa_chunk0 + kk), lb);
            tma_load_2d_pair(sbase + kOffSfb + stage * kSfbBytes, &map_sfb, 0, int32_t(t.b_chunk0 + kk), lb);
            tma_load_2d_pair(sbase + kOffSfb + stage * kSfbBytes + 512, &map_sfb, 0,
                             int32_t(t.b_chunk0 + a.b_sc_tiles + kk), lb);
          }
          __syncwarp();
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      // the leader's stages count both CTAs' copies: wait for them to land
      if (rank == 0 && lane == 0)
        for (int s = 0; s < kStages; ++s)
          if (issued & (1u << s)) mbar_drain(full_bar(s), (last_par >> s) & 1u);
    }
    __syncwarp();
  }
  // ------------------------------------------------------ MMA (leader) ---
  else if (warp == 5) {
    if (rank == 0) {
      // The whole warp runs the loop so that descriptors and TMEM addresses
      // stay warp-uniform; one elected lane issues each tcgen05 group.
      int stage = 0;
      uint32_t phase = 0;
      uint32_t tiles_done = 0, ksteps = 0;
      // Descriptors of stage 0 / K block 0, built once. A descriptor's start
      // address field holds (address >> 4) in its low bits, so moving to
      // another stage or K block is one 64-bit add; the issue loop below is
      // then a handful of instructions per MMA and keeps the tensor pipe fed.
      const uint64_t a_desc0 = smem_desc(sbase + kOffA, 16, 1024, 2);
      // B MN-major (kGroupsMKn): one 128-byte swizzle atom of N per CTA, K rows
      // 128 bytes apart in 8-row groups 1024 bytes apart, so a 32-deep K block
      // is four groups (+4096 bytes); K-major: +32 bytes per K block.
      const uint64_t b_desc0 = kMode == kGroupsMKn ? smem_desc(sbase + kOffB, kBBytes, 1024, 2)
                                                   : smem_desc(sbase + kOffB, 16, 1024, 2);
      constexpr uint64_t kBStep = kMode == kGroupsMKn ? (4096 >> 4) : (32 >> 4);
      constexpr uint32_t kIdesc = kIdescBase | (kMode == kGroupsMKn ? (1u << 16) : 0u);
      // N = 128: the pair MMA's columns [0, 64) are the first CTA's B rows [0, 64)
      // with their scales in the same TMEM columns as at N = 256
      constexpr uint32_t kIdescNarrow = (kIdesc & ~(0x3Fu << 17)) | (uint32_t(128 >> 3) << 17);
      const uint64_t sfa_desc0 = smem_desc(sbase + kOffSfa, 0, 128, 0);
      const uint64_t sfb_desc0 = smem_desc(sbase + kOffSfb, 0, 128, 0);
      for (int64_t tile = pair; tile < total_tiles; tile += npairs) {
        const TileInfo t = decode_tile<kMode>(tile, a, ends, pstart, tstart);
        if (t.nk == 0) continue;
        const uint32_t slot = tiles_done & 1u, use = tiles_done >> 1;
        // this slot's previous tile fully drained, and the previous tile's
        // shared subtile drained
        if (!mbar_wait_warp(acc_free0 + 8u * slot, (use & 1u) ^ 1u, abort_flag)) break;
        if (!mbar_wait_warp(ovl_free, (tiles_done & 1u) ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (slot ? kAccSlot1 : 0u);
        // a tile at a ragged edge with at most 64 output columns (all from the first
        // CTA's B rows) runs its MMAs at N = 128, half the tensor work; the columns
        // this leaves stale are past the output and never stored. B read MN-major
        // (the dgrad) keeps N = 256: its shared-memory layout is fixed per 128 columns.
        const int64_t cols_valid = (kMode == kGroupsK ? a.K : a.N) - t.n0;
        const uint32_t idesc = (kMode != kGroupsMKn && cols_valid <= 64) ? kIdescNarrow : kIdesc;
        bool ok = true;
        for (int kt = 0; kt < t.nk; ++kt) {
          // The TMA bytes of this stage are visible to the tensor core once
          // the stage barrier's phase completes (both are async-proxy
          // accesses ordered by the mbarrier), so no fence is needed here.
          if (!mbar_wait_warp(full_bar(stage), phase, abort_flag)) { ok = false; break; }
          // scale tiles: two-slot ring; tcgen05.cp and tcgen05.mma issued by
          // one thread execute in issue order
          const uint32_t sfa_t = tmem + kSfCol + 12u * (ksteps & 1u);
          const uint32_t sfb_t = sfa_t + 4u;
          const uint64_t ad = a_desc0 + uint64_t((stage * kABytes) >> 4);
          const uint64_t bd = b_desc0 + uint64_t((stage * kBBytes) >> 4);
          const uint32_t acc0 = kt != 0 ? 1u : 0u;
          if (elect_one()) {
            tmem_cp_32x128b_x4_pair(sfa_t, sfa_desc0 + uint64_t((stage * kSfaBytes) >> 4));
            tmem_cp_32x128b_x4_pair(sfb_t, sfb_desc0 + uint64_t((stage * kSfbBytes) >> 4));
            tmem_cp_32x128b_x4_pair(sfb_t + 4, sfb_desc0 + uint64_t((stage * kSfbBytes + 512) >> 4));
            // K block k of the 128-deep stage: +32 bytes (2 in the >>4 field)
            mma_mxf8_pair(d_tmem, ad, bd, idesc, sfa_t, sfb_t, acc0);
            mma_mxf8_pair(d_tmem, ad + 2, bd + kBStep, idesc | (1u << 4) | (1u << 29), sfa_t, sfb_t, 1u);
            mma_mxf8_pair(d_tmem, ad + 4, bd + 2 * kBStep, idesc | (2u << 4) | (2u << 29), sfa_t, sfb_t, 1u);
            mma_mxf8_pair(d_tmem, ad + 6, bd + 3 * kBStep, idesc | (3u << 4) | (3u << 29), sfa_t, sfb_t, 1u);
            tc_commit_pair(empty_bar(stage));
          }
          __syncwarp();
          ++ksteps;
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (elect_one()) tc_commit_pair(acc_full0 + 8u * slot);
        __syncwarp();
        ++tiles_done;
      }
      // all MMAs of the pair complete before either CTA releases TMEM
      if (elect_one()) {
        tc_commit_pair(done_bar);
        mbar_drain(done_bar, 0);
      }
    }
    __syncwarp();
  }
  // ----------------------------------------------------------- epilogue ---
  else {
    uint32_t tiles_done = 0;
    const int r = warp * 32 + lane;
    const uint32_t lane_base = tmem + (uint32_t(warp * 32) << 16);
    const uint32_t leader_ovl = mapa_shared(ovl_free, 0);
    const uint32_t leader_free0 = mapa_shared(acc_free0, 0);
    uint8_t* stage_buf = smem + kOffStage + warp * kStageWarpBytes;
    for (int64_t tile = pair; tile < total_tiles; tile += npairs) {
      const TileInfo t = decode_tile<kMode>(tile, a, ends, pstart, tstart);
      const int64_t row = t.m0 + kCtaM * rank + r;
      __nv_bfloat16* dst = nullptr;
      int64_t cols_valid;           // output columns of this tile (fewer than 256 at a ragged edge)
      if (kMode != kGroupsK) {
        const int64_t start = t.g ? ends[t.g - 1] : 0;
        const int64_t local = row - pstart[t.g];
        if (local < ends[t.g] - start) {
          if constexpr (kRowDests) dst = rdests.base[t.g] + local * a.N + t.n0;
          else dst = a.out + (start + local) * a.N + t.n0;
        }
        cols_valid = a.N - t.n0;
      } else {
        if (row < a.N) dst = a.out + (int64_t(t.g) * a.N + row) * a.K + t.n0;
        cols_valid = a.K - t.n0;
      }
      if (t.nk == 0) {
        store_zero_row(dst, cols_valid);
        continue;
      }
      const uint32_t slot = tiles_done & 1u, use = tiles_done >> 1;
      if (!mbar_wait(acc_full0 + 8u * slot, use & 1u, abort_flag)) break;
      tc_fence_after();
      epilogue_tile(lane_base, slot, dst, leader_ovl, leader_free0 + 8u * slot, stage_buf, lane, cols_valid);
      ++tiles_done;
    }
  }

  // ------------------------------------------------------------ teardown ---
  if constexpr (kRowDests) __threadfence_system();   // rows stored to other GPUs: visible once this ends
  tc_fence_before();
  __syncthreads();
  cluster_sync();          // no CTA leaves while the pair's MMAs or copies may touch it
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace mx
