// bf16 grouped GEMM on sm_100a tensor cores (tcgen05 kind::f16, CTA pairs,
// TMEM, TMA): the two GEMMs of the backward-override arms of the MXFP8
// grouped GEMM (ao "[moe training] Add backward_override to the MXFP8 grouped
// GEMM", Design notes): "high_precision" computes dgrad and wgrad as plain
// bf16 grouped GEMMs over the saved unpadded operands, and "dequantized" runs
// the same two GEMMs on the forward's quantized operands dequantized to bf16.
//
//   M-groups (dgrad):  out[rows of g, :] = A[rows of g, :] * B[g]
//     A bf16 [M, K] (K contiguous), B bf16 [G, K, N] (N contiguous), out [M, N].
//   K-groups (wgrad):  out[g] = A[rows of g, :]^T * B[rows of g, :]
//     A bf16 [M, N], B bf16 [M, K] (tokens are rows of both), out [G, N, K].
//
// Groups are the unpadded rows offs[g-1]..offs[g]; nothing is copied or
// transposed: operands whose contraction axis is not contiguous are read as
// "MN-major" tiles (the tensor core's transposed operand form), so the dgrad
// weight and both wgrad operands go to the MMA straight from the tensors the
// forward saved.
//
// Pipeline as in the MXFP8 kernel: clusters of two CTAs compute 256x256 tiles
// with the pair MMA (M = 256, N = 256, K = 16 per instruction, four per
// 64-deep stage); warp 4 is the TMA producer of a 6-stage ring, warp 5 of the
// leader issues the MMAs, warps 0-3 drain TMEM and store (two overlapping
// accumulator slots). Tile starts follow the unpadded groups: in M mode a
// 256-row tile may run into the next group, whose rows are computed but not
// stored; in K mode the last 64-token step of a group may hold tokens of the
// next group, whose rows of the A tile are set to zero in shared memory
// before that step's MMAs (each CTA zeroes its own half: the leader's MMA
// warp for the leader, warp 5 of the peer for the peer, on a handshake of
// two cluster barriers). An empty K group writes exact zeros.
#pragma once

#include "mx_gemm.cuh"

namespace mx {

constexpr int kHBK = 64;                                   // bf16 per 128-byte row = stage depth
constexpr int kHStages = 6;
constexpr uint32_t kHABytes = kCtaM * kHBK * 2;            // 16 KB per CTA
constexpr uint32_t kHBBytes = (kBN / 2) * kHBK * 2;        // 16 KB per CTA (half of B)
constexpr uint32_t kHChunk = 64 * 128;                     // one 64-wide MN-major box: 64 rows x 128 B
constexpr uint32_t kHTxBytes = 2 * (kHABytes + kHBBytes);  // both CTAs

constexpr uint32_t kHOffA = 0;
constexpr uint32_t kHOffB = kHOffA + kHStages * kHABytes;
constexpr uint32_t kHOffBar = kHOffB + kHStages * kHBBytes;
// full, empty, acc_full[2], acc_free[2], ovl_free, done, tail_ready, tail_done
constexpr uint32_t kHNumBars = 2 * kHStages + 8;
constexpr uint32_t kHOffMisc = kHOffBar + kHNumBars * 8;
constexpr uint32_t kHOffEnds = kHOffMisc + 64;
constexpr uint32_t kHOffTstart = kHOffEnds + 4 * kMaxGroups;
constexpr uint32_t kHOffStage = (kHOffTstart + 4 * (kMaxGroups + 1) + 127) & ~127u;
constexpr uint32_t kHGemmSmem = kHOffStage + 4 * kStageWarpBytes + 1024;
static_assert(kHGemmSmem <= 227 * 1024, "shared memory budget");

// Instruction descriptor of kind::f16: fp32 accumulator (bits [4,6) = 1),
// bf16 A and B (formats 1 in bits [7,10) and [10,13)), A / B major-ness in
// bits 15 / 16 (1 = MN-major), N>>3 in bits [17,23), M>>4 in bits [24,29).
__host__ __device__ constexpr uint32_t bf16_idesc(bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(a_mn) << 15) | (uint32_t(b_mn) << 16) |
         (uint32_t(kBN >> 3) << 17) | (uint32_t(kPairM >> 4) << 24);
}

struct HGemmArgs {
  const int32_t* offs;         // cumulative group ends, or null for one group of M rows
  __nv_bfloat16* out;
  int G;
  int64_t M, N, K;
};

struct HTile {
  int g;
  int nk;              // 64-deep K steps (0: empty K group)
  int tail;            // valid rows of the last K step (K mode), 64 if full
  int64_t m0;          // first row of the pair: A row (M mode) or output row in N (K mode)
  int64_t n0;          // first output column
  int64_t tok0;        // first token of the group (K mode)
};

template <int kMode>
__device__ __forceinline__ HTile decode_tile_bf16(int64_t tile, const HGemmArgs& a, const int32_t* ends,
                                                  const int32_t* tstart) {
  HTile t;
  if (kMode == kGroupsM) {
    const int64_t nt = ceil_div(a.N, kBN);
    const int64_t mt = tile / nt;
    t.n0 = (tile % nt) * kBN;
    int lo = 0, hi = a.G;   // largest g with tstart[g] <= mt
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (tstart[mid] <= mt) lo = mid; else hi = mid;
    }
    t.g = lo;
    const int64_t start = t.g ? ends[t.g - 1] : 0;
    t.m0 = start + (mt - tstart[t.g]) * kPairM;
    t.nk = int(ceil_div(a.K, kHBK));
    t.tail = kHBK;
    t.tok0 = 0;
  } else {
    const int64_t nt = ceil_div(a.K, kBN), mt = ceil_div(a.N, kPairM);
    const int64_t per_g = nt * mt;
    t.g = int(tile / per_g);
    const int64_t rem = tile % per_g;
    t.m0 = (rem / nt) * kPairM;
    t.n0 = (rem % nt) * kBN;
    t.tok0 = t.g ? ends[t.g - 1] : 0;
    const int64_t size = ends[t.g] - t.tok0;
    t.nk = int(ceil_div(size, kHBK));
    t.tail = int(size - int64_t(t.nk - 1) * kHBK);
  }
  return t;
}

// Zero token rows [from, 64) of one CTA's K-mode A stage (two 64-wide
// MN-major boxes of 64 rows x 128 bytes; the 128-byte swizzle permutes 16-byte
// pieces inside a row, so a whole row is zeroed regardless of it), then make
// the writes visible to the tensor core's operand reads. Whole warp.
__device__ __forceinline__ void zero_a_tail_rows(uint8_t* a_stage, int from, int lane) {
  const int pieces = (kHBK - from) * 16;        // 16-byte pieces: rows x 2 boxes x 8
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  for (int p = lane; p < pieces; p += 32) {
    const int row = from + (p >> 4), box = (p >> 3) & 1, piece = p & 7;
    *reinterpret_cast<uint4*>(a_stage + box * kHChunk + row * 128 + piece * 16) = z;
  }
  fence_proxy_async_smem();
  __syncwarp();
}

template <int kMode>
__global__ void __launch_bounds__(kGemmThreads, 1)
bf16_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                 const HGemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();      // 0 = leader of the pair
  const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + kHOffBar;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kHStages + s); };
  const uint32_t acc_full0 = bar0 + 8u * (2 * kHStages);   // + 8 * slot
  const uint32_t acc_free0 = acc_full0 + 16u;               // + 8 * slot
  const uint32_t ovl_free = acc_full0 + 32u;
  const uint32_t done_bar = acc_full0 + 40u;
  const uint32_t tail_ready = acc_full0 + 48u;             // peer: leader saw the tail stage land
  const uint32_t tail_done = acc_full0 + 56u;              // leader: peer zeroed its tail rows
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kHOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kHOffMisc + 4);
  int64_t* info = reinterpret_cast<int64_t*>(smem + kHOffMisc + 8);
  int32_t* ends = reinterpret_cast<int32_t*>(smem + kHOffEnds);
  int32_t* tstart = reinterpret_cast<int32_t*>(smem + kHOffTstart);

  // ---------------------------------------------------------------- setup --
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&map_a);
    tma_prefetch_desc(&map_b);
    for (int s = 0; s < kHStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(acc_full0, 1);
    mbar_init(acc_full0 + 8, 1);
    mbar_init(acc_free0, 8);      // four epilogue warps in each CTA of the pair
    mbar_init(acc_free0 + 8, 8);
    mbar_init(ovl_free, 8);
    mbar_init(done_bar, 1);
    mbar_init(tail_ready, 1);
    mbar_init(tail_done, 1);
    fence_barrier_init();
    *abort_flag = 0;
  }
  if (warp == 5) {
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == 0) {
    // group table: ends[g] and the first 256-row tile of each group, tstart[0..G]
    bool bad = false;
    const int G = args.offs ? args.G : 1;
    if (args.offs == nullptr) {
      if (lane == 0) {
        ends[0] = int32_t(args.M);
        tstart[0] = 0;
        tstart[1] = int32_t(ceil_div(args.M, kPairM));
      }
    } else {
      const unsigned full = 0xFFFFFFFFu;
      int64_t tcarry = 0, prev_end = 0;
      if (lane == 0) tstart[0] = 0;
      for (int base = 0; base < G; base += 32) {
        const int g = base + lane;
        const bool in = g < G;
        const int64_t e = in ? int64_t(__ldg(args.offs + g)) : 0;
        int64_t s = __shfl_up_sync(full, e, 1);
        if (lane == 0) s = prev_end;
        const int64_t size = in ? e - s : 0;
        if (in && size < 0) bad = true;
        int64_t tincl = size > 0 ? ceil_div(size, kPairM) : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int64_t u = __shfl_up_sync(full, tincl, o);
          if (lane >= o) tincl += u;
        }
        if (in) {
          ends[g] = int32_t(e);
          tstart[g + 1] = int32_t(tcarry + tincl);
        }
        tcarry = __shfl_sync(full, tcarry + tincl, 31);
        prev_end = __shfl_sync(full, e, min(31, G - 1 - base));
      }
      bad = __any_sync(full, bad);
      if (prev_end != args.M) bad = true;
    }
    if (lane == 0) {
      int64_t total;
      if (kMode == kGroupsM) total = bad ? 0 : int64_t(tstart[G]) * ceil_div(args.N, kBN);
      else total = bad ? 0 : int64_t(G) * ceil_div(args.N, kPairM) * ceil_div(args.K, kBN);
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
  HGemmArgs a = args;
  if (a.offs == nullptr) a.G = 1;

  // ----------------------------------------------------------- producer ---
  if (warp == 4) {
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued = 0, last_par = 0;
    for (int64_t tile = pair; tile < total_tiles; tile += npairs) {
      const HTile t = decode_tile_bf16<kMode>(tile, a, ends, tstart);
      const int32_t own_m = int32_t(t.m0 + kCtaM * rank);            // M mode: A row; K mode: A column
      const int32_t own_n = int32_t(t.n0 + (kBN / 2) * rank);        // B column (both modes)
      bool ok = true;
      for (int kt = 0; kt < t.nk; ++kt) {
        if (!mbar_wait_warp(empty_bar(stage), phase ^ 1u, abort_flag)) { ok = false; break; }
        const uint32_t fb = full_bar(stage);
        const uint32_t sa = sbase + kHOffA + stage * kHABytes;
        const uint32_t sb = sbase + kHOffB + stage * kHBBytes;
        if (elect_one()) {
          if (rank == 0) mbar_arrive_expect_tx(fb, kHTxBytes);
          const uint32_t lb = mapa_shared(fb, 0);
          if (kMode == kGroupsM) {
            tma_load_2d_pair(sa, &map_a, kt * kHBK, own_m, lb);                  // 128 rows x 64 K
            tma_load_3d_pair(sb, &map_b, own_n, kt * kHBK, t.g, lb);              // 64 K x 64 N
            tma_load_3d_pair(sb + kHChunk, &map_b, own_n + 64, kt * kHBK, t.g, lb);
          } else {
            const int32_t tok = int32_t(t.tok0 + int64_t(kt) * kHBK);
            tma_load_2d_pair(sa, &map_a, own_m, tok, lb);                         // 64 tokens x 64 N
            tma_load_2d_pair(sa + kHChunk, &map_a, own_m + 64, tok, lb);
            tma_load_2d_pair(sb, &map_b, own_n, tok, lb);                         // 64 tokens x 64 K
            tma_load_2d_pair(sb + kHChunk, &map_b, own_n + 64, tok, lb);
          }
        }
        __syncwarp();
        issued |= 1u << stage;
        last_par = (last_par & ~(1u << stage)) | (phase << stage);
        if (++stage == kHStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
    }
    if (rank == 0 && lane == 0)
      for (int s = 0; s < kHStages; ++s)
        if (issued & (1u << s)) mbar_drain(full_bar(s), (last_par >> s) & 1u);
    __syncwarp();
  }
  // ------------------------------------------------------ MMA (leader) ---
  else if (warp == 5 && rank == 0) {
    int stage = 0;
    uint32_t phase = 0;
    uint32_t tiles_done = 0, tails = 0;
    constexpr bool kAMn = kMode == kGroupsK;
    constexpr uint32_t kIdesc = bf16_idesc(kAMn, true);
    // K-major (128-byte rows, 8-row groups 1024 B apart): 16 K = +32 bytes.
    // MN-major (64-wide boxes 8 KB apart = LBO, 8-row groups 1024 B apart =
    // SBO): 16 K = two 8-row groups = +2048 bytes.
    const uint64_t a_desc0 = kAMn ? smem_desc(sbase + kHOffA, kHChunk, 1024, 2) : smem_desc(sbase + kHOffA, 16, 1024, 2);
    const uint64_t b_desc0 = smem_desc(sbase + kHOffB, kHChunk, 1024, 2);
    constexpr uint64_t kAStep = kAMn ? (2048 >> 4) : (32 >> 4);
    constexpr uint64_t kBStep = 2048 >> 4;
    const uint32_t peer_tail_ready = mapa_shared(tail_ready, 1);
    for (int64_t tile = pair; tile < total_tiles; tile += npairs) {
      const HTile t = decode_tile_bf16<kMode>(tile, a, ends, tstart);
      if (t.nk == 0) continue;
      const uint32_t slot = tiles_done & 1u, use = tiles_done >> 1;
      if (!mbar_wait_warp(acc_free0 + 8u * slot, (use & 1u) ^ 1u, abort_flag)) break;
      if (!mbar_wait_warp(ovl_free, (tiles_done & 1u) ^ 1u, abort_flag)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem + (slot ? kAccSlot1 : 0u);
      bool ok = true;
      for (int kt = 0; kt < t.nk; ++kt) {
        if (!mbar_wait_warp(full_bar(stage), phase, abort_flag)) { ok = false; break; }
        int nmma = 4;
        if (kMode == kGroupsK && kt == t.nk - 1 && t.tail < kHBK) {
          // rows of the next group in this step: zero them in both CTAs.
          // Every lane observes the completed stage phase itself (it is
          // complete, so this returns at once) before writing over the
          // copy's bytes.
          (void)mbar_try_wait(full_bar(stage), phase);
          fence_proxy_async_smem();
          zero_a_tail_rows(smem + kHOffA + stage * kHABytes, t.tail, lane);
          if (lane == 0) mbar_arrive_cluster(peer_tail_ready);
          __syncwarp();
          bool got = true;
          if (lane == 0) got = mbar_wait_cluster(tail_done, tails & 1u, abort_flag);
          if (__shfl_sync(0xFFFFFFFFu, got ? 1 : 0, 0) == 0) { ok = false; break; }
          (void)mbar_try_wait_cluster(tail_done, tails & 1u);   // acquire in every lane
          ++tails;
          nmma = (t.tail + 15) >> 4;      // K slices past the group are all zero
        }
        const uint64_t ad = a_desc0 + uint64_t((stage * kHABytes) >> 4);
        const uint64_t bd = b_desc0 + uint64_t((stage * kHBBytes) >> 4);
        if (elect_one()) {
          for (int k = 0; k < nmma; ++k)
            mma_bf16_pair(d_tmem, ad + k * kAStep, bd + k * kBStep, kIdesc, (kt | k) != 0 ? 1u : 0u);
          tc_commit_pair(empty_bar(stage));
        }
        __syncwarp();
        if (++stage == kHStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      if (elect_one()) tc_commit_pair(acc_full0 + 8u * slot);
      __syncwarp();
      ++tiles_done;
    }
    if (elect_one()) {
      tc_commit_pair(done_bar);
      mbar_drain(done_bar, 0);
    }
    __syncwarp();
  }
  // ------------------------------------------- tail rows of the peer CTA ---
  else if (warp == 5) {
    if (kMode == kGroupsK) {
      int stage = 0;
      uint32_t tails = 0;
      const uint32_t leader_tail_done = mapa_shared(tail_done, 0);
      for (int64_t tile = pair; tile < total_tiles; tile += npairs) {
        const HTile t = decode_tile_bf16<kMode>(tile, a, ends, tstart);
        if (t.nk == 0) continue;
        const int last = int((stage + t.nk - 1) % kHStages);
        stage = int((stage + t.nk) % kHStages);
        if (t.tail == kHBK) continue;
        bool got = true;
        if (lane == 0) got = mbar_wait_cluster(tail_ready, tails & 1u, abort_flag);
        if (__shfl_sync(0xFFFFFFFFu, got ? 1 : 0, 0) == 0) break;
        (void)mbar_try_wait_cluster(tail_ready, tails & 1u);  // acquire in every lane
        ++tails;
        fence_proxy_async_smem();          // the stage's TMA writes precede the zeros
        zero_a_tail_rows(smem + kHOffA + last * kHABytes, t.tail, lane);
        if (lane == 0) mbar_arrive_cluster(leader_tail_done);
        __syncwarp();
      }
    }
  }
  // ----------------------------------------------------------- epilogue ---
  else {
    uint32_t tiles_done = 0;
    const int r = warp * 32 + lane;
    const uint32_t lane_base = tmem + (uint32_t(warp * 32) << 16);
    const uint32_t leader_ovl = mapa_shared(ovl_free, 0);
    const uint32_t leader_free0 = mapa_shared(acc_free0, 0);
    uint8_t* stage_buf = smem + kHOffStage + warp * kStageWarpBytes;
    for (int64_t tile = pair; tile < total_tiles; tile += npairs) {
      const HTile t = decode_tile_bf16<kMode>(tile, a, ends, tstart);
      const int64_t row = t.m0 + kCtaM * rank + r;
      __nv_bfloat16* dst = nullptr;
      int64_t cols_valid;           // output columns of this tile (fewer than 256 at a ragged edge)
      if (kMode == kGroupsM) {
        if (row < ends[t.g]) dst = a.out + row * a.N + t.n0;
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
  tc_fence_before();
  __syncthreads();
  cluster_sync();          // no CTA leaves while the pair's MMAs or copies may touch it
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace mx
