// MX -> bf16 dequantization and the blocked -> logical scale unswizzle, for
// the "dequantized" backward arm (ao "[moe training] Add backward_override to
// the MXFP8 grouped GEMM", Design notes: that arm differentiates the
// quantized-forward function, so it needs the forward's operands back in
// bf16, and it needs logical (pre-blocking) scales, which the page notes no
// existing kernel recovered from the blocked layout).
//
// Element value: e4m3(q) * 2^(b - 127) rounded to bf16 (nearest, ties to
// even). The E4M3 pair is widened exactly by cvt.rn.f16x2.e4m3x2 (every E4M3
// value is an f16 value), the f16 -> f32 step is exact, the product by the
// power of two is exact in fp32 (the smallest result, 2^-136, is above the
// fp32 subnormal floor 2^-149; fp32 subnormals are kept, -ftz=false), and
// cvt.rn.bf16x2.f32 rounds once. A NaN code or the E8M0 NaN byte 255 gives
// NaN.
//
// Memory bound (1 byte read, 2 bytes written per element): a warp takes 1024
// consecutive elements of a row in two passes in which lane i converts 16
// codes, so each load instruction of the warp reads 512 contiguous bytes and
// each (256-bit per lane) store writes 1 KB.
#pragma once

#include <cuda_bf16.h>

#include "mx_common.cuh"

namespace mx {

constexpr int kDeqThreads = 256;

// 2^(b - 127) as a float: b = 0 is the subnormal 2^-127, 255 is NaN.
__device__ __forceinline__ float e8m0_value(uint32_t b) {
  if (b == 0u) return __uint_as_float(0x00400000u);
  if (b == 255u) return __uint_as_float(0x7FC00000u);
  return __uint_as_float(b << 23);
}

// Four E4M3 codes (one word, code 0 in the low byte) times `scale` -> four
// bf16 in two words (element order kept).
__device__ __forceinline__ uint2 dequant4(uint32_t codes, float scale) {
  uint32_t h01, h23;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h01) : "h"(static_cast<unsigned short>(codes & 0xFFFFu)));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h23) : "h"(static_cast<unsigned short>(codes >> 16)));
  float f[4];
  asm("{\n\t.reg .f16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\tcvt.f32.f16 %0, lo;\n\tcvt.f32.f16 %1, hi;\n\t}"
      : "=f"(f[0]), "=f"(f[1]) : "r"(h01));
  asm("{\n\t.reg .f16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\tcvt.f32.f16 %0, lo;\n\tcvt.f32.f16 %1, hi;\n\t}"
      : "=f"(f[2]), "=f"(f[3]) : "r"(h23));
  uint2 r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r.x) : "f"(f[1] * scale), "f"(f[0] * scale));
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r.y) : "f"(f[3] * scale), "f"(f[2] * scale));
  return r;
}

struct DequantArgs {
  const uint8_t* q;            // E4M3 codes, rows of C bytes
  const uint8_t* s;            // blocked scales
  __nv_bfloat16* out;          // rows_out x C
  int64_t rows_out, C;
  int64_t layout_rows;         // plain mode: rows per blocked scale layout (a stack of layouts)
  const int32_t* offs;         // grouped mode: cumulative group ends
  int G;
  int64_t m_cap;               // grouped mode: padded rows of q / s
};

// kGrouped = false: out row r is q row r; its scales are in layout r / layout_rows
//   (each layout_rows x C/32 layout of mx_scale_bytes bytes), row r % layout_rows.
// kGrouped = true: out row start_g + i is padded row p_g + i of q and of
//   blocked(m_cap, C/32); invalid offsets flag the device error and write nothing.
template <bool kGrouped>
__global__ void __launch_bounds__(kDeqThreads)
dequant_dim0_kernel(const DequantArgs a) {
  __shared__ int32_t s_ends[kGrouped ? kMaxGroups : 1];
  __shared__ int32_t s_pstart[kGrouped ? kMaxGroups : 1];
  __shared__ int s_bad;
  if (kGrouped) {
    if (threadIdx.x < 32) {
      const unsigned full = 0xFFFFFFFFu;
      const int lane = threadIdx.x;
      int64_t carry = 0, prev_end = 0;
      bool bad = false;
      for (int base = 0; base < a.G; base += 32) {
        const int g = base + lane;
        const bool in = g < a.G;
        const int64_t e = in ? int64_t(__ldg(a.offs + g)) : 0;
        int64_t st = __shfl_up_sync(full, e, 1);
        if (lane == 0) st = prev_end;
        const int64_t size = in ? e - st : 0;
        if (in && size < 0) bad = true;
        const int64_t pad = size > 0 ? ceil_to(size, 128) : 0;
        int64_t incl = pad;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int64_t t = __shfl_up_sync(full, incl, o);
          if (lane >= o) incl += t;
        }
        if (in) {
          s_ends[g] = int32_t(e);
          s_pstart[g] = int32_t(carry + incl - pad);
        }
        carry = __shfl_sync(full, carry + incl, 31);
        prev_end = __shfl_sync(full, e, min(31, a.G - 1 - base));
      }
      bad = __any_sync(full, bad);
      if (prev_end != a.rows_out || carry > a.m_cap) bad = true;
      if (lane == 0) {
        s_bad = bad ? 1 : 0;
        if (bad && blockIdx.x == 0) flag_error(kErrOffsets);
      }
    }
    __syncthreads();
    if (s_bad) return;
  }
  // Work item = one row and a chunk of 32 consecutive blocks (1024 elements)
  // of it, taken by one warp. The row's source and scale base are found once
  // per item.
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t cb = a.C / kBlock;                      // blocks per row
  const int64_t chunks = ceil_div(cb, 32);
  const int64_t items = a.rows_out * chunks;
  const int64_t sc_tiles = ceil_div(cb, 4);             // 4-column scale tiles per band
  const int64_t layout_bytes = ceil_to(a.layout_rows, 128) * ceil_to(cb, 4);
  const int64_t wstride = int64_t(gridDim.x) * (kDeqThreads / 32);
  // element offsets are multiples of 16 (32 bytes of bf16): 256-bit stores
  // need only a 32-byte aligned output (the ABI promises 16)
  const bool out_al = (reinterpret_cast<uintptr_t>(a.out) & 31u) == 0;
  for (int64_t it = int64_t(blockIdx.x) * (kDeqThreads / 32) + warp; it < items; it += wstride) {
    const int64_t r = it / chunks;
    const int64_t c0 = (it - r * chunks) * 32;            // first block of the chunk
    int64_t src_row, srow;
    const uint8_t* sbase = a.s;
    if (kGrouped) {
      int lo = 0, hi = a.G;                             // first g with ends[g] > r
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (s_ends[mid] > r) hi = mid; else lo = mid + 1;
      }
      const int64_t start = lo ? s_ends[lo - 1] : 0;
      src_row = s_pstart[lo] + (r - start);
      srow = src_row;
    } else {
      const int64_t layout = r / a.layout_rows;
      src_row = r;
      sbase += layout * layout_bytes;
      srow = r - layout * a.layout_rows;
    }
    const uint8_t* qrow = a.q + src_row * a.C;
    __nv_bfloat16* orow = a.out + r * a.C;
    const int64_t e0 = c0 * kBlock;                     // first element of the chunk
    // two passes of 512 elements: lane i takes 16 codes (16 bytes in, 32 bytes
    // out), so every load instruction of the warp reads 512 contiguous bytes
    // and every store writes 1 KB
    uint4 qv[2];
    uint32_t bv[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int64_t e = e0 + k * 512 + lane * 16;
      if (e < a.C) {
        qv[k] = ld_stream16(qrow + e);
        const int64_t c = e >> 5;
        bv[k] = sbase[(srow >> 7) * sc_tiles * 512 + (c >> 2) * 512 + in_tile(uint32_t(srow & 127), uint32_t(c))];
      }
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int64_t e = e0 + k * 512 + lane * 16;
      if (e < a.C) {
        const float scale = e8m0_value(bv[k]);
        const uint2 p0 = dequant4(qv[k].x, scale), p1 = dequant4(qv[k].y, scale);
        const uint2 p2 = dequant4(qv[k].z, scale), p3 = dequant4(qv[k].w, scale);
        __nv_bfloat16* dst = orow + e;
        if (out_al) {
          asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(dst), "r"(p0.x), "r"(p0.y),
                       "r"(p1.x), "r"(p1.y), "r"(p2.x), "r"(p2.y), "r"(p3.x), "r"(p3.y)
                       : "memory");
        } else {
          reinterpret_cast<uint4*>(dst)[0] = make_uint4(p0.x, p0.y, p1.x, p1.y);
          reinterpret_cast<uint4*>(dst)[1] = make_uint4(p2.x, p2.y, p3.x, p3.y);
        }
      }
    }
  }
}

// Logical scales S[R, C32] (row-major bytes) from their blocked layout.
__global__ void __launch_bounds__(kDeqThreads)
scales_unswizzle_kernel(const uint8_t* __restrict__ s, int64_t R, int64_t C32, uint8_t* __restrict__ out) {
  const int64_t sc_tiles = ceil_div(C32, 4);
  const int64_t total = R * C32;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = i / C32, c = i % C32;
    out[i] = s[(r >> 7) * sc_tiles * 512 + (c >> 2) * 512 + in_tile(uint32_t(r & 127), uint32_t(c))];
  }
}

}  // namespace mx
