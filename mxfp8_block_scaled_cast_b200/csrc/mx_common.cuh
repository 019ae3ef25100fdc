// Shared device helpers of libmx: the MX element/scale arithmetic on bit
// fields, the blocked scale index map, group lookup for the pad path, and the
// sticky device error flag.
//
// The cast arithmetic avoids CUDA math functions: the RCEIL exponent is an
// integer function of the bf16 bit fields of amax, the scaling is one exact
// float multiply by a power of two, and the element rounding is the PTX
// conversion cvt.rn.satfinite.e4m3x2.f32 (round to nearest even, saturating).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "mx.h"

namespace mx {

constexpr int kBlock = 32;          // elements sharing one E8M0 scale
constexpr int kMaxGroups = 1024;    // largest G the grouped entry points take

// Sticky device-side error word, read and cleared by mx_device_error().
__device__ unsigned int g_device_error;
enum : unsigned { kErrTimeout = 1u, kErrOffsets = 2u };

__device__ __forceinline__ void flag_error(unsigned bits) { atomicOr(&g_device_error, bits); }

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t x, int64_t a) { return (x + a - 1) / a; }
__host__ __device__ __forceinline__ int64_t ceil_to(int64_t x, int64_t a) { return ceil_div(x, a) * a; }

// Bytes of the blocked layout of a logical scale matrix S[rows, cols].
__host__ __device__ __forceinline__ int64_t scale_bytes(int64_t rows, int64_t cols) {
  return ceil_to(rows, 128) * ceil_to(cols, 4);
}

// Byte of S[r, c] inside its 512-byte 128x4 tile.
__device__ __forceinline__ uint32_t in_tile(uint32_t r, uint32_t c) {
  return (r & 31u) * 16u + ((r >> 5) & 3u) * 4u + (c & 3u);
}

// RCEIL E8M0 byte from the magnitude bits (sign cleared) of a finite bf16
// amax. With E the exponent field and m the 7-bit mantissa,
// amax = (1 + m/128) * 2^(E-127) and 448 = 1.75 * 2^8, so the smallest e with
// 448 * 2^e >= amax is E - 135 + [m > 96] and b = e + 127 = E - 8 + [m > 96],
// clamped at 0 (zero and tiny blocks). Finite bf16 gives b <= 247.
__device__ __forceinline__ uint32_t rceil_b(uint32_t amax_bits) {
  int e = int(amax_bits >> 7) - 8 + int((amax_bits & 0x7Fu) > 96u);
  return e < 0 ? 0u : uint32_t(e);
}

// FLOOR E8M0 byte: scale 2^(floor(log2 amax) - 8); floor(log2 amax) = E - 127
// for a normal bf16 amax, so b = E - 8, clamped at 0 (zero, tiny, subnormal).
__device__ __forceinline__ uint32_t floor_b(uint32_t amax_bits) {
  int e = int(amax_bits >> 7) - 8;
  return e < 0 ? 0u : uint32_t(e);
}

// 2^(127 - b) as a float (exact; b in [0, 247] keeps the exponent normal).
__device__ __forceinline__ float inv_scale(uint32_t b) { return __uint_as_float((254u - b) << 23); }

// Max of the magnitudes of the two bf16 halves of eight words, per half.
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t acc, uint32_t w) {
  return __vmaxu2(acc, w & 0x7FFF7FFFu);
}

// Two floats -> two E4M3 codes, `lo` in the low byte (RNE, satfinite).
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  unsigned short r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Four bf16 (two words) scaled by `inv` -> four E4M3 codes in one word.
__device__ __forceinline__ uint32_t quant4(uint32_t w0, uint32_t w1, float inv) {
  uint32_t a = cvt_e4m3x2(bf16_lo(w0) * inv, bf16_hi(w0) * inv);
  uint32_t b = cvt_e4m3x2(bf16_lo(w1) * inv, bf16_hi(w1) * inv);
  return a | (b << 16);
}

// Streaming 16-byte global load (read once).
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// ---------------------------------------------------------------------------
// Group lookup for the pad path. Group g holds rows offs[g-1]..offs[g] of the
// unpadded tensor and starts at padded row p_g = sum_{h<g} ceil(size_h/128)*128.
// For a padded row `row0` (a multiple of 128) this finds the group whose
// padded range holds it and returns the first source row and how many real
// rows of the group remain from row0 (<= 0: the tile is padding). Invalid
// offsets (decreasing, last != m_total, padded total > m_cap) set the device
// flag and make every tile padding. Runs on warp 0; the result is published
// in shared memory and the caller must __syncthreads() before reading it.
// ---------------------------------------------------------------------------
struct GroupSlot {
  long long src0;   // first source row of this tile
  long long live;   // real rows from row0 (may exceed 128 or be <= 0)
  long long pstart; // the group's first padded row
  int group;        // group index or -1
};

__device__ __forceinline__ void find_group_of_row(const int32_t* __restrict__ offs, int G,
                                                  long long m_total, long long m_cap,
                                                  long long row0, GroupSlot* out) {
  // Valid offsets keep every running sum below m_cap, which the launch bounds
  // to 65535 tiles of 128 rows, so the scan runs in 32-bit arithmetic
  // (unsigned, so that invalid offsets wrap instead of overflowing; they are
  // flagged below whatever the sums come to).
  const unsigned full = 0xFFFFFFFFu;
  const int lane = threadIdx.x & 31;
  const unsigned r0 = unsigned(row0);
  unsigned carry = 0u;
  int prev_end = 0;
  bool bad = false;
  unsigned f_src = 0u, f_pbeg = 0u;
  long long f_live = 0;
  int f_group = -1;
  for (int base = 0; base < G; base += 32) {
    const int g = base + lane;
    const bool in = g < G;
    const int e = in ? __ldg(offs + g) : 0;
    int s = __shfl_up_sync(full, e, 1);
    if (lane == 0) s = prev_end;
    const bool neg = in && (e < s || e < 0);
    if (neg) bad = true;
    const unsigned size = (in && !neg) ? unsigned(e - s) : 0u;
    const unsigned pad = (size + 127u) & ~127u;
    unsigned incl = pad;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned t = __shfl_up_sync(full, incl, o);
      if (lane >= o) incl += t;
    }
    const unsigned pend = carry + incl, pbeg = pend - pad;
    if (in && pad > 0u && r0 >= pbeg && r0 < pend) {
      f_src = unsigned(s) + (r0 - pbeg);
      f_live = (long long)size - (long long)(r0 - pbeg);
      f_pbeg = pbeg;
      f_group = g;
    }
    const int last = min(31, G - 1 - base);
    carry = __shfl_sync(full, pend, 31);
    prev_end = __shfl_sync(full, e, last);
  }
  bad = __any_sync(full, bad);
  // a total past the capacity (or one that wrapped) is invalid too
  if ((long long)prev_end != m_total || (long long)carry > m_cap || carry < unsigned(prev_end)) bad = true;
  const unsigned hit = __ballot_sync(full, f_group >= 0);
  if (lane == 0) {
    if (bad) {
      flag_error(kErrOffsets);
      out->src0 = 0; out->live = 0; out->pstart = 0; out->group = -1;
    } else if (hit == 0u) {
      out->src0 = 0; out->live = 0; out->pstart = 0; out->group = -1;
    }
  }
  if (!bad && hit != 0u && lane == __ffs(hit) - 1) {
    out->src0 = (long long)f_src; out->live = f_live; out->pstart = (long long)f_pbeg; out->group = f_group;
  }
}

}  // namespace mx
