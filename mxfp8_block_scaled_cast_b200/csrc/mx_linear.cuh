// MXFP8 linear forward / dgrad / wgrad and the per-weight quantization cache.
//
// The linear composes the casts and the grouped GEMM at one dense group
// (ao PR #4705, "MXFP8Linear training paths"; torchtitan PR #5334,
// description: one entry point serves dense and grouped MXFP8 linears):
//   forward  Y  = X W^T   X cast 1x32 along K, W cast with 32x32 blocks
//   dgrad    dX = dY W    dY cast 1x32 along N, the same 32x32 codes read
//                         MN-major with the dgrad scale view
//   wgrad    dW = dY^T X  dY and X cast 32x1 along the token axis
// dY is cast once with the fused rowwise+columnwise kernel.
//
// Weight cache ("Cache quantized weights for full AC", prime-rl PR #3388,
// Overview): with full activation checkpointing every checkpoint segment
// re-runs the forward, which used to re-quantize the weight each time. The
// cache keeps the 32x32 quantization of each weight, keyed by the weight's
// device address and shape and invalidated when the caller's version counter
// (the tensor's in-place update count) changes; it is cleared after
// backward. Quantization is a pure function of the weight bits, so a hit is
// bitwise identical to a miss.
#pragma once

#include <mutex>
#include <vector>

#include "mx_common.cuh"

struct mx_wcache {
  struct Entry {
    const void* w = nullptr;
    int64_t N = 0, K = 0;
    uint64_t version = 0;
    bool valid = false;
    uint8_t* q = nullptr;        // [N, K]
    uint8_t* s_fwd = nullptr;    // blocked(N, K/32)
    uint8_t* s_dgrad = nullptr;  // blocked(K, N/32)
  };
  std::vector<Entry> entries;
  int64_t hits = 0, misses = 0;
  std::mutex mu;
};

namespace mx {

// Device bytes of one 32x32-quantized weight (codes and both scale views),
// each piece rounded up to 256 bytes. The dgrad reads the same codes as an
// MN-major operand, so no transposed copy is kept.
inline int64_t wq_bytes(int64_t N, int64_t K) {
  return ceil_to(N * K, 256) + ceil_to(scale_bytes(N, K / kBlock), 256) + ceil_to(scale_bytes(K, N / kBlock), 256);
}

struct WeightView {
  uint8_t *q, *s_fwd, *s_dgrad;
};

inline WeightView carve_weight(uint8_t* base, int64_t N, int64_t K) {
  WeightView v;
  v.q = base;
  v.s_fwd = v.q + ceil_to(N * K, 256);
  v.s_dgrad = v.s_fwd + ceil_to(scale_bytes(N, K / kBlock), 256);
  return v;
}

}  // namespace mx

namespace mx {

// Workspace pieces of the linear, each rounded up to 256 bytes: X cast
// rowwise ([M, K] codes + blocked(M, K/32)), X cast columnwise ([K, M] +
// blocked(K, M/32)), dY cast both ways ([M, N] + blocked(M, N/32), [N, M] +
// blocked(N, M/32)).
inline int64_t linear_x_bytes(int64_t M, int64_t K) {
  return ceil_to(M * K, 256) + ceil_to(scale_bytes(M, K / kBlock), 256);
}
inline int64_t linear_xt_bytes(int64_t M, int64_t K) {
  return ceil_to(K * M, 256) + ceil_to(scale_bytes(K, M / kBlock), 256);
}
inline int64_t linear_dy_bytes(int64_t M, int64_t N) {
  return 2 * ceil_to(M * N, 256) + ceil_to(scale_bytes(M, N / kBlock), 256) + ceil_to(scale_bytes(N, M / kBlock), 256);
}

// The training pair's workspace (forward that keeps X's columnwise cast for
// its backward): X's columnwise codes and scales first -- written by the
// forward, read by the backward -- then the forward's rowwise X or the
// backward's dY casts (the larger of the two), then W's quantization.
struct LinearTrainWs {
  uint8_t *xqt, *xst;                 // [K, M], blocked(K, M/32)
  uint8_t *xq, *xs;                   // [M, K], blocked(M, K/32)      (forward)
  uint8_t *dyq, *dys, *dyqt, *dyst;   // [M, N], blocked(M, N/32), [N, M], blocked(N, M/32)  (backward)
  uint8_t* wq;                        // carve_weight(wq, N, K) when there is no cache
};

inline int64_t linear_train_ws_bytes(int64_t M, int64_t N, int64_t K) {
  const int64_t x = linear_x_bytes(M, K), dy = linear_dy_bytes(M, N);
  return linear_xt_bytes(M, K) + (x > dy ? x : dy) + wq_bytes(N, K);
}

inline LinearTrainWs carve_train_ws(void* ws, int64_t M, int64_t N, int64_t K) {
  LinearTrainWs L;
  uint8_t* p = static_cast<uint8_t*>(ws);
  L.xqt = p;
  L.xst = L.xqt + ceil_to(K * M, 256);
  uint8_t* mid = p + linear_xt_bytes(M, K);
  L.xq = mid;
  L.xs = L.xq + ceil_to(M * K, 256);
  L.dyq = mid;
  L.dys = L.dyq + ceil_to(M * N, 256);
  L.dyqt = L.dys + ceil_to(scale_bytes(M, N / kBlock), 256);
  L.dyst = L.dyqt + ceil_to(M * N, 256);
  L.wq = p + (linear_train_ws_bytes(M, N, K) - wq_bytes(N, K));
  return L;
}

}  // namespace mx
