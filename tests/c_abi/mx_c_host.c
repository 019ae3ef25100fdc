/* A plain C host program on the library's C ABI alone: include/mx.h, libmx.so
 * and the CUDA runtime, no C++ and no Python. It
 *   1. casts a bf16 matrix rowwise (mx_cast_dim0) and writes the input bits,
 *      the codes and the blocked scales to OUT.x, OUT.q and OUT.s, which the
 *      calling test checks bit for bit against the oracle;
 *   2. runs the linear forward twice -- with a caller workspace
 *      (mx_linear_fwd) and without any allocation (mx_linear_fwd_noalloc) --
 *      and requires the two outputs to be bitwise equal;
 *   3. runs the linear backward after the forward both as separate calls
 *      (mx_linear_fwd + mx_linear_bwd) and as the training pair
 *      (mx_linear_fwd_train + mx_linear_bwd_after_fwd, whose backward reuses
 *      the forward's casts) and requires y, dx and dw to be bitwise equal;
 *   4. requires an invalid call (a width that is not a multiple of 32) to
 *      return MX_ERR_UNSUPPORTED with a reason, before touching any buffer.
 * Usage: mx_c_host OUT ; exit status 0 when every check holds. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "mx.h"

#define M 256
#define K 320
#define N 192

static uint32_t state = 12345u;

/* xorshift32: a deterministic bit source (not the method's arithmetic) */
static uint32_t next_u32(void) {
  state ^= state << 13;
  state ^= state >> 17;
  state ^= state << 5;
  return state;
}

/* a finite bf16: random sign and mantissa, exponent within +-2^7 of 1 (or of 0.02 for w) */
static uint16_t random_bf16(int exp_center) {
  const uint32_t r = next_u32();
  const uint32_t sign = (r >> 31) & 1u;
  const int32_t e = exp_center + (int32_t)((r >> 16) % 15u) - 7;
  const uint32_t mant = r & 0x7Fu;
  return (uint16_t)((sign << 15) | ((uint32_t)e << 7) | mant);
}

static int write_file(const char* prefix, const char* ext, const void* data, size_t n) {
  char path[1024];
  snprintf(path, sizeof path, "%s.%s", prefix, ext);
  FILE* f = fopen(path, "wb");
  if (!f) return 1;
  const size_t w = fwrite(data, 1, n, f);
  fclose(f);
  return w != n;
}

#define CHECK_CUDA(call)                                                        \
  do {                                                                          \
    cudaError_t e_ = (call);                                                    \
    if (e_ != cudaSuccess) {                                                    \
      fprintf(stderr, "%s: %s\n", #call, cudaGetErrorString(e_));               \
      return 2;                                                                 \
    }                                                                           \
  } while (0)

#define CHECK_MX(call)                                                          \
  do {                                                                          \
    mx_status s_ = (call);                                                      \
    if (s_ != MX_OK) {                                                          \
      fprintf(stderr, "%s: status %d (%s)\n", #call, (int)s_, mx_last_error()); \
      return 3;                                                                 \
    }                                                                           \
  } while (0)

int main(int argc, char** argv) {
  if (argc != 2) {
    fprintf(stderr, "usage: %s OUT\n", argv[0]);
    return 1;
  }
  const size_t sbytes = mx_scale_bytes(M, K / 32);
  uint16_t* hx = (uint16_t*)malloc(sizeof(uint16_t) * M * K);
  uint16_t* hw = (uint16_t*)malloc(sizeof(uint16_t) * N * K);
  uint8_t* hq = (uint8_t*)malloc(M * K);
  uint8_t* hs = (uint8_t*)malloc(sbytes);
  uint16_t* hy1 = (uint16_t*)malloc(sizeof(uint16_t) * M * N);
  uint16_t* hy2 = (uint16_t*)malloc(sizeof(uint16_t) * M * N);
  uint16_t* hg1 = (uint16_t*)malloc(sizeof(uint16_t) * (M * K + N * K));
  uint16_t* hg2 = (uint16_t*)malloc(sizeof(uint16_t) * (M * K + N * K));
  uint16_t* hdy = (uint16_t*)malloc(sizeof(uint16_t) * M * N);
  if (!hx || !hw || !hq || !hs || !hy1 || !hy2 || !hg1 || !hg2 || !hdy) return 4;
  for (int i = 0; i < M * K; ++i) hx[i] = random_bf16(127);
  for (int i = 0; i < N * K; ++i) hw[i] = random_bf16(121);
  for (int i = 0; i < M * N; ++i) hdy[i] = random_bf16(120);

  void *dx, *dw, *dq, *ds, *dy1, *dy2, *ws, *ddy, *g1, *g2, *wst;
  const size_t ws_bytes = mx_linear_ws_bytes(M, N, K);
  const size_t wst_bytes = mx_linear_train_ws_bytes(M, N, K);
  CHECK_CUDA(cudaMalloc(&dx, sizeof(uint16_t) * M * K));
  CHECK_CUDA(cudaMalloc(&dw, sizeof(uint16_t) * N * K));
  CHECK_CUDA(cudaMalloc(&dq, M * K));
  CHECK_CUDA(cudaMalloc(&ds, sbytes));
  CHECK_CUDA(cudaMalloc(&dy1, sizeof(uint16_t) * M * N));
  CHECK_CUDA(cudaMalloc(&dy2, sizeof(uint16_t) * M * N));
  CHECK_CUDA(cudaMalloc(&ws, ws_bytes));
  CHECK_CUDA(cudaMalloc(&wst, wst_bytes));
  CHECK_CUDA(cudaMalloc(&ddy, sizeof(uint16_t) * M * N));
  CHECK_CUDA(cudaMalloc(&g1, sizeof(uint16_t) * (M * K + N * K)));   /* dx then dw */
  CHECK_CUDA(cudaMalloc(&g2, sizeof(uint16_t) * (M * K + N * K)));
  CHECK_CUDA(cudaMemcpy(ddy, hdy, sizeof(uint16_t) * M * N, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(dx, hx, sizeof(uint16_t) * M * K, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(dw, hw, sizeof(uint16_t) * N * K, cudaMemcpyHostToDevice));

  /* 1. the rowwise cast */
  CHECK_MX(mx_cast_dim0(dx, M, K, dq, ds, NULL));
  CHECK_MX(mx_device_error(NULL));
  CHECK_CUDA(cudaMemcpy(hq, dq, M * K, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(hs, ds, sbytes, cudaMemcpyDeviceToHost));
  if (write_file(argv[1], "x", hx, sizeof(uint16_t) * M * K) || write_file(argv[1], "q", hq, M * K) ||
      write_file(argv[1], "s", hs, sbytes))
    return 5;

  /* 2. the linear forward with a workspace and without any allocation */
  CHECK_MX(mx_linear_fwd(dx, dw, M, N, K, NULL, 0, dy1, ws, ws_bytes, NULL));
  CHECK_MX(mx_linear_fwd_noalloc(dx, dw, M, N, K, dy2, NULL));
  CHECK_MX(mx_device_error(NULL));
  CHECK_CUDA(cudaMemcpy(hy1, dy1, sizeof(uint16_t) * M * N, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(hy2, dy2, sizeof(uint16_t) * M * N, cudaMemcpyDeviceToHost));
  if (memcmp(hy1, hy2, sizeof(uint16_t) * M * N) != 0) {
    fprintf(stderr, "linear forward: workspace and allocation-free outputs differ\n");
    return 6;
  }

  /* 3. separate calls against the training pair: y, dx and dw bitwise equal */
  uint16_t* g1dw = (uint16_t*)g1 + M * K;
  uint16_t* g2dw = (uint16_t*)g2 + M * K;
  CHECK_MX(mx_linear_fwd(dx, dw, M, N, K, NULL, 0, dy1, ws, ws_bytes, NULL));
  CHECK_MX(mx_linear_bwd(ddy, dx, dw, M, N, K, NULL, 0, g1, g1dw, ws, ws_bytes, NULL));
  CHECK_MX(mx_linear_fwd_train(dx, dw, M, N, K, NULL, 0, dy2, wst, wst_bytes, NULL));
  CHECK_MX(mx_linear_bwd_after_fwd(ddy, dw, M, N, K, NULL, 0, g2, g2dw, wst, wst_bytes, NULL));
  CHECK_MX(mx_device_error(NULL));
  CHECK_CUDA(cudaMemcpy(hy1, dy1, sizeof(uint16_t) * M * N, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(hy2, dy2, sizeof(uint16_t) * M * N, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(hg1, g1, sizeof(uint16_t) * (M * K + N * K), cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(hg2, g2, sizeof(uint16_t) * (M * K + N * K), cudaMemcpyDeviceToHost));
  if (memcmp(hy1, hy2, sizeof(uint16_t) * M * N) != 0 ||
      memcmp(hg1, hg2, sizeof(uint16_t) * (M * K + N * K)) != 0) {
    fprintf(stderr, "linear: the training pair differs from the separate calls\n");
    return 8;
  }

  /* 4. an invalid call is refused on the host */
  const mx_status bad = mx_cast_dim0(dx, M, 48, dq, ds, NULL);
  if (bad != MX_ERR_UNSUPPORTED || mx_last_error() == NULL || mx_last_error()[0] == '\0') {
    fprintf(stderr, "a 48-wide cast returned %d\n", (int)bad);
    return 7;
  }

  cudaFree(dx);
  cudaFree(dw);
  cudaFree(dq);
  cudaFree(ds);
  cudaFree(dy1);
  cudaFree(dy2);
  cudaFree(ws);
  cudaFree(wst);
  cudaFree(ddy);
  cudaFree(g1);
  cudaFree(g2);
  free(hx);
  free(hw);
  free(hq);
  free(hs);
  free(hy1);
  free(hy2);
  free(hg1);
  free(hg2);
  free(hdy);
  printf("ok\n");
  return 0;
}
