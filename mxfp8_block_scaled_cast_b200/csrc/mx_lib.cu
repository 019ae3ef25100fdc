// libmx: the C ABI declared in include/mx.h.
//
// This single translation unit holds every kernel of the library (casts,
// the tcgen05 grouped GEMMs, dequantization, the linear and its weight cache) so that they
// share the sticky device error flag without relocatable device code.
// Host functions validate every argument before any launch and report the
// reason of a failure through mx_last_error().
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>

#include <cudaTypedefs.h>

#include "mx_common.cuh"
#include "mx_cast.cuh"
#include "mx_gemm.cuh"
#include "mx_gemm_bf16.cuh"
#include "mx_cast_warp.cuh"
#include "mx_dequant.cuh"
#include "mx_linear.cuh"

namespace mx {
namespace {

thread_local char g_err[512] = "";

mx_status fail(mx_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

mx_status cuda_check(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(MX_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return MX_OK;
}

#define MX_REQUIRE(cond, st, ...) \
  do {                            \
    if (!(cond)) return fail(st, __VA_ARGS__); \
  } while (0)

// Rowwise and 32x32 casts of at most this many 128x128 tiles load each slice in
// two halves (about nine waves of six CTAs per SM); larger ones load it whole.
constexpr int64_t kSplitLoadMaxTiles = 8192;

template <int kMode, bool kGrouped>
mx_status launch_cast(const CastArgs& a, int64_t col_tiles, int64_t row_tiles, int64_t depth,
                      cudaStream_t stream) {
  if (col_tiles == 0 || row_tiles == 0 || depth == 0) return MX_OK;
  // Every cast goes through the warp-sliced kernel (no CTA barrier before the
  // scale tiles, every code written as whole 32-byte sectors from registers).
  MX_REQUIRE(col_tiles < (1ll << 31) && row_tiles <= 65535 && depth <= 65535, MX_ERR_UNSUPPORTED,
             "cast grid too large (%lld x %lld x %lld tiles)", (long long)col_tiles, (long long)row_tiles,
             (long long)depth);
  const dim3 grid{unsigned(col_tiles), unsigned(row_tiles), unsigned(depth)};
  if constexpr ((kMode & kModeCol) == 0) {
    // rowwise and 32x32: split loads on launches of a few waves of tiles
    if (col_tiles * row_tiles * depth > kSplitLoadMaxTiles) {
      cast_warp_kernel<kMode, kGrouped, false><<<grid, kWarpCastThreads, kWarpCastSmem, stream>>>(a);
      return cuda_check("cast launch");
    }
  }
  cast_warp_kernel<kMode, kGrouped, true><<<grid, kWarpCastThreads, kWarpCastSmem, stream>>>(a);
  return cuda_check("cast launch");
}

CastArgs make_args(const void* x, int64_t rows_src, int64_t C, int64_t rows_out) {
  CastArgs a;
  memset(&a, 0, sizeof(a));
  a.x = static_cast<const uint16_t*>(x);
  a.rows_src = rows_src;
  a.C = C;
  a.rows_out = rows_out;
  return a;
}

mx_status check_cast_geometry(const void* x, int64_t R, int64_t C, bool rows_blocked) {
  MX_REQUIRE(R >= 0 && C > 0, MX_ERR_ARG, "sizes must be R >= 0, C > 0 (got %lld, %lld)", (long long)R,
             (long long)C);
  MX_REQUIRE(C % kBlock == 0, MX_ERR_UNSUPPORTED, "C = %lld is not a multiple of 32", (long long)C);
  MX_REQUIRE(!rows_blocked || R % kBlock == 0, MX_ERR_UNSUPPORTED,
             "R = %lld is not a multiple of 32 (columnwise blocks)", (long long)R);
  MX_REQUIRE(R == 0 || x != nullptr, MX_ERR_ARG, "null input");
  MX_REQUIRE(aligned16(x), MX_ERR_ALIGN, "input not 16-byte aligned");
  return MX_OK;
}

mx_status check_out(const void* p, bool needed, const char* name) {
  MX_REQUIRE(!needed || p != nullptr, MX_ERR_ARG, "null output %s", name);
  MX_REQUIRE(aligned16(p), MX_ERR_ALIGN, "output %s not 16-byte aligned", name);
  return MX_OK;
}

#define MX_TRY(expr)              \
  do {                            \
    mx_status st_ = (expr);       \
    if (st_ != MX_OK) return st_; \
  } while (0)

mx_status check_grouped(const void* x, int64_t M, int64_t K, const int32_t* offs, int32_t G,
                        int64_t m_cap) {
  MX_REQUIRE(M >= 0 && K > 0, MX_ERR_ARG, "sizes must be M >= 0, K > 0");
  MX_REQUIRE(K % kBlock == 0, MX_ERR_UNSUPPORTED, "K = %lld is not a multiple of 32", (long long)K);
  MX_REQUIRE(G >= 1 && G <= kMaxGroups, MX_ERR_ARG, "G = %d outside [1, %d]", G, kMaxGroups);
  MX_REQUIRE(offs != nullptr, MX_ERR_ARG, "null offsets");
  MX_REQUIRE((reinterpret_cast<uintptr_t>(offs) & 3u) == 0, MX_ERR_ALIGN, "offsets not 4-byte aligned");
  MX_REQUIRE(m_cap >= M && m_cap % 128 == 0, MX_ERR_ARG,
             "m_cap = %lld must be a multiple of 128 and >= M = %lld", (long long)m_cap, (long long)M);
  MX_REQUIRE(M == 0 || x != nullptr, MX_ERR_ARG, "null input");
  MX_REQUIRE(aligned16(x), MX_ERR_ALIGN, "input not 16-byte aligned");
  return MX_OK;
}

// A dense cast whose arguments have been checked: what its own launch would
// get. The public cast entry points prepare and launch one; the linear
// launches its weight and activation casts together (cast_multi_kernel).
struct PreparedCast {
  CastArgs a;
  int mode = -1;                  // kModeRow, kModeCol, kModeRowCol or kModeSquare
  int64_t gx = 0, gy = 0, gz = 0;  // tiles along columns, rows, experts
};

mx_status prepare_dim0(const void* x, int64_t R, int64_t C, void* q, void* s, PreparedCast* p) {
  MX_TRY(check_cast_geometry(x, R, C, false));
  MX_TRY(check_out(q, R > 0, "q"));
  MX_TRY(check_out(s, R > 0, "s"));
  p->a = make_args(x, R, C, R);
  p->a.q = static_cast<uint8_t*>(q);
  p->a.s = static_cast<uint8_t*>(s);
  p->mode = kModeRow;
  p->gx = ceil_div(C, kCastTile);
  p->gy = ceil_div(R, kCastTile);
  p->gz = 1;
  return MX_OK;
}

mx_status prepare_dim1(const void* x, int64_t R, int64_t C, void* qt, void* st, PreparedCast* p) {
  MX_TRY(check_cast_geometry(x, R, C, true));
  MX_TRY(check_out(qt, R > 0, "qt"));
  MX_TRY(check_out(st, R > 0, "st"));
  p->a = make_args(x, R, C, R);
  p->a.qt = static_cast<uint8_t*>(qt);
  p->a.st = static_cast<uint8_t*>(st);
  p->mode = kModeCol;
  p->gx = ceil_div(C, kCastTile);
  p->gy = ceil_div(R, kCastTile);
  p->gz = 1;
  return MX_OK;
}

mx_status prepare_2d(const void* x, int64_t R, int64_t C, void* q, void* s, void* qt, void* st, PreparedCast* p) {
  MX_TRY(check_cast_geometry(x, R, C, true));
  MX_TRY(check_out(q, R > 0, "q"));
  MX_TRY(check_out(s, R > 0, "s"));
  MX_TRY(check_out(qt, R > 0, "qt"));
  MX_TRY(check_out(st, R > 0, "st"));
  p->a = make_args(x, R, C, R);
  p->a.q = static_cast<uint8_t*>(q);
  p->a.s = static_cast<uint8_t*>(s);
  p->a.qt = static_cast<uint8_t*>(qt);
  p->a.st = static_cast<uint8_t*>(st);
  p->mode = kModeRowCol;
  p->gx = ceil_div(C, kCastTile);
  p->gy = ceil_div(R, kCastTile);
  p->gz = 1;
  return MX_OK;
}

mx_status prepare_w32x32(const void* w, int64_t G, int64_t N, int64_t K, void* q, void* s_fwd, void* qt,
                         void* s_dgrad, PreparedCast* p) {
  MX_REQUIRE(G >= 0, MX_ERR_ARG, "G must be >= 0");
  MX_TRY(check_cast_geometry(w, N, K, true));
  MX_REQUIRE(N > 0, MX_ERR_ARG, "N must be > 0");
  MX_TRY(check_out(q, G > 0, "q"));
  MX_TRY(check_out(s_fwd, G > 0, "s_fwd"));
  MX_TRY(check_out(qt, false, "qt"));
  MX_TRY(check_out(s_dgrad, false, "s_dgrad"));
  p->a = make_args(w, N, K, N);
  p->a.q = static_cast<uint8_t*>(q);
  p->a.s = static_cast<uint8_t*>(s_fwd);
  p->a.qt = static_cast<uint8_t*>(qt);
  p->a.st = static_cast<uint8_t*>(s_dgrad);
  p->a.x_stride = N * K;
  p->a.q_stride = N * K;
  p->a.qt_stride = N * K;
  p->a.s_stride = scale_bytes(N, K / kBlock);
  p->a.st_stride = scale_bytes(K, N / kBlock);
  p->mode = kModeSquare;
  p->gx = ceil_div(K, kCastTile);
  p->gy = ceil_div(N, kCastTile);
  p->gz = G;
  return MX_OK;
}

mx_status launch_prepared(const PreparedCast& p, cudaStream_t st) {
  switch (p.mode) {
    case kModeRow: return launch_cast<kModeRow, false>(p.a, p.gx, p.gy, p.gz, st);
    case kModeCol: return launch_cast<kModeCol, false>(p.a, p.gx, p.gy, p.gz, st);
    case kModeRowCol: return launch_cast<kModeRowCol, false>(p.a, p.gx, p.gy, p.gz, st);
    case kModeSquare: return launch_cast<kModeSquare, false>(p.a, p.gx, p.gy, p.gz, st);
    default: return fail(MX_ERR_ARG, "internal: unprepared cast");
  }
}

// Launches the prepared casts `ps[0..n)` (in order) as one grid when their
// modes are one of the linear's combinations -- (32x32, rowwise),
// (fused, columnwise), (32x32, fused, columnwise) -- and one at a time
// otherwise. Empty casts are dropped.
mx_status launch_casts(const PreparedCast* ps, int n, cudaStream_t st) {
  const PreparedCast* c[3];
  int m = 0;
  for (int i = 0; i < n; ++i)
    if (ps[i].gx > 0 && ps[i].gy > 0 && ps[i].gz > 0) {
      MX_REQUIRE(m < 3, MX_ERR_ARG, "internal: more than three casts in one launch");
      c[m++] = &ps[i];
    }
  if (m == 0) return MX_OK;
  if (m == 1) return launch_prepared(*c[0], st);
  CastJobs j;
  memset(&j, 0, sizeof(j));
  int64_t total = 0;
  for (int i = 0; i < m; ++i) {
    MX_REQUIRE(c[i]->gx < (1ll << 31) && c[i]->gy <= 65535 && c[i]->gz <= 65535, MX_ERR_UNSUPPORTED,
               "cast grid too large (%lld x %lld x %lld tiles)", (long long)c[i]->gx, (long long)c[i]->gy,
               (long long)c[i]->gz);
    j.a[i] = c[i]->a;
    j.gx[i] = uint32_t(c[i]->gx);
    j.gy[i] = uint32_t(c[i]->gy);
    j.gz[i] = uint32_t(c[i]->gz);
    total += c[i]->gx * c[i]->gy * c[i]->gz;
  }
  if (total >= (1ll << 31)) {     // beyond one 1-D grid: each cast on its own
    for (int i = 0; i < m; ++i) MX_TRY(launch_prepared(*c[i], st));
    return MX_OK;
  }
  const dim3 grid{unsigned(total), 1u, 1u}, block{unsigned(kWarpCastThreads), 1u, 1u};
  if (m == 2 && c[0]->mode == kModeSquare && c[1]->mode == kModeRow)
    cast_multi_kernel<kModeSquare, kModeRow, -1><<<grid, block, kWarpCastSmem, st>>>(j);
  else if (m == 2 && c[0]->mode == kModeRowCol && c[1]->mode == kModeCol)
    cast_multi_kernel<kModeRowCol, kModeCol, -1><<<grid, block, kWarpCastSmem, st>>>(j);
  else if (m == 3 && c[0]->mode == kModeSquare && c[1]->mode == kModeRowCol && c[2]->mode == kModeCol)
    cast_multi_kernel<kModeSquare, kModeRowCol, kModeCol><<<grid, block, kWarpCastSmem, st>>>(j);
  else {
    for (int i = 0; i < m; ++i) MX_TRY(launch_prepared(*c[i], st));
    return MX_OK;
  }
  return cuda_check("cast launch");
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// Encoded tensor maps are kept in a small table keyed by every encode
// argument, so that launches over the same buffers (every step of a
// training loop) skip the encode. A map is a pure function of its
// arguments, so a hit is exactly what a fresh encode would return.
struct MapKey {
  const void* base;
  uint64_t dims[3], strides[2];
  uint32_t box[3];
  int dtype, rank, swizzle;
};

constexpr int kMapCacheSize = 64;
struct MapCacheEntry {
  MapKey key;
  CUtensorMap map;
  bool used;
};
std::mutex g_map_mu;
MapCacheEntry g_map_cache[kMapCacheSize];
int g_map_next = 0;

mx_status encode_tiled(CUtensorMap* m, CUtensorMapDataType dtype, int rank, const void* base, const uint64_t* dims,
                       const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle swizzle) {
  MapKey key;
  memset(&key, 0, sizeof(key));
  key.base = base;
  for (int i = 0; i < rank; ++i) key.dims[i] = dims[i], key.box[i] = box[i];
  for (int i = 0; i + 1 < rank; ++i) key.strides[i] = strides[i];
  key.dtype = int(dtype);
  key.rank = rank;
  key.swizzle = int(swizzle);
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    for (auto& e : g_map_cache)
      if (e.used && memcmp(&e.key, &key, sizeof(key)) == 0) {
        *m = e.map;
        return MX_OK;
      }
  }
  auto fn = encode_fn();
  MX_REQUIRE(fn != nullptr, MX_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t d[3], st[2];
  cuuint32_t bx[3], estr[3] = {1u, 1u, 1u};
  for (int i = 0; i < rank; ++i) d[i] = dims[i], bx[i] = box[i];
  for (int i = 0; i + 1 < rank; ++i) st[i] = strides[i];
  CUresult r = fn(m, dtype, cuuint32_t(rank), const_cast<void*>(base), d, st, bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  MX_REQUIRE(r == CUDA_SUCCESS, MX_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  std::lock_guard<std::mutex> lk(g_map_mu);
  MapCacheEntry& e = g_map_cache[g_map_next];
  g_map_next = (g_map_next + 1) % kMapCacheSize;
  e.key = key;
  e.map = *m;
  e.used = true;
  return MX_OK;
}

// 2D uint8 tensor map over a row-major [outer, inner] byte matrix, box
// {128, box_outer}, 128-byte swizzle, zero fill outside the tensor.
mx_status make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_outer) {
  const uint64_t dims[2] = {inner, outer}, strides[1] = {inner};
  const uint32_t box[2] = {128u, box_outer};
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// 2D map over a blocked scale buffer viewed as [chunks, 128] 32-bit words:
// one box = one 512-byte 128x4 scale tile; rows past the buffer read as zero.
mx_status make_scale_map(CUtensorMap* m, const void* base, uint64_t chunks) {
  const uint64_t dims[2] = {128u, chunks}, strides[1] = {512u};
  const uint32_t box[2] = {128u, 1u};
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

template <int kMode, bool kRowDests = false>
mx_status launch_gemm(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& msa, const CUtensorMap& msb,
                      const GemmArgs& ga, int64_t pair_tiles_ub, cudaStream_t st,
                      const RowDestsT<kRowDests>& rd = RowDestsT<kRowDests>()) {
  static int max_pairs[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  MX_REQUIRE(e == cudaSuccess && dev < 64, MX_ERR_CUDA, "cudaGetDevice failed");
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = kGemmSmem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (max_pairs[dev] == 0) {       // once per device: shared-memory attribute and the resident pairs
    e = cudaFuncSetAttribute(mx_gemm_kernel<kMode, kRowDests>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(kGemmSmem));
    MX_REQUIRE(e == cudaSuccess, MX_ERR_CUDA, "gemm smem attribute: %s", cudaGetErrorString(e));
    cfg.gridDim = dim3(2, 1, 1);
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, mx_gemm_kernel<kMode, kRowDests>, &cfg);
    MX_REQUIRE(e == cudaSuccess && n > 0, MX_ERR_CUDA, "no CTA pair fits on this device (%s)", cudaGetErrorString(e));
    max_pairs[dev] = n;
  }
  const int64_t pairs = pair_tiles_ub < max_pairs[dev] ? pair_tiles_ub : max_pairs[dev];
  cfg.gridDim = dim3(unsigned(2 * pairs), 1, 1);
  e = cudaLaunchKernelEx(&cfg, mx_gemm_kernel<kMode, kRowDests>, ma, mb, msa, msb, ga, rd);
  MX_REQUIRE(e == cudaSuccess, MX_ERR_CUDA, "gemm launch: %s", cudaGetErrorString(e));
  return cuda_check("gemm launch");
}


// bf16 tensor map over a row-major [outer, inner] matrix (rank 2) or a stack
// [depth, outer, inner] (rank 3): boxes of 64 elements (128 bytes) x
// box_outer rows (x 1 matrix), 128-byte swizzle, zero fill outside.
mx_status make_map_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t depth,
                        uint32_t box_outer) {
  const int rank = depth > 0 ? 3 : 2;
  const uint64_t dims[3] = {inner, outer, depth}, strides[2] = {inner * 2, inner * outer * 2};
  const uint32_t box[3] = {64u, box_outer, 1u};
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, base, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int kMode>
mx_status launch_bf16_gemm(const CUtensorMap& ma, const CUtensorMap& mb, const HGemmArgs& ha, int64_t pair_tiles_ub,
                           cudaStream_t st) {
  static int max_pairs[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  MX_REQUIRE(e == cudaSuccess && dev < 64, MX_ERR_CUDA, "cudaGetDevice failed");
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = kHGemmSmem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (max_pairs[dev] == 0) {       // once per device: shared-memory attribute and the resident pairs
    e = cudaFuncSetAttribute(bf16_gemm_kernel<kMode>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kHGemmSmem));
    MX_REQUIRE(e == cudaSuccess, MX_ERR_CUDA, "bf16 gemm smem attribute: %s", cudaGetErrorString(e));
    cfg.gridDim = dim3(2, 1, 1);
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, bf16_gemm_kernel<kMode>, &cfg);
    MX_REQUIRE(e == cudaSuccess && n > 0, MX_ERR_CUDA, "no CTA pair fits on this device (%s)", cudaGetErrorString(e));
    max_pairs[dev] = n;
  }
  const int64_t pairs = pair_tiles_ub < max_pairs[dev] ? pair_tiles_ub : max_pairs[dev];
  cfg.gridDim = dim3(unsigned(2 * pairs), 1, 1);
  e = cudaLaunchKernelEx(&cfg, bf16_gemm_kernel<kMode>, ma, mb, ha);
  MX_REQUIRE(e == cudaSuccess, MX_ERR_CUDA, "bf16 gemm launch: %s", cudaGetErrorString(e));
  return cuda_check("bf16 gemm launch");
}

// Grid for a grid-stride memory-bound kernel: every CTA resident at once
// (SMs x resident CTAs per SM, from the occupancy calculator), never more
// CTAs than the work needs.
template <typename Kernel>
unsigned streaming_grid(Kernel kernel, int64_t items, int threads) {
  int dev = 0, sms = 148, per_sm = 1;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  const int64_t need = ceil_div(items, threads);
  const int64_t cap = int64_t(sms) * per_sm;
  return unsigned(need < cap ? need : cap);
}

}  // namespace
}  // namespace mx

using namespace mx;

extern "C" {

const char* mx_last_error(void) { return g_err; }

size_t mx_scale_bytes(int64_t rows, int64_t cols) {
  if (rows <= 0 || cols <= 0) return 0;
  return size_t(scale_bytes(rows, cols));
}

int64_t mx_padded_rows_capacity(int64_t m_total, int32_t groups) {
  if (m_total < 0 || groups < 0) return -1;
  return ((m_total + 127ll * groups) / 128) * 128;
}

mx_status mx_device_error(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(MX_ERR_CUDA, "stream sync: %s", cudaGetErrorString(e));
  unsigned v = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
  if (e != cudaSuccess) return fail(MX_ERR_CUDA, "device flag: %s", cudaGetErrorString(e));
  if (v & kErrTimeout) return fail(MX_ERR_TIMEOUT, "a device pipeline wait timed out");
  if (v & kErrOffsets) return fail(MX_ERR_DEVICE, "invalid group offsets seen on the device");
  g_err[0] = '\0';
  return MX_OK;
}

mx_status mx_cast_dim0(const void* x, int64_t R, int64_t C, void* q, void* s, void* stream) {
  PreparedCast p;
  MX_TRY(prepare_dim0(x, R, C, q, s, &p));
  return launch_prepared(p, static_cast<cudaStream_t>(stream));
}

mx_status mx_cast_dim1(const void* x, int64_t R, int64_t C, void* qt, void* st, void* stream) {
  PreparedCast p;
  MX_TRY(prepare_dim1(x, R, C, qt, st, &p));
  return launch_prepared(p, static_cast<cudaStream_t>(stream));
}

mx_status mx_cast_2d(const void* x, int64_t R, int64_t C, void* q, void* s, void* qt, void* st,
                     void* stream) {
  PreparedCast p;
  MX_TRY(prepare_2d(x, R, C, q, s, qt, st, &p));
  return launch_prepared(p, static_cast<cudaStream_t>(stream));
}

mx_status mx_cast_w32x32(const void* w, int64_t G, int64_t N, int64_t K, void* q, void* s_fwd, void* qt,
                         void* s_dgrad, void* stream) {
  PreparedCast p;
  MX_TRY(prepare_w32x32(w, G, N, K, q, s_fwd, qt, s_dgrad, &p));
  return launch_prepared(p, static_cast<cudaStream_t>(stream));
}

mx_status mx_cast_dim0_grouped(const void* x, int64_t M, int64_t K, const int32_t* offs, int32_t G,
                               int64_t m_cap, void* q, void* s, void* stream) {
  MX_TRY(check_grouped(x, M, K, offs, G, m_cap));
  MX_TRY(check_out(q, m_cap > 0, "q"));
  MX_TRY(check_out(s, m_cap > 0, "s"));
  CastArgs a = make_args(x, M, K, m_cap);
  a.offs = offs;
  a.G = G;
  a.q = static_cast<uint8_t*>(q);
  a.s = static_cast<uint8_t*>(s);
  return launch_cast<kModeRow, true>(a, ceil_div(K, kCastTile), m_cap / kCastTile, 1,
                                     static_cast<cudaStream_t>(stream));
}

mx_status mx_cast_dim0_grouped_scatter(const void* x, int64_t M, int64_t K, const int32_t* offs, int32_t G,
                                       int64_t m_cap, void* const* dst_q, void* const* dst_s, void* stream) {
  MX_TRY(check_grouped(x, M, K, offs, G, m_cap));
  MX_REQUIRE(dst_q != nullptr && dst_s != nullptr, MX_ERR_ARG, "null destination arrays");
  ScatterDests d;
  memset(&d, 0, sizeof(d));
  for (int32_t g = 0; g < G; ++g) {
    MX_REQUIRE(dst_q[g] != nullptr && dst_s[g] != nullptr, MX_ERR_ARG, "null destination of group %d", g);
    MX_REQUIRE(aligned16(dst_q[g]) && aligned16(dst_s[g]), MX_ERR_ALIGN,
               "destination of group %d not 16-byte aligned", g);
    d.q[g] = static_cast<uint8_t*>(dst_q[g]);
    d.s[g] = static_cast<uint8_t*>(dst_s[g]);
  }
  if (m_cap == 0) return MX_OK;
  const int64_t row_tiles = m_cap / kCastTile, col_tiles = ceil_div(K, kCastTile);
  MX_REQUIRE(col_tiles < (1ll << 31) && row_tiles <= 65535, MX_ERR_UNSUPPORTED,
             "cast grid too large (%lld x %lld tiles)", (long long)col_tiles, (long long)row_tiles);
  CastArgs a = make_args(x, M, K, m_cap);
  a.offs = offs;
  a.G = G;
  cast_scatter_kernel<<<dim3(unsigned(col_tiles), unsigned(row_tiles), 1u), kWarpCastThreads, kWarpCastSmem,
                        static_cast<cudaStream_t>(stream)>>>(a, d);
  MX_TRY(cuda_check("scatter cast launch"));
  system_fence_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>();
  return cuda_check("fence launch");
}

mx_status mx_cast_2d_grouped_scatter(const void* x, int64_t M, int64_t K, const int32_t* offs, int32_t G,
                                     int64_t m_cap, void* const* dst_q, void* const* dst_s, void* const* dst_qt,
                                     void* const* dst_st, const int64_t* dst_cap, void* stream) {
  MX_TRY(check_grouped(x, M, K, offs, G, m_cap));
  MX_REQUIRE(G <= kScatter2dMaxGroups, MX_ERR_UNSUPPORTED, "G = %d above the fused scatter's %d groups", G,
             kScatter2dMaxGroups);
  MX_REQUIRE(dst_q && dst_s && dst_qt && dst_st && dst_cap, MX_ERR_ARG, "null destination arrays");
  ScatterDests2d d;
  memset(&d, 0, sizeof(d));
  for (int32_t g = 0; g < G; ++g) {
    MX_REQUIRE(dst_q[g] && dst_s[g] && dst_qt[g] && dst_st[g], MX_ERR_ARG, "null destination of group %d", g);
    MX_REQUIRE(aligned16(dst_q[g]) && aligned16(dst_s[g]) && aligned16(dst_qt[g]) && aligned16(dst_st[g]),
               MX_ERR_ALIGN, "destination of group %d not 16-byte aligned", g);
    MX_REQUIRE(dst_cap[g] > 0 && dst_cap[g] % kCastTile == 0 && dst_cap[g] < (1ll << 31), MX_ERR_ARG,
               "destination capacity of group %d (%lld) must be a positive multiple of 128 below 2^31", g,
               (long long)dst_cap[g]);
    d.q[g] = static_cast<uint8_t*>(dst_q[g]);
    d.s[g] = static_cast<uint8_t*>(dst_s[g]);
    d.qt[g] = static_cast<uint8_t*>(dst_qt[g]);
    d.st[g] = static_cast<uint8_t*>(dst_st[g]);
    d.cap[g] = int32_t(dst_cap[g]);
  }
  if (m_cap == 0) return MX_OK;
  const int64_t row_tiles = m_cap / kCastTile, col_tiles = ceil_div(K, kCastTile);
  MX_REQUIRE(col_tiles < (1ll << 31) && row_tiles <= 65535, MX_ERR_UNSUPPORTED,
             "cast grid too large (%lld x %lld tiles)", (long long)col_tiles, (long long)row_tiles);
  CastArgs a = make_args(x, M, K, m_cap);
  a.offs = offs;
  a.G = G;
  cast_scatter2d_kernel<<<dim3(unsigned(col_tiles), unsigned(row_tiles), 1u), kWarpCastThreads, kWarpCastSmem,
                          static_cast<cudaStream_t>(stream)>>>(a, d);
  MX_TRY(cuda_check("fused scatter cast launch"));
  system_fence_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>();
  return cuda_check("fence launch");
}

mx_status mx_cast_dim1_grouped(const void* x, int64_t M, int64_t K, const int32_t* offs, int32_t G,
                               int64_t m_cap, void* qt, void* st, void* stream) {
  MX_TRY(check_grouped(x, M, K, offs, G, m_cap));
  MX_TRY(check_out(qt, m_cap > 0, "qt"));
  MX_TRY(check_out(st, m_cap > 0, "st"));
  CastArgs a = make_args(x, M, K, m_cap);
  a.offs = offs;
  a.G = G;
  a.qt = static_cast<uint8_t*>(qt);
  a.st = static_cast<uint8_t*>(st);
  return launch_cast<kModeCol, true>(a, ceil_div(K, kCastTile), m_cap / kCastTile, 1,
                                     static_cast<cudaStream_t>(stream));
}

mx_status mx_cast_2d_grouped(const void* x, int64_t M, int64_t K, const int32_t* offs, int32_t G,
                             int64_t m_cap, void* q, void* s, void* qt, void* st, void* stream) {
  MX_TRY(check_grouped(x, M, K, offs, G, m_cap));
  MX_TRY(check_out(q, m_cap > 0, "q"));
  MX_TRY(check_out(s, m_cap > 0, "s"));
  MX_TRY(check_out(qt, m_cap > 0, "qt"));
  MX_TRY(check_out(st, m_cap > 0, "st"));
  CastArgs a = make_args(x, M, K, m_cap);
  a.offs = offs;
  a.G = G;
  a.q = static_cast<uint8_t*>(q);
  a.s = static_cast<uint8_t*>(s);
  a.qt = static_cast<uint8_t*>(qt);
  a.st = static_cast<uint8_t*>(st);
  return launch_cast<kModeRowCol, true>(a, ceil_div(K, kCastTile), m_cap / kCastTile, 1,
                                        static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace mx {
namespace {
// The M-group modes of the grouped GEMM (forward, and dgrad with B read
// MN-major), arguments checked by the caller: tensor maps and the launch,
// with per-group output rows when kRowDests.
template <bool kRowDests>
mx_status grouped_mm_m_modes(const void* a_q, const void* a_s, const void* b_q, const void* b_s,
                             const int32_t* offs, int32_t G, int32_t E, int32_t mode, GemmArgs& ga, int64_t M,
                             int64_t N, int64_t K, int64_t m_cap, cudaStream_t st, const RowDestsT<kRowDests>& rd) {
  CUtensorMap map_a, map_b, map_sa, map_sb;
  const int64_t rows_a = offs ? m_cap : M;
  ga.m_cap = offs ? m_cap : ceil_to(M, kBM);
  if (rows_a == 0 || M == 0) return MX_OK;
  MX_REQUIRE(a_q && a_s && b_q && b_s, MX_ERR_ARG, "null operand");
  ga.a_sc_tiles = ceil_div(K, kBK);
  ga.b_sc_tiles = ceil_div(K, kBK);
  ga.b_sc_group_chunks = scale_bytes(N, K / kBlock) / 512;
  MX_TRY(make_map(&map_a, a_q, uint64_t(K), uint64_t(rows_a), kCtaM));
  if (mode == MX_GROUPS_M_KN)
    MX_TRY(make_map(&map_b, b_q, uint64_t(N), uint64_t(E) * uint64_t(K), kBK));
  else
    MX_TRY(make_map(&map_b, b_q, uint64_t(K), uint64_t(E) * uint64_t(N), kBN / 2));
  MX_TRY(make_scale_map(&map_sa, a_s, uint64_t(scale_bytes(rows_a, K / kBlock) / 512)));
  MX_TRY(make_scale_map(&map_sb, b_s, uint64_t(E) * uint64_t(ga.b_sc_group_chunks)));
  const int64_t pair_tiles_ub = (ceil_div(rows_a, kPairM) + (offs ? G : 0)) * ceil_div(N, kBN);
  if (mode == MX_GROUPS_M_KN)
    return launch_gemm<kGroupsMKn, kRowDests>(map_a, map_b, map_sa, map_sb, ga, pair_tiles_ub, st, rd);
  return launch_gemm<kGroupsM, kRowDests>(map_a, map_b, map_sa, map_sb, ga, pair_tiles_ub, st, rd);
}
}  // namespace
}  // namespace mx

extern "C" {

}  // extern "C"

namespace mx {
namespace {
mx_status check_grouped_gemm(int32_t mode, const int32_t* offs, int32_t G, int32_t E, int64_t M, int64_t N, int64_t K,
                             int64_t m_cap) {
  MX_REQUIRE(mode == MX_GROUPS_M || mode == MX_GROUPS_K || mode == MX_GROUPS_M_KN, MX_ERR_ARG, "unknown mode %d",
             mode);
  MX_REQUIRE(M >= 0 && N > 0 && K > 0, MX_ERR_ARG, "sizes must be M >= 0, N > 0, K > 0");
  if (offs != nullptr) {
    MX_REQUIRE(G >= 1 && G <= kMaxGroups, MX_ERR_ARG, "G = %d outside [1, %d]", G, kMaxGroups);
    MX_REQUIRE(E >= 1 && E <= G && G % E == 0, MX_ERR_ARG, "E = %d must divide G = %d", E, G);
    MX_REQUIRE(m_cap >= M && m_cap % 128 == 0 && m_cap < (1ll << 31), MX_ERR_ARG,
               "m_cap = %lld must be a multiple of 128, >= M and < 2^31", (long long)m_cap);
    MX_REQUIRE((reinterpret_cast<uintptr_t>(offs) & 3u) == 0, MX_ERR_ALIGN, "offsets not 4-byte aligned");
  } else {
    MX_REQUIRE(G == 1 && E == 1, MX_ERR_ARG, "without offsets G and E must be 1 (dense)");
    MX_REQUIRE(M < (1ll << 31), MX_ERR_ARG, "M too large");
  }
  return MX_OK;
}
}  // namespace
}  // namespace mx

extern "C" {

mx_status mx_grouped_mm_experts_to_rows(const void* a_q, const void* a_s, const void* b_q, const void* b_s,
                                        const int32_t* offs, int32_t G, int32_t E, int32_t mode,
                                        void* const* out_rows, int64_t M, int64_t N, int64_t K, int64_t m_cap,
                                        void* stream) {
  MX_REQUIRE(mode == MX_GROUPS_M || mode == MX_GROUPS_M_KN, MX_ERR_ARG,
             "per-group output rows take the M-group modes (got %d)", mode);
  MX_REQUIRE(offs != nullptr, MX_ERR_ARG, "per-group output rows need offsets");
  MX_TRY(check_grouped_gemm(mode, offs, G, E, M, N, K, m_cap));
  MX_REQUIRE(out_rows != nullptr, MX_ERR_ARG, "null output row array");
  RowDests rd;
  memset(&rd, 0, sizeof(rd));
  for (int32_t g = 0; g < G; ++g) {
    MX_REQUIRE(out_rows[g] != nullptr, MX_ERR_ARG, "null output rows of group %d", g);
    MX_REQUIRE(aligned16(out_rows[g]), MX_ERR_ALIGN, "output rows of group %d not 16-byte aligned", g);
    rd.base[g] = static_cast<__nv_bfloat16*>(out_rows[g]);
  }
  const void* ptrs[4] = {a_q, a_s, b_q, b_s};
  for (const void* p : ptrs) MX_REQUIRE(aligned16(p), MX_ERR_ALIGN, "operand not 16-byte aligned");
  MX_REQUIRE(N % kBlock == 0 && K % kBlock == 0, MX_ERR_UNSUPPORTED,
             "N = %lld and K = %lld must be multiples of 32", (long long)N, (long long)K);
  MX_REQUIRE(N < (1ll << 31) && K < (1ll << 31), MX_ERR_ARG, "N or K is 2^31 or more");
  GemmArgs ga;
  memset(&ga, 0, sizeof(ga));
  ga.offs = offs;
  ga.G = G;
  ga.E = E;
  ga.M = M;
  ga.N = N;
  ga.K = K;
  return grouped_mm_m_modes<true>(a_q, a_s, b_q, b_s, offs, G, E, mode, ga, M, N, K, m_cap,
                                  static_cast<cudaStream_t>(stream), rd);
}

mx_status mx_grouped_mm_experts(const void* a_q, const void* a_s, const void* b_q, const void* b_s,
                                const int32_t* offs, int32_t G, int32_t E, int32_t mode, void* out, int64_t M,
                                int64_t N, int64_t K, int64_t m_cap, void* stream) {
  MX_TRY(check_grouped_gemm(mode, offs, G, E, M, N, K, m_cap));
  const void* ptrs[5] = {a_q, a_s, b_q, b_s, out};
  for (const void* p : ptrs) MX_REQUIRE(aligned16(p), MX_ERR_ALIGN, "operand not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  GemmArgs ga;
  memset(&ga, 0, sizeof(ga));
  ga.offs = offs;
  ga.out = static_cast<__nv_bfloat16*>(out);
  ga.G = G;
  ga.E = E;
  ga.M = M;
  ga.N = N;
  ga.K = K;
  CUtensorMap map_a, map_b, map_sa, map_sb;
  // Every size is a multiple of 32 (the block of a scale). A size that is
  // not a multiple of the tile (256 output columns, 128-deep K steps) is the
  // pad path: TMA fills operand tiles past the tensor with zero codes (pad
  // scale bytes are 0x00), so past-the-end K adds nothing; output rows and
  // 32-column chunks past the tensor are never stored.
  MX_REQUIRE(N % kBlock == 0 && K % kBlock == 0, MX_ERR_UNSUPPORTED,
             "N = %lld and K = %lld must be multiples of 32", (long long)N, (long long)K);
  MX_REQUIRE(N < (1ll << 31) && K < (1ll << 31), MX_ERR_ARG, "N or K is 2^31 or more");
  if (mode != MX_GROUPS_K) {
    MX_REQUIRE(out != nullptr || M == 0, MX_ERR_ARG, "null output");
    return grouped_mm_m_modes<false>(a_q, a_s, b_q, b_s, offs, G, E, mode, ga, M, N, K, m_cap, st, NoRowDests());
  }
  MX_REQUIRE(out != nullptr, MX_ERR_ARG, "null output");
  const int64_t len = offs ? m_cap : M;
  MX_REQUIRE(offs || M % kBlock == 0, MX_ERR_UNSUPPORTED, "dense K-groups needs M %% 32 == 0");
  ga.m_cap = offs ? m_cap : ceil_to(M, kBM);
  if (len == 0) {
    cudaError_t e = cudaMemsetAsync(out, 0, size_t(E) * N * K * 2, st);
    MX_REQUIRE(e == cudaSuccess, MX_ERR_CUDA, "memset: %s", cudaGetErrorString(e));
    return MX_OK;
  }
  MX_REQUIRE(a_q && a_s && b_q && b_s, MX_ERR_ARG, "null operand");
  ga.a_sc_tiles = ceil_div(ceil_div(len, kBlock), 4);
  ga.b_sc_tiles = ga.a_sc_tiles;
  ga.b_sc_group_chunks = 0;
  MX_TRY(make_map(&map_a, a_q, uint64_t(len), uint64_t(N), kCtaM));
  MX_TRY(make_map(&map_b, b_q, uint64_t(len), uint64_t(K), kBN / 2));
  MX_TRY(make_scale_map(&map_sa, a_s, uint64_t(scale_bytes(N, ceil_div(len, kBlock)) / 512)));
  MX_TRY(make_scale_map(&map_sb, b_s, uint64_t(scale_bytes(K, ceil_div(len, kBlock)) / 512)));
  const int64_t pair_tiles_ub = int64_t(E) * ceil_div(N, kPairM) * ceil_div(K, kBN);
  return launch_gemm<kGroupsK>(map_a, map_b, map_sa, map_sb, ga, pair_tiles_ub, st);
}

mx_status mx_grouped_mm(const void* a_q, const void* a_s, const void* b_q, const void* b_s,
                        const int32_t* offs, int32_t G, int32_t mode, void* out, int64_t M, int64_t N,
                        int64_t K, int64_t m_cap, void* stream) {
  return mx_grouped_mm_experts(a_q, a_s, b_q, b_s, offs, G, G, mode, out, M, N, K, m_cap, stream);
}

mx_wcache* mx_wcache_create(void) { return new (std::nothrow) mx_wcache(); }

void mx_wcache_clear(mx_wcache* c) {
  if (c == nullptr) return;
  std::lock_guard<std::mutex> lk(c->mu);
  for (auto& e : c->entries) cudaFree(e.q);
  c->entries.clear();
}

void mx_wcache_evict(mx_wcache* c, const void* w) {
  if (c == nullptr) return;
  std::lock_guard<std::mutex> lk(c->mu);
  for (auto& e : c->entries)
    if (e.w == w && w != nullptr) {
      e.w = nullptr;          // unbound: the buffer waits for a miss of the same shape
      e.valid = false;
    }
}

void mx_wcache_destroy(mx_wcache* c) {
  mx_wcache_clear(c);
  delete c;
}

mx_status mx_wcache_stats(mx_wcache* c, int64_t* hits, int64_t* misses, int64_t* entries) {
  MX_REQUIRE(c != nullptr, MX_ERR_ARG, "null cache");
  std::lock_guard<std::mutex> lk(c->mu);
  if (hits) *hits = c->hits;
  if (misses) *misses = c->misses;
  if (entries) {
    int64_t bound = 0;
    for (const auto& e : c->entries) bound += e.w != nullptr;
    *entries = bound;
  }
  return MX_OK;
}

size_t mx_linear_ws_bytes(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N <= 0 || K <= 0) return 0;
  const int64_t fwd = ceil_to(M * K, 256) + ceil_to(scale_bytes(M, K / kBlock), 256);
  const int64_t bwd = 2 * ceil_to(M * N, 256) + ceil_to(scale_bytes(M, N / kBlock), 256) +
                      ceil_to(scale_bytes(N, M / kBlock), 256) + ceil_to(K * M, 256) +
                      ceil_to(scale_bytes(K, M / kBlock), 256);
  return size_t((fwd > bwd ? fwd : bwd) + wq_bytes(N, K));
}

size_t mx_linear_train_ws_bytes(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N <= 0 || K <= 0) return 0;
  return size_t(linear_train_ws_bytes(M, N, K));
}

}  // extern "C"

namespace mx {
namespace {

mx_status check_linear(int64_t M, int64_t N, int64_t K, void* ws, size_t ws_bytes, bool train = false) {
  MX_REQUIRE(M >= 0 && N > 0 && K > 0, MX_ERR_ARG, "sizes must be M >= 0, N > 0, K > 0");
  MX_REQUIRE(M % kBlock == 0, MX_ERR_UNSUPPORTED, "M = %lld is not a multiple of 32", (long long)M);
  MX_REQUIRE(N % kBlock == 0 && K % kBlock == 0, MX_ERR_UNSUPPORTED, "N and K must be multiples of 32");
  const size_t need = train ? mx_linear_train_ws_bytes(M, N, K) : mx_linear_ws_bytes(M, N, K);
  MX_REQUIRE(ws_bytes >= need, MX_ERR_ARG, "workspace too small (%zu < %zu bytes)", ws_bytes, need);
  MX_REQUIRE(ws != nullptr && aligned16(ws), MX_ERR_ALIGN, "workspace null or not 16-byte aligned");
  return MX_OK;
}

// Where this call's 32x32 quantization of W comes from: the cache (hit), a
// re-cast into the cache (miss or stale version), or a cast into the
// workspace tail (no cache). A cast to run is returned prepared (`cast.mode`
// >= 0), so that it can share a launch with the activation casts; a cache
// entry being refilled is marked invalid here and valid by commit_weight once
// its cast is launched. The caller holds the cache's lock from plan to commit.
struct WeightPlan {
  WeightView view;
  PreparedCast cast;
  mx_wcache::Entry* entry = nullptr;
  uint64_t version = 0;
};

mx_status plan_weight(const void* w, int64_t N, int64_t K, mx_wcache* cache, uint64_t version, uint8_t* ws_tail,
                      WeightPlan* out) {
  if (cache == nullptr) {
    out->view = carve_weight(ws_tail, N, K);
    return prepare_w32x32(w, 1, N, K, out->view.q, out->view.s_fwd, nullptr, out->view.s_dgrad, &out->cast);
  }
  mx_wcache::Entry* e = nullptr;
  for (auto& x : cache->entries)
    if (x.w == w && x.N == N && x.K == K) e = &x;
  if (e != nullptr && e->valid && e->version == version) {
    ++cache->hits;
    out->view = carve_weight(e->q, N, K);
    return MX_OK;
  }
  ++cache->misses;
  if (e == nullptr) {            // an evicted entry's buffer of the same shape, if any
    for (auto& x : cache->entries)
      if (x.w == nullptr && x.N == N && x.K == K) {
        e = &x;
        e->w = w;
        break;
      }
  }
  if (e == nullptr) {
    uint8_t* buf = nullptr;
    cudaError_t err = cudaMalloc(&buf, size_t(wq_bytes(N, K)));
    MX_REQUIRE(err == cudaSuccess, MX_ERR_CUDA, "weight cache allocation: %s", cudaGetErrorString(err));
    cache->entries.push_back(mx_wcache::Entry());
    e = &cache->entries.back();
    e->w = w;
    e->N = N;
    e->K = K;
    e->q = buf;
  }
  out->view = carve_weight(e->q, N, K);
  e->valid = false;
  MX_TRY(prepare_w32x32(w, 1, N, K, out->view.q, out->view.s_fwd, nullptr, out->view.s_dgrad, &out->cast));
  out->entry = e;
  out->version = version;
  return MX_OK;
}

void commit_weight(const WeightPlan& p) {
  if (p.entry != nullptr) {
    p.entry->version = p.version;
    p.entry->valid = true;
  }
}

std::unique_lock<std::mutex> lock_cache(mx_wcache* cache) {
  return cache ? std::unique_lock<std::mutex>(cache->mu) : std::unique_lock<std::mutex>();
}

}  // namespace
}  // namespace mx

extern "C" {

mx_status mx_linear_fwd(const void* x, const void* w, int64_t M, int64_t N, int64_t K, mx_wcache* cache,
                        uint64_t w_version, void* y, void* ws, size_t ws_bytes, void* stream) {
  MX_TRY(check_linear(M, N, K, ws, ws_bytes));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* p = static_cast<uint8_t*>(ws);
  uint8_t* xq = p;
  uint8_t* xs = xq + ceil_to(M * K, 256);
  uint8_t* tail = p + (mx_linear_ws_bytes(M, N, K) - wq_bytes(N, K));
  // the weight's cast (on a miss) and X's rowwise cast go out as one launch
  std::unique_lock<std::mutex> lk = lock_cache(cache);
  WeightPlan wp;
  MX_TRY(plan_weight(w, N, K, cache, w_version, tail, &wp));
  PreparedCast casts[2];
  casts[0] = wp.cast;
  if (M > 0) MX_TRY(prepare_dim0(x, M, K, xq, xs, &casts[1]));
  MX_TRY(launch_casts(casts, 2, st));
  commit_weight(wp);
  if (lk.owns_lock()) lk.unlock();
  if (M == 0) return MX_OK;
  const WeightView& wv = wp.view;
  return mx_grouped_mm(xq, xs, wv.q, wv.s_fwd, nullptr, 1, MX_GROUPS_M, y, M, N, K, 0, stream);
}

mx_status mx_linear_bwd(const void* dy, const void* x, const void* w, int64_t M, int64_t N, int64_t K,
                        mx_wcache* cache, uint64_t w_version, void* dx, void* dw, void* ws, size_t ws_bytes,
                        void* stream) {
  MX_TRY(check_linear(M, N, K, ws, ws_bytes));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* p = static_cast<uint8_t*>(ws);
  uint8_t* dyq = p;                                              // [M, N]
  uint8_t* dys = dyq + ceil_to(M * N, 256);                      // blocked(M, N/32)
  uint8_t* dyqt = dys + ceil_to(scale_bytes(M, N / kBlock), 256);  // [N, M]
  uint8_t* dyst = dyqt + ceil_to(M * N, 256);                    // blocked(N, M/32)
  uint8_t* xqt = dyst + ceil_to(scale_bytes(N, M / kBlock), 256);  // [K, M]
  uint8_t* xst = xqt + ceil_to(K * M, 256);                      // blocked(K, M/32)
  uint8_t* tail = p + (mx_linear_ws_bytes(M, N, K) - wq_bytes(N, K));
  // the weight's cast (on a miss), dY's fused cast and X's columnwise cast
  // go out as one launch
  std::unique_lock<std::mutex> lk = lock_cache(cache);
  WeightPlan wp;
  MX_TRY(plan_weight(w, N, K, cache, w_version, tail, &wp));
  PreparedCast casts[3];
  casts[0] = wp.cast;
  if (M > 0) {
    MX_TRY(prepare_2d(dy, M, N, dyq, dys, dyqt, dyst, &casts[1]));
    MX_TRY(prepare_dim1(x, M, K, xqt, xst, &casts[2]));
  }
  MX_TRY(launch_casts(casts, 3, st));
  commit_weight(wp);
  if (lk.owns_lock()) lk.unlock();
  if (M == 0) {
    cudaError_t e = cudaMemsetAsync(dw, 0, size_t(N) * K * 2, st);
    MX_REQUIRE(e == cudaSuccess, MX_ERR_CUDA, "memset: %s", cudaGetErrorString(e));
    return MX_OK;
  }
  const WeightView& wv = wp.view;
  MX_TRY(mx_grouped_mm(dyq, dys, wv.q, wv.s_dgrad, nullptr, 1, MX_GROUPS_M_KN, dx, M, K, N, 0, stream));
  return mx_grouped_mm(dyqt, dyst, xqt, xst, nullptr, 1, MX_GROUPS_K, dw, M, N, K, 0, stream);
}

mx_status mx_linear_fwd_train(const void* x, const void* w, int64_t M, int64_t N, int64_t K, mx_wcache* cache,
                              uint64_t w_version, void* y, void* ws, size_t ws_bytes, void* stream) {
  MX_TRY(check_linear(M, N, K, ws, ws_bytes, true));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const LinearTrainWs L = carve_train_ws(ws, M, N, K);
  // the weight's cast (on a miss) and X's fused rowwise + columnwise cast go
  // out as one launch; the columnwise codes stay in the workspace for the backward
  std::unique_lock<std::mutex> lk = lock_cache(cache);
  WeightPlan wp;
  MX_TRY(plan_weight(w, N, K, cache, w_version, L.wq, &wp));
  PreparedCast casts[2];
  casts[0] = wp.cast;
  if (M > 0) MX_TRY(prepare_2d(x, M, K, L.xq, L.xs, L.xqt, L.xst, &casts[1]));
  MX_TRY(launch_casts(casts, 2, st));
  commit_weight(wp);
  if (lk.owns_lock()) lk.unlock();
  if (M == 0) return MX_OK;
  const WeightView& wv = wp.view;
  return mx_grouped_mm(L.xq, L.xs, wv.q, wv.s_fwd, nullptr, 1, MX_GROUPS_M, y, M, N, K, 0, stream);
}

mx_status mx_linear_bwd_after_fwd(const void* dy, const void* w, int64_t M, int64_t N, int64_t K,
                                  mx_wcache* cache, uint64_t w_version, void* dx, void* dw, void* ws,
                                  size_t ws_bytes, void* stream) {
  MX_TRY(check_linear(M, N, K, ws, ws_bytes, true));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const LinearTrainWs L = carve_train_ws(ws, M, N, K);
  // X's columnwise cast is the forward's; the weight's quantization is the
  // forward's (workspace) or the cache's (re-cast only on a miss); dY's fused
  // cast is the one cast of this call
  std::unique_lock<std::mutex> lk = lock_cache(cache);
  WeightPlan wp;
  if (cache != nullptr) MX_TRY(plan_weight(w, N, K, cache, w_version, L.wq, &wp));
  else wp.view = carve_weight(L.wq, N, K);
  PreparedCast casts[2];
  casts[0] = wp.cast;
  if (M > 0) MX_TRY(prepare_2d(dy, M, N, L.dyq, L.dys, L.dyqt, L.dyst, &casts[1]));
  MX_TRY(launch_casts(casts, 2, st));
  commit_weight(wp);
  if (lk.owns_lock()) lk.unlock();
  if (M == 0) {
    cudaError_t e = cudaMemsetAsync(dw, 0, size_t(N) * K * 2, st);
    MX_REQUIRE(e == cudaSuccess, MX_ERR_CUDA, "memset: %s", cudaGetErrorString(e));
    return MX_OK;
  }
  const WeightView& wv = wp.view;
  MX_TRY(mx_grouped_mm(L.dyq, L.dys, wv.q, wv.s_dgrad, nullptr, 1, MX_GROUPS_M_KN, dx, M, K, N, 0, stream));
  return mx_grouped_mm(L.dyqt, L.dyst, L.xqt, L.xst, nullptr, 1, MX_GROUPS_K, dw, M, N, K, 0, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Linear forward without a caller workspace and without any allocation.
//
// Some callers cannot hand this library a workspace: a plain C host program
// that links libmx without a device allocator of its own, or a plugin that
// runs inside a runtime which reserves all device memory up front and does
// not allow further cudaMalloc calls (cudaMalloc can also synchronise the
// device, which such hosts avoid). mx_linear_fwd_noalloc serves them: its
// scratch (the quantized activations and weight) lives in the fixed array
// below, which every GPU that loads this library holds until the process
// exits.
// ---------------------------------------------------------------------------
namespace mx {
namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[MX_LINEAR_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device. In host code
// the array's name is only a host-side stand-in, so the address is obtained
// once per device (with that device current) and reused.
mx_status noalloc_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  MX_REQUIRE(e == cudaSuccess, MX_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  MX_REQUIRE(dev >= 0 && dev < kMaxDevices, MX_ERR_UNSUPPORTED, "device %d beyond %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    MX_REQUIRE(e == cudaSuccess && p != nullptr, MX_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return MX_OK;
}

}  // namespace
}  // namespace mx

extern "C" mx_status mx_linear_fwd_noalloc(const void* x, const void* w, int64_t M, int64_t N, int64_t K, void* y,
                                           void* stream) {
  MX_REQUIRE(M >= 0 && N > 0 && K > 0, MX_ERR_ARG, "sizes must be M >= 0, N > 0, K > 0");
  MX_REQUIRE(M % kBlock == 0, MX_ERR_UNSUPPORTED, "M = %lld is not a multiple of 32", (long long)M);
  MX_REQUIRE(N % kBlock == 0 && K % kBlock == 0, MX_ERR_UNSUPPORTED, "N and K must be multiples of 32");
  // Bound each factor before any product, so that no size can overflow the
  // byte count below and slip past the scratch bound.
  constexpr int64_t kScratch = int64_t(MX_LINEAR_NOALLOC_SCRATCH_BYTES);
  MX_REQUIRE(M <= kScratch / K && N <= kScratch / K, MX_ERR_UNSUPPORTED,
             "mx_linear_fwd_noalloc: M=%lld N=%lld K=%lld exceed its static scratch of %lld bytes (use "
             "mx_linear_fwd with a workspace)",
             (long long)M, (long long)N, (long long)K, (long long)kScratch);
  const int64_t xq_b = ceil_to(M * K, 256), xs_b = ceil_to(scale_bytes(M, K / kBlock), 256);
  const int64_t wq_b = ceil_to(N * K, 256), ws_b = ceil_to(scale_bytes(N, K / kBlock), 256);
  const int64_t need = xq_b + xs_b + wq_b + ws_b;
  MX_REQUIRE(need <= int64_t(MX_LINEAR_NOALLOC_SCRATCH_BYTES), MX_ERR_UNSUPPORTED,
             "mx_linear_fwd_noalloc needs %lld bytes of scratch for M=%lld N=%lld K=%lld; its static scratch "
             "holds %lld bytes (use mx_linear_fwd with a workspace)",
             (long long)need, (long long)M, (long long)N, (long long)K, (long long)MX_LINEAR_NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  MX_TRY(noalloc_scratch(&scratch));
  uint8_t* xq = static_cast<uint8_t*>(scratch);
  uint8_t* xs = xq + xq_b;
  uint8_t* wq = xs + xs_b;
  uint8_t* wsf = wq + wq_b;
  // Every scratch byte the GEMM reads is written by the two casts of this
  // call (codes and every scale byte, pads included), so nothing needs
  // clearing between calls.
  PreparedCast casts[2];
  MX_TRY(prepare_w32x32(w, 1, N, K, wq, wsf, nullptr, nullptr, &casts[0]));
  if (M > 0) MX_TRY(prepare_dim0(x, M, K, xq, xs, &casts[1]));
  MX_TRY(launch_casts(casts, 2, static_cast<cudaStream_t>(stream)));
  if (M == 0) return MX_OK;
  return mx_grouped_mm(xq, xs, wq, wsf, nullptr, 1, MX_GROUPS_M, y, M, N, K, 0, stream);
}

extern "C" mx_status mx_cast_ex(const void* x, int64_t R, int64_t C, int32_t dims, int32_t rule, void* q, void* s,
                                void* qt, void* st, void* stream) {
  MX_REQUIRE(dims >= 1 && dims <= 3, MX_ERR_ARG, "dims must be 1 (rowwise), 2 (columnwise) or 3 (both)");
  MX_REQUIRE(rule == MX_RCEIL || rule == MX_FLOOR, MX_ERR_ARG, "unknown scale rule %d", rule);
  if (rule == MX_RCEIL) {
    if (dims == 1) return mx_cast_dim0(x, R, C, q, s, stream);
    if (dims == 2) return mx_cast_dim1(x, R, C, qt, st, stream);
    return mx_cast_2d(x, R, C, q, s, qt, st, stream);
  }
  MX_TRY(check_cast_geometry(x, R, C, dims != 1));
  if (dims & 1) {
    MX_TRY(check_out(q, R > 0, "q"));
    MX_TRY(check_out(s, R > 0, "s"));
  }
  if (dims & 2) {
    MX_TRY(check_out(qt, R > 0, "qt"));
    MX_TRY(check_out(st, R > 0, "st"));
  }
  CastArgs a = make_args(x, R, C, R);
  a.q = static_cast<uint8_t*>(q);
  a.s = static_cast<uint8_t*>(s);
  a.qt = static_cast<uint8_t*>(qt);
  a.st = static_cast<uint8_t*>(st);
  cudaStream_t stm = static_cast<cudaStream_t>(stream);
  const int64_t ct = ceil_div(C, kCastTile), rt = ceil_div(R, kCastTile);
  if (dims == 1) return launch_cast<kModeRow | kModeFloor, false>(a, ct, rt, 1, stm);
  if (dims == 2) return launch_cast<kModeCol | kModeFloor, false>(a, ct, rt, 1, stm);
  return launch_cast<kModeRowCol | kModeFloor, false>(a, ct, rt, 1, stm);
}

// ------------------------------------------------ backward-override arms ---
extern "C" mx_status mx_grouped_mm_bf16(const void* a, const void* b, const int32_t* offs, int32_t G, int32_t mode,
                                        void* out, int64_t M, int64_t N, int64_t K, void* stream) {
  MX_REQUIRE(mode == MX_GROUPS_M || mode == MX_GROUPS_K, MX_ERR_ARG, "unknown mode %d", mode);
  MX_REQUIRE(M >= 0 && N > 0 && K > 0, MX_ERR_ARG, "sizes must be M >= 0, N > 0, K > 0");
  MX_REQUIRE(M < (1ll << 31) && N < (1ll << 31) && K < (1ll << 31), MX_ERR_ARG, "a size is 2^31 or more");
  if (offs != nullptr) {
    MX_REQUIRE(G >= 1 && G <= kMaxGroups, MX_ERR_ARG, "G = %d outside [1, %d]", G, kMaxGroups);
    MX_REQUIRE((reinterpret_cast<uintptr_t>(offs) & 3u) == 0, MX_ERR_ALIGN, "offsets not 4-byte aligned");
  } else {
    MX_REQUIRE(G == 1, MX_ERR_ARG, "without offsets G must be 1 (dense)");
  }
  const void* ptrs[3] = {a, b, out};
  for (const void* p : ptrs) MX_REQUIRE(aligned16(p), MX_ERR_ALIGN, "operand not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  HGemmArgs ha;
  memset(&ha, 0, sizeof(ha));
  ha.offs = offs;
  ha.out = static_cast<__nv_bfloat16*>(out);
  ha.G = G;
  ha.M = M;
  ha.N = N;
  ha.K = K;
  CUtensorMap map_a, map_b;
  if (mode == MX_GROUPS_M) {
    MX_REQUIRE(N % 32 == 0, MX_ERR_UNSUPPORTED, "N = %lld is not a multiple of 32", (long long)N);
    MX_REQUIRE(K % 8 == 0, MX_ERR_UNSUPPORTED, "K = %lld is not a multiple of 8 (16-byte rows)", (long long)K);
    if (M == 0) return MX_OK;
    MX_REQUIRE(a && b && out, MX_ERR_ARG, "null operand");
    MX_TRY(make_map_bf16(&map_a, a, uint64_t(K), uint64_t(M), 0, kCtaM));
    MX_TRY(make_map_bf16(&map_b, b, uint64_t(N), uint64_t(K), uint64_t(G), 64));
    const int64_t pair_tiles_ub = (ceil_div(M, kPairM) + (offs ? G : 0)) * ceil_div(N, kBN);
    return launch_bf16_gemm<kGroupsM>(map_a, map_b, ha, pair_tiles_ub, st);
  }
  MX_REQUIRE(N % 32 == 0 && K % 32 == 0, MX_ERR_UNSUPPORTED, "N = %lld and K = %lld must be multiples of 32",
             (long long)N, (long long)K);
  MX_REQUIRE(out != nullptr, MX_ERR_ARG, "null output");
  if (M == 0) {
    cudaError_t e = cudaMemsetAsync(out, 0, size_t(G) * N * K * 2, st);
    MX_REQUIRE(e == cudaSuccess, MX_ERR_CUDA, "memset: %s", cudaGetErrorString(e));
    return MX_OK;
  }
  MX_REQUIRE(a && b, MX_ERR_ARG, "null operand");
  MX_TRY(make_map_bf16(&map_a, a, uint64_t(N), uint64_t(M), 0, 64));
  MX_TRY(make_map_bf16(&map_b, b, uint64_t(K), uint64_t(M), 0, 64));
  const int64_t pair_tiles_ub = int64_t(G) * ceil_div(N, kPairM) * ceil_div(K, kBN);
  return launch_bf16_gemm<kGroupsK>(map_a, map_b, ha, pair_tiles_ub, st);
}

extern "C" mx_status mx_dequant_dim0(const void* q, const void* s, int64_t G, int64_t R, int64_t C, void* out,
                                     void* stream) {
  MX_REQUIRE(G >= 1 && R >= 0 && C > 0, MX_ERR_ARG, "sizes must be G >= 1, R >= 0, C > 0");
  MX_REQUIRE(C % kBlock == 0, MX_ERR_UNSUPPORTED, "C = %lld is not a multiple of 32", (long long)C);
  const void* ptrs[3] = {q, s, out};
  for (const void* p : ptrs) MX_REQUIRE(aligned16(p), MX_ERR_ALIGN, "operand not 16-byte aligned");
  if (R == 0) return MX_OK;
  MX_REQUIRE(q && s && out, MX_ERR_ARG, "null operand");
  DequantArgs da;
  memset(&da, 0, sizeof(da));
  da.q = static_cast<const uint8_t*>(q);
  da.s = static_cast<const uint8_t*>(s);
  da.out = static_cast<__nv_bfloat16*>(out);
  da.rows_out = G * R;
  da.C = C;
  da.layout_rows = R;
  const int64_t items = da.rows_out * ceil_div(C / kBlock, 32) * 32;
  dequant_dim0_kernel<false><<<streaming_grid(dequant_dim0_kernel<false>, items, kDeqThreads), kDeqThreads, 0,
                               static_cast<cudaStream_t>(stream)>>>(da);
  return cuda_check("dequant launch");
}

extern "C" mx_status mx_dequant_dim0_grouped(const void* q, const void* s, const int32_t* offs, int32_t G, int64_t M,
                                             int64_t K, int64_t m_cap, void* out, void* stream) {
  MX_TRY(check_grouped(q, M, K, offs, G, m_cap));
  MX_REQUIRE(m_cap < (1ll << 31), MX_ERR_ARG, "m_cap must be < 2^31");
  MX_REQUIRE(aligned16(s) && aligned16(out), MX_ERR_ALIGN, "operand not 16-byte aligned");
  if (M == 0) return MX_OK;
  MX_REQUIRE(s && out, MX_ERR_ARG, "null operand");
  DequantArgs da;
  memset(&da, 0, sizeof(da));
  da.q = static_cast<const uint8_t*>(q);
  da.s = static_cast<const uint8_t*>(s);
  da.out = static_cast<__nv_bfloat16*>(out);
  da.rows_out = M;
  da.C = K;
  da.layout_rows = m_cap;
  da.offs = offs;
  da.G = G;
  da.m_cap = m_cap;
  const int64_t items = M * ceil_div(K / kBlock, 32) * 32;
  dequant_dim0_kernel<true><<<streaming_grid(dequant_dim0_kernel<true>, items, kDeqThreads), kDeqThreads, 0,
                              static_cast<cudaStream_t>(stream)>>>(da);
  return cuda_check("grouped dequant launch");
}

extern "C" mx_status mx_scales_unswizzle(const void* s, int64_t R, int64_t C32, void* out, void* stream) {
  MX_REQUIRE(R >= 0 && C32 > 0, MX_ERR_ARG, "sizes must be R >= 0, C32 > 0");
  MX_REQUIRE(aligned16(s), MX_ERR_ALIGN, "scales not 16-byte aligned");
  if (R == 0) return MX_OK;
  MX_REQUIRE(s && out, MX_ERR_ARG, "null operand");
  scales_unswizzle_kernel<<<streaming_grid(scales_unswizzle_kernel, R * C32, kDeqThreads), kDeqThreads, 0,
                            static_cast<cudaStream_t>(stream)>>>(static_cast<const uint8_t*>(s), R, C32,
                                                                 static_cast<uint8_t*>(out));
  return cuda_check("unswizzle launch");
}

// ---------------------------------------------------- failure detection ---
// One thread waits, through the bounded wait every GEMM pipeline uses, on a
// barrier that nothing ever arrives on; after the wait's time limit it gives
// up, sets the sticky timeout flag and returns.
namespace mx {
namespace {
__global__ void wait_timeout_selftest_kernel() {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_word;
  if (threadIdx.x == 0) {
    abort_word = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
    (void)mbar_wait(smem_u32(&bar), 0u, &abort_word);
  }
}
}  // namespace
}  // namespace mx

extern "C" mx_status mx_selftest_wait_timeout(void* stream) {
  wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  return cuda_check("selftest launch");
}
