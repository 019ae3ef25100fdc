/*
 * mx.h -- C ABI of libmx, the sm_100a (B200) MXFP8 training hot path.
 *
 * Operations (sources: five public pull-request pages on MXFP8 training):
 *   - block-32 casts of bf16 tensors to FP8 E4M3 elements with one E8M0
 *     power-of-two scale per 32 elements under the RCEIL rule ("shared RCEIL
 *     constant", torchtitan PR #5334, description): rowwise 1x32 ("dim0"),
 *     columnwise 32x1 ("dim1", ao "[moe training] Add backward_override to
 *     the MXFP8 grouped GEMM", Summary and Design notes), the fused
 *     rowwise+columnwise cast and 32x32 weight blocks (torchtitan PR #5334,
 *     description); scales are written straight into the blocked layout the
 *     block-scaled MMA reads, so no separate scale rearrangement pass is
 *     needed (same page);
 *   - the group pad path ("pad_token_groups_for_grouped_mm", ao
 *     backward_override PR, Known follow-ups; "pad/unpad" and "M-groups /
 *     K-groups scale rearrange" kernels, ao PR #4705 stack list);
 *   - the MXFP8 scaled grouped GEMM over an offsets array and its dgrad and
 *     wgrad (ao backward_override PR, Summary; ao PR #4705, description),
 *     and the bf16 grouped GEMMs, dequantization and scale unswizzle of the
 *     backward-override arms (ao backward_override PR, Design notes);
 *   - the MXFP8 linear forward / dgrad / wgrad (ao PR #4705, "MXFP8Linear
 *     training paths"), also as a training pair whose backward reuses the
 *     forward's casts, and a per-weight quantization cache keyed by the
 *     weight's version counter ("Cache quantized weights for full AC",
 *     prime-rl PR #3388, Overview).
 *
 * Conventions shared by every entry point
 *   - All pointers except host-side handles are DEVICE pointers owned by the
 *     caller; they must be 16-byte aligned (MX_ERR_ALIGN otherwise). Tensors
 *     are dense row-major with the last dimension contiguous; a strided or
 *     stride-0 view must be made contiguous by the caller first.
 *   - bf16 inputs are raw 16-bit bf16 values; E4M3 outputs are one byte per
 *     element ("fn" encoding: bias 7, max 448, no infinities); E8M0 scale
 *     bytes are b with value 2^(b-127).
 *   - Scale buffers use the blocked layout: a logical scale matrix S[R, C] is
 *     padded to R' = ceil(R/128)*128 rows and C' = ceil(C/4)*4 columns and
 *     stored as 128x4 tiles of 512 bytes, tile (r/128, c/4) at index
 *     (r/128)*(C'/4) + c/4, byte (r%32)*16 + ((r%128)/32)*4 + c%4 inside the
 *     tile. Pad bytes are written as 0x00. mx_scale_bytes() gives the size.
 *   - Every call is asynchronous and ordered on `stream` (a cudaStream_t; NULL
 *     is the legacy default stream). Argument errors are detected on the host
 *     before any launch and leave every buffer untouched. Errors found on the
 *     device (bad offsets, a pipeline wait that timed out) set a sticky device
 *     flag that mx_device_error() reads.
 *   - Nothing here allocates device memory except the weight cache, which owns
 *     the buffers it creates and frees them in mx_wcache_clear/destroy.
 *   - Non-finite inputs are outside the contract (their outputs are
 *     unspecified but the kernels stay in bounds).
 */
#ifndef MX_H_
#define MX_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MX_API __attribute__((visibility("default")))
#else
#define MX_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MX_OK = 0,
  MX_ERR_ARG = 1,          /* a size, count or pointer is invalid             */
  MX_ERR_ALIGN = 2,        /* a pointer is not 16-byte aligned                */
  MX_ERR_UNSUPPORTED = 3,  /* a geometry this library does not handle         */
  MX_ERR_CUDA = 4,         /* a CUDA runtime call failed                      */
  MX_ERR_TIMEOUT = 5,      /* a device-side pipeline wait gave up             */
  MX_ERR_DEVICE = 6        /* the device flagged invalid data (e.g. offsets)  */
} mx_status;

/* Human-readable reason of the last non-MX_OK status returned on this host
 * thread (empty string if none). The pointer stays valid until the next call. */
MX_API const char* mx_last_error(void);

/* Bytes of the blocked layout of a logical scale matrix S[rows, cols]:
 * ceil(rows/128)*128 * ceil(cols/4)*4. */
MX_API size_t mx_scale_bytes(int64_t rows, int64_t cols);

/* Upper bound of the padded row count of M tokens in `groups` groups when
 * every group is rounded up to a multiple of 128 rows:
 * floor((M + 127*groups) / 128) * 128. */
MX_API int64_t mx_padded_rows_capacity(int64_t m_total, int32_t groups);

/* Synchronizes `stream`, then returns MX_OK, MX_ERR_TIMEOUT or MX_ERR_DEVICE
 * according to the sticky device flag, and clears the flag. */
MX_API mx_status mx_device_error(void* stream);

/* ---------------------------------------------------------------- casts --
 * dim0 (rowwise, 1x32 along the contiguous axis; ao backward_override PR,
 * Design notes, "CuTe DSL 1x32 kernel"):
 *   x  bf16 [R, C]          q  E4M3 [R, C]          s  blocked(R, C/32)
 * R >= 0, C a positive multiple of 32. */
MX_API mx_status mx_cast_dim0(const void* x, int64_t R, int64_t C,
                       void* q, void* s, void* stream);

/* dim1 (columnwise, 32x1 down each column, stored transposed so that the
 * reduced axis is contiguous; ao backward_override PR, Summary, "dim1 cast"):
 *   x  bf16 [R, C]          qt E4M3 [C, R]          st blocked(C, R/32)
 * R a multiple of 32, C a positive multiple of 32. */
MX_API mx_status mx_cast_dim1(const void* x, int64_t R, int64_t C,
                       void* qt, void* st, void* stream);

/* Fused rowwise + columnwise cast from one read of x (torchtitan PR #5334,
 * description, "fused dense rowwise/columnwise cast"). Outputs are bitwise
 * those of mx_cast_dim0 and mx_cast_dim1. Same size rules as mx_cast_dim1. */
MX_API mx_status mx_cast_2d(const void* x, int64_t R, int64_t C,
                     void* q, void* s, void* qt, void* st, void* stream);

/* 32x32 weight cast (one scale per 32x32 tile; torchtitan PR #5334,
 * description and review thread, "32x32 RCEIL weight-scale policy"), for a
 * stack of G weights w bf16 [G, N, K] (G = 1 for a dense weight):
 *   q        E4M3 [G, N, K]
 *   s_fwd    G concatenated blocked(N, K/32) buffers, S_fwd[n, kb] = S[n/32, kb]
 *   qt       E4M3 [G, K, N] (the same codes transposed) or NULL; the dgrad
 *            does not need it (mx_grouped_mm mode MX_GROUPS_M_KN reads q
 *            itself with s_dgrad)
 *   s_dgrad  G concatenated blocked(K, N/32) buffers, S_dgrad[k, nb] = S[nb, k/32],
 *            or NULL
 * N and K positive multiples of 32. */
MX_API mx_status mx_cast_w32x32(const void* w, int64_t G, int64_t N, int64_t K,
                         void* q, void* s_fwd, void* qt, void* s_dgrad,
                         void* stream);

/* Scale rule selector of mx_cast_ex. RCEIL is the rule of every other entry
 * point; FLOOR (ao backward_override PR, Known follow-ups: the other scale
 * rule, reachable there but untested) is scale 2^(floor(log2 amax) - 8), with which scaled elements
 * can exceed 448 and saturate to +-448. */
#define MX_RCEIL 0
#define MX_FLOOR 1

/* Rowwise (dims = 1), columnwise (dims = 2) or both (dims = 3) cast under the
 * given scale rule; buffers and size rules as mx_cast_dim0 / mx_cast_dim1 /
 * mx_cast_2d (the outputs of an unused direction may be NULL). */
MX_API mx_status mx_cast_ex(const void* x, int64_t R, int64_t C, int32_t dims, int32_t rule,
                            void* q, void* s, void* qt, void* st, void* stream);

/* ------------------------------------------------------- group pad path --
 * offs: device int32 [G] cumulative group ends (non-decreasing, offs[G-1] ==
 * M). Group g occupies rows offs[g-1]..offs[g] of x (offs[-1] = 0) and is
 * placed at padded row p_g = sum_{h<g} ceil(size_h/128)*128. m_cap is the
 * row capacity of the padded outputs: a multiple of 128 that is at least the
 * padded total (mx_padded_rows_capacity() always is). Pad rows/tokens are
 * written as code 0 with scale byte 0. Offsets are read on the device only;
 * invalid ones set the device flag (MX_ERR_DEVICE). 1 <= G <= 1024.
 *
 * dim0 into padded rows:   x bf16 [M, K] -> q [m_cap, K], s blocked(m_cap, K/32)
 * dim1 per group (32-token blocks start at each group start, a group's last
 * partial block is completed with zeros):
 *                          x bf16 [M, K] -> qt [K, m_cap], st blocked(K, m_cap/32)
 * 2d: both from one read.  K a positive multiple of 32. */
MX_API mx_status mx_cast_dim0_grouped(const void* x, int64_t M, int64_t K,
                               const int32_t* offs, int32_t G, int64_t m_cap,
                               void* q, void* s, void* stream);
MX_API mx_status mx_cast_dim1_grouped(const void* x, int64_t M, int64_t K,
                               const int32_t* offs, int32_t G, int64_t m_cap,
                               void* qt, void* st, void* stream);
MX_API mx_status mx_cast_2d_grouped(const void* x, int64_t M, int64_t K,
                             const int32_t* offs, int32_t G, int64_t m_cap,
                             void* q, void* s, void* qt, void* st, void* stream);

/* The MXFP8 dispatch of expert parallelism as one kernel ("Cache quantized
 * weights for full AC", prime-rl PR #3388, Overview: enable_a2a): the dim0
 * cast into padded groups above, with each group's padded rows written to
 * their own destination instead of one buffer -- the receiving rank's
 * buffer, which may be another GPU's memory mapped into this process (a peer
 * or symmetric-memory mapping; written with plain stores, no TMA).
 *   dst_q[g]  HOST array of G device pointers: group g's first padded row of
 *             codes; its rows follow at K bytes each (ceil(size_g/128)*128 rows).
 *   dst_s[g]  HOST array of G device pointers: group g's first 128-row band of
 *             blocked scales (mx_scale_bytes(128, K/32) bytes per band).
 * Every pointer must be non-NULL and 16-byte aligned (checked on the host;
 * an empty group's destination is never written). Bytes written per group
 * are exactly those its rows occupy in mx_cast_dim0_grouped's outputs; the
 * pad capacity past the last group writes nothing. The call ends with a
 * system-scope fence (a one-thread kernel after the cast, on the same
 * stream): once that is seen complete (e.g. through a collective issued
 * after the call on the same stream), other GPUs read the stores. */
MX_API mx_status mx_cast_dim0_grouped_scatter(const void* x, int64_t M, int64_t K,
                                              const int32_t* offs, int32_t G, int64_t m_cap,
                                              void* const* dst_q, void* const* dst_s, void* stream);

/* The fused grouped cast (rowwise and columnwise from one read, as
 * mx_cast_2d_grouped) with each group's outputs written to its own
 * destination: the backward dispatch of expert parallelism (prime-rl PR
 * #3388, Overview: enable_a2a), each token group's gradient cast both ways
 * straight into the buffers of the rank that holds its expert, exactly as
 * that rank's own mx_cast_2d_grouped of the received rows would write them
 * (the 32-token column blocks start at each group start on both sides).
 *   dst_q[g], dst_s[g]  as mx_cast_dim0_grouped_scatter.
 *   dst_qt[g]  HOST array of G device pointers: group g's first padded token
 *              column in the destination's columnwise codes [K, dst_cap[g]]
 *              (row stride dst_cap[g] bytes).
 *   dst_st[g]  HOST array of G device pointers: group g's first 512-byte tile
 *              in the destination's blocked(K, dst_cap[g]/32) scales.
 *   dst_cap[g] HOST array of G padded capacities of the destinations (each a
 *              positive multiple of 128 below 2^31).
 * G at most 512. Every pointer non-NULL and 16-byte aligned (checked on the
 * host; an empty group's destinations are never written). Bytes written per
 * group: its rows' codes and scale bands as in the rowwise scatter, and its
 * columns' codes and scale tiles as in mx_cast_2d_grouped's columnwise
 * outputs. The call ends with a system-scope fence (a one-thread kernel after
 * the cast, on the same stream). */
MX_API mx_status mx_cast_2d_grouped_scatter(const void* x, int64_t M, int64_t K,
                                            const int32_t* offs, int32_t G, int64_t m_cap,
                                            void* const* dst_q, void* const* dst_s,
                                            void* const* dst_qt, void* const* dst_st,
                                            const int64_t* dst_cap, void* stream);

/* -------------------------------------------------- scaled grouped GEMM --
 * The MXFP8 scaled grouped GEMM over an offsets array (ao "[moe training]
 * Add backward_override to the MXFP8 grouped GEMM", Summary: forward, dgrad
 * and wgrad of the grouped GEMM; ao PR #4705, "MXFP8 MoE grouped-mm").
 * Operands are E4M3 codes with blocked E8M0 scales, both K-major (the
 * contraction axis contiguous), as the casts above produce them. fp32
 * accumulation on the tensor cores, bf16 output (round to nearest even).
 * Deterministic: no split-K, no atomics.
 *
 * mode MX_GROUPS_M (forward and dgrad; groups split the rows):
 *   out[start_g + i, :] = sum_k A[p_g + i, k] B[g, :, k]   for i < size_g
 *   a_q [rows_a, K], a_s blocked(rows_a, K/32)   rows_a = m_cap (padded rows
 *       from mx_cast_dim0_grouped) or M when offs == NULL (dense, G = 1)
 *   b_q [G, N, K],   b_s G concatenated blocked(N, K/32) buffers
 *   out bf16 [M, N]; rows of the padded layout that are padding are not read
 *       into the output (the unpad is fused into the store).
 * mode MX_GROUPS_M_KN (dgrad straight from the forward's weight codes): as
 *   MX_GROUPS_M with B codes stored [G, K, N] (N contiguous; read by the MMA
 *   as an MN-major operand, so no transposed copy is needed) and b_s G
 *   concatenated blocked(N, K/32) buffers, i.e.
 *   out[start_g + i, n] = sum_k A[p_g + i, k] B[g, k, n].
 *   For dX = dY W of a weight W [G, Nw, Kw] cast 32x32: B = its codes q,
 *   b_s = its s_dgrad view, N = Kw, K = Nw.
 * mode MX_GROUPS_K (wgrad; groups split the contraction, "K groups"):
 *   out[g, n, k] = sum over the tokens t of group g of A[n, t] B[k, t]
 *   a_q [N, L], a_s blocked(N, L/32); b_q [K, L], b_s blocked(K, L/32) with
 *       L = m_cap (padded token columns from mx_cast_dim1_grouped) or M when
 *       offs == NULL (dense, G = 1, M a multiple of 32)
 *   out bf16 [G, N, K]; an empty group gives exact zeros.
 * Sizes: N and K multiples of 32 in every mode, each below 2^31. Sizes that
 * are not multiples of the 256x256 output tile or of the 128-deep K step
 * take the pad path of the unaligned geometry (torchtitan PR #5334, review
 * thread: the 576-wide output gradient): operand tiles past the tensor are
 * read as zero codes, whose blocked scale bytes are 0x00, so they add
 * nothing; output rows and columns past the tensor are never written.
 * offs: device int32 [G] cumulative ends (see the pad path above) or NULL.
 * Invalid offsets set the device flag and leave the output unwritten. */
#define MX_GROUPS_M 0
#define MX_GROUPS_K 1
#define MX_GROUPS_M_KN 2
MX_API mx_status mx_grouped_mm(const void* a_q, const void* a_s, const void* b_q, const void* b_s,
                               const int32_t* offs, int32_t G, int32_t mode, void* out,
                               int64_t M, int64_t N, int64_t K, int64_t m_cap, void* stream);

/* The grouped GEMM whose G groups cycle over E experts: group g uses expert
 * g % E. This is the layout in which an expert-parallel all-to-all delivers
 * tokens to the rank that holds E experts -- source rank major, expert minor
 * ("MXFP8 all-to-all", prime-rl PR #3388, Overview, enable_a2a; ao PR #4705,
 * the expert-parallel pipeline benchmark). E divides G; E == G is exactly
 * mx_grouped_mm. Operands and sizes as mx_grouped_mm, except:
 *   MX_GROUPS_M / MX_GROUPS_M_KN: b_q and b_s hold E experts (not G);
 *   MX_GROUPS_K: out bf16 [E, N, K], out[e] sums the token groups
 *     e, e + E, e + 2E, ... (an expert with only empty groups gives zeros).
 * Without offsets G = E = 1. */
MX_API mx_status mx_grouped_mm_experts(const void* a_q, const void* a_s, const void* b_q, const void* b_s,
                                       const int32_t* offs, int32_t G, int32_t E, int32_t mode, void* out,
                                       int64_t M, int64_t N, int64_t K, int64_t m_cap, void* stream);

/* The M-group modes above (MX_GROUPS_M, MX_GROUPS_M_KN; offsets required)
 * with each group's output rows at their own destination: row i of group g
 * (0 <= i < size_g) is written at out_rows[g] + i*N (bf16 elements) instead
 * of at out + (start_g + i)*N. This is the combine of expert parallelism
 * fused into the GEMM ("Cache quantized weights for full AC", prime-rl PR
 * #3388, Overview: enable_a2a): each expert output row is stored straight
 * into the rank that sent the token, tile by tile as the GEMM runs, instead
 * of a bf16 all-to-all afterwards. out_rows is a HOST array of G device
 * pointers, each non-NULL and 16-byte aligned (checked on the host; an empty
 * group's destination is never written); a destination may be another GPU's
 * memory mapped into this process (plain stores, no TMA). Bytes written per
 * group: size_g rows of N bf16; nothing else is written. The kernel ends with
 * a system-scope fence: once it is seen complete (e.g. through a collective
 * issued after it on the same stream), other GPUs read the rows. The other
 * arguments are those of mx_grouped_mm_experts. */
MX_API mx_status mx_grouped_mm_experts_to_rows(const void* a_q, const void* a_s, const void* b_q,
                                               const void* b_s, const int32_t* offs, int32_t G, int32_t E,
                                               int32_t mode, void* const* out_rows, int64_t M, int64_t N,
                                               int64_t K, int64_t m_cap, void* stream);

/* ------------------------------------------- backward-override arms -----
 * ao "[moe training] Add backward_override to the MXFP8 grouped GEMM", Design
 * notes: the "high_precision" arm computes dgrad and wgrad of the grouped GEMM
 * with two plain bf16 grouped GEMMs over the saved, unpadded bf16 operands;
 * the "dequantized" arm runs the same two GEMMs on the forward's quantized
 * operands turned back into bf16 (it needs logical scales, and the page notes
 * that no kernel turned blocked scales back into logical ones;
 * mx_scales_unswizzle does).
 *
 * bf16 grouped GEMM, fp32 accumulation on the tensor cores, bf16 output
 * (round to nearest even); deterministic (no split-K, no atomics). Groups are
 * the UNPADDED rows offs[g-1]..offs[g] (any sizes, empty groups allowed;
 * offs as for the pad path, offs[G-1] == M; NULL = one group, G = 1). No
 * operand is copied or transposed.
 * mode MX_GROUPS_M (dgrad):  out[rows of g, :] = a[rows of g, :] @ b[g]
 *   a bf16 [M, K], b bf16 [G, K, N], out bf16 [M, N].
 *   N a multiple of 32, K a positive multiple of 8.
 * mode MX_GROUPS_K (wgrad):  out[g] = a[rows of g, :]^T @ b[rows of g, :]
 *   a bf16 [M, N], b bf16 [M, K], out bf16 [G, N, K]; an empty group gives
 *   exact zeros. N and K multiples of 32.
 * M, N, K < 2^31. Invalid offsets set the device flag and leave the output
 * unwritten. */
MX_API mx_status mx_grouped_mm_bf16(const void* a, const void* b, const int32_t* offs, int32_t G,
                                    int32_t mode, void* out, int64_t M, int64_t N, int64_t K,
                                    void* stream);

/* Dequantization of rowwise-scaled codes to bf16:
 *   out[i, r, c] = bf16(e4m3(q[i, r, c]) * 2^(S_i[r, c/32] - 127))
 * rounded to nearest even (exact unless |value| < 2^-133 or the value
 * overflows bf16); a NaN code or scale byte 255 gives NaN.
 *   q E4M3 [G, R, C]; s G concatenated blocked(R, C/32) buffers (a dim0 cast
 *   with G = 1, or the s_fwd output of mx_cast_w32x32); out bf16 [G, R, C].
 * G >= 1, R >= 0, C a positive multiple of 32. */
MX_API mx_status mx_dequant_dim0(const void* q, const void* s, int64_t G, int64_t R, int64_t C,
                                 void* out, void* stream);

/* The same for the padded rows of mx_cast_dim0_grouped, gathered back to the
 * unpadded order: out[start_g + i, :] = dequant(row p_g + i).
 *   q [m_cap, K], s blocked(m_cap, K/32) -> out bf16 [M, K].
 * Size rules and offsets as mx_cast_dim0_grouped. */
MX_API mx_status mx_dequant_dim0_grouped(const void* q, const void* s, const int32_t* offs, int32_t G,
                                         int64_t M, int64_t K, int64_t m_cap, void* out, void* stream);

/* Logical scales from the blocked layout: out uint8 [R, C32] row-major,
 * out[r, c] = S[r, c] of the blocked buffer s = blocked(R, C32). */
MX_API mx_status mx_scales_unswizzle(const void* s, int64_t R, int64_t C32, void* out, void* stream);

/* ------------------------------------------------------ MXFP8 linear -----
 * Dense MXFP8 linear (ao PR #4705, "MXFP8Linear training paths"; torchtitan
 * PR #5334, description: one entry point for dense and grouped MXFP8 linears):
 *   forward  y  [M, N] = x [M, K] w [N, K]^T   x cast 1x32 (dim0), w 32x32
 *   backward dx [M, K] = dy [M, N] w           dy cast 1x32 along N
 *            dw [N, K] = dy^T x                dy and x cast 32x1 along M
 * dy is cast once by the fused rowwise+columnwise cast. The casts of one
 * call (the weight's, when it is quantized, with x's in the forward; with
 * dy's and x's in the backward) go out as one kernel launch, followed by the
 * GEMMs. All tensors bf16, row-major. M, N and K multiples of 32 (N or K off
 * the 256-wide tile, such as 576, take the GEMM's pad path).
 * ws: caller-owned device workspace of at least mx_linear_ws_bytes(M, N, K)
 * bytes (holds the quantized activations and gradients and, without a
 * cache, the quantized weight); it must stay untouched until the call's
 * work on `stream` completes.
 *
 * Weight cache ("Cache quantized weights for full AC", prime-rl PR #3388,
 * Overview): with cache != NULL the 32x32 quantization of w is kept in
 * device memory owned by the cache, keyed by (w address, N, K) and reused
 * while w_version is unchanged; a changed version re-quantizes in place.
 * Results are bitwise identical with and without a hit.
 * The key is an address, and an allocator may hand a freed weight's address
 * to a new tensor whose own update counter starts where the old one's did;
 * a hit would then return the old weight's codes. So w_version must change
 * whenever the bytes at w change OR w names a different tensor: a caller
 * either folds a per-tensor identity that is never reused into w_version,
 * or calls mx_wcache_evict(cache, w) when the tensor at w is freed (before
 * its memory can be reused). The Python binding does both.
 * mx_wcache_evict() unbinds the entries of address w without freeing them
 * (no device synchronization; a later miss of the same N, K reuses the
 * buffer, stream-ordered after the work already issued on that call's
 * stream; work on other streams that still reads the entry must be ordered
 * before that miss). Call it after a weight's backward to drop the entry
 * ("clear the cache after backward", same page). mx_wcache_clear() frees
 * every entry, bound or not (it synchronizes the device). The cache is
 * thread-safe; an entry must not be cleared while work that reads it is in
 * flight. mx_wcache_stats() counts hits, misses and bound entries. */
typedef struct mx_wcache mx_wcache;
MX_API mx_wcache* mx_wcache_create(void);
MX_API void mx_wcache_evict(mx_wcache* cache, const void* w);
MX_API void mx_wcache_clear(mx_wcache* cache);
MX_API void mx_wcache_destroy(mx_wcache* cache);
MX_API mx_status mx_wcache_stats(mx_wcache* cache, int64_t* hits, int64_t* misses, int64_t* entries);
MX_API size_t mx_linear_ws_bytes(int64_t M, int64_t N, int64_t K);
MX_API mx_status mx_linear_fwd(const void* x, const void* w, int64_t M, int64_t N, int64_t K,
                               mx_wcache* cache, uint64_t w_version, void* y,
                               void* ws, size_t ws_bytes, void* stream);
MX_API mx_status mx_linear_bwd(const void* dy, const void* x, const void* w,
                               int64_t M, int64_t N, int64_t K,
                               mx_wcache* cache, uint64_t w_version, void* dx, void* dw,
                               void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------ linear training pair -----
 * The same linear for a training step whose backward follows its forward:
 * the forward keeps, in the workspace, what the backward would otherwise
 * re-compute from x and w. The 32x32 weight cast writes both scale views at
 * once (ao PR #4705, "MXFP8Linear training paths"), so the forward's
 * quantization of w serves the dgrad; and x's columnwise cast comes out of
 * the forward's single read of x (the fused rowwise + columnwise cast).
 *   mx_linear_fwd_train     y as mx_linear_fwd; x cast rowwise and
 *                           columnwise in one launch with the weight's cast;
 *                           x's columnwise codes and scales, and (without a
 *                           cache) w's quantization, stay in ws.
 *   mx_linear_bwd_after_fwd dx, dw as mx_linear_bwd, casting only dy: x's
 *                           columnwise cast and w's quantization are the
 *                           forward's (with a cache: the cache entry, re-cast
 *                           from w only on a miss). x is not read.
 * Results are bitwise those of mx_linear_fwd + mx_linear_bwd on the same
 * x, w and dy. Contract: the backward runs on the workspace of the forward
 * whose step it completes, with nothing else using that workspace in
 * between, the same cache argument (NULL or not), and -- when a cache is
 * given -- w's bytes unchanged since that forward. Without a cache, w's bytes
 * may change in between: the backward uses the forward's quantization, as
 * the gradient of that forward's product. x may be freed or overwritten
 * once the forward's work on `stream` is done.
 * ws: caller-owned, at least mx_linear_train_ws_bytes(M, N, K) bytes -- x's
 * columnwise cast, then the larger of x's rowwise and dy's casts, then w's
 * quantization; more than mx_linear_ws_bytes when x's rowwise cast takes more
 * bytes than dy's two casts (K > 2N, up to scale padding), because the forward
 * holds both casts of x at once. Size rules and errors as mx_linear_fwd and
 * mx_linear_bwd (a workspace below mx_linear_train_ws_bytes: MX_ERR_ARG). */
MX_API size_t mx_linear_train_ws_bytes(int64_t M, int64_t N, int64_t K);
MX_API mx_status mx_linear_fwd_train(const void* x, const void* w, int64_t M, int64_t N, int64_t K,
                                     mx_wcache* cache, uint64_t w_version, void* y,
                                     void* ws, size_t ws_bytes, void* stream);
MX_API mx_status mx_linear_bwd_after_fwd(const void* dy, const void* w, int64_t M, int64_t N, int64_t K,
                                         mx_wcache* cache, uint64_t w_version, void* dx, void* dw,
                                         void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------- linear forward, no allocation --
 * No counterpart on the source pages: an addition for callers that cannot
 * allocate device memory and so cannot pass a workspace -- a plain C host
 * program linking this library without a device allocator of its own, or a
 * plugin running inside a runtime that reserves all device memory up front
 * and forbids further cudaMalloc calls (which can also synchronise the
 * device).
 *
 * Computes exactly what mx_linear_fwd computes without a cache
 * (y [M, N] = x [M, K] w [N, K]^T, x cast 1x32, w cast 32x32), but keeps
 * its scratch -- the quantized x and w and their scales,
 * ceil256(M*K) + ceil256(mx_scale_bytes(M, K/32)) + ceil256(N*K)
 * + ceil256(mx_scale_bytes(N, K/32)) bytes -- in a fixed device array of
 * MX_LINEAR_NOALLOC_SCRATCH_BYTES inside the library. Every GPU that loads
 * the library holds that array until the process exits. Sizes that need
 * more are rejected with MX_ERR_UNSUPPORTED and a message naming both
 * sizes. It calls no cudaMalloc, cudaFree or other allocating routine.
 *
 * The first call on a device looks up the array's device address on that
 * device (cudaGetSymbolAddress); make that first call before any stream
 * capture. The address is kept for the life of the process, so a caller
 * must not reset the device (cudaDeviceReset) after its first call. Every call shares the one array and leaves its contents behind
 * (each call rewrites every byte it reads, so nothing is cleared): calls
 * whose work overlaps on the GPU (other streams, other host threads) race
 * on it, so order them. Same size rules as mx_linear_fwd. */
#define MX_LINEAR_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
MX_API mx_status mx_linear_fwd_noalloc(const void* x, const void* w, int64_t M, int64_t N, int64_t K,
                                       void* y, void* stream);

/* ---------------------------------------------------- failure detection --
 * No counterpart on the source pages: a diagnostic of the library's own
 * failure detection. It launches one thread that waits, through the same
 * bounded wait the GEMM pipelines use, on a barrier nothing ever arrives
 * on; after that wait's 2-second limit the thread gives up, sets the sticky
 * device flag and returns. mx_device_error(stream) then reports
 * MX_ERR_TIMEOUT (and clears the flag); the context stays usable. */
MX_API mx_status mx_selftest_wait_timeout(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MX_H_ */
