"""Plain CPU oracle of the MXFP8 training hot path (numpy, float64).

TEST INFRASTRUCTURE ONLY: nothing in the product path imports it. It shares
no code, table or constant generator with the CUDA library; the only module
both sides use is the seeded input generator, which holds none of the
arithmetic below.

What it computes, and where each step comes from
------------------------------------------------
* MX block format: FP8 E4M3 elements that share one E8M0 power-of-two scale
  per block of 32 values ("blocked E8M0 scales", torchtitan PR #5334,
  description; "1x32" casts, ao PR "[moe training] Add backward_override to
  the MXFP8 grouped GEMM", Design notes).
* RCEIL scale rule ("shared RCEIL constant", "32x32 RCEIL weight-scale
  policy", torchtitan PR #5334, description and review thread): the scale of a
  block is the smallest power of two 2**e with 448 * 2**e >= amax, stored as
  the E8M0 byte b = e + 127 clamped to [0, 254]. 448 is the largest finite
  E4M3 value. A block whose amax is 0 gets b = 0.
* FLOOR scale rule (ao backward_override PR, Known follow-ups: the other
  scale rule, reachable but untested there): scale 2**(floor(log2(amax)) - 8); saturation to 448 is live.
* Element cast: q = round-to-nearest-even, saturating E4M3 encoding of
  x * 2**(127 - b), with the sign of zero kept.
* Block geometry: rowwise "dim0" (1x32 along the contiguous axis), columnwise
  "dim1" (32x1 down the columns, stored transposed), fused row+column (both
  from one read; "fused dense rowwise/columnwise cast", torchtitan PR #5334),
  and square 32x32 weight blocks ("32x32 RCEIL weight-scale policy", same
  page), which let one quantized weight serve both the forward GEMM and the
  dgrad GEMM.
* Blocked ("swizzled") scale layout: the pages name it ("swizzled layouts are
  directly output", torchtitan PR #5334) but do not define it. Reading taken:
  the layout the Blackwell block-scaled MMA consumes -- 128-row x 4-column
  tiles of 512 bytes, tile-major with the column tiles of a row band
  contiguous, and inside a tile byte (r % 32) * 16 + (r // 32) * 4 + c.
  Padding bytes are 0x00.
* Grouped operands and the pad path ("pad_token_groups_for_grouped_mm" and
  padded offsets, ao backward_override PR, Known follow-ups; "pad/unpad" and
  "M-groups / K-groups scale rearrange" kernels, ao PR #4705 stack list): each
  token group is placed at a row offset that is a multiple of 128, so that
  every 128-row scale tile belongs to one group; pad rows are zero.
* Scaled grouped GEMM over an offsets array (ao backward_override PR,
  Summary): Y[rows of group g] = deq(X_g) @ deq(W_g)^T; dgrad
  dX_g = dY_g @ W_g; wgrad dW_g = dY_g^T @ X_g, an empty group giving
  dW_g = 0. Computed here in float64 over the dequantized operands.
* MXFP8 linear forward / dgrad / wgrad ("MXFP8Linear training paths", ao PR
  #4705) composed from the casts above at one group.
* Backward-override arms (ao backward_override PR, Design notes): the
  high-precision arm's two bf16 grouped GEMMs over unpadded groups, the
  dequantized arm's dequantization of the forward's codes to bf16 (round to
  nearest even), and the grouped dequant that gathers padded rows back; and
  wgrad_with_hp (same PR, Known follow-ups: the existing knob that
  "high_precision" extends to both gradients), the MXFP8 dgrad beside the
  bf16 wgrad.
* Expert parallelism with the MXFP8 all-to-all ("Cache quantized weights for
  full AC", prime-rl PR #3388, Overview: enable_a2a; ao PR #4705, the
  expert-parallel pipeline benchmark): the expert-side forward and backward
  over received groups (source rank, local expert), group g served by local
  expert g % E, the wgrad's activations cast columnwise from their
  dequantized values, dW of an expert summed over its groups.

Where the pages are silent, the readings taken are listed in the repository's
design notes; each is restated beside the function that depends on it.
"""
from __future__ import annotations

import numpy as np

BLOCK = 32            # elements that share one scale
E4M3_MAX = 448.0      # largest finite E4M3 value
E8M0_BIAS = 127
E8M0_MAX_FINITE = 254  # 255 is the E8M0 NaN encoding
SCALE_TILE_ROWS = 128
SCALE_TILE_COLS = 4
GROUP_ALIGN = 128


def ceil_to(x, a):
    return ((x + a - 1) // a) * a


# --------------------------------------------------------------------------
# bf16 inputs are carried as their uint16 bit patterns
# --------------------------------------------------------------------------
def bf16_to_f64(bits) -> np.ndarray:
    """Exact value of each bf16 bit pattern, as float64."""
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# FP8 E4M3 ("fn" variant: bias 7, no infinities, NaN = S.1111.111)
# --------------------------------------------------------------------------
def e4m3_decode(codes) -> np.ndarray:
    """Value of each E4M3 code from the format definition (float64)."""
    c = np.asarray(codes).astype(np.int64)
    sign = c >> 7
    exp = (c >> 3) & 0xF
    man = c & 0x7
    subnormal = man / 8.0 * 2.0 ** (1 - 7)
    normal = (1.0 + man / 8.0) * np.exp2(exp - 7.0)
    mag = np.where(exp == 0, subnormal, normal)
    mag = np.where((exp == 0xF) & (man == 0x7), np.nan, mag)
    return np.where(sign == 1, -mag, mag)


# The 127 finite non-negative codes 0x00..0x7E; their values increase with the
# code, so nearest-value search is a sorted search.
_POS_CODES = np.arange(0x7F, dtype=np.int64)
_POS_VALUES = e4m3_decode(_POS_CODES)


def e4m3_encode(v) -> np.ndarray:
    """Round-to-nearest-even E4M3 code of each float64 value.

    Saturates to +-448 (the "satfinite" behaviour), keeps the sign of zero
    (a negative value that rounds to zero gives 0x80) and breaks ties toward
    the code whose mantissa is even. Inputs must be finite.
    """
    v = np.asarray(v, dtype=np.float64)
    if not np.all(np.isfinite(v)):
        raise ValueError("e4m3_encode: non-finite input is outside the contract")
    a = np.minimum(np.abs(v), E4M3_MAX)
    hi = np.searchsorted(_POS_VALUES, a, side="left")   # first value >= a
    hi = np.minimum(hi, len(_POS_VALUES) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _POS_VALUES[lo]
    d_hi = _POS_VALUES[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    sign = np.signbit(v).astype(np.int64)
    return (code | (sign << 7)).astype(np.uint8)


# --------------------------------------------------------------------------
# E8M0 scale under RCEIL
# --------------------------------------------------------------------------
def rceil_e8m0(amax) -> np.ndarray:
    """E8M0 byte of the RCEIL scale of blocks with the given amax.

    b = clamp(e + 127, 0, 254) with e the smallest integer such that
    448 * 2**e >= amax (i.e. e = ceil(log2(amax / 448)) in exact arithmetic).
    amax == 0 gives b = 0 (the all-zero block; reading: the pages are silent,
    the exact formula gives -inf before the clamp).

    The search starts from a float64 log2 estimate and is then settled with
    exact comparisons (448 * 2**e is exact in float64), so the result is the
    exact minimum whatever the rounding of log2.
    """
    amax = np.asarray(amax, dtype=np.float64)
    if np.any(~np.isfinite(amax)) or np.any(amax < 0):
        raise ValueError("rceil_e8m0: amax must be finite and non-negative")
    b = np.zeros(amax.shape, dtype=np.int64)
    nz = amax > 0
    if np.any(nz):
        a = amax[nz]
        e = np.ceil(np.log2(a / E4M3_MAX)).astype(np.int64)
        for _ in range(4):   # each pass moves e by at most one step
            too_big = np.ldexp(E4M3_MAX, e - 1) >= a
            e = np.where(too_big, e - 1, e)
            too_small = np.ldexp(E4M3_MAX, e) < a
            e = np.where(too_small, e + 1, e)
        assert np.all(np.ldexp(E4M3_MAX, e) >= a)
        assert np.all(np.ldexp(E4M3_MAX, e - 1) < a)
        b[nz] = np.clip(e + E8M0_BIAS, 0, E8M0_MAX_FINITE)
    return b.astype(np.uint8)


def floor_e8m0(amax) -> np.ndarray:
    """E8M0 byte of the FLOOR scale of blocks with the given amax.

    FLOOR is the other scale rule the ao backward_override page names (Known
    follow-ups: it can be selected there but has no parity test). Reading: the OCP MX rule,
    scale = 2**(floor(log2(amax)) - 8), 8 being the exponent of the largest
    power of two representable in E4M3 (256 <= 448 < 512); b = that exponent
    + 127 clamped to [0, 254]; amax == 0 gives b = 0. Scaled elements can then
    reach up to 511.x and saturate to 448.

    Computed exactly: the largest integer f with 2**f <= amax.
    """
    amax = np.asarray(amax, dtype=np.float64)
    if np.any(~np.isfinite(amax)) or np.any(amax < 0):
        raise ValueError("floor_e8m0: amax must be finite and non-negative")
    b = np.zeros(amax.shape, dtype=np.int64)
    nz = amax > 0
    if np.any(nz):
        a = amax[nz]
        f = np.floor(np.log2(a)).astype(np.int64)
        for _ in range(4):   # settle with exact comparisons
            f = np.where(np.ldexp(1.0, f) > a, f - 1, f)
            f = np.where(np.ldexp(1.0, f + 1) <= a, f + 1, f)
        assert np.all(np.ldexp(1.0, f) <= a) and np.all(np.ldexp(1.0, f + 1) > a)
        b[nz] = np.clip(f - 8 + E8M0_BIAS, 0, E8M0_MAX_FINITE)
    return b.astype(np.uint8)


SCALE_RULES = {"rceil": rceil_e8m0, "floor": floor_e8m0}


def e8m0_to_f64(b) -> np.ndarray:
    """Value 2**(b - 127) of an E8M0 byte (b = 255, NaN, never produced here)."""
    return np.exp2(np.asarray(b).astype(np.float64) - E8M0_BIAS)


def quantize_blocks(xf, axis=-1, rule="rceil"):
    """Quantize float64 blocks whose 32 elements lie along ``axis``.

    Returns (q, b): q has the shape of xf (uint8 E4M3 codes), b has ``axis``
    removed (uint8 E8M0 bytes). ``rule`` is "rceil" (default) or "floor".
    """
    xf = np.asarray(xf, dtype=np.float64)
    if xf.shape[axis] != BLOCK:
        raise ValueError("quantize_blocks: block axis must hold 32 elements")
    amax = np.max(np.abs(xf), axis=axis)
    b = SCALE_RULES[rule](amax)
    inv_scale = np.expand_dims(np.exp2(E8M0_BIAS - b.astype(np.float64)), axis)
    q = e4m3_encode(xf * inv_scale)      # exact: scaling by a power of two
    return q, b


# --------------------------------------------------------------------------
# The four casts (logical scales; the blocked layout is applied separately)
# --------------------------------------------------------------------------
def cast_dim0(x_bits, rule="rceil"):
    """Rowwise 1x32 cast of bf16 X[R, C] -> (Q[R, C], S[R, C/32])."""
    x_bits = np.asarray(x_bits, dtype=np.uint16)
    R, C = x_bits.shape
    if C % BLOCK:
        raise ValueError("cast_dim0: the row length must be a multiple of 32")
    xf = bf16_to_f64(x_bits).reshape(R, C // BLOCK, BLOCK)
    q, b = quantize_blocks(xf, axis=-1, rule=rule)
    return q.reshape(R, C), b


def cast_dim1(x_bits, rule="rceil"):
    """Columnwise 32x1 cast of bf16 X[R, C] -> (Q^T[C, R], S[C, R/32]).

    Blocks are X[32i:32i+32, c]; the output is stored transposed so that the
    reduced axis is contiguous.
    """
    x_bits = np.asarray(x_bits, dtype=np.uint16)
    R, C = x_bits.shape
    if R % BLOCK:
        raise ValueError("cast_dim1: the column length must be a multiple of 32")
    xf = bf16_to_f64(x_bits).reshape(R // BLOCK, BLOCK, C)   # [block, row-in-block, col]
    q, b = quantize_blocks(xf, axis=1, rule=rule)             # q [R/32, 32, C], b [R/32, C]
    return np.ascontiguousarray(q.reshape(R, C).T), np.ascontiguousarray(b.T)


def cast_2d(x_bits, rule="rceil"):
    """Fused rowwise + columnwise cast: exactly the pair (dim0, dim1)."""
    return cast_dim0(x_bits, rule), cast_dim1(x_bits, rule)


def cast_32x32(w_bits):
    """Square-block cast of bf16 W[..., N, K] -> (Q[..., N, K], S[..., N/32, K/32]).

    One scale per 32x32 tile; stacks [G, N, K] are cast per expert (tiles
    never cross experts).
    """
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    *lead, N, K = w_bits.shape
    if N % BLOCK or K % BLOCK:
        raise ValueError("cast_32x32: both matrix dims must be multiples of 32")
    xf = bf16_to_f64(w_bits).reshape(*lead, N // BLOCK, BLOCK, K // BLOCK, BLOCK)
    amax = np.max(np.abs(xf), axis=(-3, -1))                  # [..., N/32, K/32]
    b = rceil_e8m0(amax)
    inv_scale = np.exp2(E8M0_BIAS - b.astype(np.float64))[..., :, None, :, None]
    q = e4m3_encode(xf * inv_scale)
    return q.reshape(*lead, N, K), b


def w32_scale_views(s_tile):
    """The two per-row scale views of 32x32 tile scales S[..., N/32, K/32].

    S_fwd[n, kb] = S[n // 32, kb] scales W[N, K] along K (forward GEMM);
    S_dgrad[k, nb] = S[nb, k // 32] scales W^T[K, N] along N (dgrad GEMM).
    """
    s_tile = np.asarray(s_tile)
    s_fwd = np.repeat(s_tile, BLOCK, axis=-2)
    s_dgrad = np.repeat(np.swapaxes(s_tile, -1, -2), BLOCK, axis=-2)
    return s_fwd, s_dgrad


# --------------------------------------------------------------------------
# Blocked (swizzled) scale layout
# --------------------------------------------------------------------------
def blocked_scale_bytes(rows, cols):
    """Size of the blocked layout of a logical scale matrix S[rows, cols]."""
    return ceil_to(rows, SCALE_TILE_ROWS) * ceil_to(cols, SCALE_TILE_COLS)


def blocked_offset(r, c, cols):
    """Byte offset of logical scale S[r, c] in the blocked layout.

    Tiles of 128 rows x 4 columns hold 512 bytes; tile (r//128, c//4) sits at
    index (r//128) * ceil(cols/4) + c//4; inside a tile the byte is
    (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4.
    """
    r = np.asarray(r, dtype=np.int64)
    c = np.asarray(c, dtype=np.int64)
    col_tiles = ceil_to(cols, SCALE_TILE_COLS) // SCALE_TILE_COLS
    tile = (r // SCALE_TILE_ROWS) * col_tiles + (c // SCALE_TILE_COLS)
    rr = r % SCALE_TILE_ROWS
    return tile * 512 + (rr % 32) * 16 + (rr // 32) * 4 + (c % SCALE_TILE_COLS)


def swizzle(s):
    """Logical scales S[R, C] -> blocked byte buffer (pad bytes 0x00)."""
    s = np.asarray(s, dtype=np.uint8)
    R, C = s.shape
    buf = np.zeros(blocked_scale_bytes(R, C), dtype=np.uint8)
    rr, cc = np.indices((R, C))
    buf[blocked_offset(rr, cc, C)] = s
    return buf


def unswizzle(buf, R, C):
    """Blocked byte buffer -> logical scales S[R, C]."""
    buf = np.asarray(buf, dtype=np.uint8)
    rr, cc = np.indices((R, C))
    return buf[blocked_offset(rr, cc, C)]


def swizzle_stack(s):
    """Per-expert blocked buffers of S[G, R, C], concatenated in expert order."""
    return np.concatenate([swizzle(s[g]) for g in range(s.shape[0])])


# --------------------------------------------------------------------------
# Token groups and the pad path
# --------------------------------------------------------------------------
def group_bounds(offs):
    """(starts, ends) of each group from cumulative end offsets."""
    ends = np.asarray(offs, dtype=np.int64)
    starts = np.concatenate([[0], ends[:-1]]).astype(np.int64)
    if np.any(ends < starts):
        raise ValueError("offsets must be non-decreasing and start at >= 0")
    return starts, ends


def padded_group_starts(offs):
    """Row offset of each group in the padded layout, plus the total.

    p[0] = 0, p[g+1] = p[g] + ceil_to(size_g, 128): each group starts on a
    128-row boundary, so each 128-row scale tile holds one group only.
    """
    starts, ends = group_bounds(offs)
    padded = ceil_to(ends - starts, GROUP_ALIGN)
    return np.concatenate([[0], np.cumsum(padded)]).astype(np.int64)


def padded_rows_capacity(m_total, groups):
    """An upper bound of the padded row count that holds for any offsets."""
    return ((m_total + (GROUP_ALIGN - 1) * groups) // GROUP_ALIGN) * GROUP_ALIGN


def cast_dim0_grouped(x_bits, offs, m_cap):
    """dim0 cast of X[M, K] into the padded row layout with m_cap rows.

    Returns (Q[m_cap, K], S[m_cap, K/32]); pad rows hold q = 0 and b = 0.
    """
    x_bits = np.asarray(x_bits, dtype=np.uint16)
    M, K = x_bits.shape
    starts, ends = group_bounds(offs)
    p = padded_group_starts(offs)
    if ends[-1] != M or p[-1] > m_cap:
        raise ValueError("offsets do not cover X or the capacity is too small")
    q = np.zeros((m_cap, K), dtype=np.uint8)
    s = np.zeros((m_cap, K // BLOCK), dtype=np.uint8)
    for g in range(len(starts)):
        n = ends[g] - starts[g]
        if n == 0:
            continue
        qg, sg = cast_dim0(x_bits[starts[g]:ends[g]])
        q[p[g]:p[g] + n] = qg
        s[p[g]:p[g] + n] = sg
    return q, s


def cast_dim1_grouped(x_bits, offs, m_cap):
    """Per-group dim1 cast of X[M, K] into the padded token layout.

    Blocks of 32 tokens start at each group's start; a group's last partial
    block is completed with zeros (which leaves its amax unchanged). Returns
    (Q^T[K, m_cap], S[K, m_cap/32]); pad tokens hold q = 0, pad blocks b = 0.
    """
    x_bits = np.asarray(x_bits, dtype=np.uint16)
    M, K = x_bits.shape
    starts, ends = group_bounds(offs)
    p = padded_group_starts(offs)
    if ends[-1] != M or p[-1] > m_cap:
        raise ValueError("offsets do not cover X or the capacity is too small")
    qt = np.zeros((K, m_cap), dtype=np.uint8)
    s = np.zeros((K, m_cap // BLOCK), dtype=np.uint8)
    for g in range(len(starts)):
        n = ends[g] - starts[g]
        if n == 0:
            continue
        rows = ceil_to(n, BLOCK)
        xg = np.zeros((rows, K), dtype=np.uint16)     # bf16 +0.0 padding
        xg[:n] = x_bits[starts[g]:ends[g]]
        qg, sg = cast_dim1(xg)
        qt[:, p[g]:p[g] + rows] = qg
        s[:, p[g] // BLOCK:(p[g] + rows) // BLOCK] = sg
    return qt, s


# --------------------------------------------------------------------------
# Dequantization and the GEMMs (float64)
# --------------------------------------------------------------------------
def dequant(q, s):
    """Value of Q[..., R, C] with logical scales S[..., R, C/32] along the last axis."""
    vals = e4m3_decode(q)
    return vals * np.repeat(e8m0_to_f64(s), BLOCK, axis=-1)


def mm(a, b):
    """Dense D = A @ B^T with both operands K-contiguous, float64."""
    return np.asarray(a, np.float64) @ np.asarray(b, np.float64).T


def grouped_mm_m(a, b, offs):
    """M-groups GEMM: Y[start_g:end_g] = A[p_g : p_g + size_g] @ B[g]^T.

    a: dequantized padded rows [m_cap, K]; b: dequantized experts [G, N, K];
    offs: cumulative group ends. Returns Y[M, N] in the unpadded row order.
    """
    starts, ends = group_bounds(offs)
    p = padded_group_starts(offs)
    G, N, _ = b.shape
    y = np.zeros((ends[-1] if len(ends) else 0, N), dtype=np.float64)
    for g in range(G):
        n = ends[g] - starts[g]
        if n:
            y[starts[g]:ends[g]] = mm(a[p[g]:p[g] + n], b[g])
    return y


def grouped_mm_k(a, b, offs):
    """K-groups GEMM (wgrad): D[g] = A[:, tokens of g] @ B[:, tokens of g]^T.

    a: dequantized [N, m_cap], b: dequantized [K, m_cap] (tokens in the padded
    layout). An empty group gives D[g] = 0.
    """
    starts, ends = group_bounds(offs)
    p = padded_group_starts(offs)
    G = len(starts)
    out = np.zeros((G, a.shape[0], b.shape[0]), dtype=np.float64)
    for g in range(G):
        n = ends[g] - starts[g]
        if n:
            out[g] = mm(a[:, p[g]:p[g] + n], b[:, p[g]:p[g] + n])
    return out


def gemm_bound(ref, abs_ref):
    """Allowed |gpu - ref|: 2**-7 * |ref| + 1e-3 * (|A| @ |B|^T)."""
    return 2.0 ** -7 * np.abs(ref) + 1e-3 * abs_ref


# --------------------------------------------------------------------------
# Composite paths: MXFP8 linear and MoE grouped layer (float64 results)
# --------------------------------------------------------------------------
def linear_fwd(x_bits, w_bits):
    """Y = X W^T with X cast 1x32 (dim0) and W cast 32x32."""
    qx, sx = cast_dim0(x_bits)
    qw, st = cast_32x32(w_bits)
    s_fwd, _ = w32_scale_views(st)
    a, b = dequant(qx, sx), dequant(qw, s_fwd)
    return mm(a, b), mm(np.abs(a), np.abs(b))


def linear_dgrad(dy_bits, w_bits):
    """dX = dY W: dY cast along N (dim0), W^T scaled by the same 32x32 tiles."""
    qd, sd = cast_dim0(dy_bits)
    qw, st = cast_32x32(w_bits)
    _, s_dgrad = w32_scale_views(st)
    a = dequant(qd, sd)
    bt = dequant(np.ascontiguousarray(qw.T), s_dgrad)     # W^T [K, N]
    return mm(a, bt), mm(np.abs(a), np.abs(bt))


def linear_wgrad(dy_bits, x_bits):
    """dW = dY^T X: both operands cast along the token axis (dim1)."""
    qdt, sdt = cast_dim1(dy_bits)      # [N, M]
    qxt, sxt = cast_dim1(x_bits)       # [K, M]
    a, b = dequant(qdt, sdt), dequant(qxt, sxt)
    return mm(a, b), mm(np.abs(a), np.abs(b))


# --------------------------------------------------------------------------
# Backward overrides (ao "[moe training] Add backward_override to the MXFP8
# grouped GEMM", Design notes): the "high_precision" arm computes dgrad and
# wgrad as two plain bf16 grouped GEMMs over the saved, unpadded bf16
# operands; the "dequantized" arm runs the same two GEMMs on the quantized
# forward operands turned back into bf16, so its gradients are those of the
# function the quantized forward computes. Reading taken: "dequantize" means
# the exact value e4m3(q) * 2**(b - 127), rounded to the nearest bf16 (ties
# to even) -- the operand type of the bf16 grouped GEMM. The rounding only
# acts on magnitudes below 2**-133, the smallest bf16 subnormal, and on the
# one value above the bf16 range (256 * 2**120), which becomes infinity.
# --------------------------------------------------------------------------
BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127     # largest finite bf16
BF16_MIN_EXP = -133                            # exponent of the smallest bf16 subnormal


def round_to_bf16(x) -> np.ndarray:
    """Nearest bf16 value of each float64, ties to even, overflow to +-inf.

    bf16 keeps 8 significant bits; below 2**-126 the spacing stays 2**-133.
    The spacing of |x| is 2**(floor(log2 |x|) - 7), bounded below by 2**-133;
    np.rint rounds half to even. Zeros keep their sign; inf and NaN pass.
    """
    x = np.asarray(x, dtype=np.float64)
    out = x.copy()
    fin = np.isfinite(x) & (x != 0)
    ax = np.abs(x[fin])
    _, e = np.frexp(ax)                        # ax = m * 2**e, m in [0.5, 1)
    q_exp = np.maximum(e - 1 - 7, BF16_MIN_EXP)
    r = np.ldexp(np.rint(np.ldexp(ax, -q_exp)), q_exp)
    r = np.where(r > BF16_MAX, np.inf, r)
    out[fin] = np.copysign(r, x[fin])
    return out


def f64_to_bf16_bits(x) -> np.ndarray:
    """bf16 bit patterns of float64 values that are already bf16 values."""
    x = np.asarray(x, dtype=np.float64)
    r = round_to_bf16(x)
    if not np.array_equal(r, x, equal_nan=True):
        raise ValueError("f64_to_bf16_bits: value is not a bf16 value")
    bits = (r.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    return np.where(np.isnan(r), np.uint16(0x7FC0), bits).astype(np.uint16)


def dequant_bf16(q, s):
    """bf16 value of the MX tensor Q[..., R, C] with logical scales S[..., R, C/32].

    A NaN code (S.1111.111) or the E8M0 NaN byte 255 gives NaN.
    """
    v = dequant(q, s)
    v = np.where(np.repeat(np.asarray(s) == 255, BLOCK, axis=-1), np.nan, v)
    return round_to_bf16(v)


def dequant_dim0_grouped(q, s, offs):
    """Rows of a padded dim0 cast gathered back to the unpadded order, as bf16.

    q [m_cap, K] and logical scales s [m_cap, K/32] from cast_dim0_grouped;
    row start_g + i of the result is padded row p_g + i.
    """
    starts, ends = group_bounds(offs)
    p = padded_group_starts(offs)
    rows = np.concatenate([np.arange(p[g], p[g] + ends[g] - starts[g])
                           for g in range(len(starts))] + [np.zeros(0, np.int64)])
    return dequant_bf16(np.asarray(q)[rows], np.asarray(s)[rows])


def hp_grouped_mm_m(a, b, offs):
    """Groups split the rows: Y[start_g:end_g] = A[start_g:end_g] @ B[g].

    a [M, K], b [G, K, N] (float64); offsets are not padded. Rows outside
    every group (none when offs[-1] == M) stay zero.
    """
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    starts, ends = group_bounds(offs)
    y = np.zeros((a.shape[0], b.shape[2]), dtype=np.float64)
    for g in range(len(starts)):
        if ends[g] > starts[g]:
            y[starts[g]:ends[g]] = a[starts[g]:ends[g]] @ b[g]
    return y


def hp_grouped_mm_k(a, b, offs):
    """Groups split the contraction: D[g] = A[start_g:end_g]^T @ B[start_g:end_g].

    a [M, N], b [M, K] (float64) -> D [G, N, K]; an empty group gives zeros.
    """
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    starts, ends = group_bounds(offs)
    d = np.zeros((len(starts), a.shape[1], b.shape[1]), dtype=np.float64)
    for g in range(len(starts)):
        if ends[g] > starts[g]:
            d[g] = a[starts[g]:ends[g]].T @ b[starts[g]:ends[g]]
    return d


def moe_backward_high_precision(x_bits, w_bits, dy_bits, offs):
    """"high_precision" arm: dX = dY_g W_g per group, dW_g = dY_g^T X_g.

    x [M, K], w [G, N, K], dy [M, N] (bf16 bits). Returns
    (dX, |dY| |W|, dW, |dY|^T |X|), float64, the magnitudes for gemm_bound.
    """
    x, w, dy = bf16_to_f64(x_bits), bf16_to_f64(w_bits), bf16_to_f64(dy_bits)
    return (hp_grouped_mm_m(dy, w, offs), hp_grouped_mm_m(np.abs(dy), np.abs(w), offs),
            hp_grouped_mm_k(dy, x, offs), hp_grouped_mm_k(np.abs(dy), np.abs(x), offs))


def moe_backward_dequantized(x_bits, w_bits, dy_bits, offs):
    """"dequantized" arm: the same two GEMMs on the forward's quantized operands.

    The forward casts X rowwise (1x32) and each expert weight in 32x32 tiles;
    here those codes are dequantized to bf16 (the forward view of the weight
    scales) and used in place of X and W. Returns what
    moe_backward_high_precision returns.
    """
    qx, sx = cast_dim0(x_bits)
    qw, st = cast_32x32(w_bits)
    s_fwd, _ = w32_scale_views(st)
    xd, wd = dequant_bf16(qx, sx), dequant_bf16(qw, s_fwd)
    dy = bf16_to_f64(dy_bits)
    return (hp_grouped_mm_m(dy, wd, offs), hp_grouped_mm_m(np.abs(dy), np.abs(wd), offs),
            hp_grouped_mm_k(dy, xd, offs), hp_grouped_mm_k(np.abs(dy), np.abs(xd), offs))


def moe_backward_wgrad_hp(x_bits, w_bits, dy_bits, offs):
    """wgrad_with_hp: the weight gradient in high precision, the input gradient MXFP8.

    The MXFP8 knob that the "high_precision" override extends to both
    gradients (ao "[moe training] Add backward_override to the MXFP8 grouped
    GEMM", Known follow-ups). dX_g = dY_g W_g with dY cast rowwise (1x32, along
    N) into the padded group layout and W cast in 32x32 tiles, read through
    its dgrad scale view; dW_g = dY_g^T X_g on the bf16 operands. Returns what
    moe_backward_high_precision returns.
    """
    dy_bits = np.asarray(dy_bits, dtype=np.uint16)
    M = dy_bits.shape[0]
    G = np.asarray(w_bits).shape[0]
    m_cap = padded_rows_capacity(M, G)
    qd, sd = cast_dim0_grouped(dy_bits, offs, m_cap)
    qw, st = cast_32x32(w_bits)
    _, s_dgrad = w32_scale_views(st)
    a = dequant(qd, sd)                                              # [m_cap, N]
    b = dequant(np.ascontiguousarray(np.swapaxes(qw, 1, 2)), s_dgrad)   # [G, K, N]
    x, dy = bf16_to_f64(x_bits), bf16_to_f64(dy_bits)
    return (grouped_mm_m(a, b, offs), grouped_mm_m(np.abs(a), np.abs(b), offs),
            hp_grouped_mm_k(dy, x, offs), hp_grouped_mm_k(np.abs(dy), np.abs(x), offs))


# --------------------------------------------------------------------------
# Expert parallelism with the MXFP8 all-to-all (prime-rl PR #3388, Overview:
# MXFP8Config.enable_a2a; ao PR #4705, the expert-parallel pipeline
# benchmark). The rank that holds E experts receives the tokens of every
# source rank as groups (source, local expert), source major, so group g is
# served by local expert g % E. Reading: the dispatch carries the rowwise
# (1x32) cast of the tokens, so the forward and dgrad operands are those of
# the plain grouped GEMM; the wgrad casts the received activations
# columnwise from their dequantized (bf16) values, since the bf16 tokens
# never reach the expert's rank; dW of expert e sums its groups.
# --------------------------------------------------------------------------
def ep_expert_forward(x_bits, w_bits, offs, E):
    """Y[rows of g] = dim0(X)[rows of g] @ 32x32(W[g % E])^T.

    x [M, K] received tokens (bf16 bits) in groups `offs` (G = len(offs), a
    multiple of E); w [E, N, K]. Returns (Y, |A| |B|^T), float64.
    """
    qx, sx = cast_dim0(x_bits)
    a = dequant(qx, sx)
    qw, st = cast_32x32(w_bits)
    s_fwd, _ = w32_scale_views(st)
    b = dequant(qw, s_fwd)
    starts, ends = group_bounds(offs)
    E_, N, _ = b.shape
    if E_ != E or len(starts) % E:
        raise ValueError("G must be a multiple of E and w must hold E experts")
    y = np.zeros((a.shape[0], N))
    ya = np.zeros((a.shape[0], N))
    for g in range(len(starts)):
        r = slice(starts[g], ends[g])
        y[r] = mm(a[r], b[g % E])
        ya[r] = mm(np.abs(a[r]), np.abs(b[g % E]))
    return y, ya


def ep_expert_backward(x_bits, w_bits, dy_bits, offs, E):
    """(dX, |dX| bound, dW, |dW| bound) of the received groups, float64.

    dX[rows of g] = dim0(dY)[rows of g] @ W[g % E] with W's 32x32 codes and
    their dgrad scale view; dW[e] = sum over groups g = e, e + E, ... of
    dim1_g(dY)^T dim1_g(X~), dim1_g the per-group columnwise cast and
    X~ = bf16(dequant(dim0(X))).
    """
    starts, ends = group_bounds(offs)
    G = len(starts)
    if G % E:
        raise ValueError("G must be a multiple of E")
    qd, sd = cast_dim0(dy_bits)
    da = dequant(qd, sd)
    qw, st = cast_32x32(w_bits)
    _, s_dg = w32_scale_views(st)
    wt = dequant(np.ascontiguousarray(np.swapaxes(qw, 1, 2)), s_dg)          # [E, K, N]
    dx = np.zeros((da.shape[0], wt.shape[1]))
    dxa = np.zeros_like(dx)
    for g in range(G):
        r = slice(starts[g], ends[g])
        dx[r] = mm(da[r], wt[g % E])
        dxa[r] = mm(np.abs(da[r]), np.abs(wt[g % E]))
    qx, sx = cast_dim0(x_bits)
    x_deq = f64_to_bf16_bits(dequant_bf16(qx, sx))
    cap = int(padded_group_starts(offs)[-1])
    qa, sa = cast_dim1_grouped(dy_bits, offs, cap)
    qb, sb = cast_dim1_grouped(x_deq, offs, cap)
    a, b = dequant(qa, sa), dequant(qb, sb)
    per_group, per_group_abs = grouped_mm_k(a, b, offs), grouped_mm_k(np.abs(a), np.abs(b), offs)
    dw = per_group.reshape(G // E, E, *per_group.shape[1:]).sum(axis=0)
    dwa = per_group_abs.reshape(G // E, E, *per_group.shape[1:]).sum(axis=0)
    return dx, dxa, dw, dwa
