"""Pins of the CPU oracle against things other than itself.

Each test checks the oracle against a fact the pages or the mathematics fix:
hand-worked golden values (tests/golden/, each file citing its source),
closed forms derived independently of the oracle's search, a library routine
(torch's CPU float8_e4m3fn conversion), invariants of RCEIL scaling, and brute
force on tiny inputs. A plausible slip in the oracle (wrong tie rule, dropped
clamp, transposed operand, wrong swizzle index) fails at least one of them;
``test_planted_*`` shows that for two such slips.
"""
import os

import numpy as np
import pytest
import torch

from oracle import mx_oracle as O
from mxfp8_block_scaled_cast_b200 import synthetic as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


def _all_finite_bf16():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    exp = (bits >> 7) & 0xFF
    return bits[exp != 0xFF]


# ----------------------------------------------------------------- E4M3 ----
def test_e4m3_decode_golden():
    for code, val in _golden_rows("e4m3_codes.txt"):
        got = O.e4m3_decode(np.array([int(code, 16)]))[0]
        assert got == float(val) and np.signbit(got) == np.signbit(float(val)), code
    assert np.isnan(O.e4m3_decode(np.array([0x7F, 0xFF]))).all()


def test_e4m3_encode_roundtrips_every_finite_code():
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], dtype=np.int64)
    vals = O.e4m3_decode(codes)
    assert np.array_equal(O.e4m3_encode(vals), codes.astype(np.uint8))


def _torch_e4m3(v):
    t = torch.from_numpy(np.asarray(v, np.float64).astype(np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


@pytest.mark.parametrize("b", [0, 1, 120, 127, 134, 247, 3, 64, 190, 230])
def test_e4m3_encode_matches_torch_exhaustive_bf16(b):
    """All finite bf16 x at scale byte b: oracle code == torch's RNE cast of x/2^(b-127)."""
    x = O.bf16_to_f64(_all_finite_bf16())
    v = x * 2.0 ** (127 - b)
    keep = np.abs(v) <= 448.0          # torch's cast does not saturate; RCEIL never exceeds 448
    ours = O.e4m3_encode(v[keep])
    ref = _torch_e4m3(v[keep])
    assert np.array_equal(ours, ref)


def test_e4m3_saturates():
    assert O.e4m3_encode(np.array([460.0, 1000.0, -1e6, 464.0]) ).tolist() == [0x7E, 0x7E, 0xFE, 0x7E]


# ----------------------------------------------------------------- RCEIL ---
def _closed_form_b(bits):
    """b from the bf16 bit fields: E - 8 + [m > 96], clamped to [0, 254].

    448 = 1.75 * 2^8 and 1.75 = 1 + 96/128, so for amax = (1 + m/128) * 2^(E-127)
    the ratio amax / 448 exceeds the power of two 2^(E-135) exactly when m > 96.
    """
    E = (bits.astype(np.int64) >> 7) & 0xFF
    m = bits.astype(np.int64) & 0x7F
    return np.clip(E - 8 + (m > 96), 0, 254)


def test_rceil_matches_closed_form_on_every_bf16_amax():
    bits = _all_finite_bf16()
    bits = bits[bits < 0x8000]             # non-negative patterns (amax >= 0)
    amax = O.bf16_to_f64(bits)
    assert np.array_equal(O.rceil_e8m0(amax).astype(np.int64), _closed_form_b(bits))


def test_rceil_matches_float64_log2():
    bits = _all_finite_bf16()
    bits = bits[(bits < 0x8000) & (bits > 0)]
    amax = O.bf16_to_f64(bits)
    ref = np.clip(np.ceil(np.log2(amax / 448.0)) + 127, 0, 254)
    assert np.array_equal(O.rceil_e8m0(amax).astype(np.int64), ref.astype(np.int64))


def test_rceil_tiny_amax_reading_gives_zero():
    # amax <= 448 * 2^-127 (about 2.63e-36): the exact rule clamps to b = 0 (a
    # float32 quotient amax/448 would be subnormal there and could give 1; the
    # exact reading is kept). Just above the threshold b = 1.
    amax = np.array([9.2e-41, 1e-38, 2.6e-36, 448.0 * 2.0 ** -127, 2.7e-36, 5.0e-36])
    assert O.rceil_e8m0(amax).tolist() == [0, 0, 0, 0, 1, 1]
    assert O.rceil_e8m0(np.array([0.0]))[0] == 0


def test_worked_examples_golden():
    for amax, b, x, q in _golden_rows("rceil_worked_examples.txt"):
        got_b = O.rceil_e8m0(np.array([float(amax)]))[0]
        assert got_b == int(b), amax
        blk = np.zeros(32)
        blk[0] = float(amax)
        blk[1] = float(x)
        qq, bb = O.quantize_blocks(blk)
        assert bb == int(b)
        assert qq[1] == int(q, 16), (amax, x)


def test_scale_invariants_random_blocks():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((4096, 32)) * np.exp2(rng.integers(-40, 40, (4096, 1)))
    xb = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    xf = O.bf16_to_f64(S.bf16_bits(xb))
    q, b = O.quantize_blocks(xf)
    amax = np.abs(xf).max(axis=1)
    scale = O.e8m0_to_f64(b)
    assert np.all(scale >= amax / 448.0)                       # large enough
    assert np.all((b == 0) | (scale / 2 < amax / 448.0))       # and minimal
    deq = O.e4m3_decode(q)
    assert np.all(np.abs(deq) <= 448.0)
    # dequantized error within half an E4M3 ulp of the scaled value
    v = np.abs(xf) / scale[:, None]
    e = np.floor(np.log2(np.maximum(v, 2.0 ** -6)))
    half_ulp = 0.5 * np.exp2(e - 3)
    assert np.all(np.abs(xf - deq * scale[:, None]) <= half_ulp * scale[:, None])


def test_subnormal_block_keeps_nonzero_codes():
    # bf16 subnormals (exponent field 0) get b = 0 and are scaled by 2^127 exactly.
    bits = np.array([0x0001, 0x0040, 0x007F, 0x8003] + [0] * 28, dtype=np.uint16)
    xf = O.bf16_to_f64(bits)
    q, b = O.quantize_blocks(xf)
    assert b == 0
    vals = O.e4m3_decode(q[:4]) * 2.0 ** -127
    assert np.all(vals != 0) and vals[3] < 0


def test_floor_matches_closed_form_on_every_bf16_amax():
    """FLOOR: b = max(E - 8, 0) from the bf16 exponent field (2^(E-127) <= amax < 2^(E-126))."""
    bits = _all_finite_bf16()
    bits = bits[bits < 0x8000]
    amax = O.bf16_to_f64(bits)
    E = (bits.astype(np.int64) >> 7) & 0xFF
    assert np.array_equal(O.floor_e8m0(amax).astype(np.int64), np.maximum(E - 8, 0))


def test_floor_vs_rceil_and_saturation():
    bits = _all_finite_bf16()
    bits = bits[(bits < 0x8000) & (bits > 0)]
    amax = O.bf16_to_f64(bits)
    f, r = O.floor_e8m0(amax).astype(int), O.rceil_e8m0(amax).astype(int)
    assert np.all((r == f) | (r == f + 1))          # the two rules differ by at most one binade
    # amax 500 -> floor(log2 500) = 8 -> b = 127, scale 1: 500 saturates to 448, 460 too
    blk = np.zeros(32)
    blk[:3] = [500.0, -460.0, 300.0]
    q, b = O.quantize_blocks(blk, rule="floor")
    assert b == 127 and q[0] == 0x7E and q[1] == 0xFE and O.e4m3_decode(q[2:3])[0] == 288.0
    q, b = O.quantize_blocks(blk, rule="rceil")     # RCEIL never saturates: 500 -> scale 2
    assert b == 128 and O.e4m3_decode(q[:1])[0] == 256.0


# ------------------------------------------------------------ geometry -----
def test_dim1_equals_dim0_of_transpose():
    x = S.bf16_bits(S.tiny_activation(0))
    q1, s1 = O.cast_dim1(x)
    q0, s0 = O.cast_dim0(np.ascontiguousarray(x.T))
    assert np.array_equal(q1, q0) and np.array_equal(s1, s0)


def test_fused_is_the_pair():
    x = S.bf16_bits(S.normal_bf16((64, 96), seed=3))
    (a, b), (c, d) = O.cast_2d(x)
    ea, eb = O.cast_dim0(x)
    ec, ed = O.cast_dim1(x)
    for u, v in ((a, ea), (b, eb), (c, ec), (d, ed)):
        assert np.array_equal(u, v)


def test_tiny_config_worked_blocks():
    x = S.bf16_bits(S.tiny_activation(0))
    q, s = O.cast_dim0(x)
    assert s[0, 0] == 0 and not q[0, :32].any()               # the zero block
    assert S.bf16_bits(S.tiny_activation(0))[1, 0] == 0x476A  # bf16(6e4) = 59904
    assert s[1, 0] == 135 and q[1, 0] == 0x77


def test_32x32_brute_force():
    w = S.bf16_bits(S.normal_bf16((64, 96), 0.02, seed=5))
    q, st = O.cast_32x32(w)
    wf = O.bf16_to_f64(w)
    for i in range(2):
        for j in range(3):
            tile = wf[32 * i:32 * i + 32, 32 * j:32 * j + 32]
            amax = float(np.abs(tile).max())
            e = 0
            while 448.0 * 2.0 ** e >= amax:      # walk down then up: smallest e
                e -= 1
            while 448.0 * 2.0 ** e < amax:
                e += 1
            assert st[i, j] == e + 127
            for r in range(0, 32, 7):
                for c in range(0, 32, 5):
                    code = O.e4m3_encode(np.array([tile[r, c] / 2.0 ** e]))[0]
                    assert q[32 * i + r, 32 * j + c] == code


def test_32x32_scale_is_max_of_rowwise_scales():
    w = S.bf16_bits(S.normal_bf16((128, 256), 1.0, seed=6))
    _, st = O.cast_32x32(w)
    _, s0 = O.cast_dim0(w)
    assert np.array_equal(st, s0.reshape(4, 32, 8).max(axis=1))
    s_fwd, s_dgrad = O.w32_scale_views(st)
    assert s_fwd.shape == (128, 8) and s_dgrad.shape == (256, 4)
    assert s_fwd[37, 5] == st[1, 5] and s_dgrad[200, 3] == st[3, 6]


# ------------------------------------------------------------- swizzle -----
def test_blocked_offsets_golden():
    for r, c, C, off in _golden_rows("blocked_offsets.txt"):
        assert O.blocked_offset(int(r), int(c), int(C)) == int(off)


@pytest.mark.parametrize("R,C", [(128, 4), (256, 8), (300, 18), (16384 // 64, 18), (1, 1), (129, 5)])
def test_swizzle_is_a_bijection_onto_non_pad_bytes(R, C):
    rng = np.random.default_rng(R * 100 + C)
    s = rng.integers(1, 255, (R, C), dtype=np.uint8)
    buf = O.swizzle(s)
    assert buf.size == O.ceil_to(R, 128) * O.ceil_to(C, 4)
    assert np.array_equal(O.unswizzle(buf, R, C), s)
    rr, cc = np.indices((R, C))
    offs = O.blocked_offset(rr, cc, C).ravel()
    assert len(np.unique(offs)) == R * C
    assert np.count_nonzero(buf) == R * C               # pads stay 0x00


# ----------------------------------------------------------- pad path ------
def test_group_padding_offsets():
    offs = np.array([100, 100, 356, 357])
    p = O.padded_group_starts(offs)
    assert p.tolist() == [0, 128, 128, 384, 512]
    assert O.padded_rows_capacity(357, 4) >= p[-1]
    sizes = S.zipf_group_sizes(32, 32768, 1.2, 3, 0)
    cap = O.padded_rows_capacity(32768, 32)
    assert O.padded_group_starts(np.cumsum(sizes))[-1] <= cap


def test_grouped_dim0_places_rows_and_zero_pads():
    x = S.bf16_bits(S.normal_bf16((300, 64), seed=7))
    offs = np.array([100, 100, 250, 300])
    cap = O.padded_rows_capacity(300, 4)
    q, s = O.cast_dim0_grouped(x, offs, cap)
    p = O.padded_group_starts(offs)
    starts, ends = O.group_bounds(offs)
    for g in range(4):
        n = ends[g] - starts[g]
        qg, sg = O.cast_dim0(x[starts[g]:ends[g]]) if n else (None, None)
        if n:
            assert np.array_equal(q[p[g]:p[g] + n], qg)
            assert np.array_equal(s[p[g]:p[g] + n], sg)
    mask = np.ones(cap, bool)
    for g in range(4):
        mask[p[g]:p[g] + ends[g] - starts[g]] = False
    assert not q[mask].any() and not s[mask].any()


def test_grouped_dim1_aligned_equals_global_dim1():
    x = S.bf16_bits(S.normal_bf16((512, 64), seed=8))
    offs = np.array([128, 384, 384, 512])
    qt, st = O.cast_dim1_grouped(x, offs, 512)
    q1, s1 = O.cast_dim1(x)
    assert np.array_equal(qt, q1) and np.array_equal(st, s1)


def test_grouped_dim1_blocks_restart_at_group_start():
    x = S.bf16_bits(S.normal_bf16((70, 32), seed=9))
    offs = np.array([40, 70])
    qt, st = O.cast_dim1_grouped(x, offs, 256)
    # group 0: tokens 0..39 at columns 0..39 -> blocks [0,32) and [32,40)+zeros
    assert np.array_equal(qt[:, :32], O.cast_dim1(x[:32])[0])
    xb = np.zeros((32, 32), np.uint16)
    xb[:8] = x[32:40]
    assert np.array_equal(qt[:, 32:64], O.cast_dim1(xb)[0])
    # group 1 starts at padded column 128
    xb = np.zeros((32, 32), np.uint16)
    xb[:30] = x[40:70]
    assert np.array_equal(qt[:, 128:160], O.cast_dim1(xb)[0])
    assert not qt[:, 64:128].any() and not st[:, 2:4].any()


# --------------------------------------------------------------- GEMMs -----
def _loop_mm(a, b):
    out = np.zeros((a.shape[0], b.shape[0]))
    for i in range(a.shape[0]):
        for j in range(b.shape[0]):
            acc = 0.0
            for k in range(a.shape[1]):
                acc += a[i, k] * b[j, k]
            out[i, j] = acc
    return out


def test_grouped_mm_m_equals_loop_of_dense():
    rng = np.random.default_rng(11)
    offs = np.array([3, 3, 9])
    cap = O.padded_rows_capacity(9, 3)
    a = np.zeros((cap, 4))
    p = O.padded_group_starts(offs)
    x = rng.standard_normal((9, 4))
    a[p[0]:p[0] + 3] = x[0:3]
    a[p[2]:p[2] + 6] = x[3:9]
    b = rng.standard_normal((3, 5, 4))
    y = O.grouped_mm_m(a, b, offs)
    assert np.allclose(y[0:3], _loop_mm(x[0:3], b[0]))
    assert np.allclose(y[3:9], _loop_mm(x[3:9], b[2]))


def test_grouped_mm_k_equals_loop_and_empty_groups_are_zero():
    rng = np.random.default_rng(12)
    offs = np.array([5, 5, 12])
    p = O.padded_group_starts(offs)
    a = np.zeros((3, 384))
    b = np.zeros((4, 384))
    da = rng.standard_normal((3, 12))
    db = rng.standard_normal((4, 12))
    a[:, p[0]:p[0] + 5], b[:, p[0]:p[0] + 5] = da[:, :5], db[:, :5]
    a[:, p[2]:p[2] + 7], b[:, p[2]:p[2] + 7] = da[:, 5:], db[:, 5:]
    d = O.grouped_mm_k(a, b, offs)
    assert np.allclose(d[0], _loop_mm(da[:, :5], db[:, :5]))
    assert np.all(d[1] == 0.0)
    assert np.allclose(d[2], _loop_mm(da[:, 5:], db[:, 5:]))


def test_one_group_equals_dense_linear():
    x, w, _ = S.linear_problem(128, 64, 96, seed=2)
    xb, wb = S.bf16_bits(x), S.bf16_bits(w)
    y, _ = O.linear_fwd(xb, wb)
    qx, sx = O.cast_dim0_grouped(xb, np.array([128]), 128)
    qw, st = O.cast_32x32(wb[None])
    s_fwd, _ = O.w32_scale_views(st)
    yg = O.grouped_mm_m(O.dequant(qx, sx), O.dequant(qw, s_fwd), np.array([128]))
    assert np.array_equal(y, yg)


def test_linear_grads_match_float64_definition_within_mx_error():
    x, w, dy = S.linear_problem(64, 64, 96, seed=4)
    xb, wb, db = (S.bf16_bits(t) for t in (x, w, dy))
    xf, wf, df = (O.bf16_to_f64(t) for t in (xb, wb, db))
    for (got, _), ref in ((O.linear_fwd(xb, wb), xf @ wf.T),
                          (O.linear_dgrad(db, wb), df @ wf),
                          (O.linear_wgrad(db, xb), df.T @ xf)):
        # E4M3 keeps 3 mantissa bits: each operand is within 2^-4 relative per
        # element, so the product's relative Frobenius error stays well below 5%.
        assert got.shape == ref.shape and np.all(np.isfinite(got))
        rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        assert rel < 0.05, rel


# ---------------------------------------------------- planted mistakes -----
def test_planted_tie_rule_is_caught(monkeypatch):
    """A round-half-away encoder (a plausible slip) fails the torch pin."""
    def half_away(v):
        v = np.asarray(v, np.float64)
        a = np.minimum(np.abs(v), 448.0)
        d = np.abs(O._POS_VALUES[None, :] - a[:, None])
        code = len(O._POS_VALUES) - 1 - np.argmin(d[:, ::-1], axis=1)   # ties -> larger
        return (code | (np.signbit(v).astype(np.int64) << 7)).astype(np.uint8)
    monkeypatch.setattr(O, "e4m3_encode", half_away)
    with pytest.raises(AssertionError):
        test_e4m3_encode_matches_torch_exhaustive_bf16(127)


def test_planted_swizzle_slip_is_caught(monkeypatch):
    """Swapping the two in-tile strides (16 and 4) fails the golden offsets."""
    real = O.blocked_offset

    def wrong(r, c, cols):
        r = np.asarray(r)
        rr = r % 128
        return real(r, c, cols) - (rr % 32) * 16 - (rr // 32) * 4 + (rr % 32) * 4 + (rr // 32) * 16
    monkeypatch.setattr(O, "blocked_offset", wrong)
    with pytest.raises(AssertionError):
        test_blocked_offsets_golden()


# ------------------------------------------- backward overrides (bf16) -----
def _f32_samples(n=200000, seed=21):
    """fp32 bit patterns over every exponent (subnormals and near-ties included)."""
    rng = np.random.default_rng(seed)
    u = rng.integers(0, 2 ** 32, size=n, dtype=np.uint64).astype(np.uint32)
    # force a share of exact ties and one-off-ties of the bf16 rounding
    tie = rng.random(n) < 0.3
    low = u & np.uint32(0xFFFF)
    low = np.where(tie, np.uint32(0x8000) + rng.integers(-1, 2, size=n).astype(np.int64).astype(np.uint32),
                   low)
    u = (u & np.uint32(0xFFFF0000)) | (low & np.uint32(0xFFFF))
    f = u.view(np.float32)
    return f[np.isfinite(f)]


def test_round_to_bf16_matches_torch_conversion():
    """bf16 rounding of fp32 values (exact in float64) against torch's CPU cast."""
    f = _f32_samples()
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.round_to_bf16(f.astype(np.float64))
    assert np.array_equal(np.signbit(got), np.signbit(ref))
    assert np.array_equal(got, ref)


def test_round_to_bf16_worked_values():
    # ties to even at 1 and in the subnormal range, overflow at the top
    x = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 2.0 ** -134, 3 * 2.0 ** -134,
                  (2 - 2.0 ** -8) * 2.0 ** 127, (2 - 2.0 ** -7 - 2.0 ** -9) * 2.0 ** 127, -0.0])
    want = np.array([1.0, 1 + 2.0 ** -6, 0.0, 2.0 ** -132, np.inf, O.BF16_MAX, -0.0])
    got = O.round_to_bf16(x)
    assert np.array_equal(got, want) and np.signbit(got[-1])


def test_dequant_bf16_matches_torch_float8_decode_every_code_and_scale():
    """Every E4M3 code at every finite scale byte, against torch's float8 decode."""
    codes = np.arange(256, dtype=np.uint8)
    b = np.arange(255, dtype=np.uint8)
    q = np.repeat(codes[None, :], b.size, axis=0)                   # [255, 256]
    s = np.repeat(b[:, None], 256 // 32, axis=1)                    # [255, 8]
    got = O.dequant_bf16(q, s)
    tq = torch.from_numpy(q.copy()).view(torch.float8_e4m3fn).to(torch.float32)
    scale = torch.from_numpy(np.ldexp(1.0, b.astype(np.int64) - 127)).to(torch.float32)
    ref = (tq * scale[:, None]).to(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))
    # the E8M0 NaN byte
    assert np.all(np.isnan(O.dequant_bf16(np.ones((1, 32), np.uint8), np.array([[255]], np.uint8))))


def _loop_mm_plain(a, b):
    """C = A B by explicit sums (A [m, k], B [k, n])."""
    out = np.zeros((a.shape[0], b.shape[1]))
    for i in range(a.shape[0]):
        for j in range(b.shape[1]):
            acc = 0.0
            for k in range(a.shape[1]):
                acc += a[i, k] * b[k, j]
            out[i, j] = acc
    return out


def test_hp_grouped_mm_m_brute_force_unpadded_groups():
    rng = np.random.default_rng(31)
    offs = np.array([3, 3, 8, 11])        # sizes 3, 0, 5, 3: no padding
    a = rng.standard_normal((11, 4))
    b = rng.standard_normal((4, 4, 6))
    y = O.hp_grouped_mm_m(a, b, offs)
    assert np.allclose(y[0:3], _loop_mm_plain(a[0:3], b[0]))
    assert np.allclose(y[3:8], _loop_mm_plain(a[3:8], b[2]))
    assert np.allclose(y[8:11], _loop_mm_plain(a[8:11], b[3]))


def test_hp_grouped_mm_k_brute_force_and_empty_group():
    rng = np.random.default_rng(32)
    offs = np.array([4, 4, 9])
    a = rng.standard_normal((9, 3))
    b = rng.standard_normal((9, 5))
    d = O.hp_grouped_mm_k(a, b, offs)
    assert d.shape == (3, 3, 5)
    assert np.allclose(d[0], _loop_mm_plain(a[0:4].T, b[0:4]))
    assert np.all(d[1] == 0.0)
    assert np.allclose(d[2], _loop_mm_plain(a[4:9].T, b[4:9]))
    # the groups together are the dense product
    assert np.allclose(d.sum(0), a.T @ b)


def test_high_precision_arm_is_the_dense_gradient_at_one_group():
    x, w, dy = S.linear_problem(64, 96, 128, seed=5)
    xb, wb, db = (S.bf16_bits(t) for t in (x, w, dy))
    dx, _, dw, _ = O.moe_backward_high_precision(xb, wb[None], db, np.array([64]))
    xt, wt, dt = (torch.from_numpy(O.bf16_to_f64(t)) for t in (xb, wb, db))
    assert np.allclose(dx, (dt @ wt).numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(dw[0], (dt.T @ xt).numpy(), rtol=1e-12, atol=1e-12)


def _mx_exact_bits(shape, rng, tile):
    """bf16 values that the casts reproduce exactly: per scale block, E4M3
    values times 2**e with one element at +-448 * 2**e, so RCEIL picks e."""
    vals = O._POS_VALUES[rng.integers(0, 0x7F, size=shape)]
    vals = vals * np.where(rng.random(shape) < 0.5, -1.0, 1.0)
    R, C = shape
    th, tw = tile
    e = rng.integers(-20, 20, size=(R // th, C // tw))
    vals = vals.reshape(R // th, th, C // tw, tw)
    vals[:, 0, :, 0] = 448.0
    vals = vals * np.exp2(e)[:, None, :, None]
    return O.f64_to_bf16_bits(vals.reshape(R, C))


def test_dequantized_arm_equals_high_precision_arm_on_mx_exact_operands():
    """If X and W are MX-representable the quantized forward loses nothing, so
    the two override arms must give the same gradients."""
    rng = np.random.default_rng(33)
    xb = _mx_exact_bits((96, 64), rng, (1, 32))
    wb = np.stack([_mx_exact_bits((64, 64), rng, (32, 32)) for _ in range(2)])
    db = S.bf16_bits(S.normal_bf16((96, 64), seed=7))
    offs = np.array([40, 96])
    hp = O.moe_backward_high_precision(xb, wb, db, offs)
    dq = O.moe_backward_dequantized(xb, wb, db, offs)
    for u, v in zip(hp, dq):
        assert np.array_equal(u, v)
    # and a generic X differs (the arm does dequantize the forward's codes)
    xg = S.bf16_bits(S.normal_bf16((96, 64), seed=8))
    assert not np.array_equal(O.moe_backward_high_precision(xg, wb, db, offs)[2],
                              O.moe_backward_dequantized(xg, wb, db, offs)[2])


def test_wgrad_hp_arm_on_mx_exact_and_generic_operands():
    """wgrad_with_hp: with dY MX-exact in 1x32 blocks along N and W MX-exact in
    32x32 tiles, the MXFP8 dgrad loses nothing, so dX is the plain float64
    product per group (a torch matmul, to summation order); dW is always the
    bf16 product, so it
    equals the high-precision arm's; for a generic dY the dgrad is quantized
    and differs from the high-precision arm's."""
    rng = np.random.default_rng(34)
    offs = np.array([40, 96])                       # groups of 40 and 56 tokens (pad path)
    db = _mx_exact_bits((96, 64), rng, (1, 32))
    wb = np.stack([_mx_exact_bits((64, 128), rng, (32, 32)) for _ in range(2)])   # [G, N=64, K=128]
    xb = S.bf16_bits(S.normal_bf16((96, 128), seed=10))
    dx, adx, dw, _ = O.moe_backward_wgrad_hp(xb, wb, db, offs)
    dy_f, w_f, x_f = O.bf16_to_f64(db), O.bf16_to_f64(wb), O.bf16_to_f64(xb)
    for g, (lo, hi) in enumerate([(0, 40), (40, 96)]):
        want = (torch.from_numpy(dy_f[lo:hi]) @ torch.from_numpy(w_f[g])).numpy()
        assert np.allclose(dx[lo:hi], want, rtol=1e-12, atol=1e-300)
        want = (torch.from_numpy(dy_f[lo:hi]).T @ torch.from_numpy(x_f[lo:hi])).numpy()
        assert np.allclose(dw[g], want, rtol=1e-12, atol=1e-300)
    assert np.all(adx >= np.abs(dx))
    hp = O.moe_backward_high_precision(xb, wb, db, offs)
    assert np.array_equal(dw, hp[2])
    dg = S.bf16_bits(S.normal_bf16((96, 64), seed=11))
    mixed, full = O.moe_backward_wgrad_hp(xb, wb, dg, offs), O.moe_backward_high_precision(xb, wb, dg, offs)
    assert np.array_equal(mixed[2], full[2])
    assert not np.array_equal(mixed[0], full[0])


def test_dequant_grouped_gathers_padded_rows():
    x = S.normal_bf16((300, 64), seed=9)
    xb = S.bf16_bits(x)
    offs = np.array([37, 37, 300])
    cap = O.padded_rows_capacity(300, 3)
    qp, sp = O.cast_dim0_grouped(xb, offs, cap)
    got = O.dequant_dim0_grouped(qp, sp, offs)
    q, s = O.cast_dim0(xb)
    assert np.array_equal(got, O.dequant_bf16(q, s))


def test_planted_padded_starts_in_hp_wgrad_is_caught(monkeypatch):
    """Taking the group rows at the padded starts (as the MXFP8 GEMMs do)
    instead of the unpadded ones fails the brute force."""
    def slip(a, b, offs):
        starts, ends = O.group_bounds(offs)
        p = O.padded_group_starts(offs)
        d = np.zeros((len(starts), a.shape[1], b.shape[1]))
        for g in range(len(starts)):
            n = ends[g] - starts[g]
            d[g] = a[p[g]:p[g] + n].T @ b[p[g]:p[g] + n]
        return d
    monkeypatch.setattr(O, "hp_grouped_mm_k", slip)
    with pytest.raises(AssertionError):
        test_hp_grouped_mm_k_brute_force_and_empty_group()


# ------------------------------------------ expert parallelism (MXFP8 a2a) --
def _torch_deq(codes, scale_bytes):
    """Values of E4M3 codes [R, C] with per-32 scale bytes [R, C/32], via torch's float8 type."""
    v = torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return v * np.repeat(2.0 ** (np.asarray(scale_bytes, np.float64) - 127.0), 32, axis=-1)


def _ep_case(seed=3):
    rng = np.random.default_rng(seed)
    E, W, K, N = 2, 3, 64, 64
    counts = rng.integers(0, 40, size=W * E)
    counts[1] = 0                                    # an empty (source, expert) group
    offs = np.cumsum(counts)
    M = int(offs[-1])
    x = S.bf16_bits(S.normal_bf16((M, K), seed=seed))
    w = S.bf16_bits(S.normal_bf16((E, N, K), 0.1, seed=seed + 1))
    dy = S.bf16_bits(S.normal_bf16((M, N), 0.1, seed=seed + 2))
    return E, W, K, N, offs, x, w, dy


def test_ep_expert_forward_brute_force_uses_expert_g_mod_e():
    """Each row of group g times expert g % E, entry by entry, from codes decoded by torch."""
    E, W, K, N, offs, x, w, _ = _ep_case()
    y, _ = O.ep_expert_forward(x, w, offs, E)
    qx, sx = O.cast_dim0(x)
    xv = _torch_deq(qx, sx)
    starts, ends = O.group_bounds(offs)
    for e in range(E):
        qw, st = O.cast_32x32(w[e])
        wv = _torch_deq(qw, O.w32_scale_views(st)[0])
        for g in range(e, W * E, E):
            for i in range(starts[g], ends[g]):
                for n in range(0, N, 7):
                    assert y[i, n] == pytest.approx(sum(xv[i, k] * wv[n, k] for k in range(K)), rel=1e-12, abs=1e-300)


def test_ep_expert_backward_dx_brute_force():
    E, W, K, N, offs, x, w, dy = _ep_case(4)
    dx, _, _, _ = O.ep_expert_backward(x, w, dy, offs, E)
    qd, sd = O.cast_dim0(dy)
    dv = _torch_deq(qd, sd)
    starts, ends = O.group_bounds(offs)
    for g in range(W * E):
        qw, st = O.cast_32x32(w[g % E])
        wtv = _torch_deq(np.ascontiguousarray(qw.T), O.w32_scale_views(st)[1])    # [K, N]
        for i in range(starts[g], ends[g], 5):
            for k in range(0, K, 9):
                assert dx[i, k] == pytest.approx(sum(dv[i, n] * wtv[k, n] for n in range(N)), rel=1e-12, abs=1e-300)


def test_ep_expert_backward_dw_sums_each_experts_groups_over_sources():
    """dW[e] is the sum over sources of the per-group wgrad of group (source, e), each
    computed alone by the pinned single-group path (a swapped sum order fails)."""
    E, W, K, N, offs, x, w, dy = _ep_case(5)
    _, _, dw, _ = O.ep_expert_backward(x, w, dy, offs, E)
    qx, sx = O.cast_dim0(x)
    x_deq = O.f64_to_bf16_bits(O.dequant_bf16(qx, sx))
    starts, ends = O.group_bounds(offs)
    for e in range(E):
        want = np.zeros((N, K))
        for g in range(e, W * E, E):
            n = ends[g] - starts[g]
            if n == 0:
                continue
            one = np.array([n])
            cap = O.padded_rows_capacity(n, 1)
            qa, sa = O.cast_dim1_grouped(dy[starts[g]:ends[g]], one, cap)
            qb, sb = O.cast_dim1_grouped(x_deq[starts[g]:ends[g]], one, cap)
            want += _torch_deq(qa, sa) @ _torch_deq(qb, sb).T
        np.testing.assert_allclose(dw[e], want, rtol=1e-12, atol=1e-300)


def test_ep_one_rank_mx_exact_inputs_equal_the_plain_layer():
    """With one rank (G == E) and activations that are exact MX values, the expert-side
    backward is the plain grouped layer's: dequantizing the dispatched codes is exact."""
    E, K, N = 3, 64, 64
    sizes = [40, 0, 70]
    offs = np.cumsum(sizes)
    M = int(offs[-1])
    x0 = S.bf16_bits(S.normal_bf16((M, K), seed=9))
    qx, sx = O.cast_dim0(x0)
    x = O.f64_to_bf16_bits(O.dequant_bf16(qx, sx))                   # an exact MX tensor
    w = S.bf16_bits(S.normal_bf16((E, N, K), 0.1, seed=10))
    dy = S.bf16_bits(S.normal_bf16((M, N), 0.1, seed=11))
    y, _ = O.ep_expert_forward(x, w, offs, E)
    cap = O.padded_rows_capacity(M, E)
    q, s = O.cast_dim0_grouped(x, offs, cap)
    qw, st = O.cast_32x32(w)
    np.testing.assert_array_equal(y, O.grouped_mm_m(O.dequant(q, s), O.dequant(qw, O.w32_scale_views(st)[0]), offs))
    _, _, dw, _ = O.ep_expert_backward(x, w, dy, offs, E)
    qa, sa = O.cast_dim1_grouped(dy, offs, cap)
    qb, sb = O.cast_dim1_grouped(x, offs, cap)
    np.testing.assert_array_equal(dw, O.grouped_mm_k(O.dequant(qa, sa), O.dequant(qb, sb), offs))
