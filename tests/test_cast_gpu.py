"""Bit-exact parity of the CUDA casts with the CPU oracle.

Every comparison is on E4M3 code bytes and blocked E8M0 scale bytes (pad bytes
included). Inputs come from the seeded generators; expected values come from
``oracle/`` only.
"""
import numpy as np
import pytest
import torch

from oracle import mx_oracle as O
from mxfp8_block_scaled_cast_b200 import synthetic as S

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mx():
    from mxfp8_block_scaled_cast_b200 import mx as _mx
    _mx.lib()
    return _mx


def _np(t):
    return t.cpu().numpy()


def _dev(t):
    return t.to("cuda")


def _check_dim0(mx, xb):
    q, s = mx.cast_dim0(_dev(xb))
    eq, es = O.cast_dim0(S.bf16_bits(xb))
    assert np.array_equal(_np(q), eq)
    assert np.array_equal(_np(s), O.swizzle(es))


def _check_dim1(mx, xb):
    qt, st = mx.cast_dim1(_dev(xb))
    eq, es = O.cast_dim1(S.bf16_bits(xb))
    assert np.array_equal(_np(qt), eq)
    assert np.array_equal(_np(st), O.swizzle(es))


# ------------------------------------------------------------- dim0/dim1 ---
def test_tiny_config_all_casts(mx):
    a = S.tiny_activation(0)
    _check_dim0(mx, a)
    _check_dim1(mx, a)
    q, sf, qt, sd = mx.cast_w32x32(_dev(a))
    eq, st = O.cast_32x32(S.bf16_bits(a))
    e_fwd, e_dgrad = O.w32_scale_views(st)
    assert np.array_equal(_np(q), eq) and np.array_equal(_np(qt), eq.T)
    assert np.array_equal(_np(sf), O.swizzle(e_fwd)) and np.array_equal(_np(sd), O.swizzle(e_dgrad))


@pytest.mark.parametrize("R,C", [(128, 128), (96, 64), (256, 576), (384, 160), (32, 32), (1, 32), (130, 96)])
def test_dim0_shapes(mx, R, C):
    _check_dim0(mx, S.sweep_tensor((R, C), seed=R + C))


@pytest.mark.parametrize("R,C", [(128, 128), (96, 64), (256, 576), (384, 160), (32, 32), (160, 96)])
def test_dim1_shapes(mx, R, C):
    _check_dim1(mx, S.sweep_tensor((R, C), seed=R * 7 + C))


def test_empty_rows(mx):
    x = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    q, s = mx.cast_dim0(x)
    assert q.numel() == 0 and s.numel() == 0
    qt, st = mx.cast_dim1(x)
    assert qt.numel() == 0


def _exhaustive_blocks():
    """Blocks that run every finite bf16 amax and every bf16 element value.

    Part 1: one block per non-negative finite amax pattern; its other 31
    elements are drawn below the amax (with signs, zeros, subnormals).
    Part 2: for amax in {448 * 2^k} and a subnormal amax, blocks holding every
    bf16 value of magnitude <= amax (both signs), 31 per block behind the amax.
    """
    rng = np.random.default_rng(0)
    allb = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = allb[((allb >> 7) & 0xFF) != 0xFF]
    pos = finite[finite < 0x8000]
    blocks = []
    for a in pos:
        others = rng.integers(0, int(a) + 1, 31).astype(np.uint16)
        others |= (rng.integers(0, 2, 31).astype(np.uint16) << 15)
        blocks.append(np.concatenate([[a], others]).astype(np.uint16))
    for amax_bits in (0x43E0, 0x3BE0, 0x4BE0, 0x5FE0, 0x00FF, 0x0080, 0x7F7F, 0x0001):
        vals = finite[(finite & 0x7FFF) <= amax_bits]
        vals = np.concatenate([vals, np.zeros((-len(vals)) % 31, np.uint16)])
        for chunk in vals.reshape(-1, 31):
            blocks.append(np.concatenate([[amax_bits], chunk]).astype(np.uint16))
    blocks = np.stack(blocks)
    blocks = np.concatenate([blocks, np.zeros(((-len(blocks)) % 256, 32), np.uint16)])
    return blocks.reshape(-1, 32 * 32)           # rows of 32 blocks


def test_exhaustive_single_blocks_dim0_and_dim1(mx):
    bits = _exhaustive_blocks()
    xb = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    _check_dim0(mx, xb)
    # the same blocks down the columns
    xt = torch.from_numpy(np.ascontiguousarray(bits.reshape(-1, 32).T.reshape(32, -1)).view(np.int16))
    xt = xt.view(torch.bfloat16)
    _check_dim1(mx, xt)


# ---------------------------------------------------------------- fused ----
@pytest.mark.parametrize("R,C", [(256, 256), (16384 // 16, 576), (96, 160)])
def test_fused_2d_equals_oracle_and_split(mx, R, C):
    xb = S.sweep_tensor((R, C), seed=11)
    q, s, qt, st = mx.cast_2d(_dev(xb))
    (eq, es), (eqt, est) = O.cast_2d(S.bf16_bits(xb))
    assert np.array_equal(_np(q), eq) and np.array_equal(_np(s), O.swizzle(es))
    assert np.array_equal(_np(qt), eqt) and np.array_equal(_np(st), O.swizzle(est))
    q0, s0 = mx.cast_dim0(_dev(xb))
    q1, s1 = mx.cast_dim1(_dev(xb))
    for u, v in ((q, q0), (s, s0), (qt, q1), (st, s1)):
        assert torch.equal(u, v)


def test_fused_2d_outputs_only_16_byte_aligned(mx):
    """Code buffers at a 16-byte (not 32-byte) offset take the 128-bit store path."""
    R, C = 160, 288
    xb = S.sweep_tensor((R, C), seed=12)
    raw_q = torch.zeros(R * C + 16, dtype=torch.uint8, device="cuda")
    raw_qt = torch.zeros(R * C + 16, dtype=torch.uint8, device="cuda")
    q, qt = raw_q[16:].view(R, C), raw_qt[16:].view(C, R)
    assert q.data_ptr() % 32 == 16 and qt.data_ptr() % 32 == 16
    s = torch.empty(mx.mx_scale_bytes(R, C // 32), dtype=torch.uint8, device="cuda")
    st = torch.empty(mx.mx_scale_bytes(C, R // 32), dtype=torch.uint8, device="cuda")
    mx.mx_cast_2d(_dev(xb), q, s, qt, st)
    (eq, es), (eqt, est) = O.cast_2d(S.bf16_bits(xb))
    assert np.array_equal(_np(q), eq) and np.array_equal(_np(s), O.swizzle(es))
    assert np.array_equal(_np(qt), eqt) and np.array_equal(_np(st), O.swizzle(est))
    assert not raw_q[:16].any() and not raw_qt[:16].any()


def test_unaligned_576_grad_full(mx):
    """The 576-wide gradient (18 scale columns padded to 20) at its full size."""
    xb = S.normal_bf16((16384, 576), 1.0, seed=0)
    q, s, qt, st = mx.cast_2d(_dev(xb))
    (eq, es), (eqt, est) = O.cast_2d(S.bf16_bits(xb))
    assert s.numel() == 16384 * 20
    assert np.array_equal(_np(q), eq) and np.array_equal(_np(s), O.swizzle(es))
    assert np.array_equal(_np(qt), eqt) and np.array_equal(_np(st), O.swizzle(est))


# ---------------------------------------------------------------- 32x32 ----
@pytest.mark.parametrize("G,N,K", [(1, 256, 256), (3, 96, 160), (2, 128, 576), (1, 32, 32)])
def test_w32x32_stack(mx, G, N, K):
    wb = S.sweep_tensor((G, N, K), seed=G * N + K)
    q, sf, qt, sd = mx.cast_w32x32(_dev(wb))
    eq, st = O.cast_32x32(S.bf16_bits(wb))
    e_fwd, e_dgrad = O.w32_scale_views(st)
    assert np.array_equal(_np(q), eq)
    assert np.array_equal(_np(qt), np.ascontiguousarray(np.swapaxes(eq, 1, 2)))
    assert np.array_equal(_np(sf), O.swizzle_stack(e_fwd))
    assert np.array_equal(_np(sd), O.swizzle_stack(e_dgrad))
    q2, sf2, qt2, sd2 = mx.cast_w32x32(_dev(wb), transposed=False)
    assert torch.equal(q2, q) and torch.equal(sf2, sf) and qt2 is None


# ------------------------------------------------------------- pad path ----
def _grouped_case(sizes, K, seed):
    M = int(np.sum(sizes))
    xb = S.normal_bf16((M, K), 1.0, seed=seed)
    offs = S.offsets_from_sizes(sizes)
    return xb, offs


@pytest.mark.parametrize("sizes,K", [
    ([128, 128], 256),                       # the tiny config's offs=[128, 256]
    ([100, 0, 250, 1, 0, 37], 96),           # ragged + empty groups
    ([0, 0, 300], 64),                       # leading empties
    ([1000, 3000, 96], 576),                 # 576-wide pad path
])
def test_grouped_casts(mx, sizes, K):
    xb, offs = _grouped_case(sizes, K, seed=len(sizes) + K)
    M, G = xb.shape[0], len(sizes)
    cap = mx.mx_padded_rows_capacity(M, G)
    q, s, qt, st = mx.cast_2d_grouped(_dev(xb), _dev(offs), cap)
    bits = S.bf16_bits(xb)
    eq, es = O.cast_dim0_grouped(bits, offs.numpy(), cap)
    eqt, est = O.cast_dim1_grouped(bits, offs.numpy(), cap)
    assert np.array_equal(_np(q), eq) and np.array_equal(_np(s), O.swizzle(es))
    assert np.array_equal(_np(qt), eqt) and np.array_equal(_np(st), O.swizzle(est))
    q0, s0 = mx.cast_dim0_grouped(_dev(xb), _dev(offs), cap)
    q1, s1 = mx.cast_dim1_grouped(_dev(xb), _dev(offs), cap)
    for u, v in ((q, q0), (s, s0), (qt, q1), (st, s1)):
        assert torch.equal(u, v)


def test_grouped_zipf_unaligned_groups(mx):
    sizes = S.zipf_group_sizes(32, 8192, 1.2, 3, 0)
    xb, offs = _grouped_case(sizes, 128, seed=3)
    cap = mx.mx_padded_rows_capacity(8192, 32)
    q, s, qt, st = mx.cast_2d_grouped(_dev(xb), _dev(offs), cap)
    bits = S.bf16_bits(xb)
    eq, es = O.cast_dim0_grouped(bits, offs.numpy(), cap)
    eqt, est = O.cast_dim1_grouped(bits, offs.numpy(), cap)
    assert np.array_equal(_np(q), eq) and np.array_equal(_np(s), O.swizzle(es))
    assert np.array_equal(_np(qt), eqt) and np.array_equal(_np(st), O.swizzle(est))


def test_invalid_offsets_flag_device_error(mx):
    xb = S.normal_bf16((256, 64), seed=1).cuda()
    bad = torch.tensor([200, 100, 256], dtype=torch.int32, device="cuda")    # decreasing
    q, s = mx.cast_dim0_grouped(xb, bad, 512)
    with pytest.raises(mx.MXError) as e:
        mx.mx_device_error()
    assert e.value.status == 6
    assert not q.any()                     # every tile became padding
    short = torch.tensor([100, 200], dtype=torch.int32, device="cuda")       # does not reach M
    mx.cast_dim0_grouped(xb, short, 512)
    with pytest.raises(mx.MXError):
        mx.mx_device_error()
    mx.cast_dim0_grouped(xb, torch.tensor([256], dtype=torch.int32, device="cuda"), 256)
    mx.mx_device_error()                   # clean again


def test_host_argument_errors(mx):
    x = torch.zeros(64, 48, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mx.MXError) as e:
        mx.cast_dim0(x)                    # 48 is not a multiple of 32
    assert e.value.status == 3
    x = torch.zeros(48, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mx.MXError):
        mx.cast_dim1(x)                    # columnwise blocks need R % 32 == 0
    base = torch.zeros(64 * 64 + 8, dtype=torch.bfloat16, device="cuda")
    mis = base[1:1 + 64 * 64].view(64, 64)
    q = torch.empty(64, 64, dtype=torch.uint8, device="cuda")
    s = torch.empty(mx.mx_scale_bytes(64, 2), dtype=torch.uint8, device="cuda")
    with pytest.raises(mx.MXError) as e:
        mx.mx_cast_dim0(mis, q, s)
    assert e.value.status == 2


# ------------------------------------------------------- full-size sampled --
def _sample_rows_check_dim0(q, s, xb_dev, C, rows):
    idx = torch.as_tensor(rows, device=xb_dev.device)
    x_rows = S.bf16_bits(xb_dev[idx])
    eq, es = O.cast_dim0(x_rows)
    assert np.array_equal(_np(q[idx]), eq)
    sb = _np(s)
    rr, cc = np.meshgrid(rows, np.arange(C // 32), indexing="ij")
    assert np.array_equal(sb[O.blocked_offset(rr, cc, C // 32)], es)


@pytest.mark.parametrize("n", [8192, 16384])
def test_square_sweep_full_size_sampled(mx, n):
    """Full-size sweep tensors in the launch configuration the benchmark times."""
    xb = S.sweep_tensor((n, n), seed=5, device="cuda")
    rng = np.random.default_rng(n)
    q, s, qt, st = mx.cast_2d(xb)
    rows = np.sort(rng.choice(n, 24, replace=False))
    _sample_rows_check_dim0(q, s, xb, n, rows)
    # columnwise: sampled 32-row bands, all columns
    for band in rng.choice(n // 32, 2, replace=False):
        eqt, est = O.cast_dim1(S.bf16_bits(xb[band * 32:(band + 1) * 32]))
        assert np.array_equal(_np(qt[:, band * 32:(band + 1) * 32]), eqt)
        stb = _np(st)
        cc = np.arange(n)
        assert np.array_equal(stb[O.blocked_offset(cc, np.full(n, band), n // 32)], est[:, 0])
    q0, s0 = mx.cast_dim0(xb)
    assert torch.equal(q0, q) and torch.equal(s0, s)
    del q, s, qt, st, q0, s0
    q1, s1 = mx.cast_dim1(xb)
    band = int(rng.integers(n // 32))
    eqt, _ = O.cast_dim1(S.bf16_bits(xb[band * 32:(band + 1) * 32]))
    assert np.array_equal(_np(q1[:, band * 32:(band + 1) * 32]), eqt)


@pytest.mark.parametrize("n", [1024, 4096, 8192, 16384])
def test_sweep_every_mode_in_the_benchmark_launch(mx, n):
    """Every mode of the bandwidth sweep at every square size, in the launch the
    benchmark times: dim0 rows and dim1 32-row bands against the oracle (all of
    them at 1024^2, sampled above), the fused cast bitwise equal to the two, and
    sampled 32x32 tiles of the weight cast with both of its scale views."""
    xb = S.sweep_tensor((n, n), seed=11, device="cuda")
    rng = np.random.default_rng(n + 1)
    full = n <= 1024
    q0, s0 = mx.cast_dim0(xb)
    rows = np.arange(n) if full else np.sort(rng.choice(n, 16, replace=False))
    _sample_rows_check_dim0(q0, s0, xb, n, rows)
    q1, s1 = mx.cast_dim1(xb)
    s1b, cc = _np(s1), np.arange(n)
    for band in (range(n // 32) if full else rng.choice(n // 32, 2, replace=False)):
        eqt, est = O.cast_dim1(S.bf16_bits(xb[band * 32:(band + 1) * 32]))
        assert np.array_equal(_np(q1[:, band * 32:(band + 1) * 32]), eqt), f"dim1 band {band}"
        assert np.array_equal(s1b[O.blocked_offset(cc, np.full(n, band), n // 32)], est[:, 0])
    q, s, qt, st = mx.cast_2d(xb)
    assert torch.equal(q, q0) and torch.equal(s, s0) and torch.equal(qt, q1) and torch.equal(st, s1)
    del q, s, qt, st, q0, s0, q1, s1
    wq, wsf, wqt, wsd = mx.cast_w32x32(xb)
    sfb, sdb = _np(wsf), _np(wsd)
    for _ in range(16):
        i, j = int(rng.integers(n // 32)), int(rng.integers(n // 32))
        eq, st32 = O.cast_32x32(S.bf16_bits(xb[32 * i:32 * i + 32, 32 * j:32 * j + 32]))
        assert np.array_equal(_np(wq[32 * i:32 * i + 32, 32 * j:32 * j + 32]), eq), f"32x32 tile {i},{j}"
        assert np.array_equal(_np(wqt[32 * j:32 * j + 32, 32 * i:32 * i + 32]), eq.T)
        idx = np.arange(32)
        assert np.all(sfb[O.blocked_offset(32 * i + idx, j, n // 32)] == st32[0, 0])
        assert np.all(sdb[O.blocked_offset(32 * j + idx, i, n // 32)] == st32[0, 0])


def test_expert_stack_full_size_sampled(mx):
    """[64, 2048, 7168] expert weight stack, 32x32 cast, sampled tiles."""
    G, N, K = 64, 2048, 7168
    wb = S.sweep_tensor((G, N, K), seed=7, device="cuda")
    q, sf, qt, sd = mx.cast_w32x32(wb)
    rng = np.random.default_rng(0)
    sfb, sdb = _np(sf), _np(sd)
    per_f, per_d = mx.mx_scale_bytes(N, K // 32), mx.mx_scale_bytes(K, N // 32)
    for _ in range(12):
        g, i, j = int(rng.integers(G)), int(rng.integers(N // 32)), int(rng.integers(K // 32))
        tile = S.bf16_bits(wb[g, 32 * i:32 * i + 32, 32 * j:32 * j + 32])
        eq, st = O.cast_32x32(tile)
        assert np.array_equal(_np(q[g, 32 * i:32 * i + 32, 32 * j:32 * j + 32]), eq)
        assert np.array_equal(_np(qt[g, 32 * j:32 * j + 32, 32 * i:32 * i + 32]), eq.T)
        n_idx = 32 * i + np.arange(32)
        k_idx = 32 * j + np.arange(32)
        assert np.all(sfb[g * per_f + O.blocked_offset(n_idx, j, K // 32)] == st[0, 0])
        assert np.all(sdb[g * per_d + O.blocked_offset(k_idx, i, N // 32)] == st[0, 0])


# ------------------------------------------------------------- FLOOR rule --
@pytest.mark.parametrize("R,C", [(256, 256), (96, 160), (16384 // 16, 576)])
def test_floor_casts_match_oracle(mx, R, C):
    xb = S.sweep_tensor((R, C), seed=R + 3 * C)
    q, s, qt, st = mx.cast_floor(_dev(xb), dims=3)
    (eq, es), (eqt, est) = O.cast_2d(S.bf16_bits(xb), rule="floor")
    assert np.array_equal(_np(q), eq) and np.array_equal(_np(s), O.swizzle(es))
    assert np.array_equal(_np(qt), eqt) and np.array_equal(_np(st), O.swizzle(est))
    q0, s0, _, _ = mx.cast_floor(_dev(xb), dims=1)
    _, _, q1, s1 = mx.cast_floor(_dev(xb), dims=2)
    for u, v in ((q, q0), (s, s0), (qt, q1), (st, s1)):
        assert torch.equal(u, v)


def test_floor_exhaustive_blocks_and_saturation(mx):
    bits = _exhaustive_blocks()
    xb = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    q, s, _, _ = mx.cast_floor(_dev(xb), dims=1)
    eq, es = O.cast_dim0(bits, rule="floor")
    assert np.array_equal(_np(q), eq) and np.array_equal(_np(s), O.swizzle(es))
    # the worked saturation block: 500 and -460 at scale 1 saturate to +-448
    blk = torch.zeros(32, 32, dtype=torch.float32)
    blk[0, :3] = torch.tensor([500.0, -460.0, 300.0])
    q, s, _, _ = mx.cast_floor(_dev(blk.to(torch.bfloat16)), dims=1)
    assert q[0, :3].tolist() == [0x7E, 0xFE, int(O.e4m3_encode(np.array([300.0]))[0])]
    rq, _ = mx.cast_dim0(_dev(blk.to(torch.bfloat16)))          # RCEIL: no saturation
    assert rq[0, 0].item() != 0x7E


def test_cast_ex_rceil_matches_plain_entries(mx):
    xb = _dev(S.sweep_tensor((128, 256), seed=4))
    R, C = xb.shape
    u8 = lambda *sh: torch.empty(*sh, dtype=torch.uint8, device="cuda")
    q, s = u8(R, C), u8(mx.mx_scale_bytes(R, C // 32))
    qt, st = u8(C, R), u8(mx.mx_scale_bytes(C, R // 32))
    mx.mx_cast_ex(xb, 3, mx.MX_RCEIL, q, s, qt, st)
    e = mx.cast_2d(xb)
    for u, v in zip((q, s, qt, st), e):
        assert torch.equal(u, v)
