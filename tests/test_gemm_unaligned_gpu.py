"""The GEMMs at sizes that are not multiples of the tile: the pad path.

torchtitan PR #5334 (description and review thread) names the 576-wide
output gradient of the KV-A projection as the case that needs a path for
geometry that is not 128-aligned. Here every size only has to be a multiple
of 32 (the scale block): operand tiles past the tensor are read as zero codes
with zero scale bytes, and output rows and columns past the tensor are never
written. Each case runs the GEMM into an output filled with NaN and checks
every element against the float64 oracle (tolerance 2^-7 |ref| + 1e-3
(|A| |B|^T)); an element left unwritten stays NaN and fails.
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


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def _assert_close(got, ref, absref, what):
    assert got.shape == ref.shape, (got.shape, ref.shape)
    err = np.abs(got - ref)
    bound = O.gemm_bound(ref, absref)
    bad = ~(err <= bound)                      # NaN (an unwritten element) counts as bad
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} outside tolerance"


def _nan(*shape):
    return torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")


@pytest.mark.parametrize("sizes,N,K", [
    ([100, 0, 333], 576, 576),        # N and K both ragged (576 = 2 x 256 + 64 = 4 x 128 + 64)
    ([300, 45], 96, 96),              # smaller than one tile in N and one K step
    ([257], 576, 128),                # ragged N only
    ([128, 1, 200], 512, 160),        # ragged K only
    ([300, 45], 64, 160),             # every tile 64 columns wide (run at MMA N = 128)
    ([200, 0, 77], 320, 96),          # 256 + 64 columns
    ([130], 32, 64),                  # one 32-column tile
])
def test_forward_m_groups_ragged(mx, sizes, N, K):
    M, G = sum(sizes), len(sizes)
    xb = S.normal_bf16((M, K), seed=N + K)
    wb = S.normal_bf16((G, N, K), 0.02, seed=M)
    offs_t = S.offsets_from_sizes(sizes)
    cap = mx.mx_padded_rows_capacity(M, G)
    q, s = mx.cast_dim0_grouped(xb.cuda(), offs_t.cuda(), cap)
    wq, wsf, _, _ = mx.cast_w32x32(wb.cuda(), transposed=False)
    out = _nan(M, N)
    mx.mx_grouped_mm(q, s, wq, wsf, offs_t.cuda(), G, mx.MX_GROUPS_M, out, M, N, K, cap)
    mx.mx_device_error()
    qx, sx = O.cast_dim0_grouped(S.bf16_bits(xb), offs_t.numpy(), cap)
    qw, st = O.cast_32x32(S.bf16_bits(wb))
    a, b = O.dequant(qx, sx), O.dequant(qw, O.w32_scale_views(st)[0])
    of = offs_t.numpy()
    _assert_close(_f64(out), O.grouped_mm_m(a, b, of), O.grouped_mm_m(np.abs(a), np.abs(b), of), "forward")


@pytest.mark.parametrize("sizes,Nw,Kw", [
    ([100, 0, 333], 576, 576),        # contraction over 576 (the 576-wide gradient's dgrad)
    ([70, 190], 96, 352),
    ([300], 256, 96),                 # ragged dgrad output width
])
def test_dgrad_from_forward_codes_ragged(mx, sizes, Nw, Kw):
    """dX = dY W with W [G, Nw, Kw] read MN-major from the forward's 32x32 codes:
    the contraction is Nw, the output width Kw."""
    M, G = sum(sizes), len(sizes)
    dyb = S.normal_bf16((M, Nw), 1e-2, seed=Nw)
    wb = S.normal_bf16((G, Nw, Kw), 0.02, seed=Kw)
    offs_t = S.offsets_from_sizes(sizes)
    cap = mx.mx_padded_rows_capacity(M, G)
    q, s = mx.cast_dim0_grouped(dyb.cuda(), offs_t.cuda(), cap)
    wq, _, _, wsd = mx.cast_w32x32(wb.cuda(), transposed=False, dgrad_scales=True)
    out = _nan(M, Kw)
    mx.mx_grouped_mm(q, s, wq, wsd, offs_t.cuda(), G, mx.MX_GROUPS_M_KN, out, M, Kw, Nw, cap)
    mx.mx_device_error()
    qd, sd = O.cast_dim0_grouped(S.bf16_bits(dyb), offs_t.numpy(), cap)
    qw, st = O.cast_32x32(S.bf16_bits(wb))
    a = O.dequant(qd, sd)
    b = O.dequant(np.ascontiguousarray(np.swapaxes(qw, 1, 2)), O.w32_scale_views(st)[1])
    of = offs_t.numpy()
    _assert_close(_f64(out), O.grouped_mm_m(a, b, of), O.grouped_mm_m(np.abs(a), np.abs(b), of), "dgrad")


@pytest.mark.parametrize("sizes,N,K", [
    ([100, 0, 333], 576, 96),         # the 576-wide gradient's wgrad rows, a narrow K
    ([257, 31], 96, 576),
    ([0, 400], 544, 288),
    ([100, 200], 96, 64),             # output tiles 64 columns wide (run at MMA N = 128)
    ([257], 64, 32),
])
def test_wgrad_k_groups_ragged(mx, sizes, N, K):
    M, G = sum(sizes), len(sizes)
    dyb = S.normal_bf16((M, N), 1e-2, seed=N + 1)
    xb = S.normal_bf16((M, K), 1.0, seed=K + 1)
    offs_t = S.offsets_from_sizes(sizes)
    cap = mx.mx_padded_rows_capacity(M, G)
    dqt, dst = mx.cast_dim1_grouped(dyb.cuda(), offs_t.cuda(), cap)
    xqt, xst = mx.cast_dim1_grouped(xb.cuda(), offs_t.cuda(), cap)
    out = _nan(G, N, K)
    mx.mx_grouped_mm(dqt, dst, xqt, xst, offs_t.cuda(), G, mx.MX_GROUPS_K, out, M, N, K, cap)
    mx.mx_device_error()
    qa, sa = O.cast_dim1_grouped(S.bf16_bits(dyb), offs_t.numpy(), cap)
    qb, sb = O.cast_dim1_grouped(S.bf16_bits(xb), offs_t.numpy(), cap)
    a, b = O.dequant(qa, sa), O.dequant(qb, sb)
    of = offs_t.numpy()
    got = _f64(out)
    _assert_close(got, O.grouped_mm_k(a, b, of), O.grouped_mm_k(np.abs(a), np.abs(b), of), "wgrad")
    for g, n in enumerate(sizes):
        if n == 0:
            assert np.all(got[g] == 0.0)


@pytest.mark.parametrize("M,N,K", [(256, 576, 96), (512, 96, 576), (96, 576, 576)])
def test_linear_ragged_full_compare(mx, M, N, K):
    """The linear forward, dgrad and wgrad at N or K in {576, 96}, every element."""
    x, w, dy = S.linear_problem(M=M, N=N, K=K, seed=N + K)
    cache = mx.WeightCache()
    y = mx.linear_fwd(x.cuda(), w.cuda(), cache)
    dx, dw = mx.linear_bwd(dy.cuda(), x.cuda(), w.cuda(), cache)
    y2 = mx.linear_fwd(x.cuda(), w.cuda())
    mx.mx_device_error()
    assert torch.equal(y, y2)                                   # cache hit == miss, bitwise
    xb, wb, db = (S.bf16_bits(t) for t in (x, w, dy))
    _assert_close(_f64(y), *O.linear_fwd(xb, wb), "linear forward")
    _assert_close(_f64(dx), *O.linear_dgrad(db, wb), "linear dgrad")
    _assert_close(_f64(dw), *O.linear_wgrad(db, xb), "linear wgrad")
    cache.close()


@pytest.mark.parametrize("sizes,K,N", [([130, 0, 300], 96, 576), ([64, 200], 576, 96)])
def test_bf16_row_groups_ragged(mx, sizes, K, N):
    M, G = sum(sizes), len(sizes)
    a = S.normal_bf16((M, K), seed=K)
    b = S.normal_bf16((G, K, N), 0.05, seed=N)
    offs_t = S.offsets_from_sizes(sizes)
    out = _nan(M, N)
    mx.mx_grouped_mm_bf16(a.cuda(), b.cuda(), offs_t.cuda(), G, mx.MX_GROUPS_M, out, M, N, K)
    mx.mx_device_error()
    af, bf = O.bf16_to_f64(S.bf16_bits(a)), O.bf16_to_f64(S.bf16_bits(b))
    of = offs_t.numpy()
    _assert_close(_f64(out), O.hp_grouped_mm_m(af, bf, of), O.hp_grouped_mm_m(np.abs(af), np.abs(bf), of),
                  "bf16 row groups")


@pytest.mark.parametrize("sizes,N,K", [([1, 63, 0, 200], 576, 96), ([300], 96, 544)])
def test_bf16_token_groups_ragged(mx, sizes, N, K):
    M, G = sum(sizes), len(sizes)
    a = S.normal_bf16((M, N), seed=N + 3)
    b = S.normal_bf16((M, K), seed=K + 3)
    offs_t = S.offsets_from_sizes(sizes)
    out = _nan(G, N, K)
    mx.mx_grouped_mm_bf16(a.cuda(), b.cuda(), offs_t.cuda(), G, mx.MX_GROUPS_K, out, M, N, K)
    mx.mx_device_error()
    af, bf = O.bf16_to_f64(S.bf16_bits(a)), O.bf16_to_f64(S.bf16_bits(b))
    of = offs_t.numpy()
    _assert_close(_f64(out), O.hp_grouped_mm_k(af, bf, of), O.hp_grouped_mm_k(np.abs(af), np.abs(bf), of),
                  "bf16 token groups")


def test_sizes_not_a_multiple_of_32_are_rejected(mx):
    x = torch.zeros(64, 80, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(96, 80, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mx.MXError) as e:
        mx.linear_fwd(x, w)
    assert e.value.status == 3


def test_kva_gemms_full_size_sampled(mx):
    """The three GEMMs around the 576-wide gradient at the size bench.py times them
    (M=16384 tokens, N=576, K=7168; dense, as the linear runs them): sampled rows of
    the forward and dgrad (one in every 256-row tile, 32-column slabs in every
    256-column tile) and sampled 32-column slices of dW, against the oracle."""
    Mk, Nk, Kk = 16384, 576, 7168
    x, w, _ = S.linear_problem(Mk, Nk, Kk, seed=0, device="cuda")
    dy = S.sweep_tensor((Mk, Nk), seed=0, device="cuda")
    xq, xs, xqt, xst = mx.cast_2d(x)
    wq, wsf, _, wsd = mx.cast_w32x32(w, transposed=False, dgrad_scales=True)
    dq, ds, dqt, dst = mx.cast_2d(dy)
    y, dx, dw = _nan(Mk, Nk), _nan(Mk, Kk), _nan(Nk, Kk)
    mx.mx_grouped_mm(xq, xs, wq, wsf, None, 1, mx.MX_GROUPS_M, y, Mk, Nk, Kk, 0)
    mx.mx_grouped_mm(dq, ds, wq, wsd, None, 1, mx.MX_GROUPS_M_KN, dx, Mk, Kk, Nk, 0)
    mx.mx_grouped_mm(dqt, dst, xqt, xst, None, 1, mx.MX_GROUPS_K, dw, Mk, Nk, Kk, 0)
    mx.mx_device_error()
    rng = np.random.default_rng(5)
    rows = np.array([t * 256 + int(rng.integers(256)) for t in range(Mk // 256)] + [0, Mk - 1])
    xb, wb, db = S.bf16_bits(x), S.bf16_bits(w), S.bf16_bits(dy)
    # forward: rows x every 32-column slab of the 576 outputs (the third column tile is 64 wide)
    qx, sx = O.cast_dim0(xb[rows])
    qw, st = O.cast_32x32(wb)
    a, b = O.dequant(qx, sx), O.dequant(qw, O.w32_scale_views(st)[0])
    _assert_close(_f64(y[torch.as_tensor(rows, device="cuda")]), O.mm(a, b), O.mm(np.abs(a), np.abs(b)), "kva forward")
    # dgrad: contraction over the 576 (four full K steps and a half one), one slab per 256 columns
    qd, sd = O.cast_dim0(db[rows])
    ad = O.dequant(qd, sd)
    for t in range(Kk // 256):
        k0 = t * 256 + 32 * int(rng.integers(8))
        qws, sts = O.cast_32x32(wb[:, k0:k0 + 32])
        bt = O.dequant(np.ascontiguousarray(qws.T), O.w32_scale_views(sts)[1])
        got = _f64(dx[torch.as_tensor(rows, device="cuda")][:, k0:k0 + 32])
        _assert_close(got, O.mm(ad, bt), O.mm(np.abs(ad), np.abs(bt)), f"kva dgrad cols {k0}")
    # wgrad: all 576 rows of dW on sampled 32-column slices (the second row tile is half empty)
    qa, sa = O.cast_dim1(db)
    aw = O.dequant(qa, sa)                                                   # [576, Mk]
    for k0 in (0, 32 * int(rng.integers(1, Kk // 32 - 1)), Kk - 32):
        qb, sb = O.cast_dim1(xb[:, k0:k0 + 32])
        bw = O.dequant(qb, sb)
        _assert_close(_f64(dw[:, k0:k0 + 32]), O.mm(aw, bw), O.mm(np.abs(aw), np.abs(bw)), f"kva wgrad cols {k0}")
