"""Sizes past 2^31 elements: every offset the kernels form must be 64-bit.

* the fused rowwise + columnwise cast of a bf16 [40960, 53248] tensor
  (2.18e9 elements; torchtitan PR #5334, description: the fused
  rowwise/columnwise cast), checked bitwise against the oracle on sampled
  rows and 32-row column bands on both sides of element 2^31;
* the M-groups grouped GEMM (ao PR #4705, "MXFP8 MoE grouped-mm") with a
  [131104, 16384] bf16 output (2.15e9 elements), checked on sampled output
  rows on both sides of element 2^31 against the float64 oracle.

About 13 GB of device memory at the peak; released at the end of each test.
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


def test_fused_cast_past_2_31_elements(mx):
    R, C = 40960, 53248
    assert R * C > 2 ** 31
    xb = S.sweep_tensor((R, C), seed=21, device="cuda")
    q, s, qt, st = mx.cast_2d(xb)
    mx.mx_device_error()
    edge = 2 ** 31 // C                                 # the row holding element 2^31
    rng = np.random.default_rng(21)
    rows = np.unique(np.concatenate([[0, edge - 1, edge, edge + 1, R - 1], rng.choice(R, 6, replace=False)]))
    idx = torch.as_tensor(rows, device="cuda")
    eq, es = O.cast_dim0(S.bf16_bits(xb[idx]))
    assert np.array_equal(_np(q[idx]), eq), "rowwise codes"
    sb = _np(s)
    rr, cc = np.meshgrid(rows, np.arange(C // 32), indexing="ij")
    assert np.array_equal(sb[O.blocked_offset(rr, cc, C // 32)], es), "rowwise scales"
    del sb
    stb = _np(st)
    for band in (0, edge // 32, R // 32 - 1):
        eqt, est = O.cast_dim1(S.bf16_bits(xb[band * 32:(band + 1) * 32]))
        assert np.array_equal(_np(qt[:, band * 32:(band + 1) * 32]), eqt), f"columnwise codes, band {band}"
        cols = np.arange(C)
        assert np.array_equal(stb[O.blocked_offset(cols, np.full(C, band), R // 32)], est[:, 0]), \
            f"columnwise scales, band {band}"
    del xb, q, s, qt, st, stb
    torch.cuda.empty_cache()


def test_grouped_gemm_output_past_2_31_elements(mx):
    sizes = [70000, 61104]
    M, N, K = sum(sizes), 16384, 128
    assert M * N > 2 ** 31
    xb = S.normal_bf16((M, K), 1.0, seed=22, device="cuda")
    wb = S.normal_bf16((len(sizes), N, K), 0.02, seed=23, device="cuda")
    offs_t = S.offsets_from_sizes(sizes)
    cap = mx.mx_padded_rows_capacity(M, len(sizes))
    xq, xs = mx.cast_dim0_grouped(xb, offs_t.cuda(), cap)
    wq, wsf, _, _ = mx.cast_w32x32(wb, transposed=False)
    y = mx.grouped_mm(xq, xs, wq, wsf, offs_t.cuda(), M)
    mx.mx_device_error()
    edge = 2 ** 31 // N                                 # the output row holding element 2^31
    rng = np.random.default_rng(22)
    rows = np.unique(np.concatenate([[0, sizes[0] - 1, sizes[0], edge - 1, edge, edge + 1, M - 1],
                                     rng.choice(M, 6, replace=False)]))
    got = y[torch.as_tensor(rows, device="cuda")].float().cpu().numpy().astype(np.float64)
    # oracle: each sampled token row, cast rowwise, against its group's expert
    offs = offs_t.numpy()
    starts, ends = O.group_bounds(offs)
    qw, stile = O.cast_32x32(S.bf16_bits(wb.cpu()))
    s_fwd, _ = O.w32_scale_views(stile)
    b = O.dequant(qw, s_fwd)
    qx, sx = O.cast_dim0(S.bf16_bits(xb[torch.as_tensor(rows, device="cuda")]))
    a = O.dequant(qx, sx)
    g_of = np.searchsorted(np.asarray(ends), rows, side="right")
    ref = np.stack([O.mm(a[i:i + 1], b[g])[0] for i, g in enumerate(g_of)])
    absref = np.stack([O.mm(np.abs(a[i:i + 1]), np.abs(b[g]))[0] for i, g in enumerate(g_of)])
    bad = ~(np.abs(got - ref) <= O.gemm_bound(ref, absref))
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} sampled outputs outside tolerance"
    del xb, wb, xq, xs, wq, wsf, y
    torch.cuda.empty_cache()
