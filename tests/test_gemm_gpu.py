"""Parity of the tcgen05 MXFP8 grouped GEMM with the float64 oracle.

Tolerance (per element): |gpu - ref| <= 2^-7 |ref| + 1e-3 (|A| |B|^T), with
ref the float64 product of the oracle's own dequantized operands. The GPU
accumulates in fp32 and rounds to bf16, both well inside that bound. The
oracle never sees a GPU output: it quantizes the same seeded inputs itself.
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


def _assert_close(got, ref, absref, what=""):
    err = np.abs(got - ref)
    bound = O.gemm_bound(ref, absref)
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside tolerance, worst {np.max(err - bound)}"


def _oracle_fwd(xb, wb, offs, cap):
    qx, sx = O.cast_dim0_grouped(S.bf16_bits(xb), offs, cap)
    qw, st = O.cast_32x32(S.bf16_bits(wb))
    s_fwd, _ = O.w32_scale_views(st)
    a, b = O.dequant(qx, sx), O.dequant(qw, s_fwd)
    return O.grouped_mm_m(a, b, offs), O.grouped_mm_m(np.abs(a), np.abs(b), offs)


def _gpu_fwd(mx, xb, wb, offs_t, cap):
    q, s = mx.cast_dim0_grouped(xb.cuda(), offs_t.cuda(), cap)
    wq, wsf, _, _ = mx.cast_w32x32(wb.cuda(), transposed=False)
    return mx.grouped_mm(q, s, wq, wsf, offs_t.cuda(), xb.shape[0])


@pytest.mark.parametrize("case", ["tiny", "aligned", "ragged"])
def test_grouped_forward(mx, case):
    if case == "tiny":
        xb, wb, offs_t = S.tiny_problem(0)
    elif case == "aligned":
        xb = S.normal_bf16((1024, 512), seed=1)
        wb = S.normal_bf16((4, 768, 512), 0.02, seed=2)
        offs_t = S.offsets_from_sizes([256, 0, 512, 256])
    else:
        xb = S.normal_bf16((777, 384), seed=3)
        wb = S.normal_bf16((5, 512, 384), 0.02, seed=4)
        offs_t = S.offsets_from_sizes([100, 0, 250, 1, 426])
    M, G = xb.shape[0], wb.shape[0]
    cap = mx.mx_padded_rows_capacity(M, G)
    out = _gpu_fwd(mx, xb, wb, offs_t, cap)
    mx.mx_device_error()
    ref, absref = _oracle_fwd(xb, wb, offs_t.numpy(), cap)
    _assert_close(_f64(out), ref, absref, case)


def test_dense_single_group_and_determinism(mx):
    xb = S.normal_bf16((320, 640), seed=5)
    wb = S.normal_bf16((512, 640), 0.02, seed=6)
    q, s = mx.cast_dim0(xb.cuda())
    wq, wsf, _, _ = mx.cast_w32x32(wb.cuda(), transposed=False)
    out = mx.grouped_mm(q, s, wq, wsf, None, 320)
    out2 = mx.grouped_mm(q, s, wq, wsf, None, 320)
    assert torch.equal(out, out2)
    y, absy = O.linear_fwd(S.bf16_bits(xb), S.bf16_bits(wb))
    _assert_close(_f64(out), y, absy, "dense")


def test_grouped_dgrad(mx):
    """dX_g = dY_g W_g: dY cast along N (dim0, padded), W^T from the same 32x32 cast."""
    sizes = [130, 0, 384, 7]
    dyb = S.normal_bf16((sum(sizes), 512), 1e-2, seed=7)
    wb = S.normal_bf16((4, 512, 768), 0.02, seed=8)          # [G, N, K]
    offs_t = S.offsets_from_sizes(sizes)
    M, cap = dyb.shape[0], mx.mx_padded_rows_capacity(sum(sizes), 4)
    q, s = mx.cast_dim0_grouped(dyb.cuda(), offs_t.cuda(), cap)
    _, _, wqt, wsd = mx.cast_w32x32(wb.cuda())
    out = mx.grouped_mm(q, s, wqt, wsd, offs_t.cuda(), M)     # [M, K]
    qd, sd = O.cast_dim0_grouped(S.bf16_bits(dyb), offs_t.numpy(), cap)
    qw, st = O.cast_32x32(S.bf16_bits(wb))
    _, s_dg = O.w32_scale_views(st)
    a = O.dequant(qd, sd)
    b = O.dequant(np.ascontiguousarray(np.swapaxes(qw, 1, 2)), s_dg)
    _assert_close(_f64(out), O.grouped_mm_m(a, b, offs_t.numpy()),
                  O.grouped_mm_m(np.abs(a), np.abs(b), offs_t.numpy()), "dgrad")


@pytest.mark.parametrize("sizes,N,K", [([130, 0, 384, 7], 512, 768), ([300], 256, 1024), ([1, 600], 1024, 256)])
def test_grouped_dgrad_from_forward_codes(mx, sizes, N, K):
    """The MN-major dgrad (B = the forward's 32x32 codes [G, N, K], no transposed
    copy) against the oracle, and bitwise against the K-major dgrad on W^T codes."""
    G = len(sizes)
    dyb = S.normal_bf16((sum(sizes), N), 1e-2, seed=N + K)
    wb = S.normal_bf16((G, N, K), 0.02, seed=G + 3)           # [G, N, K]
    offs_t = S.offsets_from_sizes(sizes)
    M, cap = dyb.shape[0], mx.mx_padded_rows_capacity(sum(sizes), G)
    q, s = mx.cast_dim0_grouped(dyb.cuda(), offs_t.cuda(), cap)
    wq, _, wqt, wsd = mx.cast_w32x32(wb.cuda())
    out = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    mx.mx_grouped_mm(q, s, wq, wsd, offs_t.cuda(), G, mx.MX_GROUPS_M_KN, out, M, K, N, cap)
    ref_km = mx.grouped_mm(q, s, wqt, wsd, offs_t.cuda(), M)
    mx.mx_device_error()
    assert torch.equal(out, ref_km)
    qd, sd = O.cast_dim0_grouped(S.bf16_bits(dyb), offs_t.numpy(), cap)
    qw, st = O.cast_32x32(S.bf16_bits(wb))
    _, s_dg = O.w32_scale_views(st)
    a = O.dequant(qd, sd)
    b = O.dequant(np.ascontiguousarray(np.swapaxes(qw, 1, 2)), s_dg)
    _assert_close(_f64(out), O.grouped_mm_m(a, b, offs_t.numpy()),
                  O.grouped_mm_m(np.abs(a), np.abs(b), offs_t.numpy()), "dgrad (MN-major B)")


@pytest.mark.parametrize("sizes", [[256, 128], [100, 0, 250, 1, 37], [0, 0, 300]])
def test_grouped_wgrad_k_groups(mx, sizes):
    """dW_g = dY_g^T X_g over each group's tokens; empty groups are exact zeros."""
    M, G = sum(sizes), len(sizes)
    dyb = S.normal_bf16((M, 512), 1e-2, seed=9)
    xb = S.normal_bf16((M, 512), 1.0, seed=10)
    offs_t = S.offsets_from_sizes(sizes)
    cap = mx.mx_padded_rows_capacity(M, G)
    dqt, dst = mx.cast_dim1_grouped(dyb.cuda(), offs_t.cuda(), cap)
    xqt, xst = mx.cast_dim1_grouped(xb.cuda(), offs_t.cuda(), cap)
    out = mx.grouped_mm_wgrad(dqt, dst, xqt, xst, offs_t.cuda(), M)
    mx.mx_device_error()
    oq, os_ = O.cast_dim1_grouped(S.bf16_bits(dyb), offs_t.numpy(), cap)
    xq, xs = O.cast_dim1_grouped(S.bf16_bits(xb), offs_t.numpy(), cap)
    a, b = O.dequant(oq, os_), O.dequant(xq, xs)
    ref = O.grouped_mm_k(a, b, offs_t.numpy())
    absref = O.grouped_mm_k(np.abs(a), np.abs(b), offs_t.numpy())
    got = _f64(out)
    _assert_close(got, ref, absref, "wgrad")
    for g, n in enumerate(sizes):
        if n == 0:
            assert not out[g].any()


def test_dense_wgrad(mx):
    dyb = S.normal_bf16((640, 256), 1e-2, seed=11)
    xb = S.normal_bf16((640, 512), 1.0, seed=12)
    dqt, dst = mx.cast_dim1(dyb.cuda())
    xqt, xst = mx.cast_dim1(xb.cuda())
    out = mx.grouped_mm_wgrad(dqt, dst, xqt, xst, None, 640)
    ref, absref = O.linear_wgrad(S.bf16_bits(dyb), S.bf16_bits(xb))
    _assert_close(_f64(out[0]), ref, absref, "dense wgrad")


def test_moe_shape_reduced_full_compare(mx):
    """The MoE workload's structure (G=8, Dirichlet group sizes) at M=2048, K=N=1024."""
    xb, wb, dyb, offs_t = S.moe_problem(G=8, M=2048, N=1024, K=1024, seed=0)
    cap = mx.mx_padded_rows_capacity(2048, 8)
    out = _gpu_fwd(mx, xb, wb, offs_t, cap)
    ref, absref = _oracle_fwd(xb, wb, offs_t.numpy(), cap)
    _assert_close(_f64(out), ref, absref, "moe reduced")


def _sampled_fwd_check(mx, xb, wb, offs_t, out, n_samples, rng):
    """Checks sampled output entries against the oracle, one row/column at a time."""
    M, K = xb.shape
    G, N, _ = wb.shape
    ends = offs_t.cpu().numpy().astype(np.int64)
    rows = rng.choice(M, n_samples)
    cols = rng.choice(N, n_samples)
    outc = out.float().cpu().numpy()
    for i, j in zip(rows, cols):
        g = int(np.searchsorted(ends, i, side="right"))
        qx, sx = O.cast_dim0(S.bf16_bits(xb[i:i + 1]))
        n0 = (j // 32) * 32
        qw, st = O.cast_32x32(S.bf16_bits(wb[g, n0:n0 + 32]))
        s_fwd, _ = O.w32_scale_views(st)
        a = O.dequant(qx, sx)[0]
        b = O.dequant(qw, s_fwd)[j - n0]
        ref, absref = float(a @ b), float(np.abs(a) @ np.abs(b))
        assert abs(outc[i, j] - ref) <= 2 ** -7 * abs(ref) + 1e-3 * absref, (i, j, outc[i, j], ref)


def test_moe_full_size_sampled(mx):
    """G=8, K=N=4096, M=16384 in the benchmark's launch configuration, sampled outputs."""
    xb, wb, dyb, offs_t = S.moe_problem(seed=0, device="cuda")
    offs_d = offs_t.cuda()
    cap = mx.mx_padded_rows_capacity(16384, 8)
    q, s = mx.cast_dim0_grouped(xb, offs_d, cap)
    wq, wsf, _, _ = mx.cast_w32x32(wb, transposed=False)
    out = mx.grouped_mm(q, s, wq, wsf, offs_d, 16384)
    out2 = mx.grouped_mm(q, s, wq, wsf, offs_d, 16384)
    assert torch.equal(out, out2)
    mx.mx_device_error()
    _sampled_fwd_check(mx, xb, wb, offs_t, out, 256, np.random.default_rng(0))


def test_skewed_full_size_sampled(mx):
    """G=32, K=7168, N=2048, M=32768 with Zipf sizes and 3 empty groups (pad path)."""
    xb, wb, dyb, offs_t = S.unaligned_grouped_problem(device="cuda")
    offs_d = offs_t.cuda()
    cap = mx.mx_padded_rows_capacity(32768, 32)
    q, s = mx.cast_dim0_grouped(xb, offs_d, cap)
    wq, wsf, _, _ = mx.cast_w32x32(wb, transposed=False)
    out = mx.grouped_mm(q, s, wq, wsf, offs_d, 32768)
    mx.mx_device_error()
    _sampled_fwd_check(mx, xb, wb, offs_t, out, 192, np.random.default_rng(1))
    # wgrad on the same groups, sampled (n, k) entries of sampled groups
    dqt, dst = mx.cast_dim1_grouped(dyb, offs_d, cap)
    xqt, xst = mx.cast_dim1_grouped(xb, offs_d, cap)
    dw = mx.grouped_mm_wgrad(dqt, dst, xqt, xst, offs_d, 32768)
    mx.mx_device_error()
    ends = offs_t.numpy().astype(np.int64)
    starts = np.concatenate([[0], ends[:-1]])
    rng = np.random.default_rng(2)
    for g in rng.choice(32, 6, replace=False):
        if ends[g] == starts[g]:
            assert not dw[g].any()
            continue
        n = int(rng.integers(2048 // 32)) * 32
        k = int(rng.integers(7168 // 32)) * 32
        dy_g = S.bf16_bits(dyb[starts[g]:ends[g], n:n + 32])
        x_g = S.bf16_bits(xb[starts[g]:ends[g], k:k + 32])
        off1 = np.array([ends[g] - starts[g]])
        c = O.padded_rows_capacity(int(off1[0]), 1)
        qa, sa = O.cast_dim1_grouped(dy_g, off1, c)
        qb, sb = O.cast_dim1_grouped(x_g, off1, c)
        a, b = O.dequant(qa, sa), O.dequant(qb, sb)
        ref, absref = O.mm(a, b), O.mm(np.abs(a), np.abs(b))
        _assert_close(_f64(dw[g, n:n + 32, k:k + 32]), ref, absref, f"wgrad g={g}")


def test_skewed_dgrad_from_forward_codes_full_size_sampled(mx):
    """G=32, K=7168, N=2048, M=32768 (Zipf groups, 3 empty): the MXFP8 dgrad with the
    weight's forward codes read MN-major, sampled 32-column slices of sampled rows."""
    xb, wb, dyb, offs_t = S.unaligned_grouped_problem(device="cuda")    # w [G, N=2048, K=7168]
    offs_d = offs_t.cuda()
    G, N, K = wb.shape
    M = dyb.shape[0]
    cap = mx.mx_padded_rows_capacity(M, G)
    dq, ds = mx.cast_dim0_grouped(dyb, offs_d, cap)
    wq, _, _, wsd = mx.cast_w32x32(wb, transposed=False, dgrad_scales=True)
    dx = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    mx.mx_grouped_mm(dq, ds, wq, wsd, offs_d, G, mx.MX_GROUPS_M_KN, dx, M, K, N, cap)
    mx.mx_device_error()
    ends = offs_t.numpy().astype(np.int64)
    rng = np.random.default_rng(4)
    dxc = _f64(dx)
    for r in rng.choice(M, 24, replace=False):
        g = int(np.searchsorted(ends, r, side="right"))
        qd, sd = O.cast_dim0(S.bf16_bits(dyb[r:r + 1]))
        a = O.dequant(qd, sd)                                            # [1, N]
        k0 = int(rng.integers(K // 32)) * 32
        qw, st = O.cast_32x32(S.bf16_bits(wb[g][:, k0:k0 + 32]))         # [N, 32]
        _, s_dg = O.w32_scale_views(st)
        bt = O.dequant(np.ascontiguousarray(qw.T), s_dg)                 # W^T [32, N]
        _assert_close(dxc[r:r + 1, k0:k0 + 32], O.mm(a, bt), O.mm(np.abs(a), np.abs(bt)), f"dgrad row {r}")
