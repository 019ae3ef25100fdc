"""The largest group count the grouped entry points take (G = 1024, most
groups empty or tiny), through the pad-path casts, both MXFP8 GEMM modes and
the bf16 GEMMs, against the oracle; G = 1025 is rejected on the host."""
import numpy as np
import pytest
import torch

from oracle import mx_oracle as O
from mxfp8_block_scaled_cast_b200 import synthetic as S

pytestmark = pytest.mark.gpu

G = 1024


@pytest.fixture(scope="module")
def mx():
    from mxfp8_block_scaled_cast_b200 import mx as _mx
    _mx.lib()
    return _mx


@pytest.fixture(scope="module")
def sizes():
    rng = np.random.default_rng(1024)
    s = np.zeros(G, dtype=np.int64)
    live = rng.choice(G, 40, replace=False)            # 40 non-empty groups, 984 empty
    s[live] = rng.integers(1, 90, size=live.size)
    s[live[0]] = 300                                    # one group spans several tiles
    return s


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def _close(got, ref, absref, what):
    bad = np.abs(got - ref) > O.gemm_bound(ref, absref)
    assert not bad.any(), f"{what}: {bad.sum()} outside tolerance"


def test_grouped_casts_at_1024_groups(mx, sizes):
    M, K = int(sizes.sum()), 128
    xb = S.normal_bf16((M, K), seed=3)
    offs_t = S.offsets_from_sizes(sizes)
    cap = mx.mx_padded_rows_capacity(M, G)
    q, s, qt, st = mx.cast_2d_grouped(xb.cuda(), offs_t.cuda(), cap)
    mx.mx_device_error()
    eq, es = O.cast_dim0_grouped(S.bf16_bits(xb), offs_t.numpy(), cap)
    eqt, est = O.cast_dim1_grouped(S.bf16_bits(xb), offs_t.numpy(), cap)
    assert np.array_equal(q.cpu().numpy(), eq) and np.array_equal(s.cpu().numpy(), O.swizzle(es))
    assert np.array_equal(qt.cpu().numpy(), eqt) and np.array_equal(st.cpu().numpy(), O.swizzle(est))


def test_mxfp8_grouped_gemms_at_1024_groups(mx, sizes):
    M, N, K = int(sizes.sum()), 256, 128
    xb = S.normal_bf16((M, K), seed=4)
    wb = S.normal_bf16((G, N, K), 0.05, seed=5)
    offs_t = S.offsets_from_sizes(sizes)
    offs = offs_t.numpy()
    cap = mx.mx_padded_rows_capacity(M, G)
    q, s = mx.cast_dim0_grouped(xb.cuda(), offs_t.cuda(), cap)
    wq, wsf, _, _ = mx.cast_w32x32(wb.cuda(), transposed=False)
    y = mx.grouped_mm(q, s, wq, wsf, offs_t.cuda(), M)
    mx.mx_device_error()
    qx, sx = O.cast_dim0_grouped(S.bf16_bits(xb), offs, cap)
    qw, st = O.cast_32x32(S.bf16_bits(wb))
    s_fwd, _ = O.w32_scale_views(st)
    a, b = O.dequant(qx, sx), O.dequant(qw, s_fwd)
    _close(_f64(y), O.grouped_mm_m(a, b, offs), O.grouped_mm_m(np.abs(a), np.abs(b), offs), "forward")
    # wgrad over the same 1024 token groups: dW[g] [256, 256], zeros for the empty groups
    dyb = S.normal_bf16((M, 256), 0.1, seed=6)
    x2 = S.normal_bf16((M, 256), seed=7)
    dqt, dst = mx.cast_dim1_grouped(dyb.cuda(), offs_t.cuda(), cap)
    xqt, xst = mx.cast_dim1_grouped(x2.cuda(), offs_t.cuda(), cap)
    dw = mx.grouped_mm_wgrad(dqt, dst, xqt, xst, offs_t.cuda(), M)
    mx.mx_device_error()
    oa, osa = O.cast_dim1_grouped(S.bf16_bits(dyb), offs, cap)
    ob, osb = O.cast_dim1_grouped(S.bf16_bits(x2), offs, cap)
    p = O.padded_group_starts(offs)
    empty = torch.from_numpy(sizes == 0).cuda()
    assert not dw[empty].any()
    for g in np.flatnonzero(sizes):                    # the oracle per live group (K groups = token columns)
        blk = slice(p[g] // 32, p[g] // 32 + (int(sizes[g]) + 31) // 32)
        da = O.dequant(oa[:, p[g]:p[g] + 32 * (blk.stop - blk.start)], osa[:, blk])[:, :int(sizes[g])]
        db = O.dequant(ob[:, p[g]:p[g] + 32 * (blk.stop - blk.start)], osb[:, blk])[:, :int(sizes[g])]
        _close(_f64(dw[int(g)]), O.mm(da, db), O.mm(np.abs(da), np.abs(db)), f"wgrad g={g}")


def test_bf16_grouped_gemms_at_1024_groups(mx, sizes):
    M, N, K = int(sizes.sum()), 256, 256
    a = S.normal_bf16((M, K), seed=8)
    b = S.normal_bf16((G, K, N), 0.05, seed=9)
    offs_t = S.offsets_from_sizes(sizes)
    offs = offs_t.numpy()
    out = mx.grouped_mm_bf16(a.cuda(), b.cuda(), offs_t.cuda())
    a2 = S.normal_bf16((M, N), seed=10)
    dw = mx.grouped_mm_bf16_wgrad(a2.cuda(), a.cuda(), offs_t.cuda())
    mx.mx_device_error()
    af, bf, a2f = (O.bf16_to_f64(S.bf16_bits(t)) for t in (a, b, a2))
    _close(_f64(out), O.hp_grouped_mm_m(af, bf, offs), O.hp_grouped_mm_m(np.abs(af), np.abs(bf), offs), "rows")
    starts, ends = O.group_bounds(offs)
    empty = torch.from_numpy(sizes == 0).cuda()
    assert not dw[empty].any()
    for g in np.flatnonzero(sizes):                    # the oracle per live group (tokens of g)
        rows = slice(int(starts[g]), int(ends[g]))
        ref = a2f[rows].T @ af[rows]
        absref = np.abs(a2f[rows]).T @ np.abs(af[rows])
        _close(_f64(dw[int(g)]), ref, absref, f"tokens g={g}")


def test_1025_groups_are_rejected(mx):
    x = torch.zeros(64, 128, dtype=torch.bfloat16, device="cuda")
    offs = torch.full((G + 1,), 64, dtype=torch.int32, device="cuda")
    with pytest.raises(mx.MXError) as e:
        mx.cast_dim0_grouped(x, offs)
    assert e.value.status == 1
    b = torch.zeros(G + 1, 128, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mx.MXError) as e:
        mx.grouped_mm_bf16(x, b, offs)
    assert e.value.status == 1
