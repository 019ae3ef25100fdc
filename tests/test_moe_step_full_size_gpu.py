"""The benchmarked MoE step at its own size, checked against the oracle.

The step is the MoE grouped layer forward + backward of ao PR #4705 ("Wire
MoE and MXFP8Linear training paths to CuTeDSL by default", benchmark
commands: K=N=4096, G=8, M=16384 tokens in Dirichlet(1) groups), run exactly
as `bench.py` times it: the fused grouped casts of X and dY into the padded
group layout, the 32x32 cast of the expert weights, the forward GEMM, the
dgrad GEMM reading the forward's weight codes MN-major, and the K-groups
wgrad GEMM.

Every output tile of every GEMM launch is sampled: the launches tile each
group's padded rows in 256-row tiles and the columns in 256-column tiles, and
each (row tile, column tile) pair gets a whole 32-column slab of at least
one row, plus the first and last real row of every group. The wgrad is
checked on sixteen full 32-column slices per expert (one in every
256-column tile, every row), and an empty expert must be exact zeros. The
casts feeding the GEMMs are compared bitwise where the checks read them.

The oracle quantizes the same input bits itself (rowwise casts are per row,
columnwise per column and 32x32 per tile, so casting the sampled rows,
columns or tile rows alone gives the same codes as the whole tensor), and
the GEMM tolerance is |gpu - ref| <= 2^-7 |ref| + 1e-3 (|A| |B|^T).
"""
import numpy as np
import pytest
import torch

from oracle import mx_oracle as O
from mxfp8_block_scaled_cast_b200 import synthetic as S

pytestmark = pytest.mark.gpu

TILE = 256        # output tile edge of the GEMM launches
SLAB = 32         # sampled columns per tile


@pytest.fixture(scope="module")
def step():
    import bench
    from mxfp8_block_scaled_cast_b200 import mx
    mx.lib()
    st = bench.MoEStep(mx, torch.device("cuda"), seed=0)
    st.run()
    mx.mx_device_error()
    torch.cuda.synchronize()
    return st


def host_view(step):
    """Input bits and group geometry of a step on the host."""
    ends = step.offs.cpu().numpy().astype(np.int64)
    starts = np.concatenate([[0], ends[:-1]])
    sizes = ends - starts
    pstart = np.concatenate([[0], np.cumsum(-(-sizes // 128) * 128)])[:-1]
    return {
        "x": S.bf16_bits(step.x), "w": S.bf16_bits(step.w), "dy": S.bf16_bits(step.dy),
        "starts": starts, "ends": ends, "sizes": sizes, "pstart": pstart,
    }


@pytest.fixture(scope="module")
def host(step):
    return host_view(step)


def _close(got, ref, absref, what):
    err = np.abs(got - ref)
    bound = O.gemm_bound(ref, absref)
    bad = err > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} outside tolerance, worst {np.max(err - bound)}"


def _sampled_rows(size, rng):
    """Local rows of a group: one in every 256-row launch tile, plus the first and last."""
    padded = -(-size // 128) * 128
    rows = {0, size - 1}
    for t in range(-(-padded // TILE)):
        lo, hi = t * TILE, min(t * TILE + TILE, size)
        rows.add(int(rng.integers(lo, hi)))
    return np.array(sorted(rows), dtype=np.int64)


def _slab_cols(width, rng):
    """One 32-column slab in every 256-column tile: (slab starts, all their columns)."""
    starts = np.array([t * TILE + SLAB * int(rng.integers(TILE // SLAB)) for t in range(width // TILE)])
    return starts, (starts[:, None] + np.arange(SLAB)[None, :]).reshape(-1)


def _rows_f64(t, rows, cols):
    idx_r = torch.as_tensor(rows, device=t.device)
    idx_c = torch.as_tensor(cols, device=t.device)
    return t.index_select(0, idx_r).index_select(1, idx_c).float().cpu().numpy().astype(np.float64)


def test_step_forward_every_tile(step, host):
    rng = np.random.default_rng(10)
    G, N = step.G, step.N
    xq = step.xq.cpu().numpy()
    xs = O.unswizzle(step.xs.cpu().numpy(), step.cap, step.K // 32)
    checked = 0
    for g in range(G):
        size = int(host["sizes"][g])
        if size == 0:
            continue
        local = _sampled_rows(size, rng)
        rows = host["starts"][g] + local
        qx, sx = O.cast_dim0(host["x"][rows])
        # the fused grouped cast put these rows at their padded positions, bit-exact
        prow = host["pstart"][g] + local
        assert np.array_equal(xq[prow], qx) and np.array_equal(xs[prow], sx), f"x cast, group {g}"
        a = O.dequant(qx, sx)
        n0s, cols = _slab_cols(N, rng)
        bs = []
        for n0 in n0s:
            qw, st = O.cast_32x32(host["w"][g, n0:n0 + SLAB])
            s_fwd, _ = O.w32_scale_views(st)
            bs.append(O.dequant(qw, s_fwd))
        b = np.concatenate(bs)                                  # [16 * 32, K]
        _close(_rows_f64(step.y, rows, cols), O.mm(a, b), O.mm(np.abs(a), np.abs(b)), f"forward, group {g}")
        checked += len(rows) * len(cols)
    assert checked > 0


def test_step_dgrad_every_tile(step, host):
    rng = np.random.default_rng(11)
    G, N, K = step.G, step.N, step.K
    dq = step.dq.cpu().numpy()
    ds = O.unswizzle(step.ds.cpu().numpy(), step.cap, N // 32)
    for g in range(G):
        size = int(host["sizes"][g])
        if size == 0:
            continue
        local = _sampled_rows(size, rng)
        rows = host["starts"][g] + local
        qd, sd = O.cast_dim0(host["dy"][rows])
        prow = host["pstart"][g] + local
        assert np.array_equal(dq[prow], qd) and np.array_equal(ds[prow], sd), f"dy cast, group {g}"
        a = O.dequant(qd, sd)                                   # [r, N]
        k0s, cols = _slab_cols(K, rng)
        bts = []
        for k0 in k0s:
            qw, st = O.cast_32x32(host["w"][g][:, k0:k0 + SLAB])   # [N, 32]: whole 32x32 tiles
            _, s_dg = O.w32_scale_views(st)
            bts.append(O.dequant(np.ascontiguousarray(qw.T), s_dg))  # W^T rows [32, N]
        bt = np.concatenate(bts)
        _close(_rows_f64(step.dx, rows, cols), O.mm(a, bt), O.mm(np.abs(a), np.abs(bt)), f"dgrad, group {g}")


def test_step_wgrad_full_slices(step, host):
    rng = np.random.default_rng(12)
    G, N, K = step.G, step.N, step.K
    dqt = step.dqt.cpu().numpy()
    xqt = step.xqt.cpu().numpy()
    for g in range(G):
        size = int(host["sizes"][g])
        if size == 0:
            assert not step.dw[g].any(), f"empty group {g} must give exact zeros"
            continue
        s0, e0 = host["starts"][g], host["ends"][g]
        off1 = np.array([size])
        cap = O.padded_rows_capacity(size, 1)
        qa, sa = O.cast_dim1_grouped(host["dy"][s0:e0], off1, cap)          # [N, cap]
        p0 = host["pstart"][g]
        assert np.array_equal(dqt[:, p0:p0 + cap], qa), f"dy columnwise cast, group {g}"
        k0s, cols = _slab_cols(K, rng)
        qb, sb = O.cast_dim1_grouped(host["x"][s0:e0][:, cols], off1, cap)  # [512, cap]
        assert np.array_equal(xqt[cols, p0:p0 + cap], qb), f"x columnwise cast, group {g}"
        a, b = O.dequant(qa, sa), O.dequant(qb, sb)
        got = step.dw[g].index_select(1, torch.as_tensor(cols, device=step.dw.device))
        _close(got.float().cpu().numpy().astype(np.float64), O.mm(a, b), O.mm(np.abs(a), np.abs(b)),
               f"wgrad, group {g}")


def test_step_repeats_bitwise(step):
    """A second run of the whole step reproduces every output bit (no atomics, no split-K)."""
    y, dx, dw = step.y.clone(), step.dx.clone(), step.dw.clone()
    step.run()
    torch.cuda.synchronize()
    assert torch.equal(y, step.y) and torch.equal(dx, step.dx) and torch.equal(dw, step.dw)
