"""Out-of-bounds writes: every output lives inside a guarded allocation.

compute-sanitizer is not available here, so each output buffer of each entry
point is carved out of a larger allocation whose bands before and after it
hold a sentinel byte; after the call (and the device-error check) the bands
must be intact. Shapes are ragged on purpose -- rows and columns past a
tile, groups that are empty or end anywhere, N and K off the GEMM tile --
because that is where a kernel's masks and clamps decide whether it writes
past the end of a buffer. The values themselves are checked elsewhere
against the oracle; here only the bytes outside the outputs are.
"""
import numpy as np
import pytest
import torch

from mxfp8_block_scaled_cast_b200 import synthetic as S

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes of sentinel on each side (a multiple of 256: alignment kept)
SENTINEL = 0xA5


@pytest.fixture(scope="module")
def mx():
    from mxfp8_block_scaled_cast_b200 import mx as _mx
    _mx.lib()
    return _mx


class Guarded:
    """Device buffers carved from sentinel-filled allocations."""

    def __init__(self):
        self.bufs = []

    def u8(self, *shape):
        return self._take(int(np.prod(shape)), torch.uint8).view(*shape)

    def bf16(self, *shape):
        return self._take(2 * int(np.prod(shape)), torch.uint8).view(torch.bfloat16).view(*shape)

    def raw(self, nbytes):
        return self._take(int(nbytes), torch.uint8)

    def _take(self, nbytes, dtype):
        buf = torch.full((GUARD + nbytes + GUARD,), SENTINEL, dtype=torch.uint8, device="cuda")
        self.bufs.append((buf, nbytes))
        return buf[GUARD:GUARD + nbytes]

    def check(self, mx, what):
        mx.mx_device_error()
        torch.cuda.synchronize()
        for i, (buf, n) in enumerate(self.bufs):
            head, tail = buf[:GUARD], buf[GUARD + n:]
            assert bool((head == SENTINEL).all()) and bool((tail == SENTINEL).all()), \
                f"{what}: output {i} ({n} bytes) was written outside its bounds"


def _x(R, C, seed):
    return S.sweep_tensor((R, C), seed=seed).cuda()


@pytest.mark.parametrize("R,C", [(96, 160), (224, 576), (32, 32), (416, 96)])
def test_dense_casts_stay_in_bounds(mx, R, C):
    x = _x(R, C, R + C)
    sb = lambda r, c: mx.mx_scale_bytes(r, c // 32)
    g = Guarded()
    mx.mx_cast_dim0(x, g.u8(R, C), g.raw(sb(R, C)))
    mx.mx_cast_dim1(x, g.u8(C, R), g.raw(sb(C, R)))
    mx.mx_cast_2d(x, g.u8(R, C), g.raw(sb(R, C)), g.u8(C, R), g.raw(sb(C, R)))
    mx.mx_cast_w32x32(x, g.u8(R, C), g.raw(sb(R, C)), g.u8(C, R), g.raw(sb(C, R)))
    mx.mx_cast_ex(x, 3, mx.MX_FLOOR, g.u8(R, C), g.raw(sb(R, C)), g.u8(C, R), g.raw(sb(C, R)))
    g.check(mx, f"dense casts {R}x{C}")


def test_expert_stack_cast_stays_in_bounds(mx):
    G, N, K = 3, 96, 160
    w = S.sweep_tensor((G, N, K), seed=4).cuda()
    g = Guarded()
    mx.mx_cast_w32x32(w, g.u8(G, N, K), g.raw(G * mx.mx_scale_bytes(N, K // 32)), g.u8(G, K, N),
                      g.raw(G * mx.mx_scale_bytes(K, N // 32)))
    g.check(mx, "32x32 expert stack")


@pytest.mark.parametrize("sizes,K", [([100, 0, 250, 1, 37], 96), ([0, 0, 300], 576), ([128, 256], 160)])
def test_grouped_casts_stay_in_bounds(mx, sizes, K):
    M, G = sum(sizes), len(sizes)
    x = _x(M, K, M + K)
    offs = S.offsets_from_sizes(sizes).cuda()
    cap = mx.mx_padded_rows_capacity(M, G)
    g = Guarded()
    mx.mx_cast_dim0_grouped(x, offs, cap, g.u8(cap, K), g.raw(mx.mx_scale_bytes(cap, K // 32)))
    mx.mx_cast_dim1_grouped(x, offs, cap, g.u8(K, cap), g.raw(mx.mx_scale_bytes(K, cap // 32)))
    mx.mx_cast_2d_grouped(x, offs, cap, g.u8(cap, K), g.raw(mx.mx_scale_bytes(cap, K // 32)), g.u8(K, cap),
                          g.raw(mx.mx_scale_bytes(K, cap // 32)))
    g.check(mx, f"grouped casts {sizes} K={K}")


def _moe_operands(mx, sizes, N, K, G_w):
    """Quantized operands of a small grouped layer: groups `sizes`, G_w expert weights."""
    M, G = sum(sizes), len(sizes)
    x = S.normal_bf16((M, K), seed=M).cuda()
    w = S.normal_bf16((G_w, N, K), 0.02, seed=N).cuda()
    dy = S.normal_bf16((M, N), 0.1, seed=K).cuda()
    offs = S.offsets_from_sizes(sizes).cuda()
    cap = mx.mx_padded_rows_capacity(M, G)
    xq, xs = mx.cast_dim0_grouped(x, offs, cap)
    dq, ds = mx.cast_dim0_grouped(dy, offs, cap)
    xqt, xst = mx.cast_dim1_grouped(x, offs, cap)
    dqt, dst = mx.cast_dim1_grouped(dy, offs, cap)
    wq, wsf, _, wsd = mx.cast_w32x32(w, transposed=False, dgrad_scales=True)
    return dict(M=M, G=G, cap=cap, x=x, w=w, dy=dy, offs=offs, xq=xq, xs=xs, dq=dq, ds=ds, xqt=xqt, xst=xst,
                dqt=dqt, dst=dst, wq=wq, wsf=wsf, wsd=wsd)


@pytest.mark.parametrize("sizes,N,K", [([100, 0, 250, 1, 37], 96, 576), ([0, 300, 0], 576, 96), ([256, 128], 256, 256)])
def test_grouped_gemms_stay_in_bounds(mx, sizes, N, K):
    o = _moe_operands(mx, sizes, N, K, len(sizes))
    M, G, cap, offs = o["M"], o["G"], o["cap"], o["offs"]
    g = Guarded()
    mx.mx_grouped_mm(o["xq"], o["xs"], o["wq"], o["wsf"], offs, G, mx.MX_GROUPS_M, g.bf16(M, N), M, N, K, cap)
    mx.mx_grouped_mm(o["dq"], o["ds"], o["wq"], o["wsd"], offs, G, mx.MX_GROUPS_M_KN, g.bf16(M, K), M, K, N, cap)
    mx.mx_grouped_mm(o["dqt"], o["dst"], o["xqt"], o["xst"], offs, G, mx.MX_GROUPS_K, g.bf16(G, N, K), M, N, K, cap)
    mx.mx_grouped_mm_bf16(o["dy"], o["w"], offs, G, mx.MX_GROUPS_M, g.bf16(M, K), M, K, N)
    mx.mx_grouped_mm_bf16(o["dy"], o["x"], offs, G, mx.MX_GROUPS_K, g.bf16(G, N, K), M, N, K)
    mx.mx_dequant_dim0_grouped(o["xq"], o["xs"], offs, M, K, cap, g.bf16(M, K))
    g.check(mx, f"grouped GEMMs {sizes} N={N} K={K}")


def test_expert_cycling_gemms_stay_in_bounds(mx):
    """Groups cycling over fewer experts (the expert-parallel receive layout): E = 2, G = 6."""
    sizes, N, K, E = [70, 0, 130, 45, 300, 3], 96, 160, 2
    o = _moe_operands(mx, sizes, N, K, E)
    M, G, cap, offs = o["M"], o["G"], o["cap"], o["offs"]
    g = Guarded()
    mx.mx_grouped_mm_experts(o["xq"], o["xs"], o["wq"], o["wsf"], offs, G, E, mx.MX_GROUPS_M, g.bf16(M, N), M, N, K,
                             cap)
    mx.mx_grouped_mm_experts(o["dq"], o["ds"], o["wq"], o["wsd"], offs, G, E, mx.MX_GROUPS_M_KN, g.bf16(M, K), M, K,
                             N, cap)
    mx.mx_grouped_mm_experts(o["dqt"], o["dst"], o["xqt"], o["xst"], offs, G, E, mx.MX_GROUPS_K, g.bf16(E, N, K), M,
                             N, K, cap)
    g.check(mx, "expert-cycling GEMMs")


def test_dequant_and_unswizzle_stay_in_bounds(mx):
    G, R, C = 2, 96, 160
    w = S.sweep_tensor((G, R, C), seed=9).cuda()
    q, s, _, _ = mx.cast_w32x32(w, transposed=False)
    g = Guarded()
    mx.mx_dequant_dim0(q, s, G, R, C, g.bf16(G, R, C))
    x = _x(R, C, 10)
    xq, xs = mx.cast_dim0(x)
    mx.mx_scales_unswizzle(xs, R, C // 32, g.u8(R, C // 32))
    g.check(mx, "dequant and unswizzle")


@pytest.mark.parametrize("M,N,K", [(96, 576, 160), (256, 96, 576)])
def test_linear_stays_in_bounds(mx, M, N, K):
    x, w, dy = (t.cuda() for t in S.linear_problem(M=M, N=N, K=K, seed=M + N))
    for use_cache in (False, True):
        cache = mx.WeightCache() if use_cache else None
        g = Guarded()
        ws = g.raw(mx.mx_linear_ws_bytes(M, N, K))
        y, dx, dw = g.bf16(M, N), g.bf16(M, K), g.bf16(N, K)
        for _ in range(2):                      # a miss, then (with the cache) a hit
            mx.mx_linear_fwd(x, w, cache, 0, y, ws)
            mx.mx_linear_bwd(dy, x, w, cache, 0, dx, dw, ws)
        g.check(mx, f"linear {M}x{N}x{K} cache={use_cache}")
        if cache is not None:
            cache.close()
    g = Guarded()
    mx.mx_linear_fwd_noalloc(x, w, g.bf16(M, N))
    g.check(mx, f"linear without allocation {M}x{N}x{K}")


def test_scatter_cast_stays_in_bounds(mx):
    """The one-kernel MXFP8 dispatch: every rank's groups into every receive
    buffer (ranks emulated with local buffers), each buffer guarded."""
    from mxfp8_block_scaled_cast_b200 import ep
    W, E, K = 3, 2, 576
    rng = np.random.default_rng(5)
    counts = rng.integers(0, 300, size=(W, W * E))
    counts[1, :] = 0
    plans = [ep.DirectPlan(W, E, r, counts) for r in range(W)]
    band = ep.scale_band_bytes(K)
    g = Guarded()
    bq = [g.u8(int(plans[0].recv_rows_of[d]), K) for d in range(W)]
    bs = [g.raw(int(plans[0].recv_rows_of[d]) // 128 * band) for d in range(W)]
    for r in range(W):
        x = _x(int(counts[r].sum()), K, 30 + r)
        ep.dispatch_mxfp8_direct(x, plans[r], [b.data_ptr() for b in bq], [b.data_ptr() for b in bs])
    g.check(mx, "scatter cast")


def test_fused_scatter_cast_stays_in_bounds(mx):
    """The fused (rowwise + columnwise) scatter cast of three emulated ranks'
    dY into every rank's four guarded receive buffers (N = 96, ragged groups)."""
    from mxfp8_block_scaled_cast_b200 import ep
    W, E, N = 3, 2, 96
    rng = np.random.default_rng(7)
    counts = rng.integers(0, 300, size=(W, W * E))
    counts[1, 2] = 0
    plans = [ep.ExchangePlan(W, E, counts[r], counts[:, r * E:(r + 1) * E]) for r in range(W)]
    band = ep.scale_band_bytes(N)
    g = Guarded()
    bq = [g.raw(pl.m_cap_recv * N) for pl in plans]
    bs = [g.raw(pl.m_cap_recv // 128 * band) for pl in plans]
    bqt = [g.raw(N * pl.m_cap_recv) for pl in plans]
    bst = [g.raw(mx.mx_scale_bytes(N, pl.m_cap_recv // 32)) for pl in plans]
    ptrs = lambda bufs: [b.data_ptr() for b in bufs]
    for r in range(W):
        dy = S.normal_bf16((int(counts[r].sum()), N), 0.1, seed=r).cuda()
        ep.dispatch_2d_direct(dy, ep.DirectPlan(W, E, r, counts), ptrs(bq), ptrs(bs), ptrs(bqt), ptrs(bst))
    g.check(mx, "fused scatter cast")


def test_gemm_to_sender_rows_stays_in_bounds(mx):
    """The expert GEMMs with the combine fused: outputs and dX rows stored into
    every sender's (guarded) buffer, ranks emulated."""
    from mxfp8_block_scaled_cast_b200 import ep
    W, E, N, K = 2, 2, 96, 160
    rng = np.random.default_rng(6)
    counts = rng.integers(0, 300, size=(W, W * E))
    counts[0, 1] = 0
    g = Guarded()
    ybuf = [g.bf16(int(counts[s].sum()), N) for s in range(W)]
    dxbuf = [g.bf16(int(counts[s].sum()), K) for s in range(W)]
    for r in range(W):
        dp = ep.DirectPlan(W, E, r, counts)
        ex = dp.exchange
        x = S.normal_bf16((ex.M_recv, K), seed=r).cuda()
        dy = S.normal_bf16((ex.M_recv, N), 0.1, seed=10 + r).cuda()
        w = S.normal_bf16((E, N, K), 0.02, seed=20 + r).cuda()
        offs = torch.as_tensor(ex.offs_recv()).cuda()
        rq, rs = mx.cast_dim0_grouped(x, offs, ex.m_cap_recv)
        rs = rs.view(ex.m_cap_recv // 128, ep.scale_band_bytes(K))
        wq, wsf, _, wsd = mx.cast_w32x32(w, transposed=False, dgrad_scales=True)
        ep.expert_forward_to_senders(rq, rs, wq, wsf, dp, [b.data_ptr() for b in ybuf])
        ep.expert_backward(dy, rq, rs, wq, wsd, ex, dx_rows=dp.combine_destinations([b.data_ptr() for b in dxbuf], K))
    g.check(mx, "GEMM rows to senders")
