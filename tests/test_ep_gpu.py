"""Expert-parallel MoE layer with the MXFP8 all-to-all, on one GPU.

1. The expert side alone: received groups (source rank, local expert) through
   mx_grouped_mm_experts (group g uses expert g % E) in all three modes,
   against the oracle's ep_expert_forward / ep_expert_backward.
2. Two and four ranks emulated in one process (one stream; nothing waits on
   another kernel): every rank packs its tokens with the CUDA cast, a host-side copy
   stands in for the all-to-all (the same slices NCCL would move), the
   expert GEMMs run per rank, and each rank's y, dx and dw are checked
   against the oracle.
3. The module itself over a one-rank NCCL group (the all-to-all is a
   loopback through NCCL).

GEMM tolerance: |gpu - ref| <= 2^-7 |ref| + 1e-3 (|A| |B|^T).
"""
import os
import socket

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


def _close(got, ref, absref, what):
    bad = ~(np.abs(got - ref) <= O.gemm_bound(ref, absref))
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} outside tolerance"


@pytest.mark.parametrize("W,E,N,K", [(3, 2, 512, 256), (2, 4, 576, 96)])
def test_expert_side_groups_cycle_over_experts(mx, W, E, N, K):
    from mxfp8_block_scaled_cast_b200 import ep
    rng = np.random.default_rng(W * E + K)
    recv = rng.integers(0, 300, size=(W, E))
    recv[0, 1] = 0
    plan = ep.ExchangePlan(W, E, recv.reshape(-1), recv)        # the send side is not used here
    M = plan.M_recv
    xb = S.normal_bf16((M, K), seed=1)
    wb = S.normal_bf16((E, N, K), 0.02, seed=2)
    dyb = S.normal_bf16((M, N), 0.1, seed=3)
    offs = torch.as_tensor(plan.offs_recv()).cuda()
    rq, rs = mx.cast_dim0_grouped(xb.cuda(), offs, plan.m_cap_recv)
    wq, wsf, _, wsd = mx.cast_w32x32(wb.cuda(), transposed=False, dgrad_scales=True)
    rs = rs.view(plan.m_cap_recv // 128, ep.scale_band_bytes(K))
    y = ep.expert_forward(rq, rs, wq, wsf, plan)
    dx, dw = ep.expert_backward(dyb.cuda(), rq, rs, wq, wsd, plan)
    mx.mx_device_error()
    xbits, wbits, dbits = S.bf16_bits(xb), S.bf16_bits(wb), S.bf16_bits(dyb)
    of = plan.offs_recv()
    _close(_f64(y), *O.ep_expert_forward(xbits, wbits, of, E), "forward")
    dx_ref, dx_abs, dw_ref, dw_abs = O.ep_expert_backward(xbits, wbits, dbits, of, E)
    _close(_f64(dx), dx_ref, dx_abs, "dgrad")
    _close(_f64(dw), dw_ref, dw_abs, "wgrad (each expert sums its groups over sources)")


def _virtual_a2a(ins, in_splits, out_splits):
    """What an all-to-all delivers: rank d receives chunk d of every rank's
    input (chunks cut by that rank's input splits), in rank order."""
    W = len(ins)
    starts = [np.concatenate([[0], np.cumsum(sp)]) for sp in in_splits]
    outs = []
    for d in range(W):
        parts = [ins[s][int(starts[s][d]):int(starts[s][d + 1])] for s in range(W)]
        assert [p.shape[0] for p in parts] == [int(v) for v in out_splits[d]]
        outs.append(torch.cat(parts) if parts else ins[d][:0])
    return outs


@pytest.mark.parametrize("W,E,N,K", [(2, 3, 256, 576), (4, 2, 512, 256)])
def test_ranks_emulated_end_to_end(mx, W, E, N, K):
    from mxfp8_block_scaled_cast_b200 import ep
    rng = np.random.default_rng(7 + W)
    counts = [rng.integers(0, 260, size=W * E) for _ in range(W)]
    counts[1][2] = 0
    xs = [S.normal_bf16((int(c.sum()), K), seed=10 + r) for r, c in enumerate(counts)]
    ws = [S.normal_bf16((E, N, K), 0.02, seed=20 + r) for r in range(W)]      # rank r's local experts
    dys = [S.normal_bf16((int(c.sum()), N), 0.1, seed=30 + r) for r, c in enumerate(counts)]
    plans = [ep.ExchangePlan(W, E, counts[r], np.stack([counts[s][r * E:(r + 1) * E] for s in range(W)]))
             for r in range(W)]
    packed = [ep.pack_mxfp8(xs[r].cuda(), plans[r]) for r in range(W)]
    rq = _virtual_a2a([p[0] for p in packed], [pl.send_rows for pl in plans], [pl.recv_rows for pl in plans])
    rs = _virtual_a2a([p[1] for p in packed], [pl.send_rows // 128 for pl in plans],
                      [pl.recv_rows // 128 for pl in plans])
    wc = [mx.cast_w32x32(w.cuda(), transposed=False, dgrad_scales=True) for w in ws]
    y_recv = [ep.expert_forward(rq[r], rs[r], wc[r][0], wc[r][1], plans[r]) for r in range(W)]
    ys = _virtual_a2a(y_recv, [pl.recv_tokens for pl in plans], [pl.send_tokens for pl in plans])
    dy_recv = _virtual_a2a([d.cuda() for d in dys], [pl.send_tokens for pl in plans],
                           [pl.recv_tokens for pl in plans])
    back = [ep.expert_backward(dy_recv[r], rq[r], rs[r], wc[r][0], wc[r][3], plans[r]) for r in range(W)]
    dxs = _virtual_a2a([b[0] for b in back], [pl.recv_tokens for pl in plans], [pl.send_tokens for pl in plans])
    mx.mx_device_error()
    # the oracle, from each sender's view: token rows of global expert j use expert j % E of rank j // E
    for r in range(W):
        wall = np.concatenate([S.bf16_bits(w) for w in ws])                    # [W*E, N, K], global order
        of = np.cumsum(counts[r])
        xbits, dbits = S.bf16_bits(xs[r]), S.bf16_bits(dys[r])
        y_ref, y_abs = O.ep_expert_forward(xbits, wall, of, W * E)
        _close(_f64(ys[r]), y_ref, y_abs, f"y of rank {r}")
        dx_ref, dx_abs, _, _ = O.ep_expert_backward(xbits, wall, dbits, of, W * E)
        _close(_f64(dxs[r]), dx_ref, dx_abs, f"dx of rank {r}")
    # dW from each expert's view: its received groups, source major
    for r in range(W):
        ends = [np.cumsum(c) for c in counts]
        xr = np.concatenate([S.bf16_bits(xs[s])[(ends[s][j - 1] if j else 0):ends[s][j]]
                             for s in range(W) for j in range(r * E, (r + 1) * E)])
        dr = np.concatenate([S.bf16_bits(dys[s])[(ends[s][j - 1] if j else 0):ends[s][j]]
                             for s in range(W) for j in range(r * E, (r + 1) * E)])
        _, _, dw_ref, dw_abs = O.ep_expert_backward(xr, S.bf16_bits(ws[r]), dr, plans[r].offs_recv(), E)
        _close(_f64(back[r][1]), dw_ref, dw_abs, f"dw of rank {r}")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_module_over_a_one_rank_nccl_group(mx):
    import torch.distributed as dist
    from mxfp8_block_scaled_cast_b200 import ep
    if dist.is_initialized():
        pytest.skip("a process group already exists")
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    from datetime import timedelta
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        E, N, K = 4, 512, 256
        counts = np.array([100, 0, 333, 129])
        x = S.normal_bf16((int(counts.sum()), K), seed=40)
        w = S.normal_bf16((E, N, K), 0.02, seed=41)
        dy = S.normal_bf16((int(counts.sum()), N), 0.1, seed=42)
        layer = ep.MXFP8ExpertParallelMM()
        y = layer.forward(x.cuda(), counts, w.cuda())
        dx, dw = layer.backward(dy.cuda())
        mx.mx_device_error()
        xb, wb, db, of = S.bf16_bits(x), S.bf16_bits(w), S.bf16_bits(dy), np.cumsum(counts)
        _close(_f64(y), *O.ep_expert_forward(xb, wb, of, E), "y")
        dx_ref, dx_abs, dw_ref, dw_abs = O.ep_expert_backward(xb, wb, db, of, E)
        _close(_f64(dx), dx_ref, dx_abs, "dx")
        _close(_f64(dw), dw_ref, dw_abs, "dw")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("W,E,K", [(2, 3, 576), (4, 2, 256), (3, 1, 96), (9, 8, 64)])
def test_direct_dispatch_equals_the_all_to_all(mx, W, E, K):
    """The dispatch as one kernel (every rank's cast storing straight into every
    receive buffer), ranks emulated in one process with local buffers: each
    receive buffer is bitwise what the cast + all-to-all path delivers (up to
    W*E = 72 groups, destinations in nine buffers)."""
    from mxfp8_block_scaled_cast_b200 import ep
    rng = np.random.default_rng(60 + W)
    counts = rng.integers(0, 260, size=(W, W * E))
    counts[0, -1] = 0
    counts[W - 1, :E] = 128
    xs = [S.normal_bf16((int(counts[r].sum()), K), seed=70 + r).cuda() for r in range(W)]
    plans = [ep.ExchangePlan(W, E, counts[r], counts[:, r * E:(r + 1) * E]) for r in range(W)]
    packed = [ep.pack_mxfp8(xs[r], plans[r]) for r in range(W)]
    rq = _virtual_a2a([p[0] for p in packed], [pl.send_rows for pl in plans], [pl.recv_rows for pl in plans])
    rs = _virtual_a2a([p[1] for p in packed], [pl.send_rows // 128 for pl in plans],
                      [pl.recv_rows // 128 for pl in plans])
    band = ep.scale_band_bytes(K)
    bq = [torch.full((pl.m_cap_recv, K), 0xA5, dtype=torch.uint8, device="cuda") for pl in plans]
    bs = [torch.full((pl.m_cap_recv // 128, band), 0xA5, dtype=torch.uint8, device="cuda") for pl in plans]
    for r in range(W):
        dplan = ep.DirectPlan(W, E, r, counts)
        assert dplan.exchange.m_cap_send == plans[r].m_cap_send
        ep.dispatch_mxfp8_direct(xs[r], dplan, [b.data_ptr() for b in bq], [b.data_ptr() for b in bs])
    mx.mx_device_error()
    for d in range(W):
        assert torch.equal(bq[d], rq[d]), f"codes received by rank {d}"
        assert torch.equal(bs[d], rs[d]), f"scales received by rank {d}"


def test_module_direct_over_a_one_rank_nccl_group(mx):
    """The layer with the one-kernel dispatch into symmetric memory: outputs and
    gradients bitwise those of the all-to-all layer; a second forward before
    the backward is refused."""
    import torch.distributed as dist
    from mxfp8_block_scaled_cast_b200 import ep
    if dist.is_initialized():
        pytest.skip("a process group already exists")
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    from datetime import timedelta
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        E, N, K = 4, 512, 256
        counts = np.array([100, 0, 333, 129])
        x = S.normal_bf16((int(counts.sum()), K), seed=50).cuda()
        w = S.normal_bf16((E, N, K), 0.02, seed=51).cuda()
        dy = S.normal_bf16((int(counts.sum()), N), 0.1, seed=52).cuda()
        ref = ep.MXFP8ExpertParallelMM()
        y0 = ref.forward(x, counts, w)
        dx0, dw0 = ref.backward(dy)
        layer = ep.MXFP8ExpertParallelMM(direct=True)
        for _ in range(2):                              # the second step reuses the buffer
            y = layer.forward(x, counts, w)
            dx, dw = layer.backward(dy)
            mx.mx_device_error()
            assert torch.equal(y, y0) and torch.equal(dx, dx0) and torch.equal(dw, dw0)
        # a larger step (the symmetric buffers are regrown collectively), then a
        # smaller one (buffers larger than needed): still bitwise the all-to-all layer
        for step_counts, seed in ((np.array([300, 129, 513, 7]), 60), (np.array([0, 40, 0, 33]), 70)):
            xs = S.normal_bf16((int(step_counts.sum()), K), seed=seed).cuda()
            dys = S.normal_bf16((int(step_counts.sum()), N), 0.1, seed=seed + 1).cuda()
            y_ref = ref.forward(xs, step_counts, w)
            dx_ref, dw_ref = ref.backward(dys)
            y = layer.forward(xs, step_counts, w)
            dx, dw = layer.backward(dys)
            mx.mx_device_error()
            assert torch.equal(y, y_ref) and torch.equal(dx, dx_ref) and torch.equal(dw, dw_ref), step_counts
        layer.forward(x, counts, w)
        with pytest.raises(RuntimeError):
            layer.forward(x, counts, w)
        layer.backward(dy)
        del layer
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("W,E,N,K", [(2, 3, 256, 576), (4, 2, 576, 256)])
def test_fused_combine_equals_the_all_to_all(mx, W, E, N, K):
    """The combine fused into the expert GEMMs (each output row, and in backward
    each dX row, stored straight into the sender's buffer), ranks emulated with
    local buffers: bitwise the outputs of the all-to-all path."""
    from mxfp8_block_scaled_cast_b200 import ep
    rng = np.random.default_rng(80 + W)
    counts = rng.integers(0, 260, size=(W, W * E))
    counts[1, 0] = 0
    xs = [S.normal_bf16((int(counts[r].sum()), K), seed=90 + r).cuda() for r in range(W)]
    ws = [S.normal_bf16((E, N, K), 0.02, seed=100 + r).cuda() for r in range(W)]
    dys = [S.normal_bf16((int(counts[r].sum()), N), 0.1, seed=110 + r).cuda() for r in range(W)]
    plans = [ep.ExchangePlan(W, E, counts[r], counts[:, r * E:(r + 1) * E]) for r in range(W)]
    dplans = [ep.DirectPlan(W, E, r, counts) for r in range(W)]
    packed = [ep.pack_mxfp8(xs[r], plans[r]) for r in range(W)]
    rq = _virtual_a2a([p[0] for p in packed], [pl.send_rows for pl in plans], [pl.recv_rows for pl in plans])
    rs = _virtual_a2a([p[1] for p in packed], [pl.send_rows // 128 for pl in plans],
                      [pl.recv_rows // 128 for pl in plans])
    wc = [mx.cast_w32x32(w, transposed=False, dgrad_scales=True) for w in ws]
    # the all-to-all path
    y_recv = [ep.expert_forward(rq[r], rs[r], wc[r][0], wc[r][1], plans[r]) for r in range(W)]
    ys = _virtual_a2a(y_recv, [pl.recv_tokens for pl in plans], [pl.send_tokens for pl in plans])
    dy_recv = _virtual_a2a(dys, [pl.send_tokens for pl in plans], [pl.recv_tokens for pl in plans])
    back = [ep.expert_backward(dy_recv[r], rq[r], rs[r], wc[r][0], wc[r][3], plans[r]) for r in range(W)]
    dxs = _virtual_a2a([b[0] for b in back], [pl.recv_tokens for pl in plans], [pl.send_tokens for pl in plans])
    # fused: every expert rank stores into every sender's buffers (NaN-filled first)
    nan = lambda *sh: torch.full(sh, float("nan"), dtype=torch.bfloat16, device="cuda")
    ybuf = [nan(int(counts[s].sum()), N) for s in range(W)]
    dxbuf = [nan(int(counts[s].sum()), K) for s in range(W)]
    for r in range(W):
        ep.expert_forward_to_senders(rq[r], rs[r], wc[r][0], wc[r][1], dplans[r], [b.data_ptr() for b in ybuf])
        none, dw = ep.expert_backward(dy_recv[r], rq[r], rs[r], wc[r][0], wc[r][3], plans[r],
                                      dx_rows=dplans[r].combine_destinations([b.data_ptr() for b in dxbuf], K))
        assert none is None and torch.equal(dw, back[r][1]), f"dW of rank {r}"
    mx.mx_device_error()
    for s in range(W):
        assert torch.equal(ybuf[s], ys[s]), f"outputs of rank {s}"
        assert torch.equal(dxbuf[s], dxs[s]), f"dX of rank {s}"


@pytest.mark.parametrize("W,E,N", [(2, 3, 576), (4, 2, 256), (3, 1, 96)])
def test_direct_dy_dispatch_equals_the_experts_own_cast(mx, W, E, N):
    """The backward dispatch as one kernel (every rank's dY cast rowwise and
    columnwise straight into every expert's buffers), ranks emulated with local
    buffers: each rank's four outputs are bitwise what its own fused grouped
    cast of the dY the all-to-all delivers would write."""
    from mxfp8_block_scaled_cast_b200 import ep
    rng = np.random.default_rng(90 + W)
    counts = rng.integers(0, 260, size=(W, W * E))
    counts[0, -1] = 0
    counts[W - 1, :E] = 128
    dys = [S.normal_bf16((int(counts[r].sum()), N), 0.1, seed=95 + r).cuda() for r in range(W)]
    plans = [ep.ExchangePlan(W, E, counts[r], counts[:, r * E:(r + 1) * E]) for r in range(W)]
    dy_recv = _virtual_a2a(dys, [pl.send_tokens for pl in plans], [pl.recv_tokens for pl in plans])
    band = ep.scale_band_bytes(N)
    fill = lambda n: torch.full((n,), 0xA5, dtype=torch.uint8, device="cuda")
    bq = [fill(pl.m_cap_recv * N) for pl in plans]
    bs = [fill(pl.m_cap_recv // 128 * band) for pl in plans]
    bqt = [fill(N * pl.m_cap_recv) for pl in plans]
    bst = [fill(mx.mx_scale_bytes(N, pl.m_cap_recv // 32)) for pl in plans]
    ptrs = lambda bufs: [b.data_ptr() for b in bufs]
    for r in range(W):
        ep.dispatch_2d_direct(dys[r], ep.DirectPlan(W, E, r, counts), ptrs(bq), ptrs(bs), ptrs(bqt), ptrs(bst))
    mx.mx_device_error()
    for d, pl in enumerate(plans):
        if pl.M_recv == 0:
            continue
        offs = torch.as_tensor(pl.offs_recv()).cuda()
        q, s, qt, st = mx.cast_2d_grouped(dy_recv[d], offs, pl.m_cap_recv)
        assert torch.equal(bq[d], q.reshape(-1)), f"rowwise codes of rank {d}"
        assert torch.equal(bs[d], s.reshape(-1)), f"rowwise scales of rank {d}"
        assert torch.equal(bqt[d], qt.reshape(-1)), f"columnwise codes of rank {d}"
        assert torch.equal(bst[d], st.reshape(-1)), f"columnwise scales of rank {d}"


def test_autograd_entry_over_a_one_rank_nccl_group(mx):
    """mxfp8_expert_parallel_mm through autograd in both modes: y and the
    gradients bitwise those of the layer's own forward and backward; in the
    all-to-all mode two forwards (micro-batches) precede their backwards, run in
    reverse order, and the weight's accumulated gradient is the sum of both."""
    import torch.distributed as dist
    from mxfp8_block_scaled_cast_b200 import ep
    if dist.is_initialized():
        pytest.skip("a process group already exists")
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    from datetime import timedelta
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        E, N, K = 4, 512, 256
        counts = np.array([100, 0, 333, 129])
        M = int(counts.sum())
        x = S.normal_bf16((M, K), seed=60).cuda()
        x2 = S.normal_bf16((M, K), seed=63).cuda()
        w = S.normal_bf16((E, N, K), 0.02, seed=61).cuda()
        dy = S.normal_bf16((M, N), 0.1, seed=62).cuda()
        dy2 = S.normal_bf16((M, N), 0.1, seed=64).cuda()
        ref = ep.MXFP8ExpertParallelMM()
        y0 = ref.forward(x, counts, w)
        dx0, dw0 = ref.backward(dy)
        y2 = ref.forward(x2, counts, w)
        dx2, dw2 = ref.backward(dy2)
        for direct in (False, True):
            layer = ep.MXFP8ExpertParallelMM(direct=direct)
            xg, wg = x.clone().requires_grad_(), w.clone().requires_grad_()
            y = ep.mxfp8_expert_parallel_mm(xg, wg, counts, layer)
            y.backward(dy)
            assert torch.equal(y.detach(), y0), f"y (direct={direct})"
            assert torch.equal(xg.grad, dx0) and torch.equal(wg.grad, dw0), f"gradients (direct={direct})"
        layer = ep.MXFP8ExpertParallelMM()
        a, b = x.clone().requires_grad_(), x2.clone().requires_grad_()
        wg = w.clone().requires_grad_()
        ya = ep.mxfp8_expert_parallel_mm(a, wg, counts, layer)
        yb = ep.mxfp8_expert_parallel_mm(b, wg, counts, layer)
        yb.backward(dy2)
        ya.backward(dy)
        mx.mx_device_error()
        assert torch.equal(ya.detach(), y0) and torch.equal(yb.detach(), y2)
        assert torch.equal(a.grad, dx0) and torch.equal(b.grad, dx2)
        assert torch.equal(wg.grad, dw2 + dw0)
    finally:
        dist.destroy_process_group()
