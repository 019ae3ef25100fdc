"""Expert-parallel MXFP8 all-to-all on CPU: two gloo ranks, the exchange layout.

The MXFP8 dispatch (prime-rl PR #3388, Overview, enable_a2a) sends each
rank's tokens, cast rowwise into the padded group layout ordered by
destination rank, as codes and whole 128-row blocked scale tiles. Here the
oracle does the cast on each rank (no GPU), the library's own exchange
functions (ExchangePlan, exchange_counts, dispatch_mxfp8, combine,
dispatch_bf16) move the bytes over a real two-rank gloo group, and every
receiver checks that its buffer is bitwise the oracle's padded grouped
operand of the tokens it should hold -- groups (source rank, local expert),
source major -- and that the combine returns every row to its sender in
order.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
W, E, K = 2, 3, 96          # ranks, experts per rank, hidden size (not a multiple of 128)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _counts(rank):
    rng = np.random.default_rng(200 + rank)
    c = rng.integers(0, 300, size=W * E)
    c[rank] = 0                               # an empty group
    c[-1] = 128 * (rank + 1)                  # and an exact multiple of the tile
    return c


def _tokens(rank):
    from mxfp8_block_scaled_cast_b200 import synthetic as S
    return S.bf16_bits(S.normal_bf16((int(_counts(rank).sum()), K), seed=100 + rank))


def _worker(rank, port, q):
    try:
        sys.path.insert(0, ROOT)
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        import torch
        import torch.distributed as dist
        from oracle import mx_oracle as O
        from mxfp8_block_scaled_cast_b200 import ep
        dist.init_process_group("gloo", rank=rank, world_size=W)
        a2a = ep.dist_all_to_all()
        counts = [_counts(r) for r in range(W)]
        xs = [_tokens(r) for r in range(W)]

        recv = ep.exchange_counts(counts[rank], W, E, a2a, "cpu")
        assert np.array_equal(recv, np.stack([counts[s][rank * E:(rank + 1) * E] for s in range(W)]))
        plan = ep.ExchangePlan(W, E, counts[rank], recv)

        # pack (the oracle's rowwise cast into the send layout) and dispatch
        qs, ss = O.cast_dim0_grouped(xs[rank], plan.offs_send(), plan.m_cap_send)
        sb = O.swizzle(ss)
        assert sb.size == plan.m_cap_send // 128 * ep.scale_band_bytes(K)
        q_t = torch.from_numpy(qs)
        s_t = torch.from_numpy(sb).view(plan.m_cap_send // 128, ep.scale_band_bytes(K))
        rq, rs = ep.dispatch_mxfp8(q_t, s_t, plan, a2a)

        # what this rank must hold: source s's tokens of global experts rank*E + e, source major
        ends = [np.cumsum(c) for c in counts]
        rows, origin = [], []
        for s in range(W):
            for e in range(E):
                j = rank * E + e
                lo = ends[s][j - 1] if j else 0
                rows.append(xs[s][lo:ends[s][j]])
                origin += [(s, i) for i in range(lo, ends[s][j])]
        x_recv = np.concatenate(rows)
        assert x_recv.shape[0] == plan.M_recv
        qe, se = O.cast_dim0_grouped(x_recv, plan.offs_recv(), plan.m_cap_recv)
        assert np.array_equal(rq.numpy(), qe), "received codes differ from the padded grouped operand"
        assert np.array_equal(rs.numpy().reshape(-1), O.swizzle(se)), "received scale tiles differ"

        # combine: each received row carries its origin, and must come back to it in order
        y_recv = torch.tensor([s * 1e6 + i for s, i in origin], dtype=torch.float64).reshape(-1, 1).repeat(1, 4)
        y = ep.combine(y_recv, plan, a2a)
        want = rank * 1e6 + np.arange(plan.M, dtype=np.float64)
        assert np.array_equal(y[:, 0].numpy(), want) and np.array_equal(y[:, 3].numpy(), want)

        # dispatch of a bf16 gradient follows the same rows as the tokens
        dy = torch.from_numpy(xs[rank].astype(np.int16)).view(torch.bfloat16)
        dy_recv = ep.dispatch_bf16(dy, plan, a2a)
        assert np.array_equal(dy_recv.view(torch.int16).numpy().view(np.uint16), x_recv)
        dist.destroy_process_group()
        q.put((rank, "ok"))
    except Exception as exc:  # reported to the parent
        import traceback
        q.put((rank, traceback.format_exc()))
        raise SystemExit(1) from exc


def test_mxfp8_dispatch_layout_and_combine_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(W)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=120)
    assert res == {0: "ok", 1: "ok"}, res
    assert all(p.exitcode == 0 for p in procs)


def test_plan_sizes_on_the_host():
    from mxfp8_block_scaled_cast_b200 import ep
    send = np.array([0, 5, 128, 129, 1, 0])            # W = 2, E = 3
    recv = np.array([[3, 0, 200], [128, 7, 0]])
    p = ep.ExchangePlan(2, 3, send, recv)
    assert p.M == 263 and p.m_cap_send == 0 + 128 + 128 + 256 + 128 + 0
    assert list(p.send_rows) == [256, 384] and list(p.send_tokens) == [133, 130]
    assert p.M_recv == 338 and p.m_cap_recv == 128 + 0 + 256 + 128 + 128 + 0
    assert list(p.recv_rows) == [384, 256] and list(p.recv_tokens) == [203, 135]
    assert list(p.offs_recv()) == [3, 3, 203, 331, 338, 338] and p.G_recv == 6
    assert ep.scale_band_bytes(96) == 128 * 4 and ep.scale_band_bytes(4096) == 128 * 128


def test_module_rejects_bad_arguments_before_any_exchange():
    """Host-side checks of the layer run before any collective or kernel."""
    import pytest
    import torch
    from mxfp8_block_scaled_cast_b200 import ep
    layer = ep.MXFP8ExpertParallelMM(a2a=lambda *a: pytest.fail("no exchange expected"))
    x = torch.zeros(10, 64, dtype=torch.bfloat16)
    w = torch.zeros(2, 64, 64, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        layer.forward(x.float(), [5, 5], w)
    with pytest.raises(ValueError):
        layer.forward(x, [5, 4], w)                 # counts must cover every token
    with pytest.raises(RuntimeError):
        layer.backward(torch.zeros(10, 64, dtype=torch.bfloat16))


def _dead_peer_worker(rank, port, q, direct=False):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    import torch.distributed as dist
    from mxfp8_block_scaled_cast_b200 import ep
    dist.init_process_group("gloo", rank=rank, world_size=2, timeout=timedelta(seconds=5))
    if rank == 1:
        q.put((1, "left"))
        q.close()
        q.join_thread()                          # the message is out before the process goes
        os._exit(0)                              # dies between steps, nothing in flight
    import time
    t0 = time.monotonic()
    try:
        if direct:                               # direct mode's first exchange: the count all-gather
            ep.gather_counts(np.array([1, 2, 3, 4]), 2, ep.dist_all_gather(), "cpu")
        else:
            ep.exchange_counts(np.array([1, 2, 3, 4]), 2, 2, ep.dist_all_to_all(), "cpu")
        q.put((0, "no error"))
    except Exception as exc:                     # the collective must end with an error
        q.put((0, f"error after {time.monotonic() - t0:.0f} s: {type(exc).__name__}"))


@pytest.mark.parametrize("direct", [False, True])
def test_exchange_with_a_dead_peer_ends_with_an_error(direct):
    """A rank that leaves between steps: the other rank's first exchange of a step (the
    all-to-all of the token counts, or in direct mode their all-gather) ends with an error
    within the group's timeout instead of waiting for good."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dead_peer_worker, args=(r, port, q, direct)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    assert res[1] == "left"
    assert res[0].startswith("error"), res


def test_plan_rejects_inconsistent_counts():
    import pytest
    from mxfp8_block_scaled_cast_b200 import ep
    with pytest.raises(ValueError):
        ep.ExchangePlan(2, 2, [1, 2, 3], [[1, 1], [1, 1]])          # send counts not W*E
    with pytest.raises(ValueError):
        ep.ExchangePlan(2, 2, [1, 2, 3, -1], [[1, 1], [1, 1]])      # negative count
    with pytest.raises(ValueError):
        ep.ExchangePlan(64, 17, [0] * (64 * 17), [[0] * 17] * 64)   # more groups than the kernels take


def test_direct_plan_places_groups_in_each_receive_layout():
    """The one-kernel dispatch's placement: rank r's group for global expert
    d*E + e starts at the padded start of group (r, e) in rank d's receive
    layout -- ExchangePlan's, which the expert GEMMs read."""
    from mxfp8_block_scaled_cast_b200 import ep
    rng = np.random.default_rng(11)
    for W, E in ((3, 2), (4, 1), (2, 5)):
        c = rng.integers(0, 300, size=(W, W * E))
        c[0, :] = 0
        c[-1, 0] = 128
        for r in range(W):
            p = ep.DirectPlan(W, E, r, c)
            for d in range(W):
                ex = ep.ExchangePlan(W, E, c[d], c[:, d * E:(d + 1) * E])
                assert p.recv_rows_of[d] == ex.m_cap_recv
                starts = np.concatenate([[0], np.cumsum([-(-v // 128) * 128 for v in ex.recv_counts.reshape(-1)])])
                for e in range(E):
                    assert p.dst_row[d * E + e] == starts[r * E + e]
            K = 96
            bq = [1 << 20 * (d + 1) for d in range(W)]
            bs = [(1 << 20 * (d + 1)) + (1 << 19) for d in range(W)]
            dq, ds = p.destinations(bq, bs, K)
            for g in range(W * E):
                d = g // E
                assert dq[g] == bq[d] + int(p.dst_row[g]) * K
                assert ds[g] == bs[d] + int(p.dst_row[g]) // 128 * ep.scale_band_bytes(K)
            # the fused (backward) dispatch: the columnwise outputs at the group's padded
            # token column of rank d's [K, cap_d] codes and its 512-byte scale tile there
            bqt = [(3 << 40) + (1 << 20 * (d + 1)) for d in range(W)]
            bst = [(5 << 40) + (1 << 20 * (d + 1)) for d in range(W)]
            dq2, ds2, dqt, dst, cap = p.destinations_2d(bq, bs, bqt, bst, K)
            assert dq2 == dq and ds2 == ds
            for g in range(W * E):
                d = g // E
                assert cap[g] == p.recv_rows_of[d]
                assert dqt[g] == bqt[d] + int(p.dst_row[g])
                assert dst[g] == bst[d] + int(p.dst_row[g]) // 128 * 512
    with pytest.raises(ValueError):
        ep.DirectPlan(2, 2, 0, np.zeros((2, 3)))
    with pytest.raises(ValueError):
        ep.DirectPlan(2, 2, 2, np.zeros((2, 4)))


def _gather_worker(rank, port, q):
    try:
        sys.path.insert(0, ROOT)
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        import torch.distributed as dist
        from mxfp8_block_scaled_cast_b200 import ep
        dist.init_process_group("gloo", rank=rank, world_size=W)
        counts = [_counts(r) for r in range(W)]
        full = ep.gather_counts(counts[rank], W, ep.dist_all_gather(), "cpu")
        assert np.array_equal(full, np.stack(counts))
        recv = ep.exchange_counts(counts[rank], W, E, ep.dist_all_to_all(), "cpu")
        dp = ep.DirectPlan(W, E, rank, full)
        xp = ep.ExchangePlan(W, E, counts[rank], recv)
        assert dp.exchange.m_cap_recv == xp.m_cap_recv and dp.exchange.m_cap_send == xp.m_cap_send
        assert np.array_equal(dp.exchange.offs_recv(), xp.offs_recv())
        dist.destroy_process_group()
        q.put((rank, "ok"))
    except Exception as exc:  # reported to the parent
        import traceback
        q.put((rank, traceback.format_exc()))
        raise SystemExit(1) from exc


def test_gathered_counts_give_the_same_plan_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_worker, args=(r, port, q)) for r in range(W)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=120)
    assert res == {0: "ok", 1: "ok"}, res


def test_direct_mode_refuses_more_groups_than_the_fused_scatter_takes():
    """Direct mode dispatches dY through the fused scatter cast, which takes at
    most 512 groups (ranks x local experts): refused before any work."""
    import torch
    from mxfp8_block_scaled_cast_b200 import ep
    layer = ep.MXFP8ExpertParallelMM(direct=True, a2a=lambda *a: None, all_gather=lambda *a: None)
    E = ep.DIRECT_MAX_GROUPS + 1
    x = torch.zeros(E, 32, dtype=torch.bfloat16)
    w = torch.zeros(E, 32, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="at most 512 groups"):
        layer.forward(x, np.ones(E, dtype=np.int64), w)
