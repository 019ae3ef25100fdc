"""Expert-parallel MoE grouped GEMM with the MXFP8 all-to-all.

With expert parallelism each of W ranks holds E of the W*E experts, and an
all-to-all moves every token to the rank of its expert and its output back.
The "MXFP8 all-to-all" (prime-rl PR #3388, Overview: MXFP8Config.enable_a2a,
with notes on when it helps and when it hurts; ao PR #4705, the two-GPU
expert-parallel pipeline benchmark) carries the dispatched tokens as MXFP8 --
one E4M3 byte per element plus one E8M0 byte per 32 -- instead of two bf16
bytes.

Layout (this implementation's reading; the pages describe no layout):
  * The sender casts its tokens rowwise (1x32 along K) straight into the
    padded group layout of the pad path with one group per global expert,
    ordered by destination rank. Each destination's groups are then one
    contiguous run of whole 128-row tiles: its codes are a row range of the
    code buffer and its scales a range of whole 512-byte blocked scale tiles,
    so each piece is one slice of the all-to-all.
  * The receiver's buffer is therefore the padded grouped operand of groups
    (source rank, local expert), source major -- exactly what the grouped
    GEMM reads, with group g using local expert g % E
    (mx_grouped_mm_experts). No unpack or rearrangement pass runs. The
    rowwise cast is per row, so the received codes are bitwise the codes the
    receiver would compute from the bf16 tokens.
  * Outputs return in bf16 by the reverse all-to-all (the combine), in the
    sender's token order.
  * Backward: dY goes to the experts in bf16 (the combine's reverse), the
    receiver casts it (rowwise for dX, columnwise per group for dW), and the
    wgrad's columnwise cast of the activations reads the received codes
    dequantized to bf16 -- the receiver never sees the bf16 activations;
    that double rounding is what the MXFP8 dispatch trades for bandwidth.
    dW of expert e sums its groups from every source rank in one GEMM.

Everything that moves data is torch.distributed.all_to_all_single (NCCL over
NVLink on GPUs) -- or, with direct=True, the kernels themselves storing into
symmetric memory: the rowwise cast of the tokens into the receivers' buffers,
the expert GEMMs' epilogue storing outputs and dX rows into the senders'
buffers, and in backward the fused cast of dY (rowwise and columnwise, per
group, bitwise what the receiver's own cast would write) into the experts'
buffers, so no all-to-all is left. Every arithmetic step is a libmx kernel.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import mx

BLOCK_ROWS = 128          # rows of a blocked scale tile: the pad path's group alignment
MAX_GROUPS = 1024         # groups the grouped casts and GEMMs take (include/mx.h)
DIRECT_MAX_GROUPS = 512   # groups the fused scatter cast takes (the direct mode's dY dispatch)


def _pad(n):
    return -(-int(n) // BLOCK_ROWS) * BLOCK_ROWS


def scale_band_bytes(K: int) -> int:
    """Bytes of the blocked scales of one 128-row band of a [rows, K] rowwise cast."""
    return mx.mx_scale_bytes(BLOCK_ROWS, K // 32)


@dataclass
class ExchangePlan:
    """Sizes of one rank's all-to-alls, from the token counts.

    send_counts[j]: tokens this rank sends to global expert j (W*E entries;
    rank r holds experts r*E .. r*E + E - 1); recv_counts[s, e]: tokens rank s
    sends to this rank's local expert e."""
    W: int
    E: int
    send_counts: np.ndarray
    recv_counts: np.ndarray

    def __post_init__(self):
        self.send_counts = np.asarray(self.send_counts, dtype=np.int64).reshape(-1)
        self.recv_counts = np.asarray(self.recv_counts, dtype=np.int64)
        if self.send_counts.size != self.W * self.E or self.recv_counts.size != self.W * self.E:
            raise ValueError(f"token counts must hold W*E = {self.W * self.E} entries")
        self.recv_counts = self.recv_counts.reshape(self.W, self.E)
        if (self.send_counts < 0).any() or (self.recv_counts < 0).any():
            raise ValueError("token counts must be >= 0")
        if self.W * self.E > MAX_GROUPS:
            raise ValueError(f"W*E = {self.W * self.E} groups exceed the grouped kernels' {MAX_GROUPS}")
        pad = np.array([_pad(c) for c in self.send_counts], dtype=np.int64).reshape(self.W, self.E)
        rpad = np.array([_pad(c) for c in self.recv_counts.reshape(-1)], dtype=np.int64).reshape(self.W, self.E)
        self.M = int(self.send_counts.sum())                          # tokens sent
        self.m_cap_send = int(pad.sum())                              # padded rows of the send buffer
        self.send_rows = pad.sum(axis=1)                              # padded rows to each rank
        self.send_tokens = self.send_counts.reshape(self.W, self.E).sum(axis=1)
        self.M_recv = int(self.recv_counts.sum())                     # tokens received
        self.m_cap_recv = int(rpad.sum())
        self.recv_rows = rpad.sum(axis=1)                             # padded rows from each rank
        self.recv_tokens = self.recv_counts.sum(axis=1)

    def offs_send(self) -> np.ndarray:
        """Cumulative group ends of the send layout (one group per global expert)."""
        return np.cumsum(self.send_counts).astype(np.int32)

    def offs_recv(self) -> np.ndarray:
        """Cumulative group ends of the receive layout: groups (source rank, local expert)."""
        return np.cumsum(self.recv_counts.reshape(-1)).astype(np.int32)

    @property
    def G_recv(self) -> int:
        return self.W * self.E


def exchange_counts(send_counts, W: int, E: int, a2a, device) -> np.ndarray:
    """recv_counts [W, E] from every rank's send_counts (one small all-to-all)."""
    send = torch.as_tensor(np.asarray(send_counts, dtype=np.int64), device=device)
    recv = torch.empty(W * E, dtype=torch.int64, device=device)
    a2a(recv, send, [E] * W, [E] * W)
    return recv.cpu().numpy().reshape(W, E)


def _splits(rows):
    return [int(r) for r in rows]


def dist_all_to_all(group=None):
    """all_to_all_single over `group` (output, input, output splits, input splits), in rows."""
    import torch.distributed as dist

    def a2a(out, inp, out_splits, in_splits):
        dist.all_to_all_single(out, inp, out_splits, in_splits, group=group)
    return a2a


# ----------------------------------------------------------- the pieces --
def pack_mxfp8(x, plan: ExchangePlan):
    """Rowwise cast of x [M, K] (tokens ordered by global expert) into the send
    layout: codes [m_cap_send, K] and blocked scales viewed as [bands, band bytes]."""
    M, K = x.shape
    offs = torch.as_tensor(plan.offs_send(), device=x.device)
    q = torch.empty(plan.m_cap_send, K, dtype=torch.uint8, device=x.device)
    s = torch.empty(mx.mx_scale_bytes(plan.m_cap_send, K // 32), dtype=torch.uint8, device=x.device)
    if plan.m_cap_send:
        mx.mx_cast_dim0_grouped(x, offs, plan.m_cap_send, q, s)
    return q, s.view(plan.m_cap_send // BLOCK_ROWS, scale_band_bytes(K))


def dispatch_mxfp8(q, s, plan: ExchangePlan, a2a):
    """The MXFP8 dispatch: codes by padded rows, scales by whole 128-row bands."""
    K = q.shape[1]
    rq = torch.empty(plan.m_cap_recv, K, dtype=torch.uint8, device=q.device)
    rs = torch.empty(plan.m_cap_recv // BLOCK_ROWS, s.shape[1], dtype=torch.uint8, device=q.device)
    a2a(rq, q, _splits(plan.recv_rows), _splits(plan.send_rows))
    a2a(rs, s, _splits(plan.recv_rows // BLOCK_ROWS), _splits(plan.send_rows // BLOCK_ROWS))
    return rq, rs


# --------------------------------------- the dispatch as one kernel ---
# The same exchange without a send buffer or an all-to-all: the rowwise cast
# writes each of this rank's token groups straight into its destination's
# receive buffer (mx_cast_dim0_grouped_scatter; the buffers are mapped into
# every rank, e.g. symmetric memory over NVLink). The receive layout is the
# one above, so everything downstream is unchanged. Every rank needs every
# rank's counts to know where its groups land: one all-gather replaces the
# all-to-all of the counts.
def gather_counts(send_counts, W: int, all_gather, device) -> np.ndarray:
    """counts [W, W*E]: tokens each rank sends to each global expert (one small
    all-gather; all_gather(out [W, n], inp [n]) as torch.distributed's)."""
    send = torch.as_tensor(np.asarray(send_counts, dtype=np.int64), device=device)
    out = torch.empty(W, send.numel(), dtype=torch.int64, device=device)
    all_gather(out, send)
    return out.cpu().numpy()


def dist_all_gather(group=None):
    """all_gather over `group` into the rows of `out` (output [W, n], input [n])."""
    import torch.distributed as dist

    def ag(out, inp):
        dist.all_gather(list(out.unbind(0)), inp, group=group)
    return ag


@dataclass
class DirectPlan:
    """Where rank `rank`'s token groups land in the receive buffers, from every
    rank's counts ([W, W*E]): rank d's buffer holds groups (source s, local
    expert e) source-major, each padded to whole 128-row tiles."""
    W: int
    E: int
    rank: int
    counts: np.ndarray

    def __post_init__(self):
        c = np.asarray(self.counts, dtype=np.int64)
        if c.shape != (self.W, self.W * self.E):
            raise ValueError(f"counts must be [W, W*E] = [{self.W}, {self.W * self.E}]")
        if not 0 <= self.rank < self.W:
            raise ValueError("rank outside [0, W)")
        self.counts = c
        self.exchange = ExchangePlan(self.W, self.E, c[self.rank], c[:, self.rank * self.E:(self.rank + 1) * self.E])
        pad = np.vectorize(_pad, otypes=[np.int64])(c) if c.size else c      # [W, W*E]
        rows = pad.reshape(self.W, self.W, self.E).sum(axis=2)               # rows[s, d]: s's rows to d
        start = np.concatenate([np.zeros((1, self.W), np.int64), np.cumsum(rows, axis=0)[:-1]])  # [s, d]
        self.recv_rows_of = rows.sum(axis=0)                                 # m_cap_recv of each rank
        mine = pad[self.rank].reshape(self.W, self.E)
        within = np.concatenate([np.zeros((self.W, 1), np.int64), np.cumsum(mine, axis=1)[:, :-1]], axis=1)
        self.dst_row = (start[self.rank][:, None] + within).reshape(-1)     # per global expert g

    def destinations(self, base_q, base_s, K: int):
        """Device addresses of each group's first row of codes and first scale
        band, given every rank's receive code and scale buffer addresses."""
        band = scale_band_bytes(K)
        dq, ds = [], []
        for g, row in enumerate(self.dst_row):
            d = g // self.E
            dq.append(int(base_q[d]) + int(row) * K)
            ds.append(int(base_s[d]) + int(row) // BLOCK_ROWS * band)
        return dq, ds


    def destinations_2d(self, base_q, base_s, base_qt, base_st, K: int):
        """Destinations of the fused (rowwise + columnwise) dispatch, e.g. of dY in
        backward: each group's rowwise codes and scale bands as destinations(),
        its first padded token column in the receiving rank's columnwise codes
        [K, cap_d] and its first tile of their blocked(K, cap_d/32) scales, and
        cap_d (the receiving rank's padded capacity, the row stride there)."""
        dq, ds = self.destinations(base_q, base_s, K)
        dqt, dst, cap = [], [], []
        for g, row in enumerate(self.dst_row):
            d = g // self.E
            dqt.append(int(base_qt[d]) + int(row))
            dst.append(int(base_st[d]) + int(row) // BLOCK_ROWS * 512)
            cap.append(int(self.recv_rows_of[d]))
        return dq, ds, dqt, dst, cap

    def combine_destinations(self, out_base, width: int, itemsize: int = 2):
        """Device addresses where each group this rank receives sends its output
        rows: group (source s, local expert e) -> rank s's output buffer
        (out_base[s], [M_s, width] rows of `itemsize` bytes, in s's token
        order) at s's first token of global expert rank*E + e."""
        starts = np.concatenate([np.zeros((self.W, 1), np.int64), np.cumsum(self.counts, axis=1)[:, :-1]], axis=1)
        return [int(out_base[s]) + int(starts[s, self.rank * self.E + e]) * width * itemsize
                for s in range(self.W) for e in range(self.E)]


def dispatch_mxfp8_direct(x, plan: DirectPlan, base_q, base_s):
    """The MXFP8 dispatch as one kernel: x [M, K] (tokens ordered by global
    expert) cast rowwise straight into every rank's receive buffer (base_q[d],
    base_s[d]: rank d's codes [rows, K] and scale bands as mapped on this
    rank). The ranks must wait for one another (a collective issued after this
    on the stream) before any of them reads its buffer."""
    M, K = x.shape
    ex = plan.exchange
    if ex.m_cap_send == 0:
        return
    offs = torch.as_tensor(ex.offs_send(), device=x.device)
    dq, ds = plan.destinations(base_q, base_s, K)
    mx.mx_cast_dim0_grouped_scatter(x, offs, ex.m_cap_send, dq, ds)


def dispatch_2d_direct(t, plan: DirectPlan, base_q, base_s, base_qt, base_st):
    """The backward dispatch as one kernel: t [M, C] (tokens ordered by global
    expert; dY in backward) cast rowwise and columnwise straight into every
    rank's buffers (rank d's rowwise codes [rows, C] and scale bands, its
    columnwise codes [C, cap_d] and their scale tiles, as mapped on this rank),
    exactly as rank d's own fused grouped cast of the rows it receives would
    write them. The ranks must wait for one another before reading."""
    M, C = t.shape
    ex = plan.exchange
    if ex.m_cap_send == 0:
        return
    offs = torch.as_tensor(ex.offs_send(), device=t.device)
    dq, ds, dqt, dst, cap = plan.destinations_2d(base_q, base_s, base_qt, base_st, C)
    mx.mx_cast_2d_grouped_scatter(t, offs, ex.m_cap_send, dq, ds, dqt, dst, cap)


def expert_forward_to_senders(rq, rs, wq, wsf, plan: DirectPlan, y_base):
    """The expert GEMMs with the combine fused: each received group's outputs
    stored straight into the rank that sent its tokens (y_base[s]: rank s's
    output buffer [M_s, N] bf16 as mapped here), tile by tile as the GEMM runs.
    The ranks must wait for one another before reading their outputs."""
    ex = plan.exchange
    N, K = wq.shape[1], wq.shape[2]
    if ex.M_recv == 0:
        return
    offs = torch.as_tensor(ex.offs_recv(), device=rq.device)
    mx.mx_grouped_mm_experts_to_rows(rq, rs, wq, wsf, offs, ex.G_recv, ex.E, mx.MX_GROUPS_M,
                                     plan.combine_destinations(y_base, N), ex.M_recv, N, K, ex.m_cap_recv)


def expert_forward(rq, rs, wq, wsf, plan: ExchangePlan):
    """y_recv [M_recv, N] bf16 = each received group times its local expert (g % E)."""
    N, K = wq.shape[1], wq.shape[2]
    y = torch.empty(plan.M_recv, N, dtype=torch.bfloat16, device=rq.device)
    if plan.M_recv:
        offs = torch.as_tensor(plan.offs_recv(), device=rq.device)
        mx.mx_grouped_mm_experts(rq, rs, wq, wsf, offs, plan.G_recv, plan.E, mx.MX_GROUPS_M, y, plan.M_recv, N, K,
                                 plan.m_cap_recv)
    return y


def combine(y_recv, plan: ExchangePlan, a2a):
    """Outputs back to their senders (bf16), in the sender's token order."""
    y = torch.empty(plan.M, y_recv.shape[1], dtype=y_recv.dtype, device=y_recv.device)
    a2a(y, y_recv, _splits(plan.send_tokens), _splits(plan.recv_tokens))
    return y


def dispatch_bf16(t, plan: ExchangePlan, a2a):
    """A bf16 tensor in the sender's token order to the experts' ranks (dY in backward)."""
    out = torch.empty(plan.M_recv, t.shape[1], dtype=t.dtype, device=t.device)
    a2a(out, t, _splits(plan.recv_tokens), _splits(plan.send_tokens))
    return out


def expert_backward(dy_recv, rq, rs, wq, wsd, plan: ExchangePlan, dx_rows=None):
    """(dx_recv [M_recv, K], dw [E, N, K]) of the received groups.

    dX = dY W_e (dY cast rowwise along N, W's forward codes read MN-major);
    dW_e = sum over the groups of expert e of dY_g^T X_g, both cast columnwise
    per group, X from the received codes dequantized to bf16. With dx_rows
    (one device address per received group: where its dX rows go, e.g. into
    the senders' buffers) dX is stored there and dx_recv is None."""
    if plan.M_recv == 0:
        return expert_backward_from_codes(None, None, None, None, rq, rs, wq, wsd, plan, dx_rows)
    offs = torch.as_tensor(plan.offs_recv(), device=dy_recv.device)
    dq, ds, dqt, dst = mx.cast_2d_grouped(dy_recv, offs, plan.m_cap_recv)
    return expert_backward_from_codes(dq, ds, dqt, dst, rq, rs, wq, wsd, plan, dx_rows)


def expert_backward_from_codes(dq, ds, dqt, dst, rq, rs, wq, wsd, plan: ExchangePlan, dx_rows=None):
    """expert_backward from dY already cast both ways in the receive layout (dq
    [m_cap_recv, N] and its scales, dqt [N, m_cap_recv] and its scales: what
    the fused grouped cast of the received dY writes, or what the senders'
    dispatch_2d_direct stored there)."""
    E, N, K = wq.shape
    dev = rq.device
    dw = torch.empty(E, N, K, dtype=torch.bfloat16, device=dev)
    dx = None if dx_rows is not None else torch.empty(plan.M_recv, K, dtype=torch.bfloat16, device=dev)
    if plan.M_recv == 0:
        dw.zero_()
        return dx, dw
    offs = torch.as_tensor(plan.offs_recv(), device=dev)
    G, cap = plan.G_recv, plan.m_cap_recv
    if dx_rows is not None:
        mx.mx_grouped_mm_experts_to_rows(dq, ds, wq, wsd, offs, G, E, mx.MX_GROUPS_M_KN, dx_rows, plan.M_recv, K, N,
                                         cap)
    else:
        mx.mx_grouped_mm_experts(dq, ds, wq, wsd, offs, G, E, mx.MX_GROUPS_M_KN, dx, plan.M_recv, K, N, cap)
    x_deq = torch.empty(plan.M_recv, K, dtype=torch.bfloat16, device=dev)
    mx.mx_dequant_dim0_grouped(rq, rs.reshape(-1), offs, plan.M_recv, K, cap, x_deq)
    xqt, xst = mx.cast_dim1_grouped(x_deq, offs, cap)
    mx.mx_grouped_mm_experts(dqt, dst, xqt, xst, offs, G, E, mx.MX_GROUPS_K, dw, plan.M_recv, N, K, cap)
    return dx, dw


def return_grad(dx_recv, plan: ExchangePlan, a2a):
    """dX back to the senders (bf16), in the sender's token order."""
    return combine(dx_recv, plan, a2a)


# ------------------------------------------------------------- the layer --
class MXFP8ExpertParallelMM:
    """y[tokens of expert j] = x[tokens of expert j] @ w_j^T with the experts
    sharded over the ranks of `group` and the dispatch in MXFP8.

    forward(x [M, K] bf16 ordered by global expert, send_counts [W*E] tokens
    per global expert, w [E, N, K] bf16 local experts) -> y [M, N];
    backward(dy [M, N]) -> (dx [M, K], dw [E, N, K]). `a2a` defaults to
    torch.distributed.all_to_all_single over `group`.

    direct=True fuses the exchanges into the kernels: the dispatch is the
    rowwise cast storing each tile straight into the receiving rank's buffer,
    and the combine (and, in backward, the return of dX) is the expert GEMM's
    epilogue storing each output row straight into the rank that sent the
    token; in backward each sender casts dY rowwise and columnwise straight
    into the experts' buffers. The buffers are
    symmetric memory (every rank's mapped into every rank) written with plain
    stores (no TMA, no multicast); a one-element all-reduce, ordered on the
    stream after each such call, is the barrier before anyone reads. The
    buffers are kept and grown collectively (every rank computes the same
    sizes from the gathered counts); outputs are copied out of them, and the
    received codes the backward reads stay in them, so a second forward of
    the same layer before its backward is refused. No all-to-all is left on
    this path."""

    def __init__(self, group=None, a2a=None, direct=False, all_gather=None):
        import torch.distributed as dist
        self.group = group
        self.W = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.a2a = a2a if a2a is not None else dist_all_to_all(group)
        self.direct = direct
        self.all_gather = all_gather if all_gather is not None else (dist_all_gather(group) if direct else None)
        self._symm_bufs = {}          # direct mode: name -> (buffer, handle, bytes)
        self._saved = None

    def _symm(self, name: str, nbytes: int, device):
        """A symmetric-memory byte buffer of at least nbytes and every rank's
        address of it; (re)allocated collectively when it must grow."""
        cur = self._symm_bufs.get(name)
        if cur is None or cur[2] < nbytes:
            import torch.distributed as dist
            import torch.distributed._symmetric_memory as symm_mem
            size = max(int(nbytes), 512)
            buf = symm_mem.empty(size, dtype=torch.uint8, device=device)
            grp = self.group if self.group is not None else dist.group.WORLD
            cur = (buf, symm_mem.rendezvous(buf, grp.group_name), size)
            self._symm_bufs[name] = cur
        return cur[0], [int(p) for p in cur[1].buffer_ptrs]

    def _barrier(self, device):
        import torch.distributed as dist
        flag = torch.zeros(1, dtype=torch.float32, device=device)
        dist.all_reduce(flag, group=self.group)      # every rank's stores are in before anyone reads

    def _forward_direct(self, x, send_counts, w):
        E, N, K = w.shape
        if self.W * E > DIRECT_MAX_GROUPS:
            raise ValueError(f"direct mode takes at most {DIRECT_MAX_GROUPS} groups (ranks x local experts), "
                             f"got {self.W} x {E}")
        dev = x.device
        counts = gather_counts(send_counts, self.W, self.all_gather, dev)
        plan = DirectPlan(self.W, E, self.rank, counts)
        ex = plan.exchange
        rows = int(plan.recv_rows_of.max())
        band = scale_band_bytes(K)
        rbuf, rbase = self._symm("recv", rows * K + rows // BLOCK_ROWS * band, dev)
        dispatch_mxfp8_direct(x, plan, rbase, [b + rows * K for b in rbase])
        self._barrier(dev)
        rq = rbuf[:ex.m_cap_recv * K].view(ex.m_cap_recv, K)
        rs = rbuf[rows * K:rows * K + ex.m_cap_recv // BLOCK_ROWS * band].view(-1, band)
        wq, wsf, _, wsd = mx.cast_w32x32(w, transposed=False, dgrad_scales=True)
        m_max = int(counts.sum(axis=1).max())
        ybuf, ybase = self._symm("y", m_max * N * 2, dev)
        expert_forward_to_senders(rq, rs, wq, wsf, plan, ybase)
        self._barrier(dev)
        y = ybuf[:ex.M * N * 2].view(torch.bfloat16).view(ex.M, N).clone()
        self._saved = (plan, rq, rs, wq, wsd)
        return y

    def _backward_direct(self, dy):
        plan, rq, rs, wq, wsd = self._saved
        self._saved = None
        ex = plan.exchange
        E, N, K = wq.shape
        dev = dy.device
        # dY cast both ways by its senders straight into one symmetric buffer per
        # rank: rowwise codes [rows, N], their scale bands, columnwise codes
        # [N, cap] (this rank reads them with its own cap as the row stride)
        # and their scale tiles; every region starts on a 512-byte boundary
        rows = int(plan.recv_rows_of.max())
        band = scale_band_bytes(N)
        o_s = rows * N
        o_qt = o_s + rows // BLOCK_ROWS * band
        o_st = o_qt + N * rows
        dbuf, dbase = self._symm("dy", o_st + mx.mx_scale_bytes(N, rows // 32), dev)
        dispatch_2d_direct(dy.contiguous(), plan, dbase, [b + o_s for b in dbase], [b + o_qt for b in dbase],
                           [b + o_st for b in dbase])
        self._barrier(dev)
        cap = ex.m_cap_recv
        dq = dbuf[:cap * N].view(cap, N)
        ds = dbuf[o_s:o_s + cap // BLOCK_ROWS * band]
        dqt = dbuf[o_qt:o_qt + N * cap].view(N, cap)
        dst = dbuf[o_st:o_st + mx.mx_scale_bytes(N, cap // 32)]
        m_max = int(plan.counts.sum(axis=1).max())
        dxbuf, dxbase = self._symm("dx", m_max * K * 2, dev)
        _, dw = expert_backward_from_codes(dq, ds, dqt, dst, rq, rs, wq, wsd, ex,
                                           dx_rows=plan.combine_destinations(dxbase, K))
        self._barrier(dev)
        return dxbuf[:ex.M * K * 2].view(torch.bfloat16).view(ex.M, K).clone(), dw

    def forward(self, x, send_counts, w):
        for name, t in (("x", x), ("w", w)):
            if t.dtype != torch.bfloat16:
                raise TypeError(f"MXFP8ExpertParallelMM takes bf16 operands ({name} is {t.dtype})")
        x, w = x.contiguous(), w.contiguous()
        E = w.shape[0]
        if int(np.sum(send_counts)) != x.shape[0]:
            raise ValueError("send_counts must sum to the number of tokens")
        if self.direct:
            if self._saved is not None:
                raise RuntimeError("direct mode: the previous forward's backward has not run (its "
                                   "receive buffer would be overwritten)")
            return self._forward_direct(x, send_counts, w)
        recv = exchange_counts(send_counts, self.W, E, self.a2a, x.device)
        plan = ExchangePlan(self.W, E, send_counts, recv)
        q, s = pack_mxfp8(x, plan)
        rq, rs = dispatch_mxfp8(q, s, plan, self.a2a)
        wq, wsf, _, wsd = mx.cast_w32x32(w, transposed=False, dgrad_scales=True)
        y = combine(expert_forward(rq, rs, wq, wsf, plan), plan, self.a2a)
        self._saved = (plan, rq, rs, wq, wsd)
        return y

    def backward(self, dy):
        if self._saved is None:
            raise RuntimeError("backward before forward")
        if dy.dtype != torch.bfloat16:
            raise TypeError("MXFP8ExpertParallelMM takes a bf16 gradient")
        if self.direct:
            return self._backward_direct(dy)
        plan, rq, rs, wq, wsd = self._saved
        self._saved = None
        dy_recv = dispatch_bf16(dy.contiguous(), plan, self.a2a)
        dx_recv, dw = expert_backward(dy_recv, rq, rs, wq, wsd, plan)
        return return_grad(dx_recv, plan, self.a2a), dw


class _ExpertParallelFn(torch.autograd.Function):
    """Autograd wrapper of MXFP8ExpertParallelMM: forward and backward are the
    layer's calls, collectives included (every rank runs them in the same
    order). In the all-to-all mode the forward's state moves into the autograd
    context, so several forwards (micro-batches) may precede their backwards,
    in any order; direct mode keeps it in the layer, whose receive buffers hold
    the codes the backward reads, and so refuses a second forward before the
    backward."""

    @staticmethod
    def forward(ctx, x, w, send_counts, layer):
        y = layer.forward(x, send_counts, w)
        ctx.layer = layer
        if not layer.direct:
            ctx.state, layer._saved = layer._saved, None
        return y

    @staticmethod
    def backward(ctx, dy):
        layer, ctx.layer = ctx.layer, None
        if not layer.direct:
            layer._saved, ctx.state = ctx.state, None
        dx, dw = layer.backward(dy)
        return dx, dw, None, None


def mxfp8_expert_parallel_mm(x, w, send_counts, layer):
    """y = the expert-parallel MXFP8 MoE layer `layer` (an MXFP8ExpertParallelMM)
    on x [M, K] (tokens ordered by global expert, send_counts tokens per global
    expert) with this rank's experts w [E, N, K]; differentiable in x and w."""
    return _ExpertParallelFn.apply(x, w, send_counts, layer)
