"""The MoE layer's forward and backward captured once in a CUDA graph and
replayed under new routing.

Group boundaries are read from the offsets on the device -- the casts' group
lookup and the GEMM tile schedulers scan them there, and nothing on the host
reads a device value -- so overwriting the offsets tensor (and the tokens)
between replays re-routes the step without a new capture. Every replay must
equal an eager run of the layer on the same inputs bitwise, for each backward
arm, including routings with empty groups and one group holding every token.
"""
import numpy as np
import pytest
import torch

from mxfp8_block_scaled_cast_b200 import synthetic as S

pytestmark = pytest.mark.gpu

G, M, N, K = 4, 1024, 256, 384
ROUTINGS = [[256, 256, 256, 256], [1000, 0, 24, 0], [0, 0, 0, 1024], [77, 300, 129, 518]]


@pytest.fixture(scope="module")
def mx():
    from mxfp8_block_scaled_cast_b200 import mx as _mx
    _mx.lib()
    return _mx


@pytest.mark.parametrize("arm", [None, "high_precision", "dequantized"])
def test_step_captured_once_replays_under_new_routing(mx, arm):
    x = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    dy = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    w = S.normal_bf16((G, N, K), 0.02, seed=3, device="cuda")
    offs = torch.empty(G, dtype=torch.int32, device="cuda")

    def load(i):
        x.copy_(S.normal_bf16((M, K), seed=10 + i, device="cuda"))
        dy.copy_(S.normal_bf16((M, N), 0.1, seed=20 + i, device="cuda"))
        offs.copy_(torch.as_tensor(np.cumsum(ROUTINGS[i]), dtype=torch.int32))

    def step():
        op = mx.MXFP8GroupedMM(backward_override=arm)
        y = op.forward(x, w, offs)
        dx, dw = op.backward(dy)
        return y, dx, dw

    load(0)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):          # warm-up outside the capture
        step()
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        outs = step()
    for i in range(len(ROUTINGS)):
        load(i)
        graph.replay()
        torch.cuda.synchronize()
        ref = step()
        torch.cuda.synchronize()
        mx.mx_device_error()
        for name, got, want in zip(("y", "dx", "dw"), outs, ref):
            assert torch.equal(got, want), f"{name} under routing {ROUTINGS[i]} ({arm})"
        for g in np.flatnonzero(np.asarray(ROUTINGS[i]) == 0):
            assert not outs[2][g].any(), f"dW of empty group {g} must be exact zeros"
    del graph


@pytest.mark.parametrize("train", [False, True])
def test_linear_captured_once_replays_new_inputs(mx, train):
    """The linear forward and backward without the weight cache (the cache decides
    hit or miss on the host, once, at capture), with its workspace: one capture,
    replays on new x, w and dy bitwise equal to eager calls. Sizes off the GEMM
    tile (N = 96, K = 576) take the pad path. Both the separate calls and the
    training pair (whose backward reads the forward's casts from the workspace)."""
    Ml, Nl, Kl = 256, 96, 576
    x = torch.empty(Ml, Kl, dtype=torch.bfloat16, device="cuda")
    w = torch.empty(Nl, Kl, dtype=torch.bfloat16, device="cuda")
    dy = torch.empty(Ml, Nl, dtype=torch.bfloat16, device="cuda")
    ws = mx.linear_workspace(Ml, Nl, Kl, train=train)
    outs = [torch.empty(Ml, Nl, dtype=torch.bfloat16, device="cuda"),
            torch.empty(Ml, Kl, dtype=torch.bfloat16, device="cuda"),
            torch.empty(Nl, Kl, dtype=torch.bfloat16, device="cuda")]

    def load(i):
        x.copy_(S.normal_bf16((Ml, Kl), seed=30 + i, device="cuda"))
        w.copy_(S.normal_bf16((Nl, Kl), 0.02, seed=40 + i, device="cuda"))
        dy.copy_(S.normal_bf16((Ml, Nl), 0.1, seed=50 + i, device="cuda"))

    def step(y, dx, dw):
        if train:
            mx.mx_linear_fwd_train(x, w, None, 0, y, ws)
            mx.mx_linear_bwd_after_fwd(dy, w, None, 0, dx, dw, ws)
        else:
            mx.mx_linear_fwd(x, w, None, 0, y, ws)
            mx.mx_linear_bwd(dy, x, w, None, 0, dx, dw, ws)

    load(0)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(*outs)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(*outs)
    refs = [torch.empty_like(o) for o in outs]
    for i in range(3):
        load(i)
        graph.replay()
        torch.cuda.synchronize()
        step(*refs)
        torch.cuda.synchronize()
        mx.mx_device_error()
        for name, got, want in zip(("y", "dx", "dw"), outs, refs):
            assert torch.equal(got, want), f"linear {name}, inputs {i}"
    del graph

