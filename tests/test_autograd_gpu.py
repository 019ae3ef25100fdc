"""The autograd entry points give exactly the library calls' results."""
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


@pytest.mark.parametrize("arm", [None, "high_precision", "dequantized"])
def test_grouped_mm_autograd_equals_module(mx, arm):
    sizes = [90, 0, 333, 200, 377]
    M, G, N, K = sum(sizes), len(sizes), 256, 512
    x = S.normal_bf16((M, K), seed=1).cuda().requires_grad_()
    w = S.normal_bf16((G, N, K), 0.02, seed=2).cuda().requires_grad_()
    dy = S.normal_bf16((M, N), 0.1, seed=3).cuda()
    offs = S.offsets_from_sizes(sizes).cuda()
    y = mx.mxfp8_grouped_mm(x, w, offs, backward_override=arm)
    y.backward(dy)
    op = mx.MXFP8GroupedMM(backward_override=arm)
    y_ref = op.forward(x.detach(), w.detach(), offs)
    dx_ref, dw_ref = op.backward(dy)
    mx.mx_device_error()
    assert torch.equal(y, y_ref)
    assert torch.equal(x.grad, dx_ref) and torch.equal(w.grad, dw_ref)


def test_grouped_mm_autograd_stride0_grad(mx):
    """out.sum().backward() hands the backward an expanded (stride-0) gradient."""
    sizes = [128, 256]
    x = S.normal_bf16((384, 256), seed=4).cuda().requires_grad_()
    w = S.normal_bf16((2, 256, 256), 0.02, seed=5).cuda().requires_grad_()
    offs = S.offsets_from_sizes(sizes).cuda()
    mx.mxfp8_grouped_mm(x, w, offs).float().sum().backward()
    mx.mx_device_error()
    ones = torch.ones(384, 256, dtype=torch.bfloat16)
    op = mx.MXFP8GroupedMM()
    op.forward(x.detach(), w.detach(), offs)
    dx_ref, dw_ref = op.backward(ones.cuda())
    assert torch.equal(x.grad, dx_ref) and torch.equal(w.grad, dw_ref)


def test_linear_autograd_with_cache(mx):
    x = S.normal_bf16((256, 512), seed=6).cuda().requires_grad_()
    w = S.normal_bf16((256, 512), 0.02, seed=7).cuda().requires_grad_()
    dy = S.normal_bf16((256, 256), 0.1, seed=8).cuda()
    cache = mx.WeightCache()
    y1 = mx.mxfp8_linear(x, w, cache)
    y1.backward(dy)
    g1 = (x.grad.clone(), w.grad.clone())
    x.grad = None
    w.grad = None
    y2 = mx.mxfp8_linear(x, w, cache)                 # cache hit: bitwise the same
    y2.backward(dy)
    mx.mx_device_error()
    assert cache.stats()["hits"] >= 1
    assert torch.equal(y1, y2) and torch.equal(g1[0], x.grad) and torch.equal(g1[1], w.grad)
    ref, absref = O.linear_fwd(S.bf16_bits(x.detach().cpu()), S.bf16_bits(w.detach().cpu()))
    err = np.abs(y1.detach().float().cpu().numpy() - ref)
    assert np.all(err <= O.gemm_bound(ref, absref))
    cache.close()


def test_grouped_layer_backward_reads_the_forwards_codes_not_x(mx):
    """The MXFP8 backward of the grouped layer takes the wgrad's columnwise codes
    of x from the forward's fused cast: x overwritten between forward and backward
    leaves y, dX and dW bitwise those of an untouched run (ragged and empty groups)."""
    G, N, K = 4, 256, 384
    sizes = [300, 0, 129, 595]
    M = sum(sizes)
    x = S.normal_bf16((M, K), seed=5, device="cuda")
    w = S.normal_bf16((G, N, K), 0.02, seed=6, device="cuda")
    dy = S.normal_bf16((M, N), 0.1, seed=7, device="cuda")
    offs = S.offsets_from_sizes(sizes).cuda()
    op = mx.MXFP8GroupedMM()
    y_ref = op.forward(x, w, offs)
    ref = op.backward(dy)
    op = mx.MXFP8GroupedMM()
    y = op.forward(x, w, offs)
    x.zero_()
    got = op.backward(dy)
    mx.mx_device_error()
    assert torch.equal(y, y_ref)
    for name, a, b in zip(("dx", "dw"), got, ref):
        assert torch.equal(a, b), name


@pytest.mark.parametrize("use_reentrant", [False, True])
@pytest.mark.parametrize("arm", [None, "high_precision", "dequantized"])
def test_checkpointed_grouped_layer_is_bitwise_the_plain_run(mx, arm, use_reentrant):
    """The grouped layer under torch.utils.checkpoint (its saved codes and operands
    dropped after the forward and recomputed in the backward) gives the loss and
    both gradients bitwise equal to the plain run, for each backward arm."""
    from torch.utils.checkpoint import checkpoint
    G, N, K = 4, 256, 384
    sizes = [300, 0, 129, 595]
    M = sum(sizes)
    x0 = S.normal_bf16((M, K), seed=31, device="cuda")
    w0 = S.normal_bf16((G, N, K), 0.02, seed=32, device="cuda")
    offs = S.offsets_from_sizes(sizes).cuda()

    def layer(a, b):
        return mx.mxfp8_grouped_mm(a, b, offs, backward_override=arm)

    def run(ckpt):
        x, w = x0.clone().requires_grad_(), w0.clone().requires_grad_()
        y = checkpoint(layer, x, w, use_reentrant=use_reentrant) if ckpt else layer(x, w)
        loss = y.float().pow(2).sum()
        loss.backward()
        return loss.detach(), x.grad, w.grad

    ref = run(False)
    got = run(True)
    mx.mx_device_error()
    for name, a, b in zip(("loss", "dx", "dw"), got, ref):
        assert torch.equal(a, b), f"{name} under checkpointing ({arm}, use_reentrant={use_reentrant})"
