"""MXFP8 linear forward / dgrad / wgrad and the weight cache on the GPU.

Parity against the float64 oracle within 2^-7 |ref| + 1e-3 (|A| |B|^T); the
cache tests follow the cases named by "Cache quantized weights for full AC"
(prime-rl PR #3388, Overview): hit/miss, in-place weight update, per-tensor
isolation, and bit-identical results with and without a hit.
"""
import ctypes

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
    bad = np.abs(got - ref) > O.gemm_bound(ref, absref)
    assert not bad.any(), f"{what}: {bad.sum()} entries outside tolerance"


def test_linear_reduced_full_compare(mx):
    x, w, dy = S.linear_problem(M=512, N=512, K=256, seed=3)
    y = mx.linear_fwd(x.cuda(), w.cuda())
    dx, dw = mx.linear_bwd(dy.cuda(), x.cuda(), w.cuda())
    xb, wb, db = (S.bf16_bits(t) for t in (x, w, dy))
    _close(_f64(y), *O.linear_fwd(xb, wb), "fwd")
    _close(_f64(dx), *O.linear_dgrad(db, wb), "dgrad")
    _close(_f64(dw), *O.linear_wgrad(db, xb), "wgrad")


def _sqnr_db(ref, got):
    ref, got = ref.double(), got.double()
    return float(10 * torch.log10(ref.pow(2).sum() / (ref - got).pow(2).sum()))


def test_linear_full_size_sampled_and_sqnr(mx):
    """X[4096, 2048], W[4096, 2048], dY[4096, 4096]; sampled entries vs the oracle."""
    x, w, dy = S.linear_problem(seed=0, device="cuda")
    cache = mx.WeightCache()
    y = mx.linear_fwd(x, w, cache)
    dx, dw = mx.linear_bwd(dy, x, w, cache)
    mx.mx_device_error()
    rng = np.random.default_rng(0)
    yc, dxc, dwc = y.float().cpu().numpy(), dx.float().cpu().numpy(), dw.float().cpu().numpy()
    for _ in range(48):
        i, n, k = int(rng.integers(4096)), int(rng.integers(4096)), int(rng.integers(2048))
        n0, k0, i0 = n // 32 * 32, k // 32 * 32, i // 32 * 32
        # forward entry (i, n): row i of X (dim0) against row n of W (32x32 scales)
        qx, sx = O.cast_dim0(S.bf16_bits(x[i:i + 1]))
        qw, st = O.cast_32x32(S.bf16_bits(w[n0:n0 + 32]))
        a, b = O.dequant(qx, sx)[0], O.dequant(qw, O.w32_scale_views(st)[0])[n - n0]
        ref = a @ b
        assert abs(yc[i, n] - ref) <= 2 ** -7 * abs(ref) + 1e-3 * (np.abs(a) @ np.abs(b))
        # dgrad entry (i, k): row i of dY (dim0 along N) against column k of W
        qd, sd = O.cast_dim0(S.bf16_bits(dy[i:i + 1]))
        qw, st = O.cast_32x32(S.bf16_bits(w[:, k0:k0 + 32]))
        a = O.dequant(qd, sd)[0]
        b = O.dequant(np.ascontiguousarray(qw.T), O.w32_scale_views(st)[1])[k - k0]
        ref = a @ b
        assert abs(dxc[i, k] - ref) <= 2 ** -7 * abs(ref) + 1e-3 * (np.abs(a) @ np.abs(b))
        # wgrad entry (n, k): column n of dY and column k of X, cast down the tokens
        qa, sa = O.cast_dim1(S.bf16_bits(dy[:, n0:n0 + 32]))
        qb, sb = O.cast_dim1(S.bf16_bits(x[:, k0:k0 + 32]))
        a, b = O.dequant(qa, sa)[n - n0], O.dequant(qb, sb)[k - k0]
        ref = a @ b
        assert abs(dwc[n, k] - ref) <= 2 ** -7 * abs(ref) + 1e-3 * (np.abs(a) @ np.abs(b))
    # numerics versus the bf16 reference products (reported metric of the linear tests)
    y_ref = x.float() @ w.float().t()
    dx_ref = dy.float() @ w.float()
    dw_ref = dy.float().t() @ x.float()
    for got, ref in ((y, y_ref), (dx, dx_ref), (dw, dw_ref)):
        assert _sqnr_db(ref, got.float()) > 20.0
    cache.close()


def test_cache_hit_is_bitwise_identical_and_counted(mx):
    x, w, dy = S.linear_problem(M=1024, N=1024, K=512, seed=5, device="cuda")
    y0 = mx.linear_fwd(x, w)                       # no cache
    dx0, dw0 = mx.linear_bwd(dy, x, w)
    cache = mx.WeightCache()
    ys = [mx.linear_fwd(x, w, cache) for _ in range(3)]   # 1 miss + 2 hits (recompute)
    dx1, dw1 = mx.linear_bwd(dy, x, w, cache)             # hit
    st = cache.stats()
    assert st == {"hits": 3, "misses": 1, "entries": 1}
    for y in ys:
        assert torch.equal(y, y0)
    assert torch.equal(dx1, dx0) and torch.equal(dw1, dw0)
    cache.clear()
    assert cache.stats()["entries"] == 0
    cache.close()


def test_cache_in_place_update_and_isolation(mx):
    x, w, _ = S.linear_problem(M=256, N=512, K=256, seed=6, device="cuda")
    w2 = S.normal_bf16((512, 256), 0.02, seed=7, device="cuda")
    cache = mx.WeightCache()
    y_a = mx.linear_fwd(x, w, cache)
    y_b = mx.linear_fwd(x, w2, cache)              # different tensor: its own entry
    assert cache.stats()["entries"] == 2
    assert torch.equal(y_a, mx.linear_fwd(x, w)) and torch.equal(y_b, mx.linear_fwd(x, w2))
    v0 = w._version
    with torch.no_grad():
        w.mul_(2.0)                                # in-place update bumps the version
    assert w._version != v0
    y_c = mx.linear_fwd(x, w, cache)
    assert torch.equal(y_c, mx.linear_fwd(x, w))   # re-quantized, not the stale entry
    assert not torch.equal(y_c, y_a)
    st = cache.stats()
    assert st["misses"] == 3 and st["hits"] == 0 and st["entries"] == 2
    cache.close()


def test_stride0_grad_is_materialised(mx):
    """out.sum().backward() hands an expanded (stride-0) grad: the wrapper materialises it."""
    x, w, _ = S.linear_problem(M=256, N=256, K=256, seed=8, device="cuda")
    g = torch.full((1, 1), 0.5, dtype=torch.bfloat16, device="cuda").expand(256, 256)
    assert g.stride() == (0, 0)
    dx, dw = mx.linear_bwd(g, x, w)
    dx2, dw2 = mx.linear_bwd(g.contiguous(), x, w)
    assert torch.equal(dx, dx2) and torch.equal(dw, dw2)
    with pytest.raises(ValueError):
        mx.mx_cast_2d(g, *mx.cast_2d(g.contiguous()))  # the raw entry refuses strided views


class _DeviceMemory:
    """A fresh tensor object over existing device memory (its own version counter, at 0)."""

    def __init__(self, ptr, numel):
        self.__cuda_array_interface__ = {"shape": (numel,), "typestr": "<i2", "data": (ptr, False),
                                         "version": 3, "strides": None}


def _fresh_view(base, shape):
    t = torch.as_tensor(_DeviceMemory(base.data_ptr(), base.numel()), device=base.device)
    return t.view(torch.bfloat16).view(*shape)


def test_cache_address_reuse_by_a_new_tensor_is_a_miss(mx):
    """A weight freed and replaced by a different tensor at the same address, whose
    _version is 0 again, must not get the freed weight's codes (prime-rl PR #3388,
    Note: wrong invalidation gives silently wrong numerics)."""
    x, _, _ = S.linear_problem(M=256, N=512, K=256, seed=9, device="cuda")
    wa = S.normal_bf16((512 * 256,), 0.02, seed=10, device="cuda")
    wb = S.normal_bf16((512 * 256,), 0.02, seed=11, device="cuda")
    base = torch.empty(512 * 256, dtype=torch.bfloat16, device="cuda")
    cache = mx.WeightCache()
    base.copy_(wa)
    w = _fresh_view(base, (512, 256))
    assert w._version == 0
    y_a = mx.linear_fwd(x, w, cache)
    assert torch.equal(y_a, mx.linear_fwd(x, w, cache))            # hit
    del w                                                           # the tensor is gone ...
    base.copy_(wb)                                                  # ... its memory gets new bits
    w2 = _fresh_view(base, (512, 256))                              # and a new tensor at that address
    assert w2._version == 0
    y_b = mx.linear_fwd(x, w2, cache)
    torch.cuda.synchronize()
    assert torch.equal(y_b, mx.linear_fwd(x, w2))                  # equals the no-cache forward
    assert not torch.equal(y_b, y_a)
    st = cache.stats()
    assert st["hits"] == 1 and st["misses"] == 2
    # a live alias (a second tensor object over the same memory) is its own entry too
    w3 = _fresh_view(base, (512, 256))
    mx.linear_fwd(x, w3, cache)
    assert cache.stats()["misses"] == 3
    cache.close()


def test_cache_evict_through_the_c_abi(mx):
    """A C caller that passes the same version for a new tensor at a freed weight's
    address calls mx_wcache_evict when it frees the weight: the next call misses."""
    x, _, _ = S.linear_problem(M=128, N=256, K=256, seed=12, device="cuda")
    base = S.normal_bf16((256, 256), 0.02, seed=13, device="cuda")
    other = S.normal_bf16((256, 256), 0.02, seed=14, device="cuda")
    ws = mx.linear_workspace(128, 256, 256)
    y = torch.empty(128, 256, dtype=torch.bfloat16, device="cuda")
    cache = mx.WeightCache()
    mx.mx_linear_fwd(x, base, cache, 0, y, ws)
    mx.lib().mx_wcache_evict(cache.handle, ctypes.c_void_p(base.data_ptr()))
    base.copy_(other)
    mx.mx_linear_fwd(x, base, cache, 0, y, ws)                     # same address, same version: a miss
    torch.cuda.synchronize()
    assert torch.equal(y, mx.linear_fwd(x, other))
    st = cache.stats()
    assert st["misses"] == 2 and st["hits"] == 0 and st["entries"] == 1
    cache.close()


def test_linear_autograd_clears_the_entry_after_backward(mx):
    """mxfp8_linear drops the weight's entry once its backward ran (prime-rl PR #3388,
    Overview: the cache is cleared after backward); a recompute forward before the
    backward (activation checkpointing) still hits."""
    x = S.normal_bf16((256, 512), seed=15).cuda().requires_grad_()
    w = S.normal_bf16((256, 512), 0.02, seed=16).cuda().requires_grad_()
    dy = S.normal_bf16((256, 256), 0.1, seed=17).cuda()
    cache = mx.WeightCache()
    mx.mxfp8_linear(x, w, cache)                      # forward: miss
    y = mx.mxfp8_linear(x, w, cache)                  # recompute forward: hit
    assert cache.stats() == {"hits": 1, "misses": 1, "entries": 1}
    y.backward(dy)                                    # backward: hit, then the entry is dropped
    st = cache.stats()
    assert st["hits"] == 2 and st["entries"] == 0
    keep = mx.WeightCache(clear_after_backward=False)
    mx.mxfp8_linear(x, w, keep).backward(dy)
    assert keep.stats()["entries"] == 1
    cache.close()
    keep.close()


def _linear_inputs(M, N, K, seed):
    if M:
        return S.linear_problem(M=M, N=N, K=K, seed=seed, device="cuda")
    return (torch.empty(0, K, dtype=torch.bfloat16, device="cuda"),
            S.normal_bf16((N, K), 0.02, seed=seed, device="cuda"),
            torch.empty(0, N, dtype=torch.bfloat16, device="cuda"))


def _separate_calls(mx, x, w, dy):
    M, K = x.shape
    N = w.shape[0]
    out = [torch.empty(M, N, dtype=torch.bfloat16, device="cuda"),
           torch.empty(M, K, dtype=torch.bfloat16, device="cuda"),
           torch.empty(N, K, dtype=torch.bfloat16, device="cuda")]
    ws = mx.linear_workspace(M, N, K)
    mx.mx_linear_fwd(x, w, None, 0, out[0], ws)
    mx.mx_linear_bwd(dy, x, w, None, 0, out[1], out[2], ws)
    return out


@pytest.mark.parametrize("M,N,K", [(512, 512, 256), (256, 96, 576), (96, 256, 128), (0, 256, 256)])
@pytest.mark.parametrize("cached", [False, True])
def test_training_pair_is_bitwise_the_separate_calls(mx, M, N, K, cached):
    """mx_linear_fwd_train + mx_linear_bwd_after_fwd give y, dX and dW bitwise
    equal to mx_linear_fwd + mx_linear_bwd on the same x, w and dY. The backward
    reads neither x (zeroed after the forward here) nor, without a cache, w
    (doubled in between: the gradient stays that of the forward's product).
    Shapes: aligned, the GEMM pad path with K > 2N (the pair's larger
    workspace), M off the 128-row tile, and no tokens."""
    x, w, dy = _linear_inputs(M, N, K, seed=7)
    ref = _separate_calls(mx, x, w, dy)
    cache = mx.WeightCache() if cached else None
    ver = cache.key_version(w) if cached else 0
    got = [torch.full_like(t, float("nan")) for t in ref]
    ws = mx.linear_workspace(M, N, K, train=True)
    mx.mx_linear_fwd_train(x, w, cache, ver, got[0], ws)
    x.zero_()
    if not cached:
        w.mul_(2)
    mx.mx_linear_bwd_after_fwd(dy, w, cache, ver, got[1], got[2], ws)
    torch.cuda.synchronize()
    mx.mx_device_error()
    for name, a, b in zip(("y", "dx", "dw"), got, ref):
        assert torch.equal(a, b), f"{name} of the training pair at M={M}, N={N}, K={K}"
    if cached:
        st = cache.stats()
        assert (st["misses"], st["hits"]) == (1, 1), st     # the backward reuses the forward's entry
        cache.close()


def test_autograd_linear_runs_the_training_pair(mx):
    """mxfp8_linear under autograd: y, dX and dW bitwise those of the separate
    calls, x not saved for the backward (w and the workspace holding x's codes
    are), and a forward without gradients (mx_linear_fwd) gives the same y."""
    M, N, K = 256, 96, 576
    x, w, dy = _linear_inputs(M, N, K, seed=11)
    ref = _separate_calls(mx, x, w, dy)
    xg, wg = x.clone().requires_grad_(), w.clone().requires_grad_()
    y = mx.mxfp8_linear(xg, wg)
    saved = y.grad_fn.saved_tensors
    assert len(saved) == 2 and saved[0] is wg and saved[1].dtype == torch.uint8
    y.backward(dy)
    assert torch.equal(y.detach(), ref[0])
    assert torch.equal(xg.grad, ref[1]) and torch.equal(wg.grad, ref[2])
    with torch.no_grad():
        assert torch.equal(mx.mxfp8_linear(x, w), ref[0])
    mx.mx_device_error()


@pytest.mark.parametrize("use_reentrant", [False, True])
def test_checkpointed_segment_with_the_cache_is_bitwise_the_plain_run(mx, use_reentrant):
    """Full activation checkpointing ("Cache quantized weights for full AC",
    prime-rl PR #3388, Overview: checkpoint grad parity; the cache is cleared
    after backward so training stays bit-identical to an uncheckpointed run): a
    segment of two MXFP8 linears around a GELU, under torch.utils.checkpoint with
    a weight cache, gives the loss and every gradient bitwise equal to the same
    segment run without checkpointing and without a cache, and the backward leaves
    the cache empty; with non-reentrant checkpointing the recompute forward hits."""
    from torch.utils.checkpoint import checkpoint
    M, D, H = 256, 512, 768
    x0 = S.normal_bf16((M, D), seed=21).cuda()
    w1_0 = S.normal_bf16((H, D), 0.02, seed=22).cuda()
    w2_0 = S.normal_bf16((D, H), 0.02, seed=23).cuda()

    def segment(x, w1, w2, cache):
        h = torch.nn.functional.gelu(mx.mxfp8_linear(x, w1, cache))
        return mx.mxfp8_linear(h, w2, cache)

    def run(ckpt, cache):
        x, w1, w2 = (t.clone().requires_grad_() for t in (x0, w1_0, w2_0))
        y = checkpoint(segment, x, w1, w2, cache, use_reentrant=use_reentrant) if ckpt else segment(x, w1, w2, cache)
        loss = y.float().pow(2).sum()
        loss.backward()
        return loss.detach(), x.grad, w1.grad, w2.grad

    ref = run(False, None)
    cache = mx.WeightCache()
    got = run(True, cache)
    mx.mx_device_error()
    for name, a, b in zip(("loss", "dx", "dw1", "dw2"), got, ref):
        assert torch.equal(a, b), f"{name} under checkpointing (use_reentrant={use_reentrant})"
    st = cache.stats()
    if use_reentrant:
        # the reentrant form recomputes on detached aliases of the weights: new tensor
        # objects to the cache's per-object identity, so the recompute re-quantizes
        # (two more misses) instead of risking a stale hit; the backward then hits
        assert (st["misses"], st["hits"], st["entries"]) == (4, 2, 0), st
    else:
        assert st["misses"] == 2 and st["hits"] >= 2 and st["entries"] == 0, st
    cache.close()
