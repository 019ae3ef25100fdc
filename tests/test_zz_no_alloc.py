"""The allocation-free linear forward, checked against the workspace entry point.

mx_linear_fwd_noalloc is for callers that cannot allocate device memory (a
plain C host program without a device allocator, or a plugin inside a
runtime that owns all device memory): its scratch is a fixed array inside
the library. This file is collected last on purpose, so that a run that
stops at the first failure has already run every other test; it also passes
on its own in a fresh process (the first call does the per-device set-up).
"""
import numpy as np
import pytest
import torch

from mxfp8_block_scaled_cast_b200 import synthetic as S

pytestmark = pytest.mark.gpu


def _within_gemm_tolerance(got, ref, x, w):
    # the GEMM tolerance of the other tests, 2^-7 |ref| + 1e-3 (|A| |B|^T),
    # with |x| |w|^T standing in for the magnitude of the quantized operands
    absref = x.float().abs() @ w.float().abs().t()
    err = (got.float() - ref.float()).abs()
    return bool((err <= 2.0 ** -7 * ref.float().abs() + 1e-3 * absref).all())


def test_noalloc_forward_matches_workspace_forward_twice():
    from mxfp8_block_scaled_cast_b200 import mx
    x, w, _ = S.linear_problem(M=4096, N=4096, K=2048, seed=0, device="cuda")
    ws = mx.linear_workspace(4096, 4096, 2048)
    y_ref = torch.empty(4096, 4096, dtype=torch.bfloat16, device="cuda")
    mx.mx_linear_fwd(x, w, None, 0, y_ref, ws)
    for _ in range(2):                                   # two calls in a row share the array
        y = torch.full((4096, 4096), float("nan"), dtype=torch.bfloat16, device="cuda")
        mx.mx_linear_fwd_noalloc(x, w, y)
        torch.cuda.synchronize()
        assert _within_gemm_tolerance(y, y_ref, x, w)
        assert torch.equal(y, y_ref)                     # same kernels: identical bits
    mx.mx_device_error()


def test_noalloc_forward_other_shape_after_first():
    from mxfp8_block_scaled_cast_b200 import mx
    x, w, _ = S.linear_problem(M=96, N=512, K=256, seed=1, device="cuda")
    y_ref = mx.linear_fwd(x, w)
    y = torch.empty_like(y_ref)
    mx.mx_linear_fwd_noalloc(x, w, y)
    assert torch.equal(y, y_ref)


def test_noalloc_rejects_sizes_beyond_the_array():
    from mxfp8_block_scaled_cast_b200 import mx
    M, N, K = 8192, 4096, 4096                           # needs 48 MiB of scratch
    x = torch.zeros(M, K, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(N, K, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mx.MXError) as e:
        mx.mx_linear_fwd_noalloc(x, w, y)
    assert e.value.status == 3 and "static scratch" in str(e.value)
    assert str(mx.MX_LINEAR_NOALLOC_SCRATCH_BYTES) in str(e.value)
    assert not y.any()                                   # rejected before any launch
