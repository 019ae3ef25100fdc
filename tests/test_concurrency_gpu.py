"""The library used from several host threads at once, each on its own CUDA
stream, as a serving process would: the grouped MoE layer (casts and the
three grouped GEMMs) and the linear with a shared weight cache, on different
shapes per thread so that the tensor-map cache, the once-per-device kernel
setup and the weight cache's lock are exercised concurrently. Every result
must be bitwise the result of the same work run alone.
"""
import threading

import numpy as np
import pytest
import torch

from mxfp8_block_scaled_cast_b200 import synthetic as S

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mx():
    from mxfp8_block_scaled_cast_b200 import mx as _mx
    _mx.lib()
    return _mx


def _moe_job(mx, seed):
    rng = np.random.default_rng(seed)
    G, N, K = 4, 256 + 32 * (seed % 3), 384
    sizes = rng.integers(0, 400, size=G)
    M = int(sizes.sum())
    x = S.normal_bf16((M, K), seed=seed, device="cuda")
    w = S.normal_bf16((G, N, K), 0.02, seed=seed + 1, device="cuda")
    dy = S.normal_bf16((M, N), 0.1, seed=seed + 2, device="cuda")
    offs = S.offsets_from_sizes(sizes).cuda()

    def run():
        op = mx.MXFP8GroupedMM()
        y = op.forward(x, w, offs)
        dx, dw = op.backward(dy)
        return y, dx, dw
    return run


def _linear_job(mx, seed, cache):
    M, N, K = 256, 192 + 64 * (seed % 2), 320
    x, w, dy = S.linear_problem(M=M, N=N, K=K, seed=seed, device="cuda")

    def run():
        y = mx.mxfp8_linear(x, w, cache)
        return (y,)
    return run


def test_threads_on_their_own_streams_match_serial_runs(mx):
    cache = mx.WeightCache()
    jobs = [_moe_job(mx, s) for s in (1, 2, 3)] + [_linear_job(mx, s, cache) for s in (4, 5)]
    want = []
    for job in jobs:                        # each job alone, on the default stream
        want.append([t.clone() for t in job()])
    torch.cuda.synchronize()
    errors, got = [], [None] * len(jobs)

    def worker(i):
        try:
            stream = torch.cuda.Stream()
            with torch.cuda.stream(stream):
                outs = None
                for _ in range(10):         # repeated, so the threads' launches interleave
                    outs = jobs[i]()
                stream.synchronize()
                got[i] = [t.clone() for t in outs]
                stream.synchronize()
        except Exception as e:               # reported on the main thread
            errors.append((i, repr(e)))

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(len(jobs))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not any(t.is_alive() for t in threads), "a worker thread did not finish"
    assert not errors, errors
    mx.mx_device_error()
    for i, (g, w_) in enumerate(zip(got, want)):
        for a, b in zip(g, w_):
            assert torch.equal(a, b), f"job {i} differs from its serial run"
    cache.close()
