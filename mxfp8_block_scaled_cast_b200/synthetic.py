"""Seeded synthetic inputs shaped like the workloads on the pages.

This module only draws random numbers. It holds none of the casting or GEMM
arithmetic, so both the CUDA path and the CPU oracle can consume its output.
Every tensor is bf16 (or int32 offsets) and is a pure function of its seed,
its shape and the device it is generated on (CPU and CUDA generators give
different bits for the same seed; parity tests always generate on the CPU and
copy the bits to the GPU).

Workloads (the benchmark shapes of ao PR #4705, "Wire MoE and MXFP8Linear
training paths to CuTeDSL by default": the MoE recipe benchmark at K=N=4096,
G=8, M=16384 and the MXFP8Linear benchmark at M=4096, N=4096, K=2048):

* ``tiny``      A[256, 256] = N(0,1) * 2**k per 1x32 block, k uniform in
                [-20, 20]; block (0, 0) all zeros; element (1, 0) = 6e4;
                grouped GEMM G=2, offs=[128, 256], W[2, 256, 256] N(0, 0.02).
* ``linear``    X[4096, 2048] N(0,1); W[4096, 2048] N(0, 0.02);
                dY[4096, 4096] N(0, 1e-2).
* ``moe``       G=8, K=N=4096, M=16384: group sizes are 128 * (Dirichlet(1)
                counts over 128 units, largest-remainder rounded); X N(0,1),
                W[8, 4096, 4096] N(0, 0.02), dY[16384, 4096] N(0, 1e-2).
* ``sweep``     N(0,1) tensors of the given shape with 0.1% of the elements
                (chosen by the seed) multiplied by 1000.
* ``unaligned`` dY[16384, 576] N(0,1); grouped GEMM G=32, K=7168, N=2048,
                M=32768 with Zipf(s=1.2) sizes over 29 non-empty groups in
                shuffled positions, 3 empty groups, no non-empty size a
                multiple of 128.
"""
from __future__ import annotations

import numpy as np
import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, std=1.0, seed=0, device="cpu") -> torch.Tensor:
    """bf16 tensor of N(0, std^2) samples (drawn in fp32, rounded by torch)."""
    g = _gen(seed, device)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def sweep_tensor(shape, seed=0, device="cpu", outlier_frac=1e-3, outlier_mul=1000.0):
    """N(0,1) bf16 with a seeded 0.1% of elements scaled by 1000."""
    g = _gen(seed, device)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    mask = torch.rand(*shape, generator=g, device=device) < outlier_frac
    x = torch.where(mask, x * outlier_mul, x)
    return x.to(torch.bfloat16)


def tiny_activation(seed=0) -> torch.Tensor:
    """A[256, 256]: per-1x32-block magnitudes 2**k, one zero block, one 6e4 entry."""
    g = _gen(seed, "cpu")
    x = torch.randn(256, 256, generator=g, dtype=torch.float32)
    k = torch.randint(-20, 21, (256, 256 // 32), generator=g, dtype=torch.int64)
    x = x * torch.pow(2.0, k.to(torch.float32)).repeat_interleave(32, dim=1)
    x[0, 0:32] = 0.0
    x[1, 0] = 6e4
    return x.to(torch.bfloat16)


def tiny_problem(seed=0):
    """The tiny case: activations, two experts of 256x256 and offs=[128, 256]."""
    a = tiny_activation(seed)
    w = normal_bf16((2, 256, 256), std=0.02, seed=seed + 1)
    offs = torch.tensor([128, 256], dtype=torch.int32)
    return a, w, offs


def _largest_remainder(weights: np.ndarray, total: int) -> np.ndarray:
    """Integer counts proportional to ``weights`` that sum exactly to ``total``."""
    raw = weights / weights.sum() * total
    base = np.floor(raw).astype(np.int64)
    rem = total - int(base.sum())
    order = np.argsort(-(raw - base), kind="stable")
    base[order[:rem]] += 1
    return base


def dirichlet_group_sizes(groups=8, total=16384, unit=128, seed=0) -> np.ndarray:
    """Group sizes: multiples of ``unit`` from Dirichlet(1) weights, summing to total."""
    rng = np.random.default_rng(seed)
    w = rng.dirichlet(np.ones(groups))
    return _largest_remainder(w, total // unit) * unit


def zipf_group_sizes(groups=32, total=32768, s=1.2, empty=3, seed=0) -> np.ndarray:
    """Skewed sizes: Zipf(s) over the non-empty groups, ``empty`` zero groups.

    Re-rolls with the next seed until no non-empty size is a multiple of 128
    and every non-empty size is positive.
    """
    while True:
        rng = np.random.default_rng(seed)
        live = groups - empty
        w = np.arange(1, live + 1, dtype=np.float64) ** (-s)
        sizes_live = _largest_remainder(w, total)
        slots = rng.permutation(groups)
        sizes = np.zeros(groups, dtype=np.int64)
        sizes[slots[:live]] = rng.permutation(sizes_live)
        ok = (np.count_nonzero(sizes == 0) == empty
              and not np.any((sizes > 0) & (sizes % 128 == 0)))
        if ok:
            return sizes
        seed += 1


def offsets_from_sizes(sizes) -> torch.Tensor:
    """Cumulative end offsets (int32), the format of the grouped GEMM's offs."""
    return torch.tensor(np.cumsum(np.asarray(sizes, dtype=np.int64)), dtype=torch.int32)


def linear_problem(M=4096, N=4096, K=2048, seed=0, device="cpu"):
    x = normal_bf16((M, K), 1.0, seed, device)
    w = normal_bf16((N, K), 0.02, seed + 1, device)
    dy = normal_bf16((M, N), 1e-2, seed + 2, device)
    return x, w, dy


def moe_problem(G=8, M=16384, N=4096, K=4096, seed=0, device="cpu"):
    sizes = dirichlet_group_sizes(G, M, 128, seed)
    x = normal_bf16((M, K), 1.0, seed, device)
    w = normal_bf16((G, N, K), 0.02, seed + 1, device)
    dy = normal_bf16((M, N), 1e-2, seed + 2, device)
    return x, w, dy, offsets_from_sizes(sizes)


def unaligned_grouped_problem(G=32, M=32768, N=2048, K=7168, seed=0, device="cpu"):
    sizes = zipf_group_sizes(G, M, 1.2, 3, seed)
    x = normal_bf16((M, K), 1.0, seed, device)
    w = normal_bf16((G, N, K), 0.02, seed + 1, device)
    dy = normal_bf16((M, N), 1.0, seed + 2, device)
    return x, w, dy, offsets_from_sizes(sizes)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a bf16 tensor (copied to the host)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
