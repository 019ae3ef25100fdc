"""K-groups (wgrad) GEMM: how the output tiles of each expert are walked.

Every expert's [N, K] output is cut into 256x256 tiles that the CTA pairs
share out; a tile walks the 128-deep token steps of all the expert's groups.
These cases check the result against the float64 oracle (ao "[moe training]
Add backward_override to the MXFP8 grouped GEMM", Summary: the wgrad of the
grouped GEMM, dW_g = dY_g^T X_g over each group's tokens) where that walk has
its edges:

* more tiles per expert than CTA pairs, skewed sizes, empty experts;
* fewer tiles per expert than pairs, groups cycling over experts (E < G);
* 64 and 65 experts of one group each, sizes from empty to a few hundred.

The output is filled with NaN first, so a tile that no pair computed shows.
"""
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


def _wgrad(mx, sizes, N, K, E, seed):
    """GPU wgrad of groups `sizes` cycling over E experts, output NaN-prefilled;
    returns (out as float64, oracle dequantized A [N, cap], B [K, cap], offs)."""
    M, G = int(sum(sizes)), len(sizes)
    dyb = S.normal_bf16((M, N), 1e-2, seed=seed)
    xb = S.normal_bf16((M, K), 1.0, seed=seed + 1)
    offs_t = S.offsets_from_sizes(sizes)
    cap = mx.mx_padded_rows_capacity(M, G)
    od = offs_t.cuda()
    dqt, dst = mx.cast_dim1_grouped(dyb.cuda(), od, cap)
    xqt, xst = mx.cast_dim1_grouped(xb.cuda(), od, cap)
    out = torch.full((E, N, K), float("nan"), dtype=torch.bfloat16, device="cuda")
    mx.mx_grouped_mm_experts(dqt, dst, xqt, xst, od, G, E, mx.MX_GROUPS_K, out, M, N, K, cap)
    mx.mx_device_error()
    offs = offs_t.numpy()
    aq, as_ = O.cast_dim1_grouped(S.bf16_bits(dyb), offs, cap)
    bq, bs = O.cast_dim1_grouped(S.bf16_bits(xb), offs, cap)
    return out.float().cpu().numpy().astype(np.float64), O.dequant(aq, as_), O.dequant(bq, bs), offs


def _expert_sums(a, b, offs, E):
    """Oracle: expert e's dW is the sum of its groups' K-groups products."""
    per_group = O.grouped_mm_k(a, b, offs)
    per_group_abs = O.grouped_mm_k(np.abs(a), np.abs(b), offs)
    ref = np.stack([per_group[e::E].sum(axis=0) for e in range(E)])
    absref = np.stack([per_group_abs[e::E].sum(axis=0) for e in range(E)])
    return ref, absref


def _check(got, ref, absref, what):
    assert not np.isnan(got).any(), f"{what}: tiles left unwritten"
    bad = ~(np.abs(got - ref) <= O.gemm_bound(ref, absref))
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} outside tolerance"


def test_more_tiles_per_expert_than_pairs_skewed_and_empty(mx):
    """N = K = 2304: 81 tiles per expert (more than the 74 pairs of a B200);
    Zipf-like sizes, two empty experts, sizes not multiples of 128. Rows are
    sampled in every 256-row band (all columns), so every tile is compared."""
    sizes = [1900, 0, 700, 333, 95, 0, 1288, 41, 510, 129]
    N = K = 2304
    got, a, b, offs = _wgrad(mx, sizes, N, K, len(sizes), seed=31)
    assert not np.isnan(got).any(), "tiles left unwritten"
    rows = np.array(sorted({min(N - 1, band * 256 + d) for band in range(N // 256 + 1) for d in (0, 97, 255)}))
    ref, absref = _expert_sums(a[rows], b, offs, len(sizes))
    _check(got[:, rows, :], ref, absref, "wgrad, sampled rows")
    for e, n in enumerate(sizes):
        if n == 0:
            assert not got[e].any(), f"empty expert {e} is not exactly zero"


@pytest.mark.parametrize("E", [2, 8])
def test_fewer_tiles_per_expert_than_pairs_groups_cycle(mx, E):
    """N = K = 512 (four tiles per expert), 16 groups cycling over E experts."""
    rng = np.random.default_rng(40 + E)
    sizes = [int(v) for v in rng.integers(0, 400, size=16)]
    sizes[3] = 0
    got, a, b, offs = _wgrad(mx, sizes, 512, 512, E, seed=41)
    _check(got, *_expert_sums(a, b, offs, E), f"wgrad, E={E}")


@pytest.mark.parametrize("E", [64, 65])
def test_many_experts_one_group_each(mx, E):
    """64 and 65 experts, one group each, N = 256, K = 512 (two tiles per
    expert), sizes from empty to a few hundred."""
    rng = np.random.default_rng(50 + E)
    sizes = [int(v) for v in rng.integers(0, 300, size=E)]
    sizes[0] = 0
    sizes[-1] = 777
    got, a, b, offs = _wgrad(mx, sizes, 256, 512, E, seed=51)
    _check(got, *_expert_sums(a, b, offs, E), f"wgrad, E={E}")
