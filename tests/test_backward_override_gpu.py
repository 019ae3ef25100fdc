"""Parity of the backward-override arms (bf16 grouped GEMMs, dequantization,
scale unswizzle) with the float64 oracle.

Dequantization and the unswizzle are byte work: bit-exact. The bf16 GEMMs
use the GEMM tolerance |gpu - ref| <= 2^-7 |ref| + 1e-3 (|A| |B|) against
the float64 products of the same bf16 operands (the GPU accumulates in fp32
and rounds once to bf16). Quantized operands the GPU path starts from are
the GPU casts' outputs, which the cast tests pin bit-exactly to the oracle;
the oracle computes its side from the seeded bf16 inputs alone.
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


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def _bits(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def _assert_close(got, ref, absref, what=""):
    err = np.abs(got - ref)
    bound = O.gemm_bound(ref, absref)
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside tolerance, worst {np.max(err - bound)}"


def _assert_bf16_equal(got_t, ref_f64, what=""):
    got = _f64(got_t)
    nan = np.isnan(ref_f64)
    assert np.array_equal(np.isnan(got), nan), what
    assert np.array_equal(got[~nan], ref_f64[~nan]), what
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref_f64[~nan])), what


# ------------------------------------------------------- dequantization ----
@pytest.mark.parametrize("G,R,C", [(1, 300, 96), (3, 64, 256), (1, 1, 32)])
def test_dequant_every_code_random_scales(mx, G, R, C):
    rng = np.random.default_rng(G * 1000 + R + C)
    q = rng.integers(0, 256, size=(G, R, C), dtype=np.uint8)
    s = rng.integers(0, 256, size=(G, R, C // 32), dtype=np.uint8)    # 255 (NaN) included
    s[..., 0] = rng.integers(0, 8, size=(G, R))                       # tiny scales: bf16 rounding
    blocked = np.concatenate([O.swizzle(s[g]) for g in range(G)])
    out = mx.dequant_dim0(torch.from_numpy(q).cuda().squeeze(0) if G == 1 else torch.from_numpy(q).cuda(),
                          torch.from_numpy(blocked).cuda())
    _assert_bf16_equal(out.reshape(G, R, C), O.dequant_bf16(q, s), "dequant")


def test_dequant_output_only_16_byte_aligned(mx):
    """An output at a 16-byte (not 32-byte) offset takes the 128-bit store path."""
    rng = np.random.default_rng(5)
    R, C = 130, 96
    q = rng.integers(0, 0x7F, size=(R, C), dtype=np.uint8)
    s = rng.integers(100, 140, size=(R, C // 32), dtype=np.uint8)
    raw = torch.zeros(R * C + 8, dtype=torch.bfloat16, device="cuda")
    out = raw[8:].view(R, C)
    assert out.data_ptr() % 32 == 16
    mx.mx_dequant_dim0(torch.from_numpy(q).cuda(), torch.from_numpy(O.swizzle(s)).cuda(), 1, R, C, out)
    _assert_bf16_equal(out, O.dequant_bf16(q, s), "dequant, 16-byte aligned output")
    assert not raw[:8].any()


@pytest.mark.parametrize("sizes", [[37, 0, 263], [128, 128], [1, 2, 3, 500]])
def test_dequant_grouped_round_trip(mx, sizes):
    M = int(sum(sizes))
    xb = S.normal_bf16((M, 192), seed=len(sizes) + M)
    offs_t = S.offsets_from_sizes(sizes)
    q, s = mx.cast_dim0_grouped(xb.cuda(), offs_t.cuda())
    out = mx.dequant_dim0_grouped(q, s, offs_t.cuda(), M)
    mx.mx_device_error()
    qo, so = O.cast_dim0(S.bf16_bits(xb))
    _assert_bf16_equal(out, O.dequant_bf16(qo, so), "grouped dequant")


def test_dequant_grouped_invalid_offsets_write_nothing(mx):
    q = torch.zeros(256, 64, dtype=torch.uint8, device="cuda")
    s = torch.zeros(mx.mx_scale_bytes(256, 2), dtype=torch.uint8, device="cuda")
    out = torch.full((200, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    bad = torch.tensor([150, 100, 200], dtype=torch.int32, device="cuda")
    mx.mx_dequant_dim0_grouped(q, s, bad, 200, 64, 256, out)
    with pytest.raises(mx.MXError) as e:
        mx.mx_device_error()
    assert e.value.status == 6
    assert bool((out == 7.0).all())


@pytest.mark.parametrize("R,C32", [(300, 3), (128, 4), (5, 70)])
def test_scales_unswizzle(mx, R, C32):
    rng = np.random.default_rng(R * 7 + C32)
    s = rng.integers(0, 255, size=(R, C32), dtype=np.uint8)
    blocked = O.swizzle(s)
    out = mx.scales_unswizzle(torch.from_numpy(blocked).cuda(), R, C32)
    assert np.array_equal(out.cpu().numpy(), O.unswizzle(blocked, R, C32))
    assert np.array_equal(out.cpu().numpy(), s)


# ------------------------------------------------------- bf16 GEMMs ------
@pytest.mark.parametrize("sizes,K,N", [
    ([130, 0, 300, 270], 200, 512),     # ragged groups, K with a partial 64-step
    ([700], 64, 256),                   # one group, one K step
    ([1, 255, 256, 257, 0], 520, 256),  # tile boundaries inside and across groups
])
def test_bf16_grouped_mm_row_groups(mx, sizes, K, N):
    M, G = int(sum(sizes)), len(sizes)
    a = S.normal_bf16((M, K), seed=M + K)
    b = S.normal_bf16((G, K, N), 0.05, seed=G + N)
    offs_t = S.offsets_from_sizes(sizes)
    out = mx.grouped_mm_bf16(a.cuda(), b.cuda(), offs_t.cuda())
    out2 = mx.grouped_mm_bf16(a.cuda(), b.cuda(), offs_t.cuda())
    mx.mx_device_error()
    assert torch.equal(out, out2)
    af, bf = O.bf16_to_f64(S.bf16_bits(a)), O.bf16_to_f64(S.bf16_bits(b))
    offs = offs_t.numpy()
    _assert_close(_f64(out), O.hp_grouped_mm_m(af, bf, offs), O.hp_grouped_mm_m(np.abs(af), np.abs(bf), offs),
                  "row groups")


def test_bf16_dense_row_groups(mx):
    a = S.normal_bf16((300, 136), seed=1)
    b = S.normal_bf16((1, 136, 512), 0.05, seed=2)
    out = mx.grouped_mm_bf16(a.cuda(), b.cuda(), None)
    af, bf = O.bf16_to_f64(S.bf16_bits(a)), O.bf16_to_f64(S.bf16_bits(b))
    _assert_close(_f64(out), af @ bf[0], np.abs(af) @ np.abs(bf[0]), "dense")


@pytest.mark.parametrize("sizes,N,K", [
    ([1, 63, 0, 64, 65, 507], 256, 512),   # every tail length class, an empty group
    ([130, 70], 512, 256),
    ([0, 0, 333], 256, 256),
])
def test_bf16_grouped_mm_token_groups(mx, sizes, N, K):
    M, G = int(sum(sizes)), len(sizes)
    a = S.normal_bf16((M, N), seed=M + N + 1)
    b = S.normal_bf16((M, K), seed=M + K + 2)
    offs_t = S.offsets_from_sizes(sizes)
    out = mx.grouped_mm_bf16_wgrad(a.cuda(), b.cuda(), offs_t.cuda())
    out2 = mx.grouped_mm_bf16_wgrad(a.cuda(), b.cuda(), offs_t.cuda())
    mx.mx_device_error()
    assert torch.equal(out, out2)
    af, bf = O.bf16_to_f64(S.bf16_bits(a)), O.bf16_to_f64(S.bf16_bits(b))
    offs = offs_t.numpy()
    got = _f64(out)
    for g, n in enumerate(sizes):
        if n == 0:
            assert np.all(got[g] == 0.0) and not np.any(np.signbit(got[g]))
    _assert_close(got, O.hp_grouped_mm_k(af, bf, offs), O.hp_grouped_mm_k(np.abs(af), np.abs(bf), offs),
                  "token groups")


def test_bf16_token_groups_no_tokens(mx):
    a = torch.zeros(0, 256, dtype=torch.bfloat16, device="cuda")
    b = torch.zeros(0, 256, dtype=torch.bfloat16, device="cuda")
    offs = torch.zeros(3, dtype=torch.int32, device="cuda")
    out = mx.grouped_mm_bf16_wgrad(a, b, offs)
    assert out.shape == (3, 256, 256) and not out.any()


def test_bf16_gemm_invalid_offsets_and_host_errors(mx):
    a = S.normal_bf16((256, 64), seed=3).cuda()
    b = S.normal_bf16((2, 64, 256), seed=4).cuda()
    bad = torch.tensor([200, 100], dtype=torch.int32, device="cuda")
    out = torch.full((256, 256), 3.0, dtype=torch.bfloat16, device="cuda")
    mx.mx_grouped_mm_bf16(a, b, bad, 2, mx.MX_GROUPS_M, out, 256, 256, 64)
    with pytest.raises(mx.MXError) as e:
        mx.mx_device_error()
    assert e.value.status == 6
    assert bool((out == 3.0).all())
    with pytest.raises(mx.MXError) as e:          # N not a multiple of 32
        mx.mx_grouped_mm_bf16(a, b, None, 1, mx.MX_GROUPS_M, out, 256, 100, 64)
    assert e.value.status == 3
    with pytest.raises(mx.MXError) as e:          # K not a multiple of 8
        mx.mx_grouped_mm_bf16(a, b, None, 1, mx.MX_GROUPS_M, out, 256, 256, 60)
    assert e.value.status == 3


# ----------------------------------------------------- the module's arms --
def _moe_small(seed=0):
    sizes = [90, 0, 333, 200, 377]
    M, G, N, K = int(sum(sizes)), len(sizes), 256, 512
    x = S.normal_bf16((M, K), seed=seed)
    w = S.normal_bf16((G, N, K), 0.02, seed=seed + 1)
    dy = S.normal_bf16((M, N), 0.1, seed=seed + 2)
    return x, w, dy, S.offsets_from_sizes(sizes)


@pytest.mark.parametrize("arm", ["high_precision", "dequantized"])
def test_override_arms_match_oracle(mx, arm):
    x, w, dy, offs_t = _moe_small(5)
    op = mx.MXFP8GroupedMM(backward_override=arm)
    op.forward(x.cuda(), w.cuda(), offs_t.cuda())
    dx, dw = op.backward(dy.cuda())
    mx.mx_device_error()
    fn = O.moe_backward_high_precision if arm == "high_precision" else O.moe_backward_dequantized
    rdx, adx, rdw, adw = fn(S.bf16_bits(x), S.bf16_bits(w), S.bf16_bits(dy), offs_t.numpy())
    _assert_close(_f64(dx), rdx, adx, f"{arm} dx")
    _assert_close(_f64(dw), rdw, adw, f"{arm} dw")


def test_forward_bitwise_identical_across_overrides(mx):
    x, w, dy, offs_t = _moe_small(6)
    ys = []
    for arm in (None, "quantized", "high_precision", "dequantized"):
        op = mx.MXFP8GroupedMM(backward_override=arm)
        ys.append(op.forward(x.cuda(), w.cuda(), offs_t.cuda()))
        op.backward(dy.cuda())
    mx.mx_device_error()
    for y in ys[1:]:
        assert torch.equal(ys[0], y)


def test_stride0_grad_through_every_arm(mx):
    x, w, _, offs_t = _moe_small(7)
    dy = torch.ones(1, 1, dtype=torch.bfloat16, device="cuda").expand(x.shape[0], w.shape[1])
    grads = []
    for arm in (None, "high_precision", "dequantized"):
        op = mx.MXFP8GroupedMM(backward_override=arm)
        op.forward(x.cuda(), w.cuda(), offs_t.cuda())
        grads.append(op.backward(dy))
    mx.mx_device_error()
    ref = O.moe_backward_high_precision(S.bf16_bits(x), S.bf16_bits(w),
                                        S.bf16_bits(torch.ones(x.shape[0], w.shape[1], dtype=torch.bfloat16)),
                                        offs_t.numpy())
    _assert_close(_f64(grads[1][0]), ref[0], ref[1], "hp dx, stride-0 dy")
    _assert_close(_f64(grads[1][1]), ref[2], ref[3], "hp dw, stride-0 dy")


def test_wgrad_with_hp_matches_oracle_and_composes(mx):
    """wgrad_with_hp: dx is the MXFP8 dgrad (bitwise the default backward's), dw the
    bf16 wgrad (bitwise the high-precision arm's); with "high_precision" the flag
    changes nothing. Also through autograd and with a stride-0 dy."""
    x, w, dy, offs_t = _moe_small(9)
    out = {}
    for name, kw in (("mixed", dict(wgrad_with_hp=True)), ("quantized", {}),
                     ("hp", dict(backward_override="high_precision")),
                     ("hp_flag", dict(backward_override="high_precision", wgrad_with_hp=True))):
        op = mx.MXFP8GroupedMM(**kw)
        op.forward(x.cuda(), w.cuda(), offs_t.cuda())
        out[name] = op.backward(dy.cuda())
    mx.mx_device_error()
    rdx, adx, rdw, adw = O.moe_backward_wgrad_hp(S.bf16_bits(x), S.bf16_bits(w), S.bf16_bits(dy), offs_t.numpy())
    _assert_close(_f64(out["mixed"][0]), rdx, adx, "wgrad_with_hp dx")
    _assert_close(_f64(out["mixed"][1]), rdw, adw, "wgrad_with_hp dw")
    assert torch.equal(out["mixed"][0], out["quantized"][0])
    assert torch.equal(out["mixed"][1], out["hp"][1])
    assert torch.equal(out["hp_flag"][0], out["hp"][0]) and torch.equal(out["hp_flag"][1], out["hp"][1])

    xa = x.cuda().requires_grad_(True)
    wa = w.cuda().requires_grad_(True)
    mx.mxfp8_grouped_mm(xa, wa, offs_t.cuda(), wgrad_with_hp=True).backward(dy.cuda())
    assert torch.equal(xa.grad, out["mixed"][0]) and torch.equal(wa.grad, out["mixed"][1])

    ones = torch.ones(1, 1, dtype=torch.bfloat16, device="cuda").expand(x.shape[0], w.shape[1])
    op = mx.MXFP8GroupedMM(wgrad_with_hp=True)
    op.forward(x.cuda(), w.cuda(), offs_t.cuda())
    dx1, dw1 = op.backward(ones)
    mx.mx_device_error()
    r = O.moe_backward_wgrad_hp(S.bf16_bits(x), S.bf16_bits(w),
                                S.bf16_bits(torch.ones(x.shape[0], w.shape[1], dtype=torch.bfloat16)), offs_t.numpy())
    _assert_close(_f64(dx1), r[0], r[1], "wgrad_with_hp dx, stride-0 dy")
    _assert_close(_f64(dw1), r[2], r[3], "wgrad_with_hp dw, stride-0 dy")


def test_override_validation(mx):
    with pytest.raises(ValueError):
        mx.MXFP8GroupedMM(backward_override="fp32")
    op = mx.MXFP8GroupedMM(backward_override="dequantized")
    x, w, _, offs_t = _moe_small(8)
    with pytest.raises(TypeError):
        op.forward(x.float().cuda(), w.cuda(), offs_t.cuda())


def test_high_precision_full_size_sampled(mx):
    """G=8, K=N=4096, M=16384 (the benchmark's MoE layer), sampled outputs of both GEMMs."""
    xb, wb, dyb, offs_t = S.moe_problem(seed=0, device="cuda")
    offs_d = offs_t.cuda()
    dx = mx.grouped_mm_bf16(dyb, wb, offs_d)
    dw = mx.grouped_mm_bf16_wgrad(dyb, xb, offs_d)
    mx.mx_device_error()
    ends = offs_t.numpy().astype(np.int64)
    starts = np.concatenate([[0], ends[:-1]])
    rng = np.random.default_rng(3)
    dxc, dwc = dx.float().cpu().numpy(), dw.float().cpu().numpy()
    for r in rng.choice(16384, 48, replace=False):
        g = int(np.searchsorted(ends, r, side="right"))
        a = O.bf16_to_f64(_bits(dyb[r]))
        cols = rng.choice(4096, 16, replace=False)
        bm = O.bf16_to_f64(_bits(wb[g][:, cols]))
        ref, absref = a @ bm, np.abs(a) @ np.abs(bm)
        assert np.all(np.abs(dxc[r, cols] - ref) <= 2 ** -7 * np.abs(ref) + 1e-3 * absref), r
    for g in rng.choice(8, 4, replace=False):
        s, e = starts[g], ends[g]
        A = O.bf16_to_f64(_bits(dyb[s:e]))
        B = O.bf16_to_f64(_bits(xb[s:e]))
        for _ in range(8):
            n, k = int(rng.integers(4096)), int(rng.integers(4096))
            ref, absref = A[:, n] @ B[:, k], np.abs(A[:, n]) @ np.abs(B[:, k])
            assert abs(dwc[g, n, k] - ref) <= 2 ** -7 * abs(ref) + 1e-3 * absref, (g, n, k)


def test_high_precision_skewed_full_size_sampled(mx):
    """G=32, K=7168, N=2048, M=32768, Zipf groups with 3 empty: both bf16 gradients of
    the high-precision arm, sampled, and exact zeros for the empty groups' dW."""
    xb, wb, dyb, offs_t = S.unaligned_grouped_problem(device="cuda")    # x [M, K], w [G, N, K], dy [M, N]
    offs_d = offs_t.cuda()
    dx = mx.grouped_mm_bf16(dyb, wb, offs_d)                           # [M, K]
    dw = mx.grouped_mm_bf16_wgrad(dyb, xb, offs_d)                     # [G, N, K]
    mx.mx_device_error()
    G, N, K = wb.shape
    ends = offs_t.numpy().astype(np.int64)
    starts = np.concatenate([[0], ends[:-1]])
    rng = np.random.default_rng(6)
    dxc = dx.float().cpu().numpy()
    for r in rng.choice(dyb.shape[0], 24, replace=False):
        g = int(np.searchsorted(ends, r, side="right"))
        a = O.bf16_to_f64(_bits(dyb[r]))
        cols = rng.choice(K, 16, replace=False)
        bm = O.bf16_to_f64(_bits(wb[g][:, cols]))
        ref, absref = a @ bm, np.abs(a) @ np.abs(bm)
        assert np.all(np.abs(dxc[r, cols] - ref) <= 2 ** -7 * np.abs(ref) + 1e-3 * absref), r
    for g in range(G):
        if ends[g] == starts[g]:
            assert not dw[g].any(), g
    for g in rng.choice([g for g in range(G) if ends[g] > starts[g]], 5, replace=False):
        A = O.bf16_to_f64(_bits(dyb[starts[g]:ends[g]]))
        B = O.bf16_to_f64(_bits(xb[starts[g]:ends[g]]))
        for _ in range(6):
            n, k = int(rng.integers(N)), int(rng.integers(K))
            ref, absref = A[:, n] @ B[:, k], np.abs(A[:, n]) @ np.abs(B[:, k])
            got = float(dw[g, n, k])
            assert abs(got - ref) <= 2 ** -7 * abs(ref) + 1e-3 * absref, (g, n, k)


@pytest.mark.parametrize("M,K,sizes", [(50, 40, None), (50, 40, [20, 0, 30]), (7, 8, [7])])
def test_bf16_row_groups_tiny_shapes(mx, M, K, sizes):
    """Fewer rows than a tile and a contraction shorter than one 64-deep step:
    the operand boxes reach past the tensors and read zeros."""
    N = 256
    G = len(sizes) if sizes else 1
    a = S.normal_bf16((M, K), seed=M + K)
    b = S.normal_bf16((G, K, N), 0.05, seed=G + K)
    offs_t = S.offsets_from_sizes(sizes) if sizes else None
    out = mx.grouped_mm_bf16(a.cuda(), b.cuda(), offs_t.cuda() if sizes else None)
    mx.mx_device_error()
    af, bf = O.bf16_to_f64(S.bf16_bits(a)), O.bf16_to_f64(S.bf16_bits(b))
    offs = offs_t.numpy() if sizes else np.array([M])
    _assert_close(_f64(out), O.hp_grouped_mm_m(af, bf, offs), O.hp_grouped_mm_m(np.abs(af), np.abs(bf), offs),
                  "tiny row groups")


def test_bf16_token_groups_tiny_shapes(mx):
    """Groups of a few tokens (every one a partial 64-token step)."""
    sizes = [3, 0, 1, 10]
    M, N, K = sum(sizes), 256, 256
    a = S.normal_bf16((M, N), seed=5)
    b = S.normal_bf16((M, K), seed=6)
    offs_t = S.offsets_from_sizes(sizes)
    out = mx.grouped_mm_bf16_wgrad(a.cuda(), b.cuda(), offs_t.cuda())
    mx.mx_device_error()
    af, bf = O.bf16_to_f64(S.bf16_bits(a)), O.bf16_to_f64(S.bf16_bits(b))
    offs = offs_t.numpy()
    _assert_close(_f64(out), O.hp_grouped_mm_k(af, bf, offs), O.hp_grouped_mm_k(np.abs(af), np.abs(bf), offs),
                  "tiny token groups")


@pytest.mark.parametrize("arm,hp", [(None, False), (None, True), ("high_precision", False), ("dequantized", False)])
def test_layer_with_no_tokens(mx, arm, hp):
    """Every group empty (M = 0): the forward returns [0, N], dX [0, K], and dW
    exact zeros for every expert, under each backward arm."""
    Gz, Nz, Kz = 4, 256, 384
    x = torch.empty(0, Kz, dtype=torch.bfloat16, device="cuda")
    dy = torch.empty(0, Nz, dtype=torch.bfloat16, device="cuda")
    w = S.normal_bf16((Gz, Nz, Kz), 0.02, seed=9, device="cuda")
    offs = torch.zeros(Gz, dtype=torch.int32, device="cuda")
    op = mx.MXFP8GroupedMM(backward_override=arm, wgrad_with_hp=hp)
    y = op.forward(x, w, offs)
    dx, dw = op.backward(dy)
    torch.cuda.synchronize()
    mx.mx_device_error()
    assert tuple(y.shape) == (0, Nz) and tuple(dx.shape) == (0, Kz) and tuple(dw.shape) == (Gz, Nz, Kz)
    assert not dw.any()
