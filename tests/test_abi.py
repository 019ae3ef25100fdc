"""The C-ABI library builds, loads without a GPU and exports every entry point
that include/mx.h declares; the host-only helpers agree with the oracle."""
import ctypes
import os
import re

import numpy as np

from oracle import mx_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"^MX_API\s+[\w\s\*]+?\b(mx_\w+)\s*\(", text, flags=re.M)
    return names


def _lib():
    from mxfp8_block_scaled_cast_b200 import build
    return ctypes.CDLL(build.build_library())


def test_header_declares_the_entry_points():
    names = _declared()
    for must in ("mx_cast_dim0", "mx_cast_dim1", "mx_cast_2d", "mx_cast_w32x32",
                 "mx_cast_dim0_grouped", "mx_cast_dim1_grouped", "mx_cast_2d_grouped"):
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = _lib()
    for name in _declared():
        assert hasattr(lib, name), name


def test_binding_covers_the_header():
    from mxfp8_block_scaled_cast_b200 import mx
    assert set(_declared()) <= set(mx.exported_names())


def test_host_helpers_match_oracle():
    from mxfp8_block_scaled_cast_b200 import mx
    for r, c in ((1, 1), (128, 4), (300, 18), (16384, 128), (0, 4)):
        want = O.blocked_scale_bytes(r, c) if r > 0 else 0
        assert mx.mx_scale_bytes(r, c) == want
    for m, g in ((16384, 8), (32768, 32), (357, 4), (0, 1)):
        assert mx.mx_padded_rows_capacity(m, g) == O.padded_rows_capacity(m, g)
    assert mx.lib().mx_last_error() is not None
    assert np.int64(mx.mx_padded_rows_capacity(-1, 1)) == -1


def test_no_silent_fallback_without_the_library_or_a_gpu(monkeypatch, tmp_path):
    """The product path raises when libmx.so is missing or a tensor is on the
    host: there is no CPU implementation behind the binding."""
    import pytest
    import torch
    from mxfp8_block_scaled_cast_b200 import mx
    monkeypatch.setattr(mx, "_lib", None)
    monkeypatch.setattr(mx, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        mx.lib()
    monkeypatch.undo()
    x = torch.zeros(32, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="device tensors"):
        mx.cast_dim0(x)
    with pytest.raises(ValueError):
        mx.MXFP8GroupedMM(backward_override="fp32")


def test_host_argument_checks_return_before_any_launch():
    """Argument errors are reported from host checks alone (no device is touched:
    the pointers below are never dereferenced)."""
    from mxfp8_block_scaled_cast_b200 import mx
    L = mx.lib()
    ok16, odd = ctypes.c_void_p(0x100000), ctypes.c_void_p(0x100008)
    assert L.mx_cast_dim0(ok16, 64, 48, ok16, ok16, None) == 3          # C not a multiple of 32
    assert L.mx_cast_dim0(odd, 64, 64, ok16, ok16, None) == 2           # misaligned input
    assert L.mx_cast_dim1(ok16, 48, 64, ok16, ok16, None) == 3          # R not a multiple of 32
    assert L.mx_cast_ex(ok16, 64, 64, 3, 7, ok16, ok16, ok16, ok16, None) == 1   # unknown rule
    assert L.mx_grouped_mm(ok16, ok16, ok16, ok16, None, 1, 5, ok16, 128, 256, 128, 0, None) == 1  # mode
    assert L.mx_grouped_mm(ok16, ok16, ok16, ok16, None, 1, 0, ok16, 128, 200, 128, 0, None) == 3  # N % 32
    assert L.mx_grouped_mm_bf16(ok16, ok16, None, 1, 0, ok16, 128, 256, 60, None) == 3      # K % 8
    assert L.mx_grouped_mm_bf16(ok16, ok16, ok16, 0, 0, ok16, 128, 256, 64, None) == 1      # G = 0
    assert L.mx_dequant_dim0(ok16, ok16, 1, 4, 40, ok16, None) == 3     # C not a multiple of 32
    assert L.mx_grouped_mm_experts(ok16, ok16, ok16, ok16, ok16, 6, 4, 0, ok16, 128, 256, 128, 1024,
                                   None) == 1                           # E does not divide G
    assert L.mx_grouped_mm_experts(ok16, ok16, ok16, ok16, None, 1, 2, 0, ok16, 128, 256, 128, 0,
                                   None) == 1                           # dense needs E = 1
    assert L.mx_scales_unswizzle(odd, 4, 4, ok16, None) == 2
    # the scatter cast checks every destination on the host
    two = lambda *v: (ctypes.c_void_p * 2)(*v)
    assert L.mx_cast_dim0_grouped_scatter(ok16, 64, 64, ok16, 2, 256, None, two(0x100000, 0x100000),
                                          None) == 1                    # null destination array
    assert L.mx_cast_dim0_grouped_scatter(ok16, 64, 64, ok16, 2, 256, two(0x100000, None),
                                          two(0x100000, 0x100000), None) == 1   # null destination
    assert L.mx_cast_dim0_grouped_scatter(ok16, 64, 64, ok16, 2, 256, two(0x100000, 0x100008),
                                          two(0x100000, 0x100000), None) == 2   # misaligned destination
    # the fused scatter cast: four destinations and a capacity per group
    ok2 = two(0x100000, 0x100000)
    caps = (ctypes.c_int64 * 2)(256, 256)
    assert L.mx_cast_2d_grouped_scatter(ok16, 64, 64, ok16, 2, 256, ok2, ok2, ok2, None, caps,
                                        None) == 1                      # null destination array
    assert L.mx_cast_2d_grouped_scatter(ok16, 64, 64, ok16, 2, 256, ok2, ok2, two(0x100000, 0x100008), ok2,
                                        caps, None) == 2                # misaligned destination
    assert L.mx_cast_2d_grouped_scatter(ok16, 64, 64, ok16, 2, 256, ok2, ok2, ok2, ok2,
                                        (ctypes.c_int64 * 2)(256, 200), None) == 1   # capacity not 128-aligned
    many = (ctypes.c_void_p * 513)(*([0x100000] * 513))
    assert L.mx_cast_2d_grouped_scatter(ok16, 64, 64, ok16, 513, 128 * 513, many, many, many, many,
                                        (ctypes.c_int64 * 513)(*([256] * 513)), None) == 3   # above 512 groups
    # the GEMM with per-group output rows: M-group modes only, every destination checked
    assert L.mx_grouped_mm_experts_to_rows(ok16, ok16, ok16, ok16, ok16, 2, 2, 1, two(0x100000, 0x100000),
                                           128, 256, 128, 256, None) == 1    # K-groups mode
    assert L.mx_grouped_mm_experts_to_rows(ok16, ok16, ok16, ok16, None, 1, 1, 0, two(0x100000, 0x100000),
                                           128, 256, 128, 256, None) == 1    # no offsets
    assert L.mx_grouped_mm_experts_to_rows(ok16, ok16, ok16, ok16, ok16, 2, 2, 0, two(0x100000, 0x100004),
                                           128, 256, 128, 256, None) == 2    # misaligned destination
    # the linear training pair: its own workspace, larger than the plain pair's when K > 2N
    # (the forward holds both casts of x at once), the same where dY's casts are the larger
    Ml, Nl, Kl = 256, 96, 576
    plain, train = L.mx_linear_ws_bytes(Ml, Nl, Kl), L.mx_linear_train_ws_bytes(Ml, Nl, Kl)
    assert train > plain
    assert L.mx_linear_train_ws_bytes(4096, 4096, 2048) == L.mx_linear_ws_bytes(4096, 4096, 2048)
    assert L.mx_linear_fwd_train(ok16, ok16, Ml, Nl, Kl, None, 0, ok16, ok16, plain, None) == 1  # ws too small
    assert L.mx_linear_bwd_after_fwd(ok16, ok16, Ml, Nl, Kl, None, 0, ok16, ok16, ok16, plain, None) == 1
    assert L.mx_linear_fwd_train(ok16, ok16, 48, Nl, Kl, None, 0, ok16, ok16, train, None) == 3  # M % 32
    assert L.mx_linear_bwd_after_fwd(ok16, ok16, Ml, Nl, Kl, None, 0, ok16, ok16, odd, train, None) == 2
    msg = (L.mx_cast_dim0(ok16, 64, 48, ok16, ok16, None), L.mx_last_error())[1]
    assert b"not a multiple of 32" in msg


def test_oracle_and_product_share_no_code():
    """The oracle is independent of the CUDA path: the product package (its Python
    and its CUDA sources) never imports, includes or reads anything under oracle/,
    and the oracle imports nothing but numpy. Only tests, smoke() and bench.py's
    CPU legs may use the oracle."""
    import ast
    pkg = os.path.join(ROOT, "mxfp8_block_scaled_cast_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            path = os.path.join(dirpath, f)
            if f.endswith((".py", ".cu", ".cuh", ".h", ".c")):
                text = open(path).read()
                for tok in ("mx_oracle", "import oracle", "from oracle", "oracle/"):
                    assert tok not in text, f"{path} refers to the oracle ({tok!r})"
            if f.endswith(".py"):
                tree = ast.parse(open(path).read())
                for node in ast.walk(tree):
                    mods = [a.name for a in node.names] if isinstance(node, ast.Import) else (
                        [node.module or ""] if isinstance(node, ast.ImportFrom) else [])
                    assert not any(m.split(".")[0] == "oracle" for m in mods), f"{path} imports the oracle"
    tree = ast.parse(open(os.path.join(ROOT, "oracle", "mx_oracle.py")).read())
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            assert all(a.name.split(".")[0] in ("numpy",) for a in node.names), ast.dump(node)
        elif isinstance(node, ast.ImportFrom) and node.module not in ("__future__",):
            assert (node.module or "").split(".")[0] == "numpy", ast.dump(node)
