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
