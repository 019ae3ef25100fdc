"""The C ABI from a plain C host program (tests/c_abi/mx_c_host.c): no C++, no
Python, no torch -- include/mx.h, libmx.so and the CUDA runtime only.

Without a GPU: the program compiles as C99 with every warning an error and
links against the library's exports. On a B200: it runs, casts a bf16 matrix
rowwise (its codes and blocked scales are checked here bit for bit against the
oracle), requires the linear forward with a workspace and without any
allocation to agree bitwise, the linear training pair to agree bitwise with the separate
forward and backward calls, and requires a bad width to be refused.
"""
import os
import subprocess

import numpy as np
import pytest

from oracle import mx_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")
M, K = 256, 320


def _build(tmp_path):
    from mxfp8_block_scaled_cast_b200 import build
    lib = build.build_library()
    exe = tmp_path / "mx_c_host"
    libdir = os.path.dirname(lib)
    cmd = ["gcc", "-std=c99", "-O2", "-Wall", "-Wextra", "-Werror",
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
           os.path.join(ROOT, "tests", "c_abi", "mx_c_host.c"),
           "-L", libdir, "-lmx", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
           f"-Wl,-rpath,{libdir}:{os.path.join(CUDA, 'lib64')}", "-o", str(exe)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stdout + res.stderr
    return exe


def test_c_program_compiles_and_links(tmp_path):
    assert _build(tmp_path).exists()


@pytest.mark.gpu
def test_c_program_runs_and_matches_the_oracle(tmp_path):
    exe = _build(tmp_path)
    out = tmp_path / "run"
    res = subprocess.run([str(exe), str(out)], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0 and res.stdout.strip() == "ok", res.stdout + res.stderr
    x = np.fromfile(f"{out}.x", dtype=np.uint16).reshape(M, K)
    q = np.fromfile(f"{out}.q", dtype=np.uint8).reshape(M, K)
    s = np.fromfile(f"{out}.s", dtype=np.uint8)
    eq, es = O.cast_dim0(x)
    assert np.array_equal(q, eq), "codes of the C program's cast"
    assert np.array_equal(s, O.swizzle(es)), "blocked scales of the C program's cast"
