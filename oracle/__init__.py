"""CPU oracle for the MXFP8 training hot path.

TEST INFRASTRUCTURE ONLY. Nothing in the product path (the package
``mxfp8_block_scaled_cast_b200`` and its CUDA library) imports, links or calls
anything here. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of
``bench.py`` (``cpu_baseline`` and ``--impl reference``) use it.

The oracle is plain numpy in float64: slow, unblocked, and written so that a
reader can check each step against its definition. See ``mx_oracle`` for the
citations of every function.
"""
from . import mx_oracle  # noqa: F401
