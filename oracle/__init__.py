"""CPU oracle for NVFP4 quantization and the W4A4 block-scaled GEMM.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the product package.
"""
from .oracle import *  # noqa: F401,F403
