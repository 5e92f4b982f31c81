"""The debug build (libnvfp4_debug.so, compiled with NVFP4_DEBUG_CHECKS) in
place of a memory checker: every kernel's direct global stores are checked
against the extent of the buffer they write, and a store that would leave it
is skipped and reported as ERR_BOUNDS in the workspace status word (no trap).

The small-shape GPU parity tests -- ragged M, N and K (K = 64, 128, partial
K slabs), swapped and stream-K tiles, the CTA pair, the one-launch decode
kernel, the fused MLP, re-quantized outputs, MXFP4, W4A16, W4A8 -- run again
in a child process that loads the debug build.  They compare every result
with the oracle and assert that the status word is clean after each call,
so an out-of-bounds store fails them either way."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
MODULES = ["tests/test_quantize_gpu.py", "tests/test_gemm_gpu.py", "tests/test_linear_gpu.py",
           "tests/test_decode_gpu.py", "tests/test_requant_gpu.py", "tests/test_mx_gpu.py",
           "tests/test_w4a16_gpu.py", "tests/test_w4a8_gpu.py"]
# full-size workloads are covered by the release-build tests; here the small,
# ragged shapes where an index mistake would reach past a buffer's end
DESELECT = "not full and not workload and not timed_call and not 4096-5120 and not 8192 and not 17408"


def test_small_shape_suite_on_the_debug_build():
    lib = os.path.join(ROOT, "nvfp4_block_scaled_21_b200", "libnvfp4_debug.so")
    assert os.path.exists(lib), "libnvfp4_debug.so is not built (build(debug=True))"
    env = dict(os.environ, NVFP4_LIBRARY="debug")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-k", DESELECT,
                        "-p", "no:cacheprovider", *MODULES],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1500)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-30:])
    assert r.returncode == 0, tail
    assert " passed" in tail, tail


def test_debug_build_is_loaded_in_the_child():
    """The switch really loads the debug library (not the release one)."""
    env = dict(os.environ, NVFP4_LIBRARY="debug")
    code = ("import nvfp4_block_scaled_21_b200 as nv, os; "
            "print(nv.DEBUG_BUILD, os.path.basename(nv.LIB_PATH))")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.split() == ["True", "libnvfp4_debug.so"]
