"""The bounds-checked build (libtitans_mem_debug.so, compiled with -DTITANS_DEBUG) passes the
tensor-core parity suites (the deep memory's and the backward's included) with a clean status word: none of its checks on TMA coordinates, gate and
token indices, shared-memory and TMEM offsets fires on any parity case, and its results still match
the oracle. The suites run in a child process with TITANS_DEBUG=1, which makes the binding load the
debug library; the child also confirms from its own memory map that this library is the one loaded."""
import os
import subprocess
import sys

import pytest

from titans_long_term_b200 import build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SUITES = ["tests/test_parity_gpu.py", "tests/test_phased_gpu.py", "tests/test_chunk_gates_gpu.py",
          "tests/test_gated_gpu.py", "tests/test_stated_inputs_gpu.py", "tests/test_deep_gpu.py",
          "tests/test_backward_gpu.py"]

CHILD = r"""
import sys, pytest
from titans_long_term_b200 import mem
assert mem.DEBUG and mem.LIB_PATH.endswith("libtitans_mem_debug.so"), mem.LIB_PATH
rc = pytest.main(["-q", "-x", "-m", "gpu", "-p", "no:cacheprovider", *sys.argv[1:]])
maps = open("/proc/self/maps").read()
assert "libtitans_mem_debug.so" in maps and "libtitans_mem.so" not in maps, "wrong library loaded"
sys.exit(int(rc))
"""


def test_debug_build_passes_the_parity_suites():
    build.build(debug=True)  # no-op when it is up to date
    env = dict(os.environ, TITANS_DEBUG="1")
    res = subprocess.run([sys.executable, "-c", CHILD, *SUITES], cwd=ROOT, env=env, capture_output=True,
                         text=True, timeout=1200)
    tail = (res.stdout + res.stderr)[-3000:]
    print(tail)
    assert res.returncode == 0, tail
