"""Failure detection without a GPU fault: a wait on an mbarrier that nothing arrives on must end
after its time limit (about a second) with a recorded status, and the CUDA context must stay
usable afterwards (a forward call still matches the oracle). The kernel uses the library's own
bounded-wait helper; nothing here traps, faults or hangs."""
import ctypes
import os
import subprocess

import pytest

from parity import TOL, compare, run_gpu, run_oracle, workload_inputs
from titans_long_term_b200 import mem

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def test_bounded_wait_times_out_and_context_survives(tmp_path):
    lib = str(tmp_path / "libprobe.so")
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17", "-shared",
                    "-Xcompiler", "-fPIC", os.path.join(HERE, "csrc", "wait_timeout_probe.cu"), "-o", lib],
                   check=True)
    L = ctypes.CDLL(lib)
    st = ctypes.c_uint(0)
    ns = ctypes.c_ulonglong(0)
    assert L.run_never_arrives(ctypes.byref(st), ctypes.byref(ns)) == 0
    assert st.value == 2  # timeout recorded
    assert 0.9e9 <= ns.value <= 5e9  # gave up after about the 1 s limit
    # the context is still usable: a forward call right after matches the oracle
    w, inp = workload_inputs("mlp-d64-b2h4-t2k", T=128)
    m = mem.Memory(64, 256, 64, "bf16", 2, 4)
    gy, gst = run_gpu(m, inp, 2, 4, 64)
    ry, rst = run_oracle(inp, 64)
    compare(gy, gst, ry, rst, TOL["bf16"], what="after timeout")
