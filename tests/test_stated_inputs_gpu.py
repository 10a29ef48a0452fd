"""GPU parity at the workloads' stated input distributions, against the token-loop oracle.

The stated recipe draws k, q, v ~ N(0, I) independently per token (k, q l2-normalised) and
the gates alpha ~ U(0, 0.05), eta ~ U(0.8, 0.99), theta ~ U(0, 0.1). The 2-layer MLP memory
diverges on these inputs: the oracle's own weights grow about 100x per chunk from the third
64-token chunk on, and past about 16 tokens at chunk 1. So these tests cover the horizon over
which the method's result is finite -- one to two chunks of the chunked forward, 12 decode
steps -- where the larger theta makes the c- and d-scaled bf16 operands of the weight GEMMs
as large as they get. Every kernel runs here: the tcgen05 chunk kernel (bf16, 2e-2), the
CUDA-core chunk kernel (fp32 reference mode, 1e-4; and the wide memory in bf16) and the
cluster decode step. The linear memory's workload runs on this recipe by default, over its
whole stream (tests/test_parity_gpu.py).
"""
import pytest

from parity import TOL, compare, run_gpu, run_oracle, step_sequence
from titans_long_term_b200 import mem, synth

pytestmark = pytest.mark.gpu

STATED = "stated"


def _inputs(name, units, T, mode):
    w = synth.WORKLOADS[name]
    return w, synth.make_inputs(w, units=range(units), T=T, dtype=mode, recipe=STATED)


@pytest.mark.parametrize("name,B,H,T,chunk", [
    ("mlp-d64-b2h4-t2k", 2, 4, 64, 64),     # one chunk: y and the first update at W0
    ("mlp-d64-b2h4-t2k", 2, 4, 128, 64),    # two chunks
    ("mlp-d64-b2h4-t2k", 2, 4, 100, 64),    # ragged second chunk
    ("mlp-d64-b2h4-t2k", 2, 4, 96, 32),     # three chunks of 32
    ("mlp-d64-b2h4-t2k", 2, 4, 48, 16),     # three chunks of 16
    ("mlp-d64-b8h16-t4k", 8, 16, 128, 64),  # the 760M-class layer's 128 units, two chunks
])
def test_tensor_core_kernel_at_stated_inputs(name, B, H, T, chunk):
    w, inp = _inputs(name, B * H, T, "bf16")
    m = mem.Memory(w.d, w.h, chunk, "bf16", B, H)
    assert m.path(chunk) == mem.PATH_TC_MLP64
    gy, gst = run_gpu(m, inp, B, H, chunk)
    ry, rst = run_oracle(inp, chunk)
    worst = compare(gy, gst, ry, rst, TOL["bf16"], what=f"tc stated T={T} chunk={chunk}")
    print(f"tc stated {name} T={T} chunk={chunk}:", {k: f"{v:.2e}" for k, v in worst.items()})


@pytest.mark.parametrize("name,B,H,T,chunk,mode", [
    ("mlp-d64-b2h4-t2k", 2, 4, 128, 64, "fp32"),
    ("mlp-d64-b2h4-t2k", 2, 4, 100, 64, "fp32"),
    ("mlp-d64-b8h16-t4k", 8, 16, 128, 64, "fp32"),
    ("mlp-d128-b4h8-t16k", 2, 4, 256, 128, "fp32"),  # the wide memory's prefill shape, two chunks
    ("mlp-d128-b4h8-t16k", 2, 4, 200, 128, "fp32"),
    ("mlp-d128-b4h8-t16k", 2, 4, 256, 128, "bf16"),
])
def test_cuda_core_kernel_at_stated_inputs(name, B, H, T, chunk, mode):
    w, inp = _inputs(name, B * H, T, mode)
    m = mem.Memory(w.d, w.h, chunk, mode, B, H, cuda_cores=True)
    assert m.path(chunk) == mem.PATH_CUDA_CORES
    gy, gst = run_gpu(m, inp, B, H, chunk)
    ry, rst = run_oracle(inp, chunk)
    compare(gy, gst, ry, rst, TOL[mode], what=f"cuda cores stated {name} T={T} {mode}")


@pytest.mark.parametrize("name,mode", [("mlp-d64-b2h4-t2k", "bf16"), ("mlp-d64-b2h4-t2k", "fp32"),
                                       ("mlp-d128-b4h8-t16k", "bf16"), ("mlp-d128-b4h8-t16k", "fp32")])
def test_decode_step_at_stated_inputs(name, mode):
    """12 single-token steps (chunk = 1 semantics) from the seeded W0, every unit of a 4 x 2 batch."""
    w, inp = _inputs(name, 8, 12, mode)
    m = mem.Memory(w.d, w.h, 1, mode, 4, 2)
    assert m.path(1, step=True) == mem.PATH_STEP_CLUSTER
    gy, gst = step_sequence(m, inp, 4, 2, 12)
    ry, rst = run_oracle(inp, 1)
    compare(gy, gst, ry, rst, TOL[mode], what=f"step stated {name} {mode}")
