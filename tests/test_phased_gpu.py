"""GPU parity of the phased tensor-core kernel (the wide memory, d = 128, h = 512, bf16) against
the token-loop oracle, plus its invariants checked bitwise on the GPU."""
import pytest
import torch

from parity import TOL, compare, gpu_inputs, run_gpu, run_oracle
from titans_long_term_b200 import mem, synth

pytestmark = pytest.mark.gpu

WIDE = synth.WORKLOADS["mlp-d128-b4h8-t16k"]


@pytest.mark.parametrize("B,H,T,chunk,recipe", [
    (2, 2, 300, 128, None),      # two full chunks and a ragged one
    (2, 2, 128, 128, None),      # exactly one chunk
    (2, 2, 200, 64, None),       # chunk below the tile height: padded token rows
    (1, 3, 100, 32, None),       # odd unit count, four chunks
    (4, 8, 256, 128, None),      # the wide workload's 32 units: more tiles than SMs in P1 and P4
    (2, 4, 256, 128, "stated"),  # the stated input distributions, two chunks
])
def test_phased_kernel_matches_the_oracle(B, H, T, chunk, recipe):
    inp = synth.make_inputs(WIDE, units=range(B * H), T=T, recipe=recipe)
    m = mem.Memory(128, 512, chunk, "bf16", B, H)
    assert m.path(chunk) == mem.PATH_TC_PHASED
    gy, gst = run_gpu(m, inp, B, H, chunk)
    ry, rst = run_oracle(inp, chunk)
    worst = compare(gy, gst, ry, rst, TOL["bf16"], what=f"phased B={B} H={H} T={T} chunk={chunk}")
    print(f"phased T={T} chunk={chunk} {recipe}:", {k: f"{v:.2e}" for k, v in worst.items()})


def _run(inp, B, H, chunk=128):
    m = mem.Memory(128, 512, chunk, "bf16", B, H)
    toks, gates, state = gpu_inputs(inp, B, H)
    y = m.forward(toks["k"], toks["q"], toks["v"], gates["alpha"], gates["eta"], gates["theta"], state)
    m.sync_status()
    return y, state


def test_phased_kernel_is_deterministic_and_split_invariant():
    """Two runs agree bit for bit, and forward(T1) then forward(T2) equals forward(T1 + T2) bit for
    bit when T1 is a multiple of the chunk (the state handed between calls is the whole state)."""
    inp = synth.make_inputs(WIDE, units=range(4), T=384)
    y, s = _run(inp, 2, 2)
    y2, s2 = _run(inp, 2, 2)
    assert torch.equal(y, y2) and all(torch.equal(s[n], s2[n]) for n in s)
    first = {n: (x[:, :256] if n in ("k", "q", "v", "alpha", "eta", "theta") else x) for n, x in inp.items()}
    ya, sa = _run(first, 2, 2)
    second = {n: x[:, 256:] for n, x in inp.items() if n in ("k", "q", "v", "alpha", "eta", "theta")}
    second.update({n: t.reshape(4, *t.shape[2:]).cpu() for n, t in sa.items()})
    yb, sb = _run(second, 2, 2)
    assert torch.equal(torch.cat([ya, yb], dim=2), y)
    assert all(torch.equal(s[n], sb[n]) for n in s)


def test_phased_retrieval_does_not_write():
    """The final state does not depend on the queries (bitwise)."""
    inp = synth.make_inputs(WIDE, units=range(4), T=256)
    _, s1 = _run(inp, 2, 2)
    alt = dict(inp)
    alt["q"] = inp["k"].clone()
    _, s2 = _run(alt, 2, 2)
    assert all(torch.equal(s1[n], s2[n]) for n in s1)


def test_cuda_core_flag_still_selects_the_cuda_core_kernel():
    m = mem.Memory(128, 512, 128, "bf16", 1, 1, cuda_cores=True)
    assert m.path(128) == mem.PATH_CUDA_CORES
    assert mem.Memory(128, 512, 128, "fp32", 1, 1).path(128) == mem.PATH_CUDA_CORES
