"""The allocation-free entry point (titans_mem_forward_noalloc) against the existing entry
point (titans_mem_forward with the CUDA-core kernel), through the C ABI.

Some callers cannot allocate device memory (inside another framework's stream capture,
under an allocator that owns the device, on a path that must not synchronize); this entry
point serves them with a fixed scratch array inside the library. Two calls in a row check
that reusing the shared array leaves no trace. This file is collected last on purpose."""
import ctypes

import pytest
import torch

from parity import gpu_inputs, rel_err
from titans_long_term_b200 import mem, synth

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-4, "bf16": 2e-2}


def _run_reference(w, inp, B, H, mode, chunk):
    m = mem.Memory(w.d, w.h, chunk, mode, B, H, cuda_cores=True)
    toks, gates, state = gpu_inputs(inp, B, H)
    y = m.forward(toks["k"], toks["q"], toks["v"], gates["alpha"], gates["eta"], gates["theta"], state, chunk=chunk)
    m.sync_status()
    return y, state


def _run_noalloc(inp, B, H, mode, chunk):
    toks, gates, state = gpu_inputs(inp, B, H)
    y = mem.forward_noalloc(toks["k"], toks["q"], toks["v"], gates["alpha"], gates["eta"], gates["theta"], state,
                            chunk, mode)
    torch.cuda.synchronize()
    return y, state


@pytest.mark.parametrize("name,mode,T,units,B,H", [
    ("mlp-d64-b2h4-t2k", "fp32", 300, 8, 2, 4),
    ("mlp-d64-b2h4-t2k", "bf16", 256, 8, 2, 4),
    ("linear-d64", "fp32", 256, 1, 1, 1),
    ("mlp-d128-b4h8-t16k", "bf16", 200, 4, 2, 2),
])
def test_noalloc_matches_forward_twice(name, mode, T, units, B, H):
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w, units=range(units), T=T, dtype=mode)
    y_ref, st_ref = _run_reference(w, inp, B, H, mode, w.chunk)
    for call in range(2):  # two calls in a row share the fixed scratch array
        y, st = _run_noalloc(inp, B, H, mode, w.chunk)
        e = rel_err(y.reshape(units, -1).float().cpu().numpy(), y_ref.reshape(units, -1).float().cpu().numpy())
        assert e.max() <= TOL[mode], (call, "y", e.max())
        for n in st:
            e = rel_err(st[n].reshape(units, -1).cpu().numpy(), st_ref[n].reshape(units, -1).cpu().numpy())
            assert e.max() <= TOL[mode], (call, n, e.max())


def test_noalloc_rejects_oversized_scratch():
    """128 units of the 64-256-64 memory at chunk 64 need ~34.9 MB of scratch > 16 MiB."""
    w = synth.WORKLOADS["mlp-d64-b8h16-t4k"]
    B, H, T = 8, 16, 64
    dev = "cuda"
    k = torch.zeros(B, H, T, 64, dtype=torch.bfloat16, device=dev)
    g = torch.zeros(B, H, T, device=dev)
    st = mem.new_state(B, H, 64, 256)
    with pytest.raises(mem.TitansError) as ei:
        mem.forward_noalloc(k, k, k, g, g, g, st, 64, "bf16")
    assert ei.value.status == mem.EUNSUPPORTED
    assert "exceeds" in str(ei.value)
