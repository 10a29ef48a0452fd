"""The allocation-free entry point (titans_mem_forward_noalloc) against the existing entry
point (titans_mem_forward on the CUDA-core kernel) and the oracle, through the C ABI.

Some callers cannot allocate device memory: code inside another framework's stream capture,
under an allocator that owns the device, on a path that must not synchronize the device.
The entry point serves them with a fixed scratch array inside the library. It runs the same
kernel as the handle's CUDA-core path on the same inputs, so its results must be equal bit
for bit; two calls in a row check that reusing the shared array leaves no trace. Each
result is also held to the oracle at the usual bars. This file is collected last on purpose."""
import pytest
import torch

from parity import TOL, compare, gpu_inputs, run_oracle
from titans_long_term_b200 import mem, synth

pytestmark = pytest.mark.gpu


def _run_reference(w, inp, B, H, mode, chunk):
    m = mem.Memory(w.d, w.h, chunk, mode, B, H, cuda_cores=True)
    assert m.path(chunk) == mem.PATH_CUDA_CORES
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
    ry, rst = run_oracle(inp, w.chunk)
    for call in range(2):  # two calls in a row share the fixed scratch array
        y, st = _run_noalloc(inp, B, H, mode, w.chunk)
        assert torch.equal(y, y_ref), (call, "y differs from the handle's CUDA-core path")
        for n in st:
            assert torch.equal(st[n], st_ref[n]), (call, n, "differs from the handle's CUDA-core path")
        gy = y.reshape(units, T, w.d).float().cpu().numpy()
        gst = {n: t.reshape(units, *t.shape[2:]).cpu().numpy() for n, t in st.items()}
        compare(gy, gst, ry, rst, TOL[mode], what=f"noalloc {name} {mode} call {call}")


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
