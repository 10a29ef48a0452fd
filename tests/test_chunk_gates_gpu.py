"""Chunk-shared gates (TITANS_FLAG_CHUNK_GATES; walk-through sec. 3.2, "Parameters as the Function of
Chunks"): alpha, eta, theta given once per chunk. Every chunk kernel against the oracle run on the
gates repeated over each chunk's tokens, and bit for bit against the same kernel fed those repeated
gates per token."""
import numpy as np
import pytest
import torch

import oracle
from parity import TOL, compare, gpu_inputs
from titans_long_term_b200 import mem, synth

pytestmark = pytest.mark.gpu


def _chunk_gate_inputs(name, units, T, chunk, mode, recipe=None):
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w, units=range(units), T=T, dtype=mode, recipe=recipe)
    cg = {n: inp[n][:, ::chunk].contiguous() for n in ("alpha", "eta", "theta")}  # one value per chunk
    rep = dict(inp)
    for n in cg:
        rep[n] = torch.as_tensor(oracle.expand_chunk_gates(cg[n].numpy(), T, chunk))
    return w, inp, cg, rep


def _run(m, inp, gates, B, H, chunk):
    toks, _, state = gpu_inputs(inp, B, H)
    g = {n: t.reshape(B, H, -1).cuda().contiguous() for n, t in gates.items()}
    y = m.forward(toks["k"], toks["q"], toks["v"], g["alpha"], g["eta"], g["theta"], state, chunk=chunk)
    m.sync_status()
    return y, state


@pytest.mark.parametrize("name,B,H,T,chunk,mode,cuda_cores", [
    ("mlp-d64-b2h4-t2k", 2, 4, 200, 64, "bf16", False),    # tcgen05 chunk kernel, ragged last chunk
    ("mlp-d64-b2h4-t2k", 2, 4, 150, 32, "fp32", False),    # CUDA-core kernel, fp32 reference mode
    ("mlp-d128-b4h8-t16k", 2, 2, 300, 128, "bf16", False), # phased tensor-core kernel (wide memory)
    ("linear-d64", 1, 1, 256, 16, "fp32", False),          # linear memory
])
def test_chunk_gates_match_the_oracle_and_the_repeated_gates(name, B, H, T, chunk, mode, cuda_cores):
    w, inp, cg, rep = _chunk_gate_inputs(name, B * H, T, chunk, mode)
    mc = mem.Memory(w.d, w.h, chunk, mode, B, H, cuda_cores=cuda_cores, chunk_gates=True)
    y, st = _run(mc, inp, cg, B, H, chunk)
    mp = mem.Memory(w.d, w.h, chunk, mode, B, H, cuda_cores=cuda_cores)
    assert mp.path(chunk) == mc.path(chunk)
    y2, st2 = _run(mp, inp, {n: rep[n] for n in cg}, B, H, chunk)
    assert torch.equal(y, y2), "chunk gates differ from the same gates repeated per token"
    assert all(torch.equal(st[n], st2[n]) for n in st)
    U = B * H
    ry, rst = oracle.forward(*(rep[n] for n in ("k", "q", "v", "alpha", "eta", "theta")),
                             {n: rep[n] for n in rep if n[0] in "WS"}, chunk)
    compare(y.reshape(U, T, -1).float().cpu().numpy(),
            {n: t.reshape(U, *t.shape[2:]).float().cpu().numpy() for n, t in st.items()},
            ry, rst, TOL[mode], what=f"chunk gates {name} {mode}")


def test_chunk_gates_deep_memory():
    w = synth.WORKLOADS["mlp-d64-b2h4-t2k"]
    B, H, T, chunk, L = 2, 2, 100, 32, 3
    inp = synth.make_inputs(w, units=range(4), T=T, dtype="fp32")
    st = synth.make_deep_state(w, L, units=range(4))
    cg = {n: inp[n][:, ::chunk].contiguous() for n in ("alpha", "eta", "theta")}
    m = mem.Memory(64, 256, chunk, "fp32", B, H, layers=L, chunk_gates=True)
    dev = lambda x, *s: x.reshape(B, H, *s).cuda().contiguous()
    state = {n: dev(st[n], st[n].shape[-1]) for n in st}
    y = m.forward_deep(dev(inp["k"], T, 64), dev(inp["q"], T, 64), dev(inp["v"], T, 64),
                       *(dev(cg[n], cg[n].shape[-1]) for n in ("alpha", "eta", "theta")), state, chunk=chunk)
    m.sync_status()
    rep = {n: oracle.expand_chunk_gates(cg[n].numpy(), T, chunk) for n in cg}
    ry, rst = oracle.forward_deep(inp["k"], inp["q"], inp["v"], rep["alpha"], rep["eta"], rep["theta"],
                                  {"W": st["W"], "S": st["S"]}, chunk, L)
    compare(y.reshape(4, T, 64).cpu().numpy(), {n: t.reshape(4, -1).cpu().numpy() for n, t in state.items()},
            ry, rst, TOL["fp32"], what="chunk gates deep")


def test_chunk_gates_host_staged_forward_equals_the_device_forward():
    """titans_mem_forward_host with chunk gates (segments start at chunk columns) equals
    titans_mem_forward bit for bit."""
    w, inp, cg, _ = _chunk_gate_inputs("mlp-d64-b2h4-t2k", 8, 512, 64, "bf16")
    B, H, T = 2, 4, 512
    m = mem.Memory(64, 256, 64, "bf16", B, H, chunk_gates=True)
    y_dev, st_dev = _run(m, inp, cg, B, H, 64)
    toks, _, state = gpu_inputs(inp, B, H)
    host = {n: inp[n].reshape(B, H, T, 64).contiguous().pin_memory() for n in ("k", "q", "v")}
    hg = {n: cg[n].reshape(B, H, -1).contiguous().pin_memory() for n in cg}
    y_host = torch.empty(B, H, T, 64, dtype=torch.bfloat16).pin_memory()
    staging = {n: torch.empty_like(toks[n]) for n in toks}
    staging.update({n: torch.empty(B, H, hg[n].shape[-1], device="cuda") for n in hg})
    staging["y"] = torch.empty_like(toks["k"])
    m.forward_host(host["k"], host["q"], host["v"], hg["alpha"], hg["eta"], hg["theta"], state, y_host, staging,
                   t_seg=128)
    torch.cuda.synchronize()
    m.sync_status()
    assert torch.equal(y_host, y_dev.cpu())
    assert all(torch.equal(state[n], st_dev[n]) for n in state)
