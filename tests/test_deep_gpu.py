"""GPU parity of the deep memory (L >= 2 SiLU layers, titans_mem_init_deep / titans_mem_forward_deep)
against the oracle's deep token loop, plus its invariants."""
import numpy as np
import pytest
import torch

import oracle
from parity import TOL, compare
from titans_long_term_b200 import mem, synth

pytestmark = pytest.mark.gpu


def _inputs(name, units, T, mode, layers, recipe=None):
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w, units=range(units), T=T, dtype=mode, recipe=recipe)
    st = synth.make_deep_state(w, layers, units=range(units))
    return w, inp, st


def _gpu(w, inp, st, B, H, chunk, mode, layers, attn=None, cuda_cores=False, chunk_gates=None):
    m = mem.Memory(w.d, w.h, chunk, mode, B, H, layers=layers, cuda_cores=cuda_cores, chunk_gates=chunk_gates is not None)
    if layers > 2:  # a 2-layer handle reports the path titans_mem_forward takes
        tc = mode == "bf16" and not cuda_cores
        assert m.path(chunk) == (mem.PATH_TC_DEEP if tc else mem.PATH_DEEP_CUDA_CORES)
    T = inp["k"].shape[1]
    dev = lambda x, *s: x.reshape(B, H, *s).cuda().contiguous()
    toks = {n: dev(inp[n], T, w.d) for n in ("k", "q", "v")}
    gates = {n: dev(inp[n], T) for n in ("alpha", "eta", "theta")}
    if chunk_gates is not None:
        gates = {n: dev(chunk_gates[n], chunk_gates[n].shape[-1]) for n in chunk_gates}
    state = {n: dev(st[n], st[n].shape[-1]) for n in ("W", "S")}
    a = None if attn is None else dev(attn, T, w.d)
    y = m.forward_deep(toks["k"], toks["q"], toks["v"], gates["alpha"], gates["eta"], gates["theta"], state,
                       chunk=chunk, attn=a)
    m.sync_status()
    U = B * H
    return (y.reshape(U, T, w.d).float().cpu().numpy(),
            {n: t.reshape(U, -1).cpu().numpy() for n, t in state.items()})


def _oracle(inp, st, chunk, layers, attn=None):
    y, out = oracle.forward_deep(*(inp[n] for n in ("k", "q", "v", "alpha", "eta", "theta")),
                                 {"W": st["W"], "S": st["S"]}, chunk, layers)
    if attn is not None:
        y = oracle.mag_gate(attn.float().numpy(), y)
    return y, out


@pytest.mark.parametrize("name,B,H,T,chunk,mode,layers,recipe", [
    ("mlp-d64-b2h4-t2k", 2, 2, 150, 64, "fp32", 3, None),
    ("mlp-d64-b2h4-t2k", 2, 2, 150, 64, "bf16", 3, None),
    ("mlp-d64-b2h4-t2k", 1, 3, 100, 32, "fp32", 4, None),
    ("mlp-d64-b2h4-t2k", 2, 2, 40, 16, "bf16", 4, None),
    ("mlp-d64-b2h4-t2k", 2, 2, 64, 64, "fp32", 3, "stated"),
    ("mlp-d128-b4h8-t16k", 1, 2, 140, 128, "bf16", 3, None),
    # the tensor-core kernel: several chunks, ragged last chunk, up to 8 layers, both widths
    ("mlp-d64-b2h4-t2k", 2, 2, 300, 64, "bf16", 4, None),
    ("mlp-d64-b2h4-t2k", 1, 3, 257, 128, "bf16", 5, None),
    ("mlp-d64-b2h4-t2k", 1, 2, 70, 16, "bf16", 8, None),
    ("mlp-d64-b2h4-t2k", 2, 1, 5, 1, "bf16", 3, None),
    ("mlp-d128-b4h8-t16k", 1, 2, 300, 128, "bf16", 4, None),
    ("mlp-d64-b2h4-t2k", 1, 2, 128, 64, "bf16", 4, "stated"),
])
def test_deep_memory_matches_the_oracle(name, B, H, T, chunk, mode, layers, recipe):
    w, inp, st = _inputs(name, B * H, T, mode, layers, recipe)
    gy, gst = _gpu(w, inp, st, B, H, chunk, mode, layers)
    ry, rst = _oracle(inp, st, chunk, layers)
    compare(gy, gst, ry, rst, TOL[mode], what=f"deep L={layers} {name} {mode} T={T} chunk={chunk}")


def test_deep_at_two_layers_is_the_two_layer_memory():
    """L = 2 through the deep entry point, against the 2-layer oracle on the same W1, W2."""
    w, inp, st = _inputs("mlp-d64-b2h4-t2k", 4, 130, "fp32", 2)
    gy, gst = _gpu(w, inp, st, 2, 2, 32, "fp32", 2)
    ry, rst = oracle.forward(*(inp[n] for n in ("k", "q", "v", "alpha", "eta", "theta")),
                             {n: inp[n] for n in ("W1", "W2", "S1", "S2")}, 32)
    packed = {"W": oracle.pack_deep([rst["W1"], rst["W2"]]), "S": oracle.pack_deep([rst["S1"], rst["S2"]])}
    compare(gy, gst, ry, packed, TOL["fp32"], what="deep L=2")


def test_deep_gated_output():
    w, inp, st = _inputs("mlp-d64-b2h4-t2k", 4, 96, "bf16", 3)
    attn = synth.make_attn(w, units=range(4), T=96, dtype="bf16")
    gy, gst = _gpu(w, inp, st, 2, 2, 64, "bf16", 3, attn=attn)
    ry, rst = _oracle(inp, st, 64, 3, attn=attn)
    compare(gy, gst, ry, rst, TOL["bf16"], what="deep gated")


def test_deep_reset_is_a_fixed_point():
    """alpha = 1, eta = 0, theta = 0 on the last token of a chunk: W = S = 0 is a fixed point of any
    deep SiLU memory, so every later retrieval and the final state are exactly zero."""
    w, inp, st = _inputs("mlp-d64-b2h4-t2k", 4, 128, "fp32", 4)
    inp["alpha"][:, 63] = 1.0
    inp["eta"][:, 63] = 0.0
    inp["theta"][:, 63] = 0.0
    gy, gst = _gpu(w, inp, st, 2, 2, 64, "fp32", 4)
    assert not gy[:, 64:].any() and not gst["W"].any() and not gst["S"].any()
    assert np.abs(gy[:, :64]).max() > 0


def test_deep_handle_runs_only_the_deep_forward():
    m = mem.Memory(64, 256, 64, "fp32", 1, 1, layers=3)
    assert m.path(64, step=True) == -1
    with pytest.raises(mem.TitansError):
        z = torch.zeros(1, 1, 8, 64, device="cuda")
        g = torch.zeros(1, 1, 8, device="cuda")
        m.forward(z, z, z, g, g, g, {"W1": torch.zeros(1, 1, 256, 64, device="cuda"),
                                     "W2": torch.zeros(1, 1, 64, 256, device="cuda"),
                                     "S1": torch.zeros(1, 1, 256, 64, device="cuda"),
                                     "S2": torch.zeros(1, 1, 64, 256, device="cuda")})


def test_deep_tensor_core_kernel_against_the_cuda_core_kernel():
    """Same bf16 inputs through the tensor-core deep kernel and the fp32 CUDA-core one: both within
    the bf16 bar of the oracle, and of each other."""
    w, inp, st = _inputs("mlp-d64-b2h4-t2k", 4, 256, "bf16", 4)
    ty, tst = _gpu(w, inp, st, 2, 2, 64, "bf16", 4)
    cy, cst = _gpu(w, inp, st, 2, 2, 64, "bf16", 4, cuda_cores=True)
    ry, rst = _oracle(inp, st, 64, 4)
    compare(ty, tst, ry, rst, TOL["bf16"], what="deep tensor cores")
    compare(cy, cst, ry, rst, TOL["bf16"], what="deep CUDA cores")


def test_deep_tensor_core_kernel_with_chunk_gates_and_the_gated_output():
    w, inp, st = _inputs("mlp-d64-b2h4-t2k", 4, 192, "bf16", 3)
    cg = {n: inp[n][:, ::64].contiguous() for n in ("alpha", "eta", "theta")}
    attn = synth.make_attn(w, units=range(4), T=192, dtype="bf16")
    gy, gst = _gpu(w, inp, st, 2, 2, 64, "bf16", 3, attn=attn, chunk_gates=cg)
    rep = {n: oracle.expand_chunk_gates(cg[n].numpy(), 192, 64) for n in cg}
    y, out = oracle.forward_deep(inp["k"], inp["q"], inp["v"], rep["alpha"], rep["eta"], rep["theta"],
                                 {"W": st["W"], "S": st["S"]}, 64, 3)
    compare(gy, gst, oracle.mag_gate(attn.float().numpy(), y), out, TOL["bf16"], what="deep chunk gates, gated")


def test_deep_tensor_core_kernel_is_split_invariant():
    """forward(T1) then forward(T2) equals forward(T1 + T2) bit for bit when T1 is a multiple of the chunk."""
    w, inp, st = _inputs("mlp-d64-b2h4-t2k", 2, 256, "bf16", 4)
    full_y, full_st = _gpu(w, inp, st, 1, 2, 64, "bf16", 4)
    first = {n: inp[n][:, :128] for n in inp if n[0] not in "WS"}
    y1, st1 = _gpu(w, first, st, 1, 2, 64, "bf16", 4)
    second = {n: inp[n][:, 128:] for n in inp if n[0] not in "WS"}
    y2, st2 = _gpu(w, second, {n: torch.from_numpy(x) for n, x in st1.items()}, 1, 2, 64, "bf16", 4)
    assert np.array_equal(np.concatenate([y1, y2], axis=1), full_y)
    assert all(np.array_equal(st2[n], full_st[n]) for n in full_st)
