"""GPU parity of the memory-as-a-gate output against the oracle: o_t = attn_t * sigmoid(M(q_t)),
fused into every kernel's output store (tcgen05 chunk kernel, CUDA-core chunk kernel, cluster
decode step), through titans_mem_forward_gated / titans_mem_step_gated."""
import numpy as np
import pytest
import torch

import oracle
from parity import TOL, compare, gpu_inputs
from titans_long_term_b200 import mem, synth

pytestmark = pytest.mark.gpu


def _gated_gpu(m, inp, attn, B, H, chunk):
    toks, gates, state = gpu_inputs(inp, B, H)
    T = inp["k"].shape[1]
    a = attn.reshape(B, H, T, -1).cuda().contiguous()
    o = m.forward_gated(toks["k"], toks["q"], toks["v"], gates["alpha"], gates["eta"], gates["theta"], a, state,
                        chunk=chunk)
    m.sync_status()
    U = B * H
    return (o.reshape(U, T, -1).float().cpu().numpy(),
            {n: t.reshape(U, *t.shape[2:]).float().cpu().numpy() for n, t in state.items()})


def _gated_oracle(inp, attn, chunk):
    args = [inp[n] for n in ("k", "q", "v", "alpha", "eta", "theta")]
    st = {n: inp[n] for n in inp if n[0] in "WS"}
    return oracle.forward_gated(*args, st, chunk, attn)


@pytest.mark.parametrize("name,B,H,T,chunk,mode,cuda_cores,recipe", [
    ("mlp-d64-b2h4-t2k", 2, 4, 200, 64, "bf16", False, None),       # tcgen05 kernel, ragged
    ("mlp-d64-b2h4-t2k", 2, 4, 128, 64, "bf16", False, "stated"),   # tcgen05 kernel, stated inputs
    ("mlp-d64-b2h4-t2k", 2, 4, 150, 64, "fp32", False, None),       # CUDA-core, fp32 reference mode
    ("mlp-d64-b2h4-t2k", 2, 4, 130, 32, "bf16", True, None),        # CUDA-core with bf16 inputs
    ("mlp-d128-b4h8-t16k", 2, 2, 300, 128, "bf16", False, None),    # the wide memory
    ("linear-d64", 1, 1, 256, 16, "fp32", False, None),             # linear memory
])
def test_gated_forward(name, B, H, T, chunk, mode, cuda_cores, recipe):
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w, units=range(B * H), T=T, dtype=mode, recipe=recipe)
    attn = synth.make_attn(w, units=range(B * H), T=T, dtype=mode)
    m = mem.Memory(w.d, w.h, chunk, mode, B, H, cuda_cores=cuda_cores)
    go, gst = _gated_gpu(m, inp, attn, B, H, chunk)
    ro, rst = _gated_oracle(inp, attn, chunk)
    compare(go, gst, ro, rst, TOL[mode], what=f"gated {name} {mode} path {m.path(chunk)}")


def test_gated_forward_leaves_the_state_as_the_plain_forward_does():
    """The gate only changes the output: the final state equals titans_mem_forward's bit for bit."""
    w = synth.WORKLOADS["mlp-d64-b2h4-t2k"]
    inp = synth.make_inputs(w, T=192)
    attn = synth.make_attn(w, T=192)
    m = mem.Memory(64, 256, 64, "bf16", 2, 4)
    _, gst = _gated_gpu(m, inp, attn, 2, 4, 64)
    toks, gates, state = gpu_inputs(inp, 2, 4)
    m.forward(toks["k"], toks["q"], toks["v"], gates["alpha"], gates["eta"], gates["theta"], state)
    m.sync_status()
    for n, t in state.items():
        assert np.array_equal(t.reshape(8, *t.shape[2:]).cpu().numpy(), gst[n]), n


@pytest.mark.parametrize("cuda_cores", [False, True])
def test_gated_output_after_reset_is_half_the_attention(cuda_cores):
    """alpha = 1, eta = 0, theta = 0 on the last token of a chunk puts the MLP memory at its W = 0 fixed
    point: every later retrieval is exactly 0, so the gate is exactly 1/2 and o = attn / 2 bit for bit
    (a halving is exact in bf16)."""
    w = synth.WORKLOADS["mlp-d64-b2h4-t2k"]
    inp = synth.make_inputs(w, T=256)
    inp["alpha"][:, 127] = 1.0
    inp["eta"][:, 127] = 0.0
    inp["theta"][:, 127] = 0.0
    attn = synth.make_attn(w, T=256)
    m = mem.Memory(64, 256, 64, "bf16", 2, 4, cuda_cores=cuda_cores)
    go, _ = _gated_gpu(m, inp, attn, 2, 4, 64)
    half = (attn.float() / 2).numpy()
    assert np.array_equal(go[:, 128:], half[:, 128:])


@pytest.mark.parametrize("name,mode", [("mlp-d64-b2h4-t2k", "bf16"), ("mlp-d128-b4h8-t16k", "fp32"),
                                       ("linear-d64", "fp32")])
def test_gated_decode_steps(name, mode):
    w = synth.WORKLOADS[name]
    units = min(w.units, 8)
    B, H = (units // 2, 2) if units > 1 else (1, 1)
    steps = 10
    inp = synth.make_inputs(w, units=range(units), T=steps, dtype=mode)
    attn = synth.make_attn(w, units=range(units), T=steps, dtype=mode)
    m = mem.Memory(w.d, w.h, 1, mode, B, H)
    toks, gates, state = gpu_inputs(inp, B, H)
    a = attn.reshape(B, H, steps, -1).cuda()
    outs = []
    for t in range(steps):
        sl = lambda x: x[:, :, t].contiguous()
        outs.append(m.step_gated(sl(toks["k"]), sl(toks["q"]), sl(toks["v"]), sl(gates["alpha"]),
                                 sl(gates["eta"]), sl(gates["theta"]), sl(a), state))
    m.sync_status()
    go = torch.stack(outs, dim=2).reshape(units, steps, -1).float().cpu().numpy()
    gst = {n: t.reshape(units, *t.shape[2:]).float().cpu().numpy() for n, t in state.items()}
    ro, rst = _gated_oracle(inp, attn, 1)
    compare(go, gst, ro, rst, TOL[mode], what=f"gated step {name} {mode}")


def test_gated_rejects_null_and_misaligned_attn():
    w = synth.WORKLOADS["mlp-d64-b2h4-t2k"]
    inp = synth.make_inputs(w, units=range(8), T=64)
    m = mem.Memory(64, 256, 64, "bf16", 2, 4)
    toks, gates, state = gpu_inputs(inp, 2, 4)
    L = mem.lib()
    args = [toks["k"].data_ptr(), toks["q"].data_ptr(), toks["v"].data_ptr(), gates["alpha"].data_ptr(),
            gates["eta"].data_ptr(), gates["theta"].data_ptr(), 64, 64, state["W1"].data_ptr(),
            state["W2"].data_ptr(), state["S1"].data_ptr(), state["S2"].data_ptr()]
    out = torch.empty_like(toks["k"])
    assert L.titans_mem_forward_gated(m._h, *args, None, out.data_ptr(), None) == mem.EINVAL
    assert L.titans_mem_forward_gated(m._h, *args, toks["v"].data_ptr() + 2, out.data_ptr(), None) == mem.EINVAL
    m.sync_status()
