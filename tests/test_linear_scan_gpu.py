"""GPU parity of the linear memory's cross-chunk scan (TITANS_FLAG_CHUNK_SCAN) against the oracle's
token loop: segments of chunks compose their affine maps in parallel, a scan over the segments gives
their start states, and the segments then run their chunks in parallel."""
import time

import numpy as np
import pytest
import torch

import oracle
from parity import TOL, compare, gpu_inputs
from titans_long_term_b200 import mem, synth

pytestmark = pytest.mark.gpu


def _linear(d, B, H, T, chunk, mode, seed=7):
    """Linear memory inputs at the stated distributions (the linear memory stays bounded on them)."""
    w = synth.Workload(f"linear-d{d}-scan", d, 0, B, H, T, chunk, mode, 20250101 + seed, recipe="stated")
    return w, synth.make_inputs(w)


def _run(m, inp, B, H, chunk, attn=None, gates=None):
    toks, g, state = gpu_inputs(inp, B, H)
    if gates is not None:
        g = {n: t.reshape(B, H, -1).cuda().contiguous() for n, t in gates.items()}
    if attn is None:
        y = m.forward(toks["k"], toks["q"], toks["v"], g["alpha"], g["eta"], g["theta"], state, chunk=chunk)
    else:
        a = attn.reshape(*toks["k"].shape).cuda().contiguous()
        y = m.forward_gated(toks["k"], toks["q"], toks["v"], g["alpha"], g["eta"], g["theta"], a, state, chunk=chunk)
    m.sync_status()
    U = B * H
    return y.reshape(U, -1, m.d).float().cpu().numpy(), {n: t.reshape(U, m.d, m.d).cpu().numpy() for n, t in state.items()}


@pytest.mark.parametrize("d,B,H,T,chunk,mode", [
    (64, 1, 1, 256, 16, "fp32"),     # the linear workload's shape: 16 chunks, one per segment
    (64, 1, 1, 16384, 16, "fp32"),   # a long single stream: 1024 chunks over ~148 segments
    (64, 1, 2, 1000, 16, "fp32"),    # ragged last chunk and segment
    (64, 2, 1, 8192, 32, "bf16"),    # bf16 token streams
    (128, 1, 1, 2048, 32, "fp32"),   # the wide width
])
def test_linear_scan_matches_the_token_loop(d, B, H, T, chunk, mode):
    w, inp = _linear(d, B, H, T, chunk, mode)
    m = mem.Memory(d, 0, chunk, mode, B, H, chunk_scan=True)
    assert m.path(chunk) == mem.PATH_LINEAR_SCAN
    gy, gst = _run(m, inp, B, H, chunk)
    ry, rst = oracle.forward(*(inp[n] for n in ("k", "q", "v", "alpha", "eta", "theta")),
                             {n: inp[n] for n in ("W1", "S1")}, chunk)
    worst = compare(gy, gst, ry, rst, TOL[mode], what=f"linear scan d={d} T={T} {mode}")
    print(f"linear scan d={d} T={T} chunk={chunk} {mode}:", {k: f"{v:.2e}" for k, v in worst.items()})


def test_linear_scan_with_chunk_gates_and_the_gated_output():
    d, B, H, T, chunk = 64, 1, 2, 512, 16
    w, inp = _linear(d, B, H, T, chunk, "fp32", seed=9)
    cg = {n: inp[n][:, ::chunk].contiguous() for n in ("alpha", "eta", "theta")}
    attn = synth.make_attn(w, T=T, dtype="fp32")
    m = mem.Memory(d, 0, chunk, "fp32", B, H, chunk_scan=True, chunk_gates=True)
    gy, gst = _run(m, inp, B, H, chunk, attn=attn, gates=cg)
    rep = {n: oracle.expand_chunk_gates(cg[n].numpy(), T, chunk) for n in cg}
    ry, rst = oracle.forward_gated(inp["k"], inp["q"], inp["v"], rep["alpha"], rep["eta"], rep["theta"],
                                   {n: inp[n] for n in ("W1", "S1")}, chunk, attn)
    compare(gy, gst, ry, rst, TOL["fp32"], what="linear scan, chunk gates, gated")


def test_linear_scan_is_faster_than_the_chunk_loop_on_a_long_stream():
    """One unit, 65,536 tokens (4096 chunks of 16): the scan spreads the stream over the SMs."""
    d, T, chunk = 64, 65536, 16
    w, inp = _linear(d, 1, 1, T, chunk, "fp32", seed=11)
    times = {}
    for scan in (False, True):
        m = mem.Memory(d, 0, chunk, "fp32", 1, 1, chunk_scan=scan)
        toks, g, state = gpu_inputs(inp, 1, 1)
        args = (toks["k"], toks["q"], toks["v"], g["alpha"], g["eta"], g["theta"])
        st = {n: t.clone() for n, t in state.items()}
        m.forward(*args, st)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for _ in range(3):
            st = {n: t.clone() for n, t in state.items()}
            m.forward(*args, st)
        torch.cuda.synchronize()
        times[scan] = (time.perf_counter() - t0) / 3
    print(f"linear memory, 1 unit, T={T}: chunk loop {1e3 * times[False]:.2f} ms, scan {1e3 * times[True]:.2f} ms")
    assert times[True] < times[False]
