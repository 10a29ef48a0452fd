"""Shared helpers of the parity tests: run the CUDA library and the oracle on the same
seeded inputs and compare them.

Tolerance metric (per unit and per tensor y, W1, W2, S1, S2):
    err = max_i |x_i - r_i| / max_i |r_i|
with the bars 2e-2 for the bf16 tensor-core path and 1e-4 for the fp32 CUDA-core mode.
An all-zero reference requires an exact zero result.
"""
from __future__ import annotations

from typing import Dict, Optional, Sequence

import numpy as np
import torch

import oracle
from titans_long_term_b200 import synth

TOL = {"bf16": 2e-2, "fp32": 1e-4}


def gpu_inputs(inp: Dict[str, torch.Tensor], B: int, H: int, device="cuda"):
    T = inp["k"].shape[1]
    d = inp["k"].shape[2]
    toks = {n: inp[n].reshape(B, H, T, d).to(device).contiguous() for n in ("k", "q", "v")}
    gates = {n: inp[n].reshape(B, H, T).to(device).contiguous() for n in ("alpha", "eta", "theta")}
    state = {n: inp[n].reshape(B, H, *inp[n].shape[1:]).to(device).contiguous() for n in inp if n[0] in "WS"}
    return toks, gates, state


def run_gpu(mem, inp, B, H, chunk, stream=None):
    toks, gates, state = gpu_inputs(inp, B, H)
    y = mem.forward(toks["k"], toks["q"], toks["v"], gates["alpha"], gates["eta"], gates["theta"], state,
                    chunk=chunk, stream=stream)
    mem.sync_status(stream)
    U = B * H
    out = {n: t.reshape(U, *t.shape[2:]).float().cpu().numpy() for n, t in state.items()}
    return y.reshape(U, *y.shape[2:]).float().cpu().numpy(), out


def run_oracle(inp, chunk, units: Optional[Sequence[int]] = None, closed_form: bool = False):
    sel = slice(None) if units is None else list(units)
    args = [inp[n][sel] for n in ("k", "q", "v", "alpha", "eta", "theta")]
    st = {n: inp[n][sel] for n in inp if n[0] in "WS"}
    f = oracle.forward_closed_form if closed_form else oracle.forward
    return f(*args, st, chunk)


def rel_err(x: np.ndarray, r: np.ndarray) -> np.ndarray:
    """Per-unit max |x - r| / max |r| over all axes but the first."""
    x = np.asarray(x, np.float64).reshape(x.shape[0], -1)
    r = np.asarray(r, np.float64).reshape(r.shape[0], -1)
    num = np.abs(x - r).max(axis=1)
    den = np.abs(r).max(axis=1)
    out = np.where(den > 0, num / np.where(den > 0, den, 1.0), np.where(num > 0, np.inf, 0.0))
    return out


def compare(gy, gst, ry, rst, tol, units: Optional[Sequence[int]] = None, what=""):
    """Assert parity; returns {tensor: worst unit error}."""
    sel = slice(None) if units is None else list(units)
    worst = {}
    pairs = [("y", gy[sel], ry)] + [(n, gst[n][sel], rst[n]) for n in rst]
    for name, x, r in pairs:
        assert np.isfinite(x).all(), f"{what}: non-finite values in {name}"
        e = rel_err(x, r)
        worst[name] = float(e.max())
        assert e.max() <= tol, f"{what}: {name} max rel err {e.max():.3e} > {tol:.0e} (unit {int(e.argmax())})"
    return worst


def workload_inputs(name: str, T: Optional[int] = None, units=None, dtype: Optional[str] = None):
    w = synth.WORKLOADS[name]
    return w, synth.make_inputs(w, units=units, T=T, dtype=dtype)


def step_sequence(m, inp, B, H, steps):
    """`steps` titans_mem_step calls over the first tokens of `inp`; returns y [U, steps, d] and the state."""
    toks, gates, state = gpu_inputs(inp, B, H)
    ys = []
    for t in range(steps):
        sl = lambda x: x[:, :, t].contiguous()
        ys.append(m.step(sl(toks["k"]), sl(toks["q"]), sl(toks["v"]), sl(gates["alpha"]), sl(gates["eta"]),
                         sl(gates["theta"]), state))
    m.sync_status()
    U = B * H
    y = torch.stack(ys, dim=2).reshape(U, steps, -1).float().cpu().numpy()
    return y, {n: t.reshape(U, *t.shape[2:]).float().cpu().numpy() for n, t in state.items()}
