"""Seeded synthetic inputs for the neural long-term memory.

This module only draws random numbers and lays them out. It holds none of the
memory's arithmetic: the oracle (test infrastructure) and the CUDA path both
consume what it produces, and neither imports the other.

Workloads (named by what they are):

=============================  ======  ===========  ======  =========  =====
name                           memory  d -> h -> d  B x H   T          chunk
=============================  ======  ===========  ======  =========  =====
linear-d64                     linear  64 x 64      1 x 1   256        16
mlp-d64-b2h4-t2k               MLP     64-256-64    2 x 4   2048       64
mlp-d64-b8h16-t4k (760M-class) MLP     64-256-64    8 x 16  4096       64
mlp-d64-b1h16-t1m (long)       MLP     64-256-64    1 x 16  1,048,576  64
mlp-d128-b4h8-t16k + decode    MLP     128-512-128  4 x 8   16384      128
=============================  ======  ===========  ======  =========  =====

Two input recipes:

* "stated" -- the workloads' stated distributions: per token k, q, v ~ N(0, I_d)
  drawn independently, k and q l2-normalised; gates i.i.d. alpha ~ U(0, 0.05),
  eta ~ U(0.8, 0.99), theta ~ U(0, 0.1). The linear memory runs on it by default.
  The 2-layer MLP memories diverge on it within a few chunks (the oracle too: at
  chunk 64 the weights grow about 100x per chunk from the third chunk on, and
  past about 16 tokens at chunk 1), so the MLP parity tests use it over one or
  two chunks.
* "projected" -- the pages' construction of the token streams (Titans: Learning
  to Memorize at Test Time, walk-through sec. 3.1 "Objective" and "Retrieving a
  Memory": k_t = x_t W_K, v_t = x_t W_V, q_t = x_t W_Q; sec. 4.4 "Architectural
  Details": q and k are l2-normalised), the default of the MLP workloads, which
  stays finite over any length:
  - per unit, fixed projections W_K, W_V, W_Q [d, d] with N(0, 1/d) entries;
  - per token, x_t ~ N(0, I_d); k = l2n(x W_K), q = l2n(x W_Q), v = x W_V, so
    each element of v (and of k, q before the norm) is marginally N(0, 1);
  - gates eta ~ U(0.8, 0.99), alpha ~ U(0, 0.002), theta ~ U(0, 0.003) (wider
    ranges make the MLP's inner loop diverge or forget all content within a few
    chunks).

Both cast k, q, v to the input dtype (bf16 round-to-nearest-even by torch) last.

State: MLP W1 ~ N(0, 1/d) (fan_in d), W2 ~ N(0, 1/h) (fan_in h), S = 0;
linear memory W = 0, S = 0.

Long-stream recall structure: one extra key/value pair per unit (projected:
k* = l2n(x* W_K), v* = x* W_V; stated: k* = l2n(N(0, I)), v* ~ N(0, I)); at
every token t with t % 4096 == 4095, k_t = q_t = k*, v_t = v*.

Every (unit, 4096-token block) draws from its own counter-seeded torch CPU
generator, so any unit and any token range can be produced on its own and the
result does not depend on which other units or ranges were asked for.
"""
from __future__ import annotations

import dataclasses
import functools
from typing import Dict, Optional, Sequence

import numpy as np
import torch

BLOCK = 4096  # tokens per independently seeded block
RECALL_EVERY = 4096


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    d: int
    h: int  # 0 => linear memory
    B: int
    H: int
    T: int
    chunk: int
    dtype: str  # "bf16" or "fp32": dtype of k, q, v and y
    seed: int
    recall: bool = False
    decode_B: int = 0
    decode_steps: int = 0
    recipe: str = "projected"  # default input recipe: "stated" or "projected"

    @property
    def units(self) -> int:
        return self.B * self.H

    @property
    def linear(self) -> bool:
        return self.h == 0


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("linear-d64", 64, 0, 1, 1, 256, 16, "fp32", 20250101, recipe="stated"),
        Workload("mlp-d64-b2h4-t2k", 64, 256, 2, 4, 2048, 64, "bf16", 20250102),
        Workload("mlp-d64-b8h16-t4k", 64, 256, 8, 16, 4096, 64, "bf16", 20250103),
        Workload("mlp-d64-b1h16-t1m", 64, 256, 1, 16, 1 << 20, 64, "bf16", 20250104, recall=True),
        Workload("mlp-d128-b4h8-t16k", 128, 512, 4, 8, 16384, 128, "bf16", 20250105,
                 decode_B=256, decode_steps=1024),
    ]
}
# Index order of the five workloads (the small linear case first).
WORKLOAD_ORDER = list(WORKLOADS)


def _mix(*parts: int) -> int:
    """Counter-based seed: a fixed polynomial mix of integers, 63-bit."""
    x = 0x9E3779B97F4A7C15
    for p in parts:
        x = (x * 6364136223846793005 + (int(p) & 0xFFFFFFFFFFFFFFFF) + 1442695040888963407) & 0xFFFFFFFFFFFFFFFF
    return x & 0x7FFFFFFFFFFFFFFF


def _gen(*parts: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(_mix(*parts))
    return g


def _l2n(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True)


RECIPES = ("stated", "projected")
STATED_GATES = (0.05, 0.8, 0.99, 0.1)
PROJECTED_MLP_GATES = (0.002, 0.8, 0.99, 0.003)


def _recipe(w: Workload, recipe: Optional[str]) -> str:
    r = w.recipe if recipe is None else recipe
    if r not in RECIPES:
        raise ValueError(f"unknown input recipe {r!r}: expected one of {RECIPES}")
    return r


def _gate_ranges(w: Workload, recipe: Optional[str] = None):
    """(alpha_max, eta_lo, eta_hi, theta_max) of the uniform gate distributions."""
    if w.linear or _recipe(w, recipe) == "stated":
        return STATED_GATES
    return PROJECTED_MLP_GATES


def describe(w: Workload, recipe: Optional[str] = None) -> Dict[str, str]:
    """The input recipe in words (for benchmark records)."""
    r = _recipe(w, recipe)
    amax, elo, ehi, tmax = _gate_ranges(w, r)
    if r == "stated":
        toks = "k, q, v ~ N(0, I) i.i.d. per token; k, q l2-normalised"
    else:
        toks = "x ~ N(0, I) per token; k = l2n(x W_K), q = l2n(x W_Q), v = x W_V; W_K, W_V, W_Q ~ N(0, 1/d) per unit"
    out = {"recipe": r, "tokens": toks + f"; cast to {w.dtype}", "alpha": f"U(0, {amax:g})",
           "eta": f"U({elo:g}, {ehi:g})", "theta": f"U(0, {tmax:g})",
           "state": "W = S = 0" if w.linear else "W1 ~ N(0, 1/d), W2 ~ N(0, 1/h), S = 0"}
    if w.recall:
        out["recall"] = f"k = q = k*, v = v* at every t % {RECALL_EVERY} == {RECALL_EVERY - 1}"
    return out


@functools.lru_cache(maxsize=4096)
def _projections(w: Workload, unit: int):
    g = _gen(w.seed, unit, 0x960)
    s = 1.0 / np.sqrt(w.d)
    return tuple(torch.randn(w.d, w.d, generator=g) * s for _ in range(3))  # W_K, W_V, W_Q


def _recall_pair(w: Workload, unit: int, recipe: str):
    if recipe == "stated":
        g = _gen(w.seed, unit, 0x7EC, 0x57A7ED)
        return _l2n(torch.randn(1, w.d, generator=g))[0], torch.randn(w.d, generator=g)
    WK, WV, _ = _projections(w, unit)
    g = _gen(w.seed, unit, 0x7EC)
    x = torch.randn(1, w.d, generator=g)
    return _l2n(x @ WK)[0], (x @ WV)[0]


def _block_gen(w: Workload, unit: int, blk: int, recipe: str) -> torch.Generator:
    # The stated recipe draws from generators of its own, so its streams share nothing with the
    # projected ones.
    return _gen(w.seed, unit, blk, 0x57A7ED) if recipe == "stated" else _gen(w.seed, unit, blk)


def _draw(w: Workload, g: torch.Generator, n: int, unit: int, recipe: str):
    if recipe == "stated":
        k = _l2n(torch.randn(n, w.d, generator=g))
        q = _l2n(torch.randn(n, w.d, generator=g))
        v = torch.randn(n, w.d, generator=g)
    else:
        WK, WV, WQ = _projections(w, unit)
        x = torch.randn(n, w.d, generator=g)
        k, q, v = _l2n(x @ WK), _l2n(x @ WQ), x @ WV
    amax, elo, ehi, tmax = _gate_ranges(w, recipe)
    a = torch.rand(n, generator=g) * amax
    e = elo + torch.rand(n, generator=g) * (ehi - elo)
    t = torch.rand(n, generator=g) * tmax
    return k, q, v, a, e, t


def unit_tokens(w: Workload, unit: int, t0: int = 0, t1: Optional[int] = None,
                recipe: Optional[str] = None) -> Dict[str, torch.Tensor]:
    """fp32 token streams of one unit for tokens [t0, t1): k, q, v [n, d]; alpha, eta, theta [n].

    k and q are l2-normalised; nothing is rounded to the input dtype yet.
    """
    recipe = _recipe(w, recipe)
    t1 = w.T if t1 is None else t1
    assert 0 <= t0 <= t1
    ks, qs, vs, al, et, th = [], [], [], [], [], []
    for blk in range(t0 // BLOCK, (t1 + BLOCK - 1) // BLOCK):
        k, q, v, a, e, t = _draw(w, _block_gen(w, unit, blk, recipe), BLOCK, unit, recipe)
        lo = max(t0 - blk * BLOCK, 0)
        hi = min(t1 - blk * BLOCK, BLOCK)
        for lst, x in ((ks, k), (qs, q), (vs, v), (al, a), (et, e), (th, t)):
            lst.append(x[lo:hi])
    out = {n: torch.cat(l) if l else torch.zeros((0, w.d) if n in "kqv" else (0,))
           for n, l in zip(("k", "q", "v", "alpha", "eta", "theta"), (ks, qs, vs, al, et, th))}
    if w.recall and t1 > t0:
        ks_, vs_ = _recall_pair(w, unit, recipe)
        t = torch.arange(t0, t1)
        hit = (t % RECALL_EVERY) == (RECALL_EVERY - 1)
        idx = hit.nonzero().flatten()
        out["k"][idx] = ks_
        out["q"][idx] = ks_
        out["v"][idx] = vs_
    return out


def recall_positions(w: Workload, t0: int = 0, t1: Optional[int] = None) -> np.ndarray:
    t1 = w.T if t1 is None else t1
    t = np.arange(t0, t1)
    return t[(t % RECALL_EVERY) == (RECALL_EVERY - 1)]


def unit_state(w: Workload, unit: int) -> Dict[str, torch.Tensor]:
    """Initial fp32 memory state of one unit.

    MLP: W1 [h, d], W2 [d, h], S1, S2 zeros.  Linear: W1 = W [d, d] zeros, S1 zeros.
    """
    if w.linear:
        z = torch.zeros(w.d, w.d)
        return {"W1": z.clone(), "S1": z.clone()}
    g = _gen(w.seed, unit, 0x57A7E)
    W1 = torch.randn(w.h, w.d, generator=g) / np.sqrt(w.d)
    W2 = torch.randn(w.d, w.h, generator=g) / np.sqrt(w.h)
    return {"W1": W1, "W2": W2, "S1": torch.zeros_like(W1), "S2": torch.zeros_like(W2)}


def _cast(x: torch.Tensor, dtype: str) -> torch.Tensor:
    return x.to(torch.bfloat16) if dtype == "bf16" else x.to(torch.float32)


def make_inputs(w: Workload, units: Optional[Sequence[int]] = None, T: Optional[int] = None,
                dtype: Optional[str] = None, t0: int = 0, recipe: Optional[str] = None) -> Dict[str, torch.Tensor]:
    """Stacked CPU tensors for a list of units: k, q, v [U, T, d] in the input dtype;
    alpha, eta, theta [U, T] fp32; W1, W2, S1, S2 fp32 (W2/S2 absent for linear).

    `units` defaults to all B*H units in (b, h) row-major order, so [U, ...] reshapes
    to [B, H, ...]. `T` truncates the stream (tokens t0 .. t0+T). `recipe` overrides the
    workload's input recipe ("stated" or "projected")."""
    units = list(range(w.units)) if units is None else list(units)
    T = w.T - t0 if T is None else T
    dtype = w.dtype if dtype is None else dtype
    cols = {n: [] for n in ("k", "q", "v", "alpha", "eta", "theta")}
    for u in units:  # cast unit by unit: only one unit's fp32 stream is alive at a time
        t = unit_tokens(w, u, t0, t0 + T, recipe)
        for n in cols:
            cols[n].append(_cast(t[n], dtype) if n in ("k", "q", "v") else t[n])
        del t
    sts = [unit_state(w, u) for u in units]
    out = {n: torch.stack(cols.pop(n)) for n in ("k", "q", "v")}
    for n in ("alpha", "eta", "theta"):
        out[n] = torch.stack(cols.pop(n)).contiguous()
    for n in sts[0]:
        out[n] = torch.stack([s[n] for s in sts]).contiguous()
    return out


def decode_step_inputs(w: Workload, step: int, dtype: Optional[str] = None,
                       recipe: Optional[str] = None) -> Dict[str, torch.Tensor]:
    """Per-step decode inputs for decode_B x H units: k, q, v [decode_B*H, d]; gates [decode_B*H].

    One generator per step draws the tokens and the gates for every decode unit. Projected
    recipe: decode unit u projects its x with the projections of the prefill unit whose state
    it starts from; stated recipe: k, q, v drawn i.i.d."""
    dtype = w.dtype if dtype is None else dtype
    recipe = _recipe(w, recipe)
    n = w.decode_B * w.H
    if recipe == "stated":
        g = _gen(w.seed + 1000, step, 0x57A7ED)
        k, q, v, a, e, t = _draw(w, g, n, 0, recipe)
        return {"k": _cast(k, dtype), "q": _cast(q, dtype), "v": _cast(v, dtype), "alpha": a, "eta": e,
                "theta": t}
    src = decode_state_rows(w)
    g = _gen(w.seed + 1000, step)
    x = torch.randn(n, w.d, generator=g)
    amax, elo, ehi, tmax = _gate_ranges(w, recipe)
    a = torch.rand(n, generator=g) * amax
    e = elo + torch.rand(n, generator=g) * (ehi - elo)
    t = torch.rand(n, generator=g) * tmax
    k = torch.empty(n, w.d)
    q = torch.empty(n, w.d)
    v = torch.empty(n, w.d)
    for s_ in np.unique(src):
        rows = torch.as_tensor(np.nonzero(src == s_)[0])
        WK, WV, WQ = _projections(w, int(s_))
        xs = x[rows]
        k[rows] = _l2n(xs @ WK)
        q[rows] = _l2n(xs @ WQ)
        v[rows] = xs @ WV
    return {"k": _cast(k, dtype), "q": _cast(q, dtype), "v": _cast(v, dtype), "alpha": a, "eta": e, "theta": t}


def decode_state_rows(w: Workload) -> np.ndarray:
    """Decode unit u = b' * H + hh takes the prefill state of unit (b' // (decode_B // B)) * H + hh."""
    rep = w.decode_B // w.B
    u = np.arange(w.decode_B * w.H)
    return (u // w.H // rep) * w.H + (u % w.H)


def make_attn(w: Workload, units: Optional[Sequence[int]] = None, T: Optional[int] = None,
              dtype: Optional[str] = None, t0: int = 0) -> torch.Tensor:
    """The attention branch's output that a memory-as-a-gate layer multiplies by the gate: [U, T, d]
    in the input dtype, N(0, 1) elements, from a counter-seeded generator per (unit, 4096-token
    block), so any unit and token range can be drawn alone. It stands in for a sliding-window
    attention output, which the memory's caller computes."""
    units = list(range(w.units)) if units is None else list(units)
    T = w.T - t0 if T is None else T
    dtype = w.dtype if dtype is None else dtype
    rows = []
    for u in units:
        parts = []
        for blk in range(t0 // BLOCK, (t0 + T + BLOCK - 1) // BLOCK):
            x = torch.randn(BLOCK, w.d, generator=_gen(w.seed, u, blk, 0xA77))
            lo = max(t0 - blk * BLOCK, 0)
            hi = min(t0 + T - blk * BLOCK, BLOCK)
            parts.append(x[lo:hi])
        rows.append(_cast(torch.cat(parts) if parts else torch.zeros(0, w.d), dtype))
    return torch.stack(rows)


def deep_shapes(d: int, h: int, layers: int):
    """[out, in] of every layer of a deep memory: W_1 [h, d], W_2 .. W_{L-1} [h, h], W_L [d, h]."""
    return [(h, d)] + [(h, h)] * (layers - 2) + [(d, h)]


def make_deep_state(w: Workload, layers: int, units: Optional[Sequence[int]] = None) -> Dict[str, torch.Tensor]:
    """Initial state of a deep memory for a list of units: W [U, P] with each layer ~ N(0, 1/fan_in),
    packed layer after layer (row-major [out][in] each); S = 0. At 2 layers W_1, W_2 are the
    2-layer memory's initial weights of the same units."""
    units = list(range(w.units)) if units is None else list(units)
    rows = []
    for u in units:
        st = unit_state(w, u)
        mats = [st["W1"]]
        g = _gen(w.seed, u, 0xDEE9)
        for (o, i) in deep_shapes(w.d, w.h, layers)[1:-1]:
            mats.append(torch.randn(o, i, generator=g) / np.sqrt(i))
        mats.append(st["W2"])
        rows.append(torch.cat([m.reshape(-1) for m in mats]))
    W = torch.stack(rows).contiguous()
    return {"W": W, "S": torch.zeros_like(W)}
