"""Host-side logic on CPU: the seeded input generator and the benchmark's accounting.

The generator must give the same numbers for a token range whether it is drawn alone or as
part of a longer range, must be independent across units, and must follow the stated recipe
(l2-normalised keys and queries, gate ranges, the recall probes of the long stream, the
decode units' source rows). The benchmark's algorithmic FLOP and byte counts must equal the
figures derived in the design notes (18 d h FLOPs and 8 d + 12 bytes per head-token; 4 |W| fp32
state words per unit per call)."""
import os
import sys

import numpy as np
import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))

from titans_long_term_b200 import synth  # noqa: E402

W_SMALL = synth.WORKLOADS["mlp-d64-b2h4-t2k"]


def test_token_ranges_are_slices_of_the_full_stream():
    full = synth.unit_tokens(W_SMALL, 3, 0, 2048)
    part = synth.unit_tokens(W_SMALL, 3, 700, 1500)
    for n in full:
        assert torch.equal(full[n][700:1500], part[n])


def test_units_are_independent_and_deterministic():
    a = synth.unit_tokens(W_SMALL, 0, 0, 256)
    b = synth.unit_tokens(W_SMALL, 1, 0, 256)
    a2 = synth.unit_tokens(W_SMALL, 0, 0, 256)
    assert all(torch.equal(a[n], a2[n]) for n in a)
    assert not torch.equal(a["k"], b["k"])
    # make_inputs stacks the same per-unit streams in (b, h) order
    inp = synth.make_inputs(W_SMALL, units=[1, 0], T=256, dtype="fp32")
    assert torch.equal(inp["k"][0], b["k"]) and torch.equal(inp["k"][1], a["k"])


def test_keys_queries_normalised_and_gates_in_range():
    t = synth.unit_tokens(W_SMALL, 2, 0, 4096 if W_SMALL.T >= 4096 else W_SMALL.T)
    for n in ("k", "q"):
        norms = t[n].norm(dim=1)
        assert torch.allclose(norms, torch.ones_like(norms), atol=1e-5)
    amax, elo, ehi, tmax = synth._gate_ranges(W_SMALL)
    assert float(t["alpha"].min()) >= 0 and float(t["alpha"].max()) <= amax
    assert float(t["eta"].min()) >= elo and float(t["eta"].max()) <= ehi
    assert float(t["theta"].min()) >= 0 and float(t["theta"].max()) <= tmax
    # v is a linear image of the same x as k: not normalised, unit-scale elements
    assert 0.5 < float(t["v"].std()) < 2.0


def test_bf16_cast_happens_last():
    f32 = synth.make_inputs(W_SMALL, units=[0], T=128, dtype="fp32")
    b16 = synth.make_inputs(W_SMALL, units=[0], T=128, dtype="bf16")
    assert b16["k"].dtype == torch.bfloat16 and f32["k"].dtype == torch.float32
    assert torch.equal(f32["k"].to(torch.bfloat16), b16["k"])
    assert torch.equal(f32["alpha"], b16["alpha"])  # gates stay fp32


def test_long_stream_recall_probes():
    w = synth.WORKLOADS["mlp-d64-b1h16-t1m"]
    pos = synth.recall_positions(w, 0, 3 * synth.RECALL_EVERY)
    assert list(pos) == [synth.RECALL_EVERY - 1, 2 * synth.RECALL_EVERY - 1, 3 * synth.RECALL_EVERY - 1]
    t = synth.unit_tokens(w, 5, 0, 3 * synth.RECALL_EVERY)
    for p in pos:  # every probe repeats one key/value pair; the query asks for that key
        assert torch.equal(t["k"][p], t["k"][pos[0]]) and torch.equal(t["v"][p], t["v"][pos[0]])
        assert torch.equal(t["q"][p], t["k"][p])
    assert not torch.equal(t["k"][pos[0] - 1], t["k"][pos[0]])


def test_initial_state_recipe():
    st = synth.unit_state(W_SMALL, 0)
    assert st["W1"].shape == (W_SMALL.h, W_SMALL.d) and st["W2"].shape == (W_SMALL.d, W_SMALL.h)
    assert float(st["S1"].abs().max()) == 0 and float(st["S2"].abs().max()) == 0
    # W1 ~ N(0, 1/d), W2 ~ N(0, 1/h)
    assert abs(float(st["W1"].std()) - 1 / np.sqrt(W_SMALL.d)) < 0.1 / np.sqrt(W_SMALL.d)
    assert abs(float(st["W2"].std()) - 1 / np.sqrt(W_SMALL.h)) < 0.1 / np.sqrt(W_SMALL.h)
    lin = synth.unit_state(synth.WORKLOADS["linear-d64"], 0)
    assert set(lin) == {"W1", "S1"} and float(lin["W1"].abs().max()) == 0


def test_decode_units_and_step_inputs():
    w = synth.WORKLOADS["mlp-d128-b4h8-t16k"]
    src = synth.decode_state_rows(w)
    n = w.decode_B * w.H
    assert src.shape == (n,)
    rep = w.decode_B // w.B
    for u in (0, 7, 8, 63 * 8 + 5, n - 1):
        b, hh = divmod(u, w.H)
        assert src[u] == (b // rep) * w.H + hh
    d0 = synth.decode_step_inputs(w, 0, dtype="fp32")
    d0b = synth.decode_step_inputs(w, 0, dtype="fp32")
    d1 = synth.decode_step_inputs(w, 1, dtype="fp32")
    assert all(torch.equal(d0[k], d0b[k]) for k in d0)
    assert not torch.equal(d0["k"], d1["k"])
    assert d0["k"].shape == (n, w.d) and d0["alpha"].shape == (n,)
    norms = d0["k"].norm(dim=1)
    assert torch.allclose(norms, torch.ones_like(norms), atol=1e-5)


@pytest.fixture(scope="module")
def bench():
    import bench as b
    return b


def test_algorithmic_counts(bench):
    w = synth.WORKLOADS["mlp-d64-b8h16-t4k"]
    assert bench.flops_per_head_token(w) == 294912  # 18 d h
    assert bench.stream_bytes_per_head_token(w) == 8 * 64 + 12  # k, q, v, y bf16 + 3 fp32 gates
    assert bench.state_bytes_per_unit(w) == 512 * 1024  # W1, W2, S1, S2 fp32, read + written
    total = bench.stream_bytes_per_head_token(w) * w.units * w.T + bench.state_bytes_per_unit(w) * w.units
    assert total == 341835776  # the 342 MB per launch the roofline uses
    wide = synth.WORKLOADS["mlp-d128-b4h8-t16k"]
    assert bench.flops_per_head_token(wide) == 1179648
    assert bench.flops_per_head_token(synth.WORKLOADS["linear-d64"]) == 8 * 64 * 64


def test_kernel_hash_ignores_comments(bench, tmp_path, monkeypatch):
    src = os.path.join(os.path.dirname(HERE), "titans_long_term_b200", "csrc", "chunk_tc_mlp64.cu")
    text = open(src).read()
    d = tmp_path / "titans_long_term_b200" / "csrc"
    d.mkdir(parents=True)
    monkeypatch.setattr(bench, "HERE", str(tmp_path))
    (d / "chunk_tc_mlp64.cu").write_text(text)
    h0 = bench.kernel_sha()
    (d / "chunk_tc_mlp64.cu").write_text("// a new comment line\n\n" + text.replace("\n", "  // trailing\n", 1))
    assert bench.kernel_sha() == h0
    (d / "chunk_tc_mlp64.cu").write_text(text.replace("kThreads = 384", "kThreads = 385"))
    assert bench.kernel_sha() != h0


def test_stated_recipe_draws_independent_tokens_with_the_stated_gate_ranges():
    """The stated recipe: k, q, v ~ N(0, I) drawn independently (k, q l2-normalised) and gates
    alpha ~ U(0, 0.05), eta ~ U(0.8, 0.99), theta ~ U(0, 0.1). In the projected recipe v is a
    linear image of the same x as k, so least squares recovers v from k almost exactly; in the
    stated recipe it explains next to nothing."""
    n = 4096
    st = synth.unit_tokens(W_SMALL, 1, 0, n, recipe="stated")
    pr = synth.unit_tokens(W_SMALL, 1, 0, n, recipe="projected")
    for n_ in ("k", "q"):
        norms = st[n_].norm(dim=1)
        assert torch.allclose(norms, torch.ones_like(norms), atol=1e-5)
    assert 0.95 < float(st["v"].std()) < 1.05 and abs(float(st["v"].mean())) < 0.02

    def r2(k, v):
        sol = torch.linalg.lstsq(k.double(), v.double()).solution
        res = v.double() - k.double() @ sol
        return 1.0 - float(res.pow(2).sum() / (v.double() - v.double().mean(0)).pow(2).sum())
    assert r2(pr["k"], pr["v"]) > 0.5  # k is v's x, renormalised per token
    assert r2(st["k"], st["v"]) < 0.05
    amax, elo, ehi, tmax = synth._gate_ranges(W_SMALL, "stated")
    assert (amax, elo, ehi, tmax) == (0.05, 0.8, 0.99, 0.1)
    assert 0 <= float(st["alpha"].min()) and float(st["alpha"].max()) <= amax
    assert float(st["alpha"].max()) > 0.99 * amax  # spans the range, not the projected recipe's
    assert elo <= float(st["eta"].min()) and float(st["eta"].max()) <= ehi
    assert 0 <= float(st["theta"].min()) and float(st["theta"].max()) <= tmax
    assert float(st["theta"].max()) > 0.99 * tmax
    # its own generators: no stream shared with the projected recipe
    assert not torch.equal(st["alpha"], pr["alpha"])


def test_linear_workload_defaults_to_the_stated_recipe():
    w = synth.WORKLOADS["linear-d64"]
    assert w.recipe == "stated"
    a = synth.make_inputs(w, T=64)
    b = synth.make_inputs(w, T=64, recipe="stated")
    assert all(torch.equal(a[n], b[n]) for n in a)
    d = synth.describe(w)
    assert d["recipe"] == "stated" and d["alpha"] == "U(0, 0.05)" and d["theta"] == "U(0, 0.1)"
    assert synth.describe(W_SMALL)["theta"] == "U(0, 0.003)"
    with pytest.raises(ValueError):
        synth.make_inputs(w, T=4, recipe="nope")


def test_stated_recipe_decode_and_recall():
    w = synth.WORKLOADS["mlp-d128-b4h8-t16k"]
    a = synth.decode_step_inputs(w, 3, dtype="fp32", recipe="stated")
    b = synth.decode_step_inputs(w, 3, dtype="fp32", recipe="stated")
    assert all(torch.equal(a[n], b[n]) for n in a)
    assert a["k"].shape == (w.decode_B * w.H, w.d)
    assert float(a["theta"].max()) > 0.09
    wl = synth.WORKLOADS["mlp-d64-b1h16-t1m"]
    t = synth.unit_tokens(wl, 2, 0, 2 * synth.RECALL_EVERY, recipe="stated")
    p = synth.recall_positions(wl, 0, 2 * synth.RECALL_EVERY)
    assert torch.equal(t["k"][p[0]], t["k"][p[1]]) and torch.equal(t["q"][p[0]], t["k"][p[0]])
