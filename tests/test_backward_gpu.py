"""GPU parity of the linear memory's backward (titans_mem_backward) against the oracle's fp64
reverse-mode gradients: every input's gradient (k, q, v, the gates, the initial state) for a loss on
y and on the final state."""
import numpy as np
import pytest
import torch

import oracle
from parity import TOL, rel_err
from titans_long_term_b200 import mem, synth

pytestmark = pytest.mark.gpu


def _case(d, B, H, T, chunk, mode, seed, with_dstate):
    w = synth.Workload(f"linear-d{d}-bwd", d, 0, B, H, T, chunk, mode, 20251201 + seed, recipe="stated")
    inp = synth.make_inputs(w)
    U = B * H
    g = torch.Generator().manual_seed(seed)
    # a non-zero initial state, so that every term of the adjoint is exercised
    inp["W1"] = torch.randn(U, d, d, generator=g) / np.sqrt(d)
    inp["S1"] = torch.randn(U, d, d, generator=g) * 0.01
    dy = torch.randn(U, T, d, generator=g).to(inp["k"].dtype)
    dst = {"W1": torch.randn(U, d, d, generator=g), "S1": torch.randn(U, d, d, generator=g)} if with_dstate else {}
    return w, inp, dy, dst


@pytest.mark.parametrize("d,B,H,T,chunk,mode,with_dstate", [
    (64, 1, 2, 64, 16, "fp32", True),
    (64, 1, 2, 50, 16, "fp32", False),   # ragged last chunk, loss on y only
    (64, 2, 1, 40, 1, "fp32", True),     # chunk = 1: the per-token recurrence
    (32 * 2, 1, 1, 96, 32, "bf16", True),
    (128, 1, 1, 48, 16, "fp32", True),
])
def test_linear_backward_matches_the_oracle(d, B, H, T, chunk, mode, with_dstate):
    w, inp, dy, dst = _case(d, B, H, T, chunk, mode, d + T + chunk, with_dstate)
    U = B * H
    m = mem.Memory(d, 0, chunk, mode, B, H)
    dev = lambda x, *s: x.reshape(B, H, *s).cuda().contiguous()
    args = [dev(inp[n], T, d) for n in ("k", "q", "v")] + [dev(inp[n], T) for n in ("alpha", "eta", "theta")]
    state = {n: dev(inp[n], d, d) for n in ("W1", "S1")}
    dstate = {n: dev(x, d, d) for n, x in dst.items()}
    out = m.backward(*args, state, dev(dy, T, d), dstate, chunk=chunk)
    m.sync_status()
    ref = oracle.backward(inp["k"], inp["q"], inp["v"], inp["alpha"], inp["eta"], inp["theta"],
                          {n: inp[n] for n in ("W1", "S1")}, chunk, dy.float(), {n: x for n, x in dst.items()})
    tol = TOL[mode]
    worst = {}
    for n in ("k", "q", "v", "alpha", "eta", "theta", "W1", "S1"):
        x = out[n].reshape(U, -1).float().cpu().numpy()
        r = ref[n].reshape(U, -1)
        e = rel_err(x, r)
        worst[n] = float(e.max())
        assert np.isfinite(x).all(), n
        assert e.max() <= tol, f"d{n}: {e.max():.3e} > {tol}"
    print(f"backward d={d} T={T} chunk={chunk} {mode}:", {k: f"{v:.1e}" for k, v in worst.items()})


def _mlp_case(B, H, T, chunk, mode, seed, with_dstate, recipe=None):
    w = synth.WORKLOADS["mlp-d64-b2h4-t2k"]
    inp = synth.make_inputs(w, units=range(B * H), T=T, dtype=mode, recipe=recipe)
    U = B * H
    g = torch.Generator().manual_seed(seed)
    inp["S1"] = torch.randn(*inp["S1"].shape, generator=g) * 0.01  # a non-zero momentum, every term exercised
    inp["S2"] = torch.randn(*inp["S2"].shape, generator=g) * 0.01
    dy = torch.randn(U, T, 64, generator=g).to(inp["k"].dtype)
    dst = {n: torch.randn(*inp[n].shape, generator=g) for n in ("W1", "W2", "S1", "S2")} if with_dstate else {}
    return w, inp, dy, dst


@pytest.mark.parametrize("B,H,T,chunk,mode,with_dstate,recipe", [
    (1, 2, 40, 16, "fp32", True, None),       # ragged last chunk
    (2, 1, 64, 64, "fp32", False, None),      # one chunk, loss on y only
    (1, 2, 12, 1, "fp32", True, None),        # chunk = 1
    (1, 2, 64, 32, "fp32", True, "stated"),   # the stated gate ranges
    (1, 2, 48, 16, "bf16", True, None),       # bf16 token streams (the tensor-core backward from here on)
    (2, 2, 200, 64, "bf16", True, None),      # several chunks, ragged last chunk
    (1, 2, 64, 64, "bf16", False, None),      # one chunk, loss on y only
    (1, 2, 9, 1, "bf16", True, None),         # chunk = 1
    (1, 2, 64, 32, "bf16", True, "stated"),   # the stated gate ranges, over the two chunks the memory stays bounded
])
def test_mlp_backward_matches_the_oracle(B, H, T, chunk, mode, with_dstate, recipe):
    """The MLP memory's adjoint includes the second-order terms of the inner gradient (its update
    depends on W through g); against fp64 reverse-mode differentiation of the token loop."""
    w, inp, dy, dst = _mlp_case(B, H, T, chunk, mode, T + chunk, with_dstate, recipe)
    U = B * H
    m = mem.Memory(64, 256, chunk, mode, B, H)
    assert m.backward_path(chunk) == (mem.PATH_TC_BACKWARD if mode == "bf16" else mem.PATH_CUDA_CORES)
    dev = lambda x: x.reshape(B, H, *x.shape[1:]).cuda().contiguous()
    args = [dev(inp[n]) for n in ("k", "q", "v", "alpha", "eta", "theta")]
    state = {n: dev(inp[n]) for n in ("W1", "W2", "S1", "S2")}
    out = m.backward(*args, state, dev(dy), {n: dev(x) for n, x in dst.items()}, chunk=chunk)
    m.sync_status()
    ref = oracle.backward(inp["k"], inp["q"], inp["v"], inp["alpha"], inp["eta"], inp["theta"],
                          {n: inp[n] for n in ("W1", "W2", "S1", "S2")}, chunk, dy.float(), dst)
    worst = {}
    for n in ("k", "q", "v", "alpha", "eta", "theta", "W1", "W2", "S1", "S2"):
        x = out[n].reshape(U, -1).float().cpu().numpy()
        e = rel_err(x, ref[n].reshape(U, -1))
        worst[n] = float(e.max())
        assert np.isfinite(x).all(), n
        assert e.max() <= TOL[mode], f"d{n}: {e.max():.3e} > {TOL[mode]}"
    print(f"MLP backward T={T} chunk={chunk} {mode} {recipe}:", {k: f"{v:.1e}" for k, v in worst.items()})


def test_backward_leaves_its_inputs_alone_and_rejects_a_deep_memory():
    w, inp, dy, dst = _case(64, 1, 1, 32, 16, "fp32", 5, True)
    m = mem.Memory(64, 0, 16, "fp32", 1, 1)
    dev = lambda x, *s: x.reshape(1, 1, *s).cuda().contiguous()
    state = {n: dev(inp[n], 64, 64) for n in ("W1", "S1")}
    before = {n: t.clone() for n, t in state.items()}
    m.backward(*[dev(inp[n], 32, 64) for n in ("k", "q", "v")], *[dev(inp[n], 32) for n in ("alpha", "eta", "theta")],
               state, dev(dy, 32, 64), {n: dev(x, 64, 64) for n, x in dst.items()})
    m.sync_status()
    assert all(torch.equal(before[n], state[n]) for n in state)
    deep = mem.Memory(64, 256, 16, "fp32", 1, 1, layers=3)
    with pytest.raises(mem.TitansError) as ei:
        z = torch.zeros(1, 1, 8, 64, device="cuda")
        gz = torch.zeros(1, 1, 8, device="cuda")
        deep.backward(z, z, z, gz, gz, gz, {"W1": torch.zeros(1, 1, 256, 64, device="cuda"),
                                            "S1": torch.zeros(1, 1, 256, 64, device="cuda")}, z)
    assert ei.value.status == mem.EUNSUPPORTED


def test_mlp_backward_tensor_cores_against_cuda_cores():
    """The bf16 tensor-core backward and the fp32 CUDA-core one (TITANS_FLAG_CUDA_CORES) on the same
    inputs: each within the bf16 bar of the oracle's gradients."""
    B, H, T, chunk = 2, 2, 256, 64
    w, inp, dy, dst = _mlp_case(B, H, T, chunk, "bf16", 3, True)
    dev = lambda x: x.reshape(B, H, *x.shape[1:]).cuda().contiguous()
    args = [dev(inp[n]) for n in ("k", "q", "v", "alpha", "eta", "theta")]
    state = {n: dev(inp[n]) for n in ("W1", "W2", "S1", "S2")}
    ref = oracle.backward(inp["k"], inp["q"], inp["v"], inp["alpha"], inp["eta"], inp["theta"],
                          {n: inp[n] for n in ("W1", "W2", "S1", "S2")}, chunk, dy.float(), dst)
    for cuda_cores in (False, True):
        m = mem.Memory(64, 256, chunk, "bf16", B, H, cuda_cores=cuda_cores)
        out = m.backward(*args, state, dev(dy), {n: dev(x) for n, x in dst.items()}, chunk=chunk)
        m.sync_status()
        for n in ("k", "q", "v", "alpha", "eta", "theta", "W1", "W2", "S1", "S2"):
            e = rel_err(out[n].reshape(B * H, -1).float().cpu().numpy(), ref[n].reshape(B * H, -1))
            assert e.max() <= TOL["bf16"], f"{'CUDA cores' if cuda_cores else 'tensor cores'} d{n}: {e.max():.3e}"
