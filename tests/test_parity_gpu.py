"""GPU parity of every kernel path against the oracle, on seeded synthetic inputs at
sizes the oracle finishes in seconds (several tiles and chunks, ragged tails), plus the
method's invariants checked bitwise on the GPU."""
import numpy as np
import pytest
import torch

import oracle
from parity import TOL, compare, gpu_inputs, run_gpu, run_oracle, step_sequence, workload_inputs
from titans_long_term_b200 import mem, synth

pytestmark = pytest.mark.gpu


def make_mem(w, mode, chunk=None, cuda_cores=False, B=None, H=None):
    return mem.Memory(w.d, w.h, chunk or w.chunk, mode, B or w.B, H or w.H, cuda_cores=cuda_cores)


# ---------------------------------------------------------------- each path vs the oracle

@pytest.mark.parametrize("mode", ["fp32", "bf16"])
def test_linear_memory(mode):
    """Linear memory W in R^{64x64}, T=256, chunk=16 (CUDA-core kernel)."""
    w, inp = workload_inputs("linear-d64", dtype=mode)
    m = make_mem(w, mode)
    assert m.path() == mem.PATH_CUDA_CORES
    gy, gst = run_gpu(m, inp, w.B, w.H, w.chunk)
    ry, rst = run_oracle(inp, w.chunk)
    compare(gy, gst, ry, rst, TOL[mode], what=f"linear {mode}")


@pytest.mark.parametrize("T,chunk", [(2048, 64), (200, 64), (130, 32), (77, 16), (45, 1), (5, 64), (1, 1)])
def test_mlp64_tensor_cores(T, chunk):
    """tcgen05 kernel, d=64 h=256, B=2 H=4: full chunks, ragged last chunk, chunk < 64, T < chunk."""
    w, inp = workload_inputs("mlp-d64-b2h4-t2k", T=T)
    m = make_mem(w, "bf16", chunk=chunk)
    assert m.path(chunk) == mem.PATH_TC_MLP64
    gy, gst = run_gpu(m, inp, w.B, w.H, chunk)
    ry, rst = run_oracle(inp, chunk)
    compare(gy, gst, ry, rst, TOL["bf16"], what=f"tc T={T} chunk={chunk}")


def test_mlp64_tensor_cores_more_units_than_sms():
    """160 units (more CTAs than the 148 SMs), T = 192 with chunk 64."""
    w = synth.WORKLOADS["mlp-d64-b8h16-t4k"]
    inp = synth.make_inputs(w, units=range(160), T=192)
    m = mem.Memory(64, 256, 64, "bf16", 10, 16)
    gy, gst = run_gpu(m, inp, 10, 16, 64)
    ry, rst = run_oracle(inp, 64)
    compare(gy, gst, ry, rst, TOL["bf16"], what="160 units")


@pytest.mark.parametrize("mode,T,chunk", [("fp32", 512, 64), ("bf16", 256, 64), ("fp32", 100, 48)])
def test_mlp64_cuda_cores(mode, T, chunk):
    """CUDA-core kernel for the d=64 MLP (fp32 reference mode, and bf16 inputs when asked)."""
    w, inp = workload_inputs("mlp-d64-b2h4-t2k", T=T, dtype=mode)
    m = make_mem(w, mode, chunk=chunk, cuda_cores=True)
    assert m.path(chunk) == mem.PATH_CUDA_CORES
    gy, gst = run_gpu(m, inp, w.B, w.H, chunk)
    ry, rst = run_oracle(inp, chunk)
    compare(gy, gst, ry, rst, TOL[mode], what=f"cuda cores {mode}")


@pytest.mark.parametrize("mode", ["fp32", "bf16"])
def test_mlp128_cuda_cores(mode):
    """d=128, h=512, chunk=128 (wide memory prefill shape), 4 units, T = 300 (ragged)."""
    w = synth.WORKLOADS["mlp-d128-b4h8-t16k"]
    inp = synth.make_inputs(w, units=range(4), T=300, dtype=mode)
    m = mem.Memory(128, 512, 128, mode, 2, 2, cuda_cores=True)
    assert m.path(128) == mem.PATH_CUDA_CORES
    gy, gst = run_gpu(m, inp, 2, 2, 128)
    ry, rst = run_oracle(inp, 128)
    compare(gy, gst, ry, rst, TOL[mode], what=f"d128 {mode}")


# ---------------------------------------------------------------- decode step

@pytest.mark.parametrize("name,mode", [("mlp-d64-b2h4-t2k", "bf16"), ("mlp-d64-b2h4-t2k", "fp32"),
                                       ("mlp-d128-b4h8-t16k", "bf16"), ("mlp-d128-b4h8-t16k", "fp32"),
                                       ("linear-d64", "fp32")])
def test_decode_steps(name, mode):
    """k decode steps equal the oracle with chunk = 1 (retrieve with W_{t-1}, then update)."""
    w = synth.WORKLOADS[name]
    units = min(w.units, 8)
    inp = synth.make_inputs(w, units=range(units), T=12, dtype=mode)
    B, H = (units // 2, 2) if units > 1 else (1, 1)
    m = mem.Memory(w.d, w.h, 1, mode, B, H)
    gy, gst = step_sequence(m, inp, B, H, 12)
    ry, rst = run_oracle(inp, 1)
    compare(gy, gst, ry, rst, TOL[mode], what=f"step {name} {mode}")


# ---------------------------------------------------------------- invariants, bitwise on the GPU

def _tc_run(inp, B, H, chunk=64, q_override=None):
    m = mem.Memory(64, 256, chunk, "bf16", B, H)
    toks, gates, state = gpu_inputs(inp, B, H)
    q = toks["q"] if q_override is None else q_override
    y = m.forward(toks["k"], q, toks["v"], gates["alpha"], gates["eta"], gates["theta"], state)
    m.sync_status()
    return y, state


def test_deterministic():
    w, inp = workload_inputs("mlp-d64-b2h4-t2k", T=300)
    y1, s1 = _tc_run(inp, 2, 4)
    y2, s2 = _tc_run(inp, 2, 4)
    assert torch.equal(y1, y2) and all(torch.equal(s1[n], s2[n]) for n in s1)


def test_retrieval_does_not_write():
    """The final state is independent of the queries (bitwise)."""
    w, inp = workload_inputs("mlp-d64-b2h4-t2k", T=256)
    _, s1 = _tc_run(inp, 2, 4)
    k = inp["k"].reshape(2, 4, 256, 64).cuda().contiguous()
    _, s2 = _tc_run(inp, 2, 4, q_override=k)
    assert all(torch.equal(s1[n], s2[n]) for n in s1)


def test_continuity():
    """forward(T1) then forward(T2) == forward(T1 + T2) when T1 is a multiple of the chunk (bitwise)."""
    w, inp = workload_inputs("mlp-d64-b2h4-t2k", T=320)
    y, s = _tc_run(inp, 2, 4)
    first = {n: (x[:, :192] if n in ("k", "q", "v", "alpha", "eta", "theta") else x) for n, x in inp.items()}
    y1, s1 = _tc_run(first, 2, 4)
    second = {n: x[:, 192:] for n, x in inp.items() if n in ("k", "q", "v", "alpha", "eta", "theta")}
    second.update({n: t.reshape(8, *t.shape[2:]).cpu() for n, t in s1.items()})
    y2, s2 = _tc_run(second, 2, 4)
    assert torch.equal(torch.cat([y1, y2], dim=2), y)
    assert all(torch.equal(s[n], s2[n]) for n in s)


def test_unit_permutation():
    """Units are independent: permuting them permutes every output (bitwise)."""
    w, inp = workload_inputs("mlp-d64-b2h4-t2k", T=130)
    p = torch.tensor([5, 2, 7, 0, 1, 3, 6, 4])
    y, s = _tc_run(inp, 2, 4)
    y2, s2 = _tc_run({n: x[p] for n, x in inp.items()}, 2, 4)
    assert torch.equal(y.reshape(8, 130, 64)[p.cuda()], y2.reshape(8, 130, 64))
    for n in s:
        assert torch.equal(s[n].reshape(8, *s[n].shape[2:])[p.cuda()], s2[n].reshape(8, *s[n].shape[2:]))


def test_reset_makes_mlp_memory_zero():
    """alpha = 1, eta = 0, theta = 0 on the last token of a chunk: W = 0 is a fixed point of the MLP
    memory, so every later retrieval is exactly zero and the state stays zero."""
    w, inp = workload_inputs("mlp-d64-b2h4-t2k", T=256)
    inp["alpha"][:, 127] = 1.0
    inp["eta"][:, 127] = 0.0
    inp["theta"][:, 127] = 0.0
    y, s = _tc_run(inp, 2, 4)
    assert not y.reshape(8, 256, 64)[:, 128:].any()
    assert not any(t.any() for t in s.values())


def test_status_word_clear_and_bad_arguments():
    w, inp = workload_inputs("mlp-d64-b2h4-t2k", T=64)
    m = make_mem(w, "bf16")
    toks, gates, state = gpu_inputs(inp, 2, 4)
    with pytest.raises(mem.TitansError):  # T = 0
        mem.lib()  # noqa
        rc = mem.lib().titans_mem_forward(m._h, toks["k"].data_ptr(), toks["q"].data_ptr(), toks["v"].data_ptr(),
                                          gates["alpha"].data_ptr(), gates["eta"].data_ptr(),
                                          gates["theta"].data_ptr(), 0, 64, state["W1"].data_ptr(),
                                          state["W2"].data_ptr(), state["S1"].data_ptr(), state["S2"].data_ptr(),
                                          toks["k"].data_ptr(), None)
        mem._check(rc)
    rc = mem.lib().titans_mem_forward(m._h, toks["k"].data_ptr() + 2, toks["q"].data_ptr(), toks["v"].data_ptr(),
                                      gates["alpha"].data_ptr(), gates["eta"].data_ptr(), gates["theta"].data_ptr(),
                                      64, 64, state["W1"].data_ptr(), state["W2"].data_ptr(),
                                      state["S1"].data_ptr(), state["S2"].data_ptr(), toks["k"].data_ptr(), None)
    assert rc == mem.EINVAL  # misaligned k
    rc = mem.lib().titans_mem_forward(m._h, toks["k"].data_ptr(), toks["q"].data_ptr(), toks["v"].data_ptr(),
                                      gates["alpha"].data_ptr(), gates["eta"].data_ptr(), gates["theta"].data_ptr(),
                                      64, 65, state["W1"].data_ptr(), state["W2"].data_ptr(),
                                      state["S1"].data_ptr(), state["S2"].data_ptr(), toks["k"].data_ptr(), None)
    assert rc == mem.EUNSUPPORTED  # chunk above the handle's maximum
    m.sync_status()
