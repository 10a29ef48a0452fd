"""titans_mem_forward_host: token streams and y in host memory, T cut into chunk-aligned
segments whose copies overlap the compute. A segment boundary is a chunk boundary, so the
result must equal titans_mem_forward over the whole stream bit for bit (the continuity the
chunked recurrence has; walk-through sec. 3.2: every chunk starts from the weights the
previous one ended with)."""
import pytest
import torch

from parity import gpu_inputs
from titans_long_term_b200 import mem, synth

pytestmark = pytest.mark.gpu


def _both(name, T, mode, t_seg, pinned, B, H, chunk=None):
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w, units=range(B * H), T=T, dtype=mode)
    chunk = chunk or w.chunk
    m = mem.Memory(w.d, w.h, chunk, mode, B, H)
    toks, gates, state = gpu_inputs(inp, B, H)
    y_ref = m.forward(toks["k"], toks["q"], toks["v"], gates["alpha"], gates["eta"], gates["theta"], state)
    m.sync_status()
    _, _, state2 = gpu_inputs(inp, B, H)
    host = {n: t.cpu() for n, t in list(toks.items()) + list(gates.items())}
    y_host = torch.empty(y_ref.shape, dtype=y_ref.dtype)
    if pinned:
        host = {n: t.pin_memory() for n, t in host.items()}
        y_host = y_host.pin_memory()
    staging = {n: torch.empty_like(t) for n, t in list(toks.items()) + list(gates.items())}
    staging["y"] = torch.empty_like(y_ref)
    m.forward_host(host["k"], host["q"], host["v"], host["alpha"], host["eta"], host["theta"], state2, y_host,
                   staging, t_seg=t_seg)
    m.sync_status()
    return y_ref.cpu(), state, y_host, state2


@pytest.mark.parametrize("T,t_seg,pinned", [(1000, 256, True), (2048, 0, True), (700, 128, False), (64, 64, True)])
def test_forward_host_equals_forward_tensor_cores(T, t_seg, pinned):
    y_ref, s_ref, y, s = _both("mlp-d64-b2h4-t2k", T, "bf16", t_seg, pinned, 2, 4)
    assert torch.equal(y, y_ref)
    assert all(torch.equal(s[n], s_ref[n]) for n in s_ref)


def test_forward_host_equals_forward_fp32_wide():
    y_ref, s_ref, y, s = _both("mlp-d128-b4h8-t16k", 700, "fp32", 256, True, 1, 2)
    assert torch.equal(y, y_ref)
    assert all(torch.equal(s[n], s_ref[n]) for n in s_ref)


def test_forward_host_rejects_unaligned_segment():
    w = synth.WORKLOADS["mlp-d64-b2h4-t2k"]
    m = mem.Memory(w.d, w.h, 64, "bf16", 1, 1)
    st = mem.new_state(1, 1, w.d, w.h)
    k = torch.zeros(1, 1, 256, w.d, dtype=torch.bfloat16)
    g = torch.zeros(1, 1, 256)
    staging = {n: torch.zeros_like(k, device="cuda") for n in ("k", "q", "v", "y")}
    staging.update({n: torch.zeros_like(g, device="cuda") for n in ("alpha", "eta", "theta")})
    with pytest.raises(mem.TitansError) as e:
        m.forward_host(k, k, k, g, g, g, st, torch.empty_like(k), staging, t_seg=100)
    assert e.value.status == mem.EINVAL
