"""Python binding of the C ABI in include/titans_mem.h (argument marshalling only).

Every computation runs in the CUDA library ``libtitans_mem.so`` built in-tree by
``titans_long_term_b200/build.py``; if the library is missing this module raises
instead of falling back to anything else. PyTorch supplies device memory and the
current CUDA stream. With the environment variable ``TITANS_DEBUG=1`` the binding loads
``libtitans_mem_debug.so`` (``build.py --debug``), whose kernels check the coordinates and
offsets of their memory accesses and report a failed check in the status word.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
DEBUG = os.environ.get("TITANS_DEBUG", "0") == "1"
LIB_PATH = os.path.join(HERE, "libtitans_mem_debug.so" if DEBUG else "libtitans_mem.so")

OK, EINVAL, EUNSUPPORTED, ECUDA, EDEVICE = 0, 1, 2, 3, 4
BF16, FP32 = 0, 1
FLAG_CUDA_CORES = 1
FLAG_CHUNK_GATES = 2
FLAG_CHUNK_SCAN = 4
(PATH_TC_MLP64, PATH_CUDA_CORES, PATH_STEP_CLUSTER, PATH_TC_PHASED, PATH_DEEP_CUDA_CORES,
 PATH_LINEAR_SCAN, PATH_TC_DEEP, PATH_TC_BACKWARD) = 1, 2, 3, 4, 5, 6, 7, 8

EXPORTED = ["titans_mem_init", "titans_mem_destroy", "titans_mem_forward", "titans_mem_step",
            "titans_mem_path", "titans_mem_sync_status", "titans_last_error_string", "titans_mem_version",
            "titans_mem_forward_noalloc", "titans_mem_forward_host", "titans_mem_forward_gated",
            "titans_mem_step_gated", "titans_mem_init_deep", "titans_mem_forward_deep", "titans_mem_backward",
            "titans_mem_backward_workspace_bytes", "titans_silu_routes"]


class TitansError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"titans status {status}: {msg}")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int), ("d_hidden", ctypes.c_int), ("chunk", ctypes.c_int),
                ("mode", ctypes.c_int), ("B", ctypes.c_int), ("H", ctypes.c_int), ("flags", ctypes.c_uint)]


class DeviceBuffers(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("q", ctypes.c_void_p), ("v", ctypes.c_void_p), ("alpha", ctypes.c_void_p),
                ("eta", ctypes.c_void_p), ("theta", ctypes.c_void_p), ("y", ctypes.c_void_p)]


_lib = None


def lib():
    """Load the library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            how = " --debug" if DEBUG else ""
            raise ImportError(f"{LIB_PATH} is missing: run `python -m titans_long_term_b200.build{how}`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, l = ctypes.c_void_p, ctypes.c_int, ctypes.c_long
        L.titans_mem_init.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(vp)]
        L.titans_mem_destroy.argtypes = [vp]
        L.titans_mem_forward.argtypes = [vp, vp, vp, vp, vp, vp, vp, l, i, vp, vp, vp, vp, vp, vp]
        L.titans_mem_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.titans_mem_path.argtypes = [vp, i, i]
        L.titans_mem_forward_noalloc.argtypes = [ctypes.POINTER(Config), vp, vp, vp, vp, vp, vp, l, i, vp, vp, vp,
                                                 vp, vp, vp]
        L.titans_mem_forward_host.argtypes = [vp, vp, vp, vp, vp, vp, vp, l, i, vp, vp, vp, vp, vp,
                                              ctypes.POINTER(DeviceBuffers), l, vp]
        L.titans_mem_forward_gated.argtypes = [vp, vp, vp, vp, vp, vp, vp, l, i, vp, vp, vp, vp, vp, vp, vp]
        L.titans_mem_step_gated.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.titans_mem_init_deep.argtypes = [ctypes.POINTER(Config), i, ctypes.POINTER(vp)]
        L.titans_mem_forward_deep.argtypes = [vp, vp, vp, vp, vp, vp, vp, l, i, vp, vp, vp, vp, vp]
        L.titans_mem_backward_workspace_bytes.argtypes = [vp, l, i]
        L.titans_mem_backward_workspace_bytes.restype = ctypes.c_size_t
        L.titans_mem_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, l, i] + [vp] * 20 + [ctypes.c_size_t, vp]
        L.titans_mem_sync_status.argtypes = [vp, vp]
        L.titans_silu_routes.argtypes = [vp, vp, vp, l, vp]
        L.titans_last_error_string.restype = ctypes.c_char_p
        for f in ("titans_mem_init", "titans_mem_destroy", "titans_mem_forward", "titans_mem_step",
                  "titans_mem_path", "titans_mem_sync_status", "titans_mem_version", "titans_mem_forward_noalloc",
                  "titans_mem_forward_host", "titans_mem_forward_gated", "titans_mem_step_gated",
                  "titans_mem_init_deep", "titans_mem_forward_deep", "titans_mem_backward", "titans_silu_routes"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(status: int):
    if status != OK:
        raise TitansError(status, lib().titans_last_error_string().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


class Memory:
    """A configured memory: B*H independent units of a linear (d_hidden = 0) or
    2-layer SiLU MLP memory (d_hidden = 4d)."""

    def __init__(self, d: int, d_hidden: int, chunk: int, mode: str, B: int, H: int, cuda_cores: bool = False,
                 layers: Optional[int] = None, chunk_gates: bool = False, chunk_scan: bool = False):
        self.d, self.h, self.chunk, self.B, self.H = d, d_hidden, chunk, B, H
        self.mode = mode
        self.layers = layers or 2
        self.chunk_gates = chunk_gates
        self.dtype = torch.bfloat16 if mode == "bf16" else torch.float32
        cfg = Config(d, d_hidden, chunk, BF16 if mode == "bf16" else FP32, B, H,
                     (FLAG_CUDA_CORES if cuda_cores else 0) | (FLAG_CHUNK_GATES if chunk_gates else 0) |
                     (FLAG_CHUNK_SCAN if chunk_scan else 0))
        h = ctypes.c_void_p()
        if layers is None:
            _check(lib().titans_mem_init(ctypes.byref(cfg), ctypes.byref(h)))
        else:
            _check(lib().titans_mem_init_deep(ctypes.byref(cfg), layers, ctypes.byref(h)))
        self._h = h

    def close(self):
        if getattr(self, "_h", None):
            lib().titans_mem_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def path(self, chunk: Optional[int] = None, step: bool = False) -> int:
        return lib().titans_mem_path(self._h, chunk or self.chunk, int(step))

    def backward_path(self, chunk: Optional[int] = None) -> int:
        """Kernel titans_mem_backward runs with this chunk length."""
        return lib().titans_mem_path(self._h, chunk or self.chunk, 2)

    def _gate_lead(self, lead, chunk):
        """Shape of a gate array: one value per token, or per chunk with chunk-shared gates."""
        if not self.chunk_gates or len(lead) < 3:
            return lead
        return lead[:-1] + ((lead[-1] + chunk - 1) // chunk,)

    def _check_tensors(self, toks, gates, state, y, lead, chunk=None):
        for n, t in list(toks.items()) + [("y", y)]:
            if t.dtype != self.dtype or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != lead + (self.d,):
                raise ValueError(f"{n}: expected contiguous CUDA {self.dtype} of shape {lead + (self.d,)}")
        glead = self._gate_lead(lead, chunk or self.chunk)
        for n, t in gates.items():
            if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != glead:
                raise ValueError(f"{n}: expected contiguous CUDA float32 of shape {glead}")
        for n, t in state.items():
            if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
                raise ValueError(f"{n}: expected contiguous CUDA float32")

    def forward(self, k, q, v, alpha, eta, theta, state: Dict[str, torch.Tensor], chunk: Optional[int] = None,
                y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """k, q, v [B, H, T, d]; gates [B, H, T]; state W1, S1 (+ W2, S2) updated in place; returns y."""
        T = k.shape[-2]
        if y is None:
            y = torch.empty_like(k)
        self._check_tensors({"k": k, "q": q, "v": v}, {"alpha": alpha, "eta": eta, "theta": theta}, state, y,
                            (self.B, self.H, T), chunk)
        _check(lib().titans_mem_forward(self._h, _ptr(k), _ptr(q), _ptr(v), _ptr(alpha), _ptr(eta), _ptr(theta),
                                        T, chunk or self.chunk, _ptr(state["W1"]), _ptr(state.get("W2")),
                                        _ptr(state["S1"]), _ptr(state.get("S2")), _ptr(y), _stream(stream)))
        return y

    def forward_gated(self, k, q, v, alpha, eta, theta, attn, state: Dict[str, torch.Tensor],
                      chunk: Optional[int] = None, o: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """Memory-as-a-gate output: o = attn * sigmoid(M(q)) element-wise, attn [B, H, T, d] in the
        dtype of k (the attention branch's output); otherwise as forward(). Returns o."""
        T = k.shape[-2]
        if o is None:
            o = torch.empty_like(k)
        self._check_tensors({"k": k, "q": q, "v": v, "attn": attn}, {"alpha": alpha, "eta": eta, "theta": theta},
                            state, o, (self.B, self.H, T), chunk)
        _check(lib().titans_mem_forward_gated(self._h, _ptr(k), _ptr(q), _ptr(v), _ptr(alpha), _ptr(eta),
                                              _ptr(theta), T, chunk or self.chunk, _ptr(state["W1"]),
                                              _ptr(state.get("W2")), _ptr(state["S1"]), _ptr(state.get("S2")),
                                              _ptr(attn), _ptr(o), _stream(stream)))
        return o

    def forward_deep(self, k, q, v, alpha, eta, theta, state: Dict[str, torch.Tensor], chunk: Optional[int] = None,
                     attn: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """Deep memory (a handle made with layers=L): state {"W", "S"} [B, H, P] fp32, the layers packed
        per unit (W_1 [h, d], W_2 .. W_{L-1} [h, h], W_L [d, h]); optional attn for the gated output."""
        T = k.shape[-2]
        if y is None:
            y = torch.empty_like(k)
        toks = {"k": k, "q": q, "v": v}
        if attn is not None:
            toks["attn"] = attn
        self._check_tensors(toks, {"alpha": alpha, "eta": eta, "theta": theta}, state, y, (self.B, self.H, T), chunk)
        _check(lib().titans_mem_forward_deep(self._h, _ptr(k), _ptr(q), _ptr(v), _ptr(alpha), _ptr(eta), _ptr(theta),
                                             T, chunk or self.chunk, _ptr(state["W"]), _ptr(state["S"]), _ptr(attn),
                                             _ptr(y), _stream(stream)))
        return y

    def backward(self, k, q, v, alpha, eta, theta, state: Dict[str, torch.Tensor], dy: torch.Tensor,
                 dstate: Optional[Dict[str, torch.Tensor]] = None, chunk: Optional[int] = None,
                 stream=None) -> Dict[str, torch.Tensor]:
        """Gradients of <dy, y> + sum_n <dstate[n], final state[n]> (dstate optional) with respect to
        k, q, v, the gates and the initial state (read only). Returns a dict with keys k, q, v, alpha,
        eta, theta and the state's names."""
        T = k.shape[-2]
        chunk = chunk or self.chunk
        self._check_tensors({"k": k, "q": q, "v": v, "dy": dy}, {"alpha": alpha, "eta": eta, "theta": theta},
                            state, torch.empty_like(k), (self.B, self.H, T), chunk)
        out = {n: torch.empty_like(x) for n, x in (("k", k), ("q", q), ("v", v), ("alpha", alpha), ("eta", eta),
                                                   ("theta", theta))}
        for n in state:
            out[n] = torch.empty_like(state[n])
        nbytes = lib().titans_mem_backward_workspace_bytes(self._h, T, chunk)
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=k.device)
        ds = dstate or {}
        _check(lib().titans_mem_backward(
            self._h, _ptr(k), _ptr(q), _ptr(v), _ptr(alpha), _ptr(eta), _ptr(theta), T, chunk, _ptr(state["W1"]),
            _ptr(state.get("W2")), _ptr(state["S1"]), _ptr(state.get("S2")), _ptr(dy), _ptr(ds.get("W1")),
            _ptr(ds.get("W2")), _ptr(ds.get("S1")), _ptr(ds.get("S2")), _ptr(out["k"]), _ptr(out["q"]), _ptr(out["v"]),
            _ptr(out["alpha"]), _ptr(out["eta"]), _ptr(out["theta"]), _ptr(out["W1"]), _ptr(out.get("W2")),
            _ptr(out["S1"]), _ptr(out.get("S2")), _ptr(ws), nbytes, _stream(stream)))
        return out

    def forward_host(self, k, q, v, alpha, eta, theta, state: Dict[str, torch.Tensor], y: torch.Tensor,
                     staging: Dict[str, torch.Tensor], chunk: Optional[int] = None, t_seg: int = 0,
                     stream=None) -> torch.Tensor:
        """titans_mem_forward_host: k, q, v [B, H, T, d] and gates [B, H, T] in host memory (pinned
        for overlap), y [B, H, T, d] host output, state on the device (updated in place);
        `staging` holds device tensors k, q, v, alpha, eta, theta, y of the same shapes (scratch).
        Asynchronous on the stream: synchronize before reading y."""
        T = k.shape[-2]
        lead = (self.B, self.H, T)
        for n, t in (("k", k), ("q", q), ("v", v), ("y", y)):
            if t.is_cuda or t.dtype != self.dtype or not t.is_contiguous() or tuple(t.shape) != lead + (self.d,):
                raise ValueError(f"{n}: expected contiguous host {self.dtype} of shape {lead + (self.d,)}")
        glead = self._gate_lead(lead, chunk or self.chunk)
        for n, t in (("alpha", alpha), ("eta", eta), ("theta", theta)):
            if t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous() or tuple(t.shape) != glead:
                raise ValueError(f"{n}: expected contiguous host float32 of shape {glead}")
        self._check_tensors({n: staging[n] for n in ("k", "q", "v")},
                            {n: staging[n] for n in ("alpha", "eta", "theta")}, state, staging["y"], lead, chunk)
        dev = DeviceBuffers(*(staging[n].data_ptr() for n in ("k", "q", "v", "alpha", "eta", "theta", "y")))
        _check(lib().titans_mem_forward_host(self._h, _ptr(k), _ptr(q), _ptr(v), _ptr(alpha), _ptr(eta),
                                             _ptr(theta), T, chunk or self.chunk, _ptr(state["W1"]),
                                             _ptr(state.get("W2")), _ptr(state["S1"]), _ptr(state.get("S2")),
                                             _ptr(y), ctypes.byref(dev), t_seg, _stream(stream)))
        return y

    def step(self, k, q, v, alpha, eta, theta, state: Dict[str, torch.Tensor], y: Optional[torch.Tensor] = None,
             stream=None) -> torch.Tensor:
        """One decode token per unit: k, q, v [B, H, d]; gates [B, H]; state updated in place; returns y."""
        if y is None:
            y = torch.empty_like(k)
        self._check_tensors({"k": k, "q": q, "v": v}, {"alpha": alpha, "eta": eta, "theta": theta}, state, y,
                            (self.B, self.H))
        _check(lib().titans_mem_step(self._h, _ptr(k), _ptr(q), _ptr(v), _ptr(alpha), _ptr(eta), _ptr(theta),
                                     _ptr(state["W1"]), _ptr(state.get("W2")), _ptr(state["S1"]),
                                     _ptr(state.get("S2")), _ptr(y), _stream(stream)))
        return y

    def step_gated(self, k, q, v, alpha, eta, theta, attn, state: Dict[str, torch.Tensor],
                   o: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """One decode token per unit with the memory-as-a-gate output o = attn * sigmoid(M(q)); attn [B, H, d]."""
        if o is None:
            o = torch.empty_like(k)
        self._check_tensors({"k": k, "q": q, "v": v, "attn": attn}, {"alpha": alpha, "eta": eta, "theta": theta},
                            state, o, (self.B, self.H))
        _check(lib().titans_mem_step_gated(self._h, _ptr(k), _ptr(q), _ptr(v), _ptr(alpha), _ptr(eta), _ptr(theta),
                                           _ptr(state["W1"]), _ptr(state.get("W2")), _ptr(state["S1"]),
                                           _ptr(state.get("S2")), _ptr(attn), _ptr(o), _stream(stream)))
        return o

    def sync_status(self, stream=None):
        _check(lib().titans_mem_sync_status(self._h, _stream(stream)))


def new_state(B: int, H: int, d: int, d_hidden: int, device="cuda") -> Dict[str, torch.Tensor]:
    if d_hidden == 0:
        z = torch.zeros(B, H, d, d, device=device)
        return {"W1": z, "S1": z.clone()}
    return {"W1": torch.zeros(B, H, d_hidden, d, device=device), "W2": torch.zeros(B, H, d, d_hidden, device=device),
            "S1": torch.zeros(B, H, d_hidden, d, device=device), "S2": torch.zeros(B, H, d, d_hidden, device=device)}


def forward_noalloc(k, q, v, alpha, eta, theta, state: Dict[str, torch.Tensor], chunk: int, mode: str,
                    y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """titans_mem_forward_noalloc: the CUDA-core chunk forward with the library's fixed scratch
    array (no device allocation by the library). k, q, v [B, H, T, d]; gates [B, H, T]; state
    updated in place; returns y. Calls that overlap on the GPU race on the shared scratch."""
    B, H, T, d = k.shape
    h = state["W1"].shape[-2] if "W2" in state else 0
    if y is None:
        y = torch.empty_like(k)
    cfg = Config(d, h, chunk, BF16 if mode == "bf16" else FP32, B, H, 0)
    _check(lib().titans_mem_forward_noalloc(ctypes.byref(cfg), _ptr(k), _ptr(q), _ptr(v), _ptr(alpha), _ptr(eta),
                                            _ptr(theta), T, chunk, _ptr(state["W1"]), _ptr(state.get("W2")),
                                            _ptr(state["S1"]), _ptr(state.get("S2")), _ptr(y), _stream(stream)))
    return y


def silu_routes(h: torch.Tensor):
    """silu(2h) on the chunk kernel's two routes: (FMA-pipe tanh, hardware tanh.approx), fp32 on the device."""
    if h.dtype != torch.float32 or not h.is_cuda:
        raise TypeError("h must be a CUDA fp32 tensor")
    h = h.contiguous()
    a, b = torch.empty_like(h), torch.empty_like(h)
    _check(lib().titans_silu_routes(_ptr(h), _ptr(a), _ptr(b), h.numel(), _stream(None)))
    return a, b
