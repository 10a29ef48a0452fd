"""Oracle for the Titans neural long-term memory -- TEST INFRASTRUCTURE ONLY.

Only tests/, the smoke check (``__graft_entry__.smoke``) and bench.py's CPU
baseline leg may import this package. The product (the CUDA library and its
Python binding) never imports it and shares no code with it.

Two fp64 paths, both from the pages on "Titans: Learning to Memorize at Test Time":

* :func:`forward` -- the defining recurrence, token by token, in plain C
  (``titans_oracle.c``): per-token gradients at the chunk-start weights
  (walk-through sec. 3.2, t' = t - mod(t, b)), momentum S_t = eta_t S_{t-1} -
  theta_t grad (sec. 3.1), forgetting W_t = (1 - alpha_t) W_{t-1} + S_t
  (sec. 3.1 "Forgetting Mechanism"), retrieval y_t = M*(q_t) (sec. 3.1
  "Retrieving a Memory").
* :func:`forward_closed_form` -- the same chunk semantics unrolled over one
  chunk (the tensorized mini-batch form of sec. 3.2, extended with momentum):
  every per-token gradient is taken at the chunk-start weights, so the n
  updates of a chunk fold into per-token coefficients c_j, d_j and three
  per-chunk scalars. It is pinned to :func:`forward` by the tests (1e-12) and
  is used where the token loop would take too long.

* :func:`forward_deep` / :func:`forward_deep_closed_form` -- the deep memory
  (walk-through sec. 3.1 "Memory Architecture", L_M >= 2 layers; sec. 5.5):
  M(x) = W_L silu(W_{L-1} ... silu(W_1 x)), every hidden layer h wide, no bias,
  the L layers packed one after another per unit (:func:`deep_shapes`).
* :func:`linear_chunk_map` / :func:`forward_linear_scan` -- for the linear memory
  the chunk update is affine in the row state X = [W | S]: X -> X M_c + N_c, so
  the chunks combine by an associative scan (German summary, "Parallelisiertes
  Training": parallel associative scans; tencent review, the same): segments
  of chunks compose their maps independently, a short scan over the segments
  gives every segment's start state, and each segment then runs its chunks.
* :func:`backward` -- gradients of a scalar loss on the forward's outputs (y and
  the final state) with respect to every input (k, q, v, the gates, the initial
  state), by reverse-mode automatic differentiation in fp64 through the token
  loop written in plain PyTorch ops (the outer loop of training: walk-through
  sec. 3.1, W_K and W_V are outer-loop parameters). Pinned by central finite
  differences of the C token loop.
* :func:`mag_gate` / :func:`forward_gated` -- the gated output of the
  memory-as-a-gate architecture (walk-through sec. 4.2 "Gated Memory": o = y
  (x) M(x~), y the sliding-window attention branch's output; the tencent review's
  MAG bullet names (x) an element-wise product with a non-linear activation).
  Reading taken: o_t = attn_t * sigmoid(M(q_t)) element-wise, the logistic
  function applied to the memory's retrieval, which gates the attention output.

Pins against things other than the oracle itself are in tests/test_oracle_pins.py.
Parity of the oracle on the full-size workloads is "unpinned" beyond those pins:
no page prints a worked numerical example.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import numpy as np

from . import build as _build

_lib = None


def _open(path: str):
    lib = ctypes.CDLL(path)
    f = lib.titans_oracle_forward
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_long, ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_int] + \
        [ctypes.c_void_p] * 11 + [ctypes.c_int]
    lib.titans_oracle_threads.restype = ctypes.c_int
    return _open_deep(lib)


def _open_deep(lib):
    f = lib.titans_oracle_forward_deep
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_long, ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int] + \
        [ctypes.c_void_p] * 9 + [ctypes.c_int]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _open(_build.build())
    return _lib


def forward_from_library(path: str):
    """A forward() bound to another build of titans_oracle.c (used by the mutation tests)."""
    lib = _open(path)

    def fwd(*args, **kw):
        return forward(*args, _lib_override=lib, **kw)
    return fwd


def threads() -> int:
    return _load().titans_oracle_threads()


def _np(x, dtype) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu")
            x = x.to(torch.float64 if dtype == np.float64 else torch.float32).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=dtype))


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def forward(k, q, v, alpha, eta, theta, state: Dict, chunk: int, want_y: bool = True,
            n_threads: int = 0, _lib_override=None):
    """Token-by-token fp64 recurrence.

    k, q, v: [U, T, d]; alpha, eta, theta: [U, T]; state: dict with W1, S1 (and W2, S2 for
    the MLP), each [U, ...]. Returns (y [U, T, d] float64 or None, new state dict float64).
    """
    kf, qf, vf = (_np(x, np.float32) for x in (k, q, v))
    al, et, th = (_np(x, np.float32) for x in (alpha, eta, theta))
    U, T, d = kf.shape
    linear = "W2" not in state
    W1 = _np(state["W1"], np.float64).copy()
    S1 = _np(state["S1"], np.float64).copy()
    W2 = None if linear else _np(state["W2"], np.float64).copy()
    S2 = None if linear else _np(state["S2"], np.float64).copy()
    h = 0 if linear else W1.shape[1]
    y = np.zeros((U, T, d), np.float64) if want_y else None
    lib = _load() if _lib_override is None else _lib_override
    rc = lib.titans_oracle_forward(U, T, d, h, int(chunk), _ptr(kf), _ptr(qf), _ptr(vf),
                                       _ptr(al), _ptr(et), _ptr(th), _ptr(W1), _ptr(W2), _ptr(S1),
                                       _ptr(S2), _ptr(y), int(n_threads))
    if rc != 0:
        raise RuntimeError("oracle: bad arguments or out of memory")
    st = {"W1": W1, "S1": S1}
    if not linear:
        st.update(W2=W2, S2=S2)
    return y, st


def chunk_scalars(alpha: np.ndarray, eta: np.ndarray, theta: np.ndarray):
    """Coefficients of one chunk (last axis = the chunk's tokens, 0-based j = 0..n-1).

    Unrolling S_j = eta_j S_{j-1} - theta_j g_j and W_j = (1 - alpha_j) W_{j-1} + S_j over
    the chunk with every g_j fixed at the chunk-start weights gives
        W_end = A * W_0 + sigma * S_0 - sum_j c_j g_j
        S_end = E * S_0 - sum_j d_j g_j
    with P_j = prod_{l>j} (1 - alpha_l), Q_j = prod_{l>j} eta_l,
         r_{n-1} = 1, r_j = P_j + eta_{j+1} r_{j+1},
         c_j = theta_j r_j, d_j = theta_j Q_j,
         A = (1 - alpha_0) P_0, E = eta_0 Q_0, sigma = eta_0 r_0.
    Division-free; valid for eta = 0 and alpha = 1.
    """
    alpha = np.asarray(alpha, np.float64)
    eta = np.asarray(eta, np.float64)
    theta = np.asarray(theta, np.float64)
    n = alpha.shape[-1]
    P = np.ones_like(alpha)
    Q = np.ones_like(alpha)
    r = np.ones_like(alpha)
    for j in range(n - 2, -1, -1):
        P[..., j] = P[..., j + 1] * (1.0 - alpha[..., j + 1])
        Q[..., j] = Q[..., j + 1] * eta[..., j + 1]
        r[..., j] = P[..., j] + eta[..., j + 1] * r[..., j + 1]
    c = theta * r
    dd = theta * Q
    A = (1.0 - alpha[..., 0]) * P[..., 0]
    E = eta[..., 0] * Q[..., 0]
    sig = eta[..., 0] * r[..., 0]
    return c, dd, A, E, sig


def _silu_parts(Z):
    s = 1.0 / (1.0 + np.exp(-Z))
    return s, Z * s


def forward_closed_form(k, q, v, alpha, eta, theta, state: Dict, chunk: int, want_y: bool = True):
    """Chunk closed form in fp64, batched over units with numpy matmuls. Same arguments as forward."""
    K, Qm, V = (_np(x, np.float64) for x in (k, q, v))
    al, et, th = (_np(x, np.float64) for x in (alpha, eta, theta))
    U, T, d = K.shape
    linear = "W2" not in state
    W1 = _np(state["W1"], np.float64).copy()
    S1 = _np(state["S1"], np.float64).copy()
    if not linear:
        W2 = _np(state["W2"], np.float64).copy()
        S2 = _np(state["S2"], np.float64).copy()
    y = np.zeros((U, T, d), np.float64) if want_y else None
    tr = lambda x: np.swapaxes(x, -1, -2)
    for t0 in range(0, T, chunk):
        t1 = min(t0 + chunk, T)
        Kc, Qc, Vc = K[:, t0:t1], Qm[:, t0:t1], V[:, t0:t1]
        c, dd, A, E, sig = chunk_scalars(al[:, t0:t1], et[:, t0:t1], th[:, t0:t1])
        A, E, sig = A[:, None, None], E[:, None, None], sig[:, None, None]
        if linear:
            Yh = Kc @ tr(W1)
            G = 2.0 * (Yh - Vc)
            if want_y:
                y[:, t0:t1] = Qc @ tr(W1)
            gc = tr(G * c[..., None]) @ Kc
            gd = tr(G * dd[..., None]) @ Kc
            W1, S1 = A * W1 + sig * S1 - gc, E * S1 - gd
            continue
        Z = Kc @ tr(W1)
        s, Ak = _silu_parts(Z)
        Yh = Ak @ tr(W2)
        G = 2.0 * (Yh - Vc)
        Dl = (G @ W2) * (s * (1.0 + Z * (1.0 - s)))
        if want_y:
            _, Aq = _silu_parts(Qc @ tr(W1))
            y[:, t0:t1] = Aq @ tr(W2)
        g2c = tr(G * c[..., None]) @ Ak
        g2d = tr(G * dd[..., None]) @ Ak
        g1c = tr(Dl * c[..., None]) @ Kc
        g1d = tr(Dl * dd[..., None]) @ Kc
        W2, S2 = A * W2 + sig * S2 - g2c, E * S2 - g2d
        W1, S1 = A * W1 + sig * S1 - g1c, E * S1 - g1d
    st = {"W1": W1, "S1": S1}
    if not linear:
        st.update(W2=W2, S2=S2)
    return y, st


def mag_gate(attn, y):
    """o = attn * sigmoid(y), element-wise, in fp64: the attention branch's output `attn` gated by
    the logistic function of the memory's retrieval `y` (walk-through sec. 4.2 "Gated Memory")."""
    a = np.asarray(attn, np.float64)
    yy = np.asarray(y, np.float64)
    with np.errstate(over="ignore"):
        return a / (1.0 + np.exp(-yy))


def forward_gated(k, q, v, alpha, eta, theta, state: Dict, chunk: int, attn, n_threads: int = 0):
    """The token loop of :func:`forward` with the gated output: returns (o [U, T, d] float64, state),
    o_t = mag_gate(attn_t, M(q_t)) with M at the chunk-start weights. attn: [U, T, d]."""
    y, st = forward(k, q, v, alpha, eta, theta, state, chunk, n_threads=n_threads)
    return mag_gate(_np(attn, np.float32), y), st


def deep_shapes(d: int, h: int, layers: int):
    """[out, in] of every layer of the deep memory: W_1 [h, d], W_2 .. W_{L-1} [h, h], W_L [d, h]."""
    return [(h, d)] + [(h, h)] * (layers - 2) + [(d, h)]


def _deep_hidden(P: int, d: int, layers: int) -> int:
    """Hidden width h of a packed deep state of P elements per unit."""
    for h in range(1, 1 << 14):
        n = sum(a * b for a, b in deep_shapes(d, h, layers))
        if n == P:
            return h
        if n > P:
            break
    raise ValueError(f"a packed state of {P} elements per unit fits no {layers}-layer memory of width {d}")


def pack_deep(mats):
    """[U, out, in] per layer -> [U, P], layers one after another (row-major each)."""
    return np.concatenate([np.asarray(m, np.float64).reshape(m.shape[0], -1) for m in mats], axis=1)


def unpack_deep(W, d: int, h: int, layers: int):
    W = np.asarray(W)
    out, o = [], 0
    for (a, b) in deep_shapes(d, h, layers):
        out.append(W[:, o:o + a * b].reshape(W.shape[0], a, b))
        o += a * b
    return out


def forward_deep(k, q, v, alpha, eta, theta, state: Dict, chunk: int, layers: int, want_y: bool = True,
                 n_threads: int = 0, _lib_override=None):
    """Token-by-token fp64 recurrence of the deep memory. state: {"W": [U, P], "S": [U, P]} packed
    (pack_deep). Returns (y [U, T, d] or None, {"W", "S"} float64)."""
    kf, qf, vf = (_np(x, np.float32) for x in (k, q, v))
    al, et, th = (_np(x, np.float32) for x in (alpha, eta, theta))
    U, T, d = kf.shape
    W = _np(state["W"], np.float64).copy()
    S = _np(state["S"], np.float64).copy()
    h = _deep_hidden(W.shape[1], d, layers)
    y = np.zeros((U, T, d), np.float64) if want_y else None
    lib = _load() if _lib_override is None else _open_deep(_lib_override)
    rc = lib.titans_oracle_forward_deep(U, T, d, h, layers, int(chunk), _ptr(kf), _ptr(qf), _ptr(vf), _ptr(al),
                                        _ptr(et), _ptr(th), _ptr(W), _ptr(S), _ptr(y), int(n_threads))
    if rc != 0:
        raise RuntimeError("oracle: bad arguments or out of memory")
    return y, {"W": W, "S": S}


def forward_deep_closed_form(k, q, v, alpha, eta, theta, state: Dict, chunk: int, layers: int, want_y: bool = True):
    """Chunk closed form of the deep memory in fp64 (numpy matmuls), same arguments as forward_deep:
    per chunk every key goes forward through the chunk-start layers, the error 2 (M(k) - v) goes back
    through them, and each layer's c- and d-weighted sums of per-token outer products update W, S."""
    K, Qm, V = (_np(x, np.float64) for x in (k, q, v))
    al, et, th = (_np(x, np.float64) for x in (alpha, eta, theta))
    U, T, d = K.shape
    h = _deep_hidden(_np(state["W"], np.float64).shape[1], d, layers)
    Ws = [w.copy() for w in unpack_deep(_np(state["W"], np.float64), d, h, layers)]
    Ss = [x.copy() for x in unpack_deep(_np(state["S"], np.float64), d, h, layers)]
    y = np.zeros((U, T, d), np.float64) if want_y else None
    tr = lambda x: np.swapaxes(x, -1, -2)

    def fwd(X):
        zs, acts = [], [X]
        for l in range(layers - 1):
            z = acts[-1] @ tr(Ws[l])
            s_, a_ = _silu_parts(z)
            zs.append((z, s_))
            acts.append(a_)
        return zs, acts, acts[-1] @ tr(Ws[-1])

    for t0 in range(0, T, chunk):
        t1 = min(t0 + chunk, T)
        c, dd, A, E, sig = chunk_scalars(al[:, t0:t1], et[:, t0:t1], th[:, t0:t1])
        A, E, sig = A[:, None, None], E[:, None, None], sig[:, None, None]
        if want_y:
            y[:, t0:t1] = fwd(Qm[:, t0:t1])[2]
        zs, acts, out = fwd(K[:, t0:t1])
        delta = 2.0 * (out - V[:, t0:t1])  # dl/d out, then dl/dz of each hidden layer going back
        grads_c, grads_d = [None] * layers, [None] * layers
        for l in range(layers - 1, -1, -1):
            grads_c[l] = tr(delta * c[..., None]) @ acts[l]
            grads_d[l] = tr(delta * dd[..., None]) @ acts[l]
            if l > 0:
                z, s_ = zs[l - 1]
                delta = (delta @ Ws[l]) * (s_ * (1.0 + z * (1.0 - s_)))
        for l in range(layers):
            Ws[l], Ss[l] = A * Ws[l] + sig * Ss[l] - grads_c[l], E * Ss[l] - grads_d[l]
    return y, {"W": pack_deep(Ws), "S": pack_deep(Ss)}


def expand_chunk_gates(g, T: int, chunk: int):
    """Chunk-shared gates [U, ceil(T / chunk)] -> per-token gates [U, T]: every token of chunk c takes
    the chunk's value (walk-through sec. 3.2, "Parameters as the Function of Chunks"). The forward
    with chunk-shared gates is the token loop run on these."""
    g = np.asarray(g, np.float32)
    return np.ascontiguousarray(np.repeat(g, chunk, axis=1)[:, :T])


def linear_chunk_map(K, V, alpha, eta, theta):
    """The affine map of one chunk of the linear memory M(x) = W x on the row state X = [W | S]
    (d x 2d): X' = X M + N with (K, V: [n, d] rows k_j, v_j; C = diag(c), D = diag(d) of the chunk)
        M = [[A I - 2 K^T C K, -2 K^T D K], [sigma I, E I]]   (2d x 2d)
        N = [2 V^T C K, 2 V^T D K]                            (d x 2d)
    from W' = A W + sigma S - sum_j c_j 2 (W k_j - v_j) k_j^T and S' = E S - sum_j d_j 2 (W k_j - v_j) k_j^T."""
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    d = K.shape[1]
    c, dd, A, E, sig = chunk_scalars(alpha, eta, theta)
    I = np.eye(d)
    M = np.block([[A * I - 2.0 * K.T @ (c[:, None] * K), -2.0 * K.T @ (dd[:, None] * K)],
                  [sig * I, E * I]])
    N = np.concatenate([2.0 * V.T @ (c[:, None] * K), 2.0 * V.T @ (dd[:, None] * K)], axis=1)
    return M, N


def forward_linear_scan(k, q, v, alpha, eta, theta, state: Dict, chunk: int, segments: int, tree: bool = False):
    """Linear memory forward by the cross-chunk scan, fp64: the chunk maps of each of `segments`
    segments are composed (tree=True: pairwise, as a parallel scan would), the segment totals are
    scanned to give each segment's start state, and each segment's chunks are then applied in order
    (y_t = W q_t with the chunk-start W). Same arguments and returns as forward() for the linear
    memory."""
    K, Qm, V = (_np(x, np.float64) for x in (k, q, v))
    al, et, th = (_np(x, np.float64) for x in (alpha, eta, theta))
    U, T, d = K.shape
    W = _np(state["W1"], np.float64).copy()
    S = _np(state["S1"], np.float64).copy()
    y = np.zeros((U, T, d))
    nch = (T + chunk - 1) // chunk
    G = (nch + segments - 1) // segments
    bounds = [(s * G, min((s + 1) * G, nch)) for s in range(segments) if s * G < nch]

    def compose(m1, m2):  # apply m1 then m2
        return m1[0] @ m2[0], m1[1] @ m2[0] + m2[1]
    for u in range(U):
        maps = []
        for c in range(nch):
            t0, t1 = c * chunk, min((c + 1) * chunk, T)
            maps.append(linear_chunk_map(K[u, t0:t1], V[u, t0:t1], al[u, t0:t1], et[u, t0:t1], th[u, t0:t1]))
        seg = []
        for c0, c1 in bounds:
            ms = maps[c0:c1]
            if tree:
                while len(ms) > 1:
                    ms = [compose(ms[i], ms[i + 1]) if i + 1 < len(ms) else ms[i] for i in range(0, len(ms), 2)]
                seg.append(ms[0])
            else:
                tot = (np.eye(2 * d), np.zeros((d, 2 * d)))
                for mp in ms:
                    tot = compose(tot, mp)
                seg.append(tot)
        X = np.concatenate([W[u], S[u]], axis=1)
        for (c0, c1), (Ms, Ns) in zip(bounds, seg):
            Xc = X
            for c in range(c0, c1):
                t0, t1 = c * chunk, min((c + 1) * chunk, T)
                y[u, t0:t1] = Qm[u, t0:t1] @ Xc[:, :d].T
                Xc = Xc @ maps[c][0] + maps[c][1]
            X = X @ Ms + Ns
        W[u], S[u] = X[:, :d], X[:, d:]
    return y, {"W1": W, "S1": S}


def _torch_token_loop(k, q, v, alpha, eta, theta, state, chunk):
    """The defining recurrence in fp64 torch ops (differentiable): the same steps as the C token
    loop, with the per-token gradient written out (linear: 2 (W k - v) k^T; MLP: the chain rule)."""
    import torch
    U, T, d = k.shape
    linear = "W2" not in state
    W1, S1 = state["W1"], state["S1"]
    W2, S2 = (None, None) if linear else (state["W2"], state["S2"])
    ys = []
    for t in range(T):
        if t % chunk == 0:
            W1b, W2b = W1, W2
        kt, qt, vt = k[:, t], q[:, t], v[:, t]
        if linear:
            ys.append(torch.einsum("uij,uj->ui", W1b, qt))
            e = 2.0 * (torch.einsum("uij,uj->ui", W1b, kt) - vt)
            g1 = e[:, :, None] * kt[:, None, :]
        else:
            zq = torch.einsum("uij,uj->ui", W1b, qt)
            ys.append(torch.einsum("uij,uj->ui", W2b, zq * torch.sigmoid(zq)))
            z = torch.einsum("uij,uj->ui", W1b, kt)
            s_ = torch.sigmoid(z)
            a = z * s_
            e = 2.0 * (torch.einsum("uij,uj->ui", W2b, a) - vt)
            g2 = e[:, :, None] * a[:, None, :]
            delta = torch.einsum("uij,ui->uj", W2b, e) * s_ * (1.0 + z * (1.0 - s_))
            g1 = delta[:, :, None] * kt[:, None, :]
        at, et_, tt = alpha[:, t, None, None], eta[:, t, None, None], theta[:, t, None, None]
        S1 = et_ * S1 - tt * g1
        W1 = (1.0 - at) * W1 + S1
        if not linear:
            S2 = et_ * S2 - tt * g2
            W2 = (1.0 - at) * W2 + S2
    out = {"W1": W1, "S1": S1}
    if not linear:
        out.update(W2=W2, S2=S2)
    return torch.stack(ys, 1), out


def backward(k, q, v, alpha, eta, theta, state: Dict, chunk: int, dy, dstate: Dict):
    """Gradients of L = <dy, y> + sum_n <dstate[n], final state[n]> with respect to k, q, v, alpha,
    eta, theta and the initial state, in fp64 (reverse mode through the token loop). Returns a dict
    with keys k, q, v, alpha, eta, theta and the state's names (W1, S1, W2, S2)."""
    import torch
    f64 = lambda x: torch.as_tensor(np.asarray(_np(x, np.float64)), dtype=torch.float64).clone().requires_grad_(True)
    ins = {n: f64(x) for n, x in (("k", k), ("q", q), ("v", v), ("alpha", alpha), ("eta", eta), ("theta", theta))}
    st = {n: f64(x) for n, x in state.items()}
    y, out = _torch_token_loop(ins["k"], ins["q"], ins["v"], ins["alpha"], ins["eta"], ins["theta"], st, chunk)
    L = (y * torch.as_tensor(_np(dy, np.float64))).sum()
    for n, g in dstate.items():
        L = L + (out[n] * torch.as_tensor(_np(g, np.float64))).sum()
    L.backward()
    # an input the loss does not depend on (e.g. the initial momentum when only the first chunk's y
    # is scored) has no .grad: its gradient is zero
    g = lambda x: x.grad.numpy() if x.grad is not None else np.zeros(tuple(x.shape))
    grads = {n: g(x) for n, x in ins.items()}
    grads.update({n: g(x) for n, x in st.items()})
    return grads
