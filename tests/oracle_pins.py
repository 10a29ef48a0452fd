"""Pins for the oracle: checks against what the pages and the mathematics fix.

Each pin takes a ``fwd`` callable with the signature of ``oracle.forward`` and
raises AssertionError on a mismatch. tests/test_oracle_pins.py runs them on the
oracle; tests/test_oracle_mutants.py runs them on deliberately broken copies of
the oracle's C source and requires every copy to fail at least one pin.

Sources (pages on "Titans: Learning to Memorize at Test Time"):
  walk-through sec. 3.1 (loss, momentum, forgetting, linear memory = online
  linear regression, retrieval without update), sec. 3.2 (chunk-start
  gradients t' = t - mod(t, b); the eta = 0 tensorized form with Theta_b and
  B_b built from beta_i = prod (1 - alpha_j)); blog sec. 3.1 (MLP memory
  W2 sigma(W1 .)).
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))


def _rng(seed):
    return np.random.default_rng(seed)


def _l2n(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _mk(U, T, d, h, seed, alpha=None, eta=None, theta=None, W0_scale=1.0):
    """Random fp32-exact inputs (values are float32 so both sides see identical numbers)."""
    r = _rng(seed)
    f = lambda *s: r.standard_normal(s).astype(np.float32)
    k = _l2n(f(U, T, d)).astype(np.float32)
    q = _l2n(f(U, T, d)).astype(np.float32)
    v = f(U, T, d)
    al = (r.uniform(0, 0.05, (U, T)) if alpha is None else np.broadcast_to(alpha, (U, T))).astype(np.float32)
    et = (r.uniform(0.8, 0.99, (U, T)) if eta is None else np.broadcast_to(eta, (U, T))).astype(np.float32)
    th = (r.uniform(0, 0.1, (U, T)) if theta is None else np.broadcast_to(theta, (U, T))).astype(np.float32)
    if h == 0:
        st = {"W1": (W0_scale * r.standard_normal((U, d, d)) / np.sqrt(d)), "S1": np.zeros((U, d, d))}
    else:
        st = {"W1": W0_scale * r.standard_normal((U, h, d)) / np.sqrt(d),
              "W2": W0_scale * r.standard_normal((U, d, h)) / np.sqrt(h),
              "S1": np.zeros((U, h, d)), "S2": np.zeros((U, d, h))}
    st = {n: x.astype(np.float32).astype(np.float64) for n, x in st.items()}
    return k, q, v, np.ascontiguousarray(al), np.ascontiguousarray(et), np.ascontiguousarray(th), st


def _close(a, b, tol, what):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    scale = max(np.abs(b).max(), 1e-300)
    err = np.abs(a - b).max() / scale
    assert err <= tol, f"{what}: rel err {err:.3e} > {tol:.1e}"


# ---------------------------------------------------------------- golden (by hand)

def pin_hand_worked_d1(fwd):
    """Hand-computed linear d=1 example (tests/golden/linear_d1_hand.json), exact fractions."""
    g = json.load(open(os.path.join(HERE, "golden", "linear_d1_hand.json")))
    one = np.ones((1, 3, 1), np.float32)
    for case in g["cases"]:
        y, st = fwd(one, one, one, np.full((1, 3), 0.5, np.float32), np.full((1, 3), 0.5, np.float32),
                    np.full((1, 3), 0.25, np.float32), {"W1": np.zeros((1, 1, 1)), "S1": np.zeros((1, 1, 1))},
                    case["chunk"])
        assert np.array_equal(y.ravel(), np.array(case["y"])), (case, y.ravel())
        assert st["W1"].item() == case["W"] and st["S1"].item() == case["S"], (case, st)


# ------------------------------------------------------- linear memory = regression

def pin_orthonormal_exact_write(fwd):
    """Linear memory, alpha = eta = 0, theta = 1/2: one gradient step on ||W k - v||^2 with a
    unit key writes the pair exactly (W k = v), and steps on mutually orthogonal keys do not
    disturb each other. Holds for chunk = 1 and for all keys in one chunk."""
    d = 8
    r = _rng(1)
    Kq, _ = np.linalg.qr(r.standard_normal((d, d)))
    K = Kq.T.astype(np.float32)  # rows orthonormal (to fp32 rounding; re-orthonormalise below)
    K = np.linalg.qr(K.astype(np.float64).T)[0].T
    K32 = K.astype(np.float32)
    V = r.standard_normal((d, d)).astype(np.float32)
    for chunk in (1, d):
        y, st = fwd(K32[None], K32[None], V[None], np.zeros((1, d), np.float32), np.zeros((1, d), np.float32),
                    np.full((1, d), 0.5, np.float32), {"W1": np.zeros((1, d, d)), "S1": np.zeros((1, d, d))}, chunk)
        W = st["W1"][0]
        _close(K32.astype(np.float64) @ W.T, V, 1e-6, f"W k_i = v_i (chunk={chunk})")


def pin_lms_batch_form(fwd):
    """alpha = eta = 0, one chunk: the batched delta rule (LMS) in matrix form,
    W_n = Wbar - 2 sum_j theta_j (Wbar k_j - v_j) k_j^T = Wbar (I - 2 K^T Theta K) + 2 V^T Theta K."""
    d, n = 6, 5
    k, q, v, al, et, th, st = _mk(1, n, d, 0, 2, alpha=0.0, eta=0.0)
    _, out = fwd(k, q, v, al, et, th, st, n)
    K, V, Th, Wb = k[0].astype(np.float64), v[0].astype(np.float64), np.diag(th[0].astype(np.float64)), st["W1"][0]
    Wn = Wb @ (np.eye(d) - 2 * K.T @ Th @ K) + 2 * V.T @ Th @ K
    _close(out["W1"][0], Wn, 1e-12, "LMS batch form")


def pin_eta0_tensorized(fwd):
    """eta = 0: W_n = beta_n W_0 - sum_j theta_j (beta_n / beta_j) grad_j(W_0), the tensorized
    mini-batch form Theta_b B_b (...) of sec. 3.2 with beta_i = prod_{l<=i} (1 - alpha_l)."""
    d, n = 5, 7
    k, q, v, al, et, th, st = _mk(1, n, d, 0, 3, eta=0.0)
    _, out = fwd(k, q, v, al, et, th, st, n)
    K, V, W0 = k[0].astype(np.float64), v[0].astype(np.float64), st["W1"][0]
    beta = np.cumprod(1.0 - al[0].astype(np.float64))
    G = 2.0 * (K @ W0.T - V)  # row j: 2 (W0 k_j - v_j)
    acc = sum(th[0, j] * beta[-1] / beta[j] * np.outer(G[j], K[j]) for j in range(n))
    _close(out["W1"][0], beta[-1] * W0 - acc, 1e-12, "eta=0 tensorized form")


# ---------------------------------------------------------------- momentum, decay

def pin_geometric_impulse(fwd):
    """Only the first token writes (theta_t = 0 for t > 1), alpha and eta constant, S_0 = 0:
    S_T = -theta_1 eta^{T-1} g and W_T = (1-alpha)^T W_0 - theta_1 g ((1-alpha)^T - eta^T) / ((1-alpha) - eta),
    a geometric series; g is the first token's gradient at W_0, taken here with torch autograd."""
    for h in (0, 6):
        d, T = 4, 9
        a, e = 0.125, 0.5
        th = np.zeros((1, T), np.float32)
        th[0, 0] = 0.25
        k, q, v, al, et, _, st = _mk(1, T, d, h, 4, alpha=a, eta=e)
        _, out = fwd(k, q, v, al, et, th, st, T)
        grads = _autograd_grad(st, k[0, 0], v[0, 0])
        geo = ((1 - a) ** T - e ** T) / ((1 - a) - e)
        for name, g in grads.items():
            W0 = st[name][0]
            _close(out[name][0], (1 - a) ** T * W0 - 0.25 * g * geo, 1e-12, f"impulse {name} (h={h})")
            _close(out["S" + name[1]][0], -0.25 * e ** (T - 1) * g, 1e-12, f"impulse S (h={h})")


def pin_pure_decay(fwd):
    """theta = 0, S_0 = 0: W_T = prod(1 - alpha_t) W_0, S stays 0, and each chunk's retrieval
    uses the decayed chunk-start weights (y via torch.nn.functional on the scaled weights)."""
    for h in (0, 12):
        d, T, n = 6, 20, 6
        k, q, v, al, et, th, st = _mk(1, T, d, h, 5, theta=0.0)
        y, out = fwd(k, q, v, al, et, th, st, n)
        beta = np.cumprod(np.concatenate([[1.0], 1.0 - al[0].astype(np.float64)]))
        for name in ("W1", "W2") if h else ("W1",):
            _close(out[name][0], beta[T] * st[name][0], 1e-12, f"decay {name}")
            assert not np.any(out["S" + name[1]]), "S must stay 0"
        for t in range(T):
            sc = beta[(t // n) * n]
            ref = _torch_memory({nm: sc * st[nm][0] for nm in st if nm.startswith("W")}, q[0, t])
            _close(y[0, t], ref, 1e-12, f"decay y[{t}]")


def pin_reset(fwd):
    """alpha = 1, eta = 0, theta = 0 on the last token of a chunk empties W and S. Linear: the rest
    of the sequence equals a fresh run from W = S = 0. MLP: W = 0 is a fixed point (silu(0) = 0,
    every gradient vanishes), so every later retrieval is exactly 0 and the state stays 0."""
    d, T, n, cut = 5, 24, 4, 12
    for h in (0, 7):
        k, q, v, al, et, th, st = _mk(1, T, d, h, 6)
        al[0, cut - 1], et[0, cut - 1], th[0, cut - 1] = 1.0, 0.0, 0.0
        y, out = fwd(k, q, v, al, et, th, st, n)
        if h == 0:
            zero = {nm: np.zeros_like(x) for nm, x in st.items()}
            y2, out2 = fwd(k[:, cut:], q[:, cut:], v[:, cut:], al[:, cut:], et[:, cut:], th[:, cut:], zero, n)
            assert np.array_equal(y[:, cut:], y2) and all(np.array_equal(out[nm], out2[nm]) for nm in out)
        else:
            assert not np.any(y[:, cut:]) and not any(np.any(x) for x in out.values())


# ---------------------------------------------------------------- gradients

def _torch_memory(Ws, x):
    x = torch.as_tensor(np.asarray(x, np.float64))
    W1 = torch.as_tensor(Ws["W1"])
    if "W2" not in Ws:
        return torch.nn.functional.linear(x, W1).numpy()
    return torch.nn.functional.linear(torch.nn.functional.silu(torch.nn.functional.linear(x, W1)),
                                      torch.as_tensor(Ws["W2"])).numpy()


def _autograd_grad(st, k, v):
    """Gradient of ||M(k) - v||^2 in fp64 by torch autograd (library routine)."""
    Ws = {n: torch.tensor(st[n][0], dtype=torch.float64, requires_grad=True) for n in st if n.startswith("W")}
    x = torch.as_tensor(np.asarray(k, np.float64))
    if "W2" in Ws:
        out = torch.nn.functional.linear(torch.nn.functional.silu(torch.nn.functional.linear(x, Ws["W1"])), Ws["W2"])
    else:
        out = torch.nn.functional.linear(x, Ws["W1"])
    loss = ((out - torch.as_tensor(np.asarray(v, np.float64))) ** 2).sum()
    loss.backward()
    return {n: W.grad.numpy() for n, W in Ws.items()}


def pin_gradient_autograd(fwd):
    """One token, S_0 = 0, alpha = 0, theta = 1: S_1 = -g and W_1 = W_0 - g, so the oracle's
    per-token gradient is W_0 - W_1; it must equal torch autograd of ||M(k) - v||^2 (fp64)."""
    for h, d in ((0, 5), (9, 4), (16, 8)):
        k, q, v, al, et, th, st = _mk(1, 1, d, h, 7 + h, alpha=0.0, eta=0.5, theta=1.0, W0_scale=2.0)
        _, out = fwd(k, q, v, al, et, th, st, 1)
        g = _autograd_grad(st, k[0, 0], v[0, 0])
        for name in g:
            _close(st[name][0] - out[name][0], g[name], 1e-12, f"grad {name} (h={h})")
            _close(-out["S" + name[1]][0], g[name], 1e-12, f"S=-g {name} (h={h})")


def pin_gradient_finite_difference(fwd):
    """Same single-token read-out of the gradient, against central finite differences of the
    loss (step 1e-6, fp64) on a tiny MLP; the loss is evaluated with torch.nn.functional."""
    d, h = 3, 5
    k, q, v, al, et, th, st = _mk(1, 1, d, h, 11, alpha=0.0, eta=0.0, theta=1.0, W0_scale=2.0)
    _, out = fwd(k, q, v, al, et, th, st, 1)

    def loss(Ws):
        return float(((_torch_memory(Ws, k[0, 0]) - v[0, 0].astype(np.float64)) ** 2).sum())
    eps = 1e-6
    for name in ("W1", "W2"):
        W = {n: st[n][0].copy() for n in ("W1", "W2")}
        fd = np.zeros_like(W[name])
        for idx in np.ndindex(*W[name].shape):
            Wp = {n: x.copy() for n, x in W.items()}
            Wm = {n: x.copy() for n, x in W.items()}
            Wp[name][idx] += eps
            Wm[name][idx] -= eps
            fd[idx] = (loss(Wp) - loss(Wm)) / (2 * eps)
        _close(st[name][0] - out[name][0], fd, 1e-7, f"finite differences {name}")


def pin_autograd_recurrence(fwd):
    """Brute force on tiny inputs: the pages' update (sec. 3.1) driven by torch-autograd
    gradients taken at the chunk-start weights (sec. 3.2), y from torch.nn.functional."""
    d, h, T = 4, 8, 13
    for chunk in (1, 4, 5):
        k, q, v, al, et, th, st = _mk(2, T, d, h, 13 + chunk)
        y, out = fwd(k, q, v, al, et, th, st, chunk)
        for u in range(2):
            W = {n: st[n][u].copy() for n in ("W1", "W2")}
            S = {n: np.zeros_like(W[n]) for n in W}
            for t in range(T):
                if t % chunk == 0:
                    Wbar = {n: x.copy() for n, x in W.items()}
                _close(y[u, t], _torch_memory(Wbar, q[u, t]), 1e-12, f"brute y[{u},{t}]")
                g = _autograd_grad({n: x[None] for n, x in Wbar.items()}, k[u, t], v[u, t])
                for n in W:
                    S[n] = float(et[u, t]) * S[n] - float(th[u, t]) * g[n]
                    W[n] = (1.0 - float(al[u, t])) * W[n] + S[n]
            for n in W:
                _close(out[n][u], W[n], 1e-12, f"brute {n} chunk={chunk}")
                _close(out["S" + n[1]][u], S[n], 1e-12, f"brute S chunk={chunk}")


# ---------------------------------------------------------------- invariants

def pin_first_chunk_reads_initial_weights(fwd):
    """Every token of the first chunk retrieves with W_0: y_t = W2 silu(W1 q_t) (torch.nn.functional)."""
    d, h, n = 6, 10, 8
    k, q, v, al, et, th, st = _mk(1, 20, d, h, 17)
    y, _ = fwd(k, q, v, al, et, th, st, n)
    for t in range(n):
        _close(y[0, t], _torch_memory({nm: st[nm][0] for nm in ("W1", "W2")}, q[0, t]), 1e-12, f"y[{t}]")


def pin_retrieval_purity(fwd):
    """Retrieval does not write: the final state does not depend on the queries (bitwise)."""
    d, h, T, n = 5, 9, 17, 4
    k, q, v, al, et, th, st = _mk(1, T, d, h, 19)
    _, a = fwd(k, q, v, al, et, th, st, n)
    _, b = fwd(k, k.copy(), v, al, et, th, st, n)
    assert all(np.array_equal(a[nm], b[nm]) for nm in a)


def pin_continuity(fwd):
    """forward(T1) then forward(T2) from its final state == forward(T1 + T2), T1 % chunk == 0 (bitwise)."""
    d, h, T, n, T1 = 5, 9, 22, 4, 12
    k, q, v, al, et, th, st = _mk(1, T, d, h, 23)
    y, full = fwd(k, q, v, al, et, th, st, n)
    y1, mid = fwd(k[:, :T1], q[:, :T1], v[:, :T1], al[:, :T1], et[:, :T1], th[:, :T1], st, n)
    y2, end = fwd(k[:, T1:], q[:, T1:], v[:, T1:], al[:, T1:], et[:, T1:], th[:, T1:], mid, n)
    assert np.array_equal(np.concatenate([y1, y2], 1), y)
    assert all(np.array_equal(full[nm], end[nm]) for nm in full)


def pin_unit_equivariance(fwd):
    """Units are independent: permuting (batch, head) units permutes every output (bitwise)."""
    d, h, T, n = 4, 6, 10, 3
    k, q, v, al, et, th, st = _mk(4, T, d, h, 29)
    p = np.array([2, 0, 3, 1])
    y, a = fwd(k, q, v, al, et, th, st, n)
    y2, b = fwd(k[p], q[p], v[p], al[p], et[p], th[p], {nm: x[p] for nm, x in st.items()}, n)
    assert np.array_equal(y[p], y2) and all(np.array_equal(a[nm][p], b[nm]) for nm in a)


def pin_sign_symmetry(fwd):
    """The loss ||W2 a - v||^2 is unchanged by (W2, v) -> (-W2, -v): the error e flips sign, the
    W2 gradient 2 e a^T flips sign, and the W1 gradient (W2^T 2e) * silu' k^T does not. So negating
    W2, S2 and v negates y, W2 and S2 and leaves W1 and S1 unchanged (bitwise: only negations)."""
    d, h, T, n = 5, 8, 19, 4
    k, q, v, al, et, th, st = _mk(1, T, d, h, 31)
    st["S1"] = 0.01 * st["W1"][::-1].copy()
    st["S2"] = 0.01 * st["W2"][::-1].copy()
    y, a = fwd(k, q, v, al, et, th, st, n)
    neg = dict(st, W2=-st["W2"], S2=-st["S2"])
    y2, b = fwd(k, q, -v, al, et, th, neg, n)
    assert np.array_equal(y2, -y)
    assert np.array_equal(b["W1"], a["W1"]) and np.array_equal(b["S1"], a["S1"])
    assert np.array_equal(b["W2"], -a["W2"]) and np.array_equal(b["S2"], -a["S2"])


def pin_zero_w2_first_chunk(fwd):
    """W2_0 = 0, S_0 = 0: the memory outputs 0, so within the first chunk every W1 gradient
    vanishes and every W2 gradient is 2 (0 - v_j) a_j^T with a_j = silu(W1_0 k_j). Unrolling
    S_t = eta_t S_{t-1} - theta_t g_t, W_t = (1 - alpha_t) W_{t-1} + S_t by hand over the chunk:
      W2_n = sum_j c_j 2 v_j a_j^T,  S2_n = sum_j d_j 2 v_j a_j^T,  W1_n = prod_l (1 - alpha_l) W1_0,
    with c_j = theta_j sum_{m >= j} prod_{j < l <= m} eta_l prod_{l > m} (1 - alpha_l) and
    d_j = theta_j prod_{l > j} eta_l, evaluated here by nested loops; y = 0 in the chunk."""
    d, h, n = 4, 7, 6
    k, q, v, al, et, th, st = _mk(1, n, d, h, 37)
    st["W2"][:] = 0.0
    y, out = fwd(k, q, v, al, et, th, st, n)
    assert not np.any(y)
    W1 = st["W1"][0]
    a = [torch.nn.functional.silu(torch.tensor(W1 @ k[0, j].astype(np.float64))).numpy() for j in range(n)]
    al64, et64, th64 = (x[0].astype(np.float64) for x in (al, et, th))
    W2n = np.zeros((d, h))
    S2n = np.zeros((d, h))
    for j in range(n):
        c = 0.0
        for m in range(j, n):
            term = 1.0
            for l in range(j + 1, m + 1):
                term *= et64[l]
            for l in range(m + 1, n):
                term *= 1.0 - al64[l]
            c += term
        dj = 1.0
        for l in range(j + 1, n):
            dj *= et64[l]
        outer = 2.0 * np.outer(v[0, j].astype(np.float64), a[j])
        W2n += th64[j] * c * outer
        S2n += th64[j] * dj * outer
    _close(out["W2"][0], W2n, 1e-12, "W2 after the first chunk")
    _close(out["S2"][0], S2n, 1e-12, "S2 after the first chunk")
    _close(out["W1"][0], np.prod(1.0 - al64) * W1, 1e-12, "W1 (pure decay)")
    assert not np.any(out["S1"])


PINS = [v for k_, v in sorted(globals().items()) if k_.startswith("pin_")]
