"""Pins of the backward oracle (CPU only): its gradients against central finite differences of the
scalar loss computed by the C token loop (a separate implementation of the forward), on tiny shapes,
for the linear and the MLP memory, with momentum, forgetting and a ragged last chunk."""
import numpy as np
import pytest

import oracle
from oracle_pins import _mk


def _loss(k, q, v, al, et, th, st, chunk, dy, dst):
    y, out = oracle.forward(k, q, v, al, et, th, st, chunk)
    return float((y * dy).sum() + sum((out[n] * dst[n]).sum() for n in dst))


@pytest.mark.parametrize("h,chunk", [(0, 2), (0, 3), (5, 2), (5, 4)])
def test_backward_matches_finite_differences(h, chunk):
    d, T, U = 3, 7, 2
    k, q, v, al, et, th, st = _mk(U, T, d, h, 90 + h + chunk)
    r = np.random.default_rng(91)
    dy = r.standard_normal((U, T, d))
    dst = {n: r.standard_normal(x.shape) for n, x in st.items()}
    g = oracle.backward(k, q, v, al, et, th, st, chunk, dy, dst)
    # inputs are float32 for the C oracle: perturb in float64 copies and pass them through
    base = {"k": k.astype(np.float64), "q": q.astype(np.float64), "v": v.astype(np.float64),
            "alpha": al.astype(np.float64), "eta": et.astype(np.float64), "theta": th.astype(np.float64)}
    base.update({n: x.copy() for n, x in st.items()})
    names = ["k", "q", "v", "alpha", "eta", "theta"] + list(st)

    def L(vals):
        stv = {n: vals[n] for n in st}
        # the C oracle rounds its token inputs to float32: keep perturbations representable
        return _loss(*(vals[n] for n in names[:6]), stv, chunk, dy, dst)
    eps = 1e-3
    for n in names:
        x = base[n]
        flat = x.reshape(-1)
        idx = np.random.default_rng(7).choice(flat.size, size=min(12, flat.size), replace=False)
        for i in idx:
            vals = {m: base[m].copy() for m in names}
            vp, vm = vals[n].reshape(-1), None
            vp[i] += eps
            lp = L(vals)
            vals[n].reshape(-1)[i] -= 2 * eps
            lm = L(vals)
            fd = (lp - lm) / (2 * eps)
            ad = g[n].reshape(-1)[i]
            scale = max(1.0, np.abs(g[n]).max())
            assert abs(fd - ad) <= 2e-4 * scale, f"{n}[{i}]: autograd {ad:.6e} vs finite differences {fd:.6e}"


def test_backward_of_a_frozen_memory():
    """theta = 0 and S0 = 0: the memory never changes (W_t = beta_t W0), so k and v get no gradient
    and the queries' gradient is W_c^T dy (linear memory, chunk-start W = beta W0)."""
    d, T, U, chunk = 4, 8, 1, 4
    k, q, v, al, et, th, st = _mk(U, T, d, 0, 95, theta=0.0)
    dy = np.random.default_rng(3).standard_normal((U, T, d))
    g = oracle.backward(k, q, v, al, et, th, st, chunk, dy, {})
    assert np.abs(g["k"]).max() == 0 and np.abs(g["v"]).max() == 0
    beta = np.concatenate([[1.0], np.cumprod(1.0 - al[0].astype(np.float64))])
    for t in range(T):
        Wc = beta[(t // chunk) * chunk] * st["W1"][0]
        np.testing.assert_allclose(g["q"][0, t], Wc.T @ dy[0, t], rtol=1e-12, atol=1e-14)


def test_backward_of_an_input_the_loss_ignores_is_zero():
    """One chunk, loss on y only: y reads the initial weights, never the initial momentum, so the
    momentum's gradient is exactly zero (returned as zeros, not missing)."""
    k, q, v, al, et, th, st = _mk(1, 6, 3, 4, 97)
    dy = np.random.default_rng(5).standard_normal((1, 6, 3))
    g = oracle.backward(k, q, v, al, et, th, st, 6, dy, {})
    assert g["S1"].shape == st["S1"].shape and not g["S1"].any() and not g["S2"].any()
    assert np.abs(g["W1"]).max() > 0
