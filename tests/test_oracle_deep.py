"""Pins of the deep-memory oracle (CPU only): M(x) = W_L silu(W_{L-1} ... silu(W_1 x)), L >= 2
layers (walk-through sec. 3.1 "Memory Architecture"; sec. 5.5 "The Effect of Deep Memory").

Each pin takes a ``fwd`` with the signature of ``oracle.forward_deep`` and checks it against
something other than itself: torch fp64 autograd, central finite differences, a brute-force torch
recurrence, the W = 0 fixed point, a direct forward pass, and the 2-layer oracle at L = 2.
Plausible mistakes planted in copies of the C source must each fail at least one pin."""
import numpy as np
import pytest
import torch

import oracle
from oracle import build as obuild
from oracle_pins import _mk

D, H = 4, 8


def _deep_state(U, d, h, L, seed, scale=1.0):
    r = np.random.default_rng(seed)
    mats = [scale * r.standard_normal((U,) + sh) / np.sqrt(sh[1]) for sh in oracle.deep_shapes(d, h, L)]
    mats = [m.astype(np.float32).astype(np.float64) for m in mats]
    W = oracle.pack_deep(mats)
    return {"W": W, "S": np.zeros_like(W)}


def _torch_mlp(Ws, x):
    a = x
    for W in Ws[:-1]:
        a = torch.nn.functional.silu(a @ W.T)
    return a @ Ws[-1].T


def pin_autograd_gradient(fwd, L=3):
    """One token, chunk 1, alpha = eta = 0, theta = 1, S0 = 0: W_1 = W_0 - grad l(W_0)."""
    k, q, v, _, _, _, _ = _mk(2, 1, D, H, 11)
    st = _deep_state(2, D, H, L, 12)
    zero = np.zeros((2, 1), np.float32)
    _, out = fwd(k, q, v, zero, zero, np.ones((2, 1), np.float32), st, 1, L)
    g = st["W"] - out["W"]
    for u in range(2):
        Ws = [torch.tensor(m[u], dtype=torch.float64, requires_grad=True)
              for m in oracle.unpack_deep(st["W"], D, H, L)]
        loss = ((_torch_mlp(Ws, torch.tensor(k[u, 0], dtype=torch.float64)) -
                 torch.tensor(v[u, 0], dtype=torch.float64)) ** 2).sum()
        loss.backward()
        ref = np.concatenate([W.grad.numpy().ravel() for W in Ws])
        assert np.abs(g[u] - ref).max() <= 1e-12 * np.abs(ref).max(), f"autograd L={L}"


def pin_finite_differences(fwd, L=3):
    """The same one-token gradient against central differences of the loss (step 1e-6)."""
    k, q, v, _, _, _, _ = _mk(1, 1, D, H, 21)
    st = _deep_state(1, D, H, L, 22)
    zero = np.zeros((1, 1), np.float32)
    _, out = fwd(k, q, v, zero, zero, np.ones((1, 1), np.float32), st, 1, L)
    g = (st["W"] - out["W"])[0]
    W0 = st["W"][0]

    def loss(w):
        Ws = [torch.tensor(m[0], dtype=torch.float64) for m in oracle.unpack_deep(w[None], D, H, L)]
        return float(((_torch_mlp(Ws, torch.tensor(k[0, 0], dtype=torch.float64)) -
                       torch.tensor(v[0, 0], dtype=torch.float64)) ** 2).sum())
    eps = 1e-6
    fd = np.empty_like(W0)
    for i in range(W0.size):
        e = np.zeros_like(W0)
        e[i] = eps
        fd[i] = (loss(W0 + e) - loss(W0 - e)) / (2 * eps)
    assert np.abs(g - fd).max() <= 1e-6 * np.abs(fd).max(), f"finite differences L={L}"


def pin_brute_force_recurrence(fwd, L=3):
    """Momentum and forgetting over chunks of 1, 3 and 5 tokens: a torch loop that takes every
    token's gradient by autograd at the chunk-start weights."""
    T = 11
    k, q, v, al, et, th, _ = _mk(2, T, D, H, 31)
    st = _deep_state(2, D, H, L, 32)
    for chunk in (1, 3, 5):
        y, out = fwd(k, q, v, al, et, th, st, chunk, L)
        for u in range(2):
            Ws = [torch.tensor(m[u], dtype=torch.float64) for m in oracle.unpack_deep(st["W"], D, H, L)]
            Ss = [torch.zeros_like(W) for W in Ws]
            ys = []
            for t in range(T):
                if t % chunk == 0:
                    Wbar = [W.clone() for W in Ws]
                ys.append(_torch_mlp(Wbar, torch.tensor(q[u, t], dtype=torch.float64)))
                wg = [W.clone().requires_grad_(True) for W in Wbar]
                loss = ((_torch_mlp(wg, torch.tensor(k[u, t], dtype=torch.float64)) -
                         torch.tensor(v[u, t], dtype=torch.float64)) ** 2).sum()
                loss.backward()
                for i in range(L):
                    Ss[i] = float(et[u, t]) * Ss[i] - float(th[u, t]) * wg[i].grad
                    Ws[i] = (1.0 - float(al[u, t])) * Ws[i] + Ss[i]
            ry = torch.stack(ys).numpy()
            assert np.abs(y[u] - ry).max() <= 1e-12 * np.abs(ry).max(), f"brute force y chunk={chunk}"
            rw = np.concatenate([W.numpy().ravel() for W in Ws])
            rs = np.concatenate([S.numpy().ravel() for S in Ss])
            assert np.abs(out["W"][u] - rw).max() <= 1e-12 * np.abs(rw).max(), f"brute force W chunk={chunk}"
            assert np.abs(out["S"][u] - rs).max() <= 1e-12 * np.abs(rs).max(), f"brute force S chunk={chunk}"


def pin_reset_fixed_point(fwd, L=3):
    """alpha = 1, eta = 0, theta = 0 on the last token of a chunk: W = S = 0, a fixed point of any
    deep SiLU memory (every activation is 0), so every later retrieval and the final state are 0."""
    k, q, v, al, et, th, _ = _mk(2, 24, D, H, 41)
    al[:, 7], et[:, 7], th[:, 7] = 1.0, 0.0, 0.0
    st = _deep_state(2, D, H, L, 42)
    y, out = fwd(k, q, v, al, et, th, st, 4, L)
    assert not y[:, 8:].any() and not out["W"].any() and not out["S"].any(), "reset"
    assert np.abs(y[:, :8]).max() > 0


def pin_first_chunk_retrieval(fwd, L=4):
    """Tokens of the first chunk read the initial weights: y_t = M(q_t; W0) exactly."""
    k, q, v, al, et, th, _ = _mk(2, 9, D, H, 51)
    st = _deep_state(2, D, H, L, 52)
    y, _ = fwd(k, q, v, al, et, th, st, 9, L)
    for u in range(2):
        Ws = [torch.tensor(m[u], dtype=torch.float64) for m in oracle.unpack_deep(st["W"], D, H, L)]
        ry = _torch_mlp(Ws, torch.tensor(q[u], dtype=torch.float64)).numpy()
        assert np.abs(y[u] - ry).max() <= 1e-13 * np.abs(ry).max(), "first chunk"


DEEP_PINS = [pin_autograd_gradient, pin_finite_differences, pin_brute_force_recurrence, pin_reset_fixed_point,
             pin_first_chunk_retrieval]


@pytest.mark.parametrize("pin", DEEP_PINS, ids=lambda p: p.__name__)
def test_deep_pin(pin):
    pin(oracle.forward_deep)


@pytest.mark.parametrize("L", [3, 4])
def test_deep_pins_at_four_layers_too(L):
    pin_autograd_gradient(oracle.forward_deep, L)
    pin_reset_fixed_point(oracle.forward_deep, L)


def test_two_layers_equal_the_two_layer_oracle():
    """At L = 2 the deep recurrence is the 2-layer memory: both C paths agree bit for bit."""
    k, q, v, al, et, th, st = _mk(3, 37, 5, 12, 9)
    y2, s2 = oracle.forward(k, q, v, al, et, th, st, 6)
    packed = {"W": oracle.pack_deep([st["W1"], st["W2"]]), "S": oracle.pack_deep([st["S1"], st["S2"]])}
    yd, sd = oracle.forward_deep(k, q, v, al, et, th, packed, 6, 2)
    assert np.array_equal(yd, y2)
    assert np.array_equal(sd["W"], oracle.pack_deep([s2["W1"], s2["W2"]]))
    assert np.array_equal(sd["S"], oracle.pack_deep([s2["S1"], s2["S2"]]))


@pytest.mark.parametrize("L,chunk,T", [(3, 7, 37), (4, 5, 23), (3, 1, 9), (4, 40, 30)])
def test_deep_closed_form_matches_token_loop(L, chunk, T):
    k, q, v, al, et, th, _ = _mk(3, T, 5, 12, 60 + L)
    st = _deep_state(3, 5, 12, L, 61)
    y, a = oracle.forward_deep(k, q, v, al, et, th, st, chunk, L)
    yc, b = oracle.forward_deep_closed_form(k, q, v, al, et, th, st, chunk, L)
    assert np.abs(y - yc).max() <= 1e-12 * np.abs(y).max()
    for n in a:
        assert np.abs(a[n] - b[n]).max() <= 1e-12 * np.abs(a[n]).max(), n


SRC = open(obuild.SRC).read()
DEEP_MUTANTS = {
    "output_activation": ("        out[i] = s;\n    }\n}\n\n/*\n * Gradient of || M(k) - v ||^2 with respect to every layer",
                          "        out[i] = s * sigmoid(s);\n    }\n}\n\n/*\n * Gradient of || M(k) - v ||^2 with respect to every layer"),
    "no_silu_prime_hidden": ("                back[m] = b * s * (1.0 + zz * (1.0 - s));", "                back[m] = b;"),
    "activation_as_input": ("const double *in = l == 0 ? k : a + (size_t)(l - 1) * h;",
                            "const double *in = l == 0 ? k : a + (size_t)l * h;"),
    "backprop_untransposed": ("for (int j = 0; j < h; ++j) b += Wl[(size_t)j * h + m] * delta[j];",
                              "for (int j = 0; j < h; ++j) b += Wl[(size_t)m * h + j] * delta[j];"),
    "gradient_at_running_weights": ("deep_grad(d, h, L, Wbar, kx, vx,", "deep_grad(d, h, L, W, kx, vx,"),
    "retrieval_after_update": ("if (y) deep_forward(d, h, L, Wbar, qx,", "if (y) deep_forward(d, h, L, W, qx,"),
}


@pytest.mark.parametrize("name", sorted(DEEP_MUTANTS))
def test_deep_mutant_is_caught(name, tmp_path):
    old, new = DEEP_MUTANTS[name]
    assert SRC.count(old) == 1, f"mutation anchor not found once: {name}"
    src = tmp_path / "mutant.c"
    src.write_text(SRC.replace(old, new))
    lib = str(tmp_path / "libmutant.so")
    obuild.build(force=True, src=str(src), out=lib)
    import ctypes
    fwd_lib = ctypes.CDLL(lib)

    def fwd(*args, **kw):
        return oracle.forward_deep(*args, _lib_override=fwd_lib, **kw)
    failed = []
    for pin in DEEP_PINS:
        try:
            pin(fwd)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"deep mutant {name} passed every pin"
