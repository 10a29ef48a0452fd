"""The oracle against its pins (CPU only): hand-worked values, closed forms, torch autograd,
finite differences and invariants. See tests/oracle_pins.py for what each pin fixes."""
import numpy as np
import pytest

import oracle
from oracle_pins import PINS, _mk


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(oracle.forward)


@pytest.mark.parametrize("h,d,T,chunk", [(0, 7, 33, 5), (0, 16, 64, 16), (12, 5, 29, 4), (32, 8, 70, 16),
                                         (24, 6, 40, 40), (24, 6, 40, 1), (16, 4, 9, 64)])
def test_closed_form_matches_token_loop(h, d, T, chunk):
    """The chunk closed form (the derivation the GPU kernels follow) equals the defining
    token loop to 1e-12, including a partial last chunk and chunk = 1 / chunk > T."""
    k, q, v, al, et, th, st = _mk(3, T, d, h, 31 + h + chunk)
    y, a = oracle.forward(k, q, v, al, et, th, st, chunk)
    y2, b = oracle.forward_closed_form(k, q, v, al, et, th, st, chunk)
    assert np.abs(y - y2).max() <= 1e-12 * np.abs(y).max()
    for n in a:
        assert np.abs(a[n] - b[n]).max() <= 1e-12 * np.abs(a[n]).max(), n


def test_closed_form_degenerate_gates():
    """eta = 0 and alpha = 1 inside a chunk: the division-free scan stays exact."""
    d, h, T, n = 5, 8, 24, 6
    k, q, v, al, et, th, st = _mk(2, T, d, h, 37)
    al[:, 3] = 1.0
    et[:, 7] = 0.0
    et[:, 12] = 0.0
    al[:, 12] = 1.0
    y, a = oracle.forward(k, q, v, al, et, th, st, n)
    y2, b = oracle.forward_closed_form(k, q, v, al, et, th, st, n)
    assert np.abs(y - y2).max() <= 1e-12 * np.abs(y).max()
    for nm in a:
        assert np.abs(a[nm] - b[nm]).max() <= 1e-12 * max(np.abs(a[nm]).max(), 1e-300), nm


def test_chunk_scalars_match_direct_unroll():
    """c_j, d_j, A, E, sigma from the scan equal the brute-force unroll of one chunk with scalar
    'gradients' (S, W scalars, g_j = unit impulses)."""
    r = np.random.default_rng(41)
    n = 9
    al, et, th = r.uniform(0, 0.3, n), r.uniform(0.2, 0.99, n), r.uniform(0, 0.5, n)
    c, dd, A, E, sig = oracle.chunk_scalars(al, et, th)

    def unroll(W, S, g):
        for j in range(n):
            S = et[j] * S - th[j] * g[j]
            W = (1 - al[j]) * W + S
        return W, S
    W, S = unroll(1.0, 0.0, np.zeros(n))
    assert abs(W - A) < 1e-14 and S == 0.0
    W, S = unroll(0.0, 1.0, np.zeros(n))
    assert abs(W - sig) < 1e-14 and abs(S - E) < 1e-14
    for j in range(n):
        e = np.zeros(n)
        e[j] = 1.0
        W, S = unroll(0.0, 0.0, e)
        assert abs(-W - c[j]) < 1e-14 and abs(-S - dd[j]) < 1e-14


# ---------------------------------------------------------------- the memory-as-a-gate output

def _gate_pins(gate):
    """Pins of o = attn (x) M(x~) read as attn * sigmoid(M): values the definition fixes exactly."""
    r = np.random.default_rng(5)
    attn = r.standard_normal((3, 7, 5))
    y = 3.0 * r.standard_normal((3, 7, 5))
    # a zero attention branch gives zero output, whatever the memory says
    assert np.array_equal(gate(np.zeros_like(attn), y), np.zeros_like(attn))
    # a memory that retrieves exactly zero (e.g. the MLP at its W = 0 fixed point) halves the attention
    assert np.array_equal(gate(attn, np.zeros_like(y)), attn / 2)
    # the logistic function's symmetry sigma(-y) = 1 - sigma(y)
    np.testing.assert_allclose(gate(attn, y) + gate(attn, -y), attn, rtol=0, atol=1e-15)
    # saturation: a large positive retrieval passes the attention through, a large negative blocks it
    np.testing.assert_allclose(gate(attn, np.full_like(y, 50.0)), attn, rtol=1e-15)
    assert np.abs(gate(attn, np.full_like(y, -800.0))).max() == 0.0
    # element-wise: one element of y moves only the same element of o
    y2 = y.copy()
    y2[1, 2, 3] += 1.0
    diff = gate(attn, y2) != gate(attn, y)
    assert diff.sum() == 1 and diff[1, 2, 3]


def test_mag_gate_pins():
    _gate_pins(oracle.mag_gate)


@pytest.mark.parametrize("name,wrong", [
    ("gate_the_memory_by_the_attention", lambda a, y: y / (1.0 + np.exp(-a))),
    ("silu_instead_of_sigmoid", lambda a, y: a * y / (1.0 + np.exp(-y))),
    ("tanh_instead_of_sigmoid", lambda a, y: a * np.tanh(y)),
    ("no_activation", lambda a, y: a * y),
    ("sigmoid_of_minus_y", lambda a, y: a / (1.0 + np.exp(y))),
])
def test_mag_gate_pins_reject_plausible_mistakes(name, wrong):
    with np.errstate(over="ignore"):
        with pytest.raises(AssertionError):
            _gate_pins(wrong)


def test_gated_forward_after_reset_halves_the_attention():
    """alpha = 1, eta = 0, theta = 0 on the last token of a chunk puts the MLP memory at W = 0, its
    fixed point: every later retrieval is exactly 0, so every later gated output is attn / 2."""
    k, q, v, al, et, th, st = _mk(2, 40, 6, 12, 77)
    al[:, 15], et[:, 15], th[:, 15] = 1.0, 0.0, 0.0
    attn = np.random.default_rng(3).standard_normal((2, 40, 6)).astype(np.float32)
    o, _ = oracle.forward_gated(k, q, v, al, et, th, st, 8, attn)
    assert np.array_equal(o[:, 16:], attn[:, 16:].astype(np.float64) / 2)
    y, _ = oracle.forward(k, q, v, al, et, th, st, 8)
    assert np.abs(o[:, :16] - oracle.mag_gate(attn[:, :16], y[:, :16])).max() == 0.0


# ---------------------------------------------------------------- chunk-shared gates (the LTI variant)

def test_chunk_coefficients_with_chunk_shared_gates_are_geometric_sums():
    """With alpha, eta, theta shared by a chunk's tokens (walk-through sec. 3.2, "Parameters as the
    Function of Chunks": the system is then linear time-invariant), the coefficients have closed
    forms: P_j = (1-a)^(n-1-j), Q_j = e^(n-1-j), r_j = sum_{m=j}^{n-1} (1-a)^(n-1-m) e^(m-j)
    = ((1-a)^(n-j) - e^(n-j)) / ((1-a) - e), c_j = th r_j, d_j = th e^(n-1-j), A = (1-a)^n, E = e^n,
    sigma = e r_0. The oracle's scan must reach them; its coefficients depend on j only through
    n-1-j (a convolution kernel)."""
    for n, a, e, th in [(16, 0.03, 0.9, 0.07), (7, 0.0, 0.5, 0.1), (64, 0.01, 0.95, 0.002), (5, 0.3, 0.2, 1.0)]:
        c, dd, A, E, sig = oracle.chunk_scalars(np.full(n, a), np.full(n, e), np.full(n, th))
        j = np.arange(n)
        keep = 1.0 - a
        r = (keep ** (n - j) - e ** (n - j)) / (keep - e)
        np.testing.assert_allclose(c, th * r, rtol=1e-12)
        np.testing.assert_allclose(dd, th * e ** (n - 1 - j), rtol=1e-12)
        np.testing.assert_allclose([A, E, sig], [keep ** n, e ** n, e * r[0]], rtol=1e-12)


def test_forward_with_chunk_gates_is_the_forward_with_repeated_gates():
    """oracle.expand_chunk_gates repeats each chunk's gates over its tokens (a ragged last chunk
    included); running the token loop on them defines the chunk-shared-gate forward."""
    g = np.arange(2 * 3, dtype=np.float32).reshape(2, 3)
    x = oracle.expand_chunk_gates(g, T=7, chunk=3)
    assert x.shape == (2, 7)
    assert np.array_equal(x[0], [0, 0, 0, 1, 1, 1, 2]) and np.array_equal(x[1], [3, 3, 3, 4, 4, 4, 5])


# ---------------------------------------------------------------- the linear memory's cross-chunk scan

@pytest.mark.parametrize("T,chunk,segments", [(64, 16, 1), (100, 16, 3), (96, 8, 12), (37, 5, 4)])
@pytest.mark.parametrize("tree", [False, True])
def test_cross_chunk_scan_matches_the_token_loop(T, chunk, segments, tree):
    """The linear memory's chunk update is an affine map of [W | S]; composing the maps per segment
    (in order or pairwise) and scanning the segments gives the defining recurrence's result."""
    k, q, v, al, et, th, st = _mk(2, T, 6, 0, 71 + T)
    y, a = oracle.forward(k, q, v, al, et, th, st, chunk)
    ys, b = oracle.forward_linear_scan(k, q, v, al, et, th, st, chunk, segments, tree=tree)
    assert np.abs(ys - y).max() <= 1e-12 * np.abs(y).max()
    for n in a:
        assert np.abs(b[n] - a[n]).max() <= 1e-12 * np.abs(a[n]).max(), n


def test_chunk_map_against_the_recurrence_on_a_basis():
    """M and N of one chunk, against the token loop started from W = e_i rows / S = e_i rows with v = 0
    (the columns of M) and from W = S = 0 (N)."""
    k, q, v, al, et, th, _ = _mk(1, 9, 3, 0, 81)
    d = 3
    M, N = oracle.linear_chunk_map(k[0], v[0], al[0], et[0], th[0])
    zero = np.zeros_like(v)
    for i in range(2 * d):
        X = np.zeros((1, d, 2 * d))
        X[0, 0, i] = 1.0  # row 0 of [W | S] is the basis row e_i
        _, out = oracle.forward(k, q, zero, al, et, th, {"W1": X[:, :, :d], "S1": X[:, :, d:]}, 9)
        got = np.concatenate([out["W1"][0, 0], out["S1"][0, 0]])
        np.testing.assert_allclose(got, M[i], rtol=1e-12, atol=1e-14)
    _, out = oracle.forward(k, q, v, al, et, th, {"W1": np.zeros((1, d, d)), "S1": np.zeros((1, d, d))}, 9)
    np.testing.assert_allclose(np.concatenate([out["W1"][0], out["S1"][0]], axis=1), N, rtol=1e-12, atol=1e-14)
