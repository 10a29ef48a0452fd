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
