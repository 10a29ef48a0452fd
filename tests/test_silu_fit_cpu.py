"""The FMA-pipe tanh of the tensor-core chunk kernel's SiLU, on the CPU: its constants are the ones
the fit script generates, the fit is the Chebyshev interpolant it claims to be, and the fp32 route
meets its error bound against fp64 tanh and silu."""
import os

import numpy as np
from numpy.polynomial import polynomial as P

from titans_long_term_b200 import silu_fit

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KERNEL = os.path.join(ROOT, "titans_long_term_b200", "csrc", "chunk_tc_mlp64.cu")
BOUND = 1.1e-4  # absolute error of tanh|h| on the route


def test_kernel_constants_are_the_generated_ones():
    src = open(KERNEL).read()
    for line in silu_fit.c_constants().splitlines():
        assert line in src, line


def test_fits_interpolate_at_the_chebyshev_nodes():
    # The interpolant through n + 1 Chebyshev nodes reproduces the function there (before rounding
    # to fp32), and the two target functions are the ones named: 2^-f and (1 - e) / (1 + e).
    for fn, a, b, deg in ((lambda f: 2.0 ** (-f), -0.5, 0.5, silu_fit.DEG_EXP2),
                          (lambda e: (1 - e) / (1 + e), 0.0, 1.0, silu_fit.DEG_Q)):
        c = silu_fit.chebyshev_interpolant(fn, a, b, deg)
        k = np.arange(deg + 1)
        x = 0.5 * (b - a) * np.cos((2 * k + 1) * np.pi / (2 * (deg + 1))) + 0.5 * (a + b)
        np.testing.assert_allclose(P.polyval(x, c), fn(x), rtol=0, atol=1e-13)
    # Near-minimax: a Chebyshev interpolant's error is within a small factor of the best
    # polynomial's; here the worst errors on a dense grid.
    p, q = silu_fit.coefficients()
    f = np.linspace(-0.5, 0.5, 20001)
    assert np.max(np.abs(P.polyval(f, p.astype(np.float64)) * 2.0 ** f - 1)) < 1.1e-4
    e = np.linspace(0, 1, 20001)
    assert np.max(np.abs(P.polyval(e, q.astype(np.float64)) - (1 - e) / (1 + e))) < 1.05e-4


def test_route_error_against_fp64_tanh():
    h = np.concatenate([np.linspace(-30, 30, 1_200_001), [0.0, -0.0, 1e-38, -1e-38, 1e-7, 5.0, 1e4, 3e38, -3e38]])
    h = h.astype(np.float32)
    t = silu_fit.tanh_abs_fp32(h).astype(np.float64)
    ref = np.tanh(np.abs(h.astype(np.float64)))
    err = np.abs(t - ref)
    assert err.max() < BOUND, (err.max(), h[err.argmax()])
    assert np.all(np.isfinite(t))


def test_silu_against_fp64():
    h = np.linspace(-40, 40, 800_001).astype(np.float32)
    s = silu_fit.silu_fp32(h).astype(np.float64)
    z = 2.0 * h.astype(np.float64)
    ref = z / (1.0 + np.exp(-z))  # silu(z) = z sigmoid(z), z = 2h
    err = np.abs(s - ref)
    assert np.all(err <= np.abs(h) * BOUND + 1e-6 * np.abs(ref) + 1e-30)
    # odd part: silu(z) - silu(-z) = z for the exact function; the route keeps it to its bound
    d = silu_fit.silu_fp32(h).astype(np.float64) - silu_fit.silu_fp32(-h).astype(np.float64)
    assert np.all(np.abs(d - z) <= 1e-6 * np.abs(z) + 1e-30)
