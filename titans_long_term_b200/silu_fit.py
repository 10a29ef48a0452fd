"""Coefficients of the FMA-pipe tanh that the tensor-core chunk kernel uses for part of its SiLU.

    python -m titans_long_term_b200.silu_fit      # prints the constants as they appear in the kernel

The kernel evaluates silu(z) = h (1 + tanh h), h = z / 2. Most tanh evaluations go to the
hardware's special-function unit (tanh.approx.f32); a fixed share of the queries' evaluations uses
plain fp32 arithmetic instead, so that both units work during the SiLU phase. That route computes
tanh|h| = (1 - e) / (1 + e) with e = exp(-2|h|) = 2^-y, y = 2 log2(e) |h|, in two steps:
  - 2^-y = 2^-n * 2^-f with n = round(y) and f = y - n in [-1/2, 1/2]: 2^-f is a cubic in f and
    2^-n is applied by subtracting n from the exponent field;
  - (1 - e) / (1 + e) on e in [0, 1] is a quintic in e.
Both polynomials are Chebyshev interpolants (interpolation at the Chebyshev nodes of the first
kind, a near-minimax polynomial; Trefethen, "Approximation Theory and Approximation Practice",
ch. 4 and 16), computed here in fp64 and rounded once to fp32. The sign is restored through
silu = h + |h| tanh|h|.
"""
from __future__ import annotations

import numpy as np
from numpy.polynomial import chebyshev as _cheb
from numpy.polynomial import polynomial as _poly

LOG2E_X2 = 2.0 / np.log(2.0)  # y = LOG2E_X2 * |h|
Y_MAX = 64.0                  # e < 2^-63 there: tanh|h| = 1 in fp32
ROUND_MAGIC = 12582912.0      # 1.5 * 2^23: y + magic rounds y to an integer held in the low mantissa bits
DEG_EXP2, DEG_Q = 3, 5


def chebyshev_interpolant(fn, a: float, b: float, deg: int) -> np.ndarray:
    """Monomial coefficients (lowest first, in x) of the degree-`deg` polynomial that interpolates
    fn at the deg + 1 Chebyshev nodes of the first kind mapped to [a, b]."""
    k = np.arange(deg + 1)
    t = np.cos((2 * k + 1) * np.pi / (2 * (deg + 1)))
    x = 0.5 * (b - a) * t + 0.5 * (b + a)
    in_t = _cheb.cheb2poly(_cheb.chebfit(t, fn(x), deg))  # monomials in t = (2x - a - b) / (b - a)
    lin = np.array([-(a + b) / (b - a), 2.0 / (b - a)])
    out, acc = np.zeros(deg + 1), np.array([1.0])
    for i, ci in enumerate(in_t):
        if i > 0:
            acc = _poly.polymul(acc, lin)
        out[: len(acc)] += ci * acc
    return out


def coefficients():
    """(exp2 cubic, quintic) coefficients, lowest degree first, rounded to fp32."""
    p = chebyshev_interpolant(lambda f: 2.0 ** (-f), -0.5, 0.5, DEG_EXP2)
    q = chebyshev_interpolant(lambda e: (1.0 - e) / (1.0 + e), 0.0, 1.0, DEG_Q)
    return p.astype(np.float32), q.astype(np.float32)


def _fma32(a, b, c):
    # fp32 fused multiply-add: the fp32 product is exact in fp64, one rounding of the sum to fp32
    with np.errstate(over="ignore"):
        return (np.asarray(a, np.float64) * np.asarray(b, np.float64) + np.asarray(c, np.float64)).astype(np.float32)


def tanh_abs_fp32(h: np.ndarray) -> np.ndarray:
    """The route's steps in fp32, as the kernel takes them (for the tests)."""
    p, q = coefficients()
    h = np.asarray(h, np.float32)
    with np.errstate(over="ignore"):  # |h| near the fp32 maximum: the product is inf, clamped like on the GPU
        y = np.minimum(np.abs(h) * np.float32(LOG2E_X2), np.float32(Y_MAX)).astype(np.float32)
    r = (y + np.float32(ROUND_MAGIC)).astype(np.float32)
    f = (y - (r - np.float32(ROUND_MAGIC)).astype(np.float32)).astype(np.float32)
    s = np.full_like(f, p[-1])
    for c in p[-2::-1]:
        s = _fma32(s, f, c)
    e = (s.view(np.uint32) - (r.view(np.uint32) << np.uint32(23))).astype(np.uint32).view(np.float32)
    t = np.full_like(e, q[-1])
    for c in q[-2::-1]:
        t = _fma32(t, e, c)
    return t


def silu_fp32(h: np.ndarray) -> np.ndarray:
    """silu(2h) = h + |h| tanh|h| on the route above."""
    h = np.asarray(h, np.float32)
    return _fma32(np.abs(h), tanh_abs_fp32(h), h)


def c_constants() -> str:
    """The two coefficient lists as the kernel declares them (kP0.. for 2^-f, kQ0.. for the quintic)."""
    p, q = coefficients()
    decl = lambda name, cs: "constexpr float " + ", ".join(f"{name}{i} = {float(v):.9e}f" for i, v in enumerate(cs)) + ";"
    return decl("kP", p) + "\n" + decl("kQ", q)


if __name__ == "__main__":
    print(c_constants())
