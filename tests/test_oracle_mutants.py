"""Mutation check of the pins (CPU only): plausible mistakes planted in copies of the oracle's
C source (a dropped factor, a wrong sign, the old momentum in the weight update, a transposed
outer product, an off-by-one chunk boundary, retrieval after the update, sigmoid' for silu',
gradients at the running weights, ...) must each fail at least one pin. The mistakes are
planted only in temporary copies on the CPU; the oracle itself is never changed."""
import os
import subprocess

import pytest

import oracle
from oracle import build as obuild
from oracle_pins import PINS

SRC = open(obuild.SRC).read()

MUTANTS = {
    "no_factor_2_mlp": ("ge[i] = 2.0 * (out[i] - v[i]);", "ge[i] = (out[i] - v[i]);"),
    "no_factor_2_linear": ("double e2 = 2.0 * (out[i] - v[i]);", "double e2 = (out[i] - v[i]);"),
    "momentum_sign": ("S[i] = eta * S[i] - theta * g[i];", "S[i] = eta * S[i] + theta * g[i];"),
    "old_S_in_W": ("        S[i] = eta * S[i] - theta * g[i];\n        W[i] = (1.0 - alpha) * W[i] + S[i];",
                   "        W[i] = (1.0 - alpha) * W[i] + S[i];\n        S[i] = eta * S[i] - theta * g[i];"),
    "forget_after_add": ("W[i] = (1.0 - alpha) * W[i] + S[i];", "W[i] = (1.0 - alpha) * (W[i] + S[i]);"),
    "eta_on_gradient": ("S[i] = eta * S[i] - theta * g[i];", "S[i] = eta * (S[i] - theta * g[i]);"),
    "transposed_linear_outer": ("gW[(size_t)i * d + m] = e2 * k[m];", "gW[(size_t)m * d + i] = e2 * k[m];"),
    "chunk_off_by_one": ("if (t % chunk == 0) {", "if ((t + 1) % chunk == 0 || t == 0) {"),
    "retrieve_running_linear": ("if (linear) linear_apply(d, W1bar, qx, yt);", "if (linear) linear_apply(d, W1, qx, yt);"),
    "retrieve_running_mlp": ("else mlp_apply(d, h, W1bar, W2bar, qx, zq, a, yt);", "else mlp_apply(d, h, W1, W2, qx, zq, a, yt);"),
    "sigmoid_prime_for_silu_prime": ("delta[j] = back * s * (1.0 + z[j] * (1.0 - s));", "delta[j] = back * s * (1.0 - s);"),
    "grad_at_running_linear": ("linear_grad(d, W1bar, kx, vx, out, g1);", "linear_grad(d, W1, kx, vx, out, g1);"),
    "grad_at_running_mlp": ("mlp_grad(d, h, W1bar, W2bar, kx, vx,", "mlp_grad(d, h, W1, W2, kx, vx,"),
    "w2_grad_uses_z": ("gW2[(size_t)i * h + j] = ge[i] * a[j];", "gW2[(size_t)i * h + j] = ge[i] * z[j];"),
    "backprop_transposed_W2": ("for (int i = 0; i < d; ++i) back += W2[(size_t)i * h + j] * ge[i];",
                               "for (int i = 0; i < d; ++i) back += W2[((size_t)j * d + i) % ((size_t)d * h)] * ge[i];"),
    "silu_as_sigmoid": ("a[j] = s * sigmoid(s);", "a[j] = sigmoid(s);"),
    "missing_alpha_first_token": ("for (long t = 0; t < T; ++t) {", "for (long t = 0; t < T; ++t) { if (t == 0) { } "),
}
# "missing_alpha_first_token" above is an identity edit (a control): it must PASS every pin.


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    assert SRC.count(old) >= 1, f"mutation anchor not found: {name}"
    src = tmp_path / "mutant.c"
    src.write_text(SRC.replace(old, new))
    lib = str(tmp_path / "libmutant.so")
    obuild.build(force=True, src=str(src), out=lib)
    fwd = oracle.forward_from_library(lib)
    failed = []
    for pin in PINS:
        try:
            pin(fwd)
        except AssertionError:
            failed.append(pin.__name__)
    if name == "missing_alpha_first_token":
        assert not failed, f"identity edit must pass every pin, failed: {failed}"
    else:
        assert failed, f"mutant {name} passed every pin"
