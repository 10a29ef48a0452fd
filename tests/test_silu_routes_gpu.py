"""The chunk kernel's two SiLU routes on the GPU (titans_silu_routes): the FMA-pipe route equals its
fp32 restatement step for step, and both routes hold their error bounds against fp64 silu."""
import numpy as np
import pytest
import torch

from titans_long_term_b200 import mem, silu_fit

pytestmark = pytest.mark.gpu


def _grid():
    h = np.concatenate([np.linspace(-40, 40, 2_000_001),
                        [0.0, -0.0, 1e-38, -1e-38, 1e-20, 1e-7, -1e-7, 9.0, -9.0, 1e4, -1e4, 3e38, -3e38]])
    return h.astype(np.float32)


def test_fma_route_matches_its_fp32_steps():
    h = _grid()
    s_fma, _ = mem.silu_routes(torch.from_numpy(h).cuda())
    got = s_fma.cpu().numpy()
    want = silu_fit.silu_fp32(h)
    # Same operations in the same order; the CPU restatement rounds each fused multiply-add from
    # fp64, which can differ from one fp32 rounding by an ulp in rare ties.
    # (h near the fp32 maximum overflows to the same infinity on both.)
    close = np.abs(got.astype(np.float64) - want) <= np.spacing(np.abs(want)).astype(np.float64) + 1e-44
    assert np.all((got == want) | close)


def test_both_routes_against_fp64_silu():
    h = _grid()[:-2]  # z = 2h must stay finite for the fp64 reference
    s_fma, s_mufu = (x.cpu().numpy().astype(np.float64) for x in mem.silu_routes(torch.from_numpy(h).cuda()))
    z = 2.0 * h.astype(np.float64)
    with np.errstate(over="ignore"):
        ref = z / (1.0 + np.exp(-z))
    ah = np.abs(h.astype(np.float64))
    # tanh's absolute error times |h|: 1.1e-4 on the FMA route, 2^-10 for tanh.approx.f32 (its
    # relative error is about 2^-11 and |tanh| <= 1), plus the final fma's rounding.
    assert np.all(np.abs(s_fma - ref) <= ah * 1.1e-4 + 1e-6 * np.abs(ref) + 1e-37)
    assert np.all(np.abs(s_mufu - ref) <= ah * 2.0 ** -10 + 1e-6 * np.abs(ref) + 1e-37)


def test_routes_reject_bad_arguments():
    with pytest.raises(TypeError):
        mem.silu_routes(torch.zeros(4))
    L = mem.lib()
    assert L.titans_silu_routes(None, None, None, -1, None) == mem.EINVAL
    assert L.titans_silu_routes(None, None, None, 4, None) == mem.EINVAL
    assert L.titans_silu_routes(None, None, None, 0, None) == mem.OK
