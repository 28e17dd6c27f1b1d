"""Pins of the oracle's SwiGLU form of the preprocessing (h = SiLU(gate) * up,
SiLU(a) = a / (1 + E(-a))) against fp64 mathematics and exact special cases.

The pages give no formula for the gated activation; the oracle defines one in
fixed fp32 steps (see oracle/sharq_oracle.c, SwiGLU section).  These tests tie
its exponential E and SiLU to e^x and a / (1 + e^-a) computed in fp64."""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _ulps(got: np.ndarray, ref64: np.ndarray) -> np.ndarray:
    ref32 = ref64.astype(np.float32)
    return np.abs(got.astype(np.float64) - ref64) / np.spacing(np.abs(ref32)).astype(np.float64)


def test_exp_within_one_ulp_of_fp64():
    x = np.float32(np.linspace(-87.0, 88.0, 400001))
    e = oracle.exp(x)
    ref = np.exp(x.astype(np.float64))
    assert np.all(np.isfinite(e))
    assert _ulps(e, ref).max() <= 1.0


def test_exp_special_values_and_monotone():
    e = oracle.exp(np.float32([0.0, -0.0, 89.0, 100.0, -104.0, -200.0]))
    assert e[0] == 1.0 and e[1] == 1.0
    assert np.isinf(e[2]) and np.isinf(e[3])
    assert e[4] == 0.0 and e[5] == 0.0
    x = np.float32(np.linspace(-20.0, 20.0, 100001))
    assert np.all(np.diff(oracle.exp(x).astype(np.float64)) >= 0)


def test_silu_against_fp64():
    a = np.float32(np.linspace(-15.0, 15.0, 60001))
    got = oracle.swiglu(a, np.ones_like(a))
    ref = a.astype(np.float64) / (1.0 + np.exp(-a.astype(np.float64)))
    # a / (1 + E(-a)): one ulp in E, one rounding each for the add and the divide
    assert _ulps(got, ref).max() <= 3.0


def test_silu_exact_cases():
    big = np.float32([20.0, 37.5, 1000.0, 3.0e38])
    assert np.array_equal(oracle.swiglu(big, np.ones_like(big)), big)   # 1 + E(-a) rounds to 1
    neg = np.float32([-104.0, -1000.0])
    s = oracle.swiglu(neg, np.ones_like(neg))
    assert np.all(s == 0.0) and np.all(np.signbit(s))                   # a / inf = -0
    z = oracle.swiglu(np.float32([0.0]), np.float32([5.0]))
    assert z[0] == 0.0


def test_swiglu_product_against_fp64():
    rng = np.random.default_rng(5)
    a = np.float32(rng.standard_normal(200000) * 3)
    b = np.float32(rng.standard_normal(200000) * 3)
    got = oracle.swiglu(a, b)
    a64, b64 = a.astype(np.float64), b.astype(np.float64)
    ref = a64 / (1.0 + np.exp(-a64)) * b64
    ok = np.abs(ref) > 1e-30
    assert _ulps(got[ok], ref[ok]).max() <= 4.0


@pytest.mark.parametrize("fmt,pat", [("nvfp4", "4:8pair"), ("mxfp4", "2:4"), ("nvfp4", "8:16")])
def test_prepare_swiglu_composes_where_silu_is_identity(fmt, pat):
    """With every gate >= 20, SiLU(gate) = gate exactly, so the SwiGLU form must
    equal the plain preprocessing of gate * up rounded once to fp32."""
    rng = np.random.default_rng(6)
    t, k = 24, 512
    gate = np.float32(20.0 + rng.uniform(0.0, 40.0, (t, k)))
    up = np.float32(rng.standard_normal((t, k)))
    up[:, rng.permutation(k)[:4]] *= 30.0
    a = oracle.prepare_swiglu(gate, up, fmt, pat)
    b = oracle.prepare(np.float32(gate * up), fmt, pat)
    for f in ("meta", "bb_codes", "bb_scales", "res_codes", "res_scales", "tensor"):
        assert np.array_equal(a[f], b[f]), f
