"""The FMA-pipe 2^x of csrc/exp2_poly.cuh, pinned on the CPU.

* The header is exactly what csrc/gen_exp2_poly.py writes (so the stated
  coefficients and bounds come from the Remez fit, not hand edits).
* The float32 evaluation, emulated step by step (each fused multiply-add
  rounded once), stays within the stated relative error over [-125, 0] against
  the exact 2^x, is exact at the integers (2^n), and never leaves the normal
  float range.
* The coefficients sit next to the Taylor coefficients (ln 2)^k / k! that a
  minimax fit of 2^f on a small interval must approach."""
import importlib.util
import math
import os

import numpy as np
import pytest

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "sparse_attention_long_anchor_b200", "csrc")


@pytest.fixture(scope="module")
def gen():
    spec = importlib.util.spec_from_file_location("gen_exp2_poly", os.path.join(CSRC, "gen_exp2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


@pytest.fixture(scope="module")
def fit(gen):
    return gen.fitted()


def test_header_is_the_generators_output(gen, fit):
    with open(os.path.join(CSRC, "exp2_poly.cuh")) as fh:
        assert fh.read() == gen.header_text(fit)


@pytest.mark.parametrize("deg,bound", [(4, 3e-6), (5, 3e-7)])
def test_relative_error_bound(gen, fit, deg, bound):
    c32, fit_err = fit[deg]
    assert fit_err < bound
    assert gen.measured_bound(c32, samples=1 << 20, seed=1) < bound


@pytest.mark.parametrize("deg,bound", [(4, 3e-6), (5, 3e-7)])
def test_integers_and_range(gen, fit, deg, bound):
    c32, _ = fit[deg]
    n = np.arange(-125, 1, dtype=np.float32)
    got = gen.emulate(n, c32).astype(np.float64)
    # at f = 0 the polynomial is its constant term (the minimax fit moves it off
    # 1 by at most the fit error); scaling by 2^n is exact
    assert np.max(np.abs(got / np.exp2(n.astype(np.float64)) - 1.0)) < bound
    assert np.all(got == got[-1] * np.exp2(n.astype(np.float64)))
    very_negative = gen.emulate(np.array([-126.0, -200.0, -1e30], dtype=np.float32), c32)
    assert np.all(very_negative > 0) and np.all(very_negative < 3e-38)
    assert np.all(np.isfinite(gen.emulate(np.linspace(-125, 0, 10001, dtype=np.float32), c32)))
    # monotone on a fine grid (the pooled sums rely on order only through the band)
    xs = np.linspace(-4.0, 0.0, 40001, dtype=np.float32)
    ys = gen.emulate(xs, c32)
    assert np.all(np.diff(ys.astype(np.float64)) >= 0)


@pytest.mark.parametrize("deg", [4, 5])
def test_coefficients_near_taylor(fit, deg):
    c32, _ = fit[deg]
    for k, ck in enumerate(c32):
        taylor = math.log(2.0) ** k / math.factorial(k)
        # the fit absorbs the truncated terms into the last coefficients: within
        # 2 % of Taylor, far from any reordering or transposition of them
        assert abs(float(ck) - taylor) < 2e-2 * taylor + 1e-5, (k, float(ck), taylor)
