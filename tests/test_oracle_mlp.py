"""Pins of the oracle's gated-MLP pieces (silu * up) against library routines,
closed forms and invariants."""
import numpy as np
import pytest
from scipy.special import expit

import oracle
from verify_step_lm_b200 import synth


def test_silu_mul_equals_x_times_logistic():
    rng = np.random.default_rng(1)
    g = rng.normal(0, 4, 10000)
    u = rng.normal(0, 1, 10000)
    np.testing.assert_allclose(oracle.silu_mul(g, u), g * expit(g) * u, rtol=1e-14, atol=1e-300)


def test_silu_odd_part_and_limits():
    g = np.linspace(-30, 30, 601)
    one = np.ones_like(g)
    # silu(g) - silu(-g) = g for every g (logistic(g) + logistic(-g) = 1)
    np.testing.assert_allclose(oracle.silu_mul(g, one) - oracle.silu_mul(-g, one), g, rtol=1e-13, atol=1e-13)
    assert oracle.silu_mul(0.0, 5.0) == 0.0
    assert oracle.silu_mul(40.0, 1.0) == pytest.approx(40.0, rel=1e-15)
    assert abs(oracle.silu_mul(-800.0, 1.0)) == 0.0  # exp overflow is a clean zero, not a NaN


def test_gate_up_is_the_two_halves():
    F, Kd, M = 64, 256, 3
    W = synth.make_head(2 * F, Kd, 0.05, seed=3)
    Wq, S = synth.quantize_int4_g64(W)
    x = synth.gaussian((M, Kd), 1.0, 4)
    xb, Sb, Wqn = synth.bf16_bits(x), synth.bf16_bits(S), Wq.numpy()
    g = oracle.lm_head_int4g64(xb, Wqn[:F], Sb[:F])
    u = oracle.lm_head_int4g64(xb, Wqn[F:], Sb[F:])
    h = oracle.gate_up_int4g64(xb, Wqn, Sb, F)
    np.testing.assert_array_equal(h, oracle.silu_mul(g, u))
    cols = np.array([0, 5, 63])
    np.testing.assert_array_equal(oracle.gate_up_int4g64(xb, Wqn, Sb, F, cols=cols), h[:, cols])
