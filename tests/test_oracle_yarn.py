"""Pins of the oracle's YaRN table and rotary against facts fixed by the pages
and by mathematics (not by re-typing the oracle's formulas).

Sources: mistral.rs PR "YaRN rope scaling, 4-bit F4 packed KV cache, ...",
section 1 (llama.cpp-style corr_dims ramp, table scale 1 + 0.1 ln(factor),
golden positions 262144/262145/319999 matched to <= 5e-12); ignis
"context-and-speculation", --model-rope-scaling (attention factor on queries
and keys alike).
"""
import math

import mpmath
import numpy as np
import pytest

import oracle
from conftest import read_golden

YARN4 = dict(rope_base=1e7, rot_dim=64, factor=4.0, orig_max_pos=262144, beta_fast=32.0, beta_slow=1.0)
PLAIN = dict(rope_base=1e7, rot_dim=64, factor=1.0)


def test_table_scale_matches_printed_example():
    g, _ = read_golden("yarn_table_scale.txt")
    factor, want, dec = float(g["factor"][0]), float(g["table_scale"][0]), int(g["decimals"][0])
    _, ms, _, _ = oracle.yarn_theta(dict(YARN4, factor=factor))
    assert abs(ms - want) <= 0.5 * 10.0 ** (-dec)
    # and the same rule at the long-window factor
    _, ms4, _, _ = oracle.yarn_theta(YARN4)
    assert abs(ms4 - 1.1386294361) < 1e-10


def test_factor_one_is_textbook_rope():
    """factor 1: theta_j = base^(-2j/d) (the original RoPE frequencies), scale 1."""
    th, ms, _, _ = oracle.yarn_theta(PLAIN)
    assert ms == 1.0
    mpmath.mp.dps = 40
    for j, t in enumerate(th):
        ref = mpmath.power(mpmath.mpf(10) ** 7, mpmath.mpf(-2 * j) / 64)
        assert abs(t - float(ref)) <= 4e-16 * float(ref)


def _turns(j, d=64, base=1e7, orig=262144):
    """full turns of pair j over the original context, high precision"""
    return orig * mpmath.power(base, mpmath.mpf(-2 * j) / d) / (2 * mpmath.pi)


def test_ramp_bounds_from_rotation_counts():
    """low/high are where pairs stop completing beta_fast / beta_slow turns over
    the original context, found here by bisection on the turn count."""
    mpmath.mp.dps = 40
    cross = lambda beta: mpmath.findroot(lambda j: _turns(j) - beta, (0, 31), solver="bisect")
    c_fast, c_slow = cross(32), cross(1)
    want_low = max(0, math.floor(c_fast))
    want_high = min(63, math.ceil(c_slow))
    _, _, low, high = oracle.yarn_theta(YARN4)
    assert (low, high) == (want_low, want_high) == (14, 22)
    # pairs at or below low turn at least beta_fast times; at or above high, < beta_slow... +1 turn
    assert _turns(14) >= 32 > _turns(15)
    assert _turns(21) > 1 >= _turns(22)


def test_theta_regions():
    """j <= low keeps the trained frequency; j >= high is interpolated by 1/s;
    in between the ratio moves linearly in j (a linear ramp)."""
    th, _, low, high = oracle.yarn_theta(YARN4)
    om, _, _, _ = oracle.yarn_theta(PLAIN)
    ratio = th / om
    low, high = int(low), int(high)
    assert np.all(ratio[: low + 1] == 1.0)
    assert np.allclose(ratio[high:], 0.25, rtol=0, atol=1e-15)
    mid = ratio[low: high + 1]
    assert np.all(np.diff(mid) < 0)
    assert np.allclose(np.diff(mid, 2), 0, atol=1e-14)


def test_pythagoras_and_scale():
    c, s = oracle.yarn_table(YARN4, 262140, 64)
    _, ms, _, _ = oracle.yarn_theta(YARN4)
    assert np.allclose(c * c + s * s, ms * ms, rtol=0, atol=1e-14)


@pytest.mark.parametrize("pos", [262144, 262145, 319999, 524287, 1048575])
def test_large_positions_match_high_precision(pos):
    """The table at the pages' golden positions against a 40-digit evaluation
    of cos/sin. The angle is the position times the double angle step, rounded
    once to double; at that angle the table is exact to ~1e-16, and against the
    unrounded product it is off by at most mscale * ulp(angle) / 2."""
    th, ms, _, _ = oracle.yarn_theta(YARN4)
    c, s = oracle.yarn_table(YARN4, pos, 1)
    mpmath.mp.dps = 40
    for j in range(32):
        a_dbl = mpmath.mpf(float(pos) * float(th[j]))     # the double-rounded angle
        assert abs(c[0, j] - ms * float(mpmath.cos(a_dbl))) <= 1e-15
        assert abs(s[0, j] - ms * float(mpmath.sin(a_dbl))) <= 1e-15
        a = mpmath.mpf(pos) * mpmath.mpf(th[j])            # exact product
        bound = ms * 0.5 * np.spacing(float(a)) + 1e-15
        assert abs(c[0, j] - ms * float(mpmath.cos(a))) <= bound
        assert abs(s[0, j] - ms * float(mpmath.sin(a))) <= bound


def test_plain_table_differs_past_trained_window():
    """A longer table with the trained frequencies is not the YaRN table."""
    c1, _ = oracle.yarn_table(PLAIN, 300000, 1)
    c4, _ = oracle.yarn_table(YARN4, 300000, 1)
    assert np.max(np.abs(c1 - c4)) > 0.1


def test_rope_matches_complex_rotation():
    """NEOX rotate-half: pair (x_j, x_{j+h}) behaves as the complex number
    x_j + i x_{j+h} multiplied by mscale * e^{i p theta_j}."""
    rng = np.random.default_rng(1)
    x = rng.standard_normal((3, 2, 256))
    pos = np.array([0, 4095, 524287])
    y = oracle.rope_apply_f64(x, pos, YARN4)
    th, ms, _, _ = oracle.yarn_theta(YARN4)
    z = (x[..., :32] + 1j * x[..., 32:64]) * ms * np.exp(1j * pos[:, None, None] * th[None, None, :])
    assert np.allclose(y[..., :32], z.real, atol=1e-12)
    assert np.allclose(y[..., 32:64], z.imag, atol=1e-12)
    assert np.array_equal(y[..., 64:], x[..., 64:])


def test_rope_norm_and_relative_position():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 1, 256))
    k = rng.standard_normal((1, 1, 256))
    _, ms, _, _ = oracle.yarn_theta(YARN4)
    rq = oracle.rope_apply_f64(q, [700001], YARN4)
    n_in = np.hypot(q[..., :32], q[..., 32:64])
    n_out = np.hypot(rq[..., :32], rq[..., 32:64])
    assert np.allclose(n_out, ms * n_in, rtol=1e-13)
    dots = []
    for p, pk in [(10, 3), (262147, 262140), (1048575, 1048568)]:
        a = oracle.rope_apply_f64(q, [p], YARN4)
        b = oracle.rope_apply_f64(k, [pk], YARN4)
        dots.append(float(np.sum(a * b)))
    assert np.allclose(dots, dots[0], rtol=0, atol=1e-9)


def test_rope_composition_factor_one():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((1, 4, 256))
    a = oracle.rope_apply_f64(oracle.rope_apply_f64(x, [1000], PLAIN), [2345], PLAIN)
    b = oracle.rope_apply_f64(x, [3345], PLAIN)
    assert np.allclose(a, b, atol=1e-12)


def test_rope_bf16_is_rounded_f64():
    rng = np.random.default_rng(4)
    x32 = rng.standard_normal((5, 3, 256)).astype(np.float32)
    import workloads
    xb = workloads.f32_to_bf16_bits(x32)
    pos = np.array([1, 2, 3, 262144, 524287])
    y = oracle.rope_apply_bf16(xb, pos, YARN4)
    yf = oracle.rope_apply_f64(oracle.bf16_to_f64(xb), pos, YARN4)
    assert np.array_equal(y, oracle.f64_to_bf16(yf))
    assert np.array_equal(y[..., 64:], xb[..., 64:])
