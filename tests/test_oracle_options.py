"""Pins of the oracle's step options (bias, softplus, clamp, zero-order hold).

Sources: "精读笔记 #12：Mamba" (llm-papers-study) — section 2.2 (the zero-order
hold rule: A_bar = exp(Delta A), B_bar = (Delta A)^-1 (exp(Delta A) - I) Delta B),
section 3 (algorithm 2: Delta = softplus of a projection) and section 3.5
(theorem 1: with N = 1, A = -1, B = 1 the selective recurrence is the gate
h_t = (1 - g_t) h_{t-1} + g_t x_t with g_t a sigmoid).

Each check stands apart from the oracle's code: theorem 1 as a gate written
here with the logistic function, the hold weight as a numerical integral of
exp(A s), softplus against numpy's logaddexp, and the bias and clamp against
the already pinned plain forward on pre-processed steps.
"""
import math

import numpy as np
import pytest

import oracle

RTOL = 1e-12


def _close(a, b, rtol=RTOL):
    scale = max(1.0, float(np.max(np.abs(b))))
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= rtol * scale, f"max abs err {err:.3e} > {rtol:.1e} * {scale:.3e}"


def _problem(rng, batch=2, L=37, H=4, P=8, N=16, G=2):
    x = rng.standard_normal((batch, L, H, P))
    raw = rng.normal(-1.0, 2.0, (batch, L, H))
    A = -np.exp(rng.uniform(0, math.log(16.0), H))
    B = rng.standard_normal((batch, L, G, N)) / math.sqrt(N)
    C = rng.standard_normal((batch, L, G, N)) / math.sqrt(N)
    D = rng.normal(1.0, 0.1, H)
    h0 = rng.normal(0.0, 0.5, (batch, H, P, N))
    return x, raw, A, B, C, D, h0


def test_theorem1_gate_under_zoh_and_softplus():
    """N = 1, A = -1, B = C = 1, D = 0, Delta = softplus(z): the layer is the
    gate h_t = (1 - s(z_t)) h_{t-1} + s(z_t) x_t, y_t = h_t, s the logistic."""
    rng = np.random.default_rng(11)
    L = 200
    z = rng.normal(0.0, 3.0, (1, L, 1))
    x = rng.standard_normal((1, L, 1, 1))
    A = np.array([-1.0])
    ones = np.ones((1, L, 1, 1))
    h0 = np.array([0.7]).reshape(1, 1, 1, 1)
    y, hf = oracle.ssd_forward_ex(x, z, A, ones, ones, None, h0,
                                  oracle.DtOptions(softplus=True, zoh=True))
    h = 0.7
    ref = np.empty(L)
    for t in range(L):
        g = 1.0 / (1.0 + math.exp(-z[0, t, 0]))
        h = (1.0 - g) * h + g * x[0, t, 0, 0]
        ref[t] = h
    _close(y.reshape(L), ref)
    _close(hf.reshape(1), np.array([h]))


def test_theorem1_needs_the_hold_weight():
    """With the Euler weight (dt, not 1 - exp(-dt)) the same inputs are not
    the gate: the hold rule is what makes theorem 1 exact."""
    z = np.array([[[1.5]]])
    x = np.ones((1, 1, 1, 1))
    ones = np.ones((1, 1, 1, 1))
    y_euler, _ = oracle.ssd_forward_ex(x, z, np.array([-1.0]), ones, ones,
                                       opts=oracle.DtOptions(softplus=True))
    g = 1.0 / (1.0 + math.exp(-1.5))
    assert abs(float(y_euler.reshape(())) - g) > 0.1


@pytest.mark.parametrize("dt,A", [(0.01, -1.0), (0.3, -16.0), (2.0, -0.5), (1e-4, -3.0),
                                  (0.7, 0.0), (0.7, -1e-9), (0.2, 0.8)])
def test_hold_weight_is_the_integral_of_the_decay(dt, A):
    """Zero-order hold: B_bar = (int_0^dt exp(A s) ds) B, i.e. the weight is
    (exp(dt A) - 1) / A; checked by composite Simpson quadrature."""
    _, _, w = oracle.dt_prepare(np.array([[[dt]]]), np.array([A]), oracle.DtOptions(zoh=True))
    n = 2000
    s = np.linspace(0.0, dt, n + 1)
    f = np.exp(A * s)
    simpson = dt / (3 * n) * (f[0] + f[-1] + 4 * f[1:-1:2].sum() + 2 * f[2:-1:2].sum())
    assert abs(float(w.reshape(())) - simpson) <= 1e-12 * max(1.0, abs(simpson))


def test_softplus_matches_logaddexp_and_limits():
    v = np.concatenate([np.linspace(-40, 40, 161), [-700.0, 0.0, 700.0]]).reshape(1, -1, 1)
    dt, ell, w = oracle.dt_prepare(v, np.array([-2.0]), oracle.DtOptions(softplus=True))
    ref = np.logaddexp(0.0, v)
    _close(dt, ref, 1e-15)
    assert dt[0, -2, 0] == math.log(2.0)
    assert dt[0, -1, 0] == 700.0          # softplus(v) -> v
    assert 0.0 < dt[0, 0, 0] <= math.exp(-40.0) * (1 + 1e-15)  # -> exp(v)
    _close(ell, -2.0 * dt, 1e-15)
    _close(w, dt, 0.0)                    # Euler weight = dt


def test_bias_is_added_before_softplus_per_head():
    rng = np.random.default_rng(5)
    x, raw, A, B, C, D, h0 = _problem(rng)
    bias = rng.normal(0.0, 1.0, A.shape)
    opts = oracle.DtOptions(bias=bias, softplus=True)
    y, hf = oracle.ssd_forward_ex(x, raw, A, B, C, D, h0, opts)
    dt = np.logaddexp(0.0, raw + bias[None, None, :])
    y_ref, hf_ref = oracle.ssd_forward(x, dt, A, B, C, D, h0)
    _close(y, y_ref)
    _close(hf, hf_ref)


def test_clamp_bounds_the_step_after_softplus():
    rng = np.random.default_rng(6)
    x, raw, A, B, C, D, h0 = _problem(rng)
    opts = oracle.DtOptions(softplus=True, dt_min=0.05, dt_max=0.5)
    dt, _, _ = oracle.dt_prepare(raw, A, opts)
    assert dt.min() >= 0.05 and dt.max() <= 0.5
    assert (dt == 0.05).any() and (dt == 0.5).any()
    y, hf = oracle.ssd_forward_ex(x, raw, A, B, C, D, h0, opts)
    y_ref, hf_ref = oracle.ssd_forward(x, np.clip(np.logaddexp(0.0, raw), 0.05, 0.5), A, B, C,
                                       D, h0)
    _close(y, y_ref)
    _close(hf, hf_ref)


def test_default_options_are_the_plain_layer():
    rng = np.random.default_rng(7)
    x, raw, A, B, C, D, h0 = _problem(rng)
    dt = np.abs(raw) + 1e-3
    y, hf = oracle.ssd_forward_ex(x, dt, A, B, C, D, h0)
    y_ref, hf_ref = oracle.ssd_forward(x, dt, A, B, C, D, h0)
    assert np.array_equal(y, y_ref) and np.array_equal(hf, hf_ref)


def test_hold_forward_is_the_recurrence_with_the_hold_weight():
    """ZOH changes only the input weight; the decay stays exp(dt A)."""
    rng = np.random.default_rng(8)
    x, raw, A, B, C, D, h0 = _problem(rng)
    opts = oracle.DtOptions(softplus=True, zoh=True)
    y, hf = oracle.ssd_forward_ex(x, raw, A, B, C, D, h0, opts)
    dt = np.logaddexp(0.0, raw)
    w = (np.exp(dt * A[None, None, :]) - 1.0) / A[None, None, :]
    y_ref, hf_ref = oracle.quadratic(x, dt * A[None, None, :], w, B, C, D, h0)
    _close(y, y_ref, 1e-11)
    _close(hf, hf_ref, 1e-11)


def test_decode_steps_with_options_reproduce_forward():
    rng = np.random.default_rng(9)
    x, raw, A, B, C, D, h0 = _problem(rng, L=12)
    opts = oracle.DtOptions(bias=rng.normal(0, 1, A.shape), softplus=True, dt_min=0.01,
                            dt_max=2.0, zoh=True)
    y, hf = oracle.ssd_forward_ex(x, raw, A, B, C, D, h0, opts)
    h = h0.copy()
    for t in range(x.shape[1]):
        yt, h = oracle.ssd_step_ex(h, x[:, t], raw[:, t], A, B[:, t], C[:, t], D, opts)
        _close(yt, y[:, t])
    _close(h, hf)
