"""Pins of the oracle's selective scan (diagonal A per channel; "精读笔记 #12：
Mamba", sections 2.2 and 3, algorithm 2), each independent of its code:

* a diagonal A that is the same for every state index is the scalar-decay
  layer with one channel per head ("Mamba-2 — 注意力的远亲", section
  "把 A 简化成一个数"): the separately written SSD recurrence must agree;
* the unrolled matrix form y_t = sum_s C_t^T A_t...A_{s+1} B_s x_s (section
  "把 SSM 写成一个矩阵") with diagonal A, written out here with products;
* the N states of a channel are independent: the scan equals the sum of N
  one-state scans;
* theorem 1 (section 3.5): N = 1, A = -1, B = 1, softplus step, zero-order
  hold gives the gate (1 - s(z)) h + s(z) x;
* constant inputs: a geometric series.
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


def _problem(rng, batch=2, L=23, D=6, N=5, G=2):
    return dict(x=rng.standard_normal((batch, L, D)),
                dt=rng.normal(-1.0, 1.5, (batch, L, D)),
                A=-np.exp(rng.uniform(0, math.log(16.0), (D, N))),
                B=rng.standard_normal((batch, L, G, N)) / math.sqrt(N),
                C=rng.standard_normal((batch, L, G, N)) / math.sqrt(N),
                Dskip=rng.normal(1.0, 0.1, D), h0=rng.normal(0.0, 0.5, (batch, D, N)),
                bias=rng.normal(0.0, 0.5, D))


OPTS = [dict(softplus=True), dict(softplus=True, zoh=True),
        dict(softplus=True, zoh=True, dt_min=0.05, dt_max=0.6)]


@pytest.mark.parametrize("o", OPTS)
def test_constant_diagonal_is_the_scalar_decay_layer(o):
    rng = np.random.default_rng(1)
    p = _problem(rng)
    A = np.repeat(p["A"][:, :1], p["A"].shape[1], axis=1)  # A[d][n] = A[d][0]
    opts = oracle.DtOptions(bias=p["bias"], **o)
    y, hf = oracle.selective_scan(p["x"], p["dt"], A, p["B"], p["C"], p["Dskip"], p["h0"], opts)
    b, L, D = p["x"].shape
    y2, hf2 = oracle.ssd_forward_ex(p["x"][..., None], p["dt"], A[:, 0], p["B"], p["C"],
                                    p["Dskip"], p["h0"][:, :, None, :], opts)
    _close(y, y2[..., 0])
    _close(hf, hf2[:, :, 0, :])


@pytest.mark.parametrize("o", OPTS[:2])
def test_matrix_form_with_diagonal_A(o):
    rng = np.random.default_rng(2)
    p = _problem(rng, batch=1, L=9, D=3, N=4, G=1)
    opts = oracle.DtOptions(bias=p["bias"], **o)
    y, _ = oracle.selective_scan(p["x"], p["dt"], p["A"], p["B"], p["C"], p["Dskip"], p["h0"],
                                 opts)
    dtp, _, _ = oracle.dt_prepare(p["dt"], np.zeros(p["x"].shape[2]), opts)
    L, D, N = p["x"].shape[1], p["x"].shape[2], p["A"].shape[1]
    ref = np.zeros((L, D))
    for d in range(D):
        for t in range(L):
            acc = 0.0
            for n in range(N):
                Adn = p["A"][d, n]
                a = np.exp(dtp[0, :, d] * Adn)
                w = np.expm1(dtp[0, :, d] * Adn) / Adn if o.get("zoh") else dtp[0, :, d]
                # initial state carried through a_0 ... a_t
                acc += p["C"][0, t, 0, n] * np.prod(a[:t + 1]) * p["h0"][0, d, n]
                for s in range(t + 1):
                    acc += (p["C"][0, t, 0, n] * np.prod(a[s + 1:t + 1]) * w[s]
                            * p["B"][0, s, 0, n] * p["x"][0, s, d])
            ref[t, d] = acc + p["Dskip"][d] * p["x"][0, t, d]
    _close(y[0], ref)


def test_state_indices_are_independent():
    rng = np.random.default_rng(3)
    p = _problem(rng)
    opts = oracle.DtOptions(bias=p["bias"], softplus=True, zoh=True)
    y, hf = oracle.selective_scan(p["x"], p["dt"], p["A"], p["B"], p["C"], p["Dskip"], p["h0"],
                                  opts)
    N = p["A"].shape[1]
    y_sum = p["Dskip"][None, None, :] * p["x"]
    for n in range(N):
        yn, hn = oracle.selective_scan(p["x"], p["dt"], p["A"][:, n:n + 1],
                                       p["B"][..., n:n + 1], p["C"][..., n:n + 1], None,
                                       p["h0"][..., n:n + 1], opts)
        y_sum = y_sum + yn
        _close(hn[..., 0], hf[..., n])
    _close(y, y_sum)


def test_theorem1_gate():
    rng = np.random.default_rng(4)
    L = 100
    z = rng.normal(0.0, 3.0, (1, L, 1))
    x = rng.standard_normal((1, L, 1))
    ones = np.ones((1, L, 1, 1))
    y, _ = oracle.selective_scan(x, z, np.array([[-1.0]]), ones, ones,
                                 opts=oracle.DtOptions(softplus=True, zoh=True))
    h, ref = 0.0, np.empty(L)
    for t in range(L):
        g = 1.0 / (1.0 + math.exp(-z[0, t, 0]))
        h = (1.0 - g) * h + g * x[0, t, 0]
        ref[t] = h
    _close(y.reshape(L), ref)


def test_constant_inputs_geometric_series():
    L, dt, A, xv, Bv, Cv = 40, 0.3, -2.0, 1.5, 0.7, -1.2
    y, _ = oracle.selective_scan(np.full((1, L, 1), xv), np.full((1, L, 1), dt),
                                 np.array([[A]]), np.full((1, L, 1, 1), Bv),
                                 np.full((1, L, 1, 1), Cv), opts=oracle.DtOptions(zoh=True))
    a = math.exp(dt * A)
    w = (a - 1.0) / A
    t = np.arange(L)
    _close(y.reshape(L), Cv * Bv * w * xv * (1.0 - a ** (t + 1)) / (1.0 - a))
