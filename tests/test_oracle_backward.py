"""Pins of the oracle's backward pass: the adjoint of the recurrence against
central finite differences of the oracle's forward (p1 "把 SSM 写成一个矩阵":
the layer is a fixed function of its inputs; its derivative is fixed by the
forward alone), for the scalar loss sum dy . y + sum dh_final . h_final.
The finite differences share no code with the adjoint, so a dropped term, a
wrong decay index or a missing group sum in it fails here."""
import math

import numpy as np
import pytest

import oracle


def _problem(rng, batch=2, L=7, H=4, P=3, N=4, G=2):
    return dict(x=rng.standard_normal((batch, L, H, P)),
                dt=np.log1p(np.exp(rng.normal(-1.0, 0.7, (batch, L, H)))),
                A=-np.exp(rng.uniform(0, math.log(4.0), H)),
                B=rng.standard_normal((batch, L, G, N)) / math.sqrt(N),
                C=rng.standard_normal((batch, L, G, N)) / math.sqrt(N),
                D=rng.normal(1.0, 0.1, H), h0=rng.normal(0.0, 0.5, (batch, H, P, N)))


def _loss(p, dy, dhf):
    y, hf = oracle.ssd_forward(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["h0"])
    return float((y * dy).sum() + (hf * dhf).sum())


@pytest.mark.parametrize("G", [1, 2])
def test_backward_matches_central_differences(G):
    rng = np.random.default_rng(10 + G)
    p = _problem(rng, G=G)
    dy = rng.standard_normal(p["x"].shape)
    dhf = rng.standard_normal(p["h0"].shape)
    g = oracle.ssd_backward(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["h0"], dy, dhf)
    names = {"x": "dx", "dt": "ddt", "A": "dA", "B": "dB", "C": "dC", "D": "dD", "h0": "dh0"}
    eps = 1e-6
    for k, gk in names.items():
        num = np.empty_like(p[k])
        flat = p[k].reshape(-1)
        for i in range(flat.size):
            old = flat[i]
            flat[i] = old + eps
            lp = _loss(p, dy, dhf)
            flat[i] = old - eps
            lm = _loss(p, dy, dhf)
            flat[i] = old
            num.reshape(-1)[i] = (lp - lm) / (2 * eps)
        scale = max(1.0, float(np.abs(num).max()))
        err = float(np.abs(g[gk] - num).max())
        assert err <= 1e-7 * scale, (k, err, scale)


def test_backward_of_zero_cotangent_is_zero():
    rng = np.random.default_rng(3)
    p = _problem(rng)
    g = oracle.ssd_backward(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["h0"],
                            np.zeros_like(p["x"]), None)
    for v in g.values():
        assert not np.any(v)
