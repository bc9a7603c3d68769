"""Why the tensor-core forward splits two of its operands into bf16 hi + lo
pairs: a numpy model of the chunked forward that rounds operands where the
kernel does, checked against the fp64 oracle on the 2.7B-style layer's shapes
and value distributions.

The model follows the chunked algorithm ("Mamba-2 — 注意力的远亲", section
"两条路各走一半"): per 128-token block, the masked Gram Gm = (C B^T) o L o dt
+ D I times X (the diagonal block), plus exp(cum_i) C_i H^T (the state entering
the block), rounded to bf16; then the block's chunk state (w o X)^T B with
w_j = exp(cum_end - cum_j) dt_j is added to the decayed state. The tensor
cores see bf16 (or fp16) operands and accumulate in fp32; the model rounds
each operand accordingly and keeps the rest in fp64. It imports the oracle
only as the reference and the input generator for the inputs.

CPU only; it documents the measured error budget rather than testing code:
- the output rounding alone takes most of the 2e-2 bound (max |y| is a few
  times rms(y));
- the masked Gram rounded once to bf16 adds about as much again, so its lo
  half is needed; one fp16 rounding (11 bits) would do;
- w o X rounded once to bf16 leaves y inside the bound but moves the final
  state from ~1e-5 to ~1e-2 of its rms; its lo half keeps the state tight.
"""
import math

import numpy as np
import pytest

import oracle
import synth


def bf16(a):
    """Round to the nearest bf16 (ties to even), as float64."""
    a = np.asarray(a, np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def hilo(a):
    """A bf16 hi + lo pair: hi = bf16(a), lo = bf16(a - hi)."""
    h = bf16(a)
    return h + bf16(np.asarray(a, np.float64) - h)


def f16(a):
    return np.asarray(a, np.float64).astype(np.float16).astype(np.float64)


def exact(a):
    return np.asarray(a, np.float64)


def chunked_forward(ex, rG, rW, rH, Q=128):
    """The blocked forward with the masked Gram rounded by rG, w o X by rW and
    the entering state by rH; y rounded to bf16; the carried state fp32."""
    x, dt, A, B, C, D, h0 = (ex[k] for k in ("x", "dt", "A", "B", "C", "D", "h0"))
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    y = np.zeros_like(x)
    hf = np.zeros((b, H, P, N))
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            hc = h0[bi, h].copy() if h0 is not None else np.zeros((P, N))
            for t0 in range(0, L, Q):
                sl = slice(t0, min(L, t0 + Q))
                X, Bc, Cc, d = x[bi, sl, h], B[bi, sl, g], C[bi, sl, g], dt[bi, sl, h]
                cum = np.cumsum(d * A[h])
                seg = cum[:, None] - cum[None, :]
                Lm = np.tril(np.exp(np.minimum(seg, 0.0)))
                Gm = (Cc @ Bc.T) * Lm * d[None, :] + np.diag(np.full(len(d), D[h]))
                Yd = rG(Gm) @ X
                Yo = Cc @ rH(hc.astype(np.float32)).T
                y[bi, sl, h] = bf16(Yd + np.exp(cum)[:, None] * Yo)
                wX = X * (np.exp(cum[-1] - cum) * d)[:, None]
                S = rW(wX).T @ Bc
                hc = (math.exp(cum[-1]) * hc + S).astype(np.float32).astype(np.float64)
            hf[bi, h] = hc
    return y, hf


def rel(got, ref):
    return float(np.abs(got - ref).max() / np.sqrt(np.mean(ref * ref)))


@pytest.fixture(scope="module")
def case():
    # the 2.7B-style layer's head and state shapes and distributions, 8 blocks
    w = synth.WORKLOADS["mamba2_2p7b_layer"].with_(batch=1, seqlen=1024, nheads=4, seed=55)
    ex = synth.exact_inputs(synth.forward_inputs(w), w.dtype)
    yr, hr = oracle.ssd_forward(ex["x"], ex["dt"], ex["A"], ex["B"], ex["C"], ex["D"], ex["h0"])
    return ex, yr, hr


def _errs(case, rG, rW, rH):
    ex, yr, hr = case
    y, hf = chunked_forward(ex, rG, rW, rH)
    return rel(y, yr), rel(hf, hr)


def test_model_with_exact_operands_meets_the_oracle(case):
    # the model itself is the oracle's result up to fp32 state and bf16 output
    ey, eh = _errs(case, exact, exact, exact)
    assert ey < 2e-2 and eh < 1e-5


def test_kernel_operands_stay_inside_the_bound(case):
    # as the kernel rounds: masked Gram and w o X as hi + lo, H once to bf16
    ey, eh = _errs(case, hilo, hilo, bf16)
    ey0, _ = _errs(case, exact, exact, exact)
    assert ey < 2e-2 and eh < 1e-4
    assert ey < 1.1 * ey0  # the output rounding dominates


def test_masked_gram_in_one_bf16_rounding_eats_the_margin(case):
    ey_kernel, _ = _errs(case, hilo, hilo, bf16)
    ey_hi, _ = _errs(case, bf16, hilo, bf16)
    ey_f16, _ = _errs(case, f16, hilo, bf16)
    assert ey_hi > 1.2 * ey_kernel  # the Gram's lo half carries real weight
    assert ey_f16 < 2e-2            # one fp16 rounding (11 bits) would still pass


def test_w_x_in_one_bf16_rounding_loosens_the_state(case):
    _, eh_kernel = _errs(case, hilo, hilo, bf16)
    ey_hi, eh_hi = _errs(case, hilo, bf16, bf16)
    assert ey_hi < 2e-2
    assert eh_hi > 30 * eh_kernel and eh_hi > 1e-3
