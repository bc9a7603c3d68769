"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Every check here is independent of the oracle's own code path: printed values
from the pages, closed forms, limits, a rank property, and agreement between
the oracle's three separately written forms (recurrence, brute-force matrix,
chunked) and the decode step. A dropped term, a wrong sign or index, or a
transposed operand in any of them fails at least one test below.
"""
import math

import numpy as np
import pytest

import oracle
from tests.conftest import read_golden

RTOL = 1e-12


def _rand_problem(rng, batch, L, H, P, N, G, h0=True, D=True):
    x = rng.standard_normal((batch, L, H, P))
    dt = np.log1p(np.exp(rng.normal(-2.0, 1.0, (batch, L, H))))
    A = -np.exp(rng.uniform(0, math.log(16.0), H))
    B = rng.standard_normal((batch, L, G, N)) / math.sqrt(N)
    C = rng.standard_normal((batch, L, G, N)) / math.sqrt(N)
    Dv = rng.normal(1.0, 0.1, H) if D else None
    h0v = rng.normal(0.0, 0.5, (batch, H, P, N)) if h0 else None
    return x, dt, A, B, C, Dv, h0v


def _ell(dt, A):
    return dt * A[None, None, :]


def _close(a, b, rtol=RTOL):
    scale = max(1.0, float(np.max(np.abs(b))))
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= rtol * scale, f"max abs err {err:.3e} > {rtol:.1e} * {scale:.3e}"


# ---------------------------------------------------------------------------
# P1: the pages' worked four-token example (printed values)
# ---------------------------------------------------------------------------

def _worked():
    g = read_golden("worked_example_4tok.txt")
    x = g["x"].reshape(1, 4, 1, 1)
    ell = np.log(g["a"]).reshape(1, 4, 1)
    w = np.ones((1, 4, 1))
    B = g["B"].reshape(1, 4, 1, 2)
    C = g["C"].reshape(1, 4, 1, 2)
    return g, x, ell, w, B, C


def test_worked_example_recurrence_matches_printed_y():
    g, x, ell, w, B, C = _worked()
    y, hf = oracle.scan(x, ell, w, B, C)
    _close(y.reshape(4), g["y_recurrence"], 1e-12)
    # the state after the fourth token follows from the same printed inputs:
    # h = 0.7*[3.4, 4.6] + 4*[1, -1]
    _close(hf.reshape(2), np.array([6.38, -0.78]), 1e-12)


def test_worked_example_matrix_form_matches_printed_y():
    g, x, ell, w, B, C = _worked()
    y, _ = oracle.quadratic(x, ell, w, B, C)
    _close(y.reshape(4), g["y_matrix"], 1e-12)
    M = oracle.matrix(ell, w, B, C, 0, 0)
    _close(M @ g["x"], g["y_matrix"], 1e-12)


def test_worked_example_decay_mask_matches_printed_L():
    g, x, ell, w, B, C = _worked()
    # With N = 1 and B = C = 1, w = 1 the matrix M is the decay mask L itself.
    ones = np.ones((1, 4, 1, 1))
    L = oracle.matrix(ell, w, ones, ones, 0, 0)
    _close(L, g["L"], 1e-12)
    assert abs(L[3, 0] - 0.5 * 0.8 * 0.7) < 1e-15


def test_worked_example_chunked_and_step_forms():
    g, x, ell, w, B, C = _worked()
    for Q in (1, 2, 3, 4):
        y, _ = oracle.chunked(x, ell, w, B, C, Q)
        _close(y.reshape(4), g["y_recurrence"], 1e-12)


# ---------------------------------------------------------------------------
# P2: recurrence == brute-force quadratic form (independent code paths)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("G", [1, 2])
@pytest.mark.parametrize("L", [1, 7, 33])
def test_recurrence_equals_quadratic(G, L):
    rng = np.random.default_rng(100 + G * 10 + L)
    x, dt, A, B, C, D, h0 = _rand_problem(rng, 2, L, 4, 3, 5, G)
    ell = _ell(dt, A)
    y1, h1 = oracle.scan(x, ell, dt, B, C, D, h0)
    y2, h2 = oracle.quadratic(x, ell, dt, B, C, D, h0)
    _close(y1, y2)
    _close(h1, h2)
    y3, h3 = oracle.ssd_forward(x, dt, A, B, C, D, h0)
    _close(y3, y1, 0)  # the layer forward is the scan with ell = dt*A, w = dt
    _close(h3, h1, 0)


def test_quadratic_matches_numpy_matrix_product_per_head():
    # y = M x for each head-dim column (h0 = 0, D = 0): the matrix form itself.
    rng = np.random.default_rng(7)
    x, dt, A, B, C, _, _ = _rand_problem(rng, 1, 20, 2, 3, 4, 1, h0=False, D=False)
    ell = _ell(dt, A)
    y, _ = oracle.scan(x, ell, dt, B, C)
    for h in range(2):
        M = oracle.matrix(ell, dt, B, C, 0, h)
        assert np.allclose(np.triu(M, 1), 0.0)
        _close(M @ x[0, :, h, :], y[0, :, h, :])


# ---------------------------------------------------------------------------
# P3: chunk-size invariance of the block decomposition
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("Q", [1, 2, 3, 16, 37, 50])
def test_chunked_is_chunk_invariant(Q):
    rng = np.random.default_rng(300 + Q)
    L = 37
    x, dt, A, B, C, D, h0 = _rand_problem(rng, 2, L, 4, 5, 6, 2)
    ell = _ell(dt, A)
    y0, h0f = oracle.scan(x, ell, dt, B, C, D, h0)
    y1, h1f = oracle.chunked(x, ell, dt, B, C, Q, D, h0)
    _close(y1, y0)
    _close(h1f, h0f)


def test_chunked_stage_states_equal_prefix_recurrence():
    # H_c (state entering chunk c) must be the recurrence's state after the
    # first c*Q tokens; S_c must be chunk c's state started from zero.
    rng = np.random.default_rng(11)
    L, Q = 29, 8
    x, dt, A, B, C, D, h0 = _rand_problem(rng, 1, L, 2, 3, 4, 1)
    ell = _ell(dt, A)
    _, _, S, Hs = oracle.chunked(x, ell, dt, B, C, Q, D, h0, stages=True)
    for c in range((L + Q - 1) // Q):
        t0, t1 = c * Q, min(L, c * Q + Q)
        _, hc = oracle.scan(x[:, :t0], ell[:, :t0], dt[:, :t0], B[:, :t0], C[:, :t0], D, h0)
        _close(Hs[:, :, c], hc)
        _, sc = oracle.scan(x[:, t0:t1], ell[:, t0:t1], dt[:, t0:t1], B[:, t0:t1], C[:, t0:t1])
        _close(S[:, :, c], sc)


# ---------------------------------------------------------------------------
# P4: A = 0 is linear attention, Y = Q cumsum(K^T V) (plus h0 and skip)
# ---------------------------------------------------------------------------

def test_zero_decay_is_linear_attention_cumsum():
    rng = np.random.default_rng(4)
    batch, L, H, P, N, G = 2, 19, 3, 4, 5, 1
    x, dt, _, B, C, D, h0 = _rand_problem(rng, batch, L, H, P, N, G)
    A = np.zeros(H)
    y, hf = oracle.ssd_forward(x, dt, A, B, C, D, h0)
    # K^T V accumulated over time: kv[b,t,h,p,n] = dt x_p B_n, then cumsum.
    kv = np.einsum("bth,bthp,btn->bthpn", dt, x, B[:, :, 0, :])
    state = h0[:, None] + np.cumsum(kv, axis=1)
    ref = np.einsum("btn,bthpn->bthp", C[:, :, 0, :], state) + D[None, None, :, None] * x
    _close(y, ref)
    _close(hf, state[:, -1])


# ---------------------------------------------------------------------------
# P5: constant dt, A, x, B, C (a Toeplitz decay mask): geometric series
# ---------------------------------------------------------------------------

def test_constant_inputs_geometric_series():
    L = 40
    dt0, A0, x0, B0, C0, D0 = 0.07, -2.5, 1.3, 0.8, -0.6, 0.9
    x = np.full((1, L, 1, 1), x0)
    dt = np.full((1, L, 1), dt0)
    B = np.full((1, L, 1, 1), B0)
    C = np.full((1, L, 1, 1), C0)
    y, _ = oracle.ssd_forward(x, dt, np.array([A0]), B, C, np.array([D0]))
    a = math.exp(dt0 * A0)
    t = np.arange(L)
    ref = C0 * B0 * dt0 * x0 * (1 - a ** (t + 1)) / (1 - a) + D0 * x0
    _close(y.reshape(L), ref)


# ---------------------------------------------------------------------------
# P6: gating theorem: A = -1, dt = softplus(z)  =>  a = 1 - sigmoid(z)
# ---------------------------------------------------------------------------

def test_gating_decay_is_one_minus_sigmoid():
    rng = np.random.default_rng(6)
    L = 25
    z = rng.normal(0.0, 2.0, L)
    dt = np.log1p(np.exp(z)).reshape(1, L, 1)
    x = np.zeros((1, L, 1, 1))
    B = np.ones((1, L, 1, 1))
    C = np.ones((1, L, 1, 1))
    h0 = np.ones((1, 1, 1, 1))
    y, hf = oracle.ssd_forward(x, dt, np.array([-1.0]), B, C, None, h0)
    gate = 1.0 / (1.0 + np.exp(-z))
    ref = np.cumprod(1.0 - gate)
    _close(y.reshape(L), ref, 1e-13)
    assert abs(hf.item() - ref[-1]) <= 1e-13


# ---------------------------------------------------------------------------
# P7: step-size limits: large dt resets the state, small dt keeps it
# ---------------------------------------------------------------------------

def test_large_step_erases_history():
    rng = np.random.default_rng(71)
    x, dt, A, B, C, D, h0 = _rand_problem(rng, 1, 12, 2, 3, 4, 1)
    dt[:] = 1e3
    y, hf = oracle.ssd_forward(x, dt, A, B, C, D, h0)
    # a = exp(-1000 |A|) == 0 exactly in fp64, so h_t = dt x_t (x) B_t.
    cb = np.einsum("btgn,btgn->btg", C, B)[:, :, 0]
    ref = dt * cb[:, :, None]
    ref = ref[..., None] * x + D[None, None, :, None] * x
    _close(y, ref)
    _close(hf, dt[0, -1][None, :, None, None] * x[0, -1][None, :, :, None]
           * B[0, -1, 0][None, None, None, :])


def test_small_step_keeps_state():
    rng = np.random.default_rng(72)
    x, dt, A, B, C, D, h0 = _rand_problem(rng, 1, 12, 2, 3, 4, 1)
    dt[:] = 1e-14
    y, hf = oracle.ssd_forward(x, dt, A, B, C, None, h0)
    ref = np.einsum("btn,bhpn->bthp", C[:, :, 0], h0)
    _close(y, ref, 1e-11)
    _close(hf, h0, 1e-11)
    # monotone in between: the memory of h0 shrinks as dt grows
    fracs = []
    for d in (1e-3, 1e-2, 1e-1, 1.0):
        dt[:] = d
        _, hf = oracle.ssd_forward(np.zeros_like(x), dt, A, B, C, None, h0)
        fracs.append(np.linalg.norm(hf) / np.linalg.norm(h0))
    assert all(f1 > f2 for f1, f2 in zip(fracs, fracs[1:]))


# ---------------------------------------------------------------------------
# P8: semiseparable structure: blocks below the diagonal have rank <= N
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("N", [1, 2, 3])
def test_below_diagonal_blocks_have_rank_at_most_N(N):
    rng = np.random.default_rng(80 + N)
    L = 24
    x, dt, A, B, C, _, _ = _rand_problem(rng, 1, L, 1, 1, N, 1, h0=False, D=False)
    M = oracle.matrix(_ell(dt, A), dt, B, C, 0, 0)
    for k in range(4, L - 3, 5):
        blk = M[k:, :k]
        s = np.linalg.svd(blk, compute_uv=False)
        rank = int(np.sum(s > 1e-10 * s[0]))
        assert rank <= N, (k, rank, s[: N + 2])
    # not vacuous: the whole lower triangle has rank well above N
    s = np.linalg.svd(M, compute_uv=False)
    assert int(np.sum(s > 1e-10 * s[0])) > N + 2


# ---------------------------------------------------------------------------
# P9: state carry: split sequences and decode steps reproduce the forward
# ---------------------------------------------------------------------------

def test_split_sequence_resumes_from_final_state():
    rng = np.random.default_rng(9)
    L = 41
    x, dt, A, B, C, D, h0 = _rand_problem(rng, 2, L, 4, 3, 5, 2)
    y, hf = oracle.ssd_forward(x, dt, A, B, C, D, h0)
    for L1 in (1, 13, 40):
        ya, ha = oracle.ssd_forward(x[:, :L1], dt[:, :L1], A, B[:, :L1], C[:, :L1], D, h0)
        yb, hb = oracle.ssd_forward(x[:, L1:], dt[:, L1:], A, B[:, L1:], C[:, L1:], D, ha)
        _close(np.concatenate([ya, yb], axis=1), y)
        _close(hb, hf)


def test_decode_steps_reproduce_forward():
    rng = np.random.default_rng(19)
    L = 16
    x, dt, A, B, C, D, h0 = _rand_problem(rng, 3, L, 4, 3, 5, 2)
    y, hf = oracle.ssd_forward(x, dt, A, B, C, D, h0)
    h = h0.copy()
    for t in range(L):
        yt, h = oracle.ssd_step(h, x[:, t], dt[:, t], A, B[:, t], C[:, t], D)
        _close(yt, y[:, t])
    _close(h, hf)


# ---------------------------------------------------------------------------
# P10: skip-only cases, and the head -> group map
# ---------------------------------------------------------------------------

def test_zero_B_or_C_leaves_only_skip():
    rng = np.random.default_rng(10)
    x, dt, A, B, C, D, _ = _rand_problem(rng, 1, 9, 2, 3, 4, 1)
    y, hf = oracle.ssd_forward(x, dt, A, np.zeros_like(B), C, D)
    assert np.array_equal(y, D[None, None, :, None] * x)
    assert np.array_equal(hf, np.zeros_like(hf))
    y, _ = oracle.ssd_forward(x, dt, A, B, np.zeros_like(C), D)
    assert np.array_equal(y, D[None, None, :, None] * x)


def test_heads_use_contiguous_groups():
    # Reading: head h uses group h // (H / G). With G = 2 and H = 4, heads
    # {0, 1} see group 0 and heads {2, 3} group 1.
    rng = np.random.default_rng(12)
    x, dt, A, B, C, D, h0 = _rand_problem(rng, 2, 10, 4, 3, 5, 2)
    y, hf = oracle.ssd_forward(x, dt, A, B, C, D, h0)
    for g, hs in ((0, slice(0, 2)), (1, slice(2, 4))):
        yg, hg = oracle.ssd_forward(x[:, :, hs], dt[:, :, hs], A[hs], B[:, :, g:g + 1],
                                    C[:, :, g:g + 1], D[hs], h0[:, hs])
        _close(y[:, :, hs], yg, 0)
        _close(hf[:, hs], hg, 0)


def test_empty_sequence_returns_initial_state():
    rng = np.random.default_rng(13)
    x, dt, A, B, C, D, h0 = _rand_problem(rng, 1, 0, 2, 3, 4, 1)
    y, hf = oracle.ssd_forward(x, dt, A, B, C, D, h0)
    assert y.shape == (1, 0, 2, 3)
    assert np.array_equal(hf, h0)
