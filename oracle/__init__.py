"""fp64 CPU oracle for the scalar-decay selective SSM layer (SSD).

TEST INFRASTRUCTURE ONLY. The tests, the package smoke check and the
benchmark's CPU-baseline leg are the only callers; the product path never
imports this package, and it imports nothing from the product package.

The arithmetic lives in ``ssd_oracle.c`` (plain C, IEEE fp64, OpenMP over
independent (batch, head) lanes). This module only marshals numpy arrays.
Each function states which passage of the pages it restates:

* ``scan`` / ``ssd_forward`` / ``ssd_step`` — the sequential recurrence,
  "Mamba-2 — 注意力的远亲", sections "把 SSM 写成一个矩阵",
  "把 A 简化成一个数" and "跟着四个 token 算一次" (update the state, then read
  it), with the decay exp(dt*A) of "精读笔记 #12：Mamba", section 2.2.
* ``quadratic`` / ``matrix`` — the brute-force form M = L o (C B^T),
  same page, section "把 A 简化成一个数".
* ``chunked`` — the block decomposition of "两条路各走一半" and
  "Mamba-2 模型解读", sections 6.1 / 6.2.
* ``selective_scan`` — the diagonal-A selective scan of "精读笔记 #12：Mamba",
  sections 2.2 and 3 (the prior art of the SSD pages).
* ``dt_prepare`` / ``ssd_forward_ex`` / ``ssd_step_ex`` — the step options:
  a per-head bias, softplus ("精读笔记 #12：Mamba", section 3, algorithm 2), a
  clamp, and the zero-order-hold input weight of section 2.2.

Arrays are float64, C-contiguous, with the layouts
x, y (batch, L, H, P); dt, ell, w (batch, L, H); B, C (batch, L, G, N);
A, D (H,); states (batch, H, P, N).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile ssd_oracle.c into liboracle.so (gcc, -O2, OpenMP, no fast-math)."""
    from .build_lib import build_oracle

    return build_oracle(force=force)


def _load():
    global _lib
    if _lib is not None:
        return _lib
    src = os.path.join(_HERE, "ssd_oracle.c")
    if (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        build()
    lib = ctypes.CDLL(_LIB_PATH)
    sig = {
        "oracle_scan": [_I64] * 6 + [_D] * 9 + [ctypes.c_int],
        "oracle_ssd_forward": [_I64] * 6 + [_D] * 9 + [ctypes.c_int],
        "oracle_ssd_step": [_I64] * 5 + [_D] * 8 + [ctypes.c_int],
        "oracle_matrix": [_I64] * 7 + [_D] * 5,
        "oracle_quadratic": [_I64] * 6 + [_D] * 9 + [ctypes.c_int],
        "oracle_chunked": [_I64] * 7 + [_D] * 11 + [ctypes.c_int],
        "oracle_max_threads": [ctypes.c_int],
        "oracle_dt_prepare": [_I64] * 3 + [_D] * 3 + [ctypes.c_int, ctypes.c_double,
                                                      ctypes.c_double, ctypes.c_int] + [_D] * 3,
        "oracle_ssd_forward_ex": [_I64] * 6 + [_D] * 8 + [ctypes.c_int, ctypes.c_double,
                                                          ctypes.c_double, ctypes.c_int]
        + [_D] * 2 + [ctypes.c_int],
        "oracle_selective_scan": [_I64] * 5 + [_D] * 8 + [ctypes.c_int, ctypes.c_double,
                                                          ctypes.c_double, ctypes.c_int]
        + [_D] * 2 + [ctypes.c_int],
        "oracle_ssd_backward": [_I64] * 6 + [_D] * 16,
        "oracle_ssd_step_ex": [_I64] * 5 + [_D] * 7 + [_D, ctypes.c_int, ctypes.c_double,
                                                       ctypes.c_double, ctypes.c_int, _D,
                                                       ctypes.c_int],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    _lib = lib
    return lib


def max_threads(nthreads: int = 0) -> int:
    """Threads an oracle call uses for ``nthreads`` (0 = the OpenMP default)."""
    return int(_load().oracle_max_threads(int(nthreads)))


def _p(a):
    if a is None:
        return None
    return a.ctypes.data_as(_D)


def _f64(a, shape=None, name="array"):
    if a is None:
        return None
    a = np.ascontiguousarray(a, dtype=np.float64)
    if shape is not None and a.shape != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {a.shape}")
    return a


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"{what} failed with oracle status {rc}")


def _dims(x, B):
    batch, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    return batch, L, H, P, N, G


def scan(x, ell, w, B, C, D=None, h0=None, nthreads: int = 0):
    """Recurrence with per-step log-decay ``ell`` (a_t = exp(ell_t)) and input
    weight ``w``: h_t = a_t h_{t-1} + w_t x_t (x) B_t, y_t = C_t . h_t + D x_t.

    Returns (y, h_final)."""
    x = _f64(x, name="x")
    batch, L, H, P = x.shape
    B = _f64(B, name="B")
    G, N = B.shape[2], B.shape[3]
    ell = _f64(ell, (batch, L, H), "ell")
    w = _f64(w, (batch, L, H), "w")
    C = _f64(C, (batch, L, G, N), "C")
    D = _f64(D, (H,), "D")
    h0 = _f64(h0, (batch, H, P, N), "h0")
    y = np.empty((batch, L, H, P))
    hf = np.empty((batch, H, P, N))
    rc = _load().oracle_scan(batch, L, H, P, N, G, _p(x), _p(ell), _p(w), _p(B), _p(C),
                             _p(D), _p(h0), _p(y), _p(hf), int(nthreads))
    _check(rc, "oracle_scan")
    return y, hf


def ssd_forward(x, dt, A, B, C, D=None, h0=None, nthreads: int = 0):
    """The layer forward: the recurrence with a_t = exp(dt_t A_h), w_t = dt_t.

    Returns (y, h_final)."""
    x = _f64(x, name="x")
    batch, L, H, P = x.shape
    B = _f64(B, name="B")
    G, N = B.shape[2], B.shape[3]
    dt = _f64(dt, (batch, L, H), "dt")
    A = _f64(A, (H,), "A")
    C = _f64(C, (batch, L, G, N), "C")
    D = _f64(D, (H,), "D")
    h0 = _f64(h0, (batch, H, P, N), "h0")
    y = np.empty((batch, L, H, P))
    hf = np.empty((batch, H, P, N))
    rc = _load().oracle_ssd_forward(batch, L, H, P, N, G, _p(x), _p(dt), _p(A), _p(B),
                                    _p(C), _p(D), _p(h0), _p(y), _p(hf), int(nthreads))
    _check(rc, "oracle_ssd_forward")
    return y, hf


def ssd_step(h, x, dt, A, B, C, D=None, nthreads: int = 0):
    """One decode step. h (batch,H,P,N) is NOT modified; returns (y, h_new).

    x (batch,H,P), dt (batch,H), B/C (batch,G,N)."""
    h_new = np.array(h, dtype=np.float64, order="C", copy=True)
    batch, H, P, N = h_new.shape
    x = _f64(x, (batch, H, P), "x")
    dt = _f64(dt, (batch, H), "dt")
    A = _f64(A, (H,), "A")
    B = _f64(B, name="B")
    G = B.shape[1]
    B = _f64(B, (batch, G, N), "B")
    C = _f64(C, (batch, G, N), "C")
    D = _f64(D, (H,), "D")
    y = np.empty((batch, H, P))
    rc = _load().oracle_ssd_step(batch, H, P, N, G, _p(h_new), _p(x), _p(dt), _p(A),
                                 _p(B), _p(C), _p(D), _p(y), int(nthreads))
    _check(rc, "oracle_ssd_step")
    return y, h_new


class DtOptions:
    """Step options of the layer: raw step dt -> dt + bias[h] -> softplus ->
    clamp to [dt_min, dt_max] (when dt_max > 0); input weight dt (Euler) or
    the zero-order hold (exp(dt A) - 1) / A ("精读笔记 #12：Mamba", sections 2.2
    and 3). The defaults leave dt and the layer unchanged."""

    def __init__(self, bias=None, softplus: bool = False, dt_min: float = 0.0,
                 dt_max: float = 0.0, zoh: bool = False):
        self.bias = bias
        self.softplus = bool(softplus)
        self.dt_min = float(dt_min)
        self.dt_max = float(dt_max)
        self.zoh = bool(zoh)

    def _args(self, H):
        return (_f64(self.bias, (H,), "bias"), int(self.softplus), self.dt_min, self.dt_max,
                int(self.zoh))


def dt_prepare(dt_raw, A, opts: DtOptions):
    """Prepared steps of ``dt_raw`` (batch, L, H): returns (dt, ell, w) with
    ell = dt A the log-decay and w the input weight."""
    dt_raw = _f64(dt_raw, name="dt_raw")
    batch, L, H = dt_raw.shape
    A = _f64(A, (H,), "A")
    bias, sp, lo, hi, zoh = opts._args(H)
    dt = np.empty_like(dt_raw)
    ell = np.empty_like(dt_raw)
    w = np.empty_like(dt_raw)
    rc = _load().oracle_dt_prepare(batch, L, H, _p(dt_raw), _p(A), _p(bias), sp, lo, hi, zoh,
                                   _p(dt), _p(ell), _p(w))
    _check(rc, "oracle_dt_prepare")
    return dt, ell, w


def ssd_forward_ex(x, dt_raw, A, B, C, D=None, h0=None, opts: DtOptions = None,
                   nthreads: int = 0):
    """The layer forward on raw steps prepared by ``opts`` (see DtOptions).

    Returns (y, h_final)."""
    opts = opts or DtOptions()
    x = _f64(x, name="x")
    batch, L, H, P = x.shape
    B = _f64(B, name="B")
    G, N = B.shape[2], B.shape[3]
    dt_raw = _f64(dt_raw, (batch, L, H), "dt_raw")
    A = _f64(A, (H,), "A")
    C = _f64(C, (batch, L, G, N), "C")
    D = _f64(D, (H,), "D")
    h0 = _f64(h0, (batch, H, P, N), "h0")
    bias, sp, lo, hi, zoh = opts._args(H)
    y = np.empty((batch, L, H, P))
    hf = np.empty((batch, H, P, N))
    rc = _load().oracle_ssd_forward_ex(batch, L, H, P, N, G, _p(x), _p(dt_raw), _p(A), _p(B),
                                       _p(C), _p(D), _p(h0), _p(bias), sp, lo, hi, zoh, _p(y),
                                       _p(hf), int(nthreads))
    _check(rc, "oracle_ssd_forward_ex")
    return y, hf


def ssd_step_ex(h, x, dt_raw, A, B, C, D=None, opts: DtOptions = None, nthreads: int = 0):
    """One decode step on a raw step prepared by ``opts``. h is NOT modified;
    returns (y, h_new)."""
    opts = opts or DtOptions()
    h_new = np.array(h, dtype=np.float64, order="C", copy=True)
    batch, H, P, N = h_new.shape
    x = _f64(x, (batch, H, P), "x")
    dt_raw = _f64(dt_raw, (batch, H), "dt_raw")
    A = _f64(A, (H,), "A")
    B = _f64(B, name="B")
    G = B.shape[1]
    B = _f64(B, (batch, G, N), "B")
    C = _f64(C, (batch, G, N), "C")
    D = _f64(D, (H,), "D")
    bias, sp, lo, hi, zoh = opts._args(H)
    y = np.empty((batch, H, P))
    rc = _load().oracle_ssd_step_ex(batch, H, P, N, G, _p(h_new), _p(x), _p(dt_raw), _p(A),
                                    _p(B), _p(C), _p(D), _p(bias), sp, lo, hi, zoh, _p(y),
                                    int(nthreads))
    _check(rc, "oracle_ssd_step_ex")
    return y, h_new


def ssd_backward(x, dt, A, B, C, D, h0, dy, dh_final=None):
    """Gradients of sum dy . y + sum dh_final . h_final for the plain layer
    forward (the exact adjoint of the recurrence). Returns a dict with dx,
    ddt, dA, dB, dC, dD, dh0."""
    x = _f64(x, name="x")
    batch, L, H, P = x.shape
    B = _f64(B, name="B")
    G, N = B.shape[2], B.shape[3]
    dt = _f64(dt, (batch, L, H), "dt")
    A = _f64(A, (H,), "A")
    C = _f64(C, (batch, L, G, N), "C")
    D = _f64(D, (H,), "D")
    h0 = _f64(h0, (batch, H, P, N), "h0")
    dy = _f64(dy, (batch, L, H, P), "dy")
    dh_final = _f64(dh_final, (batch, H, P, N), "dh_final")
    out = dict(dx=np.empty_like(x), ddt=np.empty((batch, L, H)), dA=np.empty(H),
               dB=np.empty((batch, L, G, N)), dC=np.empty((batch, L, G, N)), dD=np.empty(H),
               dh0=np.empty((batch, H, P, N)))
    rc = _load().oracle_ssd_backward(batch, L, H, P, N, G, _p(x), _p(dt), _p(A), _p(B), _p(C),
                                     _p(D), _p(h0), _p(dy), _p(dh_final), _p(out["dx"]),
                                     _p(out["ddt"]), _p(out["dA"]), _p(out["dB"]),
                                     _p(out["dC"]), _p(out["dD"]), _p(out["dh0"]))
    _check(rc, "oracle_ssd_backward")
    return out


def selective_scan(x, dt_raw, A, B, C, Dskip=None, h0=None, opts: DtOptions = None,
                   nthreads: int = 0):
    """The selective scan with a diagonal A per channel ("精读笔记 #12：Mamba",
    sections 2.2 and 3): x, dt_raw (batch, L, D); A (D, N); B, C
    (batch, L, G, N); Dskip (D,); h0 (batch, D, N). Steps prepared by ``opts``
    (bias per channel). Returns (y (batch, L, D), h_final (batch, D, N))."""
    opts = opts or DtOptions()
    x = _f64(x, name="x")
    batch, L, Dc = x.shape
    A = _f64(A, name="A")
    N = A.shape[1]
    B = _f64(B, name="B")
    G = B.shape[2]
    dt_raw = _f64(dt_raw, (batch, L, Dc), "dt_raw")
    A = _f64(A, (Dc, N), "A")
    B = _f64(B, (batch, L, G, N), "B")
    C = _f64(C, (batch, L, G, N), "C")
    Dskip = _f64(Dskip, (Dc,), "Dskip")
    h0 = _f64(h0, (batch, Dc, N), "h0")
    bias, sp, lo, hi, zoh = opts._args(Dc)
    y = np.empty((batch, L, Dc))
    hf = np.empty((batch, Dc, N))
    rc = _load().oracle_selective_scan(batch, L, Dc, N, G, _p(x), _p(dt_raw), _p(A), _p(B),
                                       _p(C), _p(Dskip), _p(h0), _p(bias), sp, lo, hi, zoh,
                                       _p(y), _p(hf), int(nthreads))
    _check(rc, "oracle_selective_scan")
    return y, hf


def matrix(ell, w, B, C, b: int, h: int):
    """The L x L sequence-transformation matrix M of lane (b, h):
    M_ts = exp(sum_{k=s+1..t} ell_k) (C_t . B_s) w_s for s <= t, else 0."""
    ell = _f64(ell, name="ell")
    batch, L, H = ell.shape
    B = _f64(B, name="B")
    G, N = B.shape[2], B.shape[3]
    w = _f64(w, (batch, L, H), "w")
    C = _f64(C, (batch, L, G, N), "C")
    M = np.empty((L, L))
    rc = _load().oracle_matrix(batch, L, H, N, G, int(b), int(h), _p(ell), _p(w), _p(B),
                               _p(C), _p(M))
    _check(rc, "oracle_matrix")
    return M


def quadratic(x, ell, w, B, C, D=None, h0=None, nthreads: int = 0):
    """Brute-force quadratic form (materialised M per lane). Returns (y, h_final)."""
    x = _f64(x, name="x")
    batch, L, H, P = x.shape
    B = _f64(B, name="B")
    G, N = B.shape[2], B.shape[3]
    ell = _f64(ell, (batch, L, H), "ell")
    w = _f64(w, (batch, L, H), "w")
    C = _f64(C, (batch, L, G, N), "C")
    D = _f64(D, (H,), "D")
    h0 = _f64(h0, (batch, H, P, N), "h0")
    y = np.empty((batch, L, H, P))
    hf = np.empty((batch, H, P, N))
    rc = _load().oracle_quadratic(batch, L, H, P, N, G, _p(x), _p(ell), _p(w), _p(B), _p(C),
                                  _p(D), _p(h0), _p(y), _p(hf), int(nthreads))
    _check(rc, "oracle_quadratic")
    return y, hf


def chunked(x, ell, w, B, C, Q: int, D=None, h0=None, stages: bool = False,
            nthreads: int = 0):
    """Chunked fp64 form with block length Q. Returns (y, h_final), or with
    ``stages`` (y, h_final, S, Hs) where S[b,h,c] is chunk c's own state and
    Hs[b,h,c] the state entering chunk c."""
    x = _f64(x, name="x")
    batch, L, H, P = x.shape
    B = _f64(B, name="B")
    G, N = B.shape[2], B.shape[3]
    ell = _f64(ell, (batch, L, H), "ell")
    w = _f64(w, (batch, L, H), "w")
    C = _f64(C, (batch, L, G, N), "C")
    D = _f64(D, (H,), "D")
    h0 = _f64(h0, (batch, H, P, N), "h0")
    nc = (L + Q - 1) // Q
    y = np.empty((batch, L, H, P))
    hf = np.empty((batch, H, P, N))
    S = np.empty((batch, H, nc, P, N)) if stages else None
    Hs = np.empty((batch, H, nc, P, N)) if stages else None
    rc = _load().oracle_chunked(batch, L, H, P, N, G, int(Q), _p(x), _p(ell), _p(w), _p(B),
                                _p(C), _p(D), _p(h0), _p(y), _p(hf), _p(S), _p(Hs),
                                int(nthreads))
    _check(rc, "oracle_chunked")
    if stages:
        return y, hf, S, Hs
    return y, hf
