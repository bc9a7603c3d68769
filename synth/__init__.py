"""Seeded synthetic inputs for the SSD layer, shared by the tests, the benchmark
and the smoke check.

This module holds no arithmetic of the layer itself: it only draws random
inputs, rounds them to their storage type, and decodes stored values back to
exact float64 so that the oracle and the CUDA path consume bit-identical
inputs.

Value recipe (the plainest reading of the stated distributions):

* x ~ N(0, 1)
* dt = softplus(z + b_h): z ~ N(0, 0.5) (0.5 is the std), b_h drawn once per
  head so that softplus(b_h) is log-uniform in [1e-3, 1e-1]. dt enters the
  layer already positive.
* A_h = -exp(U(0, ln 16)), stored fp32.
* B, C ~ N(0, 1) / sqrt(N).
* D_h ~ N(1, 0.1) (std), stored fp32.
* h0 = 0, or N(0, 0.1) (std) for the long-sequence workload; the decode
  state h ~ N(0, 1), fp32.

Storage: fp32 arrays as numpy float32; bf16 arrays as numpy uint16 bit
patterns (round-to-nearest-even from the float64 draw).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np

F32 = "f32"
BF16 = "bf16"


# --------------------------------------------------------------------------
# storage-type rounding and exact decoding
# --------------------------------------------------------------------------

def bf16_bits(a: np.ndarray) -> np.ndarray:
    """float64 -> bf16 bit patterns (uint16), round to nearest, ties to even.

    Rounds the float64 significand straight to 8 bits (no double rounding).
    Values are assumed inside the fp32 normal range or zero, which holds for
    every distribution above."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    u = a.view(np.uint64).copy()
    # 52 - 7 = 45 significand bits are dropped.
    lsb = (u >> np.uint64(45)) & np.uint64(1)
    u = u + (np.uint64((1 << 44) - 1) + lsb)
    u &= ~np.uint64((1 << 45) - 1)
    f32 = u.view(np.float64).astype(np.float32)  # exact: 8 significant bits
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns as float64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def store(a: np.ndarray, dtype: str) -> np.ndarray:
    """Round a float64 draw to its storage type."""
    if dtype == F32:
        return np.ascontiguousarray(a, dtype=np.float32)
    if dtype == BF16:
        return bf16_bits(a)
    raise ValueError(f"unknown storage dtype {dtype!r}")


def exact(stored: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 value of a stored array."""
    if dtype == F32:
        return np.asarray(stored, dtype=np.float32).astype(np.float64)
    if dtype == BF16:
        return bf16_to_f64(stored)
    raise ValueError(f"unknown storage dtype {dtype!r}")


# --------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Workload:
    """Shapes, storage type and seed of one forward workload."""

    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    chunk: int
    dtype: str
    h0_std: float  # 0 means h0 = 0 (passed as NULL)
    seed: int

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    """Shapes, seed and step count of one decode workload."""

    name: str
    batch: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    steps: int
    dtype: str
    seed: int

    def with_(self, **kw) -> "DecodeWorkload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    # tiny fp32 problem: b1 L64 H2 P16 N16 G1 chunk 16
    "tiny_f32": Workload("tiny_f32", 1, 64, 2, 16, 16, 1, 16, F32, 0.0, 1000),
    # Mamba-2 ~2.7B-style layer: d_inner 5120 = 80 heads x 64
    "mamba2_2p7b_layer": Workload("mamba2_2p7b_layer", 8, 2048, 80, 64, 128, 1, 256,
                                  BF16, 0.0, 1001),
    # one long sequence with a carried-in initial state
    "long_seq_65k": Workload("long_seq_65k", 1, 65536, 32, 64, 128, 1, 256, BF16, 0.1, 1002),
    # hybrid-8B-style layer: d_inner 8192 = 128 heads x 64, 8 B/C groups
    "hybrid_8b_layer_N64": Workload("hybrid_8b_layer_N64", 4, 4096, 128, 64, 64, 8, 128,
                                    BF16, 0.0, 1003 + 64),
    "hybrid_8b_layer_N128": Workload("hybrid_8b_layer_N128", 4, 4096, 128, 64, 128, 8, 128,
                                     BF16, 0.0, 1003 + 128),
    "hybrid_8b_layer_N256": Workload("hybrid_8b_layer_N256", 4, 4096, 128, 64, 256, 8, 128,
                                     BF16, 0.0, 1003 + 256),
}

@dataclasses.dataclass(frozen=True)
class ScanWorkload:
    """Shapes, storage type and seed of one selective-scan workload (diagonal
    A per channel): `channels` channels, `dstate` states each."""

    name: str
    batch: int
    seqlen: int
    channels: int
    dstate: int
    ngroups: int
    dtype: str
    h0_std: float
    seed: int

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen

    def with_(self, **kw) -> "ScanWorkload":
        return dataclasses.replace(self, **kw)


SCAN_WORKLOADS: Dict[str, ScanWorkload] = {
    "scan_tiny_f32": ScanWorkload("scan_tiny_f32", 1, 64, 8, 16, 1, F32, 0.0, 2000),
    # Mamba ~2.8B-style layer: d_model 2560, expand 2 -> 5120 channels, N = 16
    "mamba1_2p8b_scan": ScanWorkload("mamba1_2p8b_scan", 8, 2048, 5120, 16, 1, BF16, 0.0, 2001),
}


def scan_inputs(w: ScanWorkload, seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Stored inputs of one selective-scan workload, the layer's distributions
    per channel: x (b,L,D) ~ N(0,1); dt (b,L,D) the RAW step z ~ N(0, 0.5)
    with dt_bias (D,) float32 b_d, softplus(b_d) log-uniform in [1e-3, 1e-1];
    A (D,N) float32 = -exp(U(0, ln 16)) per entry; B, C (b,L,G,N) ~ N(0,1)/sqrt(N);
    Dskip (D,) ~ N(1, 0.1); h0 (b,D,N) ~ N(0, h0_std) float32 or None."""
    seed = w.seed if seed is None else seed
    r_x, r_z, r_b, r_a, r_B, r_C, r_D, r_h = _rngs(seed, 8)
    b, L, Dc, N, G = w.batch, w.seqlen, w.channels, w.dstate, w.ngroups
    x = _draw_stored(r_x, (b, L, Dc), w.dtype)
    dt = _draw_stored(r_z, (b, L, Dc), w.dtype, 0.5)
    bias = _dt_bias(r_b, Dc).astype(np.float32)
    A = (-np.exp(r_a.uniform(0.0, math.log(16.0), size=(Dc, N)))).astype(np.float32)
    inv = 1.0 / math.sqrt(N)
    B = _draw_stored(r_B, (b, L, G, N), w.dtype, inv)
    C = _draw_stored(r_C, (b, L, G, N), w.dtype, inv)
    Dk = (1.0 + 0.1 * r_D.standard_normal(Dc)).astype(np.float32)
    h0 = None
    if w.h0_std > 0:
        h0 = (w.h0_std * r_h.standard_normal((b, Dc, N))).astype(np.float32)
    return {"x": x, "dt": dt, "dt_bias": bias, "A": A, "B": B, "C": C, "Dskip": Dk, "h0": h0}


DECODE_WORKLOADS: Dict[str, DecodeWorkload] = {
    "decode_b256": DecodeWorkload("decode_b256", 256, 128, 64, 128, 8, 64, BF16, 1004),
}


def _rngs(seed: int, n: int):
    return [np.random.Generator(np.random.PCG64(s))
            for s in np.random.SeedSequence(seed).spawn(n)]


def _softplus(v: np.ndarray) -> np.ndarray:
    # log(1 + e^v), stable for both signs; input shaping only.
    return np.logaddexp(0.0, v)


def _dt_bias(rng: np.random.Generator, nheads: int) -> np.ndarray:
    target = np.exp(rng.uniform(math.log(1e-3), math.log(1e-1), size=nheads))
    return np.log(np.expm1(target))  # softplus(b) == target


def _normal_slabs(rng, shape, scale=1.0, loc=0.0, slab_axis=1, slab=4096):
    """N(loc, scale) of `shape`, drawn slab by slab along `slab_axis` to bound
    the float64 temporaries; yields (index slice, float64 block)."""
    n = shape[slab_axis]
    for s0 in range(0, n, slab):
        s1 = min(n, s0 + slab)
        sub = list(shape)
        sub[slab_axis] = s1 - s0
        yield s0, s1, loc + scale * rng.standard_normal(size=tuple(sub))


def _draw_stored(rng, shape, dtype, scale=1.0, loc=0.0, slab_axis=1):
    out = np.empty(shape, dtype=np.float32 if dtype == F32 else np.uint16)
    idx = [slice(None)] * len(shape)
    for s0, s1, blk in _normal_slabs(rng, shape, scale, loc, slab_axis):
        idx[slab_axis] = slice(s0, s1)
        out[tuple(idx)] = store(blk, dtype)
    return out


def forward_inputs(w: Workload, seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Stored inputs of one forward workload.

    Returns x (b,L,H,P), dt (b,L,H), B, C (b,L,G,N) in w.dtype storage;
    A, D (H,) float32; h0 (b,H,P,N) float32 or None."""
    return _forward_inputs(w, seed, raw=False)


def forward_inputs_raw(w: Workload, seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """The same draws as forward_inputs, with the step left raw: dt holds z
    (stored in w.dtype) and dt_bias (H,) float32 holds b_h, so that
    softplus(z + b_h) is the step of forward_inputs up to the storage
    rounding. For the layer's step options (bias, softplus)."""
    return _forward_inputs(w, seed, raw=True)


def raw_steps(w: Workload, seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Only the raw-step fields of forward_inputs_raw (dt, dt_bias), from the
    same streams, without drawing the other inputs."""
    seed = w.seed if seed is None else seed
    _, r_z, r_b = _rngs(seed, 8)[:3]
    b, L, H = w.batch, w.seqlen, w.nheads
    bias = _dt_bias(r_b, H).astype(np.float32)
    dt = np.empty((b, L, H), dtype=np.float32 if w.dtype == F32 else np.uint16)
    for s0, s1, z in _normal_slabs(r_z, (b, L, H), 0.5):
        dt[:, s0:s1] = store(z, w.dtype)
    return {"dt": dt, "dt_bias": bias}


def _forward_inputs(w: Workload, seed: Optional[int], raw: bool) -> Dict[str, np.ndarray]:
    seed = w.seed if seed is None else seed
    r_x, r_z, r_b, r_a, r_B, r_C, r_D, r_h = _rngs(seed, 8)
    b, L, H, P, N, G = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups
    x = _draw_stored(r_x, (b, L, H, P), w.dtype)
    bias = _dt_bias(r_b, H)
    if raw:
        bias = bias.astype(np.float32)
    dt = np.empty((b, L, H), dtype=np.float32 if w.dtype == F32 else np.uint16)
    for s0, s1, z in _normal_slabs(r_z, (b, L, H), 0.5):
        dt[:, s0:s1] = store(z, w.dtype) if raw else store(_softplus(z + bias), w.dtype)
    A = (-np.exp(r_a.uniform(0.0, math.log(16.0), size=H))).astype(np.float32)
    inv = 1.0 / math.sqrt(N)
    B = _draw_stored(r_B, (b, L, G, N), w.dtype, inv)
    C = _draw_stored(r_C, (b, L, G, N), w.dtype, inv)
    D = (1.0 + 0.1 * r_D.standard_normal(H)).astype(np.float32)
    h0 = None
    if w.h0_std > 0:
        h0 = (w.h0_std * r_h.standard_normal((b, H, P, N))).astype(np.float32)
    out = {"x": x, "dt": dt, "A": A, "B": B, "C": C, "D": D, "h0": h0}
    if raw:
        out["dt_bias"] = bias
    return out


def decode_state(w: DecodeWorkload, seed: Optional[int] = None) -> np.ndarray:
    """Initial decode state h (b,H,P,N) float32, N(0,1) per element."""
    seed = w.seed if seed is None else seed
    (r,) = _rngs(seed + 7919, 1)
    h = np.empty((w.batch, w.nheads, w.headdim, w.dstate), dtype=np.float32)
    for b0 in range(0, w.batch, 16):
        b1 = min(w.batch, b0 + 16)
        h[b0:b1] = r.standard_normal((b1 - b0, w.nheads, w.headdim, w.dstate))
    return h


def decode_params(w: DecodeWorkload, seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Per-head parameters of a decode workload: A, D (H,) float32 and the
    per-head dt bias (float64, input shaping only)."""
    seed = w.seed if seed is None else seed
    r_a, r_D, r_b = _rngs(seed, 3)
    A = (-np.exp(r_a.uniform(0.0, math.log(16.0), size=w.nheads))).astype(np.float32)
    D = (1.0 + 0.1 * r_D.standard_normal(w.nheads)).astype(np.float32)
    return {"A": A, "D": D, "dt_bias": _dt_bias(r_b, w.nheads)}


def decode_step_inputs(w: DecodeWorkload, step: int,
                       seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Stored per-token inputs of decode step `step`: x (b,H,P), dt (b,H),
    B, C (b,G,N) in w.dtype storage."""
    seed = w.seed if seed is None else seed
    bias = decode_params(w, seed)["dt_bias"]
    r_x, r_z, r_B, r_C = _rngs(seed * 100003 + 1 + step, 4)
    b, H, P, N, G = w.batch, w.nheads, w.headdim, w.dstate, w.ngroups
    inv = 1.0 / math.sqrt(N)
    return {
        "x": store(r_x.standard_normal((b, H, P)), w.dtype),
        "dt": store(_softplus(0.5 * r_z.standard_normal((b, H)) + bias), w.dtype),
        "B": store(inv * r_B.standard_normal((b, G, N)), w.dtype),
        "C": store(inv * r_C.standard_normal((b, G, N)), w.dtype),
    }


def decode_step_inputs_raw(w: DecodeWorkload, step: int,
                           seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """decode_step_inputs with the step left raw: dt holds z (b,H) in w.dtype
    storage; the per-head bias is decode_params(...)["dt_bias"]."""
    seed = w.seed if seed is None else seed
    r_x, r_z, r_B, r_C = _rngs(seed * 100003 + 1 + step, 4)
    b, H, P, N, G = w.batch, w.nheads, w.headdim, w.dstate, w.ngroups
    inv = 1.0 / math.sqrt(N)
    return {
        "x": store(r_x.standard_normal((b, H, P)), w.dtype),
        "dt": store(0.5 * r_z.standard_normal((b, H)), w.dtype),
        "B": store(inv * r_B.standard_normal((b, G, N)), w.dtype),
        "C": store(inv * r_C.standard_normal((b, G, N)), w.dtype),
    }


def exact_inputs(inp: Dict[str, np.ndarray], dtype: str) -> Dict[str, np.ndarray]:
    """float64 exact values of stored inputs (fp32 fields stay fp32-exact)."""
    out = {}
    for k, v in inp.items():
        if v is None:
            out[k] = None
        elif k in ("A", "D", "h0", "h", "Dskip"):
            out[k] = np.asarray(v, dtype=np.float32).astype(np.float64)
        elif k == "dt_bias":
            out[k] = np.asarray(v).astype(np.float64)
        else:
            out[k] = exact(v, dtype)
    return out
