#!/usr/bin/env python
"""Throughput of the SSD layer (libssd) on B200, one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

A step is one ssd_forward over one batch of the workload (default: the
Mamba-2 ~2.7B-style layer, b8 L2048 H80 P64 N128 G1, chunk 256, bf16 I/O,
fp32 state). The line also carries the decode step (ssd_step, b256 H128 P64
N128 G8, fp32 state) measured in the same run, the dominant kernel's
roofline, the end-to-end number through host buffers, and the fp64 CPU
oracle timed on this host's cores.

Multi-GPU (torchrun, one process per GPU): every rank runs its own batch
(weak scaling, no data-path collective); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "SSD forward tokens/s (+% tensor peak); ssd_step tokens/s (+% HBM BW), 1 B200"
L2_BYTES = 126 * 2 ** 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------
# algorithmic counts
# --------------------------------------------------------------------------

def io_bytes(w) -> dict:
    e = 2 if w.dtype == synth.BF16 else 4
    b, L, H, P, N, G = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups
    state = b * H * P * N * 4
    return {"x": b * L * H * P * e, "y": b * L * H * P * e, "dt": b * L * H * e,
            "B": b * L * G * N * e, "C": b * L * G * N * e, "AD": 2 * H * 4,
            "h0": state if w.h0_std > 0 else 0, "h_final": state,
            "chunk_states": b * H * ((L + w.chunk - 1) // w.chunk) * P * N * 4}


def forward_min_bytes(w) -> int:
    """One read of every input and one write of every output."""
    d = io_bytes(w)
    return d["x"] + d["y"] + d["dt"] + d["B"] + d["C"] + d["AD"] + d["h0"] + d["h_final"]


def forward_flops(w) -> dict:
    """Tensor-contraction FLOPs of the chunked algorithm: causal (lower
    triangle only) and dense-tile counts. Per token and head: Gram 2QN/(H/G)
    (shared by a group), diagonal 2QP, chunk state 2NP, state->output 2NP."""
    b, L, H, P, N, G, Q = (w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups,
                           w.chunk)
    tok_heads = b * L * H
    hpg = H // G
    dense = tok_heads * (2 * Q * N / hpg + 2 * Q * P + 4 * N * P)
    causal = tok_heads * (Q * N / hpg + Q * P + 4 * N * P)
    return {"causal": causal, "dense": dense}


def kernel_bytes(name: str, w) -> int:
    """Compulsory HBM bytes of one launch of each kernel for its role."""
    d = io_bytes(w)
    if name == "simt_chunk_state":
        return d["x"] + d["dt"] + d["B"] + d["chunk_states"]
    if name == "simt_state_pass":
        return 2 * d["chunk_states"] + d["h0"] + d["h_final"]
    if name == "simt_chunk_output":
        return d["x"] + d["dt"] + d["B"] + d["C"] + d["chunk_states"] + d["y"]
    if name == "state_pass":
        # the segmented tensor-core path's inter-segment pass: each (lane,
        # segment) end state and decay read, the state entering each segment
        # written in place, h0 read, h_final written
        nseg = tc_segments(w)
        lanes = w.batch * w.nheads
        seg = lanes * nseg * w.headdim * w.dstate * 4
        return 2 * seg + lanes * nseg * 4 + d["h0"] + d["h_final"]
    if name == "tc_segment_state":
        # state-only pass of the segmented tensor-core path: x, dt, B in; one
        # fp32 state and one decay per (lane, segment) out
        nseg = tc_segments(w)
        lanes = w.batch * w.nheads
        seg_out = lanes * nseg * (w.headdim * w.dstate * 4 + 4)
        return d["x"] + d["dt"] + d["B"] + seg_out
    return forward_min_bytes(w)


def backward_flops(w, Q: int = 128) -> float:
    """Algorithmic FLOPs of the chunked adjoint (single-rounded operands, the
    causal halves of the token-by-token products). Per token and head:
    C B^T 2Q N/(H/G)/2 (shared by a group), dy x^T and M^T dy QP each, V^T C
    and V B QN each, the four state products (B R^T, X R, C H^T, dy H) and the
    two recomputed chunk states 2NP each."""
    hpg = w.nheads // w.ngroups
    P, N = w.headdim, w.dstate
    per = 2 * Q * P + 2 * Q * N + Q * N / hpg + 12 * N * P
    return float(w.batch * w.seqlen * w.nheads) * per


def backward_min_bytes(w, dh0: bool = True) -> int:
    """x, dy, dt, B and C read once, and h0 when the workload has one; the fp32
    dx, ddt, dB and dC written once, and dh0 when it is asked for (the
    benchmark's call asks for it)."""
    e = 2 if w.dtype == synth.BF16 else 4
    b, L, H, P, N, G = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups
    state = b * H * P * N * 4
    reads = (2 * b * L * H * P + b * L * H + 2 * b * L * G * N) * e
    reads += state if w.h0_std > 0 else 0
    writes = (b * L * H * P + b * L * H + 2 * b * L * G * N) * 4
    writes += state if dh0 else 0
    return reads + writes


def tc_segments(w, sms=None) -> int:
    """Segments per (batch, head) lane on the tensor-core path (the library's
    rule: one when the lanes fill the GPU twice over, else about two waves
    of CTAs, at most half the 128-token blocks)."""
    if sms is None:
        try:
            import torch

            sms = torch.cuda.get_device_properties(0).multi_processor_count
        except Exception:
            sms = 148
    lanes = w.batch * w.nheads
    nb = (w.seqlen + 127) // 128
    if lanes >= 2 * sms or nb < 4:
        return 1
    nseg = max(1, (2 * sms) // lanes)
    return max(1, min(nseg, nb // 2))


def decode_bytes(w) -> int:
    e = 2 if w.dtype == synth.BF16 else 4
    state = w.batch * w.nheads * w.headdim * w.dstate * 4
    io_ = (2 * w.batch * w.nheads * w.headdim + w.batch * w.nheads
           + 2 * w.batch * w.ngroups * w.dstate) * e + 2 * w.nheads * 4
    return 2 * state + io_


# Special-function unit results per clock per SM (exp2 and the like), from
# the CUDA arithmetic-instruction throughput table for recent compute
# capabilities; the B200's maximum SM clock.
SFU_PER_CLK_PER_SM = 16
SM_MAX_MHZ = 1965.0


def scan_alu_peak(sms: int, mhz: float = SM_MAX_MHZ) -> float:
    """State updates per second the selective scan can reach at most: each
    update takes one exp2 on the special-function units (16 per clock per SM),
    beside four fp32 FMA-pipe operations (128 per clock per SM), so the SFU
    binds."""
    return SFU_PER_CLK_PER_SM * sms * mhz * 1e6


def source_digest(paths) -> str:
    h = hashlib.sha256()
    for p in sorted(paths):
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def stored_traffic(kernel: str, workload: str = None):
    """DRAM bytes per launch from the committed ncu capture of this kernel on
    this workload ("kernel@workload"; a kernel whose bytes do not depend on
    the workload is stored under its name alone), if it was taken on the
    kernel's current source; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            tab = json.load(f)
    except (OSError, ValueError):
        return None
    ent = tab.get(f"{kernel}@{workload}") if workload else None
    ent = ent or tab.get(kernel)
    if not ent:
        return None
    try:
        if source_digest(ent["sources"]) != ent["source_digest"]:
            return None
    except (OSError, KeyError):
        return None
    return ent.get("dram_bytes_per_launch")


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ["uuid", "clocks.sm", "clocks.max.sm", "power.draw", "utilization.gpu",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.proc = None
        self.t_start = self.t_stop = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=timestamp," + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return []
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for r in csv.reader(io.StringIO(out)):
            r = [c.strip() for c in r]
            if len(r) != len(self.FIELDS) + 1:
                continue
            if self.uuid and self.uuid not in r[1]:
                continue
            rows.append(r)
        return rows

    @staticmethod
    def summarise(rows, max_mhz):
        def num(v):
            try:
                return float(v)
            except ValueError:
                return float("nan")

        load = [r for r in rows if num(r[5]) >= 50.0] or rows
        sm = [num(r[2]) for r in load if not math.isnan(num(r[2]))]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in load for i in range(4) if r[6 + i] == "Active"})
        smax = [num(r[3]) for r in rows if not math.isnan(num(r[3]))]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else max_mhz,
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(load)}


# --------------------------------------------------------------------------
# distributed plumbing
# --------------------------------------------------------------------------

class Dist:
    def __init__(self, backend="nccl"):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        if self.world > 1:
            import datetime

            import torch.distributed as dist

            dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))
            self.pg = dist

    def barrier(self, device=None):
        if self.pg is not None:
            if device is not None:
                self.pg.barrier(device_ids=[device.index])
            else:
                self.pg.barrier()

    def max(self, v: float, device) -> float:
        if self.pg is None:
            return v
        import torch

        t = torch.tensor([v], dtype=torch.float64, device=device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


def shard_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own batch (weak scaling over independent batches)."""
    return base_seed + 7919 * rank


# --------------------------------------------------------------------------
# CPU oracle baseline
# --------------------------------------------------------------------------

def oracle_forward_time(w, seed, lanes_per_step=None, min_seconds=10.0, max_passes=3,
                        steps=None, outputs=None):
    """Time the fp64 oracle on this host's cores. Returns (tokens/s, cores,
    sample description, per-pass times).

    With lanes_per_step, one pass is a fixed spread of that many (batch, head)
    lanes over their whole sequences, run as one problem with one head and
    one B/C group per lane (each lane keeps its own A, D and inputs). A dict
    passed as `outputs` receives the sampled lanes and the last pass's y
    (1, L, lanes, P) and h_final (1, lanes, P, N)."""
    import oracle

    inp = synth.forward_inputs(w, seed=seed)
    ex = synth.exact_inputs(inp, w.dtype)
    cores = oracle.max_threads()
    H = w.nheads
    if lanes_per_step is None:
        sub = ex
        lanes = w.batch * H
    else:
        lanes = lanes_per_step
        idx = np.linspace(0, w.batch * H - 1, lanes).round().astype(int)
        bs, hs = idx // H, idx % H
        g = hs // (H // w.ngroups)
        sub = {"x": np.ascontiguousarray(ex["x"][bs, :, hs, :].transpose(1, 0, 2)[None]),
               "dt": np.ascontiguousarray(ex["dt"][bs, :, hs].T[None]),
               "A": ex["A"][hs], "D": ex["D"][hs],
               "B": np.ascontiguousarray(ex["B"][bs, :, g, :].transpose(1, 0, 2)[None]),
               "C": np.ascontiguousarray(ex["C"][bs, :, g, :].transpose(1, 0, 2)[None]),
               "h0": None if ex["h0"] is None else np.ascontiguousarray(ex["h0"][bs, hs][None])}
    times = []

    def one():
        t0 = time.perf_counter()
        y, hf = oracle.ssd_forward(sub["x"], sub["dt"], sub["A"], sub["B"], sub["C"],
                                   sub["D"], sub["h0"])
        times.append(time.perf_counter() - t0)
        if outputs is not None and lanes_per_step is not None:
            outputs.update(lanes=list(zip(bs.tolist(), hs.tolist())), y=y, h_final=hf)

    if steps is not None:
        for _ in range(steps):
            one()
    else:
        one()
        while len(times) < max_passes and sum(times) < min_seconds:
            one()
    if lanes_per_step is not None:
        cores = min(cores, lanes)  # the oracle's threads run over the lanes
    tok = lanes * w.seqlen / H  # token-equivalents: one token = all H heads
    value = tok * len(times) / sum(times)
    if lanes_per_step is None:
        sample = (f"whole workload ({w.batch}x{H} (batch, head) lanes x {w.seqlen} tokens), "
                  f"{len(times)} pass(es); tokens/s counts all {H} heads of a token")
    else:
        sample = (f"{lanes} of {w.batch * H} (batch, head) lanes over whole {w.seqlen}-token "
                  f"sequences per step; tokens/s counts all {H} heads of a token")
    return value, cores, sample, times


# --------------------------------------------------------------------------
# our path
# --------------------------------------------------------------------------

def to_device(arr, device):
    import torch

    if arr is None:
        return None
    if arr.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(
            torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32)).to(device)


def to_pinned(arr):
    import torch

    if arr is None:
        return None
    if arr.dtype == np.uint16:
        t = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32))
    return t.pin_memory()


def _timed(fn, steps, device, stream, dist, profile=True):
    """K calls of fn bracketed by barrier + synchronize on both sides, timed
    with CUDA events on `stream`. Returns (ms per step, max over ranks; local
    ms; per-kernel event times; library launches)."""
    import torch

    import selective_state_space_12_b200 as ssd

    torch.cuda.synchronize(device)
    dist.barrier(device)
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    n_before = ssd.launch_count()
    if profile:
        ssd.profile_begin()
    e0.record(stream)
    for i in range(steps):
        fn(i)
    e1.record(stream)
    torch.cuda.synchronize(device)
    prof = ssd.profile_end() if profile else {}
    launches = ssd.launch_count() - n_before
    dist.barrier(device)
    torch.cuda.synchronize(device)
    ms_local = e0.elapsed_time(e1) / steps
    return dist.max(ms_local, device), ms_local, prof, launches


def bench_forward(args, dist, device, stream, peaks, peaks_src):
    import torch

    import selective_state_space_12_b200 as ssd

    w = synth.WORKLOADS[args.workload]
    if args.batch:
        w = w.with_(batch=args.batch)
    seed = shard_seed(w.seed, dist.rank)
    inp = synth.forward_inputs(w, seed=seed)
    dev = {k: to_device(v, device) for k, v in inp.items()}
    y = torch.empty_like(dev["x"])
    hf = torch.empty((w.batch, w.nheads, w.headdim, w.dstate), dtype=torch.float32,
                     device=device)
    dims = ssd.make_dims(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups,
                         dev["x"].dtype)
    ws_bytes = ssd.ssd_forward_workspace_size(dims, w.chunk)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=device)
    fwd = ssd.prepare_forward(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"],
                              dev["h0"], w.chunk, y, hf, ws, stream=stream)

    # W warm-up steps, then exactly K timed steps
    for _ in range(args.warmup):
        fwd()
    ms, ms_local, prof, launches = _timed(lambda i: fwd(), args.steps, device, stream, dist)
    tokens_all = w.tokens * dist.world

    kernels = {}
    tot = sum(t for _, t in prof.values()) or 1.0
    for k, (n, t) in prof.items():
        kernels[k] = {"launches": n, "avg_us": 1e3 * t / max(n, 1), "share": t / tot}
    roofline = None
    if prof:
        dom = max(prof.items(), key=lambda kv: kv[1][1])[0]
        n, t = prof[dom]
        avg_s = t / n * 1e-3
        kb = kernel_bytes(dom, w)
        achieved = kb / avg_s / 1e9
        roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved,
                    "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": achieved / peaks["hbm_gbs"], "traffic": stored_traffic(dom, w.name),
                    "algorithmic_bytes": kb, "avg_launch_us": avg_s * 1e6,
                    "peak_source": f"{peaks_src} (STREAM-style copy)"}
    fl = forward_flops(w)
    achieved_tf = fl["causal"] / (ms_local * 1e-3) / 1e12
    tensor = {"causal_flop_per_step": fl["causal"], "dense_tile_flop_per_step": fl["dense"],
              "achieved_tflops_causal": achieved_tf, "peak_tflops": peaks["bf16_tflops"],
              "frac_causal": achieved_tf / peaks["bf16_tflops"],
              "peak_source": f"{peaks_src} (cuBLAS bf16 burst)"}
    min_b = forward_min_bytes(w)
    hbm_whole = {"min_bytes_per_step": min_b,
                 "achieved_gbs": min_b / (ms_local * 1e-3) / 1e9,
                 "frac": min_b / (ms_local * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    out = {"w": w, "seed": seed, "ms": ms, "value": tokens_all / (ms * 1e-3),
           "roofline": roofline, "tensor": tensor, "hbm_whole_forward": hbm_whole,
           "kernels": kernels, "gpu_launches": launches, "e2e": None, "step_options": None}

    # the same workload with the step options fused (raw step, per-head bias,
    # softplus, zero-order hold): ssd_forward_ex on the same buffers
    if not args.no_options:
        raw = synth.raw_steps(w, seed=seed)
        dt_raw = to_device(raw["dt"], device)
        bias = torch.from_numpy(raw["dt_bias"]).to(device)
        opts = ssd.make_options(bias, dt_softplus=True, zoh=True)
        fwd_o = ssd.prepare_forward(dev["x"], dt_raw, dev["A"], dev["B"], dev["C"], dev["D"],
                                    dev["h0"], w.chunk, y, hf, ws, stream=stream, options=opts)
        for _ in range(args.warmup):
            fwd_o()
        ms_o, _, prof_o, launches_o = _timed(lambda i: fwd_o(), args.steps, device, stream,
                                             dist)
        out["step_options"] = {
            "options": "dt = softplus(raw + bias_h), zero-order-hold input weight",
            "value": tokens_all / (ms_o * 1e-3), "unit": "tokens/s", "ms_per_step": ms_o,
            "vs_plain_forward": ms_o / ms, "gpu_launches": launches_o,
            "kernels": {k: {"launches": n, "avg_us": 1e3 * t / max(n, 1)}
                        for k, (n, t) in prof_o.items()}}

    # end to end through host buffers: pinned host -> device, forward, -> host
    if not args.no_e2e:
        host = {k: to_pinned(v) for k, v in inp.items()}
        y_h = torch.empty(y.shape, dtype=y.dtype).pin_memory()
        hf_h = torch.empty(hf.shape, dtype=hf.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host.values() if t is not None)
        d2h = y_h.numel() * y_h.element_size() + hf_h.numel() * hf_h.element_size()

        def e2e_step(i):
            for k, t in host.items():
                if t is not None:
                    dev[k].copy_(t, non_blocking=True)
            fwd()
            y_h.copy_(y, non_blocking=True)
            hf_h.copy_(hf, non_blocking=True)

        for i in range(3):
            e2e_step(i)
        k_e2e = max(1, min(args.steps, 10))
        ms_one, _, _, _ = _timed(e2e_step, k_e2e, device, stream, dist, profile=False)

        # the library's host-to-host forward: batch slices whose uploads,
        # forwards and downloads overlap on three streams
        hfw = ssd.HostForward(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups,
                              dev["x"].dtype, chunk=w.chunk, splits=args.e2e_splits,
                              h0=host.get("h0") is not None, device=device)

        def e2e_overlap(i):
            hfw(host["x"], host["dt"], host["A"], host["B"], host["C"], host["D"], y_h, hf_h,
                h0=host.get("h0"), stream=stream)

        for i in range(3):
            e2e_overlap(i)
        ms_e2e, _, _, _ = _timed(e2e_overlap, k_e2e, device, stream, dist, profile=False)
        out["e2e"] = {"value": tokens_all / (ms_e2e * 1e-3), "unit": "tokens/s",
                      "h2d_bytes_per_step": hfw.h2d_bytes, "d2h_bytes_per_step": hfw.d2h_bytes,
                      "ms_per_step": ms_e2e, "steps": k_e2e, "splits": len(hfw.slices),
                      "path": "HostForward: pinned host -> device copies, ssd_forward (C ABI) "
                              "and y, h_final -> pinned host per batch slice, overlapped on "
                              "three streams",
                      "one_stream": {"value": tokens_all / (ms_one * 1e-3),
                                     "ms_per_step": ms_one, "h2d_bytes_per_step": h2d,
                                     "d2h_bytes_per_step": d2h}}
    return out


FORWARD_CONFIGS = ("mamba2_2p7b_layer", "long_seq_65k", "hybrid_8b_layer_N64",
                   "hybrid_8b_layer_N128", "hybrid_8b_layer_N256")


def _roofline_of(name, n, t_ms, w, peaks, peaks_src):
    """HBM roofline of one kernel: its algorithmic bytes per launch over its
    CUDA-event average."""
    avg_s = t_ms / n * 1e-3
    kb = kernel_bytes(name, w)
    achieved = kb / avg_s / 1e9
    return {"bound": "hbm", "kernel": name, "achieved": achieved, "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
            "traffic": stored_traffic(name, w.name),
            "algorithmic_bytes": kb, "avg_launch_us": avg_s * 1e6,
            "peak_source": f"{peaks_src} (STREAM-style copy)"}


def bench_forward_config(name, args, dist, device, stream, peaks, peaks_src, cpu=True):
    """One forward workload at full size: tokens/s, the dominant kernel's
    roofline (and the state pass's, when the lanes are cut into segments), the
    tensor fraction, and, on one GPU, the oracle as this workload's CPU
    baseline on four sampled lanes over whole sequences, compared with the
    GPU's output on the same lanes (max |err| / rms per lane, worst lane)."""
    import torch

    import selective_state_space_12_b200 as ssd

    w = synth.WORKLOADS[name]
    seed = shard_seed(w.seed, dist.rank)
    inp = synth.forward_inputs(w, seed=seed)
    dev = {k: to_device(v, device) for k, v in inp.items()}
    y = torch.empty_like(dev["x"])
    hf = torch.empty((w.batch, w.nheads, w.headdim, w.dstate), dtype=torch.float32,
                     device=device)
    dims = ssd.make_dims(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups,
                         dev["x"].dtype)
    ws_bytes = ssd.ssd_forward_workspace_size(dims, w.chunk)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=device)
    fwd = ssd.prepare_forward(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"],
                              dev["h0"], w.chunk, y, hf, ws, stream=stream)
    for _ in range(args.warmup):
        fwd()
    steps = max(1, min(args.steps, 20))
    ms, ms_local, prof, launches = _timed(lambda i: fwd(), steps, device, stream, dist)
    tot = sum(t for _, t in prof.values()) or 1.0
    kernels = {k: {"launches": n, "avg_us": 1e3 * t / max(n, 1), "share": t / tot}
               for k, (n, t) in prof.items()}
    dom = max(prof.items(), key=lambda kv: kv[1][1])[0]
    out = {"workload": name, "steps": steps, "ms_per_step": ms,
           "value": w.tokens * dist.world / (ms * 1e-3), "unit": "tokens/s",
           "gpu_launches": launches, "kernels": kernels,
           "roofline": _roofline_of(dom, prof[dom][0], prof[dom][1], w, peaks, peaks_src)}
    if "state_pass" in prof:
        out["state_pass_roofline"] = _roofline_of("state_pass", *prof["state_pass"], w, peaks,
                                                  peaks_src)
    fl = forward_flops(w)
    out["tensor"] = {"frac_causal": fl["causal"] / (ms_local * 1e-3) / 1e12 /
                     peaks["bf16_tflops"], "causal_flop_per_step": fl["causal"]}
    min_b = forward_min_bytes(w)
    out["hbm_whole_forward"] = {"min_bytes_per_step": min_b,
                                "frac": min_b / (ms_local * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    if cpu and dist.world == 1:
        ref = {}
        v, cores, sample, _ = oracle_forward_time(w, seed, lanes_per_step=4, steps=1,
                                                  outputs=ref)
        torch.cuda.synchronize(device)
        worst_y = worst_h = 0.0
        for k, (b, h) in enumerate(ref["lanes"]):
            yg = y[b, :, h, :].double().cpu().numpy()
            yr = ref["y"][0, :, k, :]
            hg = hf[b, h].double().cpu().numpy()
            hr = ref["h_final"][0, k]
            worst_y = max(worst_y, float(np.abs(yg - yr).max() / np.sqrt(np.mean(yr * yr))))
            worst_h = max(worst_h, float(np.abs(hg - hr).max() / np.sqrt(np.mean(hr * hr))))
        out["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                               "sample": sample}
        out["parity"] = {"lanes": [list(l) for l in ref["lanes"]],
                         "max_err_over_rms_y": worst_y, "max_err_over_rms_h_final": worst_h,
                         "bound": 1e-4 if w.dtype == synth.F32 else 2e-2}
    del dev, y, hf, ws
    return out


def bench_decode(args, dist, device, stream, peaks, peaks_src):
    import torch

    import selective_state_space_12_b200 as ssd

    dw = synth.DECODE_WORKLOADS["decode_b256"]
    if args.decode_batch:
        dw = dw.with_(batch=args.decode_batch)
    dseed = shard_seed(dw.seed, dist.rank)
    prm = synth.decode_params(dw, seed=dseed)
    h = torch.from_numpy(synth.decode_state(dw, seed=dseed)).to(device)
    A = torch.from_numpy(prm["A"]).to(device)
    D = torch.from_numpy(prm["D"]).to(device)
    n_in = dw.steps
    steps_in = [{k: to_device(v, device) for k, v in
                 synth.decode_step_inputs(dw, s, seed=dseed).items()} for s in range(n_in)]
    yd = torch.empty_like(steps_in[0]["x"])
    calls = [ssd.prepare_step(h, s["x"], s["dt"], A, s["B"], s["C"], D, yd, stream=stream)
             for s in steps_in]
    for i in range(args.warmup):
        calls[i % n_in]()
    kd = max(args.steps, n_in)
    ms_d, _, dprof, launches = _timed(lambda i: calls[i % n_in](), kd, device, stream, dist)
    db = decode_bytes(dw)
    n, t = dprof.get("ssd_step", (kd, ms_d * kd))
    k_us = t / max(n, 1) * 1e3
    achieved = db / (k_us * 1e-6) / 1e9
    opt = None
    if not args.no_options:
        # the same steps on raw dt with the step options fused (bias, softplus,
        # zero-order hold), continuing on the same state
        bias = torch.from_numpy(prm["dt_bias"].astype("float32")).to(device)
        opts = ssd.make_options(bias, dt_softplus=True, zoh=True)
        raw_dt = [to_device(synth.decode_step_inputs_raw(dw, s, seed=dseed)["dt"], device)
                  for s in range(n_in)]
        calls_o = [ssd.prepare_step(h, s["x"], r, A, s["B"], s["C"], D, yd, stream=stream,
                                    options=opts) for s, r in zip(steps_in, raw_dt)]
        for i in range(args.warmup):
            calls_o[i % n_in]()
        ms_o, _, oprof, launches_o = _timed(lambda i: calls_o[i % n_in](), kd, device, stream,
                                            dist)
        no, to = oprof.get("ssd_step", (kd, ms_o * kd))
        o_us = to / max(no, 1) * 1e3
        opt = {"options": "dt = softplus(raw + bias_h), zero-order-hold input weight",
               "value": dw.batch * dist.world / (ms_o * 1e-3), "unit": "tokens/s",
               "us_per_step": ms_o * 1e3, "gpu_launches": launches_o,
               "achieved_gbs": db / (o_us * 1e-6) / 1e9,
               "frac": db / (o_us * 1e-6) / 1e9 / peaks["hbm_gbs"]}
    return {"value": dw.batch * dist.world / (ms_d * 1e-3), "unit": "tokens/s",
            "step_options": opt,
            "workload": dw.name, "batch": dw.batch, "nheads": dw.nheads,
            "headdim": dw.headdim, "dstate": dw.dstate, "ngroups": dw.ngroups,
            "steps_timed": kd, "us_per_step": ms_d * 1e3, "gpu_launches": launches,
            "roofline": {"bound": "hbm", "kernel": "ssd_step", "achieved": achieved,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"],
                         "traffic": stored_traffic("ssd_step"), "algorithmic_bytes": db,
                         "avg_launch_us": k_us,
                         "peak_source": f"{peaks_src} (STREAM-style copy)"}}


def bench_backward(args, dist, device, stream, peaks, peaks_src):
    """The backward pass (ssd_backward) on the forward's workload."""
    import ctypes

    import torch

    import selective_state_space_12_b200 as ssd
    from selective_state_space_12_b200 import _lib

    w = synth.WORKLOADS[args.workload]
    if args.batch:
        w = w.with_(batch=args.batch)
    seed = shard_seed(w.seed, dist.rank)
    inp = synth.forward_inputs(w, seed=seed)
    dev = {k: to_device(v, device) for k, v in inp.items()}
    dy = torch.randn(dev["x"].shape, device=device).to(dev["x"].dtype)
    dims = ssd.make_dims(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups,
                         dev["x"].dtype)
    need = int(_lib.load().ssd_backward_workspace_size(ctypes.byref(dims)))
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=device)

    def step(i):
        ssd.ssd_backward(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["h0"],
                         dy, None, workspace=ws)

    for i in range(args.warmup):
        step(i)
    ms, ms_local, prof, launches = _timed(step, args.steps, device, stream, dist)
    flops, nbytes = backward_flops(w), backward_min_bytes(w)
    t_flop = flops / (peaks["bf16_tflops"] * 1e12)
    t_byte = nbytes / (peaks["hbm_gbs"] * 1e9)
    sec = ms_local * 1e-3
    roof = ({"bound": "tensor", "achieved": flops / sec / 1e12, "peak": peaks["bf16_tflops"],
             "unit": "TFLOP/s", "frac": t_flop / sec}
            if t_flop >= t_byte else
            {"bound": "hbm", "achieved": nbytes / sec / 1e9, "peak": peaks["hbm_gbs"],
             "unit": "GB/s", "frac": t_byte / sec})
    roof.update({"scope": "whole backward step (all its launches)",
                 "algorithmic_flops": flops, "algorithmic_bytes": nbytes,
                 "floor_us": 1e6 * max(t_flop, t_byte), "peak_source": peaks_src})
    return {"workload": w.name, "value": w.tokens * dist.world / (ms * 1e-3), "unit": "tokens/s",
            "ms_per_step": ms, "vs_forward": None, "gpu_launches": launches,
            "workspace_bytes": need, "roofline": roof,
            "kernels": {k: {"launches": n, "avg_us": 1e3 * t / max(n, 1)}
                        for k, (n, t) in prof.items()},
            "path": ("tensor cores (tcgen05): the chunk states and the adjoint chunk states "
                     "each chained along the lanes in one pass, then per-chunk dx/ddt and dB/dC "
                     "in one persistent kernel"
                     if any(k.startswith("tc_bwd") for k in prof) else
                     "CUDA cores: recomputed chunk states, adjoint chunk states, forward and "
                     "reverse state passes, per-chunk dx/ddt and dB/dC")}


def bench_sp(args, dist, device, stream):
    """Sequence parallelism: the long-sequence workload's one sequence split
    into consecutive pieces, one per rank (strong scaling), through
    sp_forward (state of each piece, all-gather, chain, forward)."""
    import selective_state_space_12_b200 as ssd

    w = synth.WORKLOADS["long_seq_65k"]
    inp = synth.forward_inputs(w)  # one sequence: the same draws on every rank
    L, R, r = w.seqlen, dist.world, dist.rank
    t0, t1 = r * L // R, (r + 1) * L // R
    dev = {}
    for k, v in inp.items():
        if v is None:
            dev[k] = None
        elif k in ("x", "dt", "B", "C"):
            dev[k] = to_device(v[:, t0:t1], device)
        else:
            dev[k] = to_device(v, device)

    def step(i):
        ssd.sp_forward(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["h0"],
                       chunk=w.chunk)

    for i in range(args.warmup):
        step(i)
    ms, _, prof, launches = _timed(step, args.steps, device, stream, dist)
    return {"workload": w.name, "seq_len": L, "pieces": R, "tokens_per_rank": t1 - t0,
            "value": w.tokens / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
            "scaling": "strong", "gpu_launches": launches,
            "kernels": {k: {"launches": n, "avg_us": 1e3 * t / max(n, 1)}
                        for k, (n, t) in prof.items()},
            "path": "ssd_forward_state, NCCL all-gather of end states and decays, "
                    "ssd_state_chain, ssd_forward from the entering state"}


def bench_scan(args, dist, device, stream, peaks, peaks_src):
    """The selective scan with a diagonal A per channel (the prior art the
    SSD pages compare with): Mamba ~2.8B-style layer, b8 L2048 D5120 N16,
    softplus steps and the zero-order hold, each rank its own batch."""
    import torch

    import selective_state_space_12_b200 as ssd

    w = synth.SCAN_WORKLOADS["mamba1_2p8b_scan"]
    inp = synth.scan_inputs(w, seed=shard_seed(w.seed, dist.rank))
    d = {k: to_device(v, device) for k, v in inp.items()
         if v is not None and k not in ("A", "dt_bias", "Dskip")}
    f32 = {k: torch.from_numpy(inp[k]).to(device) for k in ("A", "dt_bias", "Dskip")}
    y = torch.empty_like(d["x"])
    hf = torch.empty((w.batch, w.channels, w.dstate), dtype=torch.float32, device=device)

    def step(i):
        ssd.ssd_selective_scan(d["x"], d["dt"], f32["A"], d["B"], d["C"], f32["Dskip"], None,
                               dt_bias=f32["dt_bias"], dt_softplus=True, zoh=True, y=y,
                               h_final=hf)

    for i in range(args.warmup):
        step(i)
    ms, ms_local, prof, launches = _timed(step, args.steps, device, stream, dist)
    e = 2  # bf16 I/O
    min_b = (3 * w.batch * w.seqlen * w.channels * e + 2 * w.batch * w.seqlen * w.ngroups *
             w.dstate * e + w.batch * w.channels * w.dstate * 4 + w.channels * w.dstate * 4)
    n, t = prof.get("selective_scan", (args.steps, ms_local * args.steps))
    k_us = t / max(n, 1) * 1e3
    elems = w.batch * w.seqlen * w.channels * w.dstate  # state entries updated per step
    alu_peak = scan_alu_peak(torch.cuda.get_device_properties(device).multi_processor_count)
    return {"workload": w.name, "batch": w.batch, "seq_len": w.seqlen, "channels": w.channels,
            "dstate": w.dstate, "options": "softplus(raw + bias_d), zero-order hold",
            "value": w.tokens * dist.world / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
            "gpu_launches": launches,
            "roofline": {"bound": "alu", "kernel": "selective_scan", "avg_launch_us": k_us,
                         "achieved": elems / (k_us * 1e-6), "unit": "state updates/s",
                         "peak": alu_peak, "frac": elems / (k_us * 1e-6) / alu_peak,
                         "peak_source": "derived: 16 exp2 per clock per SM x SMs x 1965 MHz",
                         "state_updates_per_s": elems / (k_us * 1e-6),
                         "hbm_achieved_gbs": min_b / (k_us * 1e-6) / 1e9,
                         "hbm_frac": min_b / (k_us * 1e-6) / 1e9 / peaks["hbm_gbs"],
                         "algorithmic_bytes": min_b,
                         "note": "one exp2 per state entry per token: the peak is the "
                                 "special-function units' rate; HBM is far from binding, and the "
                                 "kernel is latency-bound below that peak: about 17 warps per SM "
                                 "on this workload, each walking its channels' whole sequence"}}


def run_ours(args, dist: Dist):
    import torch

    from selective_state_space_12_b200 import build as ssd_build

    if dist.rank == 0 or dist.world == 1:
        ssd_build.build()
    dist.barrier()
    device = torch.device("cuda", dist.local)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    peaks, peaks_src = load_peaks()
    props = torch.cuda.get_device_properties(device)
    uuid = str(getattr(props, "uuid", "") or "")

    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.3)
    fw = dec = None
    if args.only in ("all", "forward"):
        fw = bench_forward(args, dist, device, stream, peaks, peaks_src)
    configs = None
    if args.only == "all" and not args.no_configs:
        # every forward workload at full size, the headline one included
        configs = {}
        for name in FORWARD_CONFIGS:
            torch.cuda.empty_cache()
            configs[name] = bench_forward_config(name, args, dist, device, stream, peaks,
                                                 peaks_src, cpu=not args.no_cpu_baseline)
    clock_rows = sampler.stop()
    torch.cuda.empty_cache()
    if args.only in ("all", "decode"):
        dec = bench_decode(args, dist, device, stream, peaks, peaks_src)
    bwd = None
    if args.only in ("all", "backward") and not args.no_backward:
        torch.cuda.empty_cache()
        bwd = bench_backward(args, dist, device, stream, peaks, peaks_src)
        if fw is not None:
            bwd["vs_forward"] = bwd["ms_per_step"] / fw["ms"]
    scan = None
    if args.only in ("all", "scan") and not args.no_scan:
        torch.cuda.empty_cache()
        scan = bench_scan(args, dist, device, stream, peaks, peaks_src)
    sp = None
    if args.only in ("all", "sp") and not args.no_sp:
        torch.cuda.empty_cache()
        sp = bench_sp(args, dist, device, stream)
    clocks = ClockSampler.summarise(clock_rows, peaks.get("sm_max_mhz"))
    if fw is None:
        # one part alone (profiling cases): its own line
        metric, key, res = {
            "decode": ("ssd_step tokens/s", "decode", dec),
            "scan": ("selective scan tokens/s", "selective_scan", scan),
            "backward": ("backward tokens/s", "backward", bwd),
            "sp": ("sequence-parallel forward tokens/s", "sequence_parallel", sp),
        }[args.only]
        if res is None:
            raise SystemExit(f"--only {args.only} was skipped by its --no- flag")
        return {"metric": metric, "value": res["value"], "unit": "tokens/s",
                "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
                key: res, "clocks": clocks}

    # CPU baseline: the oracle on this host's cores (rank 0, one GPU only)
    cpu = None
    w = fw["w"]
    if dist.world == 1 and not args.no_cpu_baseline:
        v, cores, sample, _ = oracle_forward_time(w, fw["seed"])
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": sample}
    return {
        "metric": METRIC, "value": fw["value"], "unit": "tokens/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": fw["ms"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded; distributions of the stated workloads)",
        "config": {"workload": w.name, "batch_per_gpu": w.batch, "global_batch":
                   w.batch * dist.world, "seq_len": w.seqlen, "nheads": w.nheads,
                   "headdim": w.headdim, "dstate": w.dstate, "ngroups": w.ngroups,
                   "chunk": w.chunk, "h0": w.h0_std > 0,
                   "parallelism": f"independent batches x{dist.world}",
                   "l2": f"inputs larger than L2: x {io_bytes(w)['x'] / 1e6:.0f} MB and y "
                         f"{io_bytes(w)['y'] / 1e6:.0f} MB per step vs "
                         f"{L2_BYTES / 1e6:.0f} MB L2; no flush"},
        "roofline": fw["roofline"], "tensor": fw["tensor"],
        "hbm_whole_forward": fw["hbm_whole_forward"], "kernels": fw["kernels"],
        "gpu_launches": fw["gpu_launches"], "e2e": fw["e2e"],
        "step_options": fw["step_options"], "decode": dec, "sequence_parallel": sp,
        "selective_scan": scan, "backward": bwd, "forward_configs": configs,
        "cpu_baseline": cpu, "clocks": clocks,
    }


def run_reference(args, world: int):
    w = synth.WORKLOADS[args.workload]
    lanes = 64
    v, cores, sample, times = oracle_forward_time(w, w.seed, lanes_per_step=lanes,
                                                  steps=args.warmup + args.steps)
    timed = times[args.warmup:]
    ms = 1e3 * sum(timed) / len(timed)
    value = lanes * w.seqlen / w.nheads / (ms * 1e-3)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; distributions of the stated workloads)",
        "config": {"workload": w.name, "batch_per_gpu": w.batch, "seq_len": w.seqlen,
                   "nheads": w.nheads, "headdim": w.headdim, "dstate": w.dstate,
                   "ngroups": w.ngroups, "chunk": w.chunk},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "note": "fp64 sequential-recurrence oracle (C, OpenMP) on the host cores; "
                "each step is a bounded sample of the workload",
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mamba2_2p7b_layer", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--only", choices=["all", "forward", "decode", "scan", "backward", "sp"],
                    default="all",
                    help="run only one part (profiling cases)")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="override the decode workload's batch")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-splits", type=int, default=4,
                    help="batch slices of the end-to-end leg (copies overlap across slices)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the backward-pass leg")
    ap.add_argument("--no-scan", action="store_true",
                    help="skip the selective-scan leg (diagonal A per channel)")
    ap.add_argument("--no-sp", action="store_true",
                    help="skip the sequence-parallel leg (long sequence split over the ranks)")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-workload forward legs (all five forward workloads)")
    ap.add_argument("--no-options", action="store_true",
                    help="skip the step-options legs (forward and decode with raw dt)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.steps < 1:
        ap.error("--steps must be at least 1")

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return 0  # the CPU oracle runs on rank 0 only
        line = run_reference(args, int(os.environ.get("WORLD_SIZE", str(args.gpus))))
        print(json.dumps(line), flush=True)
        return 0

    dist = Dist("nccl")
    if dist.world != args.gpus:
        log(f"note: --gpus {args.gpus} but WORLD_SIZE {dist.world}; using WORLD_SIZE")
    try:
        line = run_ours(args, dist)
        if dist.rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
