"""Shared test plumbing: stored numpy inputs -> torch device tensors, the
oracle on sampled lanes, and the parity measure."""
from __future__ import annotations

import numpy as np

import oracle
import synth


def to_device(arr, dtype: str, device="cuda"):
    """A stored numpy array (float32, or uint16 bf16 bits) as a torch tensor."""
    import torch

    if arr is None:
        return None
    if arr.dtype == np.uint16:
        t = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32))
    return t.to(device)


def to_f64(t):
    """Exact float64 numpy value of a torch tensor (bf16 or fp32)."""
    import torch

    return t.detach().to(torch.float64).cpu().numpy()


def gpu_forward(inp, w, chunk=None, want_final=True, D=True, h0=True):
    from selective_state_space_12_b200 import ssd_forward

    from selective_state_space_12_b200 import ssd_device_status, ssd_last_error

    dev = {k: to_device(v, w.dtype) for k, v in inp.items()}
    y, hf = ssd_forward(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"],
                        dev["D"] if D else None, dev["h0"] if h0 else None,
                        chunk=chunk or w.chunk, want_final=want_final)
    st = ssd_device_status()
    assert st == 0, f"device status {st}: {ssd_last_error()}"
    return y, hf


def lane_inputs(ex, b, h, H, G):
    """One (b, h) lane of exact inputs as a batch-1, one-head, one-group problem."""
    g = h // (H // G)
    return dict(
        x=ex["x"][b:b + 1, :, h:h + 1, :],
        dt=ex["dt"][b:b + 1, :, h:h + 1],
        A=ex["A"][h:h + 1],
        B=ex["B"][b:b + 1, :, g:g + 1, :],
        C=ex["C"][b:b + 1, :, g:g + 1, :],
        D=ex["D"][h:h + 1] if ex.get("D") is not None else None,
        h0=ex["h0"][b:b + 1, h:h + 1] if ex.get("h0") is not None else None,
    )


def oracle_lanes(ex, lanes, H, G, nthreads=0):
    """Oracle y (L,P) and h_final (P,N) for each sampled (b, h) lane. Lanes
    run concurrently on the host cores (the oracle is a C call that releases
    the interpreter lock), each single-threaded."""
    import concurrent.futures as cf
    import os

    def one(lane):
        b, h = lane
        li = lane_inputs(ex, b, h, H, G)
        y, hf = oracle.ssd_forward(li["x"], li["dt"], li["A"], li["B"], li["C"], li["D"],
                                   li["h0"], nthreads=1)
        return y[0, :, 0, :], hf[0, 0]

    workers = nthreads or max(1, min(len(lanes), os.cpu_count() or 1))
    with cf.ThreadPoolExecutor(max_workers=workers) as pool:
        return list(pool.map(one, lanes))


def spread_lanes(batch, nheads, ngroups, count, seed, must=()):
    """`count` distinct (b, h) lanes (at most batch * nheads): the ones in
    `must` first; then (batch, group) pairs not yet covered, groups cycling
    fastest over a random order of batches, each with a random head of its
    group; then random lanes."""
    rng = np.random.default_rng(seed)
    hpg = nheads // ngroups
    count = min(count, batch * nheads)
    out = []
    for lane in must:
        lane = (int(lane[0]), int(lane[1]))
        if lane not in out:
            out.append(lane)
    covered = {(b, h // hpg) for b, h in out}
    bperm = rng.permutation(batch)
    for i in range(batch * ngroups):
        if len(out) >= count:
            break
        b, g = int(bperm[(i // ngroups) % batch]), i % ngroups
        if (b, g) in covered:
            continue
        covered.add((b, g))
        out.append((b, int(g * hpg + rng.integers(hpg))))
    while len(out) < count:
        lane = (int(rng.integers(batch)), int(rng.integers(nheads)))
        if lane not in out:
            out.append(lane)
    return out


def rel_err(got, ref):
    """max |got - ref| / rms(ref)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.max(np.abs(got - ref))) / max(rms, 1e-300)


def tolerance(dtype: str) -> float:
    """Parity bound as a fraction of rms(oracle): 1e-4 for fp32 I/O, 2e-2 for
    bf16 I/O (fp32 accumulation and state in both)."""
    return 1e-4 if dtype == synth.F32 else 2e-2
