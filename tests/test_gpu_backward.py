"""The backward pass on the GPU against the oracle's exact adjoint (itself
pinned by finite differences), through the C ABI. The GPU accumulates in fp32
from the stored inputs; each gradient must match within 1e-4 of its rms for
fp32 I/O and 1e-3 for bf16 I/O (no intermediate is rounded to bf16)."""
import numpy as np
import pytest

import oracle
import synth
from tests.helpers import to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

KEYS = ("dx", "ddt", "dA", "dB", "dC", "dD", "dh0")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from selective_state_space_12_b200 import build

    build.build()


def _rel(got, ref):
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.abs(got - ref).max()) / max(rms, 1e-30)


def _check(w, h0=True, dhf=True, tol=None, edit=None):
    from selective_state_space_12_b200 import ssd_backward, ssd_device_status, ssd_last_error

    inp = synth.forward_inputs(w)
    if edit:
        edit(inp)
    rng = np.random.default_rng(w.seed + 5)
    dy_np = synth.store(rng.standard_normal((w.batch, w.seqlen, w.nheads, w.headdim)), w.dtype)
    dhf_np = rng.standard_normal((w.batch, w.nheads, w.headdim, w.dstate)).astype(np.float32)
    dev = {k: to_device(v, w.dtype) for k, v in inp.items()}
    dy = to_device(dy_np, w.dtype)
    dhf_d = torch.from_numpy(dhf_np).cuda() if dhf else None
    g = ssd_backward(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"],
                     dev["h0"] if h0 else None, dy, dhf_d)
    st = ssd_device_status()
    assert st == 0, f"device status {st}: {ssd_last_error()}"
    ex = synth.exact_inputs(inp, w.dtype)
    ref = oracle.ssd_backward(ex["x"], ex["dt"], ex["A"], ex["B"], ex["C"], ex["D"],
                              ex["h0"] if h0 else None, synth.exact(dy_np, w.dtype),
                              dhf_np.astype(np.float64) if dhf else None)
    tol = tol or (1e-4 if w.dtype == synth.F32 else 1e-3)
    errs = {k: _rel(g[k].cpu().numpy().astype(np.float64), ref[k]) for k in KEYS}
    assert all(e <= tol for e in errs.values()), errs
    return errs


def test_backward_f32_ragged_two_groups():
    w = synth.WORKLOADS["tiny_f32"].with_(batch=2, seqlen=150, nheads=4, headdim=32, dstate=32,
                                          ngroups=2, h0_std=0.3, seed=4001)
    _check(w)


@pytest.mark.parametrize("h0,dhf", [(False, False), (True, False), (False, True)])
def test_backward_f32_optional_state_terms(h0, dhf):
    w = synth.WORKLOADS["tiny_f32"].with_(batch=1, seqlen=70, nheads=2, headdim=16, dstate=16,
                                          h0_std=0.3, seed=4002)
    _check(w, h0=h0, dhf=dhf)


def test_backward_bf16_layer_shapes():
    # the 2.7B-style layer's head and state shapes (P 64, N 128), several chunks
    w = synth.WORKLOADS["mamba2_2p7b_layer"].with_(batch=2, seqlen=300, nheads=2, h0_std=0.2,
                                                   seed=4003)
    _check(w)


def test_backward_bf16_decay_that_does_not_fall():
    # the tensor-core kernels split a chunk's decays into row and column
    # factors only where c falls along the chunk (A <= 0, no negative step);
    # here head 0 has A > 0 and head 1 one negative step in its first chunk,
    # so those chunks take the per-element exponentials
    w = synth.WORKLOADS["mamba2_2p7b_layer"].with_(batch=1, seqlen=300, nheads=2, h0_std=0.2,
                                                   seed=4006)

    def edit(inp):
        inp["A"][0] = 0.02
        inp["dt"][0, 5, 1] = synth.store(np.array([-0.01]), w.dtype)[0]

    _check(w, edit=edit)


def test_backward_f32_wide_state_takes_short_chunks():
    # P 64, N 256: the chunk tiles fit only with 32-token chunks
    w = synth.WORKLOADS["tiny_f32"].with_(batch=1, seqlen=100, nheads=2, headdim=64,
                                          dstate=256, h0_std=0.2, seed=4004)
    _check(w)


def test_backward_empty_sequence():
    from selective_state_space_12_b200 import ssd_backward

    H, P, N = 2, 16, 16
    e = lambda *s: torch.empty(s, dtype=torch.float32, device="cuda")
    dhf = torch.randn(1, H, P, N, device="cuda")
    g = ssd_backward(e(1, 0, H, P), e(1, 0, H), -torch.ones(H, device="cuda"), e(1, 0, 1, N),
                     e(1, 0, 1, N), torch.ones(H, device="cuda"), None, e(1, 0, H, P), dhf)
    torch.cuda.synchronize()
    assert torch.equal(g["dh0"], dhf)
    assert not torch.any(g["dA"]).item() and not torch.any(g["dD"]).item()


def test_backward_rejects_tiles_too_large():
    from selective_state_space_12_b200 import SSDError, ssd_backward

    H, P, N = 1, 128, 256
    e = lambda *s: torch.zeros(s, dtype=torch.float32, device="cuda")
    with pytest.raises(SSDError):
        ssd_backward(e(1, 8, H, P), e(1, 8, H), -torch.ones(H, device="cuda"), e(1, 8, 1, N),
                     e(1, 8, 1, N), None, None, e(1, 8, H, P))


def test_backward_bf16_full_length_reduced_heads():
    # the 2.7B-style layer's full sequence (L 2048, 16 chunks) and shapes, on
    # four heads of two batches; every gradient element by element
    w = synth.WORKLOADS["mamba2_2p7b_layer"].with_(batch=2, nheads=4, h0_std=0.1, seed=4020)
    _check(w)


def _lane_backward(ex, dy_ex, dhf_ex, lanes, H, G):
    """The oracle's adjoint of each sampled (b, h) lane as a one-lane problem
    (lanes run concurrently; the oracle is a C call that releases the
    interpreter lock)."""
    import concurrent.futures as cf
    import os

    from tests.helpers import lane_inputs

    def one(lane):
        b, h = lane
        li = lane_inputs(ex, b, h, H, G)
        return oracle.ssd_backward(li["x"], li["dt"], li["A"], li["B"], li["C"], li["D"],
                                   li["h0"], dy_ex[b:b + 1, :, h:h + 1, :],
                                   dhf_ex[b:b + 1, h:h + 1])

    with cf.ThreadPoolExecutor(max_workers=max(1, min(len(lanes), os.cpu_count() or 1))) as p:
        return list(p.map(one, lanes))


def test_backward_full_size_sampled_lanes():
    # The backward at the size the benchmark times it (b8 L2048 H80 P64 N128
    # G1, bf16, same launch configuration), with an initial state. dy and
    # dh_final are nonzero on eight sampled lanes only, so every other lane's
    # dx, ddt and dh0 must be exactly zero, and the shared gradients are sums
    # over the sampled lanes alone: dA and dD over the lanes of a head, dB and
    # dC over the lanes of a batch (one group). The oracle computes each
    # sampled lane's adjoint.
    from selective_state_space_12_b200 import ssd_backward, ssd_device_status, ssd_last_error

    w = synth.WORKLOADS["mamba2_2p7b_layer"].with_(h0_std=0.1, seed=4030)
    b_, L, H, P, N, G = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups
    lanes = [(0, 0), (0, 41), (3, 41), (3, 79), (5, 17), (7, 5), (7, 63), (7, 79)]
    inp = synth.forward_inputs(w)
    rng = np.random.default_rng(w.seed + 5)
    dy_np = np.zeros((b_, L, H, P), dtype=np.uint16)
    dhf_np = np.zeros((b_, H, P, N), dtype=np.float32)
    for b, h in lanes:
        dy_np[b, :, h, :] = synth.store(rng.standard_normal((L, P)), w.dtype)
        dhf_np[b, h] = rng.standard_normal((P, N)).astype(np.float32)
    dev = {k: to_device(v, w.dtype) for k, v in inp.items()}
    g = ssd_backward(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["h0"],
                     to_device(dy_np, w.dtype), torch.from_numpy(dhf_np).cuda())
    st = ssd_device_status()
    assert st == 0, f"device status {st}: {ssd_last_error()}"
    got = {k: g[k].cpu().numpy().astype(np.float64) for k in KEYS}
    ex = synth.exact_inputs(inp, w.dtype)
    ref = _lane_backward(ex, synth.exact(dy_np, w.dtype), dhf_np.astype(np.float64), lanes, H, G)
    tol = 1e-3
    sel = np.zeros((b_, H), dtype=bool)
    for (b, h), r in zip(lanes, ref):
        sel[b, h] = True
        for k, v in (("dx", got["dx"][b, :, h, :]), ("ddt", got["ddt"][b, :, h]),
                     ("dh0", got["dh0"][b, h])):
            e = _rel(v, r[k][0, :, 0] if k != "dh0" else r[k][0, 0])
            assert e <= tol, (b, h, k, e)
    # lanes without a gradient signal: exactly zero
    assert not got["dx"].transpose(0, 2, 1, 3)[~sel].any()
    assert not got["ddt"].transpose(0, 2, 1)[~sel].any()
    assert not got["dh0"][~sel].any()
    # shared gradients: sums over the sampled lanes
    heads = sorted({h for _, h in lanes})
    for k in ("dA", "dD"):
        want = np.array([sum(r[k][0] for (b, h), r in zip(lanes, ref) if h == hh)
                         for hh in heads])
        e = _rel(got[k][heads], want)
        assert e <= tol, (k, e)
    for bb in sorted({b for b, _ in lanes}):
        for k in ("dB", "dC"):
            want = sum(r[k][0] for (b, h), r in zip(lanes, ref) if b == bb)
            e = _rel(got[k][bb], want)
            assert e <= tol, (k, bb, e)
    for bb in set(range(b_)) - {b for b, _ in lanes}:
        assert not got["dB"][bb].any() and not got["dC"][bb].any()
    others = sorted(set(range(H)) - {h for _, h in lanes})
    assert not got["dA"][others].any() and not got["dD"][others].any()


@pytest.mark.parametrize("chain", ["0", "1"])
def test_backward_bf16_state_chains_and_passes(chain, monkeypatch):
    # the tensor-core chunk states as lane-walking chains (=1) or as per-chunk
    # kernels with the CUDA-core passes (=0), forced on one small problem:
    # ragged last chunk, two groups, h0 and dh_final
    monkeypatch.setenv("LIBSSD_BACKWARD_CHAIN", chain)
    w = synth.WORKLOADS["mamba2_2p7b_layer"].with_(batch=2, seqlen=300, nheads=4, ngroups=2,
                                                   h0_std=0.2, seed=4020)
    _check(w)


@pytest.mark.parametrize("path", ["simt", "tc"])
def test_backward_bf16_both_paths(path, monkeypatch):
    # bf16 P 64 N 128 takes the tensor-core per-chunk kernels unless
    # LIBSSD_BACKWARD_PATH=simt; both against the oracle (ragged, two groups)
    monkeypatch.setenv("LIBSSD_BACKWARD_PATH", path)
    w = synth.WORKLOADS["mamba2_2p7b_layer"].with_(batch=2, seqlen=300, nheads=4, ngroups=2,
                                                   h0_std=0.2, seed=4010)
    _check(w)


@pytest.mark.parametrize("L", [1, 127, 128, 129, 256])
def test_backward_bf16_tc_chunk_boundaries(L):
    # one token, a chunk short by one, exact chunks, one token into a chunk
    w = synth.WORKLOADS["mamba2_2p7b_layer"].with_(batch=1, seqlen=L, nheads=2,
                                                   h0_std=0.2, seed=4011 + L)
    _check(w)
