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


def _check(w, h0=True, dhf=True, tol=None):
    from selective_state_space_12_b200 import ssd_backward, ssd_device_status, ssd_last_error

    inp = synth.forward_inputs(w)
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
