"""The selective scan (diagonal A per channel) on the GPU against the fp64
oracle, through the C ABI ("精读笔记 #12：Mamba", sections 2.2 and 3). Bounds
as for the layer: max abs error <= 1e-4 rms (fp32 I/O), 2e-2 rms (bf16 I/O),
for y and the final state."""
import numpy as np
import pytest

import oracle
import synth
from tests.helpers import rel_err, to_device, to_f64, tolerance

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

VARIANTS = {"euler_softplus": dict(softplus=True), "zoh_softplus": dict(softplus=True, zoh=True),
            "zoh_softplus_clamp": dict(softplus=True, zoh=True, dt_limit=(0.004, 0.05))}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from selective_state_space_12_b200 import build

    build.build()


def _run(w, o, want_final=True):
    from selective_state_space_12_b200 import (ssd_device_status, ssd_last_error,
                                               ssd_selective_scan)

    inp = synth.scan_inputs(w)
    d = {k: (None if v is None else to_device(v, w.dtype)) for k, v in inp.items()
         if k not in ("A", "dt_bias", "Dskip", "h0")}
    f32 = {k: (None if inp[k] is None else torch.from_numpy(inp[k]).cuda())
           for k in ("A", "dt_bias", "Dskip", "h0")}
    y, hf = ssd_selective_scan(d["x"], d["dt"], f32["A"], d["B"], d["C"], f32["Dskip"],
                               f32["h0"], dt_bias=f32["dt_bias"],
                               dt_softplus=o.get("softplus", False), dt_limit=o.get("dt_limit"),
                               zoh=o.get("zoh", False), want_final=want_final)
    st = ssd_device_status()
    assert st == 0, f"device status {st}: {ssd_last_error()}"
    return inp, y, hf


def _oracle_opts(ex, o):
    lo, hi = o.get("dt_limit", (0.0, 0.0))
    return oracle.DtOptions(bias=ex["dt_bias"], softplus=o.get("softplus", False), dt_min=lo,
                            dt_max=hi, zoh=o.get("zoh", False))


def _check(w, o):
    inp, y, hf = _run(w, o)
    ex = synth.exact_inputs(inp, w.dtype)
    yr, hr = oracle.selective_scan(ex["x"], ex["dt"], ex["A"], ex["B"], ex["C"], ex["Dskip"],
                                   ex["h0"], _oracle_opts(ex, o))
    tol = tolerance(w.dtype)
    ey, eh = rel_err(to_f64(y), yr), rel_err(hf.cpu().numpy(), hr)
    assert ey <= tol and eh <= tol, (ey, eh)


@pytest.mark.parametrize("v", sorted(VARIANTS))
@pytest.mark.parametrize("N", [4, 8, 16])
def test_scan_f32(v, N):
    w = synth.SCAN_WORKLOADS["scan_tiny_f32"].with_(batch=2, seqlen=150, channels=72, dstate=N,
                                                    ngroups=2, h0_std=0.3, seed=3000 + N)
    _check(w, VARIANTS[v])


@pytest.mark.parametrize("v", sorted(VARIANTS))
def test_scan_bf16_reduced(v):
    w = synth.SCAN_WORKLOADS["mamba1_2p8b_scan"].with_(batch=2, seqlen=333, channels=320,
                                                       h0_std=0.2, seed=3100)
    _check(w, VARIANTS[v])


# the staged (shared-memory) kernel: fp32 and bf16, several groups whose
# channels tile its blocks, a partial last block, N = 8 and 16
STAGED = [(synth.F32, 16, 128, 2), (synth.F32, 8, 256, 2), (synth.BF16, 16, 40, 1),
          (synth.BF16, 8, 128, 2), (synth.BF16, 16, 192, 3)]


@pytest.mark.parametrize("dtype,N,D,G", STAGED)
def test_scan_staged_kernel_shapes(dtype, N, D, G):
    w = synth.SCAN_WORKLOADS["scan_tiny_f32"].with_(batch=2, seqlen=200, channels=D, dstate=N,
                                                    ngroups=G, dtype=dtype, h0_std=0.3,
                                                    seed=3300 + D + N)
    _check(w, VARIANTS["zoh_softplus"])


def test_scan_empty_sequence_copies_initial_state():
    w = synth.SCAN_WORKLOADS["scan_tiny_f32"].with_(seqlen=0, h0_std=0.5, seed=3200)
    inp, y, hf = _run(w, VARIANTS["zoh_softplus"])
    assert y.numel() == 0
    assert np.array_equal(hf.cpu().numpy(), inp["h0"])


def test_scan_full_size_sampled_channels():
    # the benchmark's workload (b8 L2048 D5120 N16, bf16, softplus + ZOH),
    # checked on sampled (batch, channel) lanes over the whole sequence
    w = synth.SCAN_WORKLOADS["mamba1_2p8b_scan"]
    o = VARIANTS["zoh_softplus"]
    inp, y, hf = _run(w, o)
    ex = synth.exact_inputs(inp, w.dtype)
    tol = tolerance(w.dtype)
    for b, dch in [(0, 0), (7, 5119), (3, 2500), (5, 1)]:
        sl = lambda a: a[b:b + 1, :, dch:dch + 1]
        oo = _oracle_opts(ex, o)
        oo.bias = ex["dt_bias"][dch:dch + 1]
        yr, hr = oracle.selective_scan(sl(ex["x"]), sl(ex["dt"]), ex["A"][dch:dch + 1],
                                       ex["B"][b:b + 1], ex["C"][b:b + 1],
                                       ex["Dskip"][dch:dch + 1], None, oo)
        ey = rel_err(to_f64(y[b, :, dch]), yr[0, :, 0])
        eh = rel_err(hf[b, dch].cpu().numpy(), hr[0, 0])
        assert ey <= tol and eh <= tol, (b, dch, ey, eh)
    assert torch.isfinite(y).all().item()
