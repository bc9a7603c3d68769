"""The tensor-core kernels' failure path, driven on purpose without faulting
anything: every wait between the forward's warp roles, and every wait of the
backward's chunk-state and per-chunk gradient kernels, is bounded, and a wait
that runs out makes the kernel stop, let its copies and tensor-core work in
flight finish, free its tensor memory, store nothing and report
SSD_ERR_TIMEOUT.
Here the bound is set to a few clock cycles, so the first wait that is not
already satisfied gives up; the device stays usable and the next call with the
default bound computes normally."""
import pytest

import oracle
import synth
from tests.helpers import rel_err, to_device, to_f64, tolerance

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

SSD_ERR_TIMEOUT = 5


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from selective_state_space_12_b200 import build

    build.build()


@pytest.mark.parametrize("nheads,seqlen", [
    (4, 3 * 128 + 5),   # few lanes: state-only pass, state pass, full pass (two kernels wait)
    (160, 2 * 128),     # more lanes than SMs: the last lanes cut in two, a cross-CTA flag
])
def test_forward_bounded_wait_reports_timeout_then_recovers(nheads, seqlen):
    from selective_state_space_12_b200 import (ssd_device_status, ssd_forward, ssd_last_error,
                                               ssd_set_wait_limit)

    w = synth.WORKLOADS["mamba2_2p7b_layer"].with_(batch=1, seqlen=seqlen, nheads=nheads,
                                                   h0_std=0.2, seed=900 + nheads)
    inp = synth.forward_inputs(w)
    d = {k: to_device(v, w.dtype) for k, v in inp.items()}
    assert ssd_device_status() == 0
    ssd_set_wait_limit(16)
    try:
        ssd_forward(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"], chunk=w.chunk)
        st = ssd_device_status()
        msg = ssd_last_error()
    finally:
        ssd_set_wait_limit(0)
    assert st == SSD_ERR_TIMEOUT, (st, msg)
    assert "gave up" in msg
    # the error word was cleared by the query; the device computes normally
    assert ssd_device_status() == 0
    y, hf = ssd_forward(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"], chunk=w.chunk)
    assert ssd_device_status() == 0
    ex = synth.exact_inputs(inp, w.dtype)
    yr, hr = oracle.ssd_forward(ex["x"], ex["dt"], ex["A"], ex["B"], ex["C"], ex["D"], ex["h0"])
    tol = tolerance(w.dtype)
    assert rel_err(to_f64(y), yr) <= tol
    assert rel_err(to_f64(hf), hr) <= tol


@pytest.mark.parametrize("batch", [2, 4])
def test_backward_bounded_wait_reports_timeout_then_recovers(batch):
    # bf16 P 64 N 128 on the tensor cores: with 160 lanes the per-chunk state
    # kernels, with 320 (more than two per SM) the lane-walking chains; then
    # the persistent per-chunk gradient kernel over 3 chunks x 80 heads x
    # batch items, more than one per SM, so its loop leaves early on the abort
    from selective_state_space_12_b200 import (ssd_backward, ssd_device_status, ssd_last_error,
                                               ssd_set_wait_limit)
    from tests.test_gpu_backward import _check

    w = synth.WORKLOADS["mamba2_2p7b_layer"].with_(batch=batch, seqlen=2 * 128 + 37, nheads=80,
                                                   h0_std=0.2, seed=950 + batch)
    inp = synth.forward_inputs(w)
    d = {k: to_device(v, w.dtype) for k, v in inp.items()}
    dy = torch.randn(d["x"].shape, device="cuda").to(d["x"].dtype)
    assert ssd_device_status() == 0
    ssd_set_wait_limit(16)
    try:
        ssd_backward(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"], dy, None)
        st = ssd_device_status()
        msg = ssd_last_error()
    finally:
        ssd_set_wait_limit(0)
    assert st == SSD_ERR_TIMEOUT, (st, msg)
    assert "gave up" in msg
    assert ssd_device_status() == 0
    # the next call with the default bound matches the oracle's adjoint
    _check(w)
