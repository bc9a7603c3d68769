"""HostForward (pinned host buffers in and out, batch slices overlapped on
three streams) gives the forward's own results."""
import numpy as np
import pytest

import synth
from tests.helpers import to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("splits,h0", [(1, False), (3, True), (4, False)])
def test_host_forward_equals_device_forward(splits, h0):
    from selective_state_space_12_b200 import HostForward, build, ssd_forward

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    w = synth.WORKLOADS["mamba2_2p7b_layer"].with_(batch=5, seqlen=300, nheads=4,
                                                   h0_std=0.3 if h0 else 0.0, seed=91)
    inp = synth.forward_inputs(w)
    dev = {k: to_device(v, w.dtype) for k, v in inp.items()}
    host = {k: (None if v is None else v.cpu().pin_memory()) for k, v in dev.items()}
    y_h = torch.empty(dev["x"].shape, dtype=dev["x"].dtype).pin_memory()
    hf_h = torch.empty((w.batch, w.nheads, w.headdim, w.dstate)).pin_memory()
    hfw = HostForward(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups,
                      dev["x"].dtype, chunk=w.chunk, splits=splits, h0=h0)
    hfw(host["x"], host["dt"], host["A"], host["B"], host["C"], host["D"], y_h, hf_h,
        h0=host["h0"])
    torch.cuda.synchronize()
    y, hf = ssd_forward(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"], dev["h0"],
                        chunk=w.chunk)
    torch.cuda.synchronize()
    # the slices run the same kernels on the same rows; only the lane-count
    # dependent work split (segments) may change rounding
    yd, yr = y_h.float().numpy(), y.float().cpu().numpy()
    rms = float(np.sqrt(np.mean(yr ** 2)))
    assert np.abs(yd - yr).max() <= 2e-2 * rms
    assert np.abs(hf_h.numpy() - hf.cpu().numpy()).max() <= 1e-3 * float(
        np.sqrt(np.mean(hf.cpu().numpy() ** 2)))
