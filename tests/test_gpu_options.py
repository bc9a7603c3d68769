"""Step options (per-head bias, softplus, clamp, zero-order-hold input
weight) on the GPU against the fp64 oracle, through the C ABI.

The kernels prepare each raw step themselves ("精读笔记 #12：Mamba", section 3:
the step is a softplus of a projection; section 2.2: the zero-order hold
B_bar = (Delta A)^-1 (exp(Delta A) - I) Delta B). Inputs are the seeded
workloads with the step left raw (synth.forward_inputs_raw). Bounds as for
the plain layer: max abs error <= 1e-4 rms (fp32 I/O), 2e-2 rms (bf16 I/O),
for y and the final state.
"""
import numpy as np
import pytest

import oracle
import synth
from tests.helpers import lane_inputs, rel_err, to_device, to_f64, tolerance

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

OPTION_SETS = {
    "softplus_bias": dict(softplus=True),
    "softplus_bias_zoh": dict(softplus=True, zoh=True),
    "softplus_bias_clamp_zoh": dict(softplus=True, zoh=True, dt_limit=(0.004, 0.05)),
}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from selective_state_space_12_b200 import build

    build.build()


def _oracle_opts(ex, o):
    lo, hi = o.get("dt_limit", (0.0, 0.0))
    return oracle.DtOptions(bias=ex["dt_bias"], softplus=o.get("softplus", False), dt_min=lo,
                            dt_max=hi, zoh=o.get("zoh", False))


def _gpu(inp, w, o, chunk=None):
    from selective_state_space_12_b200 import ssd_device_status, ssd_forward_ex, ssd_last_error

    dev = {k: to_device(v, w.dtype) for k, v in inp.items() if k != "dt_bias"}
    bias = torch.from_numpy(inp["dt_bias"]).cuda()
    y, hf = ssd_forward_ex(dev["x"], dev["dt"], dev["A"], dev["B"], dev["C"], dev["D"],
                           dev["h0"], chunk=chunk or w.chunk, dt_bias=bias,
                           dt_softplus=o.get("softplus", False), dt_limit=o.get("dt_limit"),
                           zoh=o.get("zoh", False))
    st = ssd_device_status()
    assert st == 0, f"device status {st}: {ssd_last_error()}"
    return y, hf


def _check(w, o, chunk=None):
    inp = synth.forward_inputs_raw(w)
    ex = synth.exact_inputs(inp, w.dtype)
    y, hf = _gpu(inp, w, o, chunk)
    yr, hr = oracle.ssd_forward_ex(ex["x"], ex["dt"], ex["A"], ex["B"], ex["C"], ex["D"],
                                   ex["h0"], _oracle_opts(ex, o))
    tol = tolerance(w.dtype)
    ey, eh = rel_err(to_f64(y), yr), rel_err(to_f64(hf), hr)
    assert ey <= tol and eh <= tol, (ey, eh)
    return yr


@pytest.mark.parametrize("opt", sorted(OPTION_SETS))
def test_options_f32_ragged(opt):
    w = synth.WORKLOADS["tiny_f32"].with_(batch=2, seqlen=300, nheads=4, headdim=32, dstate=32,
                                          ngroups=2, h0_std=0.3, seed=41)
    _check(w, OPTION_SETS[opt], chunk=64)


@pytest.mark.parametrize("opt", sorted(OPTION_SETS))
@pytest.mark.parametrize("name", ["mamba2_2p7b_layer", "hybrid_8b_layer_N64",
                                  "hybrid_8b_layer_N256"])
def test_options_bf16_tensor_core(name, opt):
    base = synth.WORKLOADS[name]
    w = base.with_(batch=2, seqlen=3 * base.chunk + 37, nheads=2 * base.ngroups,
                   h0_std=0.2, seed=base.seed + 23)
    _check(w, OPTION_SETS[opt])


def test_options_bf16_segmented_lanes():
    # few lanes, long sequence: the state-only pass and the segment chain
    # take the prepared steps too
    w = synth.WORKLOADS["long_seq_65k"].with_(seqlen=4096 + 77, nheads=4, seed=52)
    _check(w, OPTION_SETS["softplus_bias_zoh"])


def test_options_change_the_result():
    # the hold weight is not the Euler weight: a kernel that ignored the
    # option would fail the parity above, and here differs from it visibly
    w = synth.WORKLOADS["mamba2_2p7b_layer"].with_(batch=1, seqlen=300, nheads=2, seed=61)
    inp = synth.forward_inputs_raw(w)
    y1, _ = _gpu(inp, w, dict(softplus=True))
    y2, _ = _gpu(inp, w, dict(softplus=True, zoh=True))
    assert rel_err(to_f64(y1), to_f64(y2)) > 1e-3


def test_options_full_size_sampled_lanes():
    # the 2.7B-style layer at full size, as the benchmark's options leg runs it
    w = synth.WORKLOADS["mamba2_2p7b_layer"]
    o = OPTION_SETS["softplus_bias_zoh"]
    inp = synth.forward_inputs_raw(w)
    y, hf = _gpu(inp, w, o)
    ex = synth.exact_inputs(inp, w.dtype)
    tol = tolerance(w.dtype)
    for b, h in [(0, 0), (w.batch - 1, w.nheads - 1), (3, 41)]:
        li = lane_inputs(ex, b, h, w.nheads, w.ngroups)
        oo = _oracle_opts(ex, o)
        oo.bias = ex["dt_bias"][h:h + 1]
        yr, hr = oracle.ssd_forward_ex(li["x"], li["dt"], li["A"], li["B"], li["C"], li["D"],
                                       li["h0"], oo)
        ey = rel_err(to_f64(y[b, :, h, :]), yr[0, :, 0, :])
        eh = rel_err(to_f64(hf[b, h]), hr[0, 0])
        assert ey <= tol and eh <= tol, (b, h, ey, eh)


@pytest.mark.parametrize("dtype", [synth.F32, synth.BF16])
@pytest.mark.parametrize("P,N,G", [(64, 128, 8), (32, 48, 2)])
def test_decode_options_every_step(dtype, P, N, G):
    from selective_state_space_12_b200 import ssd_step_ex

    w = synth.DECODE_WORKLOADS["decode_b256"].with_(batch=3, nheads=16, headdim=P, dstate=N,
                                                    ngroups=G, dtype=dtype, seed=71 + N)
    prm = synth.decode_params(w)
    bias32 = prm["dt_bias"].astype(np.float32)
    h_np = synth.decode_state(w)
    h = torch.from_numpy(h_np).cuda()
    A = torch.from_numpy(prm["A"]).cuda()
    D = torch.from_numpy(prm["D"]).cuda()
    bias = torch.from_numpy(bias32).cuda()
    Af, Df = prm["A"].astype(np.float64), prm["D"].astype(np.float64)
    opts = oracle.DtOptions(bias=bias32.astype(np.float64), softplus=True, dt_min=1e-3,
                            dt_max=0.08, zoh=True)
    h_ref = h_np.astype(np.float64)
    tol = tolerance(w.dtype)
    for s in range(6):
        si = synth.decode_step_inputs_raw(w, s)
        ex = synth.exact_inputs(si, w.dtype)
        dev = {k: to_device(v, w.dtype) for k, v in si.items()}
        y = ssd_step_ex(h, dev["x"], dev["dt"], A, dev["B"], dev["C"], D, dt_bias=bias,
                        dt_softplus=True, dt_limit=(1e-3, 0.08), zoh=True)
        torch.cuda.synchronize()
        yr, h_ref = oracle.ssd_step_ex(h_ref, ex["x"], ex["dt"], Af, ex["B"], ex["C"], Df, opts)
        ey, eh = rel_err(to_f64(y), yr), rel_err(h.cpu().numpy(), h_ref)
        assert ey <= tol and eh <= tol, (s, ey, eh)
