"""ssd_forward_noalloc: the forward pass for callers that cannot allocate
device memory (it uses a fixed scratch array compiled into the library).

It must give what ssd_forward gives on the same inputs, on two calls in a row
(the second call finds the first call's leftovers in the shared scratch).
This file is named so that pytest collects it last.
"""
import ctypes

import pytest

import synth
from tests.helpers import rel_err, to_device, to_f64, tolerance

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from selective_state_space_12_b200 import _lib, build

    build.build()
    return _lib.load()


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(lib, d, w, chunk):
    from selective_state_space_12_b200 import make_dims

    y = torch.empty_like(d["x"])
    hf = torch.empty((w.batch, w.nheads, w.headdim, w.dstate), dtype=torch.float32,
                     device="cuda")
    dims = make_dims(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups,
                     d["x"].dtype)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.ssd_forward_noalloc(_p(d["x"]), _p(d["dt"]), _p(d["A"]), _p(d["B"]), _p(d["C"]),
                                 _p(d["D"]), _p(d["h0"]), chunk, _p(y), _p(hf),
                                 ctypes.byref(dims), stream)
    assert st == 0, lib.ssd_last_error()
    return y, hf


def _check_two_calls(lib, base, chunk):
    # The two entry points run the same deterministic kernels on the same
    # inputs, so their outputs must be identical bit for bit. Each call draws
    # new inputs, so the second finds the first call's leftovers in the
    # shared scratch.
    from selective_state_space_12_b200 import ssd_forward

    tol = tolerance(base.dtype)
    for call in range(2):
        w = base.with_(seed=base.seed + 31 * call)  # different inputs on each call
        inp = synth.forward_inputs(w)
        d = {k: to_device(v, w.dtype) for k, v in inp.items()}
        y_ref, hf_ref = ssd_forward(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"],
                                    chunk=chunk)
        y, hf = _noalloc(lib, d, w, chunk)
        torch.cuda.synchronize()
        ey = rel_err(to_f64(y), to_f64(y_ref))
        eh = rel_err(to_f64(hf), to_f64(hf_ref))
        assert ey <= tol and eh <= tol, (call, ey, eh)
        assert torch.equal(y, y_ref), (call, "y differs from ssd_forward", ey)
        assert torch.equal(hf, hf_ref), (call, "h_final differs from ssd_forward", eh)


@pytest.mark.parametrize("name,chunk", [("tiny_f32", 16), ("long_seq_65k", 256),
                                        ("hybrid_8b_layer_N128", 128)])
def test_noalloc_matches_ssd_forward_on_two_calls_in_a_row(lib, name, chunk):
    base = synth.WORKLOADS[name]
    if base.dtype == synth.BF16:
        # few lanes: the tensor-core path cuts each lane into segments whose
        # states pass through the scratch
        base = base.with_(batch=2, seqlen=1000, nheads=2 * base.ngroups, h0_std=0.2)
    _check_two_calls(lib, base, chunk)


def test_noalloc_matches_ssd_forward_with_lanes_cut_in_two(lib):
    # More lanes than SMs by a few, and three 128-token blocks per lane (too
    # short to be cut into segments): the last eight lanes are cut in two, and
    # each second half waits for a flag in the scratch that its first half
    # raises. A flag left raised by the previous call would let a second half
    # start from a stale state; each call clears the flags first.
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    base = synth.WORKLOADS["mamba2_2p7b_layer"].with_(batch=1, nheads=sms + 8,
                                                      seqlen=2 * 128 + 37, h0_std=0.3,
                                                      seed=5150)
    _check_two_calls(lib, base, 256)


def test_noalloc_rejects_problems_beyond_its_scratch(lib):
    from selective_state_space_12_b200 import make_dims

    # fp32 I/O always takes the CUDA-core path, whose workspace here is
    # 8*80*8*64*128*4 bytes (168 MB), far above the 32 MiB fixed scratch. Real
    # buffers are passed, so the call would be valid even if it were accepted.
    b, L, H, P, N = 8, 2048, 80, 64, 128
    f = dict(dtype=torch.float32, device="cuda")
    x = torch.zeros(b, L, H, P, **f)
    dt = torch.full((b, L, H), 0.01, **f)
    A = -torch.ones(H, **f)
    B = torch.zeros(b, L, 1, N, **f)
    C = torch.zeros(b, L, 1, N, **f)
    y = torch.empty_like(x)
    dims = make_dims(b, L, H, P, N, 1, torch.float32)
    st = lib.ssd_forward_noalloc(_p(x), _p(dt), _p(A), _p(B), _p(C), None, None, 256, _p(y), None,
                                 ctypes.byref(dims), None)
    torch.cuda.synchronize()
    assert st == 2
    assert b"fixed scratch" in lib.ssd_last_error()
