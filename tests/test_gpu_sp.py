"""Sequence parallelism on the GPU through the C ABI: ssd_forward_state (end
state from a zero state, total decay) against the fp64 oracle, and a
sequence split into pieces (ranks emulated one after another on one GPU; the
pieces' kernels never wait on one another) against the oracle's forward over
the unsplit sequence. Bounds as for the forward: 1e-4 rms (fp32 I/O), 2e-2
rms (bf16 I/O), for y and the final state."""
import socket

import numpy as np
import pytest

import oracle
import synth
from tests.helpers import rel_err, to_device, to_f64, tolerance

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from selective_state_space_12_b200 import build

    build.build()


def _dev(inp, w):
    d = {k: to_device(v, w.dtype) for k, v in inp.items() if k != "dt_bias" and v is not None}
    if inp.get("dt_bias") is not None:
        d["dt_bias"] = torch.from_numpy(inp["dt_bias"]).cuda()
    return d


def _opts(ex, step):
    if not step:
        return oracle.DtOptions()
    return oracle.DtOptions(bias=ex["dt_bias"], softplus=True, zoh=True)


CASES = {
    # name: (workload, overrides, step options)
    "bf16_tc": ("mamba2_2p7b_layer", dict(batch=2, seqlen=1000, nheads=3, seed=81), False),
    "bf16_tc_segmented": ("long_seq_65k", dict(seqlen=6000, nheads=2, seed=82), False),
    "bf16_tc_options": ("hybrid_8b_layer_N64", dict(batch=1, seqlen=700, nheads=16, seed=83),
                        True),
    "f32_simt_options": ("tiny_f32", dict(batch=2, seqlen=400, nheads=4, headdim=32, dstate=32,
                                          ngroups=2, h0_std=0.3, seed=84), True),
}


def _case(name):
    wl, kw, step = CASES[name]
    w = synth.WORKLOADS[wl].with_(**kw)
    inp = synth.forward_inputs_raw(w) if step else synth.forward_inputs(w)
    return w, inp, step


@pytest.mark.parametrize("name", sorted(CASES))
def test_forward_state_matches_oracle(name):
    from selective_state_space_12_b200 import ssd_device_status, ssd_forward_state

    w, inp, step = _case(name)
    d = _dev(inp, w)
    extra = dict(dt_bias=d["dt_bias"], dt_softplus=True, zoh=True) if step else {}
    S, lam = ssd_forward_state(d["x"], d["dt"], d["A"], d["B"], chunk=w.chunk, **extra)
    assert ssd_device_status() == 0
    ex = synth.exact_inputs(inp, w.dtype)
    o = _opts(ex, step)
    _, h_ref = oracle.ssd_forward_ex(ex["x"], ex["dt"], ex["A"], ex["B"], ex["B"], None, None, o)
    _, ell, _ = oracle.dt_prepare(ex["dt"], ex["A"], o)
    lam_ref = np.exp(ell.sum(axis=1))
    assert rel_err(S.cpu().numpy(), h_ref) <= tolerance(w.dtype)
    lam_g = lam.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(lam_g - lam_ref) <= 1e-3 * lam_ref + 1e-30), (lam_g, lam_ref)


@pytest.mark.parametrize("name", sorted(CASES))
def test_pieces_chained_equal_unsplit_forward(name):
    from selective_state_space_12_b200 import (ssd_device_status, ssd_forward, ssd_forward_ex,
                                               ssd_forward_state, ssd_state_chain)

    w, inp, step = _case(name)
    d = _dev(inp, w)
    extra = dict(dt_bias=d["dt_bias"], dt_softplus=True, zoh=True) if step else {}
    h0 = d.get("h0")
    L = w.seqlen
    cuts = [0, L // 5, L // 2 + 3, (4 * L) // 5, L]  # four ragged pieces
    R = len(cuts) - 1
    piece = lambda t, r: t[:, cuts[r]:cuts[r + 1]].contiguous()
    parts = [ssd_forward_state(piece(d["x"], r), piece(d["dt"], r), d["A"], piece(d["B"], r),
                               chunk=w.chunk, **extra) for r in range(R)]
    states = torch.stack([p[0] for p in parts])
    decays = torch.stack([p[1] for p in parts])
    ys, h_total = [], None
    for r in range(R):
        h_in, h_tot = ssd_state_chain(states, decays, r, h0=h0, want_total=(r == R - 1))
        args = (piece(d["x"], r), piece(d["dt"], r), d["A"], piece(d["B"], r),
                piece(d["C"], r), d["D"], h_in)
        if step:
            y, _ = ssd_forward_ex(*args, chunk=w.chunk, want_final=False, **extra)
        else:
            y, _ = ssd_forward(*args, chunk=w.chunk, want_final=False)
        ys.append(y)
        if h_tot is not None:
            h_total = h_tot
    assert ssd_device_status() == 0
    ex = synth.exact_inputs(inp, w.dtype)
    y_ref, h_ref = oracle.ssd_forward_ex(ex["x"], ex["dt"], ex["A"], ex["B"], ex["C"], ex["D"],
                                         ex.get("h0"), _opts(ex, step))
    tol = tolerance(w.dtype)
    ey = rel_err(to_f64(torch.cat(ys, dim=1)), y_ref)
    eh = rel_err(h_total.cpu().numpy(), h_ref)
    assert ey <= tol and eh <= tol, (ey, eh)


def test_sp_forward_on_a_one_rank_nccl_group():
    """The product orchestration (NCCL all-gather included) on one rank equals
    the plain forward."""
    import torch.distributed as dist

    from selective_state_space_12_b200 import ssd_forward, sp_forward

    w, inp, _ = _case("bf16_tc")
    d = _dev(inp, w)
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        y, hf = sp_forward(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], chunk=w.chunk)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    y_ref, hf_ref = ssd_forward(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], chunk=w.chunk)
    assert rel_err(to_f64(y), to_f64(y_ref)) <= 1e-2
    assert rel_err(hf.cpu().numpy(), hf_ref.cpu().numpy()) <= 1e-4


def test_forward_state_of_an_empty_piece():
    """A piece of no tokens has a zero end state and decay 1."""
    from selective_state_space_12_b200 import ssd_device_status, ssd_forward_state

    H, P, N = 4, 64, 128
    x = torch.empty((2, 0, H, P), dtype=torch.bfloat16, device="cuda")
    dt = torch.empty((2, 0, H), dtype=torch.bfloat16, device="cuda")
    B = torch.empty((2, 0, 1, N), dtype=torch.bfloat16, device="cuda")
    A = -torch.ones(H, device="cuda")
    S, lam = ssd_forward_state(x, dt, A, B, chunk=256)
    assert ssd_device_status() == 0
    assert torch.count_nonzero(S).item() == 0
    assert torch.all(lam == 1.0).item()
