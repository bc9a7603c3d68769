"""CUDA path vs the fp64 oracle, through the C ABI, on seeded inputs.

Bounds (max abs error as a fraction of the oracle's rms, for y and for the
final state): 1e-4 for fp32 I/O, 2e-2 for bf16 I/O.

Small problems are compared element by element; the full-size workloads, in
the launch configuration the benchmark uses, are compared on sampled
(batch, head) lanes that the oracle computes one by one over the whole
sequence.
"""
import numpy as np
import pytest

import oracle
import synth
from tests.helpers import (gpu_forward, oracle_lanes, rel_err, spread_lanes, to_device, to_f64,
                           tolerance)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from selective_state_space_12_b200 import build

    build.build()


def _full_check(w, chunk=None, D=True, h0=True, want_final=True):
    inp = synth.forward_inputs(w)
    ex = synth.exact_inputs(inp, w.dtype)
    y, hf = gpu_forward(inp, w, chunk=chunk, D=D, h0=h0, want_final=want_final)
    torch.cuda.synchronize()
    yr, hr = oracle.ssd_forward(ex["x"], ex["dt"], ex["A"], ex["B"], ex["C"],
                                ex["D"] if D else None, ex["h0"] if h0 else None)
    tol = tolerance(w.dtype)
    yg = to_f64(y)
    if D or w.dtype == synth.F32:
        ey = rel_err(yg, yr)
        assert ey <= tol, f"y: {ey:.3e} > {tol:.1e}"
    else:
        # Without the skip term, rms(y) loses the D*x part and a few outputs
        # reach ~20x rms, so rounding the exact result to bf16 alone (half an
        # ulp, up to 2^-8 |y|) exceeds 2e-2 rms. The bound adds each output's
        # own half-ulp to the stated 2e-2 rms.
        rms = float(np.sqrt(np.mean(yr * yr)))
        excess = np.abs(yg - yr) - (tol * rms + 2.0 ** -8 * np.abs(yr))
        assert float(excess.max()) <= 0.0, f"y exceeds 2e-2 rms + half-ulp by {excess.max():.3e}"
        ey = rel_err(yg, yr)
    if want_final:
        eh = rel_err(to_f64(hf), hr)
        assert eh <= tol, f"h_final: {eh:.3e} > {tol:.1e}"
    return ey


# ---------------------------------------------------------------------------
# forward, element by element
# ---------------------------------------------------------------------------

def test_forward_tiny_f32_workload():
    _full_check(synth.WORKLOADS["tiny_f32"])


@pytest.mark.parametrize("chunk", [16, 32, 64, 128, 256])
def test_forward_f32_every_chunk_ragged(chunk):
    w = synth.WORKLOADS["tiny_f32"].with_(batch=2, seqlen=300, nheads=4, headdim=32,
                                          dstate=32, ngroups=2, h0_std=0.3, seed=7 + chunk)
    _full_check(w, chunk=chunk)


@pytest.mark.parametrize("P,N", [(16, 16), (64, 128), (128, 256), (48, 80)])
def test_forward_f32_shapes(P, N):
    w = synth.WORKLOADS["tiny_f32"].with_(batch=1, seqlen=200, nheads=2, headdim=P, dstate=N,
                                          ngroups=1, h0_std=0.2, seed=P + N)
    _full_check(w, chunk=64)


@pytest.mark.parametrize("name", ["mamba2_2p7b_layer", "long_seq_65k", "hybrid_8b_layer_N64",
                                  "hybrid_8b_layer_N128", "hybrid_8b_layer_N256"])
def test_forward_bf16_reduced_workloads(name):
    # the workloads' head/state shapes and chunk, fewer tokens and heads,
    # spanning several chunks with a ragged tail
    base = synth.WORKLOADS[name]
    G = base.ngroups
    w = base.with_(batch=2, seqlen=3 * base.chunk + 37, nheads=2 * G, seed=base.seed + 11)
    _full_check(w)


def test_forward_bf16_without_D_h0_or_final_state():
    w = synth.WORKLOADS["long_seq_65k"].with_(seqlen=700, nheads=4, seed=5)
    _full_check(w, D=False, h0=False, want_final=False)


@pytest.mark.parametrize("L", [1, 2, 17, 255, 256, 257])
def test_forward_bf16_short_and_boundary_lengths(L):
    w = synth.WORKLOADS["mamba2_2p7b_layer"].with_(batch=1, seqlen=L, nheads=3, h0_std=0.5,
                                                   seed=100 + L)
    _full_check(w)


def test_forward_empty_sequence_copies_initial_state():
    from selective_state_space_12_b200 import ssd_forward

    H, P, N = 4, 64, 128
    x = torch.empty((2, 0, H, P), dtype=torch.bfloat16, device="cuda")
    dt = torch.empty((2, 0, H), dtype=torch.bfloat16, device="cuda")
    B = torch.empty((2, 0, 1, N), dtype=torch.bfloat16, device="cuda")
    A = -torch.ones(H, device="cuda")
    h0 = torch.randn(2, H, P, N, device="cuda")
    y, hf = ssd_forward(x, dt, A, B, B.clone(), None, h0, chunk=64)
    torch.cuda.synchronize()
    assert y.numel() == 0
    assert torch.equal(hf, h0)


@pytest.mark.parametrize("waves,extra", [(1, 12), (1, 60), (2, 20), (2, 70)])
def test_forward_bf16_lanes_past_a_full_wave(waves, extra):
    # lanes that would leave a partial last wave of CTAs: with fewer than two
    # waves every lane is cut into segments (state-only pass, chaining, full
    # pass from the entering state); with more, the lanes past the last full
    # wave are cut in two, the second half starting from the state the first
    # half hands over. Every lane is checked against the oracle.
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    w = synth.WORKLOADS["mamba2_2p7b_layer"].with_(batch=1, seqlen=4 * 128 + 37,
                                                   nheads=waves * sms + extra, h0_std=0.3,
                                                   seed=300 + extra)
    _full_check(w)


def test_forward_chunk_invariance_on_gpu():
    w = synth.WORKLOADS["hybrid_8b_layer_N128"].with_(batch=1, seqlen=520, nheads=16,
                                                      h0_std=0.2, seed=77)
    inp = synth.forward_inputs(w)
    ref = None
    for chunk in (32, 64, 128, 256):
        y, hf = gpu_forward(inp, w, chunk=chunk)
        got = to_f64(y)
        if ref is None:
            ref = got
        else:
            assert rel_err(got, ref) <= 2 * tolerance(w.dtype)


# ---------------------------------------------------------------------------
# forward at full size: sampled lanes, the benchmark's launch configuration
# ---------------------------------------------------------------------------

def _cut_lanes(w, sms):
    """The (b, h) lanes the tensor-core forward cuts in two at this size: with
    one segment per lane, the lanes past the last full wave of CTAs when they
    are at most half a wave (they come last in (batch, head) order)."""
    lanes = w.batch * w.nheads
    nb = -(-w.seqlen // 128)
    if lanes < 2 * sms and nb >= 4:
        return []  # few lanes: every lane is cut into segments instead
    cut = lanes % sms
    if lanes < sms or nb < 2 or cut == 0 or 2 * cut > sms:
        return []
    return [divmod(bh, w.nheads) for bh in range(lanes - cut, lanes)]


@pytest.mark.parametrize("name", ["mamba2_2p7b_layer", "long_seq_65k", "hybrid_8b_layer_N64",
                                  "hybrid_8b_layer_N128", "hybrid_8b_layer_N256"])
def test_forward_full_size_sampled_lanes(name):
    # 40 lanes per workload (all 32 on the long sequence): every (batch,
    # group) pair, and on the layers whose lane count leaves a partial wave,
    # eight lanes that the kernel cuts in two (the second half starts from the
    # state its first half hands over)
    w = synth.WORKLOADS[name]
    inp = synth.forward_inputs(w)
    y, hf = gpu_forward(inp, w)
    torch.cuda.synchronize()
    ex = synth.exact_inputs(inp, w.dtype)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    cut = _cut_lanes(w, sms)
    must = [(0, 0), (w.batch - 1, w.nheads - 1)]
    if cut:
        must += [cut[i * (len(cut) - 1) // 7] for i in range(8)]
    lanes = spread_lanes(w.batch, w.nheads, w.ngroups, 40, w.seed, must)
    assert len(lanes) == min(40, w.batch * w.nheads)
    assert {(b, h // (w.nheads // w.ngroups)) for b, h in lanes} == {
        (b, g) for b in range(w.batch) for g in range(w.ngroups)}
    ref = oracle_lanes(ex, lanes, w.nheads, w.ngroups)
    tol = tolerance(w.dtype)
    worst = 0.0
    for (b, h), (yr, hr) in zip(lanes, ref):
        ey = rel_err(to_f64(y[b, :, h, :]), yr)
        eh = rel_err(to_f64(hf[b, h]), hr)
        worst = max(worst, ey, eh)
        assert ey <= tol and eh <= tol, (b, h, ey, eh)
    # every output is finite
    assert torch.isfinite(y).all().item() and torch.isfinite(hf).all().item()


# ---------------------------------------------------------------------------
# decode step
# ---------------------------------------------------------------------------

def _decode_run(w, steps, lanes=None):
    """Run `steps` decode steps on the GPU and check y and h after each step
    against the oracle carried in fp64: on every lane, or on `lanes` only."""
    from selective_state_space_12_b200 import ssd_step

    prm = synth.decode_params(w)
    h_np = synth.decode_state(w)
    h = torch.from_numpy(h_np).cuda()
    A = torch.from_numpy(prm["A"]).cuda()
    D = torch.from_numpy(prm["D"]).cuda()
    Af = prm["A"].astype(np.float64)
    Df = prm["D"].astype(np.float64)
    hpg = w.nheads // w.ngroups
    if lanes is None:
        h_ref = h_np.astype(np.float64)
    else:
        h_ref = [h_np[b, hh].astype(np.float64)[None, None] for b, hh in lanes]
    tol = tolerance(w.dtype)
    for s in range(steps):
        si = synth.decode_step_inputs(w, s)
        ex = synth.exact_inputs(si, w.dtype)
        dev = {k: to_device(v, w.dtype) for k, v in si.items()}
        y = ssd_step(h, dev["x"], dev["dt"], A, dev["B"], dev["C"], D)
        torch.cuda.synchronize()
        if lanes is None:
            yr, h_ref = oracle.ssd_step(h_ref, ex["x"], ex["dt"], Af, ex["B"], ex["C"], Df)
            ey, eh = rel_err(to_f64(y), yr), rel_err(h.cpu().numpy(), h_ref)
            assert ey <= tol and eh <= tol, (s, ey, eh)
            continue
        for k, (b, hh) in enumerate(lanes):
            g = hh // hpg
            yk, h_ref[k] = oracle.ssd_step(
                h_ref[k], ex["x"][b, hh][None, None], ex["dt"][b, hh][None, None],
                Af[hh:hh + 1], ex["B"][b, g][None, None], ex["C"][b, g][None, None],
                Df[hh:hh + 1])
            ey = rel_err(to_f64(y[b, hh]), yk[0, 0])
            eh = rel_err(h[b, hh].cpu().numpy(), h_ref[k][0, 0])
            assert ey <= tol and eh <= tol, (s, b, hh, ey, eh)


@pytest.mark.parametrize("dtype", [synth.F32, synth.BF16])
def test_decode_small_every_step(dtype):
    w = synth.DECODE_WORKLOADS["decode_b256"].with_(batch=3, nheads=16, dtype=dtype, seed=21)
    _decode_run(w, steps=8)


@pytest.mark.parametrize("P,N,G", [(16, 16, 1), (32, 256, 2), (128, 64, 4), (64, 48, 8)])
def test_decode_shapes(P, N, G):
    w = synth.DECODE_WORKLOADS["decode_b256"].with_(batch=2, nheads=8, headdim=P, dstate=N,
                                                    ngroups=G, seed=P * N + G)
    _decode_run(w, steps=3)


def test_decode_full_size_sampled_lanes():
    # the decode workload as the benchmark runs it (b256 H128 P64 N128 G8,
    # 1 GiB fp32 state carried over 64 successive steps), checked after every
    # step on 16 lanes: two per group, in different batches, the corners
    # included
    w = synth.DECODE_WORKLOADS["decode_b256"]
    lanes = spread_lanes(w.batch, w.nheads, w.ngroups, 16, w.seed,
                         must=[(0, 0), (w.batch - 1, w.nheads - 1)])
    hpg = w.nheads // w.ngroups
    assert {h // hpg for _, h in lanes} == set(range(w.ngroups))
    _decode_run(w, steps=64, lanes=lanes)
