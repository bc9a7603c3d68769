"""The seeded input generator: determinism, storage rounding, distributions."""
import math

import numpy as np

import synth


def test_bf16_rounding_is_nearest_even_and_exact_on_decode():
    # representable values round-trip; halfway cases go to the even neighbour
    vals = np.array([1.0, -2.5, 0.0, 3.140625, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1e-3])
    bits = synth.bf16_bits(vals)
    back = synth.bf16_to_f64(bits)
    assert back[0] == 1.0 and back[1] == -2.5 and back[2] == 0.0 and back[3] == 3.140625
    assert back[4] == 1.0                      # tie -> even (1.0)
    assert back[5] == 1.0 + 4 * 2 ** -8        # tie -> even (1 + 2^-6)
    assert abs(back[6] - 1e-3) <= 2 ** -8 * 1e-3
    rng = np.random.default_rng(0)
    r = rng.standard_normal(10000)
    rb = synth.bf16_to_f64(synth.bf16_bits(r))
    assert np.all(np.abs(rb - r) <= 2 ** -8 * np.abs(r))  # half an ulp of an 8-bit significand


def test_generator_is_deterministic_and_seed_sensitive():
    w = synth.WORKLOADS["tiny_f32"]
    a = synth.forward_inputs(w)
    b = synth.forward_inputs(w)
    c = synth.forward_inputs(w, seed=w.seed + 1)
    for k in ("x", "dt", "B", "C", "A", "D"):
        assert np.array_equal(a[k], b[k])
        assert not np.array_equal(a[k], c[k])
    assert a["h0"] is None


def test_distributions_follow_the_recipe():
    w = synth.WORKLOADS["tiny_f32"].with_(batch=4, seqlen=512, nheads=8, dstate=64)
    inp = synth.forward_inputs(w)
    ex = synth.exact_inputs(inp, w.dtype)
    assert abs(ex["x"].std() - 1.0) < 0.05
    assert np.all(ex["dt"] > 0)
    assert np.all((ex["A"] <= -1.0 + 1e-6) & (ex["A"] >= -16.0 - 1e-5))
    assert abs(ex["B"].std() * math.sqrt(64) - 1.0) < 0.05
    assert abs(ex["D"].mean() - 1.0) < 0.15
    # softplus(b) log-uniform in [1e-3, 1e-1]: median dt sits well inside it
    med = np.median(ex["dt"])
    assert 1e-3 < med < 1e-1


def test_long_sequence_workload_has_initial_state():
    w = synth.WORKLOADS["long_seq_65k"].with_(seqlen=512)
    inp = synth.forward_inputs(w)
    assert inp["h0"].shape == (1, 32, 64, 128)
    assert abs(inp["h0"].std() - 0.1) < 0.01


def test_decode_inputs_shapes():
    w = synth.DECODE_WORKLOADS["decode_b256"].with_(batch=4)
    h = synth.decode_state(w)
    s0 = synth.decode_step_inputs(w, 0)
    s1 = synth.decode_step_inputs(w, 1)
    assert h.shape == (4, 128, 64, 128) and h.dtype == np.float32
    assert s0["x"].shape == (4, 128, 64) and s0["dt"].shape == (4, 128)
    assert s0["B"].shape == (4, 8, 128)
    assert not np.array_equal(s0["x"], s1["x"])
