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


def test_raw_steps_reproduce_the_plain_steps():
    # the raw draws z with the per-head bias b give the plain step softplus(z + b)
    # up to the storage rounding of z and b
    w = synth.WORKLOADS["tiny_f32"].with_(seqlen=300, nheads=5)
    plain, raw = synth.forward_inputs(w), synth.forward_inputs_raw(w)
    for k in ("x", "A", "B", "C", "D"):
        assert np.array_equal(plain[k], raw[k])
    dt = np.logaddexp(0.0, raw["dt"].astype(np.float64) + raw["dt_bias"][None, None, :])
    assert np.abs(dt - plain["dt"]).max() <= 1e-6 * np.abs(plain["dt"]).max()
    only = synth.raw_steps(w)
    assert np.array_equal(only["dt"], raw["dt"]) and np.array_equal(only["dt_bias"],
                                                                    raw["dt_bias"])


def test_scan_workload_distributions():
    w = synth.SCAN_WORKLOADS["scan_tiny_f32"].with_(seqlen=512, channels=256, h0_std=0.5)
    s = synth.scan_inputs(w)
    assert s["x"].shape == (1, 512, 256) and s["A"].shape == (256, 16)
    assert s["B"].shape == (1, 512, 1, 16) and s["h0"].shape == (1, 256, 16)
    assert np.all(s["A"] <= -1.0) and np.all(s["A"] >= -16.0)
    sp_b = np.logaddexp(0.0, s["dt_bias"].astype(np.float64))
    assert np.all(sp_b >= 1e-3 * (1 - 1e-6)) and np.all(sp_b <= 1e-1 * (1 + 1e-6))
    assert abs(float(np.std(s["dt"])) - 0.5) < 0.02
    assert abs(float(np.std(s["B"])) - 0.25) < 0.02  # N(0, 1) / sqrt(16)
    assert abs(float(np.mean(s["Dskip"])) - 1.0) < 0.03


def test_decode_raw_steps_match_decode_steps():
    w = synth.DECODE_WORKLOADS["decode_b256"].with_(batch=4, nheads=8, dtype=synth.F32)
    bias = synth.decode_params(w)["dt_bias"]
    for step in range(3):
        plain, raw = synth.decode_step_inputs(w, step), synth.decode_step_inputs_raw(w, step)
        for k in ("x", "B", "C"):
            assert np.array_equal(plain[k], raw[k])
        dt = np.logaddexp(0.0, raw["dt"].astype(np.float64) + bias[None, :])
        assert np.abs(dt - plain["dt"]).max() <= 1e-6 * np.abs(plain["dt"]).max()
