"""The benchmark's algorithmic counts (the numerators of its roofline
fractions), checked on CPU against sums worked out by hand from the layer's
tensors: one read of every input and one write of every output."""
import json

import bench
import synth


def test_forward_compulsory_bytes_of_the_2p7b_layer():
    # b 8, L 2048, H 80, P 64, N 128, G 1, bf16, no h0:
    # x and y 8*2048*80*64*2 each, dt 8*2048*80*2, B and C 8*2048*128*2 each,
    # A and D 80*4 each, h_final 8*80*64*128*4
    w = synth.WORKLOADS["mamba2_2p7b_layer"]
    want = 2 * 167_772_160 + 2_621_440 + 2 * 4_194_304 + 640 + 20_971_520
    assert want == 367_526_528
    assert bench.forward_min_bytes(w) == want


def test_forward_bytes_count_h0_and_fp32():
    w = synth.WORKLOADS["tiny_f32"].with_(batch=2, seqlen=10, nheads=4, headdim=8, dstate=16,
                                          ngroups=2, h0_std=0.5)
    x = 2 * 10 * 4 * 8 * 4
    want = 2 * x + 2 * 10 * 4 * 4 + 2 * (2 * 10 * 2 * 16 * 4) + 2 * 4 * 4 + 2 * (2 * 4 * 8 * 16 * 4)
    assert bench.forward_min_bytes(w) == want


def test_decode_bytes_of_b256():
    # the fp32 state read and written, x and y, dt, B and C per group, A and D
    w = synth.DECODE_WORKLOADS["decode_b256"]
    state = 256 * 128 * 64 * 128 * 4
    io = (2 * 256 * 128 * 64 + 256 * 128 + 2 * 256 * 8 * 128) * 2 + 2 * 128 * 4
    assert bench.decode_bytes(w) == 2 * state + io == 2_156_987_392


def test_scan_alu_peak():
    # 16 exp2 per clock on each of 148 SMs at 1965 MHz
    assert bench.scan_alu_peak(148) == 16 * 148 * 1965e6
    assert abs(bench.scan_alu_peak(148) - 4.653e12) < 1e9


def test_segment_rule():
    # one segment when the lanes fill the GPU twice over or the lane is short;
    # else about two waves of CTAs, at most half the 128-token blocks
    w = synth.WORKLOADS["mamba2_2p7b_layer"]           # 640 lanes
    assert bench.tc_segments(w, sms=148) == 1
    long = synth.WORKLOADS["long_seq_65k"]              # 1 x 32 lanes of 512 blocks
    assert bench.tc_segments(long, sms=148) == 9        # 288 CTAs: about 2 waves of 148
    assert bench.tc_segments(long.with_(seqlen=8 * 128), sms=148) == 4  # half of 8 blocks
    short = long.with_(seqlen=3 * 128)                  # 3 blocks: too short to cut
    assert bench.tc_segments(short, sms=148) == 1


def test_stored_traffic_follows_the_source_digest(tmp_path, monkeypatch):
    import json

    (tmp_path / "profiles").mkdir()
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    digest = bench.source_digest(["k.cu"])
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"k": {"sources": ["k.cu"], "source_digest": digest, "dram_bytes_per_launch": 123}}))
    assert bench.stored_traffic("k") == 123
    assert bench.stored_traffic("k", "any_workload") == 123  # workload-independent entry
    assert bench.stored_traffic("other") is None
    src.write_text("kernel v2")                         # the kernel changed since the capture
    assert bench.stored_traffic("k") is None


def test_backward_counts_of_the_2p7b_layer():
    w = synth.WORKLOADS["mamba2_2p7b_layer"]
    # reads: x and dy 8*2048*80*64 bf16 each, dt 8*2048*80, B and C 8*2048*128
    # (no h0 on this workload); writes in fp32: dx, ddt, dB, dC of the same
    # element counts, and dh0 (8*80*64*128 fp32) when asked for
    reads = (2 * 83_886_080 + 1_310_720 + 2 * 2_097_152) * 2
    writes = (83_886_080 + 1_310_720 + 2 * 2_097_152) * 4
    dh0 = 8 * 80 * 64 * 128 * 4
    assert bench.backward_min_bytes(w, dh0=False) == reads + writes == 704_118_784
    assert bench.backward_min_bytes(w) == reads + writes + dh0 == 725_090_304
    # with an initial state it is read once too
    assert bench.backward_min_bytes(w.with_(h0_std=0.1)) == 725_090_304 + dh0
    # per token and head at Q 128, P 64, N 128, 80 heads per group:
    # 2*128*64 + 2*128*128 + 128*128/80 + 12*128*64
    per = 16_384 + 32_768 + 204.8 + 98_304
    assert abs(bench.backward_flops(w) - 8 * 2048 * 80 * per) < 1.0
    assert abs(bench.backward_flops(w) / 1e9 - 193.54) < 0.01


def test_state_pass_bytes_of_the_long_sequence():
    # 32 lanes cut into 9 segments each on 148 SMs (about two waves): the
    # fp32 segment end states (64 x 128) read and the entering states written
    # in place, one decay per segment read, h0 read and h_final written
    w = synth.WORKLOADS["long_seq_65k"]
    assert bench.tc_segments(w, sms=148) == 9
    seg = 32 * 9 * 64 * 128 * 4
    state = 32 * 64 * 128 * 4
    want = 2 * seg + 32 * 9 * 4 + state + state
    import unittest.mock as um
    with um.patch.object(bench, "tc_segments", lambda w_, sms=None: 9):
        assert bench.kernel_bytes("state_pass", w) == want == 20_972_672


def test_stored_traffic_per_workload(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    (tmp_path / "k.cu").write_text("kernel")
    digest = bench.source_digest(["k.cu"])
    ent = lambda b: {"sources": ["k.cu"], "source_digest": digest, "dram_bytes_per_launch": b}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"k@w1": ent(1), "k@w2": ent(2)}))
    assert bench.stored_traffic("k", "w1") == 1 and bench.stored_traffic("k", "w2") == 2
    assert bench.stored_traffic("k", "w3") is None and bench.stored_traffic("k") is None
