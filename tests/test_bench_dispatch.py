"""Host logic of bench.py's one-process run on CPU: which legs run for each
--only value and which JSON line comes back, with the GPU legs, the clock
sampler and the device calls replaced by fakes."""
import argparse
import types

import pytest

import bench
import synth


@pytest.fixture
def fake_gpu(monkeypatch):
    torch = pytest.importorskip("torch")
    calls = []

    def leg(name, value):
        def run(*a, **k):
            calls.append(name)
            if name == "forward":
                return {"value": value, "ms": 1.0, "w": synth.WORKLOADS["mamba2_2p7b_layer"],
                        "seed": 1, "roofline": {}, "tensor": {}, "hbm_whole_forward": {},
                        "kernels": {}, "gpu_launches": 1, "e2e": {}, "step_options": {}}
            return {"value": value, "ms_per_step": 1.0}
        return run

    for name, value in (("forward", 1.0), ("decode", 2.0), ("backward", 3.0), ("scan", 4.0)):
        monkeypatch.setattr(bench, f"bench_{name}", leg(name, value))
    monkeypatch.setattr(bench, "bench_sp", leg("sp", 5.0))

    def config_leg(name, *a, **k):
        calls.append("config:" + name)
        return {"workload": name, "value": 6.0, "ms_per_step": 1.0}

    monkeypatch.setattr(bench, "bench_forward_config", config_leg)

    class Sampler:
        def __init__(self, *a):
            pass

        def start(self):
            pass

        def stop(self):
            return []

        @staticmethod
        def summarise(rows, mx):
            return {}

    monkeypatch.setattr(bench, "ClockSampler", Sampler)
    monkeypatch.setattr(bench.time, "sleep", lambda s: None)
    monkeypatch.setattr(torch.cuda, "set_device", lambda d: None)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda d=None: None)
    monkeypatch.setattr(torch.cuda, "empty_cache", lambda: None)
    monkeypatch.setattr(torch.cuda, "get_device_properties",
                        lambda d: types.SimpleNamespace(uuid="GPU-0", multi_processor_count=148))
    from selective_state_space_12_b200 import build as ssd_build

    monkeypatch.setattr(ssd_build, "build", lambda *a, **k: None)
    return calls


def _args(only, **kw):
    base = dict(only=only, no_backward=False, no_scan=False, no_sp=False, no_configs=False,
                no_cpu_baseline=True, steps=2, warmup=3)
    base.update(kw)
    return argparse.Namespace(**base)


CONFIGS = ["config:" + n for n in bench.FORWARD_CONFIGS]


@pytest.mark.parametrize("only,legs,key,value", [
    ("all", ["forward"] + CONFIGS + ["decode", "backward", "scan", "sp"], "selective_scan", 1.0),
    ("forward", ["forward"], "roofline", 1.0),
    ("decode", ["decode"], "decode", 2.0),
    ("backward", ["backward"], "backward", 3.0),
    ("scan", ["scan"], "selective_scan", 4.0),
    ("sp", ["sp"], "sequence_parallel", 5.0),
])
def test_only_runs_its_legs(fake_gpu, only, legs, key, value):
    out = bench.run_ours(_args(only), bench.Dist("gloo"))
    assert fake_gpu == legs
    assert out["value"] == value and key in out


def test_skip_flags_drop_legs_from_the_full_run(fake_gpu):
    out = bench.run_ours(_args("all", no_backward=True, no_scan=True, no_sp=True,
                               no_configs=True), bench.Dist("gloo"))
    assert fake_gpu == ["forward", "decode"]
    assert out["backward"] is None and out["selective_scan"] is None
    assert out["forward_configs"] is None


def test_the_full_run_reports_every_forward_workload(fake_gpu):
    out = bench.run_ours(_args("all"), bench.Dist("gloo"))
    assert sorted(out["forward_configs"]) == sorted(bench.FORWARD_CONFIGS)
    assert set(bench.FORWARD_CONFIGS) == {"mamba2_2p7b_layer", "long_seq_65k",
                                          "hybrid_8b_layer_N64", "hybrid_8b_layer_N128",
                                          "hybrid_8b_layer_N256"}


def test_a_part_skipped_by_its_own_flag_is_an_error(fake_gpu):
    with pytest.raises(SystemExit):
        bench.run_ours(_args("backward", no_backward=True), bench.Dist("gloo"))
