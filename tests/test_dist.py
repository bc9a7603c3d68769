"""Multi-process host logic of the benchmark on CPU, two ranks over gloo:
rank discovery, the barrier, the max over ranks used for the timed region,
per-rank seeds (each rank draws its own batch: weak scaling over independent
sequences, no data-path collective), and the reference arm under torchrun
(rank 0 alone times the oracle and prints; the other ranks exit 0)."""
import json
import os
import socket
import subprocess
import sys

import numpy as np

from tests.conftest import ROOT


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import synth

    d = bench.Dist("gloo")
    assert (d.world, d.rank) == (world, rank)
    d.barrier()
    # each rank reports its own time; the job's time is the slowest rank's
    slowest = d.max(10.0 + rank, "cpu")
    w = synth.WORKLOADS["tiny_f32"]
    seed = bench.shard_seed(w.seed, rank)
    x = synth.forward_inputs(w, seed=seed)["x"]
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"slowest": slowest, "seed": seed, "x_abs_sum": float(np.abs(x).sum())}, f)
    d.barrier()
    d.close()


def test_bench_rank_helpers_on_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp

    mp.start_processes(_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2,
                       start_method="spawn")
    r = [json.load(open(tmp_path / f"rank{i}.json")) for i in range(2)]
    assert r[0]["slowest"] == r[1]["slowest"] == 11.0
    assert r[0]["seed"] != r[1]["seed"]
    assert r[0]["x_abs_sum"] != r[1]["x_abs_sum"]  # independent batches per rank


def test_reference_arm_under_torchrun_two_ranks():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--gpus", "2", "--workload", "tiny_f32", "--steps", "1",
           "--warmup", "3"]
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, p.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
