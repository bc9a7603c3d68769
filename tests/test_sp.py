"""Sequence parallelism, host logic on two gloo ranks (CPU).

sp_forward's exchange (all-gather of each piece's end state and total decay,
in rank order) and the piece index it chains to are checked with the local
steps done by the fp64 oracle; the library's own local steps and chain
kernel are checked on the GPU (tests/test_gpu_sp.py). The whole must equal
the forward over the unsplit sequence ("两条路各走一半": only the block-end
state passes between consecutive blocks)."""
import math
import os
import socket
import sys

import numpy as np
import torch

import oracle
from tests.conftest import ROOT


class _OracleOps:
    """The three local steps of sp_forward by the fp64 oracle (test stand-in)."""

    @staticmethod
    def _opts(step_opts):
        if not step_opts:
            return oracle.DtOptions()
        lo, hi = step_opts.get("dt_limit") or (0.0, 0.0)
        bias = step_opts.get("dt_bias")
        return oracle.DtOptions(bias=None if bias is None else bias.numpy(),
                                softplus=step_opts.get("dt_softplus", False), dt_min=lo,
                                dt_max=hi, zoh=step_opts.get("zoh", False))

    def state(self, x, dt, A, B, chunk, step_opts):
        o = self._opts(step_opts)
        _, hf = oracle.ssd_forward_ex(x.numpy(), dt.numpy(), A.numpy(), B.numpy(), B.numpy(),
                                      None, None, o)
        _, ell, _ = oracle.dt_prepare(dt.numpy(), A.numpy(), o)
        return torch.from_numpy(hf), torch.from_numpy(np.exp(ell.sum(axis=1)))

    def chain(self, states, decays, part, h0, want_total):
        h = np.zeros(states.shape[1:]) if h0 is None else h0.numpy().copy()
        h_in = None
        for r in range(states.shape[0]):
            if r == part:
                h_in = h.copy()
            h = decays[r].numpy()[..., None, None] * h + states[r].numpy()
        return torch.from_numpy(h_in), (torch.from_numpy(h) if want_total else None)

    def forward(self, x, dt, A, B, C, D, h_in, chunk, step_opts):
        y, _ = oracle.ssd_forward_ex(x.numpy(), dt.numpy(), A.numpy(), B.numpy(), C.numpy(),
                                     None if D is None else D.numpy(), h_in.numpy(),
                                     self._opts(step_opts))
        return torch.from_numpy(y)


def _problem(seed=3, batch=2, L=150, H=4, P=8, N=16, G=2):
    rng = np.random.default_rng(seed)
    return dict(x=rng.standard_normal((batch, L, H, P)),
                dt=rng.normal(-3.0, 1.0, (batch, L, H)),
                A=-np.exp(rng.uniform(0, math.log(16.0), H)),
                B=rng.standard_normal((batch, L, G, N)) / math.sqrt(N),
                C=rng.standard_normal((batch, L, G, N)) / math.sqrt(N),
                D=rng.normal(1.0, 0.1, H), h0=rng.normal(0.0, 0.3, (batch, H, P, N)),
                bias=rng.normal(0.0, 0.5, H))


def _worker(rank, world, port, out_dir, cuts):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from selective_state_space_12_b200.sp import sp_forward

    dist.init_process_group("gloo", rank=rank, world_size=world)
    pr = _problem()
    t0, t1 = cuts[rank], cuts[rank + 1]
    T = {k: torch.from_numpy(v) for k, v in pr.items()}
    y, hf = sp_forward(T["x"][:, t0:t1], T["dt"][:, t0:t1], T["A"], T["B"][:, t0:t1],
                       T["C"][:, t0:t1], T["D"], T["h0"], chunk=64, dt_bias=T["bias"],
                       dt_softplus=True, zoh=True, ops=_OracleOps())
    np.save(os.path.join(out_dir, f"y{rank}.npy"), y.numpy())
    np.save(os.path.join(out_dir, f"h{rank}.npy"), hf.numpy())
    dist.barrier()
    dist.destroy_process_group()


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_sp_forward_on_two_gloo_ranks_equals_unsplit_forward(tmp_path):
    import torch.multiprocessing as mp

    cuts = [0, 61, 150]  # unequal, ragged pieces
    mp.start_processes(_worker, args=(2, _free_port(), str(tmp_path), cuts), nprocs=2,
                       start_method="spawn")
    pr = _problem()
    y_ref, h_ref = oracle.ssd_forward_ex(pr["x"], pr["dt"], pr["A"], pr["B"], pr["C"], pr["D"],
                                         pr["h0"], oracle.DtOptions(bias=pr["bias"],
                                                                    softplus=True, zoh=True))
    y = np.concatenate([np.load(tmp_path / f"y{r}.npy") for r in range(2)], axis=1)
    scale = max(1.0, float(np.abs(y_ref).max()))
    assert np.abs(y - y_ref).max() <= 1e-12 * scale
    for r in range(2):  # every rank holds the whole sequence's final state
        assert np.abs(np.load(tmp_path / f"h{r}.npy") - h_ref).max() <= 1e-12 * scale
