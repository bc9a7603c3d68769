"""Sequence parallelism: one long sequence split into consecutive pieces, one
piece per rank of a torch.distributed group.

Between consecutive blocks of the chunked algorithm only the block-end state
passes ("Mamba-2 — 注意力的远亲", section "两条路各走一半"; "Mamba-2 模型解读",
section 6.2, the block function takes an initial state and returns the final
one); pieces held by different GPUs are blocks of the same kind. Each rank:

  1. computes its piece's end state S_r (from a zero initial state) and total
     decay Lambda_r = exp(sum_t dt_t A_h)         -- ssd_forward_state
  2. all-gathers (S_r, Lambda_r) over the group   -- the one exchange
  3. chains the pieces before it: h_in = h0, then h <- Lambda_q h + S_q for
     q < r, and all of them for the final state   -- ssd_state_chain
  4. runs the forward on its piece from h_in      -- ssd_forward(_ex)

All compute is in libssd; this module only orders the calls and the
collective (NCCL on GPUs). The exchange is b*H*(P*N + 1) fp32 per rank.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch


class LibOps:
    """The three local steps, by the library (the product path)."""

    def state(self, x, dt, A, B, chunk, step_opts):
        from .ssd import ssd_forward_state

        return ssd_forward_state(x, dt, A, B, chunk=chunk, **step_opts)

    def chain(self, states, decays, part, h0, want_total):
        from .ssd import ssd_state_chain

        return ssd_state_chain(states, decays, part, h0=h0, want_total=want_total)

    def forward(self, x, dt, A, B, C, D, h_in, chunk, step_opts):
        from .ssd import ssd_forward, ssd_forward_ex

        if step_opts:
            y, _ = ssd_forward_ex(x, dt, A, B, C, D, h_in, chunk=chunk, want_final=False,
                                  **step_opts)
        else:
            y, _ = ssd_forward(x, dt, A, B, C, D, h_in, chunk=chunk, want_final=False)
        return y


def sp_forward(x: torch.Tensor, dt: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
               C: torch.Tensor, D: Optional[torch.Tensor] = None,
               h0: Optional[torch.Tensor] = None, chunk: int = 256, group=None,
               dt_bias: Optional[torch.Tensor] = None, dt_softplus: bool = False,
               dt_limit: Optional[Tuple[float, float]] = None, zoh: bool = False,
               want_final: bool = True, ops=None
               ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """The layer forward on this rank's piece of a sequence split over the
    ranks of ``group`` in rank order.

    x (b, L_r, H, P), dt (b, L_r, H), B/C (b, L_r, G, N): this rank's
    consecutive tokens; A, D, h0 (the state before the whole sequence) and
    the step options are the same on every rank. Returns (y for this rank's
    tokens, the whole sequence's final state or None); the final state is
    the same on every rank."""
    import torch.distributed as dist

    ops = ops or LibOps()
    grouped = dist.is_available() and dist.is_initialized()
    world = dist.get_world_size(group) if grouped else 1  # no group: one piece
    rank = dist.get_rank(group) if grouped else 0
    step_opts = {}
    if dt_bias is not None or dt_softplus or dt_limit is not None or zoh:
        step_opts = dict(dt_bias=dt_bias, dt_softplus=dt_softplus, dt_limit=dt_limit, zoh=zoh)
    S, lam = ops.state(x, dt, A, B, chunk, step_opts)
    if world > 1:
        S_parts = [torch.empty_like(S) for _ in range(world)]
        lam_parts = [torch.empty_like(lam) for _ in range(world)]
        dist.all_gather(S_parts, S.contiguous(), group=group)
        dist.all_gather(lam_parts, lam.contiguous(), group=group)
    else:
        S_parts, lam_parts = [S], [lam]
    states = torch.stack(S_parts)
    decays = torch.stack(lam_parts)
    h_in, h_total = ops.chain(states, decays, rank, h0, want_final)
    y = ops.forward(x, dt, A, B, C, D, h_in, chunk, step_opts)
    return y, h_total
