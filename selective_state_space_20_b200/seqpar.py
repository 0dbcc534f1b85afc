"""One sequence scanned across several GPUs (one process per GPU).

Rank r of a process group holds timesteps [r * L_r, (r + 1) * L_r) of every
(batch, channel) row -- its shard of u, delta, z, B, C.  The recurrence maps
a shard's initial state h to exp(A * S) (.) h + h_local (S the shard's sum of
delta per row, h_local its final state from a zero start), so:

1. each rank runs its shard from zero for the final state alone (the
   state-only scan: no readout or outputs) and sums its delta
   (:func:`shard_summary`);
2. the ranks all-gather those summaries (one small collective:
   batch * dim * (dstate + 2) words per rank);
3. each rank folds the summaries of the ranks before it into its true
   initial state (:func:`shard_initial_state`);
4. each rank scans its shard again from that state (:func:`shard_outputs`).

The exchange happens once per call, between the state-only pass and the
full scan of the shard; there is nothing to overlap it with, and its size is
independent of L.
Every step runs in the library's kernels; torch.distributed carries the
exchange.
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple

import torch

from . import binding


def shard_summary(u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True,
                  workspace=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """(delta sum (batch, dim) fp64, final state from zero (batch, dim, N)
    fp32) of this rank's shard.  The state comes from the state-only scan;
    where its kernel cannot run (dstate > 16, rows not whole 16-byte
    vectors) from a full scan whose outputs are dropped."""
    try:
        h_local = binding.mamba_scan_state(u, delta, A, B, delta_bias=delta_bias, delta_softplus=delta_softplus,
                                           workspace=workspace)
    except binding.MambaError as e:
        if e.code != binding.MAMBA_ERR_UNSUPPORTED:
            raise
        out = torch.empty_like(u)
        _, h_local = binding.mamba_scan_fwd(u, delta, A, B, C, D=D, z=z, delta_bias=delta_bias,
                                            delta_softplus=delta_softplus, out=out,
                                            return_last_state=True, workspace=workspace)
    sums = binding.mamba_delta_sum(delta, delta_bias, delta_softplus)
    return sums, h_local


def shard_initial_state(A, all_sums: torch.Tensor, all_h_local: torch.Tensor, rank: int,
                        h0: Optional[torch.Tensor] = None) -> Optional[torch.Tensor]:
    """The state entering shard ``rank``: the shards 0 .. rank-1 folded,
    starting from ``h0`` (the state before the whole sequence; None = zeros).
    all_sums (world, batch, dim), all_h_local (world, batch, dim, N)."""
    if rank == 0:
        return h0
    return binding.mamba_state_fold(A, all_sums[:rank].contiguous(), all_h_local[:rank].contiguous(),
                                    h_init=h0)


def shard_outputs(u, delta, A, B, C, h_in, D=None, z=None, delta_bias=None, delta_softplus=True,
                  out=None, workspace=None):
    """This rank's outputs and final state, scanned from ``h_in``."""
    return binding.mamba_scan_fwd(u, delta, A, B, C, D=D, z=z, delta_bias=delta_bias,
                                  delta_softplus=delta_softplus, out=out, return_last_state=True,
                                  workspace=workspace, h0=h_in)


def all_gather_summaries(sums: torch.Tensor, h_local: torch.Tensor, group=None):
    """Stack every rank's (sums, h_local) in rank order (torch.distributed,
    any backend)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    parts_s = [torch.empty_like(sums) for _ in range(world)]
    parts_h = [torch.empty_like(h_local) for _ in range(world)]
    dist.all_gather(parts_s, sums.contiguous(), group=group)
    dist.all_gather(parts_h, h_local.contiguous(), group=group)
    return torch.stack(parts_s), torch.stack(parts_h)


def scan_sequence_parallel(u, delta, A, B, C, D=None, z=None, delta_bias=None,
                           delta_softplus=True, h0=None, group=None, out=None, workspace=None,
                           _ops: Optional[dict] = None):
    """Selective scan of a sequence split over the ranks of ``group``: this
    rank passes its shard (u, delta, z (batch, dim, L_r); B, C (batch, N,
    L_r)) and gets its shard of the outputs and the state at the end of its
    shard (on the last rank, the sequence's final state).  ``h0`` is the
    state before the whole sequence (the same on every rank; None = zeros).

    ``_ops`` replaces the per-shard steps (keys ``summary``, ``initial``,
    ``outputs``) -- the multi-process tests run the exchange logic with CPU
    stand-ins for the kernels."""
    import torch.distributed as dist
    ops = {"summary": shard_summary, "initial": shard_initial_state, "outputs": shard_outputs}
    if _ops:
        ops.update(_ops)
    rank = dist.get_rank(group)
    sums, h_local = ops["summary"](u, delta, A, B, C, D=D, z=z, delta_bias=delta_bias,
                                   delta_softplus=delta_softplus)
    all_sums, all_h = all_gather_summaries(sums, h_local, group)
    h_in = ops["initial"](A, all_sums, all_h, rank, h0)
    return ops["outputs"](u, delta, A, B, C, h_in, D=D, z=z, delta_bias=delta_bias,
                          delta_softplus=delta_softplus, out=out)
