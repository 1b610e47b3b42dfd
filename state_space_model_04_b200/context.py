"""Context-parallel prefill: the tokens of every sequence split over the ranks of a process
group, one exchange step ("Compiler-First State Space Duality and Portable O(1)
Autoregressive Caching", "Chunked recurrence": the state entering a stretch of tokens is
the decayed sum of the states the earlier stretches leave behind, and y is linear in it).

Rank r holds consecutive tokens of every sequence, ranks in group order.  Each rank
  1. computes the state its tokens leave when started from zero and their log decay
     (ssd_prefill_local_state, tensor-core state pass),
  2. all-gathers both (one collective each: 2.6 MB of fp32 state per sequence at the
     2.7B shape, over NCCL on GPUs),
  3. folds the earlier ranks' states into its entering state (ssd_prefill_context_scan),
  4. runs the prefill from that state (ssd_prefill): its y, and the state after its tokens,
     which on the last rank is the whole sequence's final state.
"""
from __future__ import annotations

import torch

from . import ssd as _ssd


class _Kernels:
    """The library's kernels (the only product implementation of the steps)."""

    @staticmethod
    def local_state(x, dt, A, B):
        return _ssd.prefill_local_state(x, dt, A, B)

    @staticmethod
    def context_scan(rank, h_all, ld_all, h0):
        return _ssd.prefill_context_scan(rank, h_all, ld_all, h0=h0)

    @staticmethod
    def prefill(x, dt, A, B, C, D, chunk, h0):
        return _ssd.prefill(x, dt, A, B, C, D, chunk=chunk, h0=h0)


def _gather(t, world, group):
    """Rank-major stack of every rank's `t` (one all_gather)."""
    import torch.distributed as dist
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.stack(parts)


def prefill_context_parallel(x, dt, A, B, C, D, h0=None, group=None, chunk=256, ops=None):
    """This rank's share of a prefill whose sequences are split over the ranks of `group`
    (consecutive tokens per rank, ranks in group order).  x [b,T_r,H,P], dt [b,T_r,H],
    B/C [b,T_r,G,N] are this rank's tokens; A, D and h0 (the state before the first rank's
    tokens, or None) are the same on every rank.  Returns (y for this rank's tokens, the
    state after them).  Without an initialised process group it is one plain prefill."""
    import torch.distributed as dist
    ops = ops or _Kernels
    dist_on = dist.is_available() and dist.is_initialized()
    world = dist.get_world_size(group) if dist_on else 1
    rank = dist.get_rank(group) if dist_on else 0
    if world == 1:
        return ops.prefill(x, dt, A, B, C, D, chunk, h0)
    h_loc, ld = ops.local_state(x, dt, A, B)
    h_all = _gather(h_loc, world, group)
    ld_all = _gather(ld, world, group)
    h_in = ops.context_scan(rank, h_all, ld_all, h0)
    return ops.prefill(x, dt, A, B, C, D, chunk, h_in)
