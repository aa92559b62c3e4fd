"""Sequence (L) sharding of the selective scan over ranks, one GPU per rank.

Every (batch, channel) lane is independent, so splitting batches or channels across GPUs
needs no communication.  A sequence too long for one GPU is split along L instead: rank r
holds the consecutive steps [r * Ls, (r + 1) * Ls) of every lane.  The recurrence couples
the shards only through the state handed from one to the next, and the parallel-scan
derivation of the "Mamba" page (yongjin360.com/news/29389, steps 1-4) gives the exchange:
a shard is one transformation T_r = (prod Abar, h_end) of the associative combine, so

  1. each rank summarises its shard from h = 0 (``ops.selective_scan_summary``: h_end and
     the summed step, prod Abar_n = exp(A_n * sum Delta));
  2. the ranks all-gather the summaries (b * d * (N + 1) floats each -- the one data-path
     collective, 1.4 MB for the 2.8B-shaped layer);
  3. rank r folds the summaries of ranks 0..r-1 into its start state
     (``ops.selective_scan_fold``) and scans its shard from there
     (``ops.selective_scan_fwd(initial_state=...)``).

All arithmetic runs in the library's kernels; this module only moves tensors and calls
the collective.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import ops


def shard_summary(u, delta, A, B, C, delta_bias=None, delta_softplus=True, exact_zoh=False):
    """Step 1 for this rank's shard: (h_end (b, d, N), delta_sum (b, d))."""
    return ops.selective_scan_summary(u, delta, A, B, C, delta_bias=delta_bias,
                                      delta_softplus=delta_softplus, exact_zoh=exact_zoh)


def gather_summaries(h_end, delta_sum, group=None):
    """Step 2: every rank's summary, in rank order: (h_ends (world, b, d, N),
    delta_sums (world, b, d)).  One all-gather of a packed (b * d, N + 1) buffer."""
    world = dist.get_world_size(group)
    b, d, N = h_end.shape
    packed = torch.cat([h_end.reshape(b * d, N), delta_sum.reshape(b * d, 1)], dim=1).reshape(-1)
    out = torch.empty(world * packed.numel(), dtype=packed.dtype, device=packed.device)
    dist.all_gather_into_tensor(out, packed.contiguous(), group=group)
    out = out.reshape(world, b * d, N + 1)
    return (out[..., :N].reshape(world, b, d, N).contiguous(),
            out[..., N].reshape(world, b, d).contiguous())


def shard_scan(rank, h_ends, delta_sums, u, delta, A, B, C, D=None, z=None, delta_bias=None,
               delta_softplus=True, out_dtype=None, exact_zoh=False):
    """Step 3 for shard `rank`: y of the shard and the state after it."""
    h0 = ops.selective_scan_fold(h_ends[:rank], delta_sums[:rank], A) if rank > 0 else None
    return ops.selective_scan_fwd(u, delta, A, B, C, D=D, z=z, delta_bias=delta_bias,
                                  delta_softplus=delta_softplus, out_dtype=out_dtype,
                                  return_last_state=True, exact_zoh=exact_zoh, initial_state=h0)


def sharded_selective_scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None,
                               delta_softplus=True, out_dtype=None, exact_zoh=False, group=None):
    """The selective scan of a sequence split along L over the ranks of `group` (NCCL):
    this rank passes its shard (batch, dim, Ls) and gets back y for the shard and the state
    after it (on the last rank, the sequence's last state)."""
    rank = dist.get_rank(group)
    h_end, dsum = shard_summary(u, delta, A, B, C, delta_bias, delta_softplus, exact_zoh)
    h_ends, dsums = gather_summaries(h_end, dsum, group)
    return shard_scan(rank, h_ends, dsums, u, delta, A, B, C, D=D, z=z, delta_bias=delta_bias,
                      delta_softplus=delta_softplus, out_dtype=out_dtype, exact_zoh=exact_zoh)
