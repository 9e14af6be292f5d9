"""A long sequence split by blocks across ranks (one process per GPU): each
rank holds a contiguous range of every sequence's tokens in its own pool and
decodes that range (pa_decode_lse); the ranks' partial outputs and log
normalisers are gathered over torch.distributed (NCCL between GPUs) and
merged by the online-softmax rule (pa_merge_partials; study notes ch.05 §4,
the merge of partial results rescaled to a common maximum).  The exchange is
one all-gather of S x Hq x (D 16-bit values + 1 float) per rank.

Argument marshalling and one collective only: the decode and the merge run in
libpa's kernels.
"""

from __future__ import annotations

from . import _lib


def gather_partials(out, lse, group=None):
    """All-gather every rank's partial output [S, Hq, D] and log normaliser
    [S, Hq] into [world, S, Hq, D] and [world, S, Hq] (rank order), on the
    tensors' own device."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    # gathered along the first dimension (world * S rows), then viewed per rank
    outs = torch.empty((world * out.shape[0],) + tuple(out.shape[1:]), dtype=out.dtype, device=out.device)
    lses = torch.empty((world * lse.shape[0],) + tuple(lse.shape[1:]), dtype=lse.dtype, device=lse.device)
    dist.all_gather_into_tensor(outs, out.contiguous(), group=group)
    dist.all_gather_into_tensor(lses, lse.contiguous(), group=group)
    return outs.view((world,) + tuple(out.shape)), lses.view((world,) + tuple(lse.shape))


def decode_split(q, k_pool, v_pool, block_tables, seq_lens, scale: float, out, workspace, dev_status=None,
                 lse_out=None, group=None):
    """Decode this rank's token range of each sequence (its own pool, tables
    and lengths), exchange the partial results with the other ranks and
    merge them into out (the same on every rank).  q is the full query on
    every rank.  Everything runs on the current stream, the collective
    included."""
    import torch

    S, Hq, _ = q.shape
    part = torch.empty_like(q)
    lse = torch.empty((S, Hq), dtype=torch.float32, device=q.device)
    _lib.pa_decode_lse(q, k_pool, v_pool, block_tables, seq_lens, scale, part, lse, workspace, dev_status)
    outs, lses = gather_partials(part, lse, group)
    _lib.pa_merge_partials(outs, lses, out, lse_out)
