"""Sequence sharding of long contexts across GPUs (one process per GPU).

The batch is split along the tokens.  For every sequence, rank p of P holds
a contiguous range of whole key groups, and the last rank also holds the
tail with the bf16 window.  Every rank's part is then an ordinary libkvq
cache (the ranks before the last have no window: residual 0), and its key
groups are exactly those the unsharded cache would form, because every
range starts on a group boundary.

Decode runs on every rank over its own tokens (kvq_decode_attention_lse).
The ranks then all-gather their outputs and ln-sum-exp values (H_q x 129
floats per sequence), and every rank merges them with kvq_merge_partials:
the softmax over the union of the ranges, the same merge the decode applies
to its own splits and to the quantized part and the window.  New tokens are
appended on the last rank, whose window flushes exactly as the unsharded
cache's would.
"""
from __future__ import annotations

from typing import List, Tuple

import torch

from . import kvq


def shard_bounds(n: int, group: int, residual: int, parts: int) -> List[Tuple[int, int]]:
    """Token ranges [lo, hi) of the `parts` ranks for one sequence of n tokens.

    The quantized groups of the unsharded cache (n_q = G * floor(max(n - R,
    0) / G) tokens) are split as evenly as whole groups allow; the last range
    also takes the n - n_q window tokens.  Every lo is a multiple of the
    group, so rank p < parts - 1 holds only whole groups and the last rank's
    own quantized prefix ends where the unsharded cache's does."""
    if parts < 1 or group < 1 or n < 0 or residual < 0:
        raise ValueError("bad shard request")
    groups = max(n - residual, 0) // group
    cuts = [group * (groups * p // parts) for p in range(parts)] + [n]
    return [(cuts[p], cuts[p + 1]) for p in range(parts)]


def shard_residual(rank: int, parts: int, residual: int) -> int:
    """Window size of rank `rank`'s cache: only the last rank keeps one."""
    return residual if rank == parts - 1 else 0


def gather_partials(out: torch.Tensor, lse: torch.Tensor, group=None):
    """All-gather this rank's decode output [rows, 128] and ln-sum-exp [rows]:
    returns ([P, rows, 128], [P, rows]) in rank order."""
    import torch.distributed as dist
    P = dist.get_world_size(group)
    outs = [torch.empty_like(out) for _ in range(P)]
    lses = [torch.empty_like(lse) for _ in range(P)]
    dist.all_gather(outs, out.contiguous(), group=group)
    dist.all_gather(lses, lse.contiguous(), group=group)
    return torch.stack(outs), torch.stack(lses)


def decode_sharded(cache: "kvq.Cache", q: torch.Tensor, out: torch.Tensor, softmax_scale: float,
                   workspace: torch.Tensor, num_splits: int, max_len: int, group=None, stream=None):
    """Decode attention over the whole sharded sequences.

    cache: this rank's shard (bounds from shard_bounds); q: bf16 [B, H_q,
    128], the same on every rank; out: float [B, H_q, 128], written on every
    rank; max_len: an upper bound of this rank's shard lengths.  Every rank
    of `group` must call it (one all-gather of the partials).

    stream: a torch.cuda.Stream (None = the current stream).  The decode, the
    buffers, the all-gather (NCCL enqueues on torch's current stream) and the
    merge all run on it, in that order, so nothing reads a buffer before the
    step that writes it; the caller orders other streams against it."""
    import contextlib
    on_gpu = out.device.type == "cuda"
    if stream is None and on_gpu:
        stream = torch.cuda.current_stream(out.device)
    with torch.cuda.stream(stream) if on_gpu else contextlib.nullcontext():
        B, Hq = cache.shape.batch, cache.shape.num_q_heads
        rows = B * Hq
        part = torch.empty(rows, 128, dtype=torch.float32, device=out.device)
        lse = torch.empty(rows, dtype=torch.float32, device=out.device)
        cache.decode_attention_lse(q, part, lse, softmax_scale, workspace, num_splits, max_len, stream)
        outs, lses = gather_partials(part, lse, group)
        kvq.kvq_merge_partials(outs, lses, outs.shape[0], rows, out, None, stream)
