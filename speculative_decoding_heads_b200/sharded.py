"""Heads with the vocabulary split over the ranks of a process group.

"Medusa — 让大模型自己同时猜好几个 token", 核心要点: every head projects u to
the whole vocabulary and keeps its k most probable tokens.  The projection
Wout [K, V, d] dominates the heads' bytes, so G ranks each hold V/G rows of
every Wout[k]; each rank runs the heads kernel on its rows (the residual
block W1 stays whole on every rank: its bytes are K·d² against K·V·d), the
ranks all-gather their top-k lists (G·B·K·k values and ids, a few KB), and
the merge kernel selects the global top-k from the G·k candidates of each
(sequence, head).  The heads kernel computes each logit the same way for any
V, so the merged lists are those of the unsplit call bit for bit.

Tree attention can split the same way along each slice's cached prefix:
rank r attends to its window of prefix rows (the last rank also to the tree
rows), the ranks all-gather their lse values only, each rank scales its own
output by its log-sum-exp weight, and an all-reduce (sum) of the scaled
outputs gives the unsplit result (tree_attention_sharded).  That moves one
output per rank instead of gathering G of them.

Every step runs in the library's kernels; torch.distributed only moves the
gathered lists, the lse values and the sum (NCCL between GPUs, gloo on the
host for the tests).

When the caller passes `stream`, everything -- the temporaries, the kernels
and the collectives -- runs with `stream` as torch's current stream, so the
caching allocator never hands a temporary to another stream while a kernel
on `stream` may still read it.
"""

import contextlib
from typing import List, Optional, Tuple

import torch
import torch.distributed as dist

from . import (MAX_SHARDS, medusa_attention_rescale, medusa_heads_topk, medusa_heads_workspace_size,
               medusa_topk_merge, medusa_tree_attention, medusa_tree_attention_split, workspace)


def _on(stream):
    """Makes `stream` torch's current stream (no-op when None)."""
    return torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()


def shard_bounds(V: int, G: int) -> List[Tuple[int, int]]:
    """(first row, rows) of each of G shards of a V-row vocabulary: contiguous, in rank order,
    the first V % G shards one row longer."""
    if not (1 <= G <= MAX_SHARDS) or V < G:
        raise ValueError(f"cannot split {V} rows over {G} shards")
    base, extra = divmod(V, G)
    out, r0 = [], 0
    for g in range(G):
        n = base + (1 if g < extra else 0)
        out.append((r0, n))
        r0 += n
    return out


def gather_shard_lists(vals: torch.Tensor, ids: torch.Tensor, group=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """All-gather this rank's top-k lists [B, K, k] into [G, B, K, k] (rank order), written
    straight into the stacked buffers (one collective per tensor, no extra copy)."""
    G = dist.get_world_size(group)
    all_vals = torch.empty((G,) + tuple(vals.shape), dtype=vals.dtype, device=vals.device)
    all_ids = torch.empty((G,) + tuple(ids.shape), dtype=ids.dtype, device=ids.device)
    dist.all_gather(list(all_vals.unbind(0)), vals.contiguous(), group=group)
    dist.all_gather(list(all_ids.unbind(0)), ids.contiguous(), group=group)
    return all_vals, all_ids


def heads_topk_sharded(h: torch.Tensor, W1: torch.Tensor, b1: torch.Tensor, Wout_shard: torch.Tensor,
                       V: int, topk: int, group=None, ws: Optional[torch.Tensor] = None, stream=None,
                       head_logits: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """S1-S3 on this rank's rows of Wout, then the exchange and the merge.

    Wout_shard [K, n_g, d] holds rows shard_bounds(V, G)[rank] of every head (G, rank from
    `group`, or a single shard when torch.distributed is not initialised).  Returns the global
    (topk_ids [B, K, topk] int32, topk_vals [B, K, topk] fp32) on every rank, produced on
    `stream` (torch's current stream when None).  head_logits, if given, receives this rank's
    [B, K, n_g] logits."""
    G = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    bounds = shard_bounds(V, G)
    r0, n = bounds[rank]
    if Wout_shard.shape[1] != n:
        raise ValueError(f"rank {rank} of {G} holds {Wout_shard.shape[1]} rows of Wout, expected {n}")
    B, K = h.shape[0], Wout_shard.shape[0]
    dev = h.device
    with _on(stream):
        if ws is None:
            ws = workspace(medusa_heads_workspace_size(B, h.shape[1], n, K, topk), dev)
        ids = torch.empty((B, K, topk), dtype=torch.int32, device=dev)
        vals = torch.empty((B, K, topk), dtype=torch.float32, device=dev)
        medusa_heads_topk(h, W1, b1, Wout_shard, topk, ids, vals, ws, head_logits=head_logits)
        if G == 1:
            all_vals, all_ids = vals.unsqueeze(0), ids.unsqueeze(0)
        else:
            all_vals, all_ids = gather_shard_lists(vals, ids, group)
        out_ids = torch.empty_like(ids)
        out_vals = torch.empty_like(vals)
        medusa_topk_merge(all_vals, all_ids, [b[0] for b in bounds], V, out_vals, out_ids)
    return out_ids, out_vals


def tree_attention_sharded(tree, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                           seq_lens: torch.Tensor, scale: float, out: torch.Tensor, group=None, stream=None):
    """S5 with every slice's cached prefix split over the ranks of `group`.

    This rank's window (medusa_tree_attention_split) goes straight into `out`; the ranks
    all-gather their lse values ([layers, B, T, H] fp32 each); each rank scales its window output
    by exp(lse_rank - lse) in place (medusa_attention_rescale); an all-reduce (sum) of `out` then
    leaves medusa_tree_attention's result on every rank.  With one rank (or no process group) it
    is that call.  Each rank needs only its window's rows of the caches (and the last rank the
    tree rows), in the full [.., Lcap, hd] layout."""
    G = dist.get_world_size(group) if dist.is_initialized() else 1
    with _on(stream):
        if G == 1:
            medusa_tree_attention(tree, q, k_cache, v_cache, seq_lens, scale, out)
            return out
        rank = dist.get_rank(group)
        lse = torch.empty(tuple(out.shape[:-1]), dtype=torch.float32, device=out.device)
        medusa_tree_attention_split(tree, q, k_cache, v_cache, seq_lens, scale, rank, G, out, lse)
        all_l = torch.empty((G,) + tuple(lse.shape), dtype=torch.float32, device=out.device)
        dist.all_gather(list(all_l.unbind(0)), lse, group=group)
        medusa_attention_rescale(all_l, rank, out)
        dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
    return out
