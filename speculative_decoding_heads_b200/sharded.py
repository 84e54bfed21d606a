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
rows), the ranks all-gather their (output, lse) partials, and the log-sum-exp
combine gives the unsplit result (tree_attention_sharded).

Every step runs in the library's kernels; torch.distributed only moves the
gathered lists (NCCL between GPUs, gloo on the host for the tests).
"""

from typing import List, Optional, Tuple

import torch
import torch.distributed as dist

from . import (MAX_SHARDS, medusa_attention_combine, medusa_heads_topk, medusa_heads_workspace_size,
               medusa_topk_merge, medusa_tree_attention, medusa_tree_attention_split, workspace)


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
    (topk_ids [B, K, topk] int32, topk_vals [B, K, topk] fp32) on every rank.  head_logits, if
    given, receives this rank's [B, K, n_g] logits."""
    G = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    bounds = shard_bounds(V, G)
    r0, n = bounds[rank]
    if Wout_shard.shape[1] != n:
        raise ValueError(f"rank {rank} of {G} holds {Wout_shard.shape[1]} rows of Wout, expected {n}")
    B, K = h.shape[0], Wout_shard.shape[0]
    dev = h.device
    if ws is None:
        ws = workspace(medusa_heads_workspace_size(B, h.shape[1], n, K, topk), dev)
    ids = torch.empty((B, K, topk), dtype=torch.int32, device=dev)
    vals = torch.empty((B, K, topk), dtype=torch.float32, device=dev)
    medusa_heads_topk(h, W1, b1, Wout_shard, topk, ids, vals, ws, head_logits=head_logits, stream=stream)
    if G == 1:
        all_vals, all_ids = vals.unsqueeze(0), ids.unsqueeze(0)
    else:
        # The collective runs on torch's current stream: order it after the
        # heads kernel and the merge after it when the caller gave a stream.
        if stream is not None:
            torch.cuda.current_stream(dev).wait_stream(stream)
        all_vals, all_ids = gather_shard_lists(vals, ids, group)
        if stream is not None:
            stream.wait_stream(torch.cuda.current_stream(dev))
    out_ids = torch.empty_like(ids)
    out_vals = torch.empty_like(vals)
    medusa_topk_merge(all_vals, all_ids, [b[0] for b in bounds], V, out_vals, out_ids, stream=stream)
    return out_ids, out_vals


def tree_attention_sharded(tree, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                           seq_lens: torch.Tensor, scale: float, out: torch.Tensor, group=None, stream=None):
    """S5 with every slice's cached prefix split over the ranks of `group`: this rank's window
    (medusa_tree_attention_split), an all-gather of the G partial outputs and lse values, and the
    combine.  `out` [layers, B, T, H, hd] receives medusa_tree_attention's result on every rank;
    with one rank (or no process group) it is that call.  Each rank needs only its window's rows
    of the caches (and the last rank the tree rows), in the full [.., Lcap, hd] layout."""
    G = dist.get_world_size(group) if dist.is_initialized() else 1
    if G == 1:
        medusa_tree_attention(tree, q, k_cache, v_cache, seq_lens, scale, out, stream=stream)
        return out
    rank = dist.get_rank(group)
    dev = out.device
    part = torch.empty_like(out)
    lse = torch.empty(tuple(out.shape[:-1]), dtype=torch.float32, device=dev)
    medusa_tree_attention_split(tree, q, k_cache, v_cache, seq_lens, scale, rank, G, part, lse, stream=stream)
    if stream is not None:
        torch.cuda.current_stream(dev).wait_stream(stream)
    all_o = torch.empty((G,) + tuple(out.shape), dtype=torch.float32, device=dev)
    all_l = torch.empty((G,) + tuple(lse.shape), dtype=torch.float32, device=dev)
    dist.all_gather(list(all_o.unbind(0)), part, group=group)
    dist.all_gather(list(all_l.unbind(0)), lse, group=group)
    if stream is not None:
        stream.wait_stream(torch.cuda.current_stream(dev))
    medusa_attention_combine(all_o, all_l, out, stream=stream)
    return out
