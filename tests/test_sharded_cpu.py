"""Vocabulary-sharded heads on the host: the shard split, the mathematics the
merge relies on (pinned with the oracle's own top-k), the all-gather between
two gloo ranks, and the host-side argument checks of medusa_topk_merge.  No
compute call is made here."""

import ctypes
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle.medusa_oracle as O

REPO = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def mb(built):
    import speculative_decoding_heads_b200 as mb
    return mb


@pytest.fixture(scope="module")
def sh(mb):
    import speculative_decoding_heads_b200.sharded as sh
    return sh


@pytest.mark.parametrize("V,G", [(32000, 1), (32000, 2), (32000, 3), (32001, 8), (1000, 7), (64, 64)])
def test_shard_bounds_partition_the_vocabulary(sh, V, G):
    b = sh.shard_bounds(V, G)
    assert len(b) == G and b[0][0] == 0
    for (r0, n), (r1, _) in zip(b, b[1:]):
        assert r1 == r0 + n
    assert b[-1][0] + b[-1][1] == V
    sizes = [n for _, n in b]
    assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)


@pytest.mark.parametrize("V,G", [(5, 6), (100, 65), (100, 0)])
def test_shard_bounds_rejects_impossible_splits(sh, V, G):
    with pytest.raises(ValueError):
        sh.shard_bounds(V, G)


@pytest.mark.parametrize("G,k", [(2, 10), (3, 8), (7, 32), (5, 1)])
def test_topk_of_gathered_shard_lists_is_the_global_topk(G, k):
    """The merge's premise: the k best of the union of every shard's k best
    (shard-local ids offset by the shard's first row) are the k best of the
    whole row, ties included.  Values come from a small set so that ties
    inside and across shards are common."""
    rng = np.random.default_rng(1000 * G + k)
    V = 997
    z = rng.integers(-6, 7, size=(4, V)).astype(np.float64)
    z[1, :] = 0.0                       # one row of all-equal values
    z[2, ::5] = np.inf                  # many equal maxima
    bounds, r0 = [], 0
    base, extra = divmod(V, G)
    for g in range(G):
        n = base + (1 if g < extra else 0)
        bounds.append((r0, n))
        r0 += n
    cand_ids, cand_vals = [], []
    for r0, n in bounds:
        ids, vals = O.topk_desc(z[:, r0:r0 + n], k)
        cand_ids.append(ids + r0)
        cand_vals.append(vals)
    cand_ids = np.concatenate(cand_ids, axis=1)
    cand_vals = np.concatenate(cand_vals, axis=1)
    ref_ids, ref_vals = O.topk_desc(z, k)
    for row in range(z.shape[0]):
        # The candidates as a sparse row: every other id holds -inf, below
        # every candidate except equal -inf ones, which the row never has.
        dense = np.full(V, -np.inf)
        dense[cand_ids[row]] = cand_vals[row]
        ids, vals = O.topk_desc(dense[None, :], k)
        assert np.array_equal(ids[0], ref_ids[row]) and np.array_equal(vals[0], ref_vals[row])


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _lists(rank, B=2, K=3, k=4):
    g = torch.Generator().manual_seed(77 + rank)
    vals = torch.randn(B, K, k, generator=g)
    ids = torch.randint(0, 1000, (B, K, k), generator=g, dtype=torch.int32)
    return vals, ids


def _gather_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, REPO)
    import torch.distributed as dist
    import speculative_decoding_heads_b200.sharded as sh
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        vals, ids = _lists(rank)
        all_vals, all_ids = sh.gather_shard_lists(vals, ids)
        ok = all_vals.shape == (world,) + tuple(vals.shape) and all_ids.dtype == torch.int32
        for r in range(world):
            v, i = _lists(r)
            ok = ok and torch.equal(all_vals[r], v) and torch.equal(all_ids[r], i)
        q.put((rank, bool(ok)))
    finally:
        dist.destroy_process_group()


def test_gather_shard_lists_two_gloo_ranks(built):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    assert sorted(q.get(timeout=5) for _ in range(2)) == [(0, True), (1, True)]


@pytest.mark.parametrize("G,topk,row0,V,what", [
    (2, 4, [1, 50], 100, "row0[0]"),
    (2, 4, [0, 98], 100, "fewer than topk"),
    (3, 4, [0, 2, 50], 100, "fewer than topk"),
    (2, 4, [0, 60], 40, "fewer than topk"),
    (2, 33, [0, 50], 100, "topk"),
    (65, 1, list(range(65)), 100, "G, B or K"),
])
def test_merge_rejects_bad_arguments_before_launch(mb, G, topk, row0, V, what):
    vals = torch.zeros(G, 1, 1, topk)
    ids = torch.zeros(G, 1, 1, topk, dtype=torch.int32)
    out_vals = torch.zeros(1, 1, topk)
    out_ids = torch.zeros(1, 1, topk, dtype=torch.int32)
    raw = lambda t: ctypes.c_void_p(t.data_ptr())      # host memory: the checks fail before any use
    r0 = (ctypes.c_int32 * len(row0))(*row0)
    with pytest.raises(mb.MedusaError) as e:
        mb._check(mb._lib.medusa_topk_merge(raw(vals), raw(ids), r0, G, V, 1, 1, topk, raw(out_vals), raw(out_ids),
                                            None))
    assert e.value.code == mb.MEDUSA_ERR_INVALID_ARG and what in str(e.value)


def test_binding_refuses_host_tensors(mb):
    vals, ids = torch.zeros(2, 1, 1, 4), torch.zeros(2, 1, 1, 4, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensors"):
        mb.medusa_topk_merge(vals, ids, [0, 50], 100, torch.zeros(1, 1, 4), torch.zeros(1, 1, 4, dtype=torch.int32),
                             stream=_NoStream())


class _NoStream:
    """A stream stand-in for host-side checks (never reaches the device)."""
    cuda_stream = 0


def test_sharded_heads_rejects_a_wrong_shard(sh):
    h = torch.zeros(1, 256)
    W1, b1 = torch.zeros(2, 256, 256), torch.zeros(2, 256)
    Wout = torch.zeros(2, 99, 256)          # a single shard must hold all V = 100 rows
    with pytest.raises(ValueError):
        sh.heads_topk_sharded(h, W1, b1, Wout, V=100, topk=4)
