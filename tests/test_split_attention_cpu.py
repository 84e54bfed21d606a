"""Pins for the oracle of tree attention split along the cached prefix.

The split is the library's multi-GPU option (no counterpart on the pages):
rank r of G attends to its window of prefix rows (the last rank also to the
tree's own rows) and returns (O_r, lse_r); the log-sum-exp identity puts the
parts back together.  Pinned here against the already pinned unsplit oracle
(the identity must reproduce it for any G), closed forms (equal scores give
the mean of V and ln(n); a single key gives its own V and score), and the
window bookkeeping.  The host-side argument checks of medusa_attention_combine
are exercised at the end (nothing reaches a device)."""

import numpy as np
import pytest

import oracle.medusa_oracle as O

WORKED = [(0,), (1,), (0, 0), (0, 1), (1, 0), (1, 1)]


def _inputs(T, L, hd, seed=0):
    rng = np.random.default_rng(seed)
    return (rng.normal(size=(T, hd)), rng.normal(size=(L + T + 5, hd)), rng.normal(size=(L + T + 5, hd)))


@pytest.mark.parametrize("L,G", [(1024, 1), (1024, 8), (200, 3), (7, 7), (5, 3), (0, 1)])
def test_windows_partition_the_prefix(L, G):
    wins = [O.attention_window(G, r, L) for r in range(G)]
    assert wins[0][0] == 0 and wins[-1][1] == L
    for (a, b), (c, _) in zip(wins, wins[1:]):
        assert b == c and a <= b
    sizes = [b - a for a, b in wins]
    assert max(sizes) - min(sizes) <= 1


@pytest.mark.parametrize("choices,K,topk,L", [(WORKED, 2, 2, 37), (O.ranksum_choices(5, 10, 40), 5, 10, 300),
                                              (O.ranksum_choices(5, 10, 40), 5, 10, 3), ([], 3, 2, 64)])
@pytest.mark.parametrize("G", [1, 2, 3, 7])
def test_combined_windows_equal_the_unsplit_attention(choices, K, topk, L, G):
    tr = O.tree_tables(choices, K, topk)
    hd = 32
    q, k, v = _inputs(tr["T"], L, hd, seed=G)
    scale = O.attention_scale(hd)
    ref = O.tree_attention_slice(tr, q, k, v, L, scale)
    outs, lses = [], []
    for r in range(G):
        lo, hi = O.attention_window(G, r, L)
        o, l = O.tree_attention_window_slice(tr, q, k, v, L, scale, lo, hi, with_tree=(r == G - 1))
        outs.append(o)
        lses.append(l)
    got, lse = O.combine_partials(np.stack(outs), np.stack(lses))
    assert np.allclose(got, ref, atol=1e-12, rtol=1e-12)
    o1, l1 = O.tree_attention_window_slice(tr, q, k, v, L, scale, 0, L, with_tree=True)
    assert np.allclose(lse, l1, atol=1e-12) and np.allclose(o1, ref, atol=1e-12)


def test_window_closed_forms():
    tr = O.tree_tables(O.ranksum_choices(3, 2, 6), 3, 2)
    T, L, hd = tr["T"], 20, 16
    _, k, v = _inputs(T, L, hd, seed=5)
    # q = 0: every score is 0, so lse = ln(number of keys) and O is the mean of their V rows
    q0 = np.zeros((T, hd))
    o, lse = O.tree_attention_window_slice(tr, q0, k, v, L, 0.25, 4, 13, with_tree=True)
    for i in range(T):
        rows = list(range(4, 13)) + [L + j for j in range(T) if tr["anc"][i, j]]
        assert np.isclose(lse[i], np.log(len(rows)), atol=1e-14)
        assert np.allclose(o[i], v[rows].mean(axis=0), atol=1e-14)
    # one prefix key and no tree rows: O is that key's V row, lse its scaled score
    q = np.random.default_rng(9).normal(size=(T, hd))
    o, lse = O.tree_attention_window_slice(tr, q, k, v, L, 0.3, 7, 8, with_tree=False)
    assert np.allclose(o, np.broadcast_to(v[7], o.shape), atol=0)
    assert np.allclose(lse, 0.3 * (q @ k[7]), atol=1e-14)
    # an empty window: O = 0, lse = -inf, and it contributes nothing when combined
    o_e, l_e = O.tree_attention_window_slice(tr, q, k, v, L, 0.3, 5, 5, with_tree=False)
    assert not o_e.any() and np.all(l_e == -np.inf)
    got, l2 = O.combine_partials(np.stack([o_e, o]), np.stack([l_e, lse]))
    assert np.allclose(got, o, atol=0) and np.allclose(l2, lse, atol=0)


# ---------------------------------------------------------------------------
# medusa_attention_combine: host-side checks (nothing reaches a device)


@pytest.fixture(scope="module")
def mb(built):
    import speculative_decoding_heads_b200 as mb
    return mb


def _raw(t):
    """A host tensor's address: these calls fail their checks before any use of it."""
    import ctypes
    return ctypes.c_void_p(t.data_ptr())


def _combine(mb, G, rows, hd, outs, lses, out):
    mb._check(mb._lib.medusa_attention_combine(G, rows, hd, outs if outs is None else _raw(outs), _raw(lses),
                                               _raw(out), None, 0))


def _combine_args(G, rows, hd):
    import torch
    return torch.zeros(G, rows, hd), torch.zeros(G, rows), torch.zeros(rows, hd)


@pytest.mark.parametrize("G,rows,hd,what", [(65, 4, 8, "G, rows or hd"), (0, 4, 8, "G, rows or hd"),
                                            (2, 4, 6, "G, rows or hd"), (2, 4, 2048, "G, rows or hd")])
def test_combine_rejects_shapes(mb, G, rows, hd, what):
    outs, lses, out = _combine_args(max(G, 1), rows, hd)
    with pytest.raises(mb.MedusaError) as e:
        _combine(mb, G, rows, hd, outs, lses, out)
    assert e.value.code == mb.MEDUSA_ERR_INVALID_ARG and what in str(e.value)


def test_combine_rejects_overlap_and_misalignment(mb):
    import torch
    outs, lses, _ = _combine_args(2, 4, 8)
    with pytest.raises(mb.MedusaError) as e:
        _combine(mb, 2, 4, 8, outs, lses, outs[1])
    assert "overlaps" in str(e.value)
    odd = torch.zeros(4 * 8 + 1)[1:].view(4, 8)          # 4 bytes past a 16-byte boundary
    with pytest.raises(mb.MedusaError) as e:
        _combine(mb, 2, 4, 8, outs, lses, odd)
    assert "misaligned" in str(e.value)
    with pytest.raises(mb.MedusaError) as e:
        _combine(mb, 2, 4, 8, None, lses, odd)
    assert "null pointer" in str(e.value)
    with pytest.raises(ValueError, match="CUDA tensors"):
        mb.medusa_attention_combine(outs, lses, torch.zeros(4, 8))


# ---------------------------------------------------------------------------
# tree_attention_sharded's exchange on two gloo ranks: each rank's window
# output and lse, an all-gather of the lse values only, the per-rank scaling
# by exp(lse_r - lse) and an all-reduce (sum) must give the unsplit oracle.
# The two library calls are replaced by oracle stand-ins on the host, so what
# runs here is the exchange itself.


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _sharded_main(rank, world, port, q):
    import os
    import sys
    import torch
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist
    import oracle.medusa_oracle as Om
    import speculative_decoding_heads_b200.sharded as sh
    tr = Om.tree_tables(Om.ranksum_choices(3, 3, 9), 3, 3)
    L, hd, layers, B, H = 23, 8, 1, 2, 2
    rng = np.random.default_rng(11)
    qq = rng.normal(size=(layers, B, tr["T"], H, hd))
    kc = rng.normal(size=(layers, B, H, L + tr["T"], hd))
    vc = rng.normal(size=(layers, B, H, L + tr["T"], hd))
    lens = np.array([L, L - 6])
    scale = 0.4

    class _Tree:
        T = tr["T"]

    def split(tree, q, k_cache, v_cache, seq_lens, sc, r, G, out, lse, stream=None):
        for l in range(layers):
            for b in range(B):
                for e in range(H):
                    lo, hi = Om.attention_window(G, r, int(seq_lens[b]))
                    o, s = Om.tree_attention_window_slice(tr, q[l, b, :, e].numpy(), k_cache[l, b, e].numpy(),
                                                          v_cache[l, b, e].numpy(), int(seq_lens[b]), sc, lo, hi,
                                                          with_tree=(r == G - 1))
                    out[l, b, :, e] = torch.from_numpy(o)
                    lse[l, b, :, e] = torch.from_numpy(s)

    def rescale(lses, r, part, lse_out=None, stream=None):
        tot = torch.logsumexp(lses, dim=0)
        part *= torch.exp(lses[r] - tot).unsqueeze(-1)

    sh.medusa_tree_attention_split = split
    sh.medusa_attention_rescale = rescale
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out = torch.zeros((layers, B, tr["T"], H, hd), dtype=torch.float64)
        sh.tree_attention_sharded(_Tree(), torch.from_numpy(qq), torch.from_numpy(kc), torch.from_numpy(vc),
                                  torch.from_numpy(lens), scale, out)
        err = 0.0
        for l in range(layers):
            for b in range(B):
                for e in range(H):
                    ref = Om.tree_attention_slice(tr, qq[l, b, :, e], kc[l, b, e], vc[l, b, e], int(lens[b]), scale)
                    err = max(err, float(np.abs(out[l, b, :, e].numpy() - ref).max()))
        q.put((rank, err))
    finally:
        dist.destroy_process_group()


def test_sharded_attention_exchange_two_gloo_ranks(built):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sharded_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert [r for r, _ in res] == [0, 1]
    # the lse buffers are fp32, as the library's are: about 1e-7 of rounding
    assert all(err < 1e-5 for _, err in res), res
