"""Vocabulary-sharded heads on one GPU.

The G shards run one after another on the same device, each a
medusa_heads_topk call on its rows of Wout; their top-k lists are then
merged by medusa_topk_merge.  This is the per-rank arithmetic of the
multi-GPU split without the all-gather, which the gloo test covers on the
host; no kernel waits on another.  The merged lists must equal the unsplit
call bit for bit and the oracle's top-k.
"""

import numpy as np
import pytest
import torch

import oracle.medusa_oracle as O
from helpers import SMALL, pick_sub_h

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mb(built):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import speculative_decoding_heads_b200 as mb
    return mb


@pytest.fixture(scope="module")
def sh(mb):
    import speculative_decoding_heads_b200.sharded as sh
    return sh


@pytest.fixture(scope="module")
def dev(mb):
    from synth import device
    return device


def _np(t):
    return t.detach().cpu().numpy()


def _unsplit(mb, t, w):
    ws = mb.workspace(mb.medusa_heads_workspace_size(w.B, w.d, w.V, w.K, w.topk))
    ids = torch.empty(w.B, w.K, w.topk, dtype=torch.int32, device="cuda")
    vals = torch.empty(w.B, w.K, w.topk, device="cuda")
    logits = torch.empty(w.B, w.K, w.V, device="cuda")
    mb.medusa_heads_topk(t["h"], t["W1"], t["b1"], t["Wout"], w.topk, ids, vals, ws, head_logits=logits)
    return ids, vals, logits


def _sharded(mb, sh, t, w, G, logits_full=None):
    bounds = sh.shard_bounds(w.V, G)
    all_vals = torch.empty(G, w.B, w.K, w.topk, device="cuda")
    all_ids = torch.empty(G, w.B, w.K, w.topk, dtype=torch.int32, device="cuda")
    for g, (r0, n) in enumerate(bounds):
        Wg = t["Wout"][:, r0:r0 + n, :].contiguous()
        lg = torch.empty(w.B, w.K, n, device="cuda")
        ws = mb.workspace(mb.medusa_heads_workspace_size(w.B, w.d, n, w.K, w.topk))
        mb.medusa_heads_topk(t["h"], t["W1"], t["b1"], Wg, w.topk, all_ids[g], all_vals[g], ws, head_logits=lg)
        if logits_full is not None:
            torch.cuda.synchronize()
            assert torch.equal(lg, logits_full[:, :, r0:r0 + n]), f"shard {g}: logits differ from the unsplit call"
    out_ids = torch.empty(w.B, w.K, w.topk, dtype=torch.int32, device="cuda")
    out_vals = torch.empty(w.B, w.K, w.topk, device="cuda")
    mb.medusa_topk_merge(all_vals, all_ids, [b[0] for b in bounds], w.V, out_vals, out_ids)
    torch.cuda.synchronize()
    return out_ids, out_vals


@pytest.mark.parametrize("name,G", [("v7b_small", 2), ("v7b_small", 3), ("v13b_small", 5), ("tiny_f32", 2),
                                    ("b3_small", 4)])
def test_sharded_heads_match_unsplit_and_oracle(mb, sh, dev, name, G):
    w = SMALL[name]
    sub_h, u, z = pick_sub_h(w)
    ids_ref, vals_ref = O.topk_desc(z, w.topk)
    t = dev.materialise(w, sub_h=sub_h)
    ids, vals, logits = _unsplit(mb, t, w)
    out_ids, out_vals = _sharded(mb, sh, t, w, G, logits_full=logits)
    assert torch.equal(out_ids, ids) and torch.equal(out_vals, vals)
    assert np.array_equal(_np(out_ids), ids_ref)
    st, det = mb.device_status(clear=True)
    assert (st, det) == (0, 0)


def test_sharded_tie_across_shards_takes_the_lower_id(mb, sh, dev):
    """Head 0's best row copied into another shard: two equal logits in two
    shards; the merged list puts the lower token id first, as the unsplit
    call does."""
    w = SMALL["v7b_small"]
    G = 3
    sub_h, _, _ = pick_sub_h(w)
    t = dev.materialise(w, sub_h=sub_h)
    ids, _, _ = _unsplit(mb, t, w)
    torch.cuda.synchronize()
    r1 = int(ids[0, 0, 0])
    first_shard_end = sh.shard_bounds(w.V, G)[0][1]
    r2 = w.V - 1 if r1 < first_shard_end else 0
    t["Wout"][0, r2, :] = t["Wout"][0, r1, :]
    ids, vals, logits = _unsplit(mb, t, w)
    torch.cuda.synchronize()
    assert float(logits[0, 0, r1]) == float(logits[0, 0, r2])
    assert [int(x) for x in ids[0, 0, :2]] == [min(r1, r2), max(r1, r2)]
    out_ids, out_vals = _sharded(mb, sh, t, w, G, logits_full=logits)
    assert torch.equal(out_ids, ids) and torch.equal(out_vals, vals)


@pytest.mark.parametrize("G,topk", [(2, 1), (3, 10), (7, 32), (64, 4)])
def test_merge_kernel_matches_oracle_topk(mb, sh, G, topk):
    """Per-shard lists from the oracle's top-k of each slice of a logit row
    with many ties, ±inf and NaN; the merge must give the oracle's top-k of
    the whole row."""
    rng = np.random.default_rng(100 * G + topk)
    B, K = 3, 5
    V = G * topk + 37
    z = rng.integers(-4, 5, size=(B, K, V)).astype(np.float32)
    z[0, 1, ::3] = np.inf
    z[1, 2, :] = -np.inf
    z[2, 0, ::4] = np.nan
    z[2, 3, :] = 1.5
    bounds = sh.shard_bounds(V, G)
    lv, li = [], []
    for r0, n in bounds:
        ids_g, vals_g = O.topk_desc(z[..., r0:r0 + n], topk)
        li.append(ids_g.astype(np.int32))
        lv.append(vals_g.astype(np.float32))
    all_ids = torch.from_numpy(np.stack(li)).cuda()
    all_vals = torch.from_numpy(np.stack(lv)).cuda()
    out_ids = torch.empty(B, K, topk, dtype=torch.int32, device="cuda")
    out_vals = torch.empty(B, K, topk, device="cuda")
    mb.medusa_topk_merge(all_vals, all_ids, [b[0] for b in bounds], V, out_vals, out_ids)
    torch.cuda.synchronize()
    ref_ids, ref_vals = O.topk_desc(z, topk)
    assert np.array_equal(_np(out_ids), ref_ids)
    assert np.array_equal(_np(out_vals), ref_vals.astype(np.float32), equal_nan=True)


def test_single_shard_entry_point_equals_unsplit(mb, sh, dev):
    w = SMALL["v13b_small"]
    sub_h, _, _ = pick_sub_h(w)
    t = dev.materialise(w, sub_h=sub_h)
    ids, vals, _ = _unsplit(mb, t, w)
    out_ids, out_vals = sh.heads_topk_sharded(t["h"], t["W1"], t["b1"], t["Wout"], w.V, w.topk)
    torch.cuda.synchronize()
    assert torch.equal(out_ids, ids) and torch.equal(out_vals, vals)


def test_sharded_calls_on_a_side_stream_with_a_busy_allocator(mb, sh, dev):
    """heads_topk_sharded and tree_attention_sharded given their own stream: their temporaries
    belong to that stream, so allocations on the default stream right after the call (which
    would reuse freed blocks) cannot clobber what the stream's kernels still read."""
    w = SMALL["v13b_small"]
    sub_h, _, _ = pick_sub_h(w)
    t = dev.materialise(w, sub_h=sub_h)
    ref_ids, ref_vals, _ = _unsplit(mb, t, w)
    tree = mb.Tree(O.ranksum_choices(w.K, w.topk, w.n_nodes), w.K, w.topk)
    scale = O.attention_scale(w.hd)
    ref_out = torch.empty_like(t["attn_out"])
    mb.medusa_tree_attention(tree, t["q"], t["k_cache"], t["v_cache"], t["seq_lens"], scale, ref_out)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    for _ in range(3):
        side.wait_stream(torch.cuda.current_stream())
        ids, vals = sh.heads_topk_sharded(t["h"], t["W1"], t["b1"], t["Wout"], w.V, w.topk, stream=side)
        out = torch.empty_like(t["attn_out"])
        side.wait_stream(torch.cuda.current_stream())
        sh.tree_attention_sharded(tree, t["q"], t["k_cache"], t["v_cache"], t["seq_lens"], scale, out, stream=side)
        junk = [torch.full((1 << 20,), -7.0, device="cuda") for _ in range(16)]   # the default stream, busy
        side.synchronize()
        assert torch.equal(ids, ref_ids) and torch.equal(vals, ref_vals)
        assert torch.equal(out, ref_out)
        del junk
