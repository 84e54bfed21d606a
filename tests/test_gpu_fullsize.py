"""Parity at the workloads' full sizes, in the launch configuration the
benchmark times (one ``medusa_step`` over device-resident inputs).

The oracle computes what it can in full -- every head logit (S1-S3), the
tree (S4) and the posterior (S6) -- and attention (S5) and the KV
compaction (S7) on a sample of (layer, sequence, head) slices: the first and
last layer's first and last head of every sequence plus seeded random
slices, each regenerated on the host from the counter-based generator.  The
planted agreement uses the oracle's own tree tokens, so no input depends on
the CUDA path.
"""

import numpy as np
import pytest
import torch

import oracle.medusa_oracle as O
from synth import inputs as I, workloads as W
from helpers import ATTN_ATOL, check_logits, oracle_heads, oracle_tree, stored_subseeds

pytestmark = pytest.mark.gpu

# Every full workload in every acceptance mode it names (config 3 runs greedy
# and typical; config 4 sweeps trees of 16, 32, 64 and 128 nodes).
FULL = [(name, mode) for name in ("vicuna7b_bs1_L1024", "vicuna7b_bs1_L4096_typical", "vicuna13b_bs8_ragged",
                                  "vicuna33b_bs4_L8192_N16", "vicuna33b_bs4_L8192_N32",
                                  "vicuna33b_bs4_L8192_N64", "vicuna33b_bs4_L8192_N128")
        for mode in W.get(name).modes]


@pytest.fixture(scope="module")
def mb(built):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import speculative_decoding_heads_b200 as mb
    return mb


def _sample_slices(w, n_random=6):
    picks = set()
    for l in (0, w.layers - 1):
        for b in range(w.B):
            for e in (0, w.H - 1):
                picks.add((l, b, e))
    rng = np.random.default_rng(w.seed)
    for _ in range(n_random):
        picks.add((int(rng.integers(w.layers)), int(rng.integers(w.B)), int(rng.integers(w.H))))
    return sorted(picks)


@pytest.mark.parametrize("name,mode", FULL, ids=[f"{n}-{m}" for n, m in FULL])
def test_full_step(mb, name, mode):
    from synth import device
    w = W.get(name)
    sub = stored_subseeds(w)
    assert sub is not None, "full workloads carry stored sub-seeds"
    sub_h, sub_l = sub
    tr = oracle_tree(w)

    # ---- oracle: S1-S4 in full, S6 in full
    _, z = oracle_heads(w, sub_h)
    ids, vals = O.topk_desc(z, w.topk)
    lens = np.asarray(w.prefix_lens())
    toks, cand, pos = O.build_tree(tr, I.root_tokens(w), ids, lens)
    logits = I.base_logits(w, toks, tr["parent"], sub_l)
    post = O.evaluate_posterior(tr, logits, cand, mode, w.temperature, w.eps, w.alpha)

    # ---- device: the benchmark's inputs, planted with the oracle's tree tokens
    choices = O.ranksum_choices(w.K, w.topk, w.n_nodes)
    tree = mb.Tree(choices, w.K, w.topk)
    t = device.materialise(w, sub_h=sub_h, sub_logits=sub_l, with_head_logits=True)
    device.tree_outputs(t, w.B, tree.T, tree.P, tree.D)
    toks_dev = torch.from_numpy(np.ascontiguousarray(toks, dtype=np.int32)).cuda()
    device.plant(t["base_logits"], toks_dev, device.parent_tensor(tr["parent"]), w.agreement,
                 w.seed + 7919 * sub_l)
    args = mb.make_step_args(tree, t, mb.MEDUSA_TYPICAL if mode == "typical" else mb.MEDUSA_GREEDY,
                             w.temperature, w.eps, w.alpha)
    ws = mb.workspace(mb.medusa_step_workspace_size(args))
    mb.medusa_step(args, ws)
    torch.cuda.synchronize()
    st, det = mb.device_status(clear=True)
    assert (st, det) == (0, 0), f"device status {st} detail {det}"

    # S1-S3
    check_logits(t["head_logits"].cpu().numpy(), z)
    assert np.array_equal(t["topk_ids"].cpu().numpy(), ids)
    check_logits(t["topk_vals"].cpu().numpy(), vals)
    # S4
    assert np.array_equal(t["tree_tokens"].cpu().numpy(), toks)
    assert np.array_equal(t["candidates"].cpu().numpy(), cand)
    assert np.array_equal(t["position_ids"].cpu().numpy(), pos)
    # S6
    for ours, ref in [("best_path", "best_path"), ("accept_len", "accept_len"),
                      ("accepted_tokens", "accepted_tokens"), ("next_token", "next_token")]:
        assert np.array_equal(t[ours].cpu().numpy(), post[ref]), ours
    # S7: sequence lengths
    assert np.array_equal(t["seq_lens"].cpu().numpy(), lens + post["accept_len"] + 1)

    # S5 and S7 on sampled slices
    scale = O.attention_scale(w.hd)
    out = t["attn_out"]
    kc, vc = t["k_cache"], t["v_cache"]
    worst = 0.0
    for (l, b, e) in _sample_slices(w):
        L = int(lens[b])
        rows = L + tree.T
        ks = I.values(I.kv_slice(w, "k", l, b, e, rows))
        vs = I.values(I.kv_slice(w, "v", l, b, e, rows))
        ref = O.tree_attention_slice(tr, I.q_slice(w, l, b, e), ks, vs, L, scale)
        got = out[l, b, :, e, :].double().cpu().numpy()
        err = float(np.abs(got - ref).max())
        worst = max(worst, err)
        assert err <= ATTN_ATOL[w.dtype], f"slice {(l, b, e)}: max abs err {err}"
        a = int(post["accept_len"][b])
        path = tr["retrieve"][int(post["best_path"][b]), : a + 1]
        for cache, src in ((kc, ks), (vc, vs)):
            moved = cache[l, b, e, L:L + a + 1, :].float().double().cpu().numpy()
            assert np.array_equal(moved, src[L + path]), f"KV rows of slice {(l, b, e)}"
    print(f"{name}: attention max abs err over sampled slices {worst:.2e}")
