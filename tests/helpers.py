"""Shared pieces of the GPU parity tests: oracle runs of a workload and the
matching device buffers.  Inputs come only from ``synth``; expected values
come only from ``oracle``."""

from __future__ import annotations

import json
import os

import numpy as np

import oracle.medusa_oracle as O
from synth import inputs as I, workloads as W

HERE = os.path.dirname(os.path.abspath(__file__))
SUBSEEDS = os.path.join(HERE, "golden", "subseeds.json")

# Tolerances of the verification step's stated accuracy: head logits 1e-2
# relative; attention 2e-3 max-abs for bf16 inputs, 1e-5 for fp32; ids, paths
# and lengths bit-exact.
LOGIT_RTOL = 1e-2
ATTN_ATOL = {"bf16": 2e-3, "f32": 1e-5}


def stored_subseeds(w):
    """Sub-seeds chosen by golden/make_subseeds.py, for an unmodified full workload."""
    if os.path.exists(SUBSEEDS) and W.WORKLOADS.get(w.name) == w:
        d = json.load(open(SUBSEEDS))
        if w.name in d:
            return d[w.name]["sub_h"], d[w.name]["sub_logits"]
    return None


def oracle_tree(w):
    return O.tree_tables(O.ranksum_choices(w.K, w.topk, w.n_nodes), w.K, w.topk)


def oracle_heads(w, sub_h):
    h = I.values(I.hidden(w, sub_h))
    b1 = I.values(I.b1(w))
    us, zs = [], []
    for k in range(w.K):
        u, z = O.medusa_head_one(h, I.values(I.w1(w, k)), b1[k], I.values(I.wout(w, k)))
        us.append(u)
        zs.append(z)
    return np.stack(us, 1), np.stack(zs, 1)


def pick_sub_h(w, max_tries=16):
    """First sub-seed whose head logits keep every top-k gap >= 1e-4 relative."""
    st = stored_subseeds(w)
    if st is not None:
        u, z = oracle_heads(w, st[0])
        return st[0], u, z
    for s in range(max_tries):
        u, z = oracle_heads(w, s)
        if O.topk_gap_ok(z, w.topk):
            return s, u, z
    raise RuntimeError("no usable sub-seed")


def pick_logits(w, tr, toks, cand, max_tries=16):
    st = stored_subseeds(w)
    if st is not None:
        return st[1], I.base_logits(w, toks, tr["parent"], st[1])
    for s in range(max_tries):
        z = I.base_logits(w, toks, tr["parent"], s)
        if "typical" not in w.modes or O.typical_margin_ok(tr, z, cand, w.temperature, w.eps, w.alpha):
            return s, z
    raise RuntimeError("no usable logits sub-seed")


def pick_uniforms(w, tr, logits, cand, mode, top_p, max_tries=32):
    """First uniforms sub-seed whose draws sit clear inside their token's CDF interval at the
    node where each sequence's walk ends; None when that node's nucleus boundary itself is not
    clear (other logits are needed then)."""
    base = O.evaluate_posterior(tr, logits, cand, mode, w.temperature, w.eps, w.alpha, top_p)
    wts = []
    for b in range(w.B):
        last = tr["retrieve"][base["best_path"][b], base["accept_len"][b]]
        pr = O.node_statistics(logits[b, last:last + 1], w.temperature, w.eps, w.alpha)["prob"][0]
        if mode == "nucleus":
            if not O.nucleus_cut_ok(pr, top_p):
                return None
            pr = np.where(O.nucleus_mask(pr, top_p), pr, 0.0)
        wts.append(pr)
    for s in range(max_tries):
        u = I.uniforms(w, s)
        if all(O.sample_margin_ok(wts[b], float(u[b])) for b in range(w.B)):
            return s, u
    raise RuntimeError("no usable uniforms sub-seed")


def pick_nucleus_inputs(w, tr, toks, cand, top_p, sampled, max_tries=16):
    """Base logits (and uniforms when sampled) whose nucleus decisions all sit clear of their
    boundaries: every tree edge's membership and, when sampled, the final node's cut-off and draw."""
    for s in range(max_tries):
        z = I.base_logits(w, toks, tr["parent"], s)
        if not O.nucleus_margin_ok(tr, z, cand, w.temperature, top_p):
            continue
        if not sampled:
            return s, z, None
        got = pick_uniforms(w, tr, z, cand, "nucleus", top_p)
        if got is not None:
            return s, z, got[1]
    raise RuntimeError("no usable logits sub-seed for nucleus acceptance")


def check_logits(got, ref, rtol=LOGIT_RTOL):
    got = np.asarray(got, dtype=np.float64)
    scale = np.abs(ref).max()
    err = np.abs(got - ref)
    bad = err > rtol * np.abs(ref) + 1e-4 * scale
    assert not bad.any(), f"{bad.sum()} head logits off; max err {err.max():.3g} (scale {scale:.3g})"


# Small workloads that the oracle finishes in seconds but that still span
# several GEMV stages, several key tiles with a ragged tail, batch groups,
# and the tree shapes of the full workloads.
SMALL = {
    "tiny_f32": W.get("tiny_f32"),
    "v7b_small": W.shrink(W.get("vicuna7b_bs1_L1024"), name="v7b_small", d=512, V=5000, layers=2, H=4,
                          prefix=200),
    "v7b_typical_small": W.shrink(W.get("vicuna7b_bs1_L4096_typical"), name="v7b_typical_small", d=768,
                                  V=4000, layers=2, H=3, prefix=300),
    "v13b_small": W.shrink(W.get("vicuna13b_bs8_ragged"), name="v13b_small", d=512, V=4000, layers=2, H=3,
                           prefix_range=(50, 400)),
    "v33b_small": W.shrink(W.get("vicuna33b_bs4_L8192_N128"), name="v33b_small", d=768, V=3000, layers=2,
                           H=2, prefix=257),
    "b3_small": W.shrink(W.get("vicuna13b_bs8_ragged"), name="b3_small", B=3, d=256, V=1500, layers=1, H=2,
                         prefix_range=(0, 130), n_nodes=20),
}
