"""Chooses the sub-seeds of every workload with the oracle and writes subseeds.json.

A workload's hidden state is re-drawn (sub-seed ``sub_h``) until every gap
among each head's k+1 largest logits is at least 1e-4 relative, and its base
logits are re-drawn (``sub_logits``) until every tree edge's
|p - threshold| under typical acceptance is at least 1e-4 relative.  Both
sides then take the same top-k and acceptance decisions whatever their
rounding order.  Only ``oracle`` and ``synth`` are used.

    python tests/golden/make_subseeds.py [workload ...]
"""

import json
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle.medusa_oracle as O  # noqa: E402
from synth import inputs as I, workloads as W  # noqa: E402

OUT = os.path.join(HERE, "subseeds.json")


def head_logits(w, sub_h):
    h = I.values(I.hidden(w, sub_h))
    b1 = I.values(I.b1(w))
    zs = []
    for k in range(w.K):
        _, z = O.medusa_head_one(h, I.values(I.w1(w, k)), b1[k], I.values(I.wout(w, k)))
        zs.append(z)
    return np.stack(zs, axis=1)


def choose(w, max_tries=32):
    tr = O.tree_tables(O.ranksum_choices(w.K, w.topk, w.n_nodes), w.K, w.topk)
    # the head logits depend on sub_h only through h: draw the weights once
    h_all = {}
    b1 = I.values(I.b1(w))
    W1 = [I.values(I.w1(w, k)) for k in range(w.K)]
    Wo = [I.values(I.wout(w, k)) for k in range(w.K)]
    sub_h = None
    for s in range(max_tries):
        h = I.values(I.hidden(w, s))
        z = np.stack([O.medusa_head_one(h, W1[k], b1[k], Wo[k])[1] for k in range(w.K)], axis=1)
        if O.topk_gap_ok(z, w.topk):
            sub_h, h_all = s, z
            break
    if sub_h is None:
        raise RuntimeError(f"{w.name}: no sub_h within {max_tries} tries")
    ids, _ = O.topk_desc(h_all, w.topk)
    toks, cand, _ = O.build_tree(tr, I.root_tokens(w), ids, w.prefix_lens())
    sub_l = 0
    if "typical" in w.modes:
        for s in range(max_tries):
            z = I.base_logits(w, toks, tr["parent"], s)
            if O.typical_margin_ok(tr, z, cand, w.temperature, w.eps, w.alpha):
                sub_l = s
                break
        else:
            raise RuntimeError(f"{w.name}: no sub_logits within {max_tries} tries")
    return {"sub_h": sub_h, "sub_logits": sub_l}


def main(names):
    data = json.load(open(OUT)) if os.path.exists(OUT) else {}
    for n in names:
        t0 = time.time()
        data[n] = choose(W.get(n))
        print(n, data[n], f"{time.time() - t0:.1f}s", flush=True)
        with open(OUT, "w") as f:
            json.dump(data, f, indent=1, sort_keys=True)


if __name__ == "__main__":
    main(sys.argv[1:] or list(W.WORKLOADS))
