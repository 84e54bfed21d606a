"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Every oracle function is checked here against something other than itself:
the pages' worked example, closed forms, invariants the pages state, special
cases that reduce to a library routine (torch's fp64 scaled-dot-product
attention), and brute force on tiny inputs.  ``test_mutants_are_caught``
plants plausible mistakes into copies of the oracle and checks that these
pins reject every one of them.
"""

import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle.medusa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def _read_worked_example():
    d = {"sees": {}}
    with open(os.path.join(GOLDEN, "worked_example_mask.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            if key == "sees":
                d["sees"][int(vals[0])] = set(int(v) for v in vals[1:])
            else:
                d[key] = [int(v) for v in vals]
    return d


WORKED = [(0,), (1,), (0, 0), (0, 1), (1, 0), (1, 1)]


# ---------------------------------------------------------------------------
# tree and candidate assembly
# ---------------------------------------------------------------------------


def check_worked_example(O):
    g = _read_worked_example()
    tr = O.tree_tables(WORKED, K=2, topk=2)
    topk_ids = np.array([[g["head1"], g["head2"]]])
    toks, cand, pos = O.build_tree(tr, np.array(g["root"]), topk_ids, np.array([40]))
    assert list(toks[0]) == g["input"]
    for node, seen in g["sees"].items():
        visible = {int(toks[0, j]) for j in range(tr["T"]) if tr["anc"][node, j] and j != node}
        assert visible == seen, (node, visible, seen)
        assert tr["anc"][node, node], "a node sees itself"
    assert tr["P"] == g["paths"][0]
    assert [list(c) for c in cand[0]] == [[900, 11, 21], [900, 11, 22], [900, 12, 21], [900, 12, 22]]
    assert list(pos[0]) == [40, 41, 41, 42, 42, 42, 42]


def test_worked_example_mask():
    check_worked_example(O)


def test_full_tree_tiny_workload():
    ch = O.ranksum_choices(3, 2, 14)
    assert sorted(ch) == sorted(c for n in (1, 2, 3) for c in itertools.product(range(2), repeat=n))
    tr = O.tree_tables(ch, 3, 2)
    assert tr["T"] == 15 and tr["P"] == 8 and tr["D"] == 3
    assert list(np.bincount(tr["depth"])) == [1, 2, 4, 8]


def _count_tuples(length, total, topk):
    """Number of length-tuples over [0, topk) with the given sum (dynamic programming)."""
    ways = [1] + [0] * total
    for _ in range(length):
        nxt = [0] * (total + 1)
        for s, w in enumerate(ways):
            if w:
                for r in range(topk):
                    if s + r <= total:
                        nxt[s + r] += w
        ways = nxt
    return ways[total]


@pytest.mark.parametrize("K,topk,n", [(5, 10, 63), (4, 8, 48), (5, 10, 16), (5, 10, 32), (5, 10, 64),
                                      (5, 10, 128), (3, 2, 14), (2, 3, 7)])
def test_ranksum_depth_histogram(K, topk, n):
    """Depth histogram from tuple counts per (rank sum, length) group, filled in order."""
    left = n
    hist = [0] * (K + 1)
    last = None
    for s in range(K * (topk - 1) + 1):
        for length in range(1, K + 1):
            c = _count_tuples(length, s, topk)
            take = min(c, left)
            hist[length] += take
            left -= take
            if take:
                last = (s, length, take)
            if left == 0:
                break
        if left == 0:
            break
    ch = O.ranksum_choices(K, topk, n)
    tr = O.tree_tables(ch, K, topk)
    got = list(np.bincount(tr["depth"], minlength=K + 1))
    got[0] = 0
    assert got == hist
    # the partially taken group is its lexicographically smallest members
    s, length, take = last
    group = sorted(t for t in itertools.product(range(min(topk, s + 1)), repeat=length) if sum(t) == s)
    assert sorted(t for t in ch if sum(t) == s and len(t) == length) == group[:take]
    # a node is a leaf exactly when its (.., 0) child was not selected
    sel = set(ch)
    assert tr["P"] == 1 * (n == 0) + sum(1 for t in ch if t + (0,) not in sel)


def test_vicuna7b_tree_counts():
    # Hand count of the rank-sum construction (K=5, top-10, 63 nodes): rank sums
    # 0 (5 tuples), 1 (15), 2 (35), then 8 of rank sum 3 -- (3), (0,3), (1,2),
    # (2,1), (3,0), (0,0,3), (0,1,2), (0,2,1) -- give 4/10/13/15/21 nodes by depth.
    tr = O.tree_tables(O.ranksum_choices(5, 10, 63), 5, 10)
    assert list(np.bincount(tr["depth"]))[1:] == [4, 10, 13, 15, 21]
    assert tr["T"] == 64 and tr["D"] == 5


def check_tree_tables_random(O):
    for _ in range(10):
        K, topk = int(RNG.integers(1, 5)), int(RNG.integers(1, 5))
        allt = [t for n in range(1, K + 1) for t in itertools.product(range(topk), repeat=n)]
        pick = set()
        for t in RNG.permutation(len(allt))[: int(RNG.integers(1, min(40, len(allt)) + 1))]:
            t = allt[t]
            for j in range(1, len(t) + 1):
                pick.add(t[:j])
        tr = O.tree_tables(list(pick), K, topk)
        nodes = tr["nodes"]
        for i, c in enumerate(nodes):
            # tree_indices: head len(c)'s rank c[-1] in [root, head1 top-k, ...]
            assert tr["tree_indices"][i] == (0 if not c else 1 + (len(c) - 1) * topk + c[-1])
            if c:
                assert nodes[tr["parent"][i]] == c[:-1]
        for p in range(tr["P"]):
            row = [n for n in tr["retrieve"][p] if n >= 0]
            assert [len(nodes[n]) for n in row] == list(range(len(row)))
            assert all(nodes[row[j]] == nodes[row[-1]][:j] for j in range(len(row)))
        leaves = [n for p in range(tr["P"]) for n in tr["retrieve"][p] if n >= 0 and
                  len(nodes[n]) == max(len(nodes[m]) for m in tr["retrieve"][p] if m >= 0)]
        assert leaves == sorted(leaves)


def test_tree_tables_random():
    check_tree_tables_random(O)


# ---------------------------------------------------------------------------
# heads and top-k
# ---------------------------------------------------------------------------


def _silu_loop(x):
    return x / (1.0 + math.exp(-x))


def check_heads_bruteforce(O):
    B, d, V, K = 2, 4, 6, 3
    h = RNG.normal(size=(B, d))
    W1 = RNG.normal(size=(K, d, d))
    b1 = RNG.normal(size=(K, d))
    Wo = RNG.normal(size=(K, V, d))
    u, z = O.medusa_heads(h, W1, b1, Wo)
    for b in range(B):
        for k in range(K):
            for i in range(d):
                pre = sum(W1[k, i, c] * h[b, c] for c in range(d)) + b1[k, i]
                assert abs(u[b, k, i] - (h[b, i] + _silu_loop(pre))) < 1e-12
            for v in range(V):
                ref = sum(Wo[k, v, c] * u[b, k, c] for c in range(d))
                assert abs(z[b, k, v] - ref) < 1e-12


def test_heads_bruteforce():
    check_heads_bruteforce(O)


def test_heads_closed_forms():
    d, V = 4, 5
    h = RNG.normal(size=(1, d))
    Wo = RNG.normal(size=(1, V, d))
    # W1 = 0, b1 = 0: SiLU(0) = 0, so u = h
    u, z = O.medusa_heads(h, np.zeros((1, d, d)), np.zeros((1, d)), Wo)
    assert np.allclose(u[0, 0], h[0], atol=0) and np.allclose(z[0, 0], Wo[0] @ h[0], rtol=1e-15)
    # h = 0 and b1 = ln 3: SiLU(ln 3) = ln 3 * sigmoid(ln 3) = 0.75 ln 3
    u, _ = O.medusa_heads(np.zeros((1, d)), RNG.normal(size=(1, d, d)), np.full((1, d), math.log(3)), Wo)
    assert np.allclose(u, 0.75 * math.log(3), rtol=1e-14)


def check_topk(O):
    z = RNG.integers(0, 5, size=(3, 40)).astype(np.float64)   # many exact ties
    ids, vals = O.topk_desc(z, 7)
    for r in range(3):
        ref = sorted(range(40), key=lambda i: (-z[r, i], i))[:7]
        assert list(ids[r]) == ref
        assert list(vals[r]) == [z[r, i] for i in ref]


def test_topk_bruteforce():
    check_topk(O)


# ---------------------------------------------------------------------------
# tree attention
# ---------------------------------------------------------------------------


def _sdpa_rows(q, k, v, mask=None):
    """torch fp64 scaled-dot-product attention (default scale 1/sqrt(hd))."""
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None], torch.from_numpy(v)[None, None],
        attn_mask=None if mask is None else torch.from_numpy(mask)[None, None])
    return out[0, 0].numpy()


def _attn_inputs(T, L, hd, rows_extra=3):
    q = RNG.normal(size=(T, hd))
    k = RNG.normal(size=(L + T + rows_extra, hd))
    v = RNG.normal(size=(L + T + rows_extra, hd))
    return q, k, v


def check_attention_paths(O, choices, K, topk, L=9, hd=16):
    tr = O.tree_tables(choices, K, topk)
    T = tr["T"]
    q, k, v = _attn_inputs(T, L, hd)
    out = O.tree_attention_slice(tr, q, k, v, L, O.attention_scale(hd))
    for p in range(tr["P"]):
        path = [n for n in tr["retrieve"][p] if n >= 0]
        rows = list(range(L)) + [L + n for n in path]
        n = len(path)
        causal = np.tril(np.ones((n, L + n), dtype=bool), k=L)    # bottom-right aligned
        ref = _sdpa_rows(q[path], k[rows], v[rows], causal)
        assert np.allclose(out[path], ref, atol=1e-12, rtol=1e-12)


@pytest.mark.parametrize("which", ["worked", "full", "ranksum"])
def test_attention_equals_causal_along_every_path(which):
    if which == "worked":
        check_attention_paths(O, WORKED, 2, 2)
    elif which == "full":
        check_attention_paths(O, O.ranksum_choices(3, 2, 14), 3, 2)
    else:
        check_attention_paths(O, O.ranksum_choices(5, 10, 40), 5, 10, L=0)


def check_chain_and_decode(O):
    # top-1 chain: ordinary causal attention over prefix + chain
    K, L, hd = 5, 11, 32
    tr = O.tree_tables(O.ranksum_choices(K, 1, K), K, 1)
    q, k, v = _attn_inputs(tr["T"], L, hd)
    out = O.tree_attention_slice(tr, q, k, v, L, O.attention_scale(hd))
    n = tr["T"]
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k[: L + n])[None, None],
        torch.from_numpy(v[: L + n])[None, None],
        attn_mask=torch.ones(n, L + n, dtype=torch.bool).tril(L)[None, None])[0, 0].numpy()
    assert np.allclose(out, ref, atol=1e-12)
    # root only: plain decode attention over prefix + the root's own row
    tr1 = O.tree_tables([], 3, 2)
    q, k, v = _attn_inputs(1, L, hd)
    out1 = O.tree_attention_slice(tr1, q, k, v, L, O.attention_scale(hd))
    assert np.allclose(out1, _sdpa_rows(q, k[: L + 1], v[: L + 1]), atol=1e-12)


def test_chain_and_decode_special_cases():
    check_chain_and_decode(O)


# ---------------------------------------------------------------------------
# posterior
# ---------------------------------------------------------------------------


def _planted_logits(tr, toks, V, q_agree, sigma=3.0, seed=0):
    rng = np.random.default_rng(seed)
    z = rng.normal(scale=sigma, size=(toks.shape[0], tr["T"], V))
    for b in range(toks.shape[0]):
        for i in range(tr["T"]):
            kids = [c for c in range(1, tr["T"]) if tr["parent"][c] == i]
            if kids and rng.random() < q_agree:
                c = kids[rng.integers(len(kids))]
                z[b, i, toks[b, c]] = z[b, i].max() + 5
    return z


def _walk(tr, toks_b, z_b):
    """Sequential autoregressive greedy check: follow the child equal to the argmax."""
    node, path = 0, [0]
    while True:
        g = int(np.argmax(z_b[node]))
        nxt = [c for c in range(1, tr["T"]) if tr["parent"][c] == node and toks_b[c] == g]
        if not nxt:
            return path, g
        node = nxt[0]
        path.append(node)


def check_greedy_walk(O, seed):
    rng = np.random.default_rng(seed)
    K, topk, n, V = 4, 5, 30, 50
    tr = O.tree_tables(O.ranksum_choices(K, topk, n), K, topk)
    B = 3
    topk_ids = np.stack([np.stack([rng.permutation(V)[:topk] for _ in range(K)]) for _ in range(B)])
    toks, cand, _ = O.build_tree(tr, rng.integers(0, V, size=B), topk_ids, np.zeros(B, dtype=np.int64))
    z = _planted_logits(tr, toks, V, 0.8, seed=seed)
    post = O.evaluate_posterior(tr, z, cand, "greedy")
    for b in range(B):
        path, g = _walk(tr, toks[b], z[b])
        a = len(path) - 1
        assert post["accept_len"][b] == a
        assert list(post["accepted_tokens"][b][: a + 1]) == [int(toks[b, n]) for n in path]
        assert all(t == -1 for t in post["accepted_tokens"][b][a + 1:])
        assert post["next_token"][b] == g
        best = post["best_path"][b]
        assert list(tr["retrieve"][best][: a + 1]) == path
        assert all(list(tr["retrieve"][p][: a + 1]) != path for p in range(best))
        # step yields a + 1 tokens (the bonus token rides on top of them)
        assert (post["accepted_tokens"][b] >= 0).sum() == a + 1


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_greedy_equals_sequential_walk(seed):
    check_greedy_walk(O, seed)


def check_typical_closed_forms(O):
    V, eps, alpha = 64, 0.09, 0.3
    # uniform row: p = 1/V, H = ln V, threshold = min(eps, alpha / V)
    st = O.node_statistics(np.zeros((1, V)), 0.7, eps, alpha)
    assert abs(st["entropy"][0] - math.log(V)) < 1e-12
    assert abs(st["threshold"][0] - min(eps, alpha / V)) < 1e-15
    assert np.allclose(st["prob"][0], 1.0 / V)
    # two-level row at temperature T: z_0 = c, others 0
    for c, Tmp in [(2.0, 0.7), (5.0, 1.0), (-1.0, 2.0)]:
        z = np.zeros((1, V))
        z[0, 0] = c
        e = math.exp(c / Tmp)
        p0, pr = e / (e + V - 1), 1.0 / (e + V - 1)
        H = -(p0 * math.log(p0) + (V - 1) * pr * math.log(pr))
        st = O.node_statistics(z, Tmp, eps, alpha)
        assert abs(st["prob"][0, 0] - p0) < 1e-14 and abs(st["prob"][0, 1] - pr) < 1e-14
        assert abs(st["entropy"][0] - H) < 1e-12
        assert abs(st["threshold"][0] - min(eps, alpha * math.exp(-H))) < 1e-14
    # low entropy: alpha e^-H >= eps, so the threshold is eps itself
    z = np.zeros((1, V))
    z[0, 3] = 40.0
    st = O.node_statistics(z, 1.0, eps, alpha)
    assert alpha * math.exp(-st["entropy"][0]) > eps and st["threshold"][0] == eps


def test_typical_closed_forms():
    check_typical_closed_forms(O)


def check_typical_bruteforce(O, seed):
    rng = np.random.default_rng(seed)
    K, topk, V = 3, 3, 12
    tr = O.tree_tables(O.ranksum_choices(K, topk, 12), K, topk)
    topk_ids = np.stack([rng.permutation(V)[:topk] for _ in range(K)])[None]
    toks, cand, _ = O.build_tree(tr, np.array([5]), topk_ids, np.array([0]))
    z = rng.normal(scale=1.5, size=(1, tr["T"], V))
    for temp, eps, alpha in [(0.7, 0.09, 0.3), (1.3, 0.2, 0.5), (0.4, 0.05, 2.0)]:
        post = O.evaluate_posterior(tr, z, cand, "typical", temp, eps, alpha)
        accs = []
        for p in range(tr["P"]):
            acc = 0
            for j in range(1, tr["D"] + 1):
                node = tr["retrieve"][p][j]
                if node < 0:
                    break
                par = tr["retrieve"][p][j - 1]
                ex = [math.exp(z[0, par, v] / temp) for v in range(V)]
                s = sum(ex)
                probs = [x / s for x in ex]
                H = -sum(pp * math.log(pp) for pp in probs)
                if not probs[cand[0, p, j]] > min(eps, alpha * math.exp(-H)):
                    break
                acc += 1
            accs.append(acc)
        best = accs.index(max(accs))
        assert post["best_path"][0] == best and post["accept_len"][0] == max(accs)
        last = tr["retrieve"][best][max(accs)]
        assert post["next_token"][0] == int(np.argmax(z[0, last]))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_typical_bruteforce(seed):
    check_typical_bruteforce(O, seed)


# ---------------------------------------------------------------------------
# nucleus acceptance and the sampled next token
# ---------------------------------------------------------------------------


def _nucleus_brute(pr, top_p):
    """Smallest m such that the m most probable tokens (lower id first on ties) hold >= top_p."""
    order = sorted(range(len(pr)), key=lambda i: (-pr[i], i))
    for m in range(1, len(pr) + 1):
        if sum(pr[i] for i in order[:m]) >= top_p:
            return set(order[:m])
    return set(order)


def check_nucleus_mask(O):
    pr = np.array([0.2, 0.5, 0.3])
    assert list(O.nucleus_mask(pr, 0.8)) == [False, True, True]   # 0.5 + 0.3 reaches 0.8 exactly
    assert list(O.nucleus_mask(pr, 0.81)) == [True, True, True]
    assert list(O.nucleus_mask(pr, 0.5)) == [False, True, False]
    assert list(O.nucleus_mask(pr, 1e-9)) == [False, True, False]  # only the most probable token
    assert list(O.nucleus_mask(np.full(4, 0.25), 0.5)) == [True, True, False, False]   # ties by id
    rng = np.random.default_rng(7)
    for _ in range(40):
        V = int(rng.integers(2, 12))
        pr = rng.dirichlet(np.ones(V) * 0.7)
        pr[rng.integers(V)] = pr[rng.integers(V)]                 # an exact tie now and then
        pr = pr / pr.sum()
        for top_p in (0.3, 0.8, 0.95):
            got = set(np.flatnonzero(O.nucleus_mask(pr, top_p)))
            assert got == _nucleus_brute(pr, top_p), (pr, top_p)


def test_nucleus_mask():
    check_nucleus_mask(O)


def check_sample_index(O):
    w = np.array([1.0, 0.0, 3.0])
    assert O.sample_index(w, 0.0) == 0
    assert O.sample_index(w, 0.2499) == 0
    assert O.sample_index(w, 0.25) == 2          # cumulative 1.0 is not above 0.25 * 4: token 1 has no weight
    assert O.sample_index(w, 0.999) == 2
    # a fine grid of u reproduces the weights
    w = np.array([0.1, 0.0, 0.45, 0.2, 0.25])
    n = 20000
    counts = np.bincount([O.sample_index(w, (i + 0.5) / n) for i in range(n)], minlength=5)
    assert np.abs(counts / n - w / w.sum()).max() <= 1.0 / n


def test_sample_index():
    check_sample_index(O)


def check_nucleus_posterior(O, seed):
    rng = np.random.default_rng(seed)
    K, topk, V = 3, 3, 10
    tr = O.tree_tables(O.ranksum_choices(K, topk, 12), K, topk)
    topk_ids = np.stack([rng.permutation(V)[:topk] for _ in range(K)])[None]
    toks, cand, _ = O.build_tree(tr, np.array([4]), topk_ids, np.array([0]))
    z = rng.normal(scale=1.5, size=(1, tr["T"], V))
    for temp, top_p in [(0.7, 0.8), (1.3, 0.5), (0.4, 0.95)]:
        u = np.array([rng.random()])
        post = O.evaluate_posterior(tr, z, cand, "nucleus", temp, top_p=top_p, uniforms=u)
        accs = []
        probs_of = lambda node: [math.exp(z[0, node, v] / temp) / sum(math.exp(z[0, node, x] / temp) for x in range(V))
                                 for v in range(V)]
        for p in range(tr["P"]):
            acc = 0
            for j in range(1, tr["D"] + 1):
                node = tr["retrieve"][p][j]
                if node < 0:
                    break
                if cand[0, p, j] not in _nucleus_brute(probs_of(tr["retrieve"][p][j - 1]), top_p):
                    break
                acc += 1
            accs.append(acc)
        best = accs.index(max(accs))
        assert post["best_path"][0] == best and post["accept_len"][0] == max(accs)
        last = tr["retrieve"][best][max(accs)]
        pr = probs_of(last)
        nuc = _nucleus_brute(pr, top_p)
        w = [pr[v] if v in nuc else 0.0 for v in range(V)]
        tot, cum, draw = sum(w), 0.0, None
        for v in range(V):
            cum += w[v]
            if cum > u[0] * tot:
                draw = v
                break
        assert post["next_token"][0] == draw


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_nucleus_posterior_bruteforce(seed):
    check_nucleus_posterior(O, seed)


def test_nucleus_and_sampling_special_cases():
    rng = np.random.default_rng(5)
    K, topk, V = 4, 3, 40
    tr = O.tree_tables(O.ranksum_choices(K, topk, 30), K, topk)
    topk_ids = np.stack([rng.permutation(V)[:topk] for _ in range(K)])[None]
    toks, cand, _ = O.build_tree(tr, np.array([1]), topk_ids, np.array([0]))
    z = _planted_logits(tr, toks, V, 0.8, seed=5)
    greedy = O.evaluate_posterior(tr, z, cand, "greedy")
    # top_p -> 0: the nucleus is the argmax alone, so acceptance is greedy acceptance
    tiny = O.evaluate_posterior(tr, z, cand, "nucleus", 1.0, top_p=1e-12)
    for k in ("best_path", "accept_len", "accepted_tokens", "next_token"):
        assert np.array_equal(tiny[k], greedy[k]), k
    # ... and a draw from a one-token nucleus is that token, whatever u
    for u in (0.0, 0.37, 0.9999):
        assert O.evaluate_posterior(tr, z, cand, "nucleus", 1.0, top_p=1e-12,
                                    uniforms=np.array([u]))["next_token"][0] == greedy["next_token"][0]
    # top_p = 1 keeps every token: every candidate of nonzero probability is accepted
    full = O.evaluate_posterior(tr, z, cand, "nucleus", 1.0, top_p=1.0)
    assert full["accept_len"][0] == tr["D"]
    assert full["best_path"][0] == int(np.argmax((tr["retrieve"] >= 0).sum(1)))   # the first path of full depth
    # without uniforms the typical and nucleus next token is the argmax (the reading used so far)
    typ = O.evaluate_posterior(tr, z, cand, "typical", 0.7)
    assert typ["next_token"][0] == int(np.argmax(z[0, tr["retrieve"][typ["best_path"][0], typ["accept_len"][0]]]))


def check_sampling_guards(O):
    rel = O.NUCLEUS_REL
    # nucleus boundary of one distribution [0.5, 0.3, 0.2]
    assert not O.nucleus_cut_ok([0.5, 0.3, 0.2], 0.8)                 # the mass through the last member is top_p
    assert O.nucleus_cut_ok([0.5, 0.3, 0.2], 0.7)
    assert not O.nucleus_cut_ok([0.5, 0.3, 0.2], 0.5 + rel / 2)       # the mass before the last member is too close
    assert O.nucleus_cut_ok([0.5, 0.3, 0.2], 0.5 + 2 * rel)
    # the last member and the first token left out tie: which one is in depends on rounding
    assert not O.nucleus_cut_ok([0.4, 0.3, 0.3], 0.6)
    assert O.nucleus_cut_ok([0.4, 0.4, 0.2], 0.6)                     # a tie inside the nucleus is harmless
    # tree edges: one-edge tree whose child token (id 0) has mass 0.5 ranking before it
    tr = O.tree_tables([(0,)], 1, 1)
    _, cand, _ = O.build_tree(tr, np.array([3]), np.array([[[0]]]), np.array([0]))
    z = np.zeros((1, 2, 3))
    z[0, 0] = np.log([0.3, 0.5, 0.2])
    assert O.nucleus_margin_ok(tr, z, cand, 1.0, 0.5 + 2 * rel)
    assert not O.nucleus_margin_ok(tr, z, cand, 1.0, 0.5 + rel / 2)
    assert not O.nucleus_margin_ok(tr, z, cand, 1.0, 0.5 - rel / 2)
    z[0, 1] = np.log([0.5, 0.3, 0.2])                                  # the leaf's row is no parent
    assert O.nucleus_margin_ok(tr, z, cand, 1.0, 0.5 + 2 * rel)
    # the draw's interval: weights [1, 3], u * 4 = 1 exactly is a boundary
    assert not O.sample_margin_ok([1.0, 3.0], 0.25)
    assert not O.sample_margin_ok([1.0, 3.0], 0.25 - rel / 8)
    assert O.sample_margin_ok([1.0, 3.0], 0.25 + rel) and O.sample_margin_ok([1.0, 3.0], 0.1)


def test_sampling_guards():
    check_sampling_guards(O)


# ---------------------------------------------------------------------------
# accept KV
# ---------------------------------------------------------------------------


def check_accept_kv(O):
    tr = O.tree_tables(WORKED, 2, 2)
    layers, B, H, hd, L = 2, 2, 3, 8, 5
    Lcap = L + tr["T"] + 2
    kc = RNG.normal(size=(layers, B, H, Lcap, hd))
    vc = RNG.normal(size=(layers, B, H, Lcap, hd))
    lens = np.array([L, L + 1])
    # sequence 0 takes path 2 = (root, B, X after B): node_1 = 2 overlaps destination L+2
    best, alen = np.array([2, 0]), np.array([2, 1])
    k2, v2, lens2 = O.accept_kv(tr, kc, vc, lens, best, alen)
    assert list(lens2) == [L + 3, L + 3]
    for b in range(B):
        Lb = lens[b]
        src = [Lb + tr["retrieve"][best[b]][j] for j in range(alen[b] + 1)]
        for j, s in enumerate(src):
            assert np.array_equal(k2[:, b, :, Lb + j], kc[:, b, :, s])
            assert np.array_equal(v2[:, b, :, Lb + j], vc[:, b, :, s])
        untouched = [r for r in range(Lcap) if not Lb <= r <= Lb + alen[b]]
        assert np.array_equal(k2[:, b, :, untouched], kc[:, b, :, untouched])
    # After compaction, plain causal attention over the new prefix reproduces the
    # tree-attention output of every accepted node.
    q = RNG.normal(size=(layers, B, tr["T"], H, hd))
    out = O.tree_attention(tr, q, kc, vc, lens, O.attention_scale(hd))
    for b in range(B):
        for j in range(alen[b] + 1):
            node = tr["retrieve"][best[b]][j]
            n_rows = lens[b] + j + 1
            for l in range(layers):
                for e in range(H):
                    ref = _sdpa_rows(q[l, b, node, e][None], k2[l, b, e, :n_rows], v2[l, b, e, :n_rows])
                    assert np.allclose(out[l, b, node, e], ref[0], atol=1e-12)


def test_accept_kv_invariants():
    check_accept_kv(O)


# ---------------------------------------------------------------------------
# margin guards (they choose the sub-seeds that make bit-exact ids a fair
# demand: every top-k gap and every typical-acceptance margin >= 1e-4 relative)
# ---------------------------------------------------------------------------


def check_topk_gap_guard(O):
    # Well separated: fine at every k up to the row length.
    z = np.array([[10.0, 9.0, 8.0, 7.0, -3.0, 0.5]])
    assert all(O.topk_gap_ok(z, k) for k in range(1, 6))
    # The 3rd and 4th largest values are 5e-5 apart (relative): the top-3 set
    # depends on that pair, so k = 3 must be refused; k = 2 never looks at it.
    z = np.array([[10.0, 9.0, 8.0, 8.0 * (1 - 5e-5), 1.0]])
    assert O.topk_gap_ok(z, 2)
    assert not O.topk_gap_ok(z, 3)
    # A tie right after the k-th value (k = 4) decides membership; ties further
    # down the row do not.
    z = np.array([[5.0, 4.0, 3.0, 1.0, 1.0, 1.0]])
    assert O.topk_gap_ok(z, 3)
    assert not O.topk_gap_ok(z, 4)
    # Gap just under and just over 1e-4 of the larger magnitude (1.0).  The
    # first gap is above 1e-4 of the smaller value, so only a guard relative to
    # the larger one refuses it.
    g_in, g_out = 1e-4 * (1 - 5e-5), 1e-4 * (1 + 5e-5)
    assert not O.topk_gap_ok(np.array([[1.0, 1.0 - g_in, -5.0]]), 1)
    assert O.topk_gap_ok(np.array([[1.0, 1.0 - g_out, -5.0]]), 1)
    # Negative values: the magnitude counts, not the signed value.
    assert not O.topk_gap_ok(np.array([[-2.0, -2.0 * (1 + 5e-5), -9.0]]), 1)
    assert O.topk_gap_ok(np.array([[-2.0, -2.0 * (1 + 5e-4), -9.0]]), 1)
    # Every row of a batch is checked, whatever its position.
    ok_row, bad_row = [7.0, 3.0, 1.0, 0.0], [7.0, 3.0, 3.0 * (1 + 1e-5), 0.0]
    assert O.topk_gap_ok(np.array([[ok_row, ok_row], [ok_row, ok_row]]), 2)
    assert not O.topk_gap_ok(np.array([[ok_row, ok_row], [ok_row, bad_row]]), 2)


def test_topk_gap_guard():
    check_topk_gap_guard(O)


def _two_level_margin(a, V, temp, eps, alpha):
    """(p - thr) / max(p, thr) for the token with logit a in a row [a, 0, ..., 0] (closed form)."""
    e = math.exp(a / temp)
    p, r = e / (e + V - 1), 1.0 / (e + V - 1)
    H = -(p * math.log(p) + (V - 1) * r * math.log(r))
    thr = min(eps, alpha * math.exp(-H))
    return (p - thr) / max(p, thr)


def _logit_for_margin(target, V, temp, eps, alpha, lo=-3.0, hi=1.0):
    """Bisection for the logit a whose two-level margin is `target` (it grows with a here)."""
    assert _two_level_margin(lo, V, temp, eps, alpha) < target < _two_level_margin(hi, V, temp, eps, alpha)
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if _two_level_margin(mid, V, temp, eps, alpha) < target:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def check_typical_margin_guard(O):
    V, temp, eps, alpha = 8, 1.0, 0.09, 0.3
    # One-edge tree: root -> its head-1 top-1 token (token 0 of the vocabulary).
    tr = O.tree_tables([(0,)], 1, 1)
    _, cand, _ = O.build_tree(tr, np.array([3]), np.array([[[0]]]), np.array([0]))

    def ok(target, child_row=None):
        z = np.zeros((1, 2, V))
        z[0, 0, 0] = _logit_for_margin(target, V, temp, eps, alpha)
        if child_row is not None:
            z[0, 1] = child_row
        return O.typical_margin_ok(tr, z, cand, temp, eps, alpha)

    assert ok(2e-4) and ok(-2e-4)
    assert not ok(5e-5) and not ok(-5e-5)
    # Just inside 1e-4 of the larger of p and thr (but not of the smaller).
    assert not ok(1e-4 * (1 - 2e-5)) and not ok(-1e-4 * (1 - 2e-5))
    assert ok(1e-4 * (1 + 2e-5)) and ok(-1e-4 * (1 + 2e-5))
    # A leaf's own row is no edge's parent: its values never matter.
    leaf = np.zeros(V)
    leaf[5] = _logit_for_margin(0.0, V, temp, eps, alpha)
    assert ok(2e-4, leaf)


def test_typical_margin_guard():
    check_typical_margin_guard(O)


# ---------------------------------------------------------------------------
# planted mistakes must be caught
# ---------------------------------------------------------------------------


class _Mutant:
    """A copy of the oracle module namespace with one function replaced."""

    def __init__(self, **over):
        for name in dir(O):
            if not name.startswith("__"):
                setattr(self, name, getattr(O, name))
        for k, v in over.items():
            setattr(self, k, v)


def _attn_no_self(tree, q_slice, k_slice, v_slice, L_b, scale):
    t2 = dict(tree)
    t2["anc"] = tree["anc"] & ~np.eye(tree["T"], dtype=bool)
    t2["anc"][0, 0] = True
    return O.tree_attention_slice(t2, q_slice, k_slice, v_slice, L_b, scale)


def _attn_all_tree(tree, q_slice, k_slice, v_slice, L_b, scale):
    t2 = dict(tree)
    t2["anc"] = np.tril(np.ones_like(tree["anc"]))
    return O.tree_attention_slice(t2, q_slice, k_slice, v_slice, L_b, scale)


def _attn_bad_scale(tree, q_slice, k_slice, v_slice, L_b, scale):
    return O.tree_attention_slice(tree, q_slice, k_slice, v_slice, L_b, scale * 2)


def _heads_transposed(h, W1, b1, Wout):
    return O.medusa_heads(h, np.swapaxes(W1, 1, 2), b1, Wout)


def _heads_no_residual(h, W1, b1, Wout):
    u, _ = O.medusa_heads(h, W1, b1, Wout)
    u = u - np.asarray(h)[:, None, :]
    return u, np.einsum("bkd,kvd->bkv", u, Wout)


def _topk_high_id(z, k):
    ids, vals = O.topk_desc(z[..., ::-1], k)
    return z.shape[-1] - 1 - ids, vals


def _stats_log2(logits_b, temperature, eps, alpha):
    st = O.node_statistics(logits_b, temperature, eps, alpha)
    if st["entropy"] is not None:
        st["entropy"] = st["entropy"] / math.log(2)
        st["threshold"] = np.minimum(eps, alpha * np.exp(-st["entropy"]))
    return st


def _gap_top_k_only(z, k, rel=1e-4):
    return O.topk_gap_ok(z, k - 1, rel)     # looks at the k largest values, not k+1


def _gap_rel_smaller(z, k, rel=1e-4):
    flat = np.asarray(z, dtype=np.float64).reshape(-1, z.shape[-1])
    for r in range(flat.shape[0]):
        top = np.sort(flat[r])[::-1][:k + 1]
        for j in range(len(top) - 1):
            if abs(top[j] - top[j + 1]) < rel * min(abs(top[j]), abs(top[j + 1])):
                return False
    return True


def _margin_rel_smaller(tree, logits, candidates, temperature, eps, alpha, rel=1e-4):
    ret = tree["retrieve"]
    for b in range(logits.shape[0]):
        st = O.node_statistics(logits[b], temperature, eps, alpha)
        for p in range(tree["P"]):
            for j in range(1, tree["D"] + 1):
                if ret[p, j] < 0:
                    break
                pr = st["prob"][ret[p, j - 1], int(candidates[b, p, j])]
                th = st["threshold"][ret[p, j - 1]]
                if abs(pr - th) < rel * min(pr, th):
                    return False
    return True


def _nucleus_inclusive(prob_row, top_p):
    prob_row = np.asarray(prob_row, dtype=np.float64)
    order = np.lexsort((np.arange(prob_row.shape[0]), -prob_row))
    before = np.concatenate([[0.0], np.cumsum(prob_row[order])[:-1]])
    mask = np.zeros(prob_row.shape[0], dtype=bool)
    mask[order] = before <= top_p                # keeps one token too many at an exact boundary
    return mask


def _draw_by_probability(weights, u):
    w = np.asarray(weights, dtype=np.float64)
    order = np.argsort(-w, kind="stable")         # walks the CDF in probability order, not id order
    c = np.cumsum(w[order])
    return int(order[np.searchsorted(c, u * c[-1], side="right")])


def _tables_bad_index(choices, K, topk):
    tr = O.tree_tables(choices, K, topk)
    tr = dict(tr)
    tr["tree_indices"] = np.array([0] + [1 + (len(c) - 1) * topk + c[0] for c in tr["nodes"][1:]])
    return tr


MUTANTS = {
    "attention without self": (dict(tree_attention_slice=_attn_no_self),
                               [lambda M: check_attention_paths(M, WORKED, 2, 2)]),
    "attention sees the whole tree": (dict(tree_attention_slice=_attn_all_tree),
                                      [lambda M: check_attention_paths(M, WORKED, 2, 2)]),
    "attention scale": (dict(tree_attention_slice=_attn_bad_scale), [check_chain_and_decode]),
    "W1 transposed": (dict(medusa_heads=_heads_transposed), [check_heads_bruteforce]),
    "no residual": (dict(medusa_heads=_heads_no_residual), [check_heads_bruteforce]),
    "top-k ties by higher id": (dict(topk_desc=_topk_high_id), [check_topk]),
    "entropy in bits": (dict(node_statistics=_stats_log2), [check_typical_closed_forms]),
    "tree index from first rank": (dict(tree_tables=_tables_bad_index),
                                   [check_worked_example, check_tree_tables_random]),
    "gap guard over the top k only": (dict(topk_gap_ok=_gap_top_k_only), [check_topk_gap_guard]),
    "gap guard relative to the smaller value": (dict(topk_gap_ok=_gap_rel_smaller), [check_topk_gap_guard]),
    "margin guard relative to the smaller value": (dict(typical_margin_ok=_margin_rel_smaller),
                                                   [check_typical_margin_guard]),
    "nucleus keeps the token at the boundary": (dict(nucleus_mask=_nucleus_inclusive),
                                                [check_nucleus_mask, lambda M: check_nucleus_posterior(M, 0)]),
    "draw in probability order": (dict(sample_index=_draw_by_probability),
                                  [check_sample_index, lambda M: check_nucleus_posterior(M, 1)]),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutants_are_caught(name):
    over, checks = MUTANTS[name]
    M = _Mutant(**over)
    caught = False
    for chk in checks:
        try:
            chk(M)
        except AssertionError:
            caught = True
    assert caught, f"planted mistake '{name}' passed every pin"
