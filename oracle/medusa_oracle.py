"""Medusa verification step: the fp64 CPU oracle.

TEST INFRASTRUCTURE ONLY.  This module is the slow, plain definition that the
CUDA library is checked against.  Only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import it; the library itself
never does, and it shares no code with ``speculative_decoding_heads_b200``.

Every step is the direct definition, in float64, with numpy for dot
products and sorting and plain Python loops where the method is a loop.
Inputs are the exact values the GPU receives (bf16 / fp32 widened exactly).

Sources (page title, then section):
  [P3] "Medusa API参考：核心函数与类详解" -- sections MedusaConfig (head count and
       depth), MedusaModelABC (medusa_head = residual blocks + linear;
       medusa_generate defaults posterior_threshold=0.09, posterior_alpha=0.3),
       and "核心功能函数" (generate_candidates with tree_indices /
       retrieve_indices; tree_decoding with medusa_position_ids;
       evaluate_posterior).
  [P4] "Medusa — 让大模型自己同时猜好几个 token" -- sections "是什么" (K heads on
       the last hidden state, each a one-layer MLP with a residual; head k
       predicts position t+k+1), "核心要点" (per-head top-k assembled into a
       prefix tree verified under one attention mask; typical acceptance),
       "实践案例" case 1 (one round: guess, verify, keep the longest
       acceptable prefix from the root toward a leaf) and case 3 (the mask
       worked example P,A,B,X,Y,X,Y), "学到什么" (each step also yields the
       base model's own token).
  [P5] "基于 Medusa 头的投机解码架构" -- section "技术深度解析" (a chain draft
       that falls back on the first rejected token).

Readings where the pages are silent or disagree:
  * one residual block per head, u = h + SiLU(W1 h + b1), then a bias-free
    V x d projection;  Medusa head k (1-based) fills tree depth k;
  * the tree is a set of rank tuples; node (r1..rj) takes head j's
    rank-rj token; BFS layout sorts by (length, lexicographic);
  * the mask lets a tree node see the whole cached prefix, its strict
    ancestors and itself;  scale 1/sqrt(hd);
  * greedy accepts a child whose token is the argmax of its parent's base
    logits; typical accepts it when its tempered probability is strictly
    above min(eps, alpha * exp(-H)), H the natural-log entropy of the same
    tempered distribution;  ties: top-k by (value desc, id asc), argmax by
    lowest id, best path by lowest path index;  the next token is the argmax
    at the last accepted node;
  * the API's sampling='nucleus' with top_p (default 0.8) accepts a child
    whose token lies in the top_p nucleus of the parent's tempered
    distribution (the typical rule's form, with nucleus membership in place
    of the threshold);  given one caller-drawn uniform u per sequence, the
    next token is drawn instead, by inverse CDF in token-id order, from the
    last accepted node's tempered distribution (typical) or its nucleus;
  * after acceptance the a+1 accepted nodes' K/V rows move to prefix
    positions L_b..L_b+a and the sequence grows by a+1.
"""

from __future__ import annotations

import itertools
import math
from typing import Dict, List, Sequence, Tuple

import numpy as np

# ----------------------------------------------------------------------------
# Candidate tree  [P3 core functions: tree_indices, retrieve_indices,
#                  medusa_position_ids; P4 key points, case 3]
# ----------------------------------------------------------------------------


def ranksum_choices(K: int, topk: int, n_nodes: int) -> List[Tuple[int, ...]]:
    """The first ``n_nodes`` rank tuples in order of (rank sum, length, lexicographic).

    All tuples of length 1..K with entries in [0, topk) are listed and sorted;
    the first n_nodes are kept.  A tuple's parent has no larger rank sum and
    is shorter, so it sorts earlier: every prefix of this order is a
    prefix-closed tree.
    """
    allt = []
    for length in range(1, K + 1):
        allt.extend(itertools.product(range(topk), repeat=length))
    allt.sort(key=lambda t: (sum(t), len(t), t))
    if n_nodes > len(allt):
        raise ValueError("more nodes requested than tuples exist")
    return [tuple(t) for t in allt[:n_nodes]]


def tree_tables(choices: Sequence[Sequence[int]], K: int, topk: int) -> Dict[str, np.ndarray]:
    """Index tables of the candidate tree given as rank tuples.

    Node 0 is the root (the base model's own token); nodes 1..N are the
    tuples sorted by (length, lexicographic).  Returns
      nodes        list of tuples, nodes[0] = ()
      depth[T]     tuple length
      parent[T]    index of the tuple without its last rank (-1 for root)
      tree_indices[T]  index into [root, head1 top-k, ..., headK top-k]
      retrieve[P, D+1] node indices along each root-to-leaf path (pad -1),
                   paths ordered by their leaf's index
      anc[T, T]    bool, anc[i, j] = node j is node i or one of its ancestors
    """
    nodes = sorted({tuple(int(r) for r in c) for c in choices}, key=lambda c: (len(c), c))
    if len(nodes) != len(choices):
        raise ValueError("duplicate choices")
    for c in nodes:
        if not 1 <= len(c) <= K or any(not 0 <= r < topk for r in c):
            raise ValueError(f"choice {c} outside K={K}, topk={topk}")
    nodes = [()] + nodes
    index = {c: i for i, c in enumerate(nodes)}
    for c in nodes[1:]:
        if c[:-1] not in index:
            raise ValueError(f"choice {c} has no parent in the tree")
    T = len(nodes)
    depth = np.array([len(c) for c in nodes], dtype=np.int64)
    parent = np.array([-1] + [index[c[:-1]] for c in nodes[1:]], dtype=np.int64)
    tree_indices = np.array([0] + [1 + (len(c) - 1) * topk + c[-1] for c in nodes[1:]],
                            dtype=np.int64)
    has_child = np.zeros(T, dtype=bool)
    for i in range(1, T):
        has_child[parent[i]] = True
    leaves = [i for i in range(T) if not has_child[i]]
    D = int(depth.max())
    retrieve = np.full((len(leaves), D + 1), -1, dtype=np.int64)
    for p, leaf in enumerate(leaves):
        c = nodes[leaf]
        for j in range(len(c) + 1):
            retrieve[p, j] = index[c[:j]]
    anc = np.zeros((T, T), dtype=bool)
    for i, ci in enumerate(nodes):
        for j, cj in enumerate(nodes):
            anc[i, j] = len(cj) <= len(ci) and ci[:len(cj)] == cj
    return dict(nodes=nodes, depth=depth, parent=parent, tree_indices=tree_indices,
                retrieve=retrieve, anc=anc, T=T, P=len(leaves), D=D, K=K, topk=topk)


# ----------------------------------------------------------------------------
# S1-S3: heads and per-head top-k  [P3 MedusaModelABC: residual block + linear;
#        P4 "是什么": one-layer MLP with residual on the last hidden state]
# ----------------------------------------------------------------------------


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def medusa_head_one(h: np.ndarray, W1: np.ndarray, b1: np.ndarray, Wout: np.ndarray):
    """One head on every sequence: u = h + SiLU(W1 h + b1), z = Wout u.

    h [B, d]; W1 [d, d] (out x in); b1 [d]; Wout [V, d].  Returns u [B, d],
    z [B, V], all float64.
    """
    h = np.asarray(h, dtype=np.float64)
    u = h + silu(h @ np.asarray(W1, dtype=np.float64).T + np.asarray(b1, dtype=np.float64))
    z = u @ np.asarray(Wout, dtype=np.float64).T
    return u, z


def medusa_heads(h, W1, b1, Wout):
    """All K heads: u [B, K, d] and head logits z [B, K, V] (float64)."""
    K = W1.shape[0]
    us, zs = [], []
    for k in range(K):
        u, z = medusa_head_one(h, W1[k], b1[k], Wout[k])
        us.append(u)
        zs.append(z)
    return np.stack(us, axis=1), np.stack(zs, axis=1)


def topk_desc(z: np.ndarray, k: int):
    """The k largest entries of each row of z, by value descending then id ascending."""
    z = np.asarray(z, dtype=np.float64)
    lead = z.shape[:-1]
    flat = z.reshape(-1, z.shape[-1])
    ids = np.empty((flat.shape[0], k), dtype=np.int64)
    vals = np.empty((flat.shape[0], k), dtype=np.float64)
    col = np.arange(flat.shape[1])
    for r in range(flat.shape[0]):
        order = np.lexsort((col, -flat[r]))[:k]
        ids[r] = order
        vals[r] = flat[r, order]
    return ids.reshape(lead + (k,)), vals.reshape(lead + (k,))


# ----------------------------------------------------------------------------
# S4: candidate assembly  [P3 generate_candidates: tree_indices gather,
#     retrieve_indices paths; tree_decoding: medusa_position_ids]
# ----------------------------------------------------------------------------


def build_tree(tree, root_tokens, topk_ids, seq_lens):
    """tree_tokens [B, T], candidates [B, P, D+1] (pad -1), position_ids [B, T]."""
    root_tokens = np.asarray(root_tokens, dtype=np.int64)
    topk_ids = np.asarray(topk_ids, dtype=np.int64)
    B = root_tokens.shape[0]
    T, P, D = tree["T"], tree["P"], tree["D"]
    tree_tokens = np.empty((B, T), dtype=np.int64)
    candidates = np.full((B, P, D + 1), -1, dtype=np.int64)
    position_ids = np.empty((B, T), dtype=np.int64)
    for b in range(B):
        flat = [int(root_tokens[b])] + [int(t) for t in topk_ids[b].reshape(-1)]
        for i in range(T):
            tree_tokens[b, i] = flat[tree["tree_indices"][i]]
            position_ids[b, i] = int(seq_lens[b]) + int(tree["depth"][i])
        for p in range(P):
            for j in range(D + 1):
                n = tree["retrieve"][p, j]
                if n >= 0:
                    candidates[b, p, j] = tree_tokens[b, n]
    return tree_tokens, candidates, position_ids


# ----------------------------------------------------------------------------
# S5: tree attention  [P4 key points: one forward under a tree mask;
#     case 3: "X after A" sees only P and A]
# ----------------------------------------------------------------------------


def tree_attention_slice(tree, q_slice, k_slice, v_slice, L_b: int, scale: float):
    """Attention of the T tree queries of one (layer, sequence, head).

    q_slice [T, hd]; k_slice, v_slice [>= L_b+T, hd] with the tree's own
    K/V at rows L_b..L_b+T-1.  Node i attends to rows 0..L_b-1 (the cached
    prefix) and to L_b+j for every j that is i or an ancestor of i.  A plain
    softmax over exactly that set, max subtracted.  Returns O [T, hd].
    """
    T = tree["T"]
    q = np.asarray(q_slice, dtype=np.float64)
    kk = np.asarray(k_slice, dtype=np.float64)
    vv = np.asarray(v_slice, dtype=np.float64)
    out = np.empty((T, q.shape[1]), dtype=np.float64)
    for i in range(T):
        rows = list(range(L_b)) + [L_b + j for j in range(T) if tree["anc"][i, j]]
        s = (kk[rows] @ q[i]) * scale
        w = np.exp(s - s.max())
        w /= w.sum()
        out[i] = w @ vv[rows]
    return out


def tree_attention(tree, q, k_cache, v_cache, seq_lens, scale):
    """All slices.  q [layers, B, T, H, hd]; caches [layers, B, H, Lcap, hd]."""
    layers, B, T, H, hd = q.shape
    out = np.empty((layers, B, T, H, hd), dtype=np.float64)
    for l in range(layers):
        for b in range(B):
            for e in range(H):
                out[l, b, :, e, :] = tree_attention_slice(
                    tree, q[l, b, :, e, :], k_cache[l, b, e], v_cache[l, b, e],
                    int(seq_lens[b]), scale)
    return out


# S5 split along the cached prefix (several ranks share one slice's keys).
# The pages have no counterpart: this is the library's multi-GPU option.  Its
# definition is the restriction of tree_attention_slice to a key subset, and
# putting the parts back together is the log-sum-exp identity.


def attention_window(G: int, r: int, L_b: int):
    """Prefix rows [lo, hi) of rank r of G: lo = floor(L_b r / G), hi = floor(L_b (r+1) / G).
    The tree's own rows belong to the last rank only."""
    return (L_b * r) // G, (L_b * (r + 1)) // G


def tree_attention_window_slice(tree, q_slice, k_slice, v_slice, L_b: int, scale: float,
                                lo: int, hi: int, with_tree: bool):
    """Attention of the T tree queries over prefix rows lo..hi-1 and, when with_tree, the tree
    rows each node may see (itself and its ancestors).  Returns (O [T, hd] normalised over that
    set, lse [T] = ln sum exp(scale q.k) over it); a query with no key gets O = 0, lse = -inf."""
    T = tree["T"]
    q = np.asarray(q_slice, dtype=np.float64)
    kk = np.asarray(k_slice, dtype=np.float64)
    vv = np.asarray(v_slice, dtype=np.float64)
    out = np.zeros((T, q.shape[1]), dtype=np.float64)
    lse = np.full(T, -np.inf)
    for i in range(T):
        rows = list(range(lo, hi))
        if with_tree:
            rows += [L_b + j for j in range(T) if tree["anc"][i, j]]
        if not rows:
            continue
        s = (kk[rows] @ q[i]) * scale
        m = s.max()
        w = np.exp(s - m)
        lse[i] = m + np.log(w.sum())
        out[i] = (w / w.sum()) @ vv[rows]
    return out, lse


def combine_partials(outs, lses):
    """Attention over the union of G disjoint key sets from each set's (O_r, lse_r):
    lse = ln sum_r exp(lse_r) and O = sum_r exp(lse_r - lse) O_r.
    outs [G, ..., hd], lses [G, ...]; entries with lse_r = -inf contribute nothing."""
    outs = np.asarray(outs, dtype=np.float64)
    lses = np.asarray(lses, dtype=np.float64)
    m = lses.max(axis=0)
    safe = np.where(np.isfinite(m), m, 0.0)
    w = np.exp(lses - safe)                      # exp(-inf) = 0
    tot = w.sum(axis=0)
    with np.errstate(divide="ignore"):
        lse = np.where(tot > 0, safe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    wn = np.where(tot > 0, w / np.where(tot > 0, tot, 1.0), 0.0)
    return (wn[..., None] * outs).sum(axis=0), lse


# ----------------------------------------------------------------------------
# S6: posterior  [P3 evaluate_posterior (posterior_threshold, posterior_alpha);
#     P4 key points (typical acceptance), case 1 step 4 (longest acceptable
#     prefix from the root toward a leaf), lessons (the step's own token)]
# ----------------------------------------------------------------------------


def node_statistics(logits_b: np.ndarray, temperature: float, eps: float, alpha: float):
    """Per tree node of one sequence: argmax, tempered probabilities, entropy, threshold.

    logits_b [T, V].  p = softmax(z / temperature); H = -sum p ln p (terms
    with p = 0 contribute 0); threshold = min(eps, alpha * exp(-H)).
    """
    z = np.asarray(logits_b, dtype=np.float64)
    argmax = np.argmax(z, axis=1)
    prob = ent = thr = None
    if temperature is not None and temperature > 0:
        y = z / temperature
        y = y - y.max(axis=1, keepdims=True)
        e = np.exp(y)
        prob = e / e.sum(axis=1, keepdims=True)
        with np.errstate(divide="ignore", invalid="ignore"):
            plogp = np.where(prob > 0, prob * np.log(prob), 0.0)
        ent = -plogp.sum(axis=1)
        thr = np.minimum(eps, alpha * np.exp(-ent))
    return dict(argmax=argmax, prob=prob, entropy=ent, threshold=thr)


def nucleus_mask(prob_row: np.ndarray, top_p: float) -> np.ndarray:
    """The top-p nucleus of one distribution, as a boolean mask over the vocabulary.

    Tokens are taken in order of probability (descending, lower id first on
    equal values) for as long as the mass of the tokens taken before them is
    below top_p: the shortest such prefix whose mass reaches top_p.
    """
    prob_row = np.asarray(prob_row, dtype=np.float64)
    order = np.lexsort((np.arange(prob_row.shape[0]), -prob_row))
    before = np.concatenate([[0.0], np.cumsum(prob_row[order])[:-1]])
    mask = np.zeros(prob_row.shape[0], dtype=bool)
    mask[order] = before < top_p
    return mask


def sample_index(weights: np.ndarray, u: float) -> int:
    """An inverse-CDF draw in token-id order: the first v whose cumulative
    weight exceeds u * (total weight), u in [0, 1).  Zero weights are never drawn."""
    c = np.cumsum(np.asarray(weights, dtype=np.float64))
    return int(np.searchsorted(c, u * c[-1], side="right"))


def evaluate_posterior(tree, logits, candidates, mode: str, temperature=0.0,
                       eps=0.09, alpha=0.3, top_p=0.8, uniforms=None):
    """Best path, accept length, accepted tokens and next token per sequence.

    logits [B, T, V] base-model logits at each tree node; candidates
    [B, P, D+1] from ``build_tree``.  For path p and depth j the child token
    candidates[b, p, j] is accepted when (greedy) it equals the argmax of its
    parent's logits, (typical) its tempered probability at the parent is
    strictly above the parent's threshold, or (nucleus) it lies in the top_p
    nucleus of the parent's tempered distribution.  acc_p counts the leading
    accepted depths; the best path is the lowest p with the largest acc_p;
    a = acc_best.  accepted_tokens = candidates[b, best, 0..a] padded with -1.
    next_token is taken at node n = retrieve[best, a]: the argmax of its logits
    when ``uniforms`` is None or in greedy mode; otherwise an inverse-CDF draw
    with uniforms[b] from n's tempered distribution (typical) or from that
    distribution restricted to its nucleus (nucleus).
    """
    B, T, V = logits.shape
    P, D = tree["P"], tree["D"]
    ret = tree["retrieve"]
    best = np.zeros(B, dtype=np.int64)
    alen = np.zeros(B, dtype=np.int64)
    accepted = np.full((B, D + 1), -1, dtype=np.int64)
    nxt = np.zeros(B, dtype=np.int64)
    accs = np.zeros((B, P), dtype=np.int64)
    if mode not in ("greedy", "typical", "nucleus"):
        raise ValueError(mode)
    for b in range(B):
        st = node_statistics(logits[b], temperature if mode != "greedy" else None, eps, alpha)
        nucleus = {}
        for p in range(P):
            acc = 0
            for j in range(1, D + 1):
                node = ret[p, j]
                if node < 0:
                    break
                par = ret[p, j - 1]
                tok = int(candidates[b, p, j])
                if mode == "greedy":
                    ok = tok == st["argmax"][par]
                elif mode == "typical":
                    ok = st["prob"][par, tok] > st["threshold"][par]
                else:
                    if par not in nucleus:
                        nucleus[par] = nucleus_mask(st["prob"][par], top_p)
                    ok = bool(nucleus[par][tok])
                if not ok:
                    break
                acc += 1
            accs[b, p] = acc
        bp = int(np.argmax(accs[b]))          # first maximum = lowest path index
        best[b] = bp
        alen[b] = accs[b, bp]
        accepted[b, :alen[b] + 1] = candidates[b, bp, :alen[b] + 1]
        last = ret[bp, alen[b]]
        if uniforms is None or mode == "greedy":
            nxt[b] = st["argmax"][last]
        else:
            w = st["prob"][last]
            if mode == "nucleus":
                w = np.where(nucleus_mask(w, top_p), w, 0.0)
            nxt[b] = sample_index(w, float(uniforms[b]))
    return dict(best_path=best, accept_len=alen, accepted_tokens=accepted,
                next_token=nxt, path_accept=accs)


# ----------------------------------------------------------------------------
# S7: keep the accepted prefix's K/V  [P4 case 1 step 4; P5 technical
#     analysis: a rejected draft falls back]
# ----------------------------------------------------------------------------


def accept_kv(tree, k_cache, v_cache, seq_lens, best_path, accept_len):
    """New caches and lengths after acceptance (inputs are not modified).

    For every layer, sequence b and head: row L_b + j of the new cache is the
    old row L_b + retrieve[best_b, j] for j = 0..a_b; all other rows are kept.
    The new length is L_b + a_b + 1.
    """
    k_new = np.array(k_cache, copy=True)
    v_new = np.array(v_cache, copy=True)
    lens = np.array(seq_lens, dtype=np.int64, copy=True)
    B = k_cache.shape[1]
    for b in range(B):
        L = int(seq_lens[b])
        a = int(accept_len[b])
        src = [L + int(tree["retrieve"][best_path[b], j]) for j in range(a + 1)]
        for j, s in enumerate(src):
            k_new[:, b, :, L + j, :] = k_cache[:, b, :, s, :]
            v_new[:, b, :, L + j, :] = v_cache[:, b, :, s, :]
        lens[b] = L + a + 1
    return k_new, v_new, lens


# ----------------------------------------------------------------------------
# Margin checks used to choose sub-seeds (the decisions both sides take must
# not sit within 1e-4 relative of a boundary).
# ----------------------------------------------------------------------------


def topk_gap_ok(z: np.ndarray, k: int, rel: float = 1e-4) -> bool:
    """True when every gap among the k+1 largest values of each row is >= rel."""
    flat = np.asarray(z, dtype=np.float64).reshape(-1, z.shape[-1])
    for r in range(flat.shape[0]):
        top = np.sort(flat[r])[::-1][:k + 1]
        for j in range(len(top) - 1):
            if abs(top[j] - top[j + 1]) < rel * max(abs(top[j]), abs(top[j + 1])):
                return False
    return True


def typical_margin_ok(tree, logits, candidates, temperature, eps, alpha,
                      rel: float = 1e-4) -> bool:
    """True when every tree edge's |p - threshold| is >= rel * max(p, threshold)."""
    B = logits.shape[0]
    ret = tree["retrieve"]
    for b in range(B):
        st = node_statistics(logits[b], temperature, eps, alpha)
        for p in range(tree["P"]):
            for j in range(1, tree["D"] + 1):
                if ret[p, j] < 0:
                    break
                par = ret[p, j - 1]
                pr = st["prob"][par, int(candidates[b, p, j])]
                th = st["threshold"][par]
                if abs(pr - th) < rel * max(pr, th):
                    return False
    return True


# The nucleus decisions are comparisons of sums of tempered probabilities
# with top_p.  Summed in fp32 over at most 65536 tokens, as the GPU does, such
# a sum is off by at most a few 1e-6 of the total mass, so these guards keep
# every such decision at least 1e-5 of the total mass away from its boundary.
NUCLEUS_REL = 1e-5


def nucleus_margin_ok(tree, logits, candidates, temperature, top_p, rel: float = NUCLEUS_REL) -> bool:
    """True when, on every tree edge, the tempered mass of the tokens ranking
    before the child's token (larger probability, or equal and lower id) is at
    least rel away from top_p, so its nucleus membership holds under any
    summation order.  logits [B, T, V]; candidates [B, P, D+1]."""
    ret = tree["retrieve"]
    for b in range(logits.shape[0]):
        st = node_statistics(logits[b], temperature, 0.0, 0.0)
        for p in range(tree["P"]):
            for j in range(1, tree["D"] + 1):
                if ret[p, j] < 0:
                    break
                pr = st["prob"][ret[p, j - 1]]
                tok = int(candidates[b, p, j])
                ids = np.arange(pr.shape[0])
                before = pr[(pr > pr[tok]) | ((pr == pr[tok]) & (ids < tok))].sum()
                if abs(before - top_p) < rel:
                    return False
    return True


def nucleus_cut_ok(prob_row, top_p, rel: float = NUCLEUS_REL) -> bool:
    """True when one distribution's nucleus boundary is clear: top_p is at
    least rel from the mass before its last member and from the mass through
    it, and that member's probability is above the next token's by at least
    1e-6 relative (so no rounding can reorder the two)."""
    pr = np.asarray(prob_row, dtype=np.float64)
    order = np.lexsort((np.arange(pr.shape[0]), -pr))
    cum = np.cumsum(pr[order])
    m = min(int(np.searchsorted(cum, top_p, side="left")), pr.shape[0] - 1)   # first prefix reaching top_p
    before = cum[m - 1] if m > 0 else 0.0
    if top_p - before < rel or cum[m] - top_p < rel:
        return False
    return not (m + 1 < pr.shape[0] and pr[order[m]] - pr[order[m + 1]] < 1e-6 * pr[order[m]])


def sample_margin_ok(weights, u: float, rel: float = NUCLEUS_REL) -> bool:
    """True when u * total lies at least rel * total inside the drawn token's CDF interval."""
    c = np.cumsum(np.asarray(weights, dtype=np.float64))
    x = u * c[-1]
    v = int(np.searchsorted(c, x, side="right"))
    lo = c[v - 1] if v > 0 else 0.0
    return x - lo >= rel * c[-1] and c[v] - x >= rel * c[-1]


def attention_scale(hd: int) -> float:
    return 1.0 / math.sqrt(hd)
