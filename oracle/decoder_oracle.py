"""The base model's forward over the tree tokens: the fp64 CPU oracle.

TEST INFRASTRUCTURE ONLY, like medusa_oracle: only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import it, and it shares no code with ``speculative_decoding_heads_b200``.

Sources (page title, then section):
  [P3] "Medusa API参考：核心函数与类详解" -- "核心功能函数": tree_decoding runs
       the base model once over every tree token, at the tree's position ids
       (prefix length + depth), under the tree mask, against the cached K/V;
       its output logits feed evaluate_posterior.
  [P4] "Medusa — 让大模型自己同时猜好几个 token" -- "实践案例" case 1 step 3 (one
       forward verifies all candidates at once).
  [P5] "基于 Medusa 头的投机解码架构" -- "性能基准测试": the base models are
       Vicuna-7B/13B/33B.

The pages name the base model but not its layers.  The plainest reading is
the Vicuna (LLaMA) decoder layer, restated here from its published
definition: pre-norm RMSNorm (Zhang & Sennrich 2019), multi-head attention
whose queries and keys are rotated by RoPE (Su et al. 2021, the half-split
pairing LLaMA uses, base 10000), and a SwiGLU feed-forward (Shazeer 2020),
each added back to the residual stream; a final RMSNorm and a bias-free LM
head give the logits.  Attention over the cache and the tree is the S5
definition of medusa_oracle (tree_attention_slice).  Every function is the
direct definition in float64.
"""

import numpy as np

from oracle import medusa_oracle as O

ROPE_BASE = 10000.0
RMS_EPS = 1e-6


def rms_norm(x: np.ndarray, w: np.ndarray, eps: float = RMS_EPS) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * w over the last axis."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * np.asarray(w, dtype=np.float64)


def rope(x: np.ndarray, pos, base: float = ROPE_BASE) -> np.ndarray:
    """Rotary position embedding of vectors x [..., n, hd] at integer positions pos [n].

    Pair i (i < hd/2) is (x[i], x[i + hd/2]), rotated by the angle pos * base^(-2i/hd)."""
    x = np.asarray(x, dtype=np.float64)
    hd = x.shape[-1]
    half = hd // 2
    inv = base ** (-np.arange(half, dtype=np.float64) * 2.0 / hd)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]          # [n, hd/2]
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def swiglu_mlp(h: np.ndarray, W_gate: np.ndarray, W_up: np.ndarray, W_down: np.ndarray) -> np.ndarray:
    """W_down (SiLU(W_gate h) * (W_up h)); weights out x in."""
    h = np.asarray(h, dtype=np.float64)
    g = h @ np.asarray(W_gate, dtype=np.float64).T
    u = h @ np.asarray(W_up, dtype=np.float64).T
    return (O.silu(g) * u) @ np.asarray(W_down, dtype=np.float64).T


def decoder_layer(tree, x, layer, k_cache, v_cache, L_b: int, H: int):
    """One decoder layer over the T tree tokens of one sequence.

    x [T, D] residual stream of the tree tokens; layer: dict with attn_norm [D], Wq, Wk, Wv, Wo
    [D, D], mlp_norm [D], W_gate, W_up [F, D], W_down [D, F]; k_cache, v_cache [H, >= L_b+T, hd]
    hold this layer's post-RoPE keys and values of the prefix in rows 0..L_b-1.  The tree tokens'
    own keys and values are written at rows L_b..L_b+T-1 (copies are returned, the inputs are not
    modified).  Node i sits at position L_b + depth(i).  Returns (x_out [T, D], k_cache, v_cache).
    """
    x = np.asarray(x, dtype=np.float64)
    T, D = x.shape
    hd = D // H
    pos = L_b + np.asarray(tree["depth"])
    kc = np.array(k_cache, dtype=np.float64)
    vc = np.array(v_cache, dtype=np.float64)
    h = rms_norm(x, layer["attn_norm"])
    q = (h @ np.asarray(layer["Wq"], dtype=np.float64).T).reshape(T, H, hd).transpose(1, 0, 2)
    k = (h @ np.asarray(layer["Wk"], dtype=np.float64).T).reshape(T, H, hd).transpose(1, 0, 2)
    v = (h @ np.asarray(layer["Wv"], dtype=np.float64).T).reshape(T, H, hd).transpose(1, 0, 2)
    q = rope(q, pos)
    k = rope(k, pos)
    kc[:, L_b:L_b + T, :] = k
    vc[:, L_b:L_b + T, :] = v
    scale = O.attention_scale(hd)
    att = np.stack([O.tree_attention_slice(tree, q[e], kc[e], vc[e], L_b, scale) for e in range(H)], axis=1)
    x = x + att.reshape(T, D) @ np.asarray(layer["Wo"], dtype=np.float64).T
    x = x + swiglu_mlp(rms_norm(x, layer["mlp_norm"]), layer["W_gate"], layer["W_up"], layer["W_down"])
    return x, kc, vc


def tree_forward(tree, tokens, embed, layers, final_norm, lm_head, k_caches, v_caches, L_b: int, H: int):
    """The whole base-model forward of one sequence's tree tokens: embedding, every decoder layer,
    the final RMSNorm and the LM head.  tokens [T] (tree_tokens of the sequence); embed [V, D];
    k_caches / v_caches: per layer [H, >= L_b+T, hd].  Returns (logits [T, V], hidden [T, D],
    updated caches) -- the logits are the base logits evaluate_posterior reads."""
    x = np.asarray(embed, dtype=np.float64)[np.asarray(tokens)]
    kcs, vcs = [], []
    for li, layer in enumerate(layers):
        x, kc, vc = decoder_layer(tree, x, layer, k_caches[li], v_caches[li], L_b, H)
        kcs.append(kc)
        vcs.append(vc)
    hid = rms_norm(x, final_norm)
    return hid @ np.asarray(lm_head, dtype=np.float64).T, x, kcs, vcs


# ----------------------------------------------------------------------------
# The generation loop  [P3 MedusaModelABC.medusa_generate: repeat the step;
#     P4 实践案例 case 1 (guess, verify, keep the accepted prefix) and 学到什么
#     (each step also yields the base model's own token)]
# ----------------------------------------------------------------------------


def chain_tree(n: int):
    """The tree of n tokens in a row (node i at depth i, seeing nodes 0..i): a causal forward."""
    return {"T": n, "depth": np.arange(n), "anc": np.tril(np.ones((n, n), dtype=bool))}


def _empty_caches(model, Lcap):
    D = model["embed"].shape[1]
    H = model["H"]
    shape = (H, Lcap, D // H)
    return [np.zeros(shape) for _ in model["layers"]], [np.zeros(shape) for _ in model["layers"]]


def _forward(model, tree, tokens, kcs, vcs, L):
    return tree_forward(tree, tokens, model["embed"], model["layers"], model["final_norm"], model["lm_head"],
                        kcs, vcs, L, model["H"])


def greedy_decode(model, prompt, n_new: int, Lcap: int):
    """Plain greedy decoding with the base model: n_new tokens after the prompt, one forward each."""
    kcs, vcs = _empty_caches(model, Lcap)
    logits, _, kcs, vcs = _forward(model, chain_tree(len(prompt)), np.asarray(prompt), kcs, vcs, 0)
    L = len(prompt)
    out = [int(np.argmax(logits[-1]))]
    while len(out) < n_new:
        logits, _, kcs, vcs = _forward(model, chain_tree(1), np.asarray(out[-1:]), kcs, vcs, L)
        L += 1
        out.append(int(np.argmax(logits[-1])))
    return out


def medusa_generate(model, heads, choices, K: int, topk: int, prompt, n_new: int, Lcap: int, mode: str = "greedy",
                    temperature: float = 0.0, eps: float = 0.09, alpha: float = 0.3, top_p: float = 0.8,
                    uniforms=None, trace=None):
    """Medusa decoding of one sequence, built from the step's oracle functions.

    After the prompt's forward, the base model's arg-max is the first root.  Each step: the heads
    on the last accepted token's final hidden state (after the final RMSNorm), their top-k, the
    candidate tree rooted at the base model's next token, the base model's forward over the tree at
    the cache length (S5 inside it), acceptance in ``mode`` (greedy, typical or nucleus, as
    ``evaluate_posterior``; with ``uniforms[s]`` the next token of step s is drawn), and the KV
    compaction.  The step emits the root and the a accepted tokens.  ``trace``, when a list, gets
    (logits [T, V], candidates [P, D+1], best path, accept length, head logits [K, V]) of every step.
    Returns (tokens [n_new], accept length of every step)."""
    tr = O.tree_tables(choices, K, topk)
    kcs, vcs = _empty_caches(model, Lcap)
    logits, x, kcs, vcs = _forward(model, chain_tree(len(prompt)), np.asarray(prompt), kcs, vcs, 0)
    L = len(prompt)
    h = rms_norm(x[-1:], model["final_norm"])
    root = int(np.argmax(logits[-1]))
    out, accepts = [], []
    while len(out) < n_new:
        if L + tr["T"] > Lcap:
            raise ValueError("cache capacity too small for the next tree")
        _, z = O.medusa_heads(h, heads["W1"], heads["b1"], heads["Wout"])
        ids, _ = O.topk_desc(z, topk)
        toks, cand, _ = O.build_tree(tr, [root], ids, [L])
        logits, x, kcs, vcs = _forward(model, tr, toks[0], kcs, vcs, L)
        u = None if uniforms is None else np.asarray([uniforms[len(accepts)]], dtype=np.float64)
        post = O.evaluate_posterior(tr, logits[None], cand, mode, temperature, eps, alpha, top_p, u)
        a, best = int(post["accept_len"][0]), int(post["best_path"][0])
        if trace is not None:
            trace.append((logits, cand[0], best, a, z[0]))
        k_new, v_new, _ = O.accept_kv(tr, np.stack(kcs)[:, None], np.stack(vcs)[:, None], [L], [best], [a])
        kcs = [k_new[l, 0] for l in range(len(kcs))]
        vcs = [v_new[l, 0] for l in range(len(vcs))]
        out.extend(int(t) for t in post["accepted_tokens"][0, :a + 1])
        node = int(tr["retrieve"][best, a])
        h = rms_norm(x[node:node + 1], model["final_norm"])
        root = int(post["next_token"][0])
        L += a + 1
        accepts.append(a)
    return out[:n_new], accepts


def medusa_generate_greedy(model, heads, choices, K: int, topk: int, prompt, n_new: int, Lcap: int):
    """Greedy Medusa decoding of one sequence (``medusa_generate`` in greedy mode).
    Returns (tokens [n_new], accept length of every step)."""
    return medusa_generate(model, heads, choices, K, topk, prompt, n_new, Lcap)
