"""Pins for the oracle of the base model's forward over the tree tokens.

The decisive pin: under the tree mask, every node's output equals an ordinary
causal forward over the cached prefix plus that node's root-to-leaf path at
positions L, L+1, ... -- the definition of verifying all candidates in one
forward.  The causal forward here is written separately, from torch's fp64
scaled-dot-product attention with a causal mask, so that a wrong mask, a
wrong position or a wrong cache row fails it.  Closed forms pin RMSNorm,
RoPE and the SwiGLU feed-forward.  The generation loop is pinned by
losslessness: greedy Medusa decoding emits the base model's greedy tokens."""

import numpy as np
import pytest
import torch

import oracle.decoder_oracle as D
import oracle.medusa_oracle as O

WORKED = [(0,), (1,), (0, 0), (0, 1), (1, 0), (1, 1)]


def _layer(rng, Dm, F, s=0.2):
    return {"attn_norm": 1.0 + 0.1 * rng.normal(size=Dm), "Wq": s * rng.normal(size=(Dm, Dm)),
            "Wk": s * rng.normal(size=(Dm, Dm)), "Wv": s * rng.normal(size=(Dm, Dm)),
            "Wo": s * rng.normal(size=(Dm, Dm)), "mlp_norm": 1.0 + 0.1 * rng.normal(size=Dm),
            "W_gate": s * rng.normal(size=(F, Dm)), "W_up": s * rng.normal(size=(F, Dm)),
            "W_down": s * rng.normal(size=(Dm, F))}


def _rope_ref(x, pos, base=D.ROPE_BASE):
    """RoPE as complex multiplication: pair (x[i], x[i+hd/2]) times exp(1j pos theta_i)."""
    hd = x.shape[-1]
    half = hd // 2
    theta = base ** (-np.arange(half) * 2.0 / hd)
    z = (x[..., :half] + 1j * x[..., half:]) * np.exp(1j * np.asarray(pos)[:, None] * theta[None, :])
    return np.concatenate([z.real, z.imag], axis=-1)


def _rms_ref(x, w):
    """RMSNorm by torch's own routine (eps 1e-6, as the pages' Vicuna bases use)."""
    t = torch.from_numpy(np.asarray(x, dtype=np.float64))
    return torch.nn.functional.rms_norm(t, (t.shape[-1],), weight=torch.from_numpy(np.asarray(w, np.float64)),
                                        eps=1e-6).numpy()


def _silu_ref(x):
    return torch.nn.functional.silu(torch.from_numpy(np.asarray(x, dtype=np.float64))).numpy()


def _causal_forward(tokens, embed, layers, k_caches, v_caches, L, H, final_norm=None, lm_head=None):
    """A plain causal decoder over a token sequence at positions L.. with a prefix cache, written
    without the oracle's helpers (torch's RMSNorm, SiLU and attention; RoPE as complex
    multiplication).  Returns the residual stream, and the logits when the head is given."""
    x = embed[np.asarray(tokens)].astype(np.float64)
    n, Dm = x.shape
    hd = Dm // H
    pos = L + np.arange(n)
    for li, ly in enumerate(layers):
        h = _rms_ref(x, ly["attn_norm"])
        q = _rope_ref((h @ ly["Wq"].T).reshape(n, H, hd).transpose(1, 0, 2), pos)
        k = _rope_ref((h @ ly["Wk"].T).reshape(n, H, hd).transpose(1, 0, 2), pos)
        v = (h @ ly["Wv"].T).reshape(n, H, hd).transpose(1, 0, 2)
        K = np.concatenate([k_caches[li][:, :L], k], axis=1)
        V = np.concatenate([v_caches[li][:, :L], v], axis=1)
        mask = torch.ones(n, L + n, dtype=torch.bool).tril(L)
        att = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None],
            attn_mask=mask[None, None])[0].numpy()
        x = x + att.transpose(1, 0, 2).reshape(n, Dm) @ ly["Wo"].T
        hm = _rms_ref(x, ly["mlp_norm"])
        x = x + (_silu_ref(hm @ ly["W_gate"].T) * (hm @ ly["W_up"].T)) @ ly["W_down"].T
    if lm_head is None:
        return x
    return x, _rms_ref(x, final_norm) @ np.asarray(lm_head).T


@pytest.mark.parametrize("choices,K,topk,L", [(WORKED, 2, 2, 9), (O.ranksum_choices(4, 3, 20), 4, 3, 17),
                                              (O.ranksum_choices(3, 2, 8), 3, 2, 0)])
def test_tree_forward_equals_causal_forward_along_every_path(choices, K, topk, L):
    rng = np.random.default_rng(L + len(choices))
    tr = O.tree_tables(choices, K, topk)
    T, Dm, F, H, Vv, nl = tr["T"], 32, 48, 4, 50, 2
    hd = Dm // H
    embed = rng.normal(size=(Vv, Dm))
    layers = [_layer(rng, Dm, F) for _ in range(nl)]
    tokens = rng.integers(0, Vv, size=T)
    kcs = [rng.normal(size=(H, L + T + 3, hd)) for _ in range(nl)]
    vcs = [rng.normal(size=(H, L + T + 3, hd)) for _ in range(nl)]
    final_norm, lm_head = 1.0 + 0.1 * rng.normal(size=Dm), rng.normal(size=(Vv, Dm))
    logits, hid, kc_out, _ = D.tree_forward(tr, tokens, embed, layers, final_norm, lm_head, kcs, vcs, L, H)
    for p in range(tr["P"]):
        path = [n for n in tr["retrieve"][p] if n >= 0]
        ref, ref_logits = _causal_forward(tokens[path], embed, layers, kcs, vcs, L, H, final_norm, lm_head)
        assert np.allclose(hid[path], ref, atol=1e-10, rtol=1e-10), p
        assert np.allclose(logits[path], ref_logits, atol=1e-9, rtol=1e-9), p
    # the prefix rows of the caches are untouched; the tree rows now hold the tree's keys
    for li in range(nl):
        assert np.array_equal(kc_out[li][:, :L], kcs[li][:, :L])
        assert not np.allclose(kc_out[li][:, L:L + T], kcs[li][:, L:L + T])
    assert logits.shape == (T, Vv)


def test_rms_norm_closed_forms():
    rng = np.random.default_rng(1)
    x = rng.normal(size=(5, 64))
    y = D.rms_norm(x, np.ones(64), eps=0.0)
    assert np.allclose(np.sqrt((y * y).mean(axis=-1)), 1.0, atol=1e-14)
    assert np.allclose(D.rms_norm(7.5 * x, np.ones(64), eps=0.0), y, atol=1e-14)
    w = rng.normal(size=64)
    assert np.allclose(D.rms_norm(x, w, eps=0.0), y * w, atol=1e-14)
    assert np.allclose(D.rms_norm(np.full((1, 4), 3.0), np.ones(4), eps=0.0), 1.0)


def test_rope_closed_forms():
    rng = np.random.default_rng(2)
    hd, n = 16, 7
    x = rng.normal(size=(n, hd))
    pos = np.arange(3, 3 + n)
    y = D.rope(x, pos)
    assert np.allclose(y, _rope_ref(x, pos), atol=1e-13)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), atol=1e-13)
    assert np.allclose(D.rope(x, np.zeros(n)), x, atol=0)
    # scores depend only on the position difference
    qv, kv = rng.normal(size=(1, hd)), rng.normal(size=(1, hd))
    s1 = D.rope(qv, [11]) @ D.rope(kv, [4]).T
    s2 = D.rope(qv, [107]) @ D.rope(kv, [100]).T
    assert np.allclose(s1, s2, atol=1e-12)
    # the first pair turns by exactly pos radians (theta_0 = 1)
    e0 = np.zeros((1, hd))
    e0[0, 0] = 1.0
    r = D.rope(e0, [0.5])
    assert np.isclose(r[0, 0], np.cos(0.5)) and np.isclose(r[0, hd // 2], np.sin(0.5))


def test_swiglu_closed_form():
    h = np.array([[2.0, -1.0]])
    Wg = np.array([[1.0, 0.0]])          # gate = 2
    Wu = np.array([[0.0, -3.0]])         # up = 3
    Wd = np.array([[1.0], [0.5]])
    out = D.swiglu_mlp(h, Wg, Wu, Wd)
    silu2 = 2.0 / (1.0 + np.exp(-2.0))
    assert np.allclose(out, [[3.0 * silu2, 1.5 * silu2]], atol=1e-15)


def test_root_only_tree_is_one_decode_step():
    rng = np.random.default_rng(4)
    tr = O.tree_tables([], 3, 2)         # T = 1: the root
    Dm, F, H, Vv, L = 16, 24, 2, 20, 6
    embed = rng.normal(size=(Vv, Dm))
    layers = [_layer(rng, Dm, F)]
    kcs = [rng.normal(size=(H, L + 2, Dm // H))]
    vcs = [rng.normal(size=(H, L + 2, Dm // H))]
    _, hid, _, _ = D.tree_forward(tr, np.array([5]), embed, layers, np.ones(Dm), np.eye(Vv, Dm), kcs, vcs, L, H)
    ref = _causal_forward(np.array([5]), embed, layers, kcs, vcs, L, H)
    assert np.allclose(hid, ref, atol=1e-12)


def _model(rng, V, Dm=16, F=24, H=2, nl=2, s=0.3):
    return {"embed": rng.normal(size=(V, Dm)), "layers": [_layer(rng, Dm, F, s) for _ in range(nl)],
            "final_norm": np.ones(Dm), "lm_head": rng.normal(size=(V, Dm)), "H": H}


def _heads(rng, K, V, Dm=16, s=0.5):
    return {"W1": s * rng.normal(size=(K, Dm, Dm)), "b1": s * rng.normal(size=(K, Dm)),
            "Wout": rng.normal(size=(K, V, Dm))}


def _copy_heads(model, K):
    """Heads that propose the base model's current prediction at every depth (u = h, Wout = LM head)."""
    Dm = model["embed"].shape[1]
    return {"W1": np.zeros((K, Dm, Dm)), "b1": np.zeros((K, Dm)),
            "Wout": np.repeat(model["lm_head"][None], K, axis=0)}


@pytest.mark.parametrize("seed,V,K,topk,n_nodes,kind", [
    (0, 4, 3, 2, 10, "random"), (1, 5, 4, 3, 20, "random"), (3, 50, 3, 2, 8, "random"),
    (0, 4, 3, 2, 10, "copy"), (1, 5, 4, 3, 20, "copy"), (2, 6, 2, 2, 6, "copy"), (4, 8, 5, 2, 16, "copy")])
def test_greedy_medusa_generation_is_lossless(seed, V, K, topk, n_nodes, kind):
    """Greedy Medusa decoding emits exactly the base model's greedy tokens, whatever the heads
    propose: the base model decides.  Random heads are mostly rejected; heads that repeat the base
    model's current prediction are accepted whenever the base model repeats itself, so accepted
    paths, the KV compaction and the positions of later steps are exercised."""
    rng = np.random.default_rng(seed)
    model = _model(rng, V)
    heads = _heads(rng, K, V) if kind == "random" else _copy_heads(model, K)
    prompt = rng.integers(0, V, size=5)
    n_new = 24
    ref = D.greedy_decode(model, prompt, n_new, Lcap=64)
    choices = O.ranksum_choices(K, topk, n_nodes)
    got, accepts = D.medusa_generate_greedy(model, heads, choices, K, topk, prompt, n_new, Lcap=160)
    assert got == ref
    assert len(accepts) <= n_new and all(0 <= a <= K for a in accepts)
    if kind == "copy":
        assert sum(accepts) > 0, "no proposal was ever accepted: the case would not exercise acceptance"


@pytest.mark.parametrize("mode", ["typical", "nucleus"])
def test_sampled_generation_at_low_temperature_is_greedy(mode):
    """At a temperature far below the logit gaps the tempered distribution is one-hot: typical
    acceptance keeps exactly the arg-max child (its probability ~1 is above min(eps, alpha)), the
    nucleus holds the arg-max alone, and a draw with u in [0.1, 0.9] returns the arg-max.  So
    sampled Medusa generation reduces to greedy generation, token for token and step for step."""
    rng = np.random.default_rng(11)
    V, K, topk = 6, 3, 2
    model = _model(rng, V)
    heads = _copy_heads(model, K)
    prompt = rng.integers(0, V, size=5)
    choices = O.ranksum_choices(K, topk, 10)
    ref, ref_acc = D.medusa_generate_greedy(model, heads, choices, K, topk, prompt, 20, Lcap=96)
    u = 0.1 + 0.8 * rng.random(40)
    trace = []
    got, acc = D.medusa_generate(model, heads, choices, K, topk, prompt, 20, 96, mode=mode, temperature=1e-3,
                                 uniforms=u, trace=trace)
    assert got == ref and acc == ref_acc and sum(acc) > 0
    assert [step[3] for step in trace] == acc


def test_sampled_generation_draws_from_the_tempered_distribution():
    """With a high temperature the drawn roots leave the greedy path: every emitted root is the
    inverse-CDF draw of its step's uniform from the tempered distribution at the previous step's
    last accepted node."""
    rng = np.random.default_rng(12)
    V, K, topk = 6, 2, 2
    model = _model(rng, V)
    heads = _heads(rng, K, V)
    prompt = rng.integers(0, V, size=4)
    choices = O.ranksum_choices(K, topk, 4)
    tr = O.tree_tables(choices, K, topk)
    u = rng.random(30)
    trace = []
    got, acc = D.medusa_generate(model, heads, choices, K, topk, prompt, 16, 96, mode="typical",
                                 temperature=1.5, uniforms=u, trace=trace)
    greedy, _ = D.medusa_generate_greedy(model, heads, choices, K, topk, prompt, 16, Lcap=96)
    assert got != greedy
    pos = 0
    for s, (logits, cand, best, a, _) in enumerate(trace[:-1]):
        pos += a + 1
        if pos >= len(got):
            break
        node = tr["retrieve"][best, a]
        z = logits[node] / 1.5
        w = np.exp(z - z.max())
        assert got[pos] == O.sample_index(w, u[s])   # the next step's root


# ---- planted mistakes in the decoder oracle: each must fail the path pin ----
def _flawed_layer(flaw):
    """The oracle's decoder layer with one plausible mistake planted."""
    def layer(tree, x, ly, k_cache, v_cache, L_b, H):
        x = np.asarray(x, dtype=np.float64)
        T, Dm = x.shape
        hd = Dm // H
        depth = np.asarray(tree["depth"])
        pos = depth if flaw == "positions without the prefix length" else L_b + depth
        kc, vc = np.array(k_cache, dtype=np.float64), np.array(v_cache, dtype=np.float64)
        h = D.rms_norm(x, ly["attn_norm"])
        q = (h @ ly["Wq"].T).reshape(T, H, hd).transpose(1, 0, 2)
        k = (h @ ly["Wk"].T).reshape(T, H, hd).transpose(1, 0, 2)
        v = (h @ ly["Wv"].T).reshape(T, H, hd).transpose(1, 0, 2)
        q = D.rope(q, pos)
        if flaw != "rotation of q only":
            k = D.rope(k, pos)
        rows = L_b + (depth if flaw == "tree keys at rows L + depth" else np.arange(T))
        kc[:, rows, :] = k
        vc[:, rows, :] = v
        att = np.stack([O.tree_attention_slice(tree, q[e], kc[e], vc[e], L_b, O.attention_scale(hd))
                        for e in range(H)], axis=1)
        proj = att.reshape(T, Dm) @ ly["Wo"].T
        x = proj if flaw == "no residual around attention" else x + proj
        hm = h if flaw == "feed-forward on the attention's normalised input" else D.rms_norm(x, ly["mlp_norm"])
        x = x + D.swiglu_mlp(hm, ly["W_gate"], ly["W_up"], ly["W_down"])
        return x, kc, vc
    return layer


def _forward_without_final_norm(tree, tokens, embed, layers, final_norm, lm_head, k_caches, v_caches, L_b, H):
    x = np.asarray(embed, dtype=np.float64)[np.asarray(tokens)]
    for li, ly in enumerate(layers):
        x, _, _ = D.decoder_layer(tree, x, ly, k_caches[li], v_caches[li], L_b, H)
    return x @ np.asarray(lm_head).T, x, None, None


def _rope_adjacent_pairs(x, pos, base=D.ROPE_BASE):
    """RoPE pairing dimensions (2i, 2i + 1) instead of (i, i + hd/2)."""
    x = np.asarray(x, dtype=np.float64)
    hd = x.shape[-1]
    inv = base ** (-np.arange(hd // 2) * 2.0 / hd)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]
    a, b = x[..., 0::2], x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2], y[..., 1::2] = a * np.cos(ang) - b * np.sin(ang), a * np.sin(ang) + b * np.cos(ang)
    return y


DECODER_MUTANTS = {
    **{f: ("decoder_layer", _flawed_layer(f)) for f in (
        "positions without the prefix length", "rotation of q only", "tree keys at rows L + depth",
        "no residual around attention", "feed-forward on the attention's normalised input")},
    "no final norm before the LM head": ("tree_forward", _forward_without_final_norm),
    "rotation pairs adjacent dimensions": ("rope", _rope_adjacent_pairs),
}


def test_unflawed_copy_passes_the_path_pin(monkeypatch):
    # the harness itself: the layer copy above, with no flaw planted, satisfies the pin
    monkeypatch.setattr(D, "decoder_layer", _flawed_layer(None))
    test_tree_forward_equals_causal_forward_along_every_path(WORKED, 2, 2, 9)


@pytest.mark.parametrize("name", sorted(DECODER_MUTANTS))
def test_decoder_mutants_are_caught(monkeypatch, name):
    attr, fn = DECODER_MUTANTS[name]
    monkeypatch.setattr(D, attr, fn)
    with pytest.raises(AssertionError):
        test_tree_forward_equals_causal_forward_along_every_path(WORKED, 2, 2, 9)
