"""Greedy Medusa generation of one sequence on the GPU (medusa_generate_greedy).

Small LLaMA-shaped base models (hd 128, two heads, two layers) with bf16 weights:
- **Lossless on the device.** The tokens equal those of the same call with the root-only tree, in
  which every step accepts nothing and emits the base model's own token: plain greedy decoding.
  The base model decides in both runs. A token's logits do not depend on the other tree tokens
  (masked keys add exact zeros), so the two runs take the same decisions.
- **Against the oracle.** The tokens equal the fp64 oracle's greedy decoding. The seed is chosen so
  that every decision on the oracle's trajectory has a top-1/top-2 logit gap above twice the forward's
  error bound, since the device rounds its intermediates to bf16.
- **Acceptance.** Heads that repeat the base model's current prediction get proposals accepted, so
  the compaction and the positions of later steps are exercised.
- **Sampled acceptance (medusa_generate).**
  - Typical and nucleus acceptance at a temperature far below the logit gaps reduce to greedy
    decoding on the device.
  - Typical acceptance at temperature 0.7 matches the oracle's sampled generation. Its seeds keep,
    on the oracle's trajectory:
    - every head top-k gap clear;
    - every typical decision |p - threshold| above 25% of max(p, threshold);
    - every draw 10% of the mass inside its token's interval.

    Those margins are well above what the device's bf16 intermediates can move (4e-2 of the logits'
    RMS at most, divided by the temperature).
"""

import numpy as np
import pytest
import torch

import oracle.decoder_oracle as Dm
import oracle.medusa_oracle as O

pytestmark = pytest.mark.gpu

D, F, NL, H = 256, 384, 2, 2
MAX_TOL = 4e-2   # the base forward's largest-error bound, relative to the logits' RMS


@pytest.fixture(scope="module")
def mb(built):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import speculative_decoding_heads_b200 as mb
    return mb


def _bf(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def _model(rng, V, s=0.06):
    layers = [{"attn_norm": _bf(1.0 + 0.1 * rng.normal(size=D)), "Wq": _bf(s * rng.normal(size=(D, D))),
               "Wk": _bf(s * rng.normal(size=(D, D))), "Wv": _bf(s * rng.normal(size=(D, D))),
               "Wo": _bf(s * rng.normal(size=(D, D))), "mlp_norm": _bf(1.0 + 0.1 * rng.normal(size=D)),
               "W_gate": _bf(s * rng.normal(size=(F, D))), "W_up": _bf(s * rng.normal(size=(F, D))),
               "W_down": _bf(s * rng.normal(size=(D, F)))} for _ in range(NL)]
    return {"embed": _bf(rng.normal(size=(V, D))), "layers": layers, "final_norm": _bf(np.ones(D)),
            "lm_head": _bf(0.3 * rng.normal(size=(V, D))), "H": H}


def _oracle_greedy_gaps(model, prompt, n_new, Lcap):
    """The oracle's greedy tokens and the smallest top-1/top-2 gap along the way, relative to the
    logits' RMS (the oracle's own plain greedy decoding, step by step)."""
    kcs, vcs = Dm._empty_caches(model, Lcap)
    logits, _, kcs, vcs = Dm._forward(model, Dm.chain_tree(len(prompt)), np.asarray(prompt), kcs, vcs, 0)
    L, out, gap = len(prompt), [], np.inf
    row = logits[-1]
    while True:
        top2 = np.sort(row)[-2:]
        gap = min(gap, (top2[1] - top2[0]) / np.sqrt(np.mean(row ** 2)))
        out.append(int(np.argmax(row)))
        if len(out) == n_new:
            return out, gap
        logits, _, kcs, vcs = Dm._forward(model, Dm.chain_tree(1), np.asarray(out[-1:]), kcs, vcs, L)
        L += 1
        row = logits[-1]


def _device(mb, model, heads, choices, K, topk):
    cuda = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float32)).cuda()
    dec = mb.Decoder(cuda(model["embed"]), [{k: cuda(v) for k, v in ly.items()} for ly in model["layers"]],
                     cuda(model["final_norm"]), cuda(model["lm_head"]))
    hd = {k: cuda(v).to(torch.bfloat16).contiguous() for k, v in heads.items()}
    return dec, hd, mb.Tree(choices, K, topk)


def _generate(mb, dec, hd, tree, prompt, n_new, Lcap):
    kc = torch.zeros((NL, 1, H, Lcap, 128), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    toks, acc = mb.medusa_generate_greedy(tree, dec, hd["W1"], hd["b1"], hd["Wout"], prompt, n_new, kc, vc,
                                          max_steps=n_new)
    assert mb.device_status(clear=True) == (0, 0)
    return toks, acc


def _heads(rng, model, K, kind):
    V = model["lm_head"].shape[0]
    if kind == "copy":   # u = h, Wout = the LM head: every head proposes the base model's prediction
        return {"W1": np.zeros((K, D, D)), "b1": np.zeros((K, D)), "Wout": np.repeat(model["lm_head"][None], K, 0)}
    return {"W1": _bf(0.05 * rng.normal(size=(K, D, D))), "b1": _bf(0.05 * rng.normal(size=(K, D))),
            "Wout": _bf(0.3 * rng.normal(size=(K, V, D)))}


def _clear_seed(V, n_prompt, n_new, Lcap, need_repeat=False, tries=60):
    """First model seed whose oracle greedy trajectory keeps every gap above the bound (and, for
    heads that repeat the base model's prediction, repeats a token somewhere, where they are right)."""
    for seed in range(tries):
        rng = np.random.default_rng(1000 + seed)
        model = _model(rng, V)
        prompt = rng.integers(0, V, size=n_prompt).tolist()
        ref, gap = _oracle_greedy_gaps(model, prompt, n_new, Lcap)
        repeats = any(a == b for a, b in zip(ref[:-1], ref[1:]))
        if gap > 2 * MAX_TOL and (repeats or not need_repeat):
            return rng, model, prompt, ref
    raise RuntimeError("no seed with clear greedy decisions")


@pytest.mark.parametrize("V,n_prompt,K,topk,n_nodes,kind", [
    (12, 5, 3, 2, 10, "random"),
    (12, 20, 3, 2, 10, "copy"),     # the prompt in two chains (17 + 3)
    (16, 9, 4, 3, 20, "copy"),
    (8, 6, 5, 2, 16, "copy"),
])
def test_generate_is_lossless_and_matches_the_oracle(mb, V, n_prompt, K, topk, n_nodes, kind):
    n_new = 24
    choices = O.ranksum_choices(K, topk, n_nodes)
    T = len(choices) + 1
    Lcap = n_prompt + n_new + T + 2
    rng, model, prompt, ref = _clear_seed(V, n_prompt, n_new, Lcap, need_repeat=kind == "copy")
    heads = _heads(rng, model, K, kind)
    dec, hd, tree = _device(mb, model, heads, choices, K, topk)
    got, accepts = _generate(mb, dec, hd, tree, prompt, n_new, Lcap)
    # plain greedy on the device: the root-only tree with one head
    dec1, hd1, tree1 = _device(mb, model, _heads(rng, model, 1, "random"), [], 1, 1)
    plain, acc1 = _generate(mb, dec1, hd1, tree1, prompt, n_new, n_prompt + n_new + 3)
    assert all(a == 0 for a in acc1) and len(acc1) == n_new
    assert got == plain
    assert got == ref
    assert all(0 <= a <= tree.D for a in accepts) and sum(a + 1 for a in accepts) >= n_new
    if kind == "copy":
        assert sum(accepts) > 0, "no proposal was accepted: the case would not exercise acceptance"


def test_generate_refuses_bad_arguments(mb):
    rng = np.random.default_rng(7)
    model = _model(rng, 12)
    choices = O.ranksum_choices(3, 2, 10)
    dec, hd, tree = _device(mb, model, _heads(rng, model, 3, "random"), choices, 3, 2)
    kc = torch.zeros((NL, 1, H, 20, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mb.MedusaError):   # the prompt and one tree do not fit in Lcap 20
        mb.medusa_generate_greedy(tree, dec, hd["W1"], hd["b1"], hd["Wout"], list(range(10)), 4, kc, kc.clone())
    kc = torch.zeros((NL, 1, H, 64, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mb.MedusaError):   # a prompt token outside [0, V)
        mb.medusa_generate_greedy(tree, dec, hd["W1"], hd["b1"], hd["Wout"], [1, 12], 4, kc, kc.clone())
    with pytest.raises(ValueError):       # heads of the wrong count
        mb.medusa_generate_greedy(tree, dec, hd["W1"][:2], hd["b1"], hd["Wout"], [1, 2], 4, kc, kc.clone())
    assert mb.device_status(clear=True) == (0, 0)


def test_sampled_generation_at_low_temperature_is_greedy(mb):
    V, n_prompt, K, topk, n_nodes, n_new = 12, 6, 3, 2, 10, 20
    choices = O.ranksum_choices(K, topk, n_nodes)
    Lcap = n_prompt + n_new + len(choices) + 3
    rng, model, prompt, ref = _clear_seed(V, n_prompt, n_new, Lcap, need_repeat=True)
    dec, hd, tree = _device(mb, model, _heads(rng, model, K, "copy"), choices, K, topk)
    greedy, g_acc = _generate(mb, dec, hd, tree, prompt, n_new, Lcap)
    assert greedy == ref and sum(g_acc) > 0
    u = (0.1 + 0.8 * rng.random(n_new)).tolist()
    for mode in (mb.MEDUSA_TYPICAL, mb.MEDUSA_NUCLEUS):
        kc = torch.zeros((NL, 1, H, Lcap, 128), dtype=torch.bfloat16, device="cuda")
        toks, acc = mb.medusa_generate(tree, dec, hd["W1"], hd["b1"], hd["Wout"], prompt, n_new, kc, kc.clone(),
                                       mode=mode, temperature=1e-3, uniforms=u, max_steps=n_new)
        assert mb.device_status(clear=True) == (0, 0)
        assert toks == greedy and acc == g_acc, mode


def _topk_clear(z, k, rel):
    """The k+1 largest values of every row are rel * RMS apart (the top-k set and its order hold)."""
    for row in np.atleast_2d(z):
        top = np.sort(row)[::-1][:k + 1]
        if np.min(top[:-1] - top[1:]) < rel * np.sqrt(np.mean(row ** 2)):
            return False
    return True


def _sampled_seed(V, K, topk, n_nodes, n_prompt, n_new, temp, tries=300):
    """A model, prompt and uniforms whose typical-acceptance trajectory (oracle) keeps the
    margins the module docstring lists."""
    choices = O.ranksum_choices(K, topk, n_nodes)
    tr = O.tree_tables(choices, K, topk)
    Lcap = n_prompt + n_new + tr["T"] + 2
    for seed in range(tries):
        rng = np.random.default_rng(5000 + seed)
        model = _model(rng, V)
        prompt = rng.integers(0, V, size=n_prompt).tolist()
        kcs, vcs = Dm._empty_caches(model, Lcap)
        logits0 = Dm._forward(model, Dm.chain_tree(n_prompt), np.asarray(prompt), kcs, vcs, 0)[0][-1]
        if not _topk_clear(logits0, topk, 2 * MAX_TOL):   # the first root and the first heads' top-k
            continue
        heads = _heads(rng, model, K, "copy")
        u = 0.05 + 0.9 * rng.random(n_new)
        trace = []
        got, acc = Dm.medusa_generate(model, heads, choices, K, topk, prompt, n_new, Lcap, mode="typical",
                                      temperature=temp, uniforms=u, trace=trace)
        ok = True
        for s, (logits, cand, best, a, z) in enumerate(trace):
            st = O.node_statistics(logits, temp, 0.09, 0.3)
            ret = tr["retrieve"]
            ok = ok and _topk_clear(z, topk, 2 * MAX_TOL)
            for p in range(tr["P"]):
                for j in range(1, tr["D"] + 1):
                    if ret[p, j] < 0:
                        break
                    pr, th = st["prob"][ret[p, j - 1], int(cand[p, j])], st["threshold"][ret[p, j - 1]]
                    ok = ok and abs(pr - th) >= 0.25 * max(pr, th)
            ok = ok and O.sample_margin_ok(st["prob"][ret[best, a]], float(u[s]), rel=0.1)
            if not ok:
                break
        if ok and sum(acc) > 0:
            return model, choices, heads, prompt, u, got, acc, Lcap
    raise RuntimeError("no seed with clear sampled decisions")


def test_typical_generation_matches_the_oracle(mb):
    V, K, topk, n_nodes, n_prompt, n_new, temp = 8, 2, 2, 4, 5, 10, 0.7
    model, choices, heads, prompt, u, ref, ref_acc, Lcap = _sampled_seed(V, K, topk, n_nodes, n_prompt, n_new, temp)
    dec, hd, tree = _device(mb, model, heads, choices, K, topk)
    kc = torch.zeros((NL, 1, H, Lcap, 128), dtype=torch.bfloat16, device="cuda")
    toks, acc = mb.medusa_generate(tree, dec, hd["W1"], hd["b1"], hd["Wout"], prompt, n_new, kc, kc.clone(),
                                   mode=mb.MEDUSA_TYPICAL, temperature=temp, uniforms=u.tolist(), max_steps=n_new)
    assert mb.device_status(clear=True) == (0, 0)
    assert toks == ref
    assert acc == ref_acc[:len(acc)]
