"""Parity of every C-ABI call with the fp64 oracle, on small workloads that
span several tiles and ragged tails, plus edge cases and error paths.

All tests call the CUDA library through its C ABI (ctypes binding) on the
same seeded inputs the oracle reads: the device inputs come from the device
generator, which ``test_device_generator_matches_host`` ties bit for bit to
the host generator the oracle reads.
"""

import numpy as np
import pytest
import torch

import oracle.medusa_oracle as O
from synth import gen, inputs as I
from helpers import (ATTN_ATOL, SMALL, check_logits, oracle_tree, pick_logits, pick_nucleus_inputs, pick_sub_h,
                     pick_uniforms)

TOP_P = 0.8   # the pages' default

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mb(built):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import speculative_decoding_heads_b200 as mb
    return mb


@pytest.fixture(scope="module")
def dev(mb):
    from synth import device
    return device


def _tree(mb, w):
    return mb.Tree(O.ranksum_choices(w.K, w.topk, w.n_nodes), w.K, w.topk)


def _np(t):
    return t.detach().cpu().numpy()


def _status_clean(mb):
    st, det = mb.device_status(clear=True)
    assert (st, det) == (0, 0), f"device status {st} detail {det}"


# ---------------------------------------------------------------------------


def test_device_generator_matches_host(mb, dev):
    for dt, bf in ((torch.bfloat16, True), (torch.float32, False)):
        t = torch.empty(300_001, dtype=dt, device="cuda")
        dev.fill_normal(t, 17, 5, 0.02, offset=123)
        got = _np(t.view(torch.int16)).view(np.uint16) if bf else _np(t)
        ref = gen.normal_bf16_bits(17, 5, 300_001, 0.02, offset=123) if bf else \
            gen.normal_f32(17, 5, 300_001, 0.02, offset=123)
        assert np.array_equal(got, ref)
    w = SMALL["v13b_small"]
    tr = oracle_tree(w)
    toks = np.random.default_rng(3).integers(0, w.V, size=(w.B, tr["T"]))
    raw = I.base_logits_raw(w)
    host = gen.plant_agreement(raw.copy(), toks, tr["parent"], w.agreement, w.seed)
    d = torch.from_numpy(raw.copy()).cuda()
    dev.plant(d, torch.from_numpy(toks.astype(np.int32)).cuda(), dev.parent_tensor(tr["parent"]),
              w.agreement, w.seed)
    assert np.array_equal(_np(d), host)


@pytest.mark.parametrize("name", sorted(SMALL))
def test_heads_topk(mb, dev, name):
    w = SMALL[name]
    sub_h, u, z = pick_sub_h(w)
    ids_ref, vals_ref = O.topk_desc(z, w.topk)
    t = dev.materialise(w, sub_h=sub_h)
    ws = mb.workspace(mb.medusa_heads_workspace_size(w.B, w.d, w.V, w.K, w.topk))
    for rep in range(2):                        # the second call checks the counters were reset
        t["topk_ids"].fill_(-7)
        mb.medusa_heads_topk(t["h"], t["W1"], t["b1"], t["Wout"], w.topk, t["topk_ids"], t["topk_vals"], ws,
                             head_logits=t["head_logits"])
        torch.cuda.synchronize()
        assert np.array_equal(_np(t["topk_ids"]), ids_ref), f"call {rep}"
    check_logits(_np(t["head_logits"]), z)
    check_logits(_np(t["topk_vals"]), vals_ref)
    # without the optional logits output
    t["topk_ids"].fill_(-7)
    mb.medusa_heads_topk(t["h"], t["W1"], t["b1"], t["Wout"], w.topk, t["topk_ids"], t["topk_vals"], ws)
    torch.cuda.synchronize()
    assert np.array_equal(_np(t["topk_ids"]), ids_ref)
    _status_clean(mb)


@pytest.mark.parametrize("B", [4, 5])
def test_heads_topk_wide_rows(mb, dev, B):
    # d 5120 (640 16-byte vectors, 4-row stages): with 2-4 sequences per launch
    # one vector per consumer thread (26 warps); B 5 runs groups of 4 and 1.
    from synth.workloads import shrink
    w = shrink(SMALL["v13b_small"], name=f"heads_wide_B{B}", d=5120, V=1500, B=B)
    sub_h, u, z = pick_sub_h(w)
    ids_ref, vals_ref = O.topk_desc(z, w.topk)
    t = dev.materialise(w, sub_h=sub_h)
    ws = mb.workspace(mb.medusa_heads_workspace_size(w.B, w.d, w.V, w.K, w.topk))
    mb.medusa_heads_topk(t["h"], t["W1"], t["b1"], t["Wout"], w.topk, t["topk_ids"], t["topk_vals"], ws,
                         head_logits=t["head_logits"])
    torch.cuda.synchronize()
    assert np.array_equal(_np(t["topk_ids"]), ids_ref)
    check_logits(_np(t["head_logits"]), z)
    check_logits(_np(t["topk_vals"]), vals_ref)
    _status_clean(mb)


@pytest.mark.parametrize("B", [2, 16, 17, 33])
def test_heads_topk_tensor_core_passes(mb, dev, B):
    # bf16 heads from two sequences up run on the tensor cores in passes of
    # at most 16 sequences (two launches each): B 2 is the smallest pass,
    # 16 a full one, 17 and 33 end in a one-sequence pass.  At 33 sequences
    # two heads of top-4 keep the gap guard satisfiable.
    from synth.workloads import shrink
    extra = {"K": 2, "topk": 4} if B > 17 else {}
    w = shrink(SMALL["v13b_small"], name=f"heads_tc_B{B}", d=512, V=2100, B=B, **extra)
    sub_h, u, z = pick_sub_h(w, max_tries=32)
    ids_ref, vals_ref = O.topk_desc(z, w.topk)
    t = dev.materialise(w, sub_h=sub_h)
    ws = mb.workspace(mb.medusa_heads_workspace_size(w.B, w.d, w.V, w.K, w.topk))
    mb.medusa_heads_topk(t["h"], t["W1"], t["b1"], t["Wout"], w.topk, t["topk_ids"], t["topk_vals"], ws,
                         head_logits=t["head_logits"])
    torch.cuda.synchronize()
    assert np.array_equal(_np(t["topk_ids"]), ids_ref)
    check_logits(_np(t["head_logits"]), z)
    check_logits(_np(t["topk_vals"]), vals_ref)
    _status_clean(mb)


@pytest.mark.parametrize("name", sorted(SMALL))
def test_build_tree(mb, dev, name):
    w = SMALL[name]
    tr = oracle_tree(w)
    rng = np.random.default_rng(5)
    ids = np.stack([np.stack([rng.permutation(w.V)[:w.topk] for _ in range(w.K)]) for _ in range(w.B)])
    root = rng.integers(0, w.V, size=w.B)
    lens = w.prefix_lens()
    toks, cand, pos = O.build_tree(tr, root, ids, lens)
    tree = _tree(mb, w)
    t = dev.tree_outputs({}, w.B, tree.T, tree.P, tree.D)
    c = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()
    mb.medusa_build_tree(tree, c(root), c(ids), c(lens), t["tree_tokens"], t["candidates"], t["position_ids"])
    torch.cuda.synchronize()
    assert np.array_equal(_np(t["tree_tokens"]), toks)
    assert np.array_equal(_np(t["candidates"]), cand)
    assert np.array_equal(_np(t["position_ids"]), pos)


def _attention_case(mb, dev, w, tree_choices=None):
    tr = oracle_tree(w) if tree_choices is None else O.tree_tables(tree_choices, w.K, w.topk)
    t = dev.materialise(w, fill=False)
    dev.fill_normal(t["q"], w.seed, gen.TID_Q, w.q_sigma)
    dev.fill_normal(t["k_cache"], w.seed, gen.TID_KCACHE, w.kv_sigma)
    dev.fill_normal(t["v_cache"], w.seed, gen.TID_VCACHE, w.kv_sigma)
    tree = _tree(mb, w) if tree_choices is None else mb.Tree(tree_choices, w.K, w.topk)
    scale = O.attention_scale(w.hd)
    mb.medusa_tree_attention(tree, t["q"], t["k_cache"], t["v_cache"], t["seq_lens"], scale, t["attn_out"])
    torch.cuda.synchronize()
    q = I.values(I.queries(w))
    kc = I.values(I.kv_cache(w, "k"))
    vc = I.values(I.kv_cache(w, "v"))
    ref = O.tree_attention(tr, q, kc, vc, w.prefix_lens(), scale)
    got = _np(t["attn_out"].float()).astype(np.float64)
    err = np.abs(got - ref).max()
    assert err <= ATTN_ATOL[w.dtype], f"max abs error {err:.3g}"
    _status_clean(mb)
    return err


@pytest.mark.parametrize("name", sorted(SMALL))
def test_tree_attention(mb, dev, name):
    _attention_case(mb, dev, SMALL[name])


@pytest.mark.parametrize("shape", [("v7b_small", 2, 160, 200, 1), ("v13b_small", 1, 37, 131, 9),
                                   ("v33b_small", 1, 90, 150, 2)])
def test_tree_attention_many_slices(mb, dev, shape):
    # More work items than SMs: every persistent CTA walks several (Q, K/V,
    # S, P and O buffers change hands between them).  T 64; T 49 with ragged
    # prefixes and an uneven split; T 129 in two 128-token row groups.
    from synth.workloads import shrink
    name, layers, H, prefix, B = shape
    kw = dict(layers=layers, H=H, B=B)
    if name == "v13b_small":
        kw["prefix_range"] = (prefix // 4, prefix)
    else:
        kw["prefix"] = prefix
    _attention_case(mb, dev, shrink(SMALL[name], **kw))


@pytest.mark.parametrize("variant", ["T200_two_row_groups", "T256_max", "T100_L0", "hd64_bf16_generic",
                                     "hd256_f32", "chain_L0", "exact_capacity", "T129_tail", "T130_tail",
                                     "T130_tail_L0"])
def test_tree_attention_edges(mb, dev, variant):
    base = SMALL["v7b_small"]
    from synth.workloads import shrink
    if variant.startswith("T129_tail") or variant.startswith("T130_tail"):
        # one or two rows past a 128-row group: a 128-row pass and a 64-row pass
        n = 128 if variant.startswith("T129") else 129
        w = shrink(base, K=5, topk=10, n_nodes=n, prefix=0 if variant.endswith("L0") else 201, layers=2, H=3)
        assert w.T == n + 1
        _attention_case(mb, dev, w)
    elif variant == "T200_two_row_groups":
        w = shrink(base, K=5, topk=10, n_nodes=199, prefix=70, layers=1, H=2)
        _attention_case(mb, dev, w)
    elif variant == "T256_max":
        # the largest tree (MEDUSA_MAX_T tokens): two full 128-token row groups
        w = shrink(base, K=5, topk=10, n_nodes=255, prefix=100, layers=1, H=2)
        assert w.T == 256
        _attention_case(mb, dev, w)
    elif variant == "T100_L0":
        # every key is a tree key: the masked path on every step
        w = shrink(base, K=5, topk=10, n_nodes=99, prefix=0, layers=1, H=3)
        _attention_case(mb, dev, w)
    elif variant == "hd64_bf16_generic":
        _attention_case(mb, dev, shrink(base, hd=64, layers=1, H=3, prefix=90))
    elif variant == "hd256_f32":
        _attention_case(mb, dev, shrink(SMALL["tiny_f32"], hd=256, H=2, prefix=33))
    elif variant == "chain_L0":
        w = shrink(base, K=5, topk=1, n_nodes=5, prefix=0, layers=1, H=2)
        _attention_case(mb, dev, w)
    else:
        # Lcap = L + T exactly, and L + T a multiple of the 128-key step
        w = shrink(base, prefix=128 - 64, layers=1, H=2)
        assert w.Lcap == 128
        _attention_case(mb, dev, w)


MODES = {"greedy": 0, "typical": 1, "nucleus": 2}


def _posterior_case(mb, w, mode, agreement=None, sampled=False):
    from synth.workloads import shrink
    if agreement is not None:
        w = shrink(w, agreement=agreement)
    tr = oracle_tree(w)
    sub_h, u, z = pick_sub_h(w)
    ids, _ = O.topk_desc(z, w.topk)
    toks, cand, _ = O.build_tree(tr, I.root_tokens(w), ids, w.prefix_lens())
    if mode == "nucleus":
        _, logits, uni = pick_nucleus_inputs(w, tr, toks, cand, TOP_P, sampled)
    else:
        _, logits = pick_logits(w, tr, toks, cand)
        uni = pick_uniforms(w, tr, logits, cand, mode, TOP_P)[1] if sampled else None
    ref = O.evaluate_posterior(tr, logits, cand, mode, w.temperature, w.eps, w.alpha, TOP_P, uni)
    tree = _tree(mb, w)
    c = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()
    B, D1 = w.B, tree.D + 1
    out = {k: torch.full(s, -9, dtype=torch.int32, device="cuda") for k, s in
           [("best", (B,)), ("alen", (B,)), ("acc", (B, D1)), ("next", (B,))]}
    ws = mb.workspace(mb.medusa_posterior_workspace_size(tree, B))
    mb.medusa_evaluate_posterior(tree, torch.from_numpy(logits).cuda(), c(cand), MODES[mode],
                                 out["best"], out["alen"], out["acc"], out["next"], ws,
                                 temperature=w.temperature, eps=w.eps, alpha=w.alpha, top_p=TOP_P,
                                 uniforms=None if uni is None else torch.from_numpy(uni.astype(np.float32)).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(_np(out["best"]), ref["best_path"])
    assert np.array_equal(_np(out["alen"]), ref["accept_len"])
    assert np.array_equal(_np(out["acc"]), ref["accepted_tokens"])
    assert np.array_equal(_np(out["next"]), ref["next_token"])
    _status_clean(mb)
    return ref


@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("mode", ["greedy", "typical"])
def test_posterior(mb, name, mode):
    w = SMALL[name]
    if mode == "typical" and "typical" not in w.modes:
        from synth.workloads import shrink
        w = shrink(w, modes=("typical",))
    _posterior_case(mb, w, mode)


@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("mode,sampled", [("nucleus", False), ("nucleus", True), ("typical", True)])
def test_posterior_nucleus_and_sampled(mb, name, mode, sampled):
    """Nucleus acceptance (top_p 0.8) and the next token drawn with a caller uniform."""
    _posterior_case(mb, SMALL[name], mode, sampled=sampled)


@pytest.mark.parametrize("V", [40001, 65540])
@pytest.mark.parametrize("mode,sampled", [("greedy", False), ("typical", False), ("nucleus", True),
                                          ("typical", True)])
def test_posterior_vocab_shapes(mb, V, mode, sampled):
    # V = 40001: rows not 16-byte aligned (one logit per load), more than one
    # 32768-logit chunk per row; V = 65540: 16-byte loads over three chunks.
    from synth.workloads import shrink
    w = shrink(SMALL["b3_small"], name=f"b3_V{V}", V=V, modes=(mode,))
    _posterior_case(mb, w, mode, sampled=sampled)


@pytest.mark.parametrize("mode,sampled", [("nucleus", False), ("nucleus", True), ("typical", True)])
def test_posterior_vicuna7b_shape(mb, mode, sampled):
    """The posterior alone at the Vicuna-7B step's shape (64 tree tokens, V 32000)."""
    from synth.workloads import WORKLOADS, shrink
    w = shrink(WORKLOADS["vicuna7b_bs1_L1024"], name="v7b_post", d=256, layers=1, H=1, prefix=16)
    _posterior_case(mb, w, mode, sampled=sampled)


@pytest.mark.parametrize("agreement,expect", [(0.0, "none"), (1.0, "leaf")])
def test_posterior_extremes(mb, agreement, expect):
    ref = _posterior_case(mb, SMALL["v13b_small"], "greedy", agreement)
    if expect == "none":
        # nothing planted: a random N(0, 9) row's argmax almost never is a child
        assert (ref["accept_len"] <= 1).all()
    else:
        # every internal node agrees with one child: the walk always reaches a leaf
        assert (ref["accept_len"] >= 1).all()


@pytest.mark.parametrize("name", ["v7b_small", "v13b_small", "tiny_f32", "b3_small"])
def test_accept_kv(mb, dev, name):
    w = SMALL[name]
    tr = oracle_tree(w)
    rng = np.random.default_rng(9)
    best = rng.integers(0, tr["P"], size=w.B)
    depth_of = [int((tr["retrieve"][p] >= 0).sum()) - 1 for p in range(tr["P"])]
    alen = np.array([rng.integers(0, depth_of[p] + 1) for p in best])
    alen[0] = depth_of[best[0]]                 # one sequence takes its whole path
    t = dev.materialise(w, fill=False)
    dev.fill_normal(t["k_cache"], w.seed, gen.TID_KCACHE, w.kv_sigma)
    dev.fill_normal(t["v_cache"], w.seed, gen.TID_VCACHE, w.kv_sigma)
    tree = _tree(mb, w)
    c = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()
    mb.medusa_accept_kv(tree, t["k_cache"], t["v_cache"], t["seq_lens"], c(best), c(alen))
    torch.cuda.synchronize()
    kc, vc = I.kv_cache(w, "k"), I.kv_cache(w, "v")
    k2, v2, lens2 = O.accept_kv(tr, kc, vc, w.prefix_lens(), best, alen)
    view = (lambda x: _np(x.view(torch.int16)).view(np.uint16)) if w.dtype == "bf16" else _np
    assert np.array_equal(view(t["k_cache"]), k2)
    assert np.array_equal(view(t["v_cache"]), v2)
    assert np.array_equal(_np(t["seq_lens"]), lens2)
    _status_clean(mb)


def test_accept_kv_overlap_worked_example(mb, dev):
    """Path (root, B, X after B): node_1 = 2 is also destination 2."""
    from synth.workloads import shrink
    choices = [(0,), (1,), (0, 0), (0, 1), (1, 0), (1, 1)]
    w = shrink(SMALL["v7b_small"], K=2, topk=2, n_nodes=6, layers=2, H=2, prefix=5)
    tr = O.tree_tables(choices, 2, 2)
    tree = mb.Tree(choices, 2, 2)
    t = dev.materialise(w, fill=False)
    dev.fill_normal(t["k_cache"], w.seed, gen.TID_KCACHE, w.kv_sigma)
    dev.fill_normal(t["v_cache"], w.seed, gen.TID_VCACHE, w.kv_sigma)
    best, alen = np.array([2]), np.array([2])
    assert tr["retrieve"][2][1] == 2
    c = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()
    mb.medusa_accept_kv(tree, t["k_cache"], t["v_cache"], t["seq_lens"], c(best), c(alen))
    torch.cuda.synchronize()
    k2, _, _ = O.accept_kv(tr, I.kv_cache(w, "k"), I.kv_cache(w, "v"), w.prefix_lens(), best, alen)
    assert np.array_equal(_np(t["k_cache"].view(torch.int16)).view(np.uint16), k2)


STEP_CASES = [(n, SMALL[n].modes[-1], False) for n in sorted(SMALL)] + [
    ("v7b_small", "nucleus", True), ("v13b_small", "nucleus", False), ("b3_small", "typical", True)]


@pytest.mark.parametrize("name,mode,sampled", STEP_CASES, ids=[f"{n}-{m}{'-sampled' if s else ''}"
                                                               for n, m, s in STEP_CASES])
def test_step(mb, dev, name, mode, sampled):
    """medusa_step end to end against the oracle's S1..S7 (S6 and S7 share one launch)."""
    w = SMALL[name]
    tr = oracle_tree(w)
    sub_h, u, z = pick_sub_h(w)
    ids, _ = O.topk_desc(z, w.topk)
    lens = w.prefix_lens()
    toks, cand, pos = O.build_tree(tr, I.root_tokens(w), ids, lens)
    if mode == "nucleus":
        sub_l, logits, uni = pick_nucleus_inputs(w, tr, toks, cand, TOP_P, sampled)
    else:
        sub_l, logits = pick_logits(w, tr, toks, cand)
        uni = pick_uniforms(w, tr, logits, cand, mode, TOP_P)[1] if sampled else None
    post = O.evaluate_posterior(tr, logits, cand, mode, w.temperature, w.eps, w.alpha, TOP_P, uni)
    q = I.values(I.queries(w))
    kc_raw, vc_raw = I.kv_cache(w, "k"), I.kv_cache(w, "v")
    scale = O.attention_scale(w.hd)
    attn = O.tree_attention(tr, q, I.values(kc_raw), I.values(vc_raw), lens, scale)
    k2, v2, lens2 = O.accept_kv(tr, kc_raw, vc_raw, lens, post["best_path"], post["accept_len"])

    tree = _tree(mb, w)
    t = dev.materialise(w, sub_h=sub_h, sub_logits=sub_l)
    t["base_logits"].copy_(torch.from_numpy(logits))
    dev.tree_outputs(t, w.B, tree.T, tree.P, tree.D)
    if uni is not None:
        t["uniforms"] = torch.from_numpy(uni.astype(np.float32)).cuda()
    args = mb.make_step_args(tree, t, MODES[mode], w.temperature, w.eps, w.alpha, top_p=TOP_P)
    ws = mb.workspace(mb.medusa_step_workspace_size(args))
    mb.medusa_step(args, ws)
    torch.cuda.synchronize()
    assert np.array_equal(_np(t["topk_ids"]), ids)
    check_logits(_np(t["head_logits"]), z)
    assert np.array_equal(_np(t["tree_tokens"]), toks)
    assert np.array_equal(_np(t["candidates"]), cand)
    assert np.array_equal(_np(t["position_ids"]), pos)
    err = np.abs(_np(t["attn_out"].float()).astype(np.float64) - attn).max()
    assert err <= ATTN_ATOL[w.dtype], err
    for k_ours, k_ref in [("best_path", "best_path"), ("accept_len", "accept_len"),
                          ("accepted_tokens", "accepted_tokens"), ("next_token", "next_token")]:
        assert np.array_equal(_np(t[k_ours]), post[k_ref]), k_ours
    view = (lambda x: _np(x.view(torch.int16)).view(np.uint16)) if w.dtype == "bf16" else _np
    assert np.array_equal(view(t["k_cache"]), k2)
    assert np.array_equal(view(t["v_cache"]), v2)
    assert np.array_equal(_np(t["seq_lens"]), lens2)
    _status_clean(mb)


# ---------------------------------------------------------------------------
# error paths: rejected on the host, nothing launched
# ---------------------------------------------------------------------------


def test_invalid_arguments_launch_nothing(mb, dev):
    w = SMALL["v7b_small"]
    t = dev.materialise(w, fill=False)
    ws = mb.workspace(mb.medusa_heads_workspace_size(w.B, w.d, w.V, w.K, w.topk))
    t["topk_ids"].fill_(-5)
    ids33 = torch.full((w.B, w.K, 33), -5, dtype=torch.int32, device="cuda")
    vals33 = torch.zeros((w.B, w.K, 33), device="cuda")
    cases = [
        (dict(topk=33, ids=ids33, vals=vals33), mb.MEDUSA_ERR_INVALID_ARG),
        (dict(ws=mb.workspace(256)), mb.MEDUSA_ERR_INVALID_ARG),
        (dict(h=t["h"][:, :100].contiguous(), W1=t["W1"][:, :100, :100].contiguous(),
              b1=t["b1"][:, :100].contiguous(), Wout=t["Wout"][:, :, :100].contiguous()), mb.MEDUSA_ERR_UNSUPPORTED),
    ]
    for over, code in cases:
        kw = dict(h=t["h"], W1=t["W1"], b1=t["b1"], Wout=t["Wout"], topk=w.topk, ws=ws, ids=t["topk_ids"],
                  vals=t["topk_vals"])
        kw.update(over)
        with pytest.raises(mb.MedusaError) as ei:
            mb.medusa_heads_topk(kw["h"], kw["W1"], kw["b1"], kw["Wout"], kw["topk"], kw["ids"], kw["vals"],
                                 kw["ws"])
        assert ei.value.code == code
    torch.cuda.synchronize()
    assert (t["topk_ids"] == -5).all() and (ids33 == -5).all()
    tree = _tree(mb, w)
    logits = torch.zeros((w.B, tree.T, w.V), device="cuda")
    cand = torch.zeros((w.B, tree.P, tree.D + 1), dtype=torch.int32, device="cuda")
    o = torch.full((w.B, tree.D + 1), -5, dtype=torch.int32, device="cuda")
    pws = mb.workspace(mb.medusa_posterior_workspace_size(tree, w.B))
    with pytest.raises(mb.MedusaError) as ei:
        mb.medusa_evaluate_posterior(tree, logits, cand, mb.MEDUSA_TYPICAL, o[:, 0], o[:, 1], o, o[:, 2], pws,
                                     temperature=0.0)
    assert ei.value.code == mb.MEDUSA_ERR_INVALID_ARG
    with pytest.raises(mb.MedusaError):
        mb.medusa_evaluate_posterior(tree, logits, cand, 7, o[:, 0], o[:, 1], o, o[:, 2], pws)
    torch.cuda.synchronize()
    assert (o == -5).all()


def test_device_check_on_overflowing_sequence(mb, dev):
    """seq_lens[b] + T > Lcap is caught on the device: status set, slice left alone."""
    w = SMALL["v7b_small"]
    t = dev.materialise(w, fill=False)
    tree = _tree(mb, w)
    t["seq_lens"].fill_(w.Lcap - tree.T + 1)
    t["attn_out"].fill_(0)
    mb.medusa_tree_attention(tree, t["q"], t["k_cache"], t["v_cache"], t["seq_lens"], 0.1, t["attn_out"])
    st, det = mb.device_status(clear=True)
    assert st == mb.MEDUSA_ERR_DEVICE_CHECK
    assert (t["attn_out"] == 0).all()
    _status_clean(mb)


def test_step_host_matches_device_step(mb, dev):
    # medusa_step_host copies q, the tree's K/V rows (one 3-D copy per
    # sequence into the caches) and the base logits on a second stream while
    # the heads run; the step waits for them through the two input-ready
    # events.  Its results equal a step over device-resident inputs.
    w = SMALL["v7b_small"]
    sub_h, _, _ = pick_sub_h(w)
    tree = _tree(mb, w)
    t = dev.materialise(w, sub_h=sub_h)
    dev.tree_outputs(t, w.B, tree.T, tree.P, tree.D)
    args = mb.make_step_args(tree, t, mb.MEDUSA_GREEDY)
    ws = mb.workspace(mb.medusa_step_workspace_size(args))
    lens0 = t["seq_lens"].clone()
    kc0, vc0 = t["k_cache"].clone(), t["v_cache"].clone()
    mb.medusa_step(args, ws)
    torch.cuda.synchronize()
    ref = {k: t[k].clone() for k in ("best_path", "accept_len", "accepted_tokens", "next_token", "attn_out",
                                     "seq_lens", "k_cache", "v_cache")}
    pin = lambda x: x.cpu().pin_memory()
    L = lens0.cpu()
    host_in = {"h": pin(t["h"]), "root_tokens": pin(t["root_tokens"]), "seq_lens": pin(lens0),
               "q": pin(t["q"]), "base_logits": pin(t["base_logits"]),
               "k_tree": pin(torch.stack([kc0[:, b, :, int(L[b]):int(L[b]) + w.T] for b in range(w.B)], 1)),
               "v_tree": pin(torch.stack([vc0[:, b, :, int(L[b]):int(L[b]) + w.T] for b in range(w.B)], 1))}
    host_out = {k: torch.empty_like(t[k], device="cpu").pin_memory()
                for k in ("best_path", "accept_len", "accepted_tokens", "next_token", "seq_lens")}
    # clobber every input the host step must bring in, and the tree rows of the caches
    for k in ("q", "base_logits", "attn_out", "h"):
        t[k].fill_(float("nan"))
    for k in ("best_path", "accept_len", "accepted_tokens", "next_token", "root_tokens"):
        t[k].fill_(-9)
    t["seq_lens"].fill_(0)
    kc, vc = kc0.clone(), vc0.clone()
    for b in range(w.B):
        kc[:, b, :, int(L[b]):int(L[b]) + w.T] = float("nan")
        vc[:, b, :, int(L[b]):int(L[b]) + w.T] = float("nan")
    t["k_cache"].copy_(kc)
    t["v_cache"].copy_(vc)
    stream = torch.cuda.Stream()
    mb.medusa_step_host(args, ws, host_in, host_out, stream)
    stream.synchronize()
    for k in host_out:
        assert torch.equal(host_out[k], ref[k].cpu()), k
    assert torch.equal(t["attn_out"], ref["attn_out"])
    assert torch.equal(t["seq_lens"], ref["seq_lens"])
    assert torch.equal(t["k_cache"], ref["k_cache"])
    assert torch.equal(t["v_cache"], ref["v_cache"])
    _status_clean(mb)


def test_step_host_single_stream(mb, dev):
    # With no copy stream every copy goes on the step's stream ahead of the
    # step; the results equal the two-stream form's.
    import ctypes
    w = SMALL["v13b_small"]
    sub_h, _, _ = pick_sub_h(w)
    tree = _tree(mb, w)
    t = dev.materialise(w, sub_h=sub_h)
    dev.tree_outputs(t, w.B, tree.T, tree.P, tree.D)
    args = mb.make_step_args(tree, t, mb.MEDUSA_GREEDY)
    ws = mb.workspace(mb.medusa_step_workspace_size(args))
    lens0 = t["seq_lens"].clone()
    kc0, vc0 = t["k_cache"].clone(), t["v_cache"].clone()
    pin = lambda x: x.cpu().pin_memory()
    L = lens0.cpu()
    host_in = {"h": pin(t["h"]), "root_tokens": pin(t["root_tokens"]), "seq_lens": pin(lens0),
               "q": pin(t["q"]), "base_logits": pin(t["base_logits"]),
               "k_tree": pin(torch.stack([kc0[:, b, :, int(L[b]):int(L[b]) + w.T] for b in range(w.B)], 1)),
               "v_tree": pin(torch.stack([vc0[:, b, :, int(L[b]):int(L[b]) + w.T] for b in range(w.B)], 1))}
    outs = []
    for single in (False, True):
        t["seq_lens"].copy_(lens0)
        t["k_cache"].copy_(kc0)
        t["v_cache"].copy_(vc0)
        host_out = {k: torch.full_like(t[k], -7, device="cpu").pin_memory()
                    for k in ("best_path", "accept_len", "accepted_tokens", "next_token", "seq_lens")}
        stream = torch.cuda.Stream()
        if single:
            io = mb.StepHostIO()
            for k, x in host_in.items():
                setattr(io, k, x.data_ptr())
            for k, x in host_out.items():
                setattr(io, "seq_lens_out" if k == "seq_lens" else k, x.data_ptr())
            io.copy_stream = None
            st = mb._lib.medusa_step_host(ctypes.byref(args), ctypes.byref(io), ws.data_ptr(), ws.numel(),
                                          stream.cuda_stream)
            assert st == mb.MEDUSA_OK, mb._lib.medusa_last_error()
        else:
            mb.medusa_step_host(args, ws, host_in, host_out, stream)
        stream.synchronize()
        outs.append((host_out, t["k_cache"].clone(), t["attn_out"].clone()))
    for k in outs[0][0]:
        assert torch.equal(outs[0][0][k], outs[1][0][k]), k
    assert (outs[1][0]["accept_len"] >= 0).all()
    assert torch.equal(outs[0][1], outs[1][1])
    assert torch.equal(outs[0][2], outs[1][2])
    _status_clean(mb)


def test_step_host_refuses_device_buffers_and_overflow(mb, dev):
    # io must hold host memory; a host length that would put the tree rows
    # past Lcap is refused; both before anything is enqueued.
    import ctypes
    w = SMALL["v7b_small"]
    tree = _tree(mb, w)
    t = dev.materialise(w)
    dev.tree_outputs(t, w.B, tree.T, tree.P, tree.D)
    args = mb.make_step_args(tree, t, mb.MEDUSA_GREEDY)
    ws = mb.workspace(mb.medusa_step_workspace_size(args))
    before = {k: t[k].clone() for k in ("best_path", "seq_lens", "k_cache")}
    io = mb.StepHostIO()
    io.h = t["h"].data_ptr()   # device memory where host memory is required
    st = mb._lib.medusa_step_host(ctypes.byref(args), ctypes.byref(io), ws.data_ptr(), ws.numel(),
                                  torch.cuda.current_stream().cuda_stream)
    assert st == mb.MEDUSA_ERR_INVALID_ARG
    lens = torch.full((w.B,), w.Lcap - tree.T + 1, dtype=torch.int32).pin_memory()
    kt = torch.zeros((w.layers, w.B, w.H, tree.T, w.hd), dtype=t["k_cache"].dtype).pin_memory()
    with pytest.raises(mb.MedusaError):
        mb.medusa_step_host(args, ws, {"seq_lens": lens, "k_tree": kt}, {})
    with pytest.raises(ValueError):
        mb.medusa_step_host(args, ws, {"h": t["h"]}, {})
    torch.cuda.synchronize()
    for k, v in before.items():
        assert torch.equal(t[k], v), k
    _status_clean(mb)
