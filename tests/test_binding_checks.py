"""Host-side checks of the Python binding: every tensor argument's shape,
dtype and layout are checked before any call reaches the C ABI (which takes
bare pointers and sizes, so a tensor smaller than the sizes imply would be
read or written past its end on the device).  CPU tensors are enough here:
each case must fail its check with ValueError before the binding looks at
where the tensor lives."""

import pytest
import torch


@pytest.fixture(scope="module")
def mb(built):
    import speculative_decoding_heads_b200 as mb
    return mb


@pytest.fixture(scope="module")
def tree(mb):
    t = mb.Tree([(0,), (1,), (0, 0), (0, 1), (1, 0), (1, 1)], 2, 2, upload=False)
    yield t
    t.close()


B, d, V, K, topk = 2, 256, 300, 2, 2
bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32


def _heads(**over):
    a = dict(h=torch.zeros(B, d, dtype=bf), W1=torch.zeros(K, d, d, dtype=bf), b1=torch.zeros(K, d, dtype=bf),
             Wout=torch.zeros(K, V, d, dtype=bf), ids=torch.zeros(B, K, topk, dtype=i32),
             vals=torch.zeros(B, K, topk, dtype=f32), ws=torch.zeros(4096, dtype=torch.uint8), logits=None)
    a.update(over)
    return a


HEADS_CASES = {
    "W1 fp32 with bf16 h": dict(W1=torch.zeros(K, d, d, dtype=f32)),
    "b1 wrong length": dict(b1=torch.zeros(K, d + 8, dtype=bf)),
    "Wout fp32": dict(Wout=torch.zeros(K, V, d, dtype=f32)),
    "W1 transposed view": dict(W1=torch.zeros(K, d, d, dtype=bf).transpose(1, 2)),
    "Wout strided": dict(Wout=torch.zeros(K, 2 * V, d, dtype=bf)[:, ::2]),
    "topk_ids too small": dict(ids=torch.zeros(B, K, topk - 1, dtype=i32)),
    "topk_ids int64": dict(ids=torch.zeros(B, K, topk, dtype=torch.int64)),
    "topk_vals bf16": dict(vals=torch.zeros(B, K, topk, dtype=bf)),
    "head_logits short": dict(logits=torch.zeros(B, K, V - 1, dtype=f32)),
    "head_logits bf16": dict(logits=torch.zeros(B, K, V, dtype=bf)),
    "workspace strided": dict(ws=torch.zeros(8192, dtype=torch.uint8)[::2]),
}


@pytest.mark.parametrize("case", sorted(HEADS_CASES))
def test_heads_refuses(mb, case):
    a = _heads(**HEADS_CASES[case])
    with pytest.raises(ValueError):
        mb.medusa_heads_topk(a["h"], a["W1"], a["b1"], a["Wout"], topk, a["ids"], a["vals"], a["ws"],
                             head_logits=a["logits"])
    with pytest.raises(ValueError):
        if case.startswith("workspace"):
            raise ValueError("no workspace in this call")
        mb.medusa_heads_topk_noalloc(a["h"], a["W1"], a["b1"], a["Wout"], topk, a["ids"], a["vals"],
                                     head_logits=a["logits"])


def test_heads_well_formed_reaches_the_device_check(mb):
    a = _heads()
    with pytest.raises(ValueError, match="CUDA tensors"):
        mb.medusa_heads_topk(a["h"], a["W1"], a["b1"], a["Wout"], topk, a["ids"], a["vals"], a["ws"])


def _attn(tree, layers=2, H=3, hd=128, Lcap=40, dt=bf, **over):
    a = dict(q=torch.zeros(layers, B, tree.T, H, hd, dtype=dt),
             k=torch.zeros(layers, B, H, Lcap, hd, dtype=dt), v=torch.zeros(layers, B, H, Lcap, hd, dtype=dt),
             lens=torch.zeros(B, dtype=i32), out=torch.zeros(layers, B, tree.T, H, hd, dtype=f32))
    a.update(over)
    return a


ATTN_CASES = {
    "q fp32 with bf16 caches": lambda tr: dict(q=torch.zeros(2, B, tr.T, 3, 128, dtype=f32)),
    "q with another tree size": lambda tr: dict(q=torch.zeros(2, B, tr.T + 1, 3, 128, dtype=bf)),
    "v_cache shorter": lambda tr: dict(v=torch.zeros(2, B, 3, 39, 128, dtype=bf)),
    "k_cache heads-major mismatch": lambda tr: dict(k=torch.zeros(2, 3, B, 40, 128, dtype=bf)),
    "out bf16": lambda tr: dict(out=torch.zeros(2, B, tr.T, 3, 128, dtype=bf)),
    "out too small": lambda tr: dict(out=torch.zeros(2, B, tr.T, 3, 64, dtype=f32)),
    "seq_lens int64": lambda tr: dict(lens=torch.zeros(B, dtype=torch.int64)),
    "k_cache strided": lambda tr: dict(k=torch.zeros(2, B, 3, 80, 128, dtype=bf)[:, :, :, ::2]),
}


@pytest.mark.parametrize("case", sorted(ATTN_CASES))
def test_attention_refuses(mb, tree, case):
    a = _attn(tree, **ATTN_CASES[case](tree))
    with pytest.raises(ValueError):
        mb.medusa_tree_attention(tree, a["q"], a["k"], a["v"], a["lens"], 0.1, a["out"])
    lse = torch.zeros(a["out"].shape[:-1], dtype=f32)
    with pytest.raises(ValueError):
        mb.medusa_tree_attention_split(tree, a["q"], a["k"], a["v"], a["lens"], 0.1, 0, 2, a["out"], lse)


def test_split_refuses_a_wrong_lse(mb, tree):
    a = _attn(tree)
    with pytest.raises(ValueError, match="lse"):
        mb.medusa_tree_attention_split(tree, a["q"], a["k"], a["v"], a["lens"], 0.1, 0, 2, a["out"],
                                       torch.zeros(2, B, tree.T, 2, dtype=f32))


def test_accept_kv_refuses(mb, tree):
    a = _attn(tree)
    one = torch.zeros(B, dtype=i32)
    with pytest.raises(ValueError):
        mb.medusa_accept_kv(tree, a["k"], a["v"][:, :, :, :30].contiguous(), a["lens"], one, one)
    with pytest.raises(ValueError):
        mb.medusa_accept_kv(tree, a["k"], a["v"].float(), a["lens"], one, one)
    with pytest.raises(ValueError):
        mb.medusa_accept_kv(tree, a["k"], a["v"], a["lens"], torch.zeros(B + 1, dtype=i32), one)


def _post(tree, **over):
    D1 = tree.D + 1
    a = dict(logits=torch.zeros(B, tree.T, V, dtype=f32), cand=torch.zeros(B, tree.P, D1, dtype=i32),
             best=torch.zeros(B, dtype=i32), alen=torch.zeros(B, dtype=i32), acc=torch.zeros(B, D1, dtype=i32),
             nxt=torch.zeros(B, dtype=i32), ws=torch.zeros(1024, dtype=torch.uint8))
    a.update(over)
    return a


POST_CASES = {
    "logits bf16": lambda tr: dict(logits=torch.zeros(B, tr.T, V, dtype=bf)),
    "logits for another tree": lambda tr: dict(logits=torch.zeros(B, tr.T - 1, V, dtype=f32)),
    "candidates short": lambda tr: dict(cand=torch.zeros(B, tr.P - 1, tr.D + 1, dtype=i32)),
    "accepted_tokens short": lambda tr: dict(acc=torch.zeros(B, tr.D, dtype=i32)),
    "next_token int64": lambda tr: dict(nxt=torch.zeros(B, dtype=torch.int64)),
    "logits strided": lambda tr: dict(logits=torch.zeros(B, tr.T, 2 * V, dtype=f32)[:, :, ::2]),
}


@pytest.mark.parametrize("case", sorted(POST_CASES))
def test_posterior_refuses(mb, tree, case):
    a = _post(tree, **POST_CASES[case](tree))
    with pytest.raises(ValueError):
        mb.medusa_evaluate_posterior(tree, a["logits"], a["cand"], mb.MEDUSA_GREEDY, a["best"], a["alen"], a["acc"],
                                     a["nxt"], a["ws"])


def test_build_tree_refuses(mb, tree):
    ok = dict(root=torch.zeros(B, dtype=i32), ids=torch.zeros(B, tree.K, tree.topk, dtype=i32),
              lens=torch.zeros(B, dtype=i32), toks=torch.zeros(B, tree.T, dtype=i32),
              cand=torch.zeros(B, tree.P, tree.D + 1, dtype=i32), pos=torch.zeros(B, tree.T, dtype=i32))
    for key, bad in [("ids", torch.zeros(B, tree.K, tree.topk + 1, dtype=i32)),
                     ("toks", torch.zeros(B, tree.T - 1, dtype=i32)),
                     ("cand", torch.zeros(B, tree.P, tree.D, dtype=i32)),
                     ("pos", torch.zeros(B, tree.T, dtype=torch.int64))]:
        a = dict(ok, **{key: bad})
        with pytest.raises(ValueError):
            mb.medusa_build_tree(tree, a["root"], a["ids"], a["lens"], a["toks"], a["cand"], a["pos"])


def test_merge_combine_and_rescale_refuse(mb):
    G = 2
    vals, ids = torch.zeros(G, B, K, topk), torch.zeros(G, B, K, topk, dtype=i32)
    with pytest.raises(ValueError):
        mb.medusa_topk_merge(vals, ids.long(), [0, 150], V, torch.zeros(B, K, topk), torch.zeros(B, K, topk, dtype=i32))
    with pytest.raises(ValueError):
        mb.medusa_topk_merge(vals, ids, [0, 150], V, torch.zeros(B, K, topk + 1), torch.zeros(B, K, topk, dtype=i32))
    outs, lses = torch.zeros(G, 10, 8), torch.zeros(G, 10)
    with pytest.raises(ValueError):
        mb.medusa_attention_combine(outs, torch.zeros(G, 9), torch.zeros(10, 8))
    with pytest.raises(ValueError):
        mb.medusa_attention_combine(outs, lses, torch.zeros(10, 4))
    with pytest.raises(ValueError):
        mb.medusa_attention_rescale(lses, 0, torch.zeros(11, 8))
    with pytest.raises(ValueError):
        mb.medusa_attention_rescale(lses.double(), 0, torch.zeros(10, 8))


# The base forward and the generation loop check their arguments against the
# model's sizes before anything reaches the C ABI, so a stand-in model with
# the sizes (D 128: one head; F 256; V 16; two layers) is enough here.
_DEC_D, _DEC_V, _DEC_LAYERS, _DEC_LCAP = 128, 16, 2, 40


@pytest.fixture(scope="module")
def dec_model(mb):
    from types import SimpleNamespace
    return SimpleNamespace(D=_DEC_D, F=256, V=_DEC_V, tensors=[{}] * _DEC_LAYERS, c=mb.DecoderModel())


def _decode_args(tree, Bd=2, **over):
    cache = (_DEC_LAYERS, Bd, _DEC_D // 128, _DEC_LCAP, 128)
    a = dict(toks=torch.zeros(Bd, tree.T, dtype=i32), kc=torch.zeros(cache, dtype=bf), vc=torch.zeros(cache, dtype=bf),
             lens=torch.zeros(Bd, dtype=i32), logits=torch.zeros(Bd * tree.T, _DEC_V), hidden=None,
             ws=torch.zeros(4096, dtype=torch.uint8))
    a.update(over)
    return a


DECODE_CASES = {
    "tree tokens of another tree": lambda t: dict(toks=torch.zeros(2, t.T + 1, dtype=i32)),
    "tree tokens int64": lambda t: dict(toks=torch.zeros(2, t.T, dtype=torch.int64)),
    "cache of another layer count": lambda t: dict(kc=torch.zeros(_DEC_LAYERS + 1, 2, 1, _DEC_LCAP, 128, dtype=bf)),
    "cache fp32": lambda t: dict(vc=torch.zeros(_DEC_LAYERS, 2, 1, _DEC_LCAP, 128)),
    "v cache shorter than k cache": lambda t: dict(vc=torch.zeros(_DEC_LAYERS, 2, 1, _DEC_LCAP - 1, 128, dtype=bf)),
    "cache not contiguous": lambda t: dict(kc=torch.zeros(_DEC_LAYERS, 2, 1, 128, _DEC_LCAP, dtype=bf).transpose(3, 4)),
    "lengths for another batch": lambda t: dict(lens=torch.zeros(3, dtype=i32)),
    "logits too short": lambda t: dict(logits=torch.zeros(2 * t.T - 1, _DEC_V)),
    "hidden of the wrong width": lambda t: dict(hidden=torch.zeros(2 * t.T, _DEC_D + 1)),
}


def _decode(mb, tree, model, a):
    mb.medusa_tree_decode(tree, model, a["toks"], a["kc"], a["vc"], a["lens"], a["logits"], a["ws"], hidden=a["hidden"])


@pytest.mark.parametrize("case", sorted(DECODE_CASES))
def test_tree_decode_refuses(mb, tree, dec_model, case):
    # each case fails its own check, before the one on where tensors live
    with pytest.raises(ValueError) as e:
        _decode(mb, tree, dec_model, _decode_args(tree, **DECODE_CASES[case](tree)))
    assert "CUDA tensors" not in str(e.value)


def test_tree_decode_well_formed_reaches_the_device_check(mb, tree, dec_model):
    with pytest.raises(ValueError, match="CUDA tensors"):
        _decode(mb, tree, dec_model, _decode_args(tree, hidden=torch.zeros(2 * tree.T, _DEC_D)))


def _gen_args(tree, **over):
    cache = (_DEC_LAYERS, 1, _DEC_D // 128, _DEC_LCAP, 128)
    a = dict(W1=torch.zeros(tree.K, _DEC_D, _DEC_D, dtype=bf), b1=torch.zeros(tree.K, _DEC_D, dtype=bf),
             Wout=torch.zeros(tree.K, _DEC_V, _DEC_D, dtype=bf), prompt=[1, 2, 3], n_new=4,
             kc=torch.zeros(cache, dtype=bf), vc=torch.zeros(cache, dtype=bf), uniforms=None,
             ws=torch.zeros(4096, dtype=torch.uint8))
    a.update(over)
    return a


GENERATE_CASES = {
    "W1 for another head count": lambda t: dict(W1=torch.zeros(t.K + 1, _DEC_D, _DEC_D, dtype=bf)),
    "b1 fp32": lambda t: dict(b1=torch.zeros(t.K, _DEC_D)),
    "Wout over another vocabulary": lambda t: dict(Wout=torch.zeros(t.K, _DEC_V + 1, _DEC_D, dtype=bf)),
    "caches for two sequences": lambda t: dict(kc=torch.zeros(_DEC_LAYERS, 2, 1, _DEC_LCAP, 128, dtype=bf)),
    "empty prompt": lambda t: dict(prompt=[]),
    "nothing to generate": lambda t: dict(n_new=0),
    "fewer uniforms than steps": lambda t: dict(uniforms=[0.5] * 3),
}


def _generate(mb, tree, model, a):
    mb.medusa_generate(tree, model, a["W1"], a["b1"], a["Wout"], a["prompt"], a["n_new"], a["kc"], a["vc"],
                       mb.MEDUSA_TYPICAL, temperature=0.7, uniforms=a["uniforms"], ws=a["ws"])


@pytest.mark.parametrize("case", sorted(GENERATE_CASES))
def test_generate_refuses(mb, tree, dec_model, case):
    with pytest.raises(ValueError) as e:
        _generate(mb, tree, dec_model, _gen_args(tree, **GENERATE_CASES[case](tree)))
    assert "CUDA tensors" not in str(e.value)


def test_generate_well_formed_reaches_the_device_check(mb, tree, dec_model):
    with pytest.raises(ValueError, match="CUDA tensors"):
        _generate(mb, tree, dec_model, _gen_args(tree, uniforms=[0.5] * 4))


# The step's arguments (make_step_args): every field against the tree and
# the head/attention shapes (layers 2, H 1, hd 128, Lcap 40).
def _step(tree, **over):
    L_, H_, hd_, Lc = 2, 1, 128, 40
    T, P, D = tree.T, tree.P, tree.D
    a = dict(h=torch.zeros(B, d, dtype=bf), W1=torch.zeros(tree.K, d, d, dtype=bf), b1=torch.zeros(tree.K, d, dtype=bf),
             Wout=torch.zeros(tree.K, V, d, dtype=bf), root_tokens=torch.zeros(B, dtype=i32),
             q=torch.zeros(L_, B, T, H_, hd_, dtype=bf), k_cache=torch.zeros(L_, B, H_, Lc, hd_, dtype=bf),
             v_cache=torch.zeros(L_, B, H_, Lc, hd_, dtype=bf), seq_lens=torch.zeros(B, dtype=i32),
             base_logits=torch.zeros(B, T, V), topk_ids=torch.zeros(B, tree.K, tree.topk, dtype=i32),
             topk_vals=torch.zeros(B, tree.K, tree.topk), tree_tokens=torch.zeros(B, T, dtype=i32),
             candidates=torch.zeros(B, P, D + 1, dtype=i32), position_ids=torch.zeros(B, T, dtype=i32),
             attn_out=torch.zeros(L_, B, T, H_, hd_), best_path=torch.zeros(B, dtype=i32),
             accept_len=torch.zeros(B, dtype=i32), accepted_tokens=torch.zeros(B, D + 1, dtype=i32),
             next_token=torch.zeros(B, dtype=i32), uniforms=None)
    a.update(over)
    return a


STEP_CASES = {
    "Wout for another head count": lambda t: dict(Wout=torch.zeros(t.K + 1, V, d, dtype=bf)),
    "q fp32 with bf16 h": lambda t: dict(q=torch.zeros(2, B, t.T, 1, 128)),
    "base logits over another vocabulary": lambda t: dict(base_logits=torch.zeros(B, t.T, V + 1)),
    "root tokens int64": lambda t: dict(root_tokens=torch.zeros(B, dtype=torch.int64)),
    "candidates for another path count": lambda t: dict(candidates=torch.zeros(B, t.P + 1, t.D + 1, dtype=i32)),
    "accepted tokens too short": lambda t: dict(accepted_tokens=torch.zeros(B, t.D, dtype=i32)),
    "position ids for another tree": lambda t: dict(position_ids=torch.zeros(B, t.T + 1, dtype=i32)),
    "uniforms for another batch": lambda t: dict(uniforms=torch.zeros(B + 1)),
}


@pytest.mark.parametrize("case", sorted(STEP_CASES))
def test_step_args_refuse(mb, tree, case):
    with pytest.raises(ValueError) as e:
        mb.make_step_args(tree, _step(tree, **STEP_CASES[case](tree)), mb.MEDUSA_GREEDY)
    assert "CUDA tensors" not in str(e.value)


def test_step_args_well_formed_reach_the_device_check(mb, tree):
    with pytest.raises(ValueError, match="CUDA tensors"):
        mb.make_step_args(tree, _step(tree, uniforms=torch.zeros(B)), mb.MEDUSA_TYPICAL)


# The host-buffer step checks its host buffers against the step's shapes
# before anything is enqueued.
def _host_step_args(mb, tree):
    a = mb.StepArgs()
    a._shape = {"B": B, "d": d, "V": V, "T": tree.T, "D": tree.D, "layers": 2, "H": 1, "hd": 128, "dtype": bf}
    return a


HOST_CASES = {
    "an unknown input": lambda t: ({"k_cache": torch.zeros(1)}, {}),
    "q of another tree": lambda t: ({"q": torch.zeros(2, B, t.T + 1, 1, 128, dtype=bf)}, {}),
    "tree rows fp32": lambda t: ({"k_tree": torch.zeros(2, B, 1, t.T, 128)}, {}),
    "base logits over another vocabulary": lambda t: ({"base_logits": torch.zeros(B, t.T, V - 1)}, {}),
    "accepted tokens too short": lambda t: ({}, {"accepted_tokens": torch.zeros(B, t.D, dtype=i32)}),
    "lengths out as int64": lambda t: ({}, {"seq_lens": torch.zeros(B, dtype=torch.int64)}),
}


@pytest.mark.parametrize("case", sorted(HOST_CASES))
def test_host_step_refuses(mb, tree, case):
    host_in, host_out = HOST_CASES[case](tree)
    with pytest.raises(ValueError):
        mb.medusa_step_host(_host_step_args(mb, tree), torch.zeros(16, dtype=torch.uint8), host_in, host_out)


def test_host_step_well_formed_passes_the_buffer_checks(mb, tree):
    # well-formed host buffers get past every buffer check (here, without a GPU, the failure comes later
    # and is not one of those checks)
    host_in = {"h": torch.zeros(B, d, dtype=bf), "q": torch.zeros(2, B, tree.T, 1, 128, dtype=bf),
               "base_logits": torch.zeros(B, tree.T, V)}
    host_out = {"accepted_tokens": torch.zeros(B, tree.D + 1, dtype=i32), "seq_lens": torch.zeros(B, dtype=i32)}
    with pytest.raises(Exception) as e:
        mb.medusa_step_host(_host_step_args(mb, tree), torch.zeros(16, dtype=torch.uint8), host_in, host_out)
    assert not isinstance(e.value, ValueError), e.value


# The base model's weights are checked against D, F and V before they are
# packed (D 128, F 256, V 16, two layers).
def _dec_weights(**over):
    Dm, Fm, Vm = 128, 256, 16
    layer = dict(attn_norm=torch.ones(Dm), mlp_norm=torch.ones(Dm), Wq=torch.zeros(Dm, Dm), Wk=torch.zeros(Dm, Dm),
                 Wv=torch.zeros(Dm, Dm), Wo=torch.zeros(Dm, Dm), W_gate=torch.zeros(Fm, Dm), W_up=torch.zeros(Fm, Dm),
                 W_down=torch.zeros(Dm, Fm))
    a = dict(embed=torch.zeros(Vm, Dm), layers=[dict(layer), dict(layer)], final_norm=torch.ones(Dm),
             lm_head=torch.zeros(Vm, Dm))
    for k, v in over.items():
        if k.startswith("layer1_"):
            a["layers"][1][k[len("layer1_"):]] = v
        else:
            a[k] = v
    return a


DECODER_CASES = {
    "width not a multiple of 128": dict(embed=torch.zeros(16, 96)),
    "LM head over another vocabulary": dict(lm_head=torch.zeros(17, 128)),
    "final norm too short": dict(final_norm=torch.ones(127)),
    "second layer's down projection too narrow": dict(layer1_W_down=torch.zeros(128, 128)),
    "second layer's up projection of another width": dict(layer1_W_up=torch.zeros(128, 128)),
    "second layer without an output projection": dict(layer1_Wo=None),
    "second layer's attention norm too long": dict(layer1_attn_norm=torch.ones(129)),
}


@pytest.mark.parametrize("case", sorted(DECODER_CASES))
def test_decoder_refuses_inconsistent_weights(mb, case):
    a = _dec_weights(**DECODER_CASES[case])
    with pytest.raises(ValueError) as e:
        mb.Decoder(a["embed"], a["layers"], a["final_norm"], a["lm_head"])
    assert "CUDA tensors" not in str(e.value)


def test_decoder_well_formed_reaches_the_device_check(mb):
    a = _dec_weights()
    with pytest.raises(ValueError, match="CUDA tensors"):
        mb.Decoder(a["embed"], a["layers"], a["final_norm"], a["lm_head"])
