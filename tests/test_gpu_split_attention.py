"""Tree attention split along the cached prefix, on one GPU.

Each rank's window is one medusa_tree_attention_split call (the G calls run
one after another; none waits on another), and medusa_attention_combine
merges the G partials.  Checked against the oracle's window partials, its
log-sum-exp combine and the unsplit oracle, and against the unsplit call.
"""

import numpy as np
import pytest
import torch

import oracle.medusa_oracle as O
from synth import gen, inputs as I
from helpers import ATTN_ATOL, SMALL, oracle_tree

pytestmark = pytest.mark.gpu
LSE_ATOL = 1e-3


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


def _np(t):
    return t.detach().cpu().numpy().astype(np.float64)


def _case(mb, dev, w):
    t = dev.materialise(w, fill=False)
    dev.fill_normal(t["q"], w.seed, gen.TID_Q, w.q_sigma)
    dev.fill_normal(t["k_cache"], w.seed, gen.TID_KCACHE, w.kv_sigma)
    dev.fill_normal(t["v_cache"], w.seed, gen.TID_VCACHE, w.kv_sigma)
    tree = mb.Tree(O.ranksum_choices(w.K, w.topk, w.n_nodes), w.K, w.topk)
    return t, tree


def _split(mb, t, tree, scale, G):
    shape = tuple(t["attn_out"].shape)
    outs = torch.empty((G,) + shape, device="cuda")
    lses = torch.empty((G,) + shape[:-1], device="cuda")
    for r in range(G):
        mb.medusa_tree_attention_split(tree, t["q"], t["k_cache"], t["v_cache"], t["seq_lens"], scale, r, G,
                                       outs[r], lses[r])
    out = torch.empty(shape, device="cuda")
    lse = torch.empty(shape[:-1], device="cuda")
    mb.medusa_attention_combine(outs, lses, out, lse)
    torch.cuda.synchronize()
    return outs, lses, out, lse


def _shrunk(name, **kw):
    from synth.workloads import shrink
    return shrink(SMALL[name], **kw)


CASES = [("v7b_small", 1), ("v7b_small", 2), ("v7b_small", 3), ("v13b_small", 5), ("b3_small", 4),
         ("v7b_many", 3)]


@pytest.mark.parametrize("name,G", CASES)
def test_split_attention_matches_oracle_and_unsplit(mb, dev, name, G):
    w = _shrunk("v7b_small", layers=2, H=160, prefix=200) if name == "v7b_many" else SMALL[name]
    tr = oracle_tree(w)
    t, tree = _case(mb, dev, w)
    scale = O.attention_scale(w.hd)
    mb.medusa_tree_attention(tree, t["q"], t["k_cache"], t["v_cache"], t["seq_lens"], scale, t["attn_out"])
    outs, lses, out, lse = _split(mb, t, tree, scale, G)
    st, det = mb.device_status(clear=True)
    assert (st, det) == (0, 0)

    q = I.values(I.queries(w))
    kc = I.values(I.kv_cache(w, "k"))
    vc = I.values(I.kv_cache(w, "v"))
    lens = w.prefix_lens()
    ref = O.tree_attention(tr, q, kc, vc, lens, scale)
    assert np.abs(_np(out) - ref).max() <= ATTN_ATOL[w.dtype]
    assert np.abs(_np(out) - _np(t["attn_out"])).max() <= ATTN_ATOL[w.dtype]

    # per-rank partials and the combined lse on sampled slices
    rng = np.random.default_rng(G)
    picks = {(0, 0, 0), (w.layers - 1, w.B - 1, w.H - 1)}
    picks |= {(int(rng.integers(w.layers)), int(rng.integers(w.B)), int(rng.integers(w.H))) for _ in range(4)}
    for (l, b, e) in sorted(picks):
        L = int(lens[b])
        qs, ks, vs = q[l, b, :, e, :], kc[l, b, e], vc[l, b, e]
        parts_o, parts_l = [], []
        for r in range(G):
            lo, hi = O.attention_window(G, r, L)
            o_r, l_r = O.tree_attention_window_slice(tr, qs, ks, vs, L, scale, lo, hi, with_tree=(r == G - 1))
            assert np.abs(_np(outs[r, l, b, :, e, :]) - o_r).max() <= ATTN_ATOL[w.dtype], (l, b, e, r)
            assert np.abs(_np(lses[r, l, b, :, e]) - l_r).max() <= LSE_ATOL, (l, b, e, r)
            parts_o.append(o_r)
            parts_l.append(l_r)
        _, lse_ref = O.combine_partials(np.stack(parts_o), np.stack(parts_l))
        assert np.abs(_np(lse[l, b, :, e]) - lse_ref).max() <= LSE_ATOL, (l, b, e)


def test_combine_kernel_matches_oracle_with_empty_windows(mb):
    rng = np.random.default_rng(3)
    G, rows, hd = 5, 700, 128
    outs = rng.normal(size=(G, rows, hd)).astype(np.float32)
    lses = rng.normal(scale=4.0, size=(G, rows)).astype(np.float32)
    lses[:, 10] = -np.inf                     # no window held a key
    lses[1:, 11] = -np.inf                    # one window only
    lses[0, 12:40] = -np.inf                  # some windows empty
    ref_o, ref_l = O.combine_partials(outs.astype(np.float64), lses.astype(np.float64))
    out = torch.empty(rows, hd, device="cuda")
    lse = torch.empty(rows, device="cuda")
    mb.medusa_attention_combine(torch.from_numpy(outs).cuda(), torch.from_numpy(lses).cuda(), out, lse)
    torch.cuda.synchronize()
    assert np.allclose(_np(out), ref_o, atol=1e-5, rtol=1e-5)
    got_l = _np(lse)
    assert np.all(got_l[10] == -np.inf) and not _np(out)[10].any()
    fin = np.isfinite(ref_l)
    assert np.allclose(got_l[fin], ref_l[fin], atol=1e-5, rtol=1e-5)


def test_split_with_an_empty_window_sets_the_device_check(mb, dev):
    w = SMALL["b3_small"]                     # one sequence has a 14-token prefix
    t, tree = _case(mb, dev, w)
    shape = tuple(t["attn_out"].shape)
    out = torch.empty(shape, device="cuda")
    lse = torch.empty(shape[:-1], device="cuda")
    mb.medusa_tree_attention_split(tree, t["q"], t["k_cache"], t["v_cache"], t["seq_lens"],
                                   O.attention_scale(w.hd), 0, 16, out, lse)
    torch.cuda.synchronize()
    st, _ = mb.device_status(clear=True)
    assert st == mb.MEDUSA_ERR_DEVICE_CHECK


@pytest.mark.parametrize("name", ["tiny_f32", "v33b_small"])
def test_split_rejects_unsupported_shapes(mb, dev, name):
    w = SMALL[name]
    t, tree = _case(mb, dev, w)
    shape = tuple(t["attn_out"].shape)
    with pytest.raises(mb.MedusaError) as e:
        mb.medusa_tree_attention_split(tree, t["q"], t["k_cache"], t["v_cache"], t["seq_lens"],
                                       O.attention_scale(w.hd), 0, 2, torch.empty(shape, device="cuda"),
                                       torch.empty(shape[:-1], device="cuda"))
    assert e.value.code == mb.MEDUSA_ERR_UNSUPPORTED


@pytest.mark.parametrize("name,G", [("v7b_small", 2), ("v13b_small", 3), ("b3_small", 4)])
def test_rescaled_partials_sum_to_the_combine(mb, dev, name, G):
    """medusa_attention_rescale: each rank scales its own window output; the sum over ranks (what
    the all-reduce computes) equals medusa_attention_combine's output and lse."""
    w = SMALL[name]
    t, tree = _case(mb, dev, w)
    outs, lses, out, lse = _split(mb, t, tree, O.attention_scale(w.hd), G)
    acc = torch.zeros_like(out)
    lse2 = torch.empty_like(lse)
    for r in range(G):
        part = outs[r].clone()
        mb.medusa_attention_rescale(lses, r, part, lse2)
        acc += part
    torch.cuda.synchronize()
    assert (acc - out).abs().max().item() <= 1e-5
    assert torch.allclose(lse2, lse, atol=1e-6, rtol=0)


def test_rescale_kernel_matches_oracle_with_empty_windows(mb):
    rng = np.random.default_rng(4)
    G, rows, hd = 4, 500, 128
    outs = rng.normal(size=(G, rows, hd)).astype(np.float32)
    lses = rng.normal(scale=4.0, size=(G, rows)).astype(np.float32)
    lses[:, 10] = -np.inf
    lses[1:, 11] = -np.inf
    lses[0, 12:40] = -np.inf
    ref_o, ref_l = O.combine_partials(outs.astype(np.float64), lses.astype(np.float64))
    lg = torch.from_numpy(lses).cuda()
    acc = torch.zeros(rows, hd, device="cuda")
    lse = torch.empty(rows, device="cuda")
    for r in range(G):
        part = torch.from_numpy(outs[r]).cuda()
        mb.medusa_attention_rescale(lg, r, part, lse)
        acc += part
    torch.cuda.synchronize()
    assert np.allclose(_np(acc), ref_o, atol=1e-5, rtol=1e-5)
    got_l = _np(lse)
    assert np.all(got_l[10] == -np.inf) and not _np(acc)[10].any()
    fin = np.isfinite(ref_l)
    assert np.allclose(got_l[fin], ref_l[fin], atol=1e-5, rtol=1e-5)
