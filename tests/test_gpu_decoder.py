"""The base model's forward over the tree tokens (tree_decoding) on the GPU
against the fp64 decoder oracle.

Small LLaMA-shaped models (hd 128, two heads, two layers) over B sequences'
trees at ragged cache lengths: the logits, the final residual stream and the
k/v rows the forward writes into the caches.  The kernels round the
normalised activations, q/k/v, the attention output and the SwiGLU
activation to bf16 between their fp32-accumulated products; the oracle keeps
everything in fp64.  Each such rounding moves its operand by at most 2^-9
relative, i.e. the product it feeds by about 2^-9/sqrt(3) of its RMS; about
six of them per layer, adding in quadrature over two layers and the LM head,
give an RMS error near 5e-3 of the output's RMS.  The bounds below are twice
that for the RMS and eight times for the largest element.
"""

import numpy as np
import pytest
import torch

import oracle.decoder_oracle as Dm
import oracle.medusa_oracle as O

pytestmark = pytest.mark.gpu

RMS_TOL, MAX_TOL = 1e-2, 4e-2


@pytest.fixture(scope="module")
def mb(built):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import speculative_decoding_heads_b200 as mb
    return mb


def _bf(a):
    """Round to bf16 (as the device tensors hold it) and back to fp64."""
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def _model(rng, D, F, V, nl, s=0.06):
    layers = []
    for _ in range(nl):
        layers.append({"attn_norm": _bf(1.0 + 0.1 * rng.normal(size=D)), "Wq": _bf(s * rng.normal(size=(D, D))),
                       "Wk": _bf(s * rng.normal(size=(D, D))), "Wv": _bf(s * rng.normal(size=(D, D))),
                       "Wo": _bf(s * rng.normal(size=(D, D))), "mlp_norm": _bf(1.0 + 0.1 * rng.normal(size=D)),
                       "W_gate": _bf(s * rng.normal(size=(F, D))), "W_up": _bf(s * rng.normal(size=(F, D))),
                       "W_down": _bf(s * rng.normal(size=(D, F)))})
    return (_bf(rng.normal(size=(V, D))), layers, _bf(1.0 + 0.1 * rng.normal(size=D)),
            _bf(s * rng.normal(size=(V, D))))


def _close(got, ref, what):
    err = got - ref
    rms = np.sqrt(np.mean(ref * ref))
    e_rms, e_max = np.sqrt(np.mean(err * err)) / rms, np.abs(err).max() / rms
    assert e_rms <= RMS_TOL and e_max <= MAX_TOL, f"{what}: rms err {e_rms:.2e}, max err {e_max:.2e} of the RMS"
    return e_rms, e_max


@pytest.mark.parametrize("B,lens,choices,lcap", [
    (2, [37, 70], ("ranksum", 3, 2, 14), 0),        # T 15: one pass of 64 tokens
    (4, [5, 130, 64, 0], ("ranksum", 4, 3, 20), 0),  # T 21: 84 tokens, one pass of 128; an empty prefix
    (1, [300], ("ranksum", 5, 10, 63), 0),           # T 64: the 7B tree, one full pass
    (3, [10, 200, 77], ("ranksum", 5, 10, 63), 0),   # 192 tokens: one pass of 256
    (5, [3, 90, 0, 41, 260], ("ranksum", 5, 10, 63), 0),   # 320 tokens: passes of 256 and 64 rows
    (3, [0, 1, 700], ("ranksum", 3, 2, 14), 800),    # a larger cache, with near-empty prefixes
    (1, [900], ("ranksum", 5, 10, 63), 1000),        # the 7B tree over a longer prefix
])
def test_tree_decode_matches_oracle(mb, B, lens, choices, lcap):
    rng = np.random.default_rng(B * 100 + len(choices))
    D, F, V, nl, H = 256, 384, 1000, 2, 2
    _, K, topk, n = choices
    ch = O.ranksum_choices(K, topk, n)
    tr = O.tree_tables(ch, K, topk)
    T = tr["T"]
    Lcap = max(max(lens) + T + 3, lcap)
    embed, layers, final_norm, lm_head = _model(rng, D, F, V, nl)
    tokens = rng.integers(0, V, size=(B, T))
    kc = _bf(rng.normal(size=(nl, B, H, Lcap, 128)))
    vc = _bf(rng.normal(size=(nl, B, H, Lcap, 128)))
    # oracle, one sequence at a time
    ref_logits, ref_hid, ref_k, ref_v = [], [], [], []
    for b in range(B):
        lg, hid, kcs, vcs = Dm.tree_forward(tr, tokens[b], embed, layers, final_norm, lm_head,
                                            [kc[l, b] for l in range(nl)], [vc[l, b] for l in range(nl)], lens[b], H)
        ref_logits.append(lg)
        ref_hid.append(hid)
        ref_k.append(np.stack(kcs))
        ref_v.append(np.stack(vcs))
    ref_logits, ref_hid = np.concatenate(ref_logits), np.concatenate(ref_hid)
    # device
    tree = mb.Tree(ch, K, topk)
    cuda = lambda a, dt: torch.from_numpy(np.asarray(a)).to(device="cuda", dtype=dt)
    model = mb.Decoder(cuda(embed, torch.float32), [{k: cuda(v, torch.float32) for k, v in ly.items()} for ly in layers],
                       cuda(final_norm, torch.float32), cuda(lm_head, torch.float32))
    k_dev, v_dev = cuda(kc, torch.bfloat16), cuda(vc, torch.bfloat16)
    logits = torch.empty((B * T, V), device="cuda")
    hidden = torch.empty((B * T, D), device="cuda")
    ws = mb.workspace(mb.medusa_tree_decode_workspace_size(tree, model, B))
    mb.medusa_tree_decode(tree, model, cuda(tokens, torch.int32), k_dev, v_dev, cuda(lens, torch.int32), logits, ws,
                          hidden=hidden)
    torch.cuda.synchronize()
    assert mb.device_status(clear=True) == (0, 0)
    e1 = _close(logits.double().cpu().numpy(), ref_logits, "logits")
    e2 = _close(hidden.double().cpu().numpy(), ref_hid, "final residual stream")
    kd, vd = k_dev.double().cpu().numpy(), v_dev.double().cpu().numpy()
    for b in range(B):
        L = lens[b]
        for l in range(nl):
            # prefix rows and rows past the tree untouched; the tree's own rows as the oracle's
            assert np.array_equal(kd[l, b, :, :L], kc[l, b, :, :L]) and np.array_equal(vd[l, b, :, :L], vc[l, b, :, :L])
            assert np.array_equal(kd[l, b, :, L + T:], kc[l, b, :, L + T:])
            _close(kd[l, b, :, L:L + T], ref_k[b][l][:, L:L + T], f"k rows of layer {l}, sequence {b}")
            _close(vd[l, b, :, L:L + T], ref_v[b][l][:, L:L + T], f"v rows of layer {l}, sequence {b}")
    # the greedy choice agrees wherever the oracle's top two logits are well apart
    top2 = np.sort(ref_logits, axis=1)[:, -2:]
    clear = (top2[:, 1] - top2[:, 0]) > 2 * MAX_TOL * np.sqrt(np.mean(ref_logits ** 2))
    assert clear.any()
    assert np.array_equal(logits.cpu().numpy().argmax(1)[clear], ref_logits.argmax(1)[clear])
    print(f"B {B} T {T}: logits rms/max err {e1[0]:.1e}/{e1[1]:.1e}, hidden {e2[0]:.1e}/{e2[1]:.1e}")


def test_tree_decode_rejects_overflow_on_device(mb):
    rng = np.random.default_rng(9)
    D, F, V, nl = 128, 128, 300, 1
    ch = O.ranksum_choices(3, 2, 6)
    tree = mb.Tree(ch, 3, 2)
    embed, layers, final_norm, lm_head = _model(rng, D, F, V, nl)
    cuda = lambda a, dt: torch.from_numpy(np.asarray(a)).to(device="cuda", dtype=dt)
    model = mb.Decoder(cuda(embed, torch.float32), [{k: cuda(v, torch.float32) for k, v in ly.items()} for ly in layers],
                       cuda(final_norm, torch.float32), cuda(lm_head, torch.float32))
    Lcap = 20
    kc = torch.zeros((nl, 1, 1, Lcap, 128), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    logits = torch.empty((tree.T, V), device="cuda")
    ws = mb.workspace(mb.medusa_tree_decode_workspace_size(tree, model, 1))
    mb.medusa_tree_decode(tree, model, torch.zeros((1, tree.T), dtype=torch.int32, device="cuda"), kc, vc,
                          torch.tensor([Lcap - tree.T + 1], dtype=torch.int32, device="cuda"), logits, ws)
    torch.cuda.synchronize()
    st, _ = mb.device_status(clear=True)
    assert st == mb.MEDUSA_ERR_DEVICE_CHECK
    assert not kc.any() and not vc.any(), "nothing is written past the cache"
