"""The seeded input generator: determinism, distribution, bf16 rounding, slices.

The generator holds none of the method's arithmetic; these checks make sure
the draws are what the workload recipe says (N(0, sigma^2), uniform ids,
ragged prefix lengths) and that any slice can be regenerated on its own.
"""

import numpy as np
import torch

from synth import gen, inputs, workloads


def test_deterministic_and_distinct_streams():
    a = gen.normal_f32(7, 3, 1000, 1.0)
    b = gen.normal_f32(7, 3, 1000, 1.0)
    c = gen.normal_f32(7, 4, 1000, 1.0)
    d = gen.normal_f32(8, 3, 1000, 1.0)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c) and not np.array_equal(a, d)


def test_known_splitmix_values():
    # splitmix64 reference outputs for state increments from 0 (public test vector:
    # seed 0 gives 0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F)
    with np.errstate(over="ignore"):
        xs = gen._mix64(np.arange(1, 4, dtype=np.uint64) * gen.GAMMA)
    assert [int(x) for x in xs] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_normal_moments_and_range():
    x = gen.normal_f32(1, 1, 2_000_000, 3.0).astype(np.float64)
    assert abs(x.mean()) < 0.01
    assert abs(x.std() - 3.0) < 0.01
    assert np.abs(x).max() <= 3.0 * 2 * np.sqrt(3) + 1e-6   # Irwin-Hall support


def test_bf16_rounding_matches_torch():
    x = gen.normal_f32(2, 2, 100_000, 0.02)
    ours = gen.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(gen.normal_bf16_bits(2, 2, 100_000, 0.02), ours)


def test_chunked_and_sampled_agree():
    n = (1 << 22) + 12345                     # crosses a chunk boundary
    full = gen.normal_bf16_bits(5, 9, n, 1.0)
    idx = np.array([0, 1, (1 << 22) - 1, 1 << 22, n - 1])
    assert np.array_equal(gen.f32_to_bf16_bits(gen.normal_at(5, 9, idx, 1.0, False)), full[idx])
    part = gen.normal_bf16_bits(5, 9, 1000, 1.0, offset=(1 << 22) - 500)
    assert np.array_equal(part, full[(1 << 22) - 500:(1 << 22) + 500])


def test_uniform_ranges():
    r = gen.uniform_int(3, 9, 100_000, 32000)
    assert r.min() >= 0 and r.max() < 32000 and abs(r.mean() - 16000) < 200
    u = gen.uniform_01(3, 10, 100_000)
    assert u.min() >= 0 and u.max() < 1 and abs(u.mean() - 0.5) < 0.01


def test_ragged_prefix_lengths():
    w = workloads.get("vicuna13b_bs8_ragged")
    L = w.prefix_lens()
    assert L.shape == (8,) and L.min() >= 256 and L.max() <= 4096
    assert np.array_equal(L, w.prefix_lens())


def test_planting_makes_child_the_argmax():
    tree_tokens = np.array([[5, 1, 2, 3, 4]])
    parent = np.array([-1, 0, 0, 1, 1])
    z = gen.normal_f32(11, 8, 5 * 10, 3.0).reshape(1, 5, 10)
    before = z.copy()
    gen.plant_agreement(z, tree_tokens, parent, 1.0, 11)
    for i, kids in [(0, [1, 2]), (1, [3, 4])]:
        tok = int(np.argmax(z[0, i]))
        assert tok in [tree_tokens[0, c] for c in kids]
        assert z[0, i, tok] == np.float32(before[0, i].max() + np.float32(5.0))
    for i in (2, 3, 4):                         # leaves are never changed
        assert np.array_equal(z[0, i], before[0, i])
    z2 = before.copy()
    gen.plant_agreement(z2, tree_tokens, parent, 0.0, 11)
    assert np.array_equal(z2, before)


def test_workload_metric_bytes():
    w = workloads.get("vicuna7b_bs1_L1024")
    assert w.metric_bytes() == 2_048_958_464
    assert w.T == 64 and w.Lcap == 1088


def test_slice_helpers_match_full_draws():
    w = workloads.shrink(workloads.get("vicuna7b_bs1_L1024"), layers=2, H=3, prefix=10, n_nodes=5, d=256, V=100)
    kc = inputs.values(inputs.kv_cache(w, "k"))
    assert np.array_equal(inputs.values(inputs.kv_slice(w, "k", 1, 0, 2)), kc[1, 0, 2])
    q = inputs.values(inputs.queries(w))
    assert np.array_equal(inputs.q_slice(w, 1, 0, 2), q[1, 0, :, 2, :])
    wk = inputs.values(inputs.wout(w, 1))
    assert np.array_equal(inputs.wout_rows(w, 1, np.array([0, 7])), wk[[0, 7]])
