"""The C ABI on a machine without a GPU: the library loads, exports every
symbol the header declares, and its host-side tree builder agrees exactly
with the oracle's independent one.  No compute call is made here."""

import ctypes
import itertools
import os
import re

import numpy as np
import pytest

import oracle.medusa_oracle as O

REPO = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(REPO, "include", "medusa_b200.h")


@pytest.fixture(scope="module")
def mb(built):
    import speculative_decoding_heads_b200 as mb
    return mb


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(medusa_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(mb):
    declared = header_functions()
    assert declared, "header parse found no functions"
    lib = ctypes.CDLL(mb.LIB_PATH)
    missing = [f for f in declared if not hasattr(lib, f)]
    assert not missing, missing
    assert sorted(mb.EXPORTED) == declared


def test_abi_version(mb):
    assert mb.abi_version() == 7


def _compare_tables(mb, choices, K, topk):
    ref = O.tree_tables(choices, K, topk)
    t = mb.Tree(choices, K, topk, upload=False)
    assert (t.T, t.P, t.D) == (ref["T"], ref["P"], ref["D"])
    tab = t.tables()
    assert tab["tree_indices"] == list(ref["tree_indices"])
    assert tab["parent"] == list(ref["parent"])
    assert tab["depth"] == list(ref["depth"])
    assert tab["retrieve"] == [list(r) for r in ref["retrieve"]]
    W = (ref["T"] + 63) // 64
    for i in range(ref["T"]):
        bits = [(tab["anc"][i][j // 64] >> (j % 64)) & 1 for j in range(ref["T"])]
        assert bits == [int(x) for x in ref["anc"][i]]
        assert len(tab["anc"][i]) == W
    t.close()


@pytest.mark.parametrize("K,topk,n", [(3, 2, 14), (5, 10, 63), (4, 8, 48), (5, 10, 16), (5, 10, 32),
                                      (5, 10, 64), (5, 10, 128), (5, 1, 5), (2, 2, 6), (16, 32, 255)])
def test_ranksum_and_tables_match_oracle(mb, K, topk, n):
    ours = mb.medusa_tree_choices_ranksum(K, topk, n)
    if K * topk <= 60:
        assert ours == O.ranksum_choices(K, topk, n)
    _compare_tables(mb, ours, K, topk)


def test_worked_example_tables(mb):
    _compare_tables(mb, [(0,), (1,), (0, 0), (0, 1), (1, 0), (1, 1)], 2, 2)


def test_random_trees_match_oracle(mb):
    rng = np.random.default_rng(7)
    for _ in range(25):
        K, topk = int(rng.integers(1, 6)), int(rng.integers(1, 6))
        allt = [t for n in range(1, K + 1) for t in itertools.product(range(topk), repeat=n)]
        pick = set()
        for i in rng.permutation(len(allt))[: int(rng.integers(0, min(60, len(allt)) + 1))]:
            t = allt[i]
            for j in range(1, len(t) + 1):
                pick.add(t[:j])
        choices = list(pick)
        rng.shuffle(choices)
        _compare_tables(mb, choices, K, topk)


@pytest.mark.parametrize("choices,K,topk", [
    ([(0, 1)], 2, 2),                 # parent (0,) missing
    ([(0,), (0,)], 2, 2),             # duplicate
    ([(2,)], 2, 2),                   # rank >= topk
    ([(0, 0, 0)], 2, 2),              # longer than K
    ([(0,)], 0, 2),                   # K out of range
    ([(0,)], 2, 33),                  # topk above the maximum
])
def test_tree_create_rejects_bad_trees(mb, choices, K, topk):
    with pytest.raises(mb.MedusaError) as ei:
        mb.Tree(choices, K, topk, upload=False)
    assert ei.value.code == mb.MEDUSA_ERR_INVALID_ARG


def test_ranksum_rejects_too_many_nodes(mb):
    with pytest.raises(mb.MedusaError):
        mb.medusa_tree_choices_ranksum(2, 2, 7)          # only 6 tuples exist
    with pytest.raises(mb.MedusaError):
        mb.medusa_tree_choices_ranksum(5, 10, 256)       # T would exceed 256


def test_decoder_pack_rows(mb):
    # q/k/v: within each head of 128 rows, row 2j holds feature j and row 2j+1 feature j + 64
    rows = mb.medusa_decoder_pack_rows(0, 256)
    assert sorted(rows) == list(range(256))
    for r in range(256):
        head, lr = divmod(r, 128)
        assert rows[r] == head * 128 + (lr // 2 if lr % 2 == 0 else 64 + lr // 2)
    # gate/up: row 2j is gate row j, row 2j+1 is up row j (index F + j of [W_gate; W_up])
    F = 384
    gu = mb.medusa_decoder_pack_rows(1, 2 * F)
    assert sorted(gu) == list(range(2 * F))
    assert gu[:4] == [0, F, 1, F + 1] and gu[-1] == 2 * F - 1
    with pytest.raises(mb.MedusaError):
        mb.medusa_decoder_pack_rows(0, 100)
