"""The five synthetic Medusa verification-step workloads and their input recipe.

Each workload gives the shapes, dtypes, seeds and value distributions of one
verification step.  The shapes are those of Vicuna-7B / 13B / 33B (hidden
size, vocabulary, layers, attention heads, head dim 128); weights and
activations are random draws from ``synth.gen`` because no trained weights or
evaluation prompts are used.  Nothing here computes any part of the method:
the candidate tree is described only by its construction parameters
(K heads, top-k per head, node count), and each side builds it on its own.
"""

from __future__ import annotations

import dataclasses
from typing import Optional, Tuple

import numpy as np

from . import gen


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: str            # "f32" or "bf16" (weights, hidden state, q, K/V)
    B: int                # sequences
    d: int                # hidden size
    V: int                # vocabulary
    K: int                # Medusa heads
    topk: int             # candidates per head
    n_nodes: int          # tree nodes excluding the root
    layers: int
    H: int                # attention heads
    hd: int               # head dim
    prefix: Optional[int]               # fixed cached prefix length L_b (None: ragged)
    prefix_range: Optional[Tuple[int, int]] = None  # ragged L_b ~ U[lo, hi]
    seed: int = 1000
    w_sigma: float = 0.02
    h_sigma: float = 1.0
    kv_sigma: float = 1.0
    q_sigma: float = 1.0
    logit_sigma: float = 3.0
    agreement: float = 0.7
    modes: Tuple[str, ...] = ("greedy",)
    temperature: float = 0.7
    eps: float = 0.09
    alpha: float = 0.3

    @property
    def T(self) -> int:
        return self.n_nodes + 1

    def prefix_lens(self) -> np.ndarray:
        """Cached prefix length L_b of every sequence (int64 [B])."""
        if self.prefix is not None:
            return np.full(self.B, self.prefix, dtype=np.int64)
        lo, hi = self.prefix_range
        return lo + gen.uniform_int(self.seed, gen.TID_SEQLEN, self.B, hi - lo + 1)

    @property
    def Lcap(self) -> int:
        """Rows per (layer, sequence, head) slice of the KV cache."""
        return int(self.prefix_lens().max()) + self.T

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def metric_bytes(self) -> int:
        """Head weights read once plus the K/V rows the attention must read."""
        w = self.K * (self.d * self.d + self.d + self.V * self.d) * self.elem_bytes
        kv_rows = int((self.prefix_lens() + self.T).sum())
        kv = 2 * self.layers * self.H * self.hd * kv_rows * self.elem_bytes
        return w + kv


def _vicuna7b(**kw):
    base = dict(dtype="bf16", B=1, d=4096, V=32000, K=5, topk=10, n_nodes=63,
                layers=32, H=32, hd=128, prefix=1024)
    base.update(kw)
    return base


WORKLOADS = {
    "tiny_f32": Workload(name="tiny_f32", dtype="f32", B=1, d=256, V=1000, K=3, topk=2,
                         n_nodes=14, layers=1, H=4, hd=64, prefix=64, seed=1000),
    "vicuna7b_bs1_L1024": Workload(name="vicuna7b_bs1_L1024", seed=1001, **_vicuna7b()),
    "vicuna7b_bs1_L4096_typical": Workload(name="vicuna7b_bs1_L4096_typical", seed=1002,
                                           logit_sigma=2.0, agreement=0.6,
                                           modes=("typical",), **_vicuna7b(prefix=4096)),
    "vicuna13b_bs8_ragged": Workload(name="vicuna13b_bs8_ragged", dtype="bf16", B=8, d=5120,
                                     V=32000, K=4, topk=8, n_nodes=48, layers=40, H=40, hd=128,
                                     prefix=None, prefix_range=(256, 4096), seed=1003,
                                     modes=("greedy", "typical")),
}
for _n in (16, 32, 64, 128):
    WORKLOADS[f"vicuna33b_bs4_L8192_N{_n}"] = Workload(
        name=f"vicuna33b_bs4_L8192_N{_n}", dtype="bf16", B=4, d=6656, V=32000, K=5, topk=10,
        n_nodes=_n, layers=60, H=52, hd=128, prefix=8192, seed=1004, agreement=0.65)

# The workload the single-GPU benchmark times (Vicuna-7B shape, batch 1).
BENCH_WORKLOAD = "vicuna7b_bs1_L1024"


def get(name: str) -> Workload:
    return WORKLOADS[name]


def shrink(w: Workload, **kw) -> Workload:
    """A smaller copy of a workload (parity cases the oracle finishes in seconds)."""
    return dataclasses.replace(w, **kw)
