"""Host materialisation of a workload's inputs (numpy).

Weights, hidden state, queries and K/V come back as the element type the GPU
reads: float32 arrays for "f32" workloads, uint16 bf16 bit patterns for
"bf16" ones (``values()`` widens either exactly to float64 for the oracle).
Base logits are always float32.  Sub-seeds re-draw the hidden state
(``sub_h``) or the base logits (``sub_logits``) when a draw lands too close to
a decision boundary.
"""

from __future__ import annotations

import numpy as np

from . import gen
from .workloads import Workload


def _tid(base: int, sub: int) -> int:
    return base + gen.SUBSEED_STRIDE * sub


def draw(w: Workload, tensor_id: int, shape, sigma: float, sub: int = 0, offset: int = 0):
    n = int(np.prod(shape))
    tid = _tid(tensor_id, sub)
    if w.dtype == "f32":
        return gen.normal_f32(w.seed, tid, n, sigma, offset).reshape(shape)
    return gen.normal_bf16_bits(w.seed, tid, n, sigma, offset).reshape(shape)


def values(a: np.ndarray) -> np.ndarray:
    """Exact float64 values of an array produced by ``draw``."""
    if a.dtype == np.uint16:
        return gen.bf16_bits_to_f32(a).astype(np.float64)
    return np.asarray(a, dtype=np.float64)


def hidden(w: Workload, sub_h: int = 0):
    return draw(w, gen.TID_H, (w.B, w.d), w.h_sigma, sub_h)


def w1(w: Workload, k: int = None):
    """W1 [K, d, d] (out x in), or head k's [d, d] slice."""
    if k is None:
        return draw(w, gen.TID_W1, (w.K, w.d, w.d), w.w_sigma)
    return draw(w, gen.TID_W1, (w.d, w.d), w.w_sigma, offset=k * w.d * w.d)


def b1(w: Workload):
    return draw(w, gen.TID_B1, (w.K, w.d), w.w_sigma)


def wout(w: Workload, k: int = None):
    """Wout [K, V, d], or head k's [V, d] slice."""
    if k is None:
        return draw(w, gen.TID_WOUT, (w.K, w.V, w.d), w.w_sigma)
    return draw(w, gen.TID_WOUT, (w.V, w.d), w.w_sigma, offset=k * w.V * w.d)


def wout_rows(w: Workload, k: int, rows: np.ndarray) -> np.ndarray:
    """Exact float64 values of the given rows of head k's Wout (sampled checks)."""
    rows = np.asarray(rows, dtype=np.int64)
    idx = (k * w.V * w.d + rows[:, None] * w.d + np.arange(w.d)[None, :]).reshape(-1)
    v = gen.normal_at(w.seed, gen.TID_WOUT, idx, w.w_sigma, w.dtype == "bf16")
    return v.astype(np.float64).reshape(len(rows), w.d)


def root_tokens(w: Workload) -> np.ndarray:
    return gen.uniform_int(w.seed, gen.TID_ROOT, w.B, w.V)


def q_shape(w: Workload):
    return (w.layers, w.B, w.T, w.H, w.hd)


def cache_shape(w: Workload):
    return (w.layers, w.B, w.H, w.Lcap, w.hd)


def queries(w: Workload):
    return draw(w, gen.TID_Q, q_shape(w), w.q_sigma)


def kv_cache(w: Workload, which: str):
    tid = gen.TID_KCACHE if which == "k" else gen.TID_VCACHE
    return draw(w, tid, cache_shape(w), w.kv_sigma)


def _slice_offset(w: Workload, l: int, b: int, e: int) -> int:
    return ((l * w.B + b) * w.H + e) * w.Lcap * w.hd


def kv_slice(w: Workload, which: str, l: int, b: int, e: int, rows: int = None):
    """One (layer, sequence, head) slice [rows, hd] of the K or V cache."""
    tid = gen.TID_KCACHE if which == "k" else gen.TID_VCACHE
    rows = w.Lcap if rows is None else rows
    return draw(w, tid, (rows, w.hd), w.kv_sigma, offset=_slice_offset(w, l, b, e))


def q_slice(w: Workload, l: int, b: int, e: int):
    """Queries [T, hd] of one (layer, sequence, head)."""
    T, H, hd = w.T, w.H, w.hd
    base = ((l * w.B + b) * T) * H * hd + e * hd
    idx = (base + np.arange(T)[:, None] * H * hd + np.arange(hd)[None, :]).reshape(-1)
    v = gen.normal_at(w.seed, gen.TID_Q, idx, w.q_sigma, w.dtype == "bf16")
    return v.astype(np.float64).reshape(T, hd)


def base_logits_raw(w: Workload, sub_logits: int = 0) -> np.ndarray:
    """Unplanted base logits [B, T, V] fp32, N(0, logit_sigma^2)."""
    n = w.B * w.T * w.V
    return gen.normal_f32(w.seed, _tid(gen.TID_BASE_LOGITS, sub_logits), n,
                          w.logit_sigma).reshape(w.B, w.T, w.V)


def base_logits(w: Workload, tree_tokens: np.ndarray, parent: np.ndarray,
                sub_logits: int = 0) -> np.ndarray:
    """Base logits with the workload's planted agreement at every tree node."""
    z = base_logits_raw(w, sub_logits)
    return gen.plant_agreement(z, tree_tokens, parent, w.agreement,
                               w.seed + 7919 * sub_logits)


def uniforms(w: Workload, sub: int = 0) -> np.ndarray:
    """One U[0, 1) draw per sequence (exact multiples of 2^-24, so fp32 holds them exactly)."""
    return gen.uniform_01(w.seed, _tid(gen.TID_UNIFORM, sub), w.B)
