"""Seeded, counter-based synthetic input generator (host side, numpy).

This module produces every input of the Medusa verification step that the
tests and the benchmark feed to both the CUDA library and the oracle: the
hidden state, head weights, attention queries, the KV cache, base logits,
root tokens and ragged prefix lengths.  It holds none of the method's
arithmetic; it only draws numbers.

Definition (restated identically by ``synth/csrc/synth.cu`` for the device):

* ``mix64(x)`` is the splitmix64 output function (Vigna's public
  finaliser): ``x ^= x >> 30; x *= 0xBF58476D1CE4E5B9; x ^= x >> 27;
  x *= 0x94D049BB133111EB; x ^= x >> 31`` in wrapping 64-bit arithmetic.
* A stream is keyed by ``(seed, tensor_id)``:
  ``key = mix64(mix64(seed) + tensor_id * GAMMA)`` with the golden gamma
  ``GAMMA = 0x9E3779B97F4A7C15``.
* Element ``i`` of a stream is ``x_i = mix64(key + (i + 1) * GAMMA)``.
* Normal(0, sigma^2): split ``x_i`` into four 16-bit fields ``b0..b3``;
  ``c = b0 + b1 + b2 + b3 - 131070`` is an exact integer with mean 0 and
  variance ``(65536^2 - 1) / 3``; the value is the single IEEE fp32 product
  ``float32(c) * float32(sigma * sqrt(3) / 65536)`` (Irwin-Hall of order 4,
  unit variance to 1e-10).  One fp32 multiply is correctly rounded on both
  host and device, so the two sides agree bit for bit.
* bf16 values are the round-to-nearest-even of that fp32 value, done with
  integer arithmetic on the bit pattern.
* Uniform integer in ``[0, n)``: ``((x_i >> 32) * n) >> 32``.
* Uniform real in ``[0, 1)``: ``(x_i >> 40) * 2^-24`` (exact in fp32).

Large tensors are produced in chunks on a thread pool (numpy releases the
GIL inside its ufuncs), and any slice can be regenerated on its own from the
flat indices, which is how parity checks at full size sample outputs.
"""

from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
M1 = np.uint64(0xBF58476D1CE4E5B9)
M2 = np.uint64(0x94D049BB133111EB)
_S30 = np.uint64(30)
_S27 = np.uint64(27)
_S31 = np.uint64(31)
_S16 = np.uint64(16)
_S32 = np.uint64(32)
_S40 = np.uint64(40)
_MASK16 = np.uint64(0xFFFF)

# Tensor ids of the step's inputs.  A sub-seed s (used to re-draw a tensor
# whose values would sit too close to a decision boundary) shifts the id by
# 64 * s, so every (tensor, sub-seed) pair is its own stream.
TID_H = 1
TID_W1 = 2
TID_B1 = 3
TID_WOUT = 4
TID_Q = 5
TID_KCACHE = 6
TID_VCACHE = 7
TID_BASE_LOGITS = 8
TID_ROOT = 9
TID_PLANT = 10
TID_SEQLEN = 11
TID_UNIFORM = 12          # one draw per sequence for the sampled next token
TID_DECODER = 1 << 20     # base-model weights: TID_DECODER + 9 * layer + matrix index; embed, final norm, LM head after
SUBSEED_STRIDE = 64

_CHUNK = 1 << 22


def _mix64(x: np.ndarray) -> np.ndarray:
    x = x ^ (x >> _S30)
    x = x * M1
    x = x ^ (x >> _S27)
    x = x * M2
    return x ^ (x >> _S31)


def stream_key(seed: int, tensor_id: int) -> np.uint64:
    """Key of the stream (seed, tensor_id)."""
    with np.errstate(over="ignore"):
        s = _mix64(np.array([seed], dtype=np.uint64))[0]
        k = _mix64(np.array([s + np.uint64(tensor_id) * GAMMA], dtype=np.uint64))[0]
    return np.uint64(k)


def raw64(seed: int, tensor_id: int, idx: np.ndarray) -> np.ndarray:
    """The 64-bit draws x_i for the flat indices ``idx`` (uint64 array)."""
    key = stream_key(seed, tensor_id)
    idx = np.asarray(idx, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(key + (idx + np.uint64(1)) * GAMMA)


def normal_scale(sigma: float) -> np.float32:
    """The fp32 constant that maps the centred Irwin-Hall integer to N(0, sigma^2)."""
    return np.float32(sigma * math.sqrt(3.0) / 65536.0)


def _normal_from_raw(x: np.ndarray, sigma: float) -> np.ndarray:
    c = ((x & _MASK16) + ((x >> _S16) & _MASK16) + ((x >> _S32) & _MASK16)
         + (x >> np.uint64(48))).astype(np.int64) - 131070
    return c.astype(np.float32) * normal_scale(sigma)


def f32_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16, returned as uint16 bit patterns."""
    b = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    return ((b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _pool_workers() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def _chunked(n: int, fn, out: np.ndarray) -> np.ndarray:
    starts = list(range(0, n, _CHUNK))
    if len(starts) <= 1:
        if n:
            out[:n] = fn(0, n)
        return out

    def work(s):
        e = min(n, s + _CHUNK)
        out[s:e] = fn(s, e)

    with ThreadPoolExecutor(_pool_workers()) as ex:
        list(ex.map(work, starts))
    return out


def normal_f32(seed: int, tensor_id: int, n: int, sigma: float, offset: int = 0) -> np.ndarray:
    """n consecutive N(0, sigma^2) fp32 draws starting at flat index ``offset``."""
    out = np.empty(n, dtype=np.float32)

    def fn(s, e):
        idx = np.arange(offset + s, offset + e, dtype=np.uint64)
        return _normal_from_raw(raw64(seed, tensor_id, idx), sigma)

    return _chunked(n, fn, out)


def normal_bf16_bits(seed: int, tensor_id: int, n: int, sigma: float, offset: int = 0) -> np.ndarray:
    """n consecutive N(0, sigma^2) draws rounded to bf16 (uint16 bit patterns)."""
    out = np.empty(n, dtype=np.uint16)

    def fn(s, e):
        idx = np.arange(offset + s, offset + e, dtype=np.uint64)
        return f32_to_bf16_bits(_normal_from_raw(raw64(seed, tensor_id, idx), sigma))

    return _chunked(n, fn, out)


def normal_at(seed: int, tensor_id: int, idx: np.ndarray, sigma: float, bf16: bool) -> np.ndarray:
    """Draws at arbitrary flat indices, as fp32 (bf16-rounded when ``bf16``)."""
    v = _normal_from_raw(raw64(seed, tensor_id, np.asarray(idx, dtype=np.uint64)), sigma)
    if bf16:
        return bf16_bits_to_f32(f32_to_bf16_bits(v))
    return v


def uniform_int(seed: int, tensor_id: int, n: int, hi: int, offset: int = 0) -> np.ndarray:
    """n integers uniform in [0, hi) (multiply-shift of the high 32 bits)."""
    idx = np.arange(offset, offset + n, dtype=np.uint64)
    x = raw64(seed, tensor_id, idx) >> _S32
    with np.errstate(over="ignore"):
        return ((x * np.uint64(hi)) >> _S32).astype(np.int64)


def uniform_01(seed: int, tensor_id: int, n: int, offset: int = 0) -> np.ndarray:
    """n reals uniform in [0, 1), each an exact multiple of 2^-24 (fp64 array)."""
    idx = np.arange(offset, offset + n, dtype=np.uint64)
    x = raw64(seed, tensor_id, idx) >> _S40
    return x.astype(np.float64) * (2.0 ** -24)


def plant_agreement(logits: np.ndarray, tree_tokens: np.ndarray, parent: np.ndarray,
                    q: float, seed: int, boost: float = 5.0) -> np.ndarray:
    """Plant head/base agreement into synthetic base logits, in place.

    ``logits`` is [B, T, V] fp32; ``tree_tokens`` [B, T]; ``parent`` [T]
    (parent[0] = -1).  For every sequence b and every node i that has
    children, draw u1 = U[0,1) at flat index 2*(b*T+i); when u1 < q, pick one
    child uniformly with u2 (index 2*(b*T+i)+1) and set that child's token
    logit in row (b, i) to (the row's maximum before the change) + boost.
    Leaves are never changed.  This stands in for a base model that agrees
    with the heads' guess with probability q at every node.
    """
    B, T, V = logits.shape
    children = [[] for _ in range(T)]
    for c in range(1, T):
        children[int(parent[c])].append(c)
    u = uniform_01(seed, TID_PLANT, 2 * B * T).reshape(B, T, 2)
    for b in range(B):
        for i in range(T):
            ch = children[i]
            if not ch or u[b, i, 0] >= q:
                continue
            c = ch[min(len(ch) - 1, int(u[b, i, 1] * len(ch)))]
            tok = int(tree_tokens[b, c])
            logits[b, i, tok] = np.float32(logits[b, i].max() + np.float32(boost))
    return logits
