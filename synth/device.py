"""Device-side synthetic inputs: the CUDA restatement of ``synth.gen``.

``fill_normal`` writes the same values ``gen.normal_f32`` /
``gen.normal_bf16_bits`` produce, directly into a device tensor, so that
multi-GB workloads (the KV cache of the 33B-shaped workload is ~53 GB) need
no host round trip.  ``plant`` is the device version of
``gen.plant_agreement``.  ``materialise`` allocates every input and output
buffer of one verification step for a workload.  Nothing here computes any
part of the Medusa step.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from . import gen
from .workloads import Workload

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmedusa_synth.so")
_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"{_LIB_PATH} missing; run the package build first")
        _lib = ctypes.CDLL(_LIB_PATH)
        _lib.synth_normal.restype = ctypes.c_int
        _lib.synth_normal.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint64,
                                      ctypes.c_uint64, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p]
        _lib.synth_plant.restype = ctypes.c_int
        _lib.synth_plant.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.c_double,
                                     ctypes.c_uint64, ctypes.c_uint64, ctypes.c_float,
                                     ctypes.c_void_p]
    return _lib


def _stream(stream):
    return ctypes.c_void_p((stream or torch.cuda.current_stream()).cuda_stream)


def fill_normal(t: torch.Tensor, seed: int, tensor_id: int, sigma: float, offset: int = 0,
                stream=None) -> torch.Tensor:
    assert t.is_cuda and t.is_contiguous() and t.dtype in (torch.float32, torch.bfloat16)
    rc = lib().synth_normal(ctypes.c_void_p(t.data_ptr()), t.numel(), int(t.dtype == torch.bfloat16),
                            seed, tensor_id, offset, float(gen.normal_scale(sigma)), _stream(stream))
    if rc != 0:
        raise RuntimeError(f"synth_normal failed with CUDA error {rc}")
    return t


def plant(logits: torch.Tensor, tree_tokens: torch.Tensor, parent: torch.Tensor, q: float,
          seed: int, boost: float = 5.0, stream=None) -> torch.Tensor:
    B, T, V = logits.shape
    rc = lib().synth_plant(ctypes.c_void_p(logits.data_ptr()), B, T, V,
                           ctypes.c_void_p(tree_tokens.data_ptr()), ctypes.c_void_p(parent.data_ptr()),
                           float(q), seed, gen.TID_PLANT, float(boost), _stream(stream))
    if rc != 0:
        raise RuntimeError(f"synth_plant failed with CUDA error {rc}")
    return logits


def _tdt(w: Workload):
    return torch.float32 if w.dtype == "f32" else torch.bfloat16


def materialise(w: Workload, sub_h: int = 0, sub_logits: int = 0, device="cuda",
                with_head_logits: bool = True, fill: bool = True) -> dict:
    """Every buffer of one step of ``w`` on the device; inputs drawn by the generator.

    ``base_logits`` hold the unplanted N(0, sigma^2) draws; the caller plants
    agreement once the tree tokens are known (``plant``).  ``fill=False``
    leaves the big inputs unfilled (sized buffers only).
    """
    dt = _tdt(w)
    T = w.T
    t = {}
    z = lambda shape, dtype: torch.empty(shape, dtype=dtype, device=device)
    t["h"] = z((w.B, w.d), dt)
    t["W1"] = z((w.K, w.d, w.d), dt)
    t["b1"] = z((w.K, w.d), dt)
    t["Wout"] = z((w.K, w.V, w.d), dt)
    t["q"] = z((w.layers, w.B, T, w.H, w.hd), dt)
    t["k_cache"] = z((w.layers, w.B, w.H, w.Lcap, w.hd), dt)
    t["v_cache"] = z((w.layers, w.B, w.H, w.Lcap, w.hd), dt)
    t["base_logits"] = z((w.B, T, w.V), torch.float32)
    t["root_tokens"] = torch.tensor(gen.uniform_int(w.seed, gen.TID_ROOT, w.B, w.V), dtype=torch.int32,
                                    device=device)
    t["seq_lens"] = torch.tensor(w.prefix_lens(), dtype=torch.int32, device=device)
    t["seq_lens0"] = t["seq_lens"].clone()
    if fill:
        sh = gen.SUBSEED_STRIDE
        fill_normal(t["h"], w.seed, gen.TID_H + sh * sub_h, w.h_sigma)
        fill_normal(t["W1"], w.seed, gen.TID_W1, w.w_sigma)
        fill_normal(t["b1"], w.seed, gen.TID_B1, w.w_sigma)
        fill_normal(t["Wout"], w.seed, gen.TID_WOUT, w.w_sigma)
        fill_normal(t["q"], w.seed, gen.TID_Q, w.q_sigma)
        fill_normal(t["k_cache"], w.seed, gen.TID_KCACHE, w.kv_sigma)
        fill_normal(t["v_cache"], w.seed, gen.TID_VCACHE, w.kv_sigma)
        fill_normal(t["base_logits"], w.seed, gen.TID_BASE_LOGITS + sh * sub_logits, w.logit_sigma)
    i32 = torch.int32
    t["head_logits"] = z((w.B, w.K, w.V), torch.float32) if with_head_logits else None
    t["topk_ids"] = z((w.B, w.K, w.topk), i32)
    t["topk_vals"] = z((w.B, w.K, w.topk), torch.float32)
    t["attn_out"] = z((w.layers, w.B, T, w.H, w.hd), torch.float32)
    return t


def tree_outputs(t: dict, B: int, T: int, P: int, D: int, device="cuda") -> dict:
    i32 = torch.int32
    t["tree_tokens"] = torch.empty((B, T), dtype=i32, device=device)
    t["candidates"] = torch.empty((B, P, D + 1), dtype=i32, device=device)
    t["position_ids"] = torch.empty((B, T), dtype=i32, device=device)
    t["best_path"] = torch.empty((B,), dtype=i32, device=device)
    t["accept_len"] = torch.empty((B,), dtype=i32, device=device)
    t["accepted_tokens"] = torch.empty((B, D + 1), dtype=i32, device=device)
    t["next_token"] = torch.empty((B,), dtype=i32, device=device)
    return t


def parent_tensor(parent, device="cuda") -> torch.Tensor:
    return torch.tensor(np.asarray(parent, dtype=np.int32), dtype=torch.int32, device=device)
