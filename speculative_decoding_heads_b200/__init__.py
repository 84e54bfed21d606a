"""Python binding of libmedusa_b200 (one Medusa verification step on B200).

Argument marshalling only: every function passes device pointers, sizes and
the current CUDA stream to the C ABI declared in ``include/medusa_b200.h``;
all computation happens in the library's sm_100a kernels.  There is no
fallback: importing this package fails when the shared library is missing.

Tensors are torch tensors on the CUDA device (torch is used for device
memory and streams only).  Names follow the C ABI.
"""

from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmedusa_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libmedusa_b200.so not found at {LIB_PATH}; build it with "
        "`python -m speculative_decoding_heads_b200._build` (nvcc, sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)
ABI_VERSION = 7   # layout of medusa_step_args_t (StepArgs below) and of every signature
_lib.medusa_abi_version.restype = ctypes.c_int
if _lib.medusa_abi_version() != ABI_VERSION:
    raise ImportError(f"{LIB_PATH} has ABI version {_lib.medusa_abi_version()}, this binding needs "
                      f"{ABI_VERSION}; rebuild it")

MEDUSA_OK = 0
MEDUSA_ERR_INVALID_ARG = 1
MEDUSA_ERR_UNSUPPORTED = 2
MEDUSA_ERR_CUDA = 3
MEDUSA_ERR_TIMEOUT = 4
MEDUSA_ERR_DEVICE_CHECK = 5
MEDUSA_F32 = 0
MEDUSA_BF16 = 1
MEDUSA_GREEDY = 0
MEDUSA_TYPICAL = 1
MEDUSA_NUCLEUS = 2
MAX_T, MAX_K, MAX_TOPK, MAX_B, MAX_SHARDS = 256, 16, 32, 64, 64

# Every symbol the header declares (checked by the CPU tests).
EXPORTED = [
    "medusa_last_error", "medusa_abi_version", "medusa_device_status", "medusa_test_heads_wait",
    "medusa_tree_choices_ranksum", "medusa_tree_create", "medusa_tree_destroy",
    "medusa_tree_info", "medusa_tree_tables",
    "medusa_heads_workspace_size", "medusa_heads_topk", "medusa_heads_topk_noalloc",
    "medusa_topk_merge", "medusa_build_tree",
    "medusa_attention_workspace_size", "medusa_tree_attention",
    "medusa_tree_attention_split", "medusa_attention_combine", "medusa_attention_rescale",
    "medusa_posterior_workspace_size", "medusa_evaluate_posterior",
    "medusa_accept_kv",
    "medusa_decoder_pack_rows", "medusa_tree_decode_workspace_size", "medusa_tree_decode",
    "medusa_step_workspace_size", "medusa_step", "medusa_step_host",
    "medusa_generate_workspace_size", "medusa_generate_greedy", "medusa_generate",
]

_vp = ctypes.c_void_p
_i32 = ctypes.c_int
_f32 = ctypes.c_float
_sz = ctypes.c_size_t
_pi32 = ctypes.POINTER(ctypes.c_int32)
_pu64 = ctypes.POINTER(ctypes.c_uint64)


class StepArgs(ctypes.Structure):
    """Mirror of ``medusa_step_args_t``."""
    _fields_ = [
        ("tree", _vp),
        ("B", _i32), ("d", _i32), ("V", _i32), ("K", _i32), ("topk", _i32),
        ("layers", _i32), ("H", _i32), ("hd", _i32), ("Lcap", _i32),
        ("dtype", _i32),
        ("h", _vp), ("W1", _vp), ("b1", _vp), ("Wout", _vp),
        ("root_tokens", _vp),
        ("q", _vp), ("k_cache", _vp), ("v_cache", _vp),
        ("seq_lens", _vp),
        ("base_logits", _vp),
        ("scale", _f32),
        ("mode", _i32),
        ("temperature", _f32), ("eps", _f32), ("alpha", _f32),
        ("head_logits", _vp), ("topk_ids", _vp), ("topk_vals", _vp),
        ("tree_tokens", _vp), ("candidates", _vp), ("position_ids", _vp),
        ("attn_out", _vp),
        ("best_path", _vp), ("accept_len", _vp), ("accepted_tokens", _vp), ("next_token", _vp),
        ("attn_inputs_ready", _vp), ("posterior_inputs_ready", _vp),
        ("top_p", _f32), ("uniforms", _vp),
    ]


class StepHostIO(ctypes.Structure):
    """Mirror of ``medusa_step_host_io_t`` (host pointers)."""
    _fields_ = [("h", _vp), ("root_tokens", _vp), ("seq_lens", _vp), ("uniforms", _vp), ("q", _vp),
                ("k_tree", _vp), ("v_tree", _vp), ("base_logits", _vp),
                ("best_path", _vp), ("accept_len", _vp), ("accepted_tokens", _vp), ("next_token", _vp),
                ("seq_lens_out", _vp), ("copy_stream", _vp)]


class DecoderLayer(ctypes.Structure):
    """Mirror of ``medusa_decoder_layer_t`` (device pointers)."""
    _fields_ = [("attn_norm", _vp), ("wqkv", _vp), ("wo", _vp), ("mlp_norm", _vp), ("wgu", _vp), ("wdown", _vp)]


class DecoderModel(ctypes.Structure):
    """Mirror of ``medusa_decoder_t``."""
    _fields_ = [("layers", _i32), ("D", _i32), ("F", _i32), ("V", _i32), ("embed", _vp),
                ("layer", ctypes.POINTER(DecoderLayer)), ("final_norm", _vp), ("lm_head", _vp)]


def _sig(name, restype, argtypes):
    fn = getattr(_lib, name)
    fn.restype = restype
    fn.argtypes = argtypes
    return fn


_sig("medusa_last_error", ctypes.c_char_p, [])
_sig("medusa_abi_version", _i32, [])
_sig("medusa_device_status", _i32, [_pi32, _pi32, _i32])
_sig("medusa_test_heads_wait", _i32, [_i32, ctypes.c_longlong])
_sig("medusa_tree_choices_ranksum", _i32, [_i32, _i32, _i32, _pi32, _pi32])
_sig("medusa_tree_create", _i32, [_pi32, _pi32, _i32, _i32, _i32, _i32, ctypes.POINTER(_vp)])
_sig("medusa_tree_destroy", None, [_vp])
_sig("medusa_tree_info", _i32, [_vp, _pi32, _pi32, _pi32])
_sig("medusa_tree_tables", _i32, [_vp, _pi32, _pi32, _pi32, _pi32, _pu64])
_sig("medusa_heads_workspace_size", _sz, [_i32] * 5)
_sig("medusa_heads_topk", _i32, [_vp, _vp, _vp, _vp] + [_i32] * 5 + [_i32, _vp, _vp, _vp, _vp, _sz, _vp])
_sig("medusa_heads_topk_noalloc", _i32, [_vp, _vp, _vp, _vp] + [_i32] * 5 + [_i32, _vp, _vp, _vp, _vp])
_sig("medusa_topk_merge", _i32, [_vp, _vp, _pi32] + [_i32] * 5 + [_vp, _vp, _vp])
_sig("medusa_build_tree", _i32, [_vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp])
_sig("medusa_attention_workspace_size", _sz, [_vp, _i32, _i32, _i32, _i32, _i32])
_sig("medusa_tree_attention", _i32,
     [_vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _i32, _vp, _f32, _vp, _vp, _sz, _vp])
_sig("medusa_tree_attention_split", _i32,
     [_vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _i32, _vp, _f32, _i32, _i32, _vp, _vp, _vp])
_sig("medusa_attention_combine", _i32, [_i32, ctypes.c_int64, _i32, _vp, _vp, _vp, _vp, _vp])
_sig("medusa_attention_rescale", _i32, [_i32, _i32, ctypes.c_int64, _i32, _vp, _vp, _vp, _vp])
_sig("medusa_posterior_workspace_size", _sz, [_vp, _i32])
_sig("medusa_evaluate_posterior", _i32,
     [_vp, _i32, _i32, _vp, _vp, _i32, _f32, _f32, _f32, _f32, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp])
_sig("medusa_accept_kv", _i32, [_vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _i32, _vp, _vp, _vp, _vp])
_sig("medusa_decoder_pack_rows", _i32, [_i32, _i32, _pi32])
_sig("medusa_tree_decode_workspace_size", _sz, [_vp, ctypes.POINTER(DecoderModel), _i32])
_sig("medusa_tree_decode", _i32, [_vp, ctypes.POINTER(DecoderModel), _i32, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp,
                                   _sz, _vp])
_sig("medusa_generate_workspace_size", _sz, [_vp, ctypes.POINTER(DecoderModel)])
_sig("medusa_generate_greedy", _i32, [_vp, ctypes.POINTER(DecoderModel), _vp, _vp, _vp, _pi32, _i32, _i32, _vp, _vp,
                                      _i32, _pi32, _pi32, _i32, _pi32, _vp, _sz, _vp])
_sig("medusa_generate", _i32, [_vp, ctypes.POINTER(DecoderModel), _vp, _vp, _vp, _i32, _f32, _f32, _f32, _f32,
                               ctypes.POINTER(ctypes.c_float), _pi32, _i32, _i32, _vp, _vp, _i32, _pi32, _pi32, _i32,
                               _pi32, _vp, _sz, _vp])
_sig("medusa_step_workspace_size", _sz, [ctypes.POINTER(StepArgs)])
_sig("medusa_step", _i32, [ctypes.POINTER(StepArgs), _vp, _sz, _vp])
_sig("medusa_step_host", _i32, [ctypes.POINTER(StepArgs), ctypes.POINTER(StepHostIO), _vp, _sz, _vp])


class MedusaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[{code}] {msg}")
        self.code = code


def _check(st: int):
    if st != MEDUSA_OK:
        raise MedusaError(st, (_lib.medusa_last_error() or b"").decode())


def _p(t: Optional[torch.Tensor]):
    """Device pointer of a tensor argument (None stays NULL).  Every tensor the C ABI takes is
    device memory: a host tensor is refused here, before anything is enqueued."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libmedusa_b200 tensor arguments must be CUDA tensors (got one on the host)")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"libmedusa_b200 tensor argument on {t.device}, but the current device is "
                         f"cuda:{torch.cuda.current_device()} (the kernels run there)")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MEDUSA_BF16
    if t.dtype == torch.float32:
        return MEDUSA_F32
    raise MedusaError(MEDUSA_ERR_UNSUPPORTED, f"unsupported dtype {t.dtype}")


# Shape, dtype and layout of every tensor argument are checked here, before
# any call: the C ABI takes bare pointers and sizes, so a tensor smaller than
# the sizes say (a wrong shape, a 2-byte dtype where 4 bytes are read) would
# be read or written past its end on the device, and a strided view would be
# read as if it were dense.


def _require(cond: bool, msg: str):
    if not cond:
        raise ValueError(msg)


def _spec(name: str, t: Optional[torch.Tensor], shape, dtype: Optional[torch.dtype]):
    """`t` must have exactly `shape` (and `dtype`, unless None) and be contiguous."""
    _require(isinstance(t, torch.Tensor), f"{name} must be a tensor")
    _require(tuple(t.shape) == tuple(int(x) for x in shape),
             f"{name} has shape {tuple(t.shape)}, expected {tuple(int(x) for x in shape)}")
    _require(dtype is None or t.dtype == dtype, f"{name} has dtype {t.dtype}, expected {dtype}")
    _require(t.is_contiguous(), f"{name} must be contiguous")


def _nbytes(name: str, t: torch.Tensor) -> int:
    """Byte size of a contiguous workspace tensor (any element type)."""
    _require(isinstance(t, torch.Tensor) and t.is_contiguous(), f"{name} must be a contiguous tensor")
    return t.numel() * t.element_size()


def _heads_specs(h, W1, b1, Wout, topk, topk_ids, topk_vals, head_logits):
    _require(h.dim() == 2 and Wout.dim() == 3, "h must be [B, d] and Wout [K, V, d]")
    B, d = h.shape
    K, V = Wout.shape[0], Wout.shape[1]
    _dtype(h)
    _spec("h", h, (B, d), h.dtype)
    _spec("W1", W1, (K, d, d), h.dtype)
    _spec("b1", b1, (K, d), h.dtype)
    _spec("Wout", Wout, (K, V, d), h.dtype)
    _spec("topk_ids", topk_ids, (B, K, topk), torch.int32)
    _spec("topk_vals", topk_vals, (B, K, topk), torch.float32)
    if head_logits is not None:
        _spec("head_logits", head_logits, (B, K, V), torch.float32)
    return B, d, K, V


def _attention_specs(tree, q, k_cache, v_cache, seq_lens, out):
    _require(q.dim() == 5 and k_cache.dim() == 5,
             "q must be [layers, B, T, H, hd] and the caches [layers, B, H, Lcap, hd]")
    layers, B, T, H, hd = q.shape
    _require(T == tree.T, f"q holds {T} tree tokens per sequence; the tree has {tree.T}")
    Lcap = k_cache.shape[3]
    _dtype(q)
    _spec("q", q, (layers, B, T, H, hd), q.dtype)
    _spec("k_cache", k_cache, (layers, B, H, Lcap, hd), q.dtype)
    _spec("v_cache", v_cache, (layers, B, H, Lcap, hd), q.dtype)
    _spec("seq_lens", seq_lens, (B,), torch.int32)
    _spec("out", out, (layers, B, T, H, hd), torch.float32)
    return layers, B, T, H, hd, Lcap


def abi_version() -> int:
    return _lib.medusa_abi_version()


def device_status(clear: bool = True) -> Tuple[int, int]:
    st, det = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(_lib.medusa_device_status(ctypes.byref(st), ctypes.byref(det), int(clear)))
    return st.value, det.value


def medusa_test_heads_wait(extra_arrivals: int, limit_ns: int):
    """Test hook of the failure-detection path (see the C header): (1, 10**6) makes the batch-1 heads
    kernel's wait between its two phases run out after 1 ms; (0, 0) restores the defaults."""
    _check(_lib.medusa_test_heads_wait(int(extra_arrivals), int(limit_ns)))


# ---------------------------------------------------------------------------
# tree
# ---------------------------------------------------------------------------


def _pack_choices(choices: Sequence[Sequence[int]], K: int):
    n = len(choices)
    ranks = (ctypes.c_int32 * max(1, n * K))()
    lens = (ctypes.c_int32 * max(1, n))()
    for i, c in enumerate(choices):
        lens[i] = len(c)
        for j, r in enumerate(c):
            if j < K:
                ranks[i * K + j] = int(r)
    return ranks, lens


def medusa_tree_choices_ranksum(K: int, topk: int, n_nodes: int) -> List[Tuple[int, ...]]:
    ranks = (ctypes.c_int32 * max(1, n_nodes * K))()
    lens = (ctypes.c_int32 * max(1, n_nodes))()
    _check(_lib.medusa_tree_choices_ranksum(K, topk, n_nodes, ranks, lens))
    return [tuple(ranks[i * K + j] for j in range(lens[i])) for i in range(n_nodes)]


class Tree:
    """A candidate tree (``medusa_tree_t``); ``upload=False`` keeps it host-only."""

    def __init__(self, choices: Sequence[Sequence[int]], K: int, topk: int, upload: bool = True):
        ranks, lens = _pack_choices(choices, K)
        h = ctypes.c_void_p()
        _check(_lib.medusa_tree_create(ranks, lens, len(choices), K, topk, int(upload), ctypes.byref(h)))
        self._h = h
        self.K, self.topk = K, topk
        T, P, D = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
        _check(_lib.medusa_tree_info(h, ctypes.byref(T), ctypes.byref(P), ctypes.byref(D)))
        self.T, self.P, self.D = T.value, P.value, D.value
        self.W = (self.T + 63) // 64

    @property
    def handle(self):
        return self._h

    def tables(self):
        T, P, D, W = self.T, self.P, self.D, self.W
        ti = (ctypes.c_int32 * T)()
        par = (ctypes.c_int32 * T)()
        dep = (ctypes.c_int32 * T)()
        ret = (ctypes.c_int32 * (P * (D + 1)))()
        anc = (ctypes.c_uint64 * (T * W))()
        _check(_lib.medusa_tree_tables(self._h, ti, par, dep, ret, anc))
        return dict(tree_indices=list(ti), parent=list(par), depth=list(dep),
                    retrieve=[list(ret[p * (D + 1):(p + 1) * (D + 1)]) for p in range(P)],
                    anc=[list(anc[i * W:(i + 1) * W]) for i in range(T)])

    def close(self):
        if getattr(self, "_h", None):
            _lib.medusa_tree_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ---------------------------------------------------------------------------
# step calls
# ---------------------------------------------------------------------------


def workspace(nbytes: int, device=None) -> torch.Tensor:
    """A zero-filled device workspace of at least ``nbytes`` (256-byte aligned)."""
    return torch.zeros(max(256, int(nbytes)), dtype=torch.uint8, device=device or "cuda")


def medusa_heads_workspace_size(B, d, V, K, topk) -> int:
    return int(_lib.medusa_heads_workspace_size(B, d, V, K, topk))


def medusa_heads_topk(h, W1, b1, Wout, topk, topk_ids, topk_vals, ws, head_logits=None, stream=None):
    B, d, K, V = _heads_specs(h, W1, b1, Wout, topk, topk_ids, topk_vals, head_logits)
    nbytes = _nbytes("ws", ws)
    _check(_lib.medusa_heads_topk(_p(h), _p(W1), _p(b1), _p(Wout), B, d, V, K, topk, _dtype(h),
                                  _p(head_logits), _p(topk_ids), _p(topk_vals), _p(ws),
                                  nbytes, _stream(stream)))


def medusa_heads_topk_noalloc(h, W1, b1, Wout, topk, topk_ids, topk_vals, head_logits=None, stream=None):
    """medusa_heads_topk without a workspace (the library's fixed scratch array)."""
    B, d, K, V = _heads_specs(h, W1, b1, Wout, topk, topk_ids, topk_vals, head_logits)
    _check(_lib.medusa_heads_topk_noalloc(_p(h), _p(W1), _p(b1), _p(Wout), B, d, V, K, topk, _dtype(h),
                                          _p(head_logits), _p(topk_ids), _p(topk_vals), _stream(stream)))


def medusa_topk_merge(vals, ids, row0: Sequence[int], V: int, out_vals, out_ids, stream=None):
    """Global top-k from gathered per-shard lists: vals/ids [G, B, K, topk] (shard-local ids),
    row0[g] the first vocabulary row of shard g; writes out_vals/out_ids [B, K, topk]."""
    _require(vals.dim() == 4, "vals must be [G, B, K, topk]")
    G, B, K, topk = vals.shape
    _spec("vals", vals, (G, B, K, topk), torch.float32)
    _spec("ids", ids, (G, B, K, topk), torch.int32)
    _spec("out_vals", out_vals, (B, K, topk), torch.float32)
    _spec("out_ids", out_ids, (B, K, topk), torch.int32)
    if len(row0) != G:
        raise ValueError(f"row0 has {len(row0)} entries for {G} shards")
    r0 = (ctypes.c_int32 * G)(*[int(x) for x in row0])
    _check(_lib.medusa_topk_merge(_p(vals), _p(ids), r0, G, V, B, K, topk, _p(out_vals), _p(out_ids),
                                  _stream(stream)))


def medusa_build_tree(tree: Tree, root_tokens, topk_ids, seq_lens, tree_tokens, candidates,
                      position_ids, stream=None):
    _require(root_tokens.dim() == 1, "root_tokens must be [B]")
    B = root_tokens.shape[0]
    _spec("root_tokens", root_tokens, (B,), torch.int32)
    _spec("topk_ids", topk_ids, (B, tree.K, tree.topk), torch.int32)
    _spec("seq_lens", seq_lens, (B,), torch.int32)
    _spec("tree_tokens", tree_tokens, (B, tree.T), torch.int32)
    _spec("candidates", candidates, (B, tree.P, tree.D + 1), torch.int32)
    _spec("position_ids", position_ids, (B, tree.T), torch.int32)
    _check(_lib.medusa_build_tree(tree.handle, root_tokens.shape[0], _p(root_tokens), _p(topk_ids),
                                  _p(seq_lens), _p(tree_tokens), _p(candidates), _p(position_ids),
                                  _stream(stream)))


def medusa_attention_workspace_size(tree: Tree, layers, B, H, hd, dtype) -> int:
    return int(_lib.medusa_attention_workspace_size(tree.handle, layers, B, H, hd, dtype))


def medusa_tree_attention(tree: Tree, q, k_cache, v_cache, seq_lens, scale, out, ws=None, stream=None):
    layers, B, T, H, hd, Lcap = _attention_specs(tree, q, k_cache, v_cache, seq_lens, out)
    nbytes = 0 if ws is None else _nbytes("ws", ws)
    _check(_lib.medusa_tree_attention(tree.handle, layers, B, H, hd, _dtype(q), _p(q), _p(k_cache),
                                      _p(v_cache), Lcap, _p(seq_lens), float(scale), _p(out), _p(ws),
                                      nbytes, _stream(stream)))


def medusa_tree_attention_split(tree: Tree, q, k_cache, v_cache, seq_lens, scale, rank: int, G: int, out, lse,
                                stream=None):
    """Attention over window `rank` of G of each slice's cached prefix (the tree rows with the last
    window): out [layers, B, T, H, hd] normalised over the window, lse [layers, B, T, H]."""
    layers, B, T, H, hd, Lcap = _attention_specs(tree, q, k_cache, v_cache, seq_lens, out)
    _spec("lse", lse, (layers, B, T, H), torch.float32)
    _check(_lib.medusa_tree_attention_split(tree.handle, layers, B, H, hd, _dtype(q), _p(q), _p(k_cache),
                                            _p(v_cache), Lcap, _p(seq_lens), float(scale), int(rank), int(G),
                                            _p(out), _p(lse), _stream(stream)))


def medusa_attention_combine(outs, lses, out, lse_out=None, stream=None):
    """outs [G, ..., hd], lses [G, ...] (the same leading shape) -> out [..., hd], lse_out [...]."""
    _require(outs.dim() >= 2 and lses.dim() == outs.dim() - 1, "outs must be [G, ..., hd] and lses [G, ...]")
    G, hd = outs.shape[0], outs.shape[-1]
    _spec("outs", outs, outs.shape, torch.float32)
    _spec("lses", lses, tuple(outs.shape[:-1]), torch.float32)
    _spec("out", out, tuple(outs.shape[1:]), torch.float32)
    if lse_out is not None:
        _spec("lse_out", lse_out, tuple(outs.shape[1:-1]), torch.float32)
    rows = lses[0].numel()
    _check(_lib.medusa_attention_combine(G, rows, hd, _p(outs), _p(lses), _p(out), _p(lse_out),
                                         _stream(stream)))


def medusa_attention_rescale(lses, rank: int, part, lse_out=None, stream=None):
    """lses [G, ...] (every rank's lse, rank order), part [..., hd] (this rank's window output,
    the same leading shape), scaled in place by exp(lse_rank - lse) so that the G ranks' parts sum
    to the combined output; lse_out [...] receives lse."""
    _require(lses.dim() >= 1 and part.dim() == lses.dim(), "lses must be [G, ...] and part [..., hd]")
    G, hd = lses.shape[0], part.shape[-1]
    _spec("lses", lses, (G,) + tuple(part.shape[:-1]), torch.float32)
    _spec("part", part, part.shape, torch.float32)
    if lse_out is not None:
        _spec("lse_out", lse_out, tuple(part.shape[:-1]), torch.float32)
    rows = lses[0].numel()
    _check(_lib.medusa_attention_rescale(G, int(rank), rows, hd, _p(lses), _p(part), _p(lse_out), _stream(stream)))


def medusa_posterior_workspace_size(tree: Tree, B) -> int:
    return int(_lib.medusa_posterior_workspace_size(tree.handle, B))


def medusa_evaluate_posterior(tree: Tree, logits, candidates, mode, best_path, accept_len,
                              accepted_tokens, next_token, ws, temperature=0.0, eps=0.09,
                              alpha=0.3, top_p=0.8, uniforms=None, stream=None):
    """S6.  ``uniforms`` [B] fp32 in [0, 1) (optional): the next token is drawn with them (typical
    and nucleus modes) instead of taken as the arg-max."""
    _require(logits.dim() == 3, "logits must be [B, T, V]")
    B, T, V = logits.shape
    _require(T == tree.T, f"logits hold {T} tree nodes per sequence; the tree has {tree.T}")
    _spec("logits", logits, (B, T, V), torch.float32)
    _spec("candidates", candidates, (B, tree.P, tree.D + 1), torch.int32)
    for name, t in (("best_path", best_path), ("accept_len", accept_len), ("next_token", next_token)):
        _spec(name, t, (B,), torch.int32)
    _spec("accepted_tokens", accepted_tokens, (B, tree.D + 1), torch.int32)
    if uniforms is not None:
        _spec("uniforms", uniforms, (B,), torch.float32)
    nbytes = _nbytes("ws", ws)
    _check(_lib.medusa_evaluate_posterior(tree.handle, B, V, _p(logits), _p(candidates), int(mode),
                                          float(temperature), float(eps), float(alpha), float(top_p),
                                          _p(uniforms), _p(best_path), _p(accept_len), _p(accepted_tokens),
                                          _p(next_token), _p(ws), nbytes, _stream(stream)))


def medusa_accept_kv(tree: Tree, k_cache, v_cache, seq_lens, best_path, accept_len, stream=None):
    _require(k_cache.dim() == 5, "the caches must be [layers, B, H, Lcap, hd]")
    layers, B, H, Lcap, hd = k_cache.shape
    _dtype(k_cache)
    _spec("k_cache", k_cache, k_cache.shape, k_cache.dtype)
    _spec("v_cache", v_cache, k_cache.shape, k_cache.dtype)
    for name, t in (("seq_lens", seq_lens), ("best_path", best_path), ("accept_len", accept_len)):
        _spec(name, t, (B,), torch.int32)
    _check(_lib.medusa_accept_kv(tree.handle, layers, B, H, hd, _dtype(k_cache), _p(k_cache),
                                 _p(v_cache), Lcap, _p(seq_lens), _p(best_path), _p(accept_len),
                                 _stream(stream)))


# ---------------------------------------------------------------------------
# the base model's forward over the tree tokens
# ---------------------------------------------------------------------------


def medusa_decoder_pack_rows(which: int, n: int) -> List[int]:
    """Source row of every packed row (which 0: one of Wq/Wk/Wv with n = D rows; which 1: [W_gate;
    W_up] with n = 2F rows), as the C call documents."""
    out = (ctypes.c_int32 * n)()
    _check(_lib.medusa_decoder_pack_rows(int(which), int(n), out))
    return list(out)


class Decoder:
    """A base model for ``medusa_tree_decode``: bf16 device tensors, hd = 128.

    ``layers`` is a list of dicts with attn_norm [D], Wq, Wk, Wv, Wo [D, D], mlp_norm [D],
    W_gate, W_up [F, D], W_down [D, F] (out x in); they are packed here (a row reordering, done
    once when the model is set up) into the layout the kernels read."""

    def __init__(self, embed, layers, final_norm, lm_head):
        # Every tensor's shape against D, F and V before anything is packed: the kernels read
        # D x F (and so on) elements from each pointer.
        _require(isinstance(embed, torch.Tensor) and embed.dim() == 2, "embed must be [V, D]")
        V, D = embed.shape
        _require(D > 0 and D % 128 == 0, f"D = {D}: the model's width must be a multiple of the head size 128")
        _require(len(layers) >= 1, "the model needs at least one layer")
        _require(isinstance(layers[0].get("W_gate"), torch.Tensor) and layers[0]["W_gate"].dim() == 2,
                 "W_gate must be [F, D]")
        F = layers[0]["W_gate"].shape[0]
        for name, t, shape in (("lm_head", lm_head, (V, D)), ("final_norm", final_norm, (D,))):
            _require(isinstance(t, torch.Tensor) and tuple(t.shape) == shape,
                     f"{name} must have shape {shape}")
        want = {"attn_norm": (D,), "mlp_norm": (D,), "Wq": (D, D), "Wk": (D, D), "Wv": (D, D), "Wo": (D, D),
                "W_gate": (F, D), "W_up": (F, D), "W_down": (D, F)}
        for i, ly in enumerate(layers):
            for name, shape in want.items():
                t = ly.get(name)
                _require(isinstance(t, torch.Tensor) and tuple(t.shape) == shape,
                         f"layer {i}: {name} must have shape {shape}"
                         + (f", got {tuple(t.shape)}" if isinstance(t, torch.Tensor) else ""))
        dev = embed.device
        iq = torch.tensor(medusa_decoder_pack_rows(0, D), dtype=torch.long, device=dev)
        igu = torch.tensor(medusa_decoder_pack_rows(1, 2 * F), dtype=torch.long, device=dev)
        bf = lambda t: t.to(device=dev, dtype=torch.bfloat16).contiguous()
        self.tensors = []
        for ly in layers:
            wqkv = torch.cat([bf(ly["Wq"])[iq], bf(ly["Wk"])[iq], bf(ly["Wv"])[iq]], 0).contiguous()
            wgu = torch.cat([bf(ly["W_gate"]), bf(ly["W_up"])], 0)[igu].contiguous()
            self.tensors.append(dict(attn_norm=bf(ly["attn_norm"]), wqkv=wqkv, wo=bf(ly["Wo"]),
                                     mlp_norm=bf(ly["mlp_norm"]), wgu=wgu, wdown=bf(ly["W_down"])))
        self.embed, self.final_norm, self.lm_head = bf(embed), bf(final_norm), bf(lm_head)
        self.D, self.F, self.V = D, F, V
        arr = (DecoderLayer * len(layers))()
        for i, t in enumerate(self.tensors):
            for k, v in t.items():
                _spec(k, v, v.shape, torch.bfloat16)
                setattr(arr[i], k, _p(v).value)
        self._layers = arr
        self.c = DecoderModel(len(layers), D, F, V, _p(self.embed).value, arr, _p(self.final_norm).value,
                              _p(self.lm_head).value)


def medusa_tree_decode_workspace_size(tree: Tree, model: Decoder, B: int) -> int:
    return int(_lib.medusa_tree_decode_workspace_size(tree.handle, ctypes.byref(model.c), int(B)))


def medusa_tree_decode(tree: Tree, model: Decoder, tree_tokens, k_cache, v_cache, seq_lens, logits, ws,
                       hidden=None, stream=None):
    """The base model's forward over the tree tokens: tree_tokens [B, T] int32; caches
    [layers, B, H, Lcap, 128] bf16 (the tree's k/v are written at rows seq_lens[b] + node);
    logits [B*T, V] fp32; hidden [B*T, D] fp32 (optional, the residual stream after the last layer)."""
    _require(tree_tokens.dim() == 2 and tree_tokens.shape[1] == tree.T, "tree_tokens must be [B, T]")
    B = tree_tokens.shape[0]
    D, V, H = model.D, model.V, model.D // 128
    _spec("tree_tokens", tree_tokens, (B, tree.T), torch.int32)
    _require(k_cache.dim() == 5, "caches must be [layers, B, H, Lcap, 128]")
    Lcap = k_cache.shape[3]
    shape = (len(model.tensors), B, H, Lcap, 128)
    _spec("k_cache", k_cache, shape, torch.bfloat16)
    _spec("v_cache", v_cache, shape, torch.bfloat16)
    _spec("seq_lens", seq_lens, (B,), torch.int32)
    _spec("logits", logits, (B * tree.T, V), torch.float32)
    if hidden is not None:
        _spec("hidden", hidden, (B * tree.T, D), torch.float32)
    nbytes = _nbytes("ws", ws)
    _check(_lib.medusa_tree_decode(tree.handle, ctypes.byref(model.c), B, _p(tree_tokens), _p(k_cache), _p(v_cache),
                                   Lcap, _p(seq_lens), _p(logits), _p(hidden), _p(ws), nbytes, _stream(stream)))


def medusa_generate_workspace_size(tree: Tree, model: Decoder) -> int:
    return int(_lib.medusa_generate_workspace_size(tree.handle, ctypes.byref(model.c)))


def medusa_generate_greedy(tree: Tree, model: Decoder, W1, b1, Wout, prompt, n_new: int, k_cache, v_cache,
                           ws=None, max_steps=None, stream=None):
    """``medusa_generate`` in greedy mode."""
    return medusa_generate(tree, model, W1, b1, Wout, prompt, n_new, k_cache, v_cache, MEDUSA_GREEDY, ws=ws,
                           max_steps=max_steps, stream=stream)


def medusa_generate(tree: Tree, model: Decoder, W1, b1, Wout, prompt, n_new: int, k_cache, v_cache,
                    mode: int = MEDUSA_GREEDY, temperature=0.0, eps=0.09, alpha=0.3, top_p=0.8, uniforms=None,
                    ws=None, max_steps=None, stream=None):
    """Medusa decoding of one sequence (``medusa_generate``), acceptance in ``mode`` with the next
    token of step s drawn with ``uniforms[s]`` (host floats, at least max_steps of them) if given: prompt (host ints),
    heads W1 [K, D, D], b1 [K, D], Wout [K, V, D] bf16 with K = tree.K, caches [layers, 1, H, Lcap,
    128] bf16 (overwritten from row 0).  Returns (the first n_new emitted tokens, the accept length
    of every step)."""
    K, D, V = tree.K, model.D, model.V
    _spec("W1", W1, (K, D, D), torch.bfloat16)
    _spec("b1", b1, (K, D), torch.bfloat16)
    _spec("Wout", Wout, (K, V, D), torch.bfloat16)
    _require(k_cache.dim() == 5, "caches must be [layers, 1, H, Lcap, 128]")
    Lcap = k_cache.shape[3]
    shape = (len(model.tensors), 1, D // 128, Lcap, 128)
    _spec("k_cache", k_cache, shape, torch.bfloat16)
    _spec("v_cache", v_cache, shape, torch.bfloat16)
    prompt = [int(x) for x in prompt]
    _require(len(prompt) >= 1 and n_new >= 1, "the prompt and n_new must be non-empty")
    max_steps = int(max_steps if max_steps is not None else n_new)
    if ws is None:
        ws = workspace(medusa_generate_workspace_size(tree, model))
    nbytes = _nbytes("ws", ws)
    pr = (ctypes.c_int32 * len(prompt))(*prompt)
    out = (ctypes.c_int32 * n_new)()
    acc = (ctypes.c_int32 * max_steps)()
    n = ctypes.c_int32(0)
    uni = None
    if uniforms is not None:
        uniforms = [float(x) for x in uniforms]
        _require(len(uniforms) >= max_steps, "uniforms needs one value per step (max_steps of them)")
        uni = (ctypes.c_float * len(uniforms))(*uniforms)
    st = _lib.medusa_generate(tree.handle, ctypes.byref(model.c), _p(W1), _p(b1), _p(Wout), int(mode),
                              float(temperature), float(eps), float(alpha), float(top_p), uni, pr, len(prompt),
                              int(n_new), _p(k_cache), _p(v_cache), Lcap, out, acc, max_steps,
                              ctypes.byref(n), _p(ws), nbytes, _stream(stream))
    _check(st)
    return list(out), list(acc[:n.value])


def make_step_args(tree: Tree, t: dict, mode: int, temperature=0.0, eps=0.09, alpha=0.3,
                   scale=None, top_p=0.8) -> StepArgs:
    """Builds ``medusa_step_args_t`` from a dict of device tensors (the keys are the fields'
    names; ``head_logits`` and ``uniforms`` may be absent or None)."""
    layers, B, T, H, hd, Lcap = _attention_specs(tree, t["q"], t["k_cache"], t["v_cache"], t["seq_lens"],
                                                 t["attn_out"])
    _require(t["q"].dtype == t["h"].dtype, "q and the caches must have the dtype of h and the weights")
    _heads_specs(t["h"], t["W1"], t["b1"], t["Wout"], tree.topk, t["topk_ids"], t["topk_vals"],
                 t.get("head_logits"))
    _require(t["Wout"].shape[0] == tree.K, f"Wout holds {t['Wout'].shape[0]} heads; the tree has {tree.K}")
    V = t["Wout"].shape[1]
    _spec("root_tokens", t["root_tokens"], (B,), torch.int32)
    _spec("base_logits", t["base_logits"], (B, T, V), torch.float32)
    for name, shape in (("tree_tokens", (B, T)), ("position_ids", (B, T)), ("candidates", (B, tree.P, tree.D + 1)),
                        ("best_path", (B,)), ("accept_len", (B,)), ("next_token", (B,)),
                        ("accepted_tokens", (B, tree.D + 1))):
        _spec(name, t[name], shape, torch.int32)
    if t.get("uniforms") is not None:
        _spec("uniforms", t["uniforms"], (B,), torch.float32)
    a = StepArgs()
    a.tree = tree.handle
    a.B, a.d = t["h"].shape
    a.K, a.V = t["Wout"].shape[0], t["Wout"].shape[1]
    a.topk = tree.topk
    a.layers, a.H, a.hd, a.Lcap = layers, H, hd, t["k_cache"].shape[3]
    a.dtype = _dtype(t["h"])
    for name in ("h", "W1", "b1", "Wout", "root_tokens", "q", "k_cache", "v_cache", "seq_lens",
                 "base_logits", "topk_ids", "topk_vals", "tree_tokens", "candidates",
                 "position_ids", "attn_out", "best_path", "accept_len", "accepted_tokens",
                 "next_token"):
        setattr(a, name, _p(t[name]).value)
    a.head_logits = _p(t["head_logits"]).value if t.get("head_logits") is not None else None
    a.scale = float(scale if scale is not None else hd ** -0.5)
    a.mode = int(mode)
    a.temperature, a.eps, a.alpha = float(temperature), float(eps), float(alpha)
    a.top_p = float(top_p)
    a._shape = {"B": B, "d": a.d, "V": V, "T": T, "D": tree.D, "layers": layers, "H": H, "hd": hd,
                "dtype": t["h"].dtype}
    if t.get("uniforms") is not None:
        a.uniforms = _p(t["uniforms"]).value
    return a


def medusa_step_workspace_size(args: StepArgs) -> int:
    return int(_lib.medusa_step_workspace_size(ctypes.byref(args)))


def medusa_step(args: StepArgs, ws, stream=None):
    nbytes = _nbytes("ws", ws)
    _check(_lib.medusa_step(ctypes.byref(args), _p(ws), nbytes, _stream(stream)))


def medusa_step_host(args: StepArgs, ws, host_in: dict, host_out: dict, stream=None, copy_stream=None):
    """One step through ``medusa_step_host`` with host buffers.

    ``host_in`` maps input names to host tensors (page-locked for copies that
    overlap the step): ``h``, ``root_tokens``, ``seq_lens``, ``uniforms``,
    ``q``, ``base_logits``, and the tree tokens' own key / value rows as
    ``k_tree`` / ``v_tree`` [layers, B, H, T, hd], which the library places
    at each sequence's length in the caches.  ``host_out`` maps result names
    (``best_path``, ``accept_len``, ``accepted_tokens``, ``next_token``,
    ``seq_lens``) to host tensors the results are copied into.  Absent inputs
    are already on the device; absent results are not copied.  The copies of
    q, the tree rows and the base logits go on ``copy_stream`` (created on
    first use when omitted) while the heads run.  The caller synchronises
    ``stream`` before reading ``host_out``."""
    sh = args._shape
    B, T, D = sh["B"], sh["T"], sh["D"]
    shapes = {"h": ((B, sh["d"]), sh["dtype"]), "root_tokens": ((B,), torch.int32),
              "seq_lens": ((B,), torch.int32), "uniforms": ((B,), torch.float32),
              "q": ((sh["layers"], B, T, sh["H"], sh["hd"]), sh["dtype"]),
              "k_tree": ((sh["layers"], B, sh["H"], T, sh["hd"]), sh["dtype"]),
              "v_tree": ((sh["layers"], B, sh["H"], T, sh["hd"]), sh["dtype"]),
              "base_logits": ((B, T, sh["V"]), torch.float32),
              "best_path": ((B,), torch.int32), "accept_len": ((B,), torch.int32),
              "accepted_tokens": ((B, D + 1), torch.int32), "next_token": ((B,), torch.int32)}
    io = StepHostIO()
    for group, names in ((host_in, ("h", "root_tokens", "seq_lens", "uniforms", "q", "k_tree", "v_tree",
                                    "base_logits")),
                         (host_out, ("best_path", "accept_len", "accepted_tokens", "next_token", "seq_lens"))):
        extra = set(group) - set(names)
        _require(not extra, f"medusa_step_host: unknown buffers {sorted(extra)}")
        for name in names:
            x = group.get(name)
            if x is None:
                continue
            shape, dtype = shapes[name]
            _spec(name, x, shape, dtype)
            _require(not x.is_cuda, f"medusa_step_host: {name} must be a host tensor")
            setattr(io, "seq_lens_out" if group is host_out and name == "seq_lens" else name, x.data_ptr())
    s = stream or torch.cuda.current_stream()
    if copy_stream is None:
        if getattr(args, "_copy_stream", None) is None:
            args._copy_stream = torch.cuda.Stream()
        copy_stream = args._copy_stream
    io.copy_stream = copy_stream.cuda_stream
    nbytes = _nbytes("ws", ws)
    _check(_lib.medusa_step_host(ctypes.byref(args), ctypes.byref(io), _p(ws), nbytes, _stream(s)))