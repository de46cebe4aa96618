"""B200-native (sm_100a) hot path of DeepSeek-V4's hybrid compressed attention.

CSA: 4x softmax-gated KV pooling to FP8/BF16, an exact FP4 lightning indexer,
exact top-k, attention over the selected entries plus a 128-token window.
HCA: 128x pooling, dense attention over every compressed entry plus the window.

This module is a thin ctypes binding over ``libhca_b200.so`` (see
``include/hca.h`` for the contract of every call).  It only marshals torch
tensors into pointers and sizes; every step of the path runs in the CUDA
kernels.  Importing it without the built library raises ImportError: there
is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhca_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m long_context_attention_hca_b200.build` "
        "(nvcc, sm_100a); this package has no CPU fallback")

_lib = ctypes.CDLL(LIB_PATH)

HCA_OK, HCA_ERR_INVALID_ARG, HCA_ERR_UNSUPPORTED, HCA_ERR_CUDA, HCA_ERR_WORKSPACE, HCA_ERR_SCRATCH_LIMIT = range(6)

EXPORTED = (
    "hca_status_string", "hca_last_cuda_error", "csa_compress", "hca_compress", "lightning_index",
    "topk_select_workspace_size", "topk_select", "lightning_index_topk_workspace_size", "lightning_index_topk",
    "compressed_attn_decode_workspace_size",
    "compressed_attn_decode", "compressed_attn_prefill_workspace_size", "compressed_attn_prefill",
)


class Layout(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("d_rope", ctypes.c_int32), ("scale_group", ctypes.c_int32)]


class CacheStruct(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("rope", ctypes.c_void_p),
                ("capacity", ctypes.c_int64)]


_V, _I32, _I64, _F, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
_lib.hca_status_string.argtypes = [ctypes.c_int]
_lib.hca_status_string.restype = ctypes.c_char_p
_lib.hca_last_cuda_error.argtypes = []
_lib.hca_last_cuda_error.restype = ctypes.c_int
_lib.hca_take_device_error.argtypes = []
_lib.hca_take_device_error.restype = ctypes.c_int


BUDGET_DENSE_DECODE, BUDGET_SPARSE_DECODE = 0, 1
_lib.hca_set_launch_budget.argtypes = [ctypes.c_int, ctypes.c_int]
_lib.hca_set_launch_budget.restype = ctypes.c_int


def set_launch_budget(op: int, max_ctas: int) -> int:
    """Cap the CTAs of decode attention launches (op: BUDGET_DENSE_DECODE or
    BUDGET_SPARSE_DECODE; 0 = default).  Process-wide; returns the previous value."""
    prev = int(_lib.hca_set_launch_budget(op, max_ctas))
    if prev < 0:
        raise ValueError("set_launch_budget: unknown op or negative budget")
    return prev


def take_device_error() -> int:
    """Read and clear the device error word (non-zero: a kernel gave up a bounded wait)."""
    return int(_lib.hca_take_device_error())
for _name in ("csa_compress", "hca_compress"):
    getattr(_lib, _name).argtypes = [_V, _V, _I64, _V, _I32, _I64, Layout, CacheStruct, _I64, _V]
    getattr(_lib, _name).restype = ctypes.c_int
_lib.lightning_index.argtypes = [_V, _V, _V, _V, _V, _V, _I32, _I32, _I64, _I32, _I32, _I32, _V, _V]
_lib.lightning_index.restype = ctypes.c_int
_lib.topk_select_workspace_size.argtypes = [_I32, _I64, _I32]
_lib.topk_select_workspace_size.restype = _SZ
_lib.topk_select.argtypes = [_V, _V, _I32, _I64, _I32, _I32, _V, _V, _V, _SZ, _V]
_lib.topk_select.restype = ctypes.c_int
_lib.compressed_attn_decode_workspace_size.argtypes = [_I32, _I32, Layout, _I32, _I32]
_lib.compressed_attn_decode_workspace_size.restype = _SZ
_lib.compressed_attn_decode.argtypes = [_V, _I32, _I32, Layout, CacheStruct, _V, _I32, _V, _I32, _V, _I32, _F,
                                        _V, _V, _V, _SZ, _V]
_lib.compressed_attn_decode.restype = ctypes.c_int
_lib.compressed_attn_prefill_workspace_size.argtypes = [_I32, _I32, Layout]
_lib.compressed_attn_prefill_workspace_size.restype = _SZ
_lib.compressed_attn_prefill.argtypes = [_V, _I32, _I32, _I32, _I32, Layout, CacheStruct, _V, _I32, _V, _V, _I32,
                                         _F, _V, _V, _SZ, _V]
_lib.compressed_attn_prefill.restype = ctypes.c_int


class HCAError(RuntimeError):
    pass


def _check(status: int, what: str):
    if status != HCA_OK:
        msg = _lib.hca_status_string(status).decode()
        if status == HCA_ERR_CUDA:
            msg += f" (cudaError {_lib.hca_last_cuda_error()})"
        raise HCAError(f"{what}: {msg}")


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, name):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")


# ------------------------------------------------------------------ KV cache
LAYOUT_512 = (512, 64, 64)
LAYOUT_128 = (128, 32, 32)


class KVCache:
    """Compressed-entry cache of B sequences (structure of arrays):
    codes uint8 [B][capacity][d-d_rope] (FP8 e4m3fn), scales fp32
    [B][capacity][(d-d_rope)/g], rope bf16 [B][capacity][d_rope]."""

    def __init__(self, B: int, capacity: int, layout=LAYOUT_512, device="cuda", zero=False):
        d, dr, g = layout
        alloc = torch.zeros if zero else torch.empty
        self.B, self.capacity, self.layout = B, capacity, tuple(layout)
        self.codes = alloc((B, capacity, d - dr), dtype=torch.uint8, device=device)
        self.scales = alloc((B, capacity, (d - dr) // g), dtype=torch.float32, device=device)
        self.rope = alloc((B, capacity, dr), dtype=torch.bfloat16, device=device)

    @property
    def c_layout(self) -> Layout:
        return Layout(*self.layout)

    @property
    def c_struct(self) -> CacheStruct:
        return CacheStruct(self.codes.data_ptr(), self.scales.data_ptr(), self.rope.data_ptr(), self.capacity)

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.codes, self.scales, self.rope))

    def sequence(self, b: int) -> "KVCache":
        """View of one sequence as a B = 1 cache (no copy)."""
        v = KVCache.__new__(KVCache)
        v.B, v.capacity, v.layout = 1, self.capacity, self.layout
        v.codes, v.scales, v.rope = self.codes[b:b + 1], self.scales[b:b + 1], self.rope[b:b + 1]
        return v


# ------------------------------------------------------------------ calls
def _compress(fn, m, x, gate, pos_bias, n_blocks, cache: KVCache, entry_begin=0, stream=None):
    _need(x, torch.bfloat16, "x"); _need(gate, torch.bfloat16, "gate"); _need(pos_bias, torch.float32, "pos_bias")
    B, T, d = x.shape
    if gate.shape != x.shape or tuple(pos_bias.shape) != (m, d) or cache.B < B:
        raise ValueError("shape mismatch")
    _check(fn(_p(x), _p(gate), T, _p(pos_bias), B, n_blocks, cache.c_layout, cache.c_struct, entry_begin,
              _stream(stream)), fn.__name__)


def csa_compress(x, gate, pos_bias, n_blocks, cache, entry_begin=0, stream=None):
    """Pool n_blocks blocks of 4 tokens per sequence (x, gate: [B][T][d] bf16,
    row 0 = first token of block entry_begin) into cache entries."""
    _compress(_lib.csa_compress, 4, x, gate, pos_bias, n_blocks, cache, entry_begin, stream)


def hca_compress(x, gate, pos_bias, n_blocks, cache, entry_begin=0, stream=None):
    """Same as csa_compress with blocks of 128 tokens."""
    _compress(_lib.hca_compress, 128, x, gate, pos_bias, n_blocks, cache, entry_begin, stream)


def lightning_index(q_codes, q_sf, w, k_codes, k_sf, q_pos, m, scores=None, stream=None):
    """Index scores [B][Tq][Nc] fp32 (-inf for entries whose block ends after the query)."""
    for t, dt, n in ((q_codes, torch.uint8, "q_codes"), (q_sf, torch.uint8, "q_sf"), (w, torch.float32, "w"),
                     (k_codes, torch.uint8, "k_codes"), (k_sf, torch.uint8, "k_sf"), (q_pos, torch.int32, "q_pos")):
        _need(t, dt, n)
    B, Tq, Hi, cb = q_codes.shape
    Nc = k_codes.shape[1]
    if scores is None:
        scores = torch.empty((B, Tq, Nc), dtype=torch.float32, device=q_codes.device)
    _need(scores, torch.float32, "scores")
    _check(_lib.lightning_index(_p(q_codes), _p(q_sf), _p(w), _p(k_codes), _p(k_sf), _p(q_pos), B, Tq, Nc, Hi,
                                cb * 2, m, _p(scores), _stream(stream)), "lightning_index")
    return scores


def topk_workspace_size(R, Nc, k) -> int:
    return int(_lib.topk_select_workspace_size(R, Nc, k))


def topk_select(scores, q_pos, m, k, idx=None, count=None, ws=None, stream=None):
    """scores [R][Nc] (any leading shape flattened), q_pos [R] -> (idx [R][k] ascending, -1 padded; count [R]).
    ws: optional uint8 workspace of topk_workspace_size(R, Nc, k) bytes (allocated here when None)."""
    _need(scores, torch.float32, "scores"); _need(q_pos, torch.int32, "q_pos")
    Nc = scores.shape[-1]
    R = scores.numel() // Nc if Nc else q_pos.numel()
    if idx is None:
        idx = torch.empty((R, k), dtype=torch.int32, device=scores.device)
    if count is None:
        count = torch.empty((R,), dtype=torch.int32, device=scores.device)
    ws_bytes = topk_workspace_size(R, Nc, k)
    if ws_bytes and (ws is None or ws.numel() < ws_bytes):
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=scores.device)
    elif not ws_bytes:
        ws = None
    _check(_lib.topk_select(_p(scores), _p(q_pos), R, Nc, m, k, _p(idx), _p(count), _p(ws), ws_bytes,
                            _stream(stream)), "topk_select")
    return idx, count


_lib.lightning_index_topk_workspace_size.argtypes = [_I32, _I64, _I32]
_lib.lightning_index_topk_workspace_size.restype = _SZ
_lib.lightning_index_topk.argtypes = [_V, _V, _V, _V, _V, _V, _I32, _I64, _I32, _I32, _I32, _I32, _V, _V, _V, _V, _SZ,
                                      _V, _V]
_lib.lightning_index_topk.restype = ctypes.c_int


def lightning_index_topk(q_codes, q_sf, w, k_codes, k_sf, q_pos, m, k, scores=None, idx=None, count=None, ws=None,
                         index_done=None, stream=None):
    """Decode (one query per sequence): index scores and top-k in one call.
    q_codes [B][1][Hi][c/2], q_sf [B][1][Hi][c/32], w [B][1][Hi]; k_codes [B][Nc][c/2], k_sf [B][Nc][c/32];
    q_pos [B] or [B][1].  index_done: optional torch.cuda.Event recorded once the scores
    are written (it must have been recorded once before, so that it exists).
    Returns (scores [B][1][Nc], idx [B][k], count [B])."""
    ev = None
    if index_done is not None:
        ev = ctypes.c_void_p(index_done.cuda_event)
        if not ev.value:
            raise ValueError("lightning_index_topk: index_done has no CUDA event yet (record it once first)")
    for t, dt, n in ((q_codes, torch.uint8, "q_codes"), (q_sf, torch.uint8, "q_sf"), (w, torch.float32, "w"),
                     (k_codes, torch.uint8, "k_codes"), (k_sf, torch.uint8, "k_sf"), (q_pos, torch.int32, "q_pos")):
        _need(t, dt, n)
    B, Tq, Hi, half_c = q_codes.shape
    if Tq != 1:
        raise ValueError("lightning_index_topk: one query per sequence")
    Nc = k_codes.shape[1]
    dev = q_codes.device
    if scores is None:
        scores = torch.empty((B, 1, Nc), dtype=torch.float32, device=dev)
    if idx is None:
        idx = torch.empty((B, k), dtype=torch.int32, device=dev)
    if count is None:
        count = torch.empty((B,), dtype=torch.int32, device=dev)
    need = int(_lib.lightning_index_topk_workspace_size(B, Nc, k))
    if need and (ws is None or ws.numel() < need):
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
    elif not need:
        ws = None
    _check(_lib.lightning_index_topk(_p(q_codes), _p(q_sf), _p(w), _p(k_codes), _p(k_sf), _p(q_pos), B, Nc, Hi,
                                     2 * half_c, m, k, _p(scores), _p(idx), _p(count), _p(ws), need, ev,
                                     _stream(stream)), "lightning_index_topk")
    return scores, idx, count


def decode_workspace_size(B, H, layout, max_comp, W) -> int:
    return int(_lib.compressed_attn_decode_workspace_size(B, H, Layout(*layout), max_comp, W))


def compressed_attn_decode(q, cache: KVCache, n_comp, max_comp, window, softmax_scale, idx=None,
                           out=None, lse=None, ws=None, stream=None):
    """Decode attention: q [B][H][d] bf16, window [B][W][d] bf16; idx [B][>=max_comp] int32 (CSA)
    or None (HCA, dense over entries 0..n_comp[b]-1).  Returns out [B][H][d] bf16."""
    _need(q, torch.bfloat16, "q"); _need(n_comp, torch.int32, "n_comp"); _need(window, torch.bfloat16, "window")
    B, H, d = q.shape
    W = window.shape[1]
    if out is None:
        out = torch.empty_like(q)
    need = decode_workspace_size(B, H, cache.layout, max_comp, W)
    if need and (ws is None or ws.numel() < need):
        ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    stride = 0
    if idx is not None:
        _need(idx, torch.int32, "idx")
        stride = idx.shape[-1]
    _check(_lib.compressed_attn_decode(_p(q), B, H, cache.c_layout, cache.c_struct, _p(idx), stride, _p(n_comp),
                                       max_comp, _p(window), W, float(softmax_scale), _p(out), _p(lse),
                                       _p(ws) if need else None, need, _stream(stream)), "compressed_attn_decode")
    return out


def compressed_attn_prefill(q, p0, m, cache: KVCache, raw, W, softmax_scale, idx=None, count=None, out=None,
                            stream=None):
    """Prefill attention for one sequence: q [Tq][H][d] bf16 at positions p0..p0+Tq-1; raw [(W-1)+Tq][d]
    bf16 raw tokens from position p0-(W-1); idx [Tq][k] + count [Tq] (CSA) or None (HCA dense causal)."""
    _need(q, torch.bfloat16, "q"); _need(raw, torch.bfloat16, "raw")
    Tq, H, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    stride = 0
    if idx is not None:
        _need(idx, torch.int32, "idx"); _need(count, torch.int32, "count")
        stride = idx.shape[-1]
    _check(_lib.compressed_attn_prefill(_p(q), Tq, H, p0, m, cache.c_layout, cache.c_struct, _p(idx), stride,
                                        _p(count), _p(raw), W, float(softmax_scale), _p(out), None, 0,
                                        _stream(stream)), "compressed_attn_prefill")
    return out
