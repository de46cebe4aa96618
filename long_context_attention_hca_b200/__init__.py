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
    "compressed_attn_decode", "compressed_attn_prefill",
    "csa_compress_ex", "hca_compress_ex", "kv_token_prep", "compressed_attn_decode_ex", "compressed_attn_prefill_ex",
    "kv_state_append", "csa_compress_overlap", "indexer_key_compress",
    "lightning_index_ex", "topk_select_ex_workspace_size", "topk_select_ex",
    "lightning_index_topk_ex_workspace_size", "lightning_index_topk_ex", "hca_decode_step_host",
)


class Layout(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("d_rope", ctypes.c_int32), ("scale_group", ctypes.c_int32)]


class CacheStruct(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("rope", ctypes.c_void_p),
                ("capacity", ctypes.c_int64)]


class EntryExtrasStruct(ctypes.Structure):
    _fields_ = [("norm_w", ctypes.c_void_p), ("norm_eps", ctypes.c_float), ("inv_freq", ctypes.c_void_p)]


class AttnExtrasStruct(ctypes.Structure):
    _fields_ = [("q_norm_w", ctypes.c_void_p), ("norm_eps", ctypes.c_float), ("sink", ctypes.c_void_p),
                ("inv_freq", ctypes.c_void_p), ("q_pos", ctypes.c_void_p), ("win_len", ctypes.c_void_p)]


class EntryExtras:
    """Section 9 extras of stored vectors (compressed entries, window tokens):
    norm_w fp32 [d] (RMSNorm weight) or None, eps, inv_freq fp32 [d_rope/2]
    (RoPE frequencies) or None."""

    def __init__(self, norm_w=None, eps=1e-6, inv_freq=None):
        for t, n in ((norm_w, "norm_w"), (inv_freq, "inv_freq")):
            if t is not None:
                _need(t, torch.float32, n)
        self.norm_w, self.eps, self.inv_freq = norm_w, float(eps), inv_freq

    def c_struct(self):
        return EntryExtrasStruct(_ptr_or_none(self.norm_w), self.eps, _ptr_or_none(self.inv_freq))


class AttnExtras:
    """Section 9 extras of core attention: q_norm_w fp32 [d] (query-head
    RMSNorm) or None, eps, sink fp32 [H] (sink logit per head) or None,
    inv_freq fp32 [d_rope/2] or None (query and output RoPE), q_pos int32 [B]
    (decode: each sequence's query position; required with inv_freq),
    win_len int32 [B] (decode: valid window rows, a window not yet full) or None."""

    def __init__(self, q_norm_w=None, eps=1e-6, sink=None, inv_freq=None, q_pos=None, win_len=None):
        for t, n, dt in ((q_norm_w, "q_norm_w", torch.float32), (sink, "sink", torch.float32),
                         (inv_freq, "inv_freq", torch.float32), (q_pos, "q_pos", torch.int32),
                         (win_len, "win_len", torch.int32)):
            if t is not None:
                _need(t, dt, n)
        self.q_norm_w, self.eps, self.sink, self.inv_freq, self.q_pos = q_norm_w, float(eps), sink, inv_freq, q_pos
        self.win_len = win_len

    def c_struct(self):
        return AttnExtrasStruct(_ptr_or_none(self.q_norm_w), self.eps, _ptr_or_none(self.sink),
                                _ptr_or_none(self.inv_freq), _ptr_or_none(self.q_pos), _ptr_or_none(self.win_len))


def _ptr_or_none(t):
    return None if t is None else t.data_ptr()


_V, _I32, _I64, _F, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
_lib.hca_status_string.argtypes = [ctypes.c_int]
_lib.hca_status_string.restype = ctypes.c_char_p
_lib.hca_last_cuda_error.argtypes = []
_lib.hca_last_cuda_error.restype = ctypes.c_int
_lib.hca_take_device_error.argtypes = []
_lib.hca_take_device_error.restype = ctypes.c_int


BUDGET_DENSE_DECODE, BUDGET_SPARSE_DECODE, BUDGET_DECODE_INDEX = 0, 1, 2
_lib.hca_set_launch_budget.argtypes = [ctypes.c_int, ctypes.c_int]
_lib.hca_set_launch_budget.restype = ctypes.c_int


def set_launch_budget(op: int, max_ctas: int) -> int:
    """Cap the CTAs of decode launches (op: BUDGET_DENSE_DECODE, BUDGET_SPARSE_DECODE
    or BUDGET_DECODE_INDEX; 0 = default).  Process-wide; returns the previous value."""
    prev = int(_lib.hca_set_launch_budget(op, max_ctas))
    if prev < 0:
        raise ValueError("set_launch_budget: unknown op or negative budget")
    return prev


_lib.hca_set_early_query.argtypes = [ctypes.c_int]
_lib.hca_set_early_query.restype = ctypes.c_int


def set_early_query(on: bool) -> bool:
    """Let a sparse decode attention (tensor-core path) load its query before it
    waits for the kernel queued just before it; the query must then be complete
    before that kernel starts.  Process-wide; returns the previous setting."""
    prev = int(_lib.hca_set_early_query(1 if on else 0))
    if prev < 0:
        raise ValueError("set_early_query: on must be 0 or 1")
    return bool(prev)


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
_lib.compressed_attn_prefill.argtypes = [_V, _I32, _I32, _I32, _I32, Layout, CacheStruct, _V, _I32, _V, _V, _I32,
                                         _F, _V, _V]
_lib.compressed_attn_prefill.restype = ctypes.c_int


for _name in ("csa_compress_ex", "hca_compress_ex"):
    getattr(_lib, _name).argtypes = [_V, _V, _I64, _V, _I32, _I64, Layout, CacheStruct, _I64,
                                     ctypes.POINTER(EntryExtrasStruct), _V]
    getattr(_lib, _name).restype = ctypes.c_int
_lib.kv_token_prep.argtypes = [_V, _V, _I64, Layout, ctypes.POINTER(EntryExtrasStruct), _V, _V]
_lib.kv_token_prep.restype = ctypes.c_int
_lib.compressed_attn_decode_ex.argtypes = [_V, _I32, _I32, Layout, CacheStruct, _V, _I32, _V, _I32, _V, _I32, _F,
                                           ctypes.POINTER(AttnExtrasStruct), _V, _V, _V, _SZ, _V]
_lib.compressed_attn_decode_ex.restype = ctypes.c_int
_lib.compressed_attn_prefill_ex.argtypes = [_V, _I32, _I32, _I32, _I32, Layout, CacheStruct, _V, _I32, _V, _V, _I32,
                                            _F, ctypes.POINTER(AttnExtrasStruct), _V, _V]
_lib.compressed_attn_prefill_ex.restype = ctypes.c_int


_lib.kv_state_append.argtypes = [_V, _V, _V, _I32, _I32, _I64, _V, _I32, _V, _V, _I32, _V]
_lib.kv_state_append.restype = ctypes.c_int
_lib.lightning_index_ex.argtypes = [_V, _V, _V, _V, _V, _V, _I32, _I32, _I64, _I32, _I32, _I32, _I32, _V, _V]
_lib.lightning_index_ex.restype = ctypes.c_int
_lib.topk_select_ex_workspace_size.argtypes = [_I32, _I64, _I32, _I32]
_lib.topk_select_ex_workspace_size.restype = _SZ
_lib.topk_select_ex.argtypes = [_V, _I32, _V, _I32, _I64, _I32, _I32, _V, _V, _V, _SZ, _V]
_lib.topk_select_ex.restype = ctypes.c_int
_lib.lightning_index_topk_ex_workspace_size.argtypes = [_I32, _I64, _I32, _I32]
_lib.lightning_index_topk_ex_workspace_size.restype = _SZ
_lib.lightning_index_topk_ex.argtypes = [_V, _V, _V, _V, _V, _V, _I32, _I64, _I32, _I32, _I32, _I32, _I32, _V, _V, _V,
                                         _V, _SZ, _V, _V]
_lib.lightning_index_topk_ex.restype = ctypes.c_int
_lib.csa_compress_overlap.argtypes = [_V, _V, _V, _V, _V, _V, _I64, _V, _I32, _I64, Layout, CacheStruct, _I64, _V]
_lib.csa_compress_overlap.restype = ctypes.c_int
_lib.indexer_key_compress.argtypes = [_V, _V, _V, _V, _V, _V, _I64, _V, _I32, _I64, _I32, _V, _V, _I64, _I64, _V]
_lib.indexer_key_compress.restype = ctypes.c_int


class DecodeStepPlan(ctypes.Structure):
    """hca_decode_step_plan (include/hca.h): device state and buffers of a
    host-to-host decode step of one CSA and one HCA layer."""
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("Hi", ctypes.c_int32), ("c", ctypes.c_int32),
                ("k", ctypes.c_int32), ("W", ctypes.c_int32), ("softmax_scale", ctypes.c_float),
                ("layout", Layout), ("csa_cache", CacheStruct), ("csa_entries", ctypes.c_int64),
                ("k_codes", ctypes.c_void_p), ("k_sf", ctypes.c_void_p), ("csa_window", ctypes.c_void_p),
                ("hca_cache", CacheStruct), ("hca_n", ctypes.c_void_p), ("hca_max", ctypes.c_int32),
                ("hca_window", ctypes.c_void_p), ("q_pos", ctypes.c_void_p), ("q_csa", ctypes.c_void_p),
                ("q_hca", ctypes.c_void_p), ("iq_codes", ctypes.c_void_p), ("iq_sf", ctypes.c_void_p),
                ("iq_w", ctypes.c_void_p), ("scores", ctypes.c_void_p), ("idx", ctypes.c_void_p),
                ("count", ctypes.c_void_p), ("topk_ws", ctypes.c_void_p), ("topk_ws_bytes", ctypes.c_size_t),
                ("ws_csa", ctypes.c_void_p), ("ws_csa_bytes", ctypes.c_size_t), ("ws_hca", ctypes.c_void_p),
                ("ws_hca_bytes", ctypes.c_size_t), ("out_csa", ctypes.c_void_p), ("out_hca", ctypes.c_void_p),
                ("side_stream", ctypes.c_void_p), ("ev_fork", ctypes.c_void_p), ("ev_index", ctypes.c_void_p),
                ("ev_q", ctypes.c_void_p), ("ev_join", ctypes.c_void_p), ("hca_ctas", ctypes.c_int32),
                ("ev_iq", ctypes.c_void_p), ("packed", ctypes.c_int32)]


_lib.hca_decode_step_host.argtypes = [ctypes.POINTER(DecodeStepPlan), _V, _V, _V, _V, _V, _V, _V, _V]
_lib.hca_decode_step_host.restype = ctypes.c_int


def decode_step_host(plan: DecodeStepPlan, h_q_csa, h_q_hca, h_iq, h_out_csa, h_out_hca, stream=None):
    """hca_decode_step_host: pinned host tensors in (queries, indexer query
    (codes, sf, w)), pinned host outputs out."""
    qc, qs, w = h_iq
    _check(_lib.hca_decode_step_host(ctypes.byref(plan), _p(h_q_csa), _p(h_q_hca), _p(qc), _p(qs), _p(w),
                                     _p(h_out_csa), _p(h_out_hca), _stream(stream)), "hca_decode_step_host")


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
def _compress(fn, fn_ex, m, x, gate, pos_bias, n_blocks, cache: KVCache, entry_begin=0, stream=None, extras=None):
    _need(x, torch.bfloat16, "x"); _need(gate, torch.bfloat16, "gate"); _need(pos_bias, torch.float32, "pos_bias")
    B, T, d = x.shape
    if gate.shape != x.shape or tuple(pos_bias.shape) != (m, d) or cache.B < B:
        raise ValueError("shape mismatch")
    if extras is None:
        _check(fn(_p(x), _p(gate), T, _p(pos_bias), B, n_blocks, cache.c_layout, cache.c_struct, entry_begin,
                  _stream(stream)), fn.__name__)
    else:
        ex = extras.c_struct()
        _check(fn_ex(_p(x), _p(gate), T, _p(pos_bias), B, n_blocks, cache.c_layout, cache.c_struct, entry_begin,
                     ctypes.byref(ex), _stream(stream)), fn_ex.__name__)


def csa_compress(x, gate, pos_bias, n_blocks, cache, entry_begin=0, stream=None, extras=None):
    """Pool n_blocks blocks of 4 tokens per sequence (x, gate: [B][T][d] bf16,
    row 0 = first token of block entry_begin) into cache entries.  extras: an
    EntryExtras (entry RMSNorm / RoPE before storage) or None."""
    _compress(_lib.csa_compress, _lib.csa_compress_ex, 4, x, gate, pos_bias, n_blocks, cache, entry_begin, stream,
              extras)


def hca_compress(x, gate, pos_bias, n_blocks, cache, entry_begin=0, stream=None, extras=None):
    """Same as csa_compress with blocks of 128 tokens."""
    _compress(_lib.hca_compress, _lib.hca_compress_ex, 128, x, gate, pos_bias, n_blocks, cache, entry_begin, stream,
              extras)


def kv_token_prep(x, pos, layout, extras: EntryExtras, out=None, stream=None):
    """Window tokens for the state cache: x [n][d] bf16, pos [n] int32 -> out
    [n][d] bf16 (RMSNorm and RoPE at each token's position)."""
    _need(x, torch.bfloat16, "x"); _need(pos, torch.int32, "pos")
    n = x.shape[0]
    if out is None:
        out = torch.empty_like(x)
    ex = extras.c_struct()
    _check(_lib.kv_token_prep(_p(x), _p(pos), n, Layout(*layout), ctypes.byref(ex), _p(out), _stream(stream)),
           "kv_token_prep")
    return out


def lightning_index(q_codes, q_sf, w, k_codes, k_sf, q_pos, m, scores=None, stream=None, score_bf16=False):
    """Index scores [B][Tq][Nc] (-inf for entries whose block ends after the
    query): fp32, or bf16 (the note's BF16 index scores) with score_bf16."""
    for t, dt, n in ((q_codes, torch.uint8, "q_codes"), (q_sf, torch.uint8, "q_sf"), (w, torch.float32, "w"),
                     (k_codes, torch.uint8, "k_codes"), (k_sf, torch.uint8, "k_sf"), (q_pos, torch.int32, "q_pos")):
        _need(t, dt, n)
    B, Tq, Hi, cb = q_codes.shape
    Nc = k_codes.shape[1]
    sdt = torch.bfloat16 if score_bf16 else torch.float32
    if scores is None:
        scores = torch.empty((B, Tq, Nc), dtype=sdt, device=q_codes.device)
    _need(scores, sdt, "scores")
    _check(_lib.lightning_index_ex(_p(q_codes), _p(q_sf), _p(w), _p(k_codes), _p(k_sf), _p(q_pos), B, Tq, Nc, Hi,
                                   cb * 2, m, int(bool(score_bf16)), _p(scores), _stream(stream)), "lightning_index")
    return scores


def topk_workspace_size(R, Nc, k, score_bf16=False) -> int:
    return int(_lib.topk_select_ex_workspace_size(R, Nc, k, int(bool(score_bf16))))


def topk_select(scores, q_pos, m, k, idx=None, count=None, ws=None, stream=None):
    """scores [R][Nc] (any leading shape flattened) fp32, or bf16 (the note's
    BF16 index scores), q_pos [R] -> (idx [R][k] ascending, -1 padded; count [R]).
    ws: optional uint8 workspace of topk_workspace_size(R, Nc, k, bf16) bytes
    (allocated here when None)."""
    _need(q_pos, torch.int32, "q_pos")
    bf = scores.dtype == torch.bfloat16
    _need(scores, torch.bfloat16 if bf else torch.float32, "scores")
    Nc = scores.shape[-1]
    R = scores.numel() // Nc if Nc else q_pos.numel()
    if idx is None:
        idx = torch.empty((R, k), dtype=torch.int32, device=scores.device)
    if count is None:
        count = torch.empty((R,), dtype=torch.int32, device=scores.device)
    ws_bytes = topk_workspace_size(R, Nc, k, bf)
    if ws_bytes and (ws is None or ws.numel() < ws_bytes):
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=scores.device)
    elif not ws_bytes:
        ws = None
    _check(_lib.topk_select_ex(_p(scores), int(bf), _p(q_pos), R, Nc, m, k, _p(idx), _p(count), _p(ws), ws_bytes,
                               _stream(stream)), "topk_select")
    return idx, count


_lib.lightning_index_topk_workspace_size.argtypes = [_I32, _I64, _I32]
_lib.lightning_index_topk_workspace_size.restype = _SZ
_lib.lightning_index_topk.argtypes = [_V, _V, _V, _V, _V, _V, _I32, _I64, _I32, _I32, _I32, _I32, _V, _V, _V, _V, _SZ,
                                      _V, _V]
_lib.lightning_index_topk.restype = ctypes.c_int


def lightning_index_topk(q_codes, q_sf, w, k_codes, k_sf, q_pos, m, k, scores=None, idx=None, count=None, ws=None,
                         index_done=None, stream=None, score_bf16=False):
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
    sdt = torch.bfloat16 if score_bf16 else torch.float32
    if scores is None:
        scores = torch.empty((B, 1, Nc), dtype=sdt, device=dev)
    _need(scores, sdt, "scores")
    if idx is None:
        idx = torch.empty((B, k), dtype=torch.int32, device=dev)
    if count is None:
        count = torch.empty((B,), dtype=torch.int32, device=dev)
    need = int(_lib.lightning_index_topk_ex_workspace_size(B, Nc, k, int(bool(score_bf16))))
    if need and (ws is None or ws.numel() < need):
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
    elif not need:
        ws = None
    _check(_lib.lightning_index_topk_ex(_p(q_codes), _p(q_sf), _p(w), _p(k_codes), _p(k_sf), _p(q_pos), B, Nc, Hi,
                                        2 * half_c, m, k, int(bool(score_bf16)), _p(scores), _p(idx), _p(count),
                                        _p(ws), need, ev, _stream(stream)), "lightning_index_topk")
    return scores, idx, count


def decode_workspace_size(B, H, layout, max_comp, W) -> int:
    return int(_lib.compressed_attn_decode_workspace_size(B, H, Layout(*layout), max_comp, W))


def compressed_attn_decode(q, cache: KVCache, n_comp, max_comp, window, softmax_scale, idx=None,
                           out=None, lse=None, ws=None, stream=None, extras=None):
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
    if extras is None:
        _check(_lib.compressed_attn_decode(_p(q), B, H, cache.c_layout, cache.c_struct, _p(idx), stride, _p(n_comp),
                                           max_comp, _p(window), W, float(softmax_scale), _p(out), _p(lse),
                                           _p(ws) if need else None, need, _stream(stream)), "compressed_attn_decode")
    else:
        ex = extras.c_struct()
        _check(_lib.compressed_attn_decode_ex(_p(q), B, H, cache.c_layout, cache.c_struct, _p(idx), stride,
                                              _p(n_comp), max_comp, _p(window), W, float(softmax_scale),
                                              ctypes.byref(ex), _p(out), _p(lse), _p(ws) if need else None, need,
                                              _stream(stream)), "compressed_attn_decode_ex")
    return out


def compressed_attn_prefill(q, p0, m, cache: KVCache, raw, W, softmax_scale, idx=None, count=None, out=None,
                            stream=None, extras=None):
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
    if extras is None:
        _check(_lib.compressed_attn_prefill(_p(q), Tq, H, p0, m, cache.c_layout, cache.c_struct, _p(idx), stride,
                                            _p(count), _p(raw), W, float(softmax_scale), _p(out),
                                            _stream(stream)), "compressed_attn_prefill")
    else:
        ex = extras.c_struct()
        _check(_lib.compressed_attn_prefill_ex(_p(q), Tq, H, p0, m, cache.c_layout, cache.c_struct, _p(idx), stride,
                                               _p(count), _p(raw), W, float(softmax_scale), ctypes.byref(ex), _p(out),
                                               _stream(stream)), "compressed_attn_prefill_ex")
    return out


def kv_state_append(x, gate, pos, window, tail_x=None, tail_gate=None, win_x=None, stream=None):
    """State-cache append of one token per sequence at position pos: x, gate
    [B][d] bf16 -> window ring [B][W][d] row pos % W (win_x instead of x when
    given), and the block tail [B][m][d] row pos % m when tail_x is given."""
    _need(x, torch.bfloat16, "x")
    B, d = x.shape
    W = window.shape[1] if window is not None else 0
    m = tail_x.shape[1] if tail_x is not None else 0
    _check(_lib.kv_state_append(_p(x), _p(gate), _p(win_x), B, d, int(pos), _p(window), W, _p(tail_x), _p(tail_gate),
                                m, _stream(stream)), "kv_state_append")


def _overlap_check(xa, za, xb, zb, a_prev, za_prev, bias, d):
    """Streams may be views into longer sequences: rows contiguous, one common
    sequence stride (passed to the library as x_seq_stride)."""
    stride0 = xa.stride(0)
    for t, n in ((xa, "xa"), (za, "za"), (xb, "xb"), (zb, "zb"), (a_prev, "a_prev"), (za_prev, "za_prev")):
        if t is None:
            continue
        if t.dtype != torch.bfloat16 or not t.is_cuda:
            raise TypeError(f"{n}: expected a CUDA bf16 tensor")
        if t.dim() != 3 or t.shape[2] != d or t.stride(2) != 1 or t.stride(1) != d or t.stride(0) != stride0:
            raise ValueError(f"{n}: rows must be contiguous with the common sequence stride")
    _need(bias, torch.float32, "pos_bias")
    if not (xa.shape == za.shape == xb.shape == zb.shape) or tuple(bias.shape) != (8, d):
        raise ValueError("shape mismatch")
    if (a_prev is None) != (za_prev is None):
        raise ValueError("a_prev and za_prev go together")


def csa_compress_overlap(xa, za, xb, zb, pos_bias, n_blocks, cache: KVCache, entry_begin=0, a_prev=None,
                         za_prev=None, stream=None):
    """The note's overlapped CSA compressor (section 7): entry entry_begin+j
    pools block j-1 of stream a and block j of stream b.  xa, za, xb, zb
    [B][T][d] bf16 (row 0 = first token of block entry_begin); a_prev, za_prev:
    views with the same sequence stride whose rows 0..3 are stream a's block
    before entry_begin (None: the first entry has no a-half); pos_bias [8][d]."""
    B, T, d = xb.shape
    _overlap_check(xa, za, xb, zb, a_prev, za_prev, pos_bias, d)
    _check(_lib.csa_compress_overlap(_p(xa), _p(za), _p(xb), _p(zb), _p(a_prev), _p(za_prev), xa.stride(0) // d,
                                     _p(pos_bias), B, n_blocks, cache.c_layout, cache.c_struct, entry_begin,
                                     _stream(stream)), "csa_compress_overlap")


def indexer_key_compress(xa, za, xb, zb, pos_bias, n_blocks, k_codes, k_sf, entry_begin=0, a_prev=None,
                         za_prev=None, stream=None):
    """Indexer keys (note section 7, K^IComp): the overlapped compressor over
    c-channel key streams [B][T][c], stored FP4 into k_codes [B][cap][c/2]
    and k_sf [B][cap][c/32] (uint8) at entries entry_begin..."""
    B, T, c = xb.shape
    _overlap_check(xa, za, xb, zb, a_prev, za_prev, pos_bias, c)
    _need(k_codes, torch.uint8, "k_codes"); _need(k_sf, torch.uint8, "k_sf")
    _check(_lib.indexer_key_compress(_p(xa), _p(za), _p(xb), _p(zb), _p(a_prev), _p(za_prev), xa.stride(0) // c,
                                     _p(pos_bias), B, n_blocks, c, _p(k_codes), _p(k_sf), k_codes.shape[1],
                                     entry_begin, _stream(stream)), "indexer_key_compress")

