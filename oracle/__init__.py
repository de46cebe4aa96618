"""CPU oracle for the DeepSeek-V4 CSA/HCA hot path.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The GPU product path (``long_context_attention_hca_b200``) never
imports it and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain C, fp64 for attention, the defined
fp32 sequences where the GPU must match bit for bit); this module only builds
it with gcc and marshals numpy arrays.  Every function cites the passage it
follows in its docstring; see ``oracle.c`` for the readings taken where the
pages leave a step open.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against closed forms, library routines (torch / numpy fp64) or brute force.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

GCC_FLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", *GCC_FLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def set_threads(n: int) -> int:
    """Threads of the oracle's parallel loops (n <= 0: all cores).  Results
    do not depend on it: each output is computed by one thread in the same
    sequence.  Returns the thread count now in effect."""
    lib().oracle_set_threads(int(n))
    return int(lib().oracle_max_threads())


def _P(t):
    return ctypes.POINTER(t)


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            u8p, u16p, i32p, i64p = _P(ctypes.c_uint8), _P(ctypes.c_uint16), _P(ctypes.c_int32), _P(ctypes.c_int64)
            fp, dp = _P(ctypes.c_float), _P(ctypes.c_double)
            L.oracle_set_threads.argtypes = [ctypes.c_int]
            L.oracle_set_threads.restype = None
            L.oracle_max_threads.argtypes = []
            L.oracle_max_threads.restype = ctypes.c_int
            L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
            L.oracle_bf16_to_f32.restype = ctypes.c_float
            L.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
            L.oracle_f32_to_bf16.restype = ctypes.c_uint16
            L.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
            L.oracle_e4m3_value.restype = ctypes.c_double
            L.oracle_f32_to_e4m3.argtypes = [ctypes.c_float]
            L.oracle_f32_to_e4m3.restype = ctypes.c_uint8
            L.oracle_e2m1_value.argtypes = [ctypes.c_int]
            L.oracle_e2m1_value.restype = ctypes.c_double
            L.oracle_ue8m0_value.argtypes = [ctypes.c_uint8]
            L.oracle_ue8m0_value.restype = ctypes.c_double
            L.oracle_const.argtypes = [ctypes.c_int]
            L.oracle_const.restype = ctypes.c_float
            L.oracle_f64_to_bf16_array.argtypes = [dp, u16p, ctypes.c_int64]
            L.oracle_f64_to_bf16_array.restype = None
            L.oracle_f32_to_bf16_array.argtypes = [fp, u16p, ctypes.c_int64]
            L.oracle_f32_to_bf16_array.restype = None
            L.oracle_f32_to_e4m3_array.argtypes = [fp, u8p, ctypes.c_int64]
            L.oracle_f32_to_e4m3_array.restype = None
            L.oracle_exp_neg_array.argtypes = [fp, fp, ctypes.c_int64]
            L.oracle_exp_neg_array.restype = None
            L.oracle_exp_neg.argtypes = [ctypes.c_float]
            L.oracle_exp_neg.restype = ctypes.c_float
            L.oracle_pool_block.argtypes = [u16p, u16p, fp, ctypes.c_int, ctypes.c_int, fp, dp, dp]
            L.oracle_pool_block.restype = None
            L.oracle_quant_entry.argtypes = [fp, ctypes.c_int, ctypes.c_int, ctypes.c_int, u8p, fp, u16p]
            L.oracle_quant_entry.restype = None
            L.oracle_compress.argtypes = [u16p, u16p, ctypes.c_int64, fp, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          u8p, fp, u16p, ctypes.c_int64, ctypes.c_int64]
            L.oracle_compress.restype = ctypes.c_double
            L.oracle_fp4_dot.argtypes = [u8p, u8p, u8p, u8p, ctypes.c_int, _P(ctypes.c_int)]
            L.oracle_fp4_dot.restype = ctypes.c_float
            L.oracle_index_scores.argtypes = [u8p, u8p, fp, u8p, u8p, i32p, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, fp]
            L.oracle_index_scores.restype = ctypes.c_int64
            L.oracle_topk.argtypes = [fp, i32p, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                      i32p, i32p]
            L.oracle_topk.restype = None
            L.oracle_attend.argtypes = [u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        u8p, fp, u16p, i64p, ctypes.c_int64, u16p, ctypes.c_int64,
                                        ctypes.c_float, dp, dp]
            L.oracle_attend.restype = None
            L.oracle_attend_ex.argtypes = [u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           u8p, fp, u16p, i64p, ctypes.c_int64, u16p, ctypes.c_int64,
                                           ctypes.c_float, fp, ctypes.c_float, fp, fp, ctypes.c_int64, dp, dp]
            L.oracle_attend_ex.restype = None
            L.oracle_rmsnorm_f32.argtypes = [fp, ctypes.c_int, fp, ctypes.c_float, fp]
            L.oracle_rmsnorm_f32.restype = None
            L.oracle_rope_f64.argtypes = [dp, ctypes.c_int, ctypes.c_int64, fp, ctypes.c_int, dp]
            L.oracle_rope_f64.restype = None
            L.oracle_token_prep.argtypes = [u16p, i64p, ctypes.c_int64, ctypes.c_int, ctypes.c_int, fp,
                                            ctypes.c_float, fp, u16p]
            L.oracle_token_prep.restype = None
            L.oracle_compress_ex.argtypes = [u16p, u16p, ctypes.c_int64, fp, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, u8p, fp, u16p,
                                             ctypes.c_int64, ctypes.c_int64, fp, ctypes.c_float, fp, ctypes.c_int64]
            L.oracle_compress_ex.restype = ctypes.c_double
            L.oracle_f32_to_e2m1.argtypes = [ctypes.c_float]
            L.oracle_f32_to_e2m1.restype = ctypes.c_uint8
            L.oracle_fp4_quant_block.argtypes = [fp, u8p, u8p]
            L.oracle_fp4_quant_block.restype = None
            L.oracle_compress_overlap.argtypes = [u16p, u16p, u16p, u16p, u16p, u16p, ctypes.c_int64, fp,
                                                  ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                                                  ctypes.c_int, ctypes.c_int, u8p, fp, u16p, ctypes.c_int64,
                                                  ctypes.c_int64]
            L.oracle_compress_overlap.restype = ctypes.c_double
            L.oracle_index_key_compress.argtypes = [u16p, u16p, u16p, u16p, u16p, u16p, ctypes.c_int64, fp,
                                                    ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int, u8p,
                                                    u8p, ctypes.c_int64, ctypes.c_int64]
            L.oracle_index_key_compress.restype = None
            _lib = L
    return _lib


def _ptr(a: np.ndarray, ct):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.POINTER(ct))


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- scalars
def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> fp32 (exact widening)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(x) -> np.ndarray:
    """fp32 -> bf16 bits, round to nearest even (oracle.c)."""
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().oracle_f32_to_bf16_array(_ptr(x, ctypes.c_float), _ptr(out, ctypes.c_uint16), x.size)
    return out


def e4m3_value(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    f = lib().oracle_e4m3_value
    return np.array([f(int(c)) for c in codes.ravel()], dtype=np.float64).reshape(codes.shape)


def f32_to_e4m3(x) -> np.ndarray:
    """fp32 -> e4m3fn codes, RN-even, saturating at 448 (oracle.c)."""
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().oracle_f32_to_e4m3_array(_ptr(x, ctypes.c_float), _ptr(out, ctypes.c_uint8), x.size)
    return out


def e2m1_value(nib: int) -> float:
    return lib().oracle_e2m1_value(int(nib))


def exp_neg(z) -> np.ndarray:
    """The defined exp E(z), z <= 0 (Cody-Waite + degree-7 Taylor, fp32)."""
    z = _c(z, np.float32)
    out = np.empty(z.shape, np.float32)
    lib().oracle_exp_neg_array(_ptr(z, ctypes.c_float), _ptr(out, ctypes.c_float), z.size)
    return out


def constant(which: int) -> np.float32:
    return np.float32(lib().oracle_const(int(which)))


# ---------------------------------------------------------------- pooling
def pool_block(x_bits: np.ndarray, gate_bits: np.ndarray, bias: np.ndarray):
    """Softmax-gated pooling of one block ("DeepSeek V4 ..." note, section 8
    HCA equations).  x_bits, gate_bits: [m][d] bf16 bits; bias [m][d] fp32.
    Returns (y fp32 [d] in the defined fp32 sequence, y64 fp64 [d])."""
    x_bits, gate_bits, bias = _c(x_bits, np.uint16), _c(gate_bits, np.uint16), _c(bias, np.float32)
    m, d = x_bits.shape
    y = np.empty(d, np.float32)
    y64 = np.empty(d, np.float64)
    lib().oracle_pool_block(_ptr(x_bits, ctypes.c_uint16), _ptr(gate_bits, ctypes.c_uint16),
                            _ptr(bias, ctypes.c_float), m, d, _ptr(y, ctypes.c_float), _ptr(y64, ctypes.c_double),
                            None)
    return y, y64


def quant_entry(y: np.ndarray, d_rope: int, g: int):
    """FP8 e4m3 per-g-channel amax/448 scaling of the non-RoPE dims, bf16 RoPE
    dims ("DeepSeek V4 ..." note, section 9, KV storage precision).
    Returns (codes uint8 [d-d_rope], scales fp32 [(d-d_rope)/g], rope bf16 bits [d_rope])."""
    y = _c(y, np.float32)
    d = y.shape[0]
    dn = d - d_rope
    codes = np.empty(dn, np.uint8)
    scales = np.empty(dn // g, np.float32)
    rope = np.empty(d_rope, np.uint16)
    lib().oracle_quant_entry(_ptr(y, ctypes.c_float), d, d_rope, g, _ptr(codes, ctypes.c_uint8),
                             _ptr(scales, ctypes.c_float), _ptr(rope, ctypes.c_uint16))
    return codes, scales, rope


def _opt(a, dtype, ct):
    if a is None:
        return None, None
    a = _c(a, dtype)
    return a, _ptr(a, ct)


def compress(x_bits, gate_bits, bias, m, n_blocks, d_rope, g, cap=None, entry_begin=0,
             norm_w=None, eps=1e-6, inv_freq=None, pos_entry0=-1):
    """Pool + quantise n_blocks entries for each sequence.
    x_bits, gate_bits: [B][T][d] bf16 bits whose row 0 is the first token of
    block ``entry_begin``.  norm_w [d] / inv_freq [d_rope/2] (optional): the
    note's section 9 entry RMSNorm and partial RoPE (entry e at position e*m)
    before storage; pos_entry0 >= 0 places the first pooled block at entry
    index pos_entry0 for RoPE.  Returns (codes [B][cap][dn], scales [B][cap][dn/g],
    rope [B][cap][d_rope], worst fp32-vs-fp64 relative deviation)."""
    x_bits, gate_bits, bias = _c(x_bits, np.uint16), _c(gate_bits, np.uint16), _c(bias, np.float32)
    nw, nw_p = _opt(norm_w, np.float32, ctypes.c_float)
    fq, fq_p = _opt(inv_freq, np.float32, ctypes.c_float)
    B, T, d = x_bits.shape
    assert n_blocks * m <= T
    cap = entry_begin + n_blocks if cap is None else cap
    dn = d - d_rope
    codes = np.zeros((B, cap, dn), np.uint8)
    scales = np.zeros((B, cap, dn // g), np.float32)
    rope = np.zeros((B, cap, d_rope), np.uint16)
    worst = lib().oracle_compress_ex(_ptr(x_bits, ctypes.c_uint16), _ptr(gate_bits, ctypes.c_uint16), T,
                                     _ptr(bias, ctypes.c_float), m, B, n_blocks, d, d_rope, g,
                                     _ptr(codes, ctypes.c_uint8), _ptr(scales, ctypes.c_float),
                                     _ptr(rope, ctypes.c_uint16), cap, entry_begin, nw_p, float(eps), fq_p,
                                     int(pos_entry0))
    return codes, scales, rope, worst


def rmsnorm_f32(y, w, eps=1e-6):
    """RMSNorm of one vector in the defined fp32 sequence (pairwise-tree sum of
    rounded squares, IEEE sqrt, (y / r) * w); note section 9."""
    y, w = _c(y, np.float32), _c(w, np.float32)
    out = np.empty_like(y)
    lib().oracle_rmsnorm_f32(_ptr(y, ctypes.c_float), y.shape[0], _ptr(w, ctypes.c_float), float(eps),
                             _ptr(out, ctypes.c_float))
    return out


def rope_f64(v, pos, inv_freq, sign=1):
    """Partial RoPE of n_r values: pairs (2i, 2i+1) rotated by sign*pos*inv_freq[i], fp64."""
    v, inv_freq = _c(v, np.float64), _c(inv_freq, np.float32)
    out = np.empty_like(v)
    lib().oracle_rope_f64(_ptr(v, ctypes.c_double), v.shape[0], int(pos), _ptr(inv_freq, ctypes.c_float),
                          int(sign), _ptr(out, ctypes.c_double))
    return out


def token_prep(x_bits, pos, d_rope, norm_w=None, eps=1e-6, inv_freq=None):
    """Window tokens for the state cache: RMSNorm and partial RoPE at each
    token's position, stored bf16.  x_bits [n][d] bf16 bits, pos [n]."""
    x_bits = _c(x_bits, np.uint16)
    n, d = x_bits.shape
    pos = _c(pos, np.int64).reshape(-1)
    nw, nw_p = _opt(norm_w, np.float32, ctypes.c_float)
    fq, fq_p = _opt(inv_freq, np.float32, ctypes.c_float)
    out = np.empty_like(x_bits)
    lib().oracle_token_prep(_ptr(x_bits, ctypes.c_uint16), _ptr(pos, ctypes.c_int64), n, d, d_rope, nw_p,
                            float(eps), fq_p, _ptr(out, ctypes.c_uint16))
    return out


# ---------------------------------------------------------------- indexer
def fp4_dot(qc, qs, kc, ks):
    """Exact FP4 e2m1 dot with ue8m0 per-32 scales (one head, one key).
    Returns (fp32 dot, inexact flag)."""
    qc, qs, kc, ks = (_c(a, np.uint8) for a in (qc, qs, kc, ks))
    c = qc.shape[0] * 2
    flag = ctypes.c_int(0)
    v = lib().oracle_fp4_dot(_ptr(qc, ctypes.c_uint8), _ptr(qs, ctypes.c_uint8), _ptr(kc, ctypes.c_uint8),
                             _ptr(ks, ctypes.c_uint8), c, ctypes.byref(flag))
    return np.float32(v), bool(flag.value)


def index_scores(q_codes, q_sf, w, k_codes, k_sf, q_pos, m):
    """Lightning-indexer scores I_{t,s} ("DeepSeek V4 ..." note, section 7).
    q_codes [B][Tq][Hi][c/2], q_sf [B][Tq][Hi][c/32], w [B][Tq][Hi],
    k_codes [B][Nc][c/2], k_sf [B][Nc][c/32], q_pos [B][Tq] -> scores [B][Tq][Nc]
    (-inf where the entry's block ends after the query).  Returns (scores, n_inexact)."""
    q_codes, q_sf, k_codes, k_sf = (_c(a, np.uint8) for a in (q_codes, q_sf, k_codes, k_sf))
    w, q_pos = _c(w, np.float32), _c(q_pos, np.int32)
    B, Tq, Hi, cb = q_codes.shape
    Nc = k_codes.shape[1]
    scores = np.empty((B, Tq, Nc), np.float32)
    n_inexact = lib().oracle_index_scores(_ptr(q_codes, ctypes.c_uint8), _ptr(q_sf, ctypes.c_uint8),
                                          _ptr(w, ctypes.c_float), _ptr(k_codes, ctypes.c_uint8),
                                          _ptr(k_sf, ctypes.c_uint8), _ptr(q_pos, ctypes.c_int32),
                                          B, Tq, Nc, Hi, cb * 2, m, _ptr(scores, ctypes.c_float))
    return scores, int(n_inexact)


def topk(scores, q_pos, m, k):
    """Top-k over eligible entries, ties to the lower index, indices ascending,
    padded with -1 ("DeepSeek V4 ..." note, section 7, Top-k selection).
    scores [R][Nc] fp32, q_pos [R] -> (idx [R][k] int32, count [R] int32)."""
    scores, q_pos = _c(scores, np.float32), _c(q_pos, np.int32)
    R, Nc = scores.shape
    idx = np.empty((R, k), np.int32)
    count = np.empty(R, np.int32)
    lib().oracle_topk(_ptr(scores, ctypes.c_float), _ptr(q_pos, ctypes.c_int32), R, Nc, m, k,
                      _ptr(idx, ctypes.c_int32), _ptr(count, ctypes.c_int32))
    return idx, count


# ---------------------------------------------------------------- attention
def attend(q_bits, codes, scales, rope, ent, win_bits, softmax_scale, g, q_norm_w=None, eps=1e-6, sink=None,
           inv_freq=None, q_pos=0):
    """Shared key-value MQA attention of one query token (H heads) over the
    listed compressed entries plus raw window tokens, one joint softmax, fp64
    ("DeepSeek V4 ..." note, sections 7-9; HF blog figures 3 and 4).
    q_bits [H][d] bf16 bits; codes/scales/rope: one sequence's cache;
    ent: entry indices; win_bits [n_win][d] bf16 bits.
    Optional note section 9 extras: q_norm_w [d] (query-head RMSNorm), sink [H]
    (per-head sink logit), inv_freq [d_rope/2] with q_pos (the query's RoPE
    dims rotated to q_pos, the output's rotated back).
    Returns (out fp64 [H][d], lse fp64 [H])."""
    q_bits = _c(q_bits, np.uint16)
    qn, qn_p = _opt(q_norm_w, np.float32, ctypes.c_float)
    sk, sk_p = _opt(sink, np.float32, ctypes.c_float)
    fq, fq_p = _opt(inv_freq, np.float32, ctypes.c_float)
    H, d = q_bits.shape
    codes, scales, rope = _c(codes, np.uint8), _c(scales, np.float32), _c(rope, np.uint16)
    d_rope = rope.shape[-1]
    ent = _c(ent, np.int64).reshape(-1)
    win_bits = _c(win_bits, np.uint16).reshape(-1, d)
    out = np.empty((H, d), np.float64)
    lse = np.empty(H, np.float64)
    lib().oracle_attend_ex(_ptr(q_bits, ctypes.c_uint16), H, d, d_rope, g, _ptr(codes, ctypes.c_uint8),
                           _ptr(scales, ctypes.c_float), _ptr(rope, ctypes.c_uint16), _ptr(ent, ctypes.c_int64),
                           ent.shape[0], _ptr(win_bits, ctypes.c_uint16), win_bits.shape[0],
                           float(softmax_scale), qn_p, float(eps), sk_p, fq_p, int(q_pos),
                           _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double))
    return out, lse


def round_bf16(x64: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 bits, rounded once to nearest (ties to even)."""
    x = np.ascontiguousarray(np.asarray(x64, dtype=np.float64))
    out = np.empty(x.shape, np.uint16)
    lib().oracle_f64_to_bf16_array(_ptr(x, ctypes.c_double), _ptr(out, ctypes.c_uint16), x.size)
    return out


# ---------------------------------------------------------------- causal key sets
def causal_keys(p: int, m: int, W: int, n_cap: int = None):
    """Keys visible to a query at absolute position p ("DeepSeek V4 ..." note,
    section 7: compressed entries plus the sliding window of the last n_win
    uncompressed tokens; an entry exists once its block is complete).
      entries: s = 0 .. min(n_cap, (p+1)//m) - 1, i.e. every block whose last
               token (s+1)m - 1 is at or before p (m = 0: none, the branch is off)
      window : raw positions max(0, p-W+1) .. p
    Returns (entry indices, first window position, last window position + 1)."""
    if m and m > 0:
        e = (p + 1) // m
        if n_cap is not None:
            e = min(e, n_cap)
    else:
        e = 0
    first = max(0, p - W + 1)
    return np.arange(max(e, 0)), first, p + 1


# ---------------------------------------------------------------- overlapped compressor (section 7)
def f32_to_e2m1(v) -> int:
    """e2m1 code of one fp32 value: nearest-even, saturating at +-6, sign kept."""
    return int(lib().oracle_f32_to_e2m1(float(np.float32(v))))


def fp4_quant_block(v):
    """One 32-element block -> (16 code bytes, ue8m0 byte): the OCP MX rule
    X = floor(log2 amax) - 2, codes e2m1(v / 2^X)."""
    v = _c(v, np.float32)
    assert v.shape == (32,)
    codes = np.empty(16, np.uint8)
    sf = np.empty(1, np.uint8)
    lib().oracle_fp4_quant_block(_ptr(v, ctypes.c_float), _ptr(codes, ctypes.c_uint8), _ptr(sf, ctypes.c_uint8))
    return codes, int(sf[0])


def _overlap_args(xa, za, xb, zb, a_prev, za_prev):
    xa, za, xb, zb = (_c(a, np.uint16) for a in (xa, za, xb, zb))
    ap = zp = None
    if a_prev is not None:
        ap, zp = _c(a_prev, np.uint16), _c(za_prev, np.uint16)
    return xa, za, xb, zb, ap, zp


def compress_overlap(xa, za, xb, zb, bias, m, n_blocks, d_rope, g, a_prev=None, za_prev=None, cap=None,
                     entry_begin=0):
    """The note's overlapped CSA compressor (section 7, two streams, 2m-token
    windows; reading in oracle.c): entry entry_begin+j pools block j-1 of
    stream a and block j of stream b (rows from row 0 = block entry_begin;
    a_prev / za_prev [B][>=m][d]: stream a's block before it, or None).
    bias [2m][d].  Returns (codes, scales, rope, worst fp32-vs-fp64 deviation)."""
    xa, za, xb, zb, ap, zp = _overlap_args(xa, za, xb, zb, a_prev, za_prev)
    bias = _c(bias, np.float32)
    B, T, d = xb.shape
    assert xa.shape == xb.shape and n_blocks * m <= T and bias.shape == (2 * m, d)
    assert ap is None or ap.shape[1] == T
    cap = entry_begin + n_blocks if cap is None else cap
    dn = d - d_rope
    codes = np.zeros((B, cap, dn), np.uint8)
    scales = np.zeros((B, cap, dn // g), np.float32)
    rope = np.zeros((B, cap, d_rope), np.uint16)
    u16 = lambda a: None if a is None else _ptr(a, ctypes.c_uint16)
    worst = lib().oracle_compress_overlap(u16(xa), u16(za), u16(xb), u16(zb), u16(ap), u16(zp), T,
                                          _ptr(bias, ctypes.c_float), m, B, n_blocks, d, d_rope, g,
                                          _ptr(codes, ctypes.c_uint8), _ptr(scales, ctypes.c_float),
                                          _ptr(rope, ctypes.c_uint16), cap, entry_begin)
    return codes, scales, rope, worst


def index_key_compress(xa, za, xb, zb, bias, m, n_blocks, a_prev=None, za_prev=None, cap=None, entry_begin=0):
    """Indexer keys K^IComp (note section 7): the overlapped compressor over
    c-channel indexer-key streams, stored FP4 (e2m1 + ue8m0 per 32).
    Returns (k_codes [B][cap][c/2], k_sf [B][cap][c/32])."""
    xa, za, xb, zb, ap, zp = _overlap_args(xa, za, xb, zb, a_prev, za_prev)
    bias = _c(bias, np.float32)
    B, T, c = xb.shape
    assert n_blocks * m <= T and bias.shape == (2 * m, c) and c % 32 == 0
    assert ap is None or ap.shape[1] == T
    cap = entry_begin + n_blocks if cap is None else cap
    kc = np.zeros((B, cap, c // 2), np.uint8)
    ks = np.zeros((B, cap, c // 32), np.uint8)
    u16 = lambda a: None if a is None else _ptr(a, ctypes.c_uint16)
    lib().oracle_index_key_compress(u16(xa), u16(za), u16(xb), u16(zb), u16(ap), u16(zp), T,
                                    _ptr(bias, ctypes.c_float), m, B, n_blocks, c, _ptr(kc, ctypes.c_uint8),
                                    _ptr(ks, ctypes.c_uint8), cap, entry_begin)
    return kc, ks

