"""Build the five synthetic workloads on the GPU from the seeded recipes in
``hca_inputs`` and the package's own compression kernels.

Used by the GPU tests, ``bench.py`` and the smoke check.  Building a decode
state is setup (not timed): raw KV and gate logits of every context token are
drawn on the device, pooled into the FP8/BF16 caches by ``csa_compress`` /
``hca_compress`` and dropped, keeping only the last W raw tokens (the
window).  ``on_raw(layer, ratio, x, gate, bias)`` lets a caller copy raw
blocks to the host (for the oracle) while they still exist.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, List, Optional

import torch

import hca_inputs as inp
from long_context_attention_hca_b200 import AttnExtras, EntryExtras, KVCache, csa_compress, hca_compress, kv_token_prep
from long_context_attention_hca_b200.pipeline import (CSA_RATIO, HCA_RATIO, DecodeLayer, PrefillState,
                                                       pro_layer_ratios)


@dataclasses.dataclass
class DecodeWorkload:
    wl: inp.Workload
    layers: List[DecodeLayer]
    ratios: List[int]
    q: List[torch.Tensor]                 # per layer [B][H][d] bf16
    iq: List[Optional[tuple]]             # per CSA layer (codes [B][1][Hi][c/2], sf, w [B][1][Hi])
    extras: Optional[List[AttnExtras]] = None     # per layer, section 9 extras of the attention call
    s9: Optional[List[dict]] = None               # per layer, the section 9 parameters (hca_inputs)
    raw_window: Optional[List[torch.Tensor]] = None   # per layer, the window before token preparation


def _compress(ratio, x, gate, bias, cache, n_blocks, extras=None):
    (csa_compress if ratio == CSA_RATIO else hca_compress)(x, gate, bias, n_blocks, cache, extras=extras)


def build_decode(wl: inp.Workload, device="cuda", on_raw: Optional[Callable] = None,
                 section9: bool = False) -> DecodeWorkload:
    """Decode state at position wl.t: every sequence holds tokens 0..t (t+1
    tokens, all blocks complete).  Single-layer workloads pair one CSA and one
    HCA path over the same raw KV (each with its own positional bias); the
    stack workload has independent inputs per layer.  section9: the note's
    section 9 extras are on: entries RMS-normalised and rotated when stored,
    window tokens prepared likewise, and the attention calls take the query
    RMSNorm, RoPE and sink (parameters from hca_inputs.section9_params)."""
    B, T, layout = wl.B, wl.t + 1, (wl.d, wl.d_rope, wl.g)
    stack = wl.layers > 1
    ratios = pro_layer_ratios(wl.layers) if stack else [CSA_RATIO, HCA_RATIO]
    layers, q, iq = [], [], []
    extras, s9s, raw_windows = [], [], []
    x = gate = None
    for li, r in enumerate(ratios):
        raw_layer = li if stack else 0
        if x is None or stack:
            x = gate = None
            torch.cuda.empty_cache()
            x, gate = inp.raw_kv(wl, B, T, layer=raw_layer, device=device)
        bias = inp.pos_bias(wl, r, layer=li if stack else 0, device=device)
        n_ent = T // r
        cache = KVCache(B, n_ent, layout, device=device)
        s9 = inp.section9_params(wl, layer=li if stack else 0, device=device) if section9 else None
        ee = EntryExtras(s9["kv_norm_w"], s9["eps"], s9["inv_freq"]) if section9 else None
        _compress(r, x, gate, bias, cache, n_ent, ee)
        if on_raw is not None:
            on_raw(li, r, x, gate, bias)
        window = x[:, T - wl.W:T].contiguous()
        if section9:
            raw_windows.append(window)
            pos = torch.arange(T - wl.W, T, dtype=torch.int32, device=device).repeat(B)
            window = kv_token_prep(window.view(B * wl.W, wl.d), pos, layout, ee).view(B, wl.W, wl.d)
            s9s.append(s9)
            extras.append(AttnExtras(s9["q_norm_w"], s9["eps"], s9["sink"], s9["inv_freq"],
                                     torch.full((B,), wl.t, dtype=torch.int32, device=device)))
        kc = ks = None
        if r == CSA_RATIO:
            kc, ks = inp.indexer_keys(wl, B, n_ent, layer=li, device=device)
        layers.append(DecodeLayer(r, cache, n_ent, window, kc, ks))
        q.append(inp.queries(wl, B, layer=li if stack else 0, device=device))
        if r == CSA_RATIO:
            qc, qs, w = inp.indexer_queries(wl, B, layer=li, device=device)
            iq.append((qc.view(B, 1, wl.Hi, wl.c // 2), qs.view(B, 1, wl.Hi, wl.c // 32), w.view(B, 1, wl.Hi)))
        else:
            iq.append(None)
        if stack:
            x = gate = None
    x = gate = None
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    if section9:
        return DecodeWorkload(wl, layers, ratios, q, iq, extras, s9s, raw_windows)
    return DecodeWorkload(wl, layers, ratios, q, iq)


@dataclasses.dataclass
class PrefillWorkload:
    wl: inp.Workload
    state: PrefillState
    raw_chunk: torch.Tensor               # [1][Tq][d]
    gate_chunk: torch.Tensor
    raw_window: torch.Tensor              # [(W-1)+Tq][d]
    q: torch.Tensor                       # [Tq][H][d]
    iq: tuple                             # ([1][Tq][Hi][c/2], sf, [1][Tq][Hi])
    x_all: Optional[torch.Tensor] = None  # kept when keep_raw=True (tests)
    gate_all: Optional[torch.Tensor] = None
    s9: Optional[dict] = None             # section 9 parameters when on
    raw_window_unprepared: Optional[torch.Tensor] = None


def build_prefill(wl: inp.Workload, device="cuda", keep_raw=False, section9: bool = False) -> PrefillWorkload:
    """One sequence with p0 = wl.t cached tokens already compressed into both
    caches, and the next Tq tokens (the chunk) still raw.  section9: entries
    and window tokens stored with the note's section 9 extras (the state
    holds the parameters; PrefillRunner takes the attention extras)."""
    p0, Tq, layout = wl.t, wl.Tq, (wl.d, wl.d_rope, wl.g)
    T = p0 + Tq
    x, gate = inp.raw_kv(wl, 1, T, device=device)
    b4 = inp.pos_bias(wl, CSA_RATIO, device=device)
    b128 = inp.pos_bias(wl, HCA_RATIO, device=device)
    csa = KVCache(1, T // CSA_RATIO, layout, device=device, zero=True)
    hca = KVCache(1, T // HCA_RATIO, layout, device=device, zero=True)
    s9 = inp.section9_params(wl, device=device) if section9 else None
    ee = EntryExtras(s9["kv_norm_w"], s9["eps"], s9["inv_freq"]) if section9 else None
    csa_compress(x, gate, b4, p0 // CSA_RATIO, csa, extras=ee)
    hca_compress(x, gate, b128, p0 // HCA_RATIO, hca, extras=ee)
    kc, ks = inp.indexer_keys(wl, 1, T // CSA_RATIO, device=device)
    st = PrefillState(csa, hca, kc, ks, b4, b128, ee)
    raw_chunk = x[:, p0:T].contiguous()
    gate_chunk = gate[:, p0:T].contiguous()
    raw_window = x[0, p0 - (wl.W - 1):T].contiguous()
    raw_unprepared = None
    if section9:
        raw_unprepared = raw_window
        pos = torch.arange(p0 - (wl.W - 1), T, dtype=torch.int32, device=device)
        raw_window = kv_token_prep(raw_window, pos, layout, ee)
    q = inp.queries(wl, Tq, device=device)
    qc, qs, w = inp.indexer_queries(wl, Tq, device=device)
    iq = (qc.view(1, Tq, wl.Hi, wl.c // 2), qs.view(1, Tq, wl.Hi, wl.c // 32), w.view(1, Tq, wl.Hi))
    pw = PrefillWorkload(wl, st, raw_chunk, gate_chunk, raw_window, q, iq, s9=s9,
                         raw_window_unprepared=raw_unprepared)
    if keep_raw:
        pw.x_all, pw.gate_all = x, gate
    torch.cuda.synchronize()
    return pw
