"""Host-side orchestration of the hot path: one decode step of a CSA and an
HCA layer, a chunked-prefill pass, and the 61-layer decode stack.

Everything here is launch plumbing around the C-ABI calls of this package:
buffers are allocated once, the CSA chain (indexer -> top-k -> attention)
and the HCA attention are queued on two streams (they share no data), and a
whole step can be captured into one CUDA graph.

Layer schedule ("DeepSeek V4 ..." reading note, section 8 table; Hugging
Face blog, "Hybrid attention: CSA and HCA"): in the 61-layer Pro stack,
layers 0 and 1 use the 128x compressor (HCA) and from layer 2 on even layers
are CSA (4x) and odd layers HCA.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import torch

from . import (KVCache, compressed_attn_decode, compressed_attn_prefill, csa_compress, decode_workspace_size,
               hca_compress, lightning_index, lightning_index_topk, topk_select, topk_workspace_size,
               set_launch_budget, BUDGET_DENSE_DECODE)

CSA_RATIO = 4
HCA_RATIO = 128


def pro_layer_ratios(n_layers: int = 61) -> List[int]:
    """compress_ratio of each layer of the Pro stack (4 = CSA, 128 = HCA)."""
    return [HCA_RATIO if (i < 2 or i % 2 == 1) else CSA_RATIO for i in range(n_layers)]


def kv_resident_bytes(B, n_tokens, ratios, d=512, d_rope=64, g=64, c=128, W=128) -> int:
    """Bytes one decode state holds: compressed entries (FP8 codes + fp32
    scales + bf16 RoPE), FP4 indexer keys + ue8m0 scales for CSA layers, and
    the raw bf16 window."""
    dn = d - d_rope
    entry = dn + 4 * (dn // g) + 2 * d_rope
    ikey = c // 2 + c // 32
    total = 0
    for r in ratios:
        ne = n_tokens // r
        total += B * ne * entry
        if r == CSA_RATIO:
            total += B * ne * ikey
        total += B * W * d * 2
    return total


def gqa_bf16_bytes(B, n_tokens, n_layers, kv_heads=8, head_dim=128) -> int:
    """The same context as a grouped-query-attention cache in bf16 (K and V)."""
    return B * n_tokens * n_layers * 2 * kv_heads * head_dim * 2


@dataclasses.dataclass
class DecodeLayer:
    """Resident decode state of one attention layer."""
    ratio: int                          # 4 (CSA) or 128 (HCA)
    cache: KVCache
    n_entries: int                      # complete blocks per sequence
    window: torch.Tensor                # [B][W][d] bf16, last W raw tokens
    k_codes: Optional[torch.Tensor] = None   # CSA: indexer keys [B][Nc][c/2]
    k_sf: Optional[torch.Tensor] = None      # CSA: [B][Nc][c/32]


class DecodeRunner:
    """Queues one decode step over a list of layers.  Per layer: CSA ->
    lightning_index, topk_select, compressed_attn_decode(sparse); HCA ->
    compressed_attn_decode(dense).  CSA chains run on `side`, a stream of
    higher priority, and HCA on the current stream; the step ends with both
    joined.  An HCA launch waits for the indexer queued before it: the
    indexer fills every SM anyway, and the top-k that follows it needs whole
    clusters of free SMs, which the HCA CTAs (one per SM) would otherwise
    hold when the indexer drains."""

    def __init__(self, layers: List[DecodeLayer], B: int, H: int, k: int, pos: int, softmax_scale: float,
                 device="cuda", schedule: str = "after_index", dense_budget: int = 0, fused_select: bool = True):
        """schedule: "after_index" -- an HCA launch waits for the indexer queued
        before it; "hca_first" -- all HCA launches are queued first and start at
        once, with dense_budget (if > 0) capping their CTAs so that the CSA
        chain runs beside them on the remaining SMs."""
        if schedule not in ("after_index", "hca_first"):
            raise ValueError(schedule)
        self.schedule = schedule
        if dense_budget:
            set_launch_budget(BUDGET_DENSE_DECODE, dense_budget)
        self.layers, self.B, self.H, self.k, self.pos = layers, B, H, k, pos
        self.scale = softmax_scale
        d = layers[0].cache.layout[0]
        self.d = d
        dev = torch.device(device)
        self.q_pos = torch.full((B, 1), pos, dtype=torch.int32, device=dev)
        self.out = [torch.empty((B, H, d), dtype=torch.bfloat16, device=dev) for _ in layers]
        self.n_dense = {}
        self.scores, self.idx, self.count, self.ws, self.topk_ws, self.fused_select = {}, {}, {}, {}, {}, {}
        self.index_done = {}
        W = layers[0].window.shape[1]
        for li, L in enumerate(layers):
            if L.ratio == CSA_RATIO:
                self.scores[li] = torch.empty((B, 1, L.n_entries), dtype=torch.float32, device=dev)
                self.idx[li] = torch.empty((B, k), dtype=torch.int32, device=dev)
                self.count[li] = torch.empty((B,), dtype=torch.int32, device=dev)
                self.topk_ws[li] = torch.empty(max(topk_workspace_size(B, L.n_entries, k), 16), dtype=torch.uint8,
                                               device=dev)
                # the fused index + top-k call pays off when top-k takes the histogram path
                self.fused_select[li] = fused_select and topk_workspace_size(B, L.n_entries, k) > 0
                # recorded inside the fused call once the scores exist (created here, outside any capture)
                self.index_done[li] = torch.cuda.Event()
                self.index_done[li].record(torch.cuda.current_stream(dev))
                mc = min(k, L.n_entries)
            else:
                self.n_dense[li] = torch.full((B,), L.n_entries, dtype=torch.int32, device=dev)
                mc = L.n_entries
            nbytes = decode_workspace_size(B, H, L.cache.layout, mc, W)
            self.ws[li] = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
        lo, hi = torch.cuda.Stream.priority_range()
        self.side = torch.cuda.Stream(device=dev, priority=hi)
        self.copy_in = torch.cuda.Stream(device=dev)     # step_host: attention queries in
        self.copy_out = torch.cuda.Stream(device=dev)    # step_host: outputs out
        self.kernels_per_step = self._count_kernels()

    def _count_kernels(self) -> int:
        """Kernels of this library launched per step: attention (+ split combine) per
        layer; per CSA layer the indexer and the top-k (three kernels on the
        histogram path, one on the cluster path)."""
        n = 0
        for li, L in enumerate(self.layers):
            mc = min(self.k, L.n_entries) if L.ratio == CSA_RATIO else L.n_entries
            split = decode_workspace_size(self.B, self.H, L.cache.layout, mc, L.window.shape[1]) > 0
            n += 1 + int(split)
            if L.ratio == CSA_RATIO:
                wide = topk_workspace_size(self.B, L.n_entries, self.k) > 0
                # indexer + (histogram,) mark, resolve on the histogram path; else the cluster kernel
                n += 1 + ((2 if self.fused_select[li] else 3) if wide else 1)
        return n

    def step_host(self, h_q: List[torch.Tensor], h_iq: List[Optional[tuple]], h_out: List[torch.Tensor],
                  d_q: List[torch.Tensor], d_iq: List[Optional[tuple]]):
        """One decode step from pinned host memory to pinned host memory.  The
        indexer queries (a few hundred bytes) are copied first, on the current
        stream; the attention queries stream in on a copy stream while the
        indexer runs, and each layer's output streams out as soon as its
        attention is done.  d_q / d_iq are the device buffers of the inputs."""
        main = torch.cuda.current_stream()
        for a, b in zip(d_iq, h_iq):
            if a is not None:
                for x, y in zip(a, b):
                    x.copy_(y, non_blocking=True)
        self.copy_in.wait_stream(main)
        q_ready = {}
        with torch.cuda.stream(self.copy_in):
            for li, (a, b) in enumerate(zip(d_q, h_q)):
                a.copy_(b, non_blocking=True)
                q_ready[li] = torch.cuda.Event()
                q_ready[li].record(self.copy_in)
        self.copy_out.wait_stream(main)

        def on_out(li, stream):
            done = torch.cuda.Event()
            done.record(stream)
            self.copy_out.wait_event(done)
            with torch.cuda.stream(self.copy_out):
                h_out[li].copy_(self.out[li], non_blocking=True)

        self.step(d_q, d_iq, q_ready=q_ready, on_out=on_out)
        main.wait_stream(self.copy_in)
        main.wait_stream(self.copy_out)
        return h_out

    def step(self, q: List[torch.Tensor], iq: List[Optional[tuple]], events: Optional[dict] = None,
             q_ready: Optional[dict] = None, on_out=None):
        """q[li]: [B][H][d] bf16; iq[li]: (codes [B][1][Hi][c/2], sf, w [B][1][Hi]) for CSA layers.
        events: if a dict is given, timing events (recorded as graph nodes
        when captured) bracket each launch: events[name] = (start, end) with
        name in indexer/topk/csa_attn/hca_attn (suffixed by the layer index
        when there are several layers).  q_ready: optional {layer: event} that
        an attention launch waits for (its query copy); on_out(layer, stream):
        called after each attention launch (to stream the output out)."""
        main = torch.cuda.current_stream()
        self.side.wait_stream(main)
        multi = len(self.layers) > 2

        def timed(name, li, fn):
            if events is None:
                return fn()
            key = f"{name}{li}" if multi else name
            a = torch.cuda.Event(enable_timing=True, external=True)
            b = torch.cuda.Event(enable_timing=True, external=True)
            a.record()
            fn()
            b.record()
            events[key] = (a, b)

        after_index = None
        order = list(range(len(self.layers)))
        if self.schedule == "hca_first":
            order = [li for li in order if self.layers[li].ratio != CSA_RATIO] + \
                    [li for li in order if self.layers[li].ratio == CSA_RATIO]
        for li in order:
            L = self.layers[li]
            if L.ratio == CSA_RATIO:
                with torch.cuda.stream(self.side):
                    qc, qs, w = iq[li]
                    if self.fused_select[li]:
                        # indexer (with the top-k's key histogram) + top-k passes in one call
                        timed("index_topk", li, lambda: lightning_index_topk(
                            qc, qs, w, L.k_codes, L.k_sf, self.q_pos.view(-1), CSA_RATIO, self.k,
                            scores=self.scores[li], idx=self.idx[li], count=self.count[li], ws=self.topk_ws[li],
                            index_done=self.index_done[li], stream=self.side))
                        after_index = self.index_done[li]
                    else:
                        timed("indexer", li, lambda: lightning_index(qc, qs, w, L.k_codes, L.k_sf, self.q_pos,
                                                                     CSA_RATIO, scores=self.scores[li]))
                        after_index = torch.cuda.Event()
                        after_index.record(self.side)
                        timed("topk", li, lambda: topk_select(self.scores[li].view(self.B, -1), self.q_pos.view(-1),
                                                              CSA_RATIO, self.k, idx=self.idx[li],
                                                              count=self.count[li], ws=self.topk_ws[li]))
                    if q_ready is not None:
                        self.side.wait_event(q_ready[li])
                    timed("csa_attn", li, lambda: compressed_attn_decode(
                        q[li], L.cache, self.count[li], min(self.k, L.n_entries), L.window, self.scale,
                        idx=self.idx[li], out=self.out[li], ws=self.ws[li]))
                    if on_out is not None:
                        on_out(li, self.side)
            else:
                if after_index is not None and self.schedule == "after_index":
                    main.wait_event(after_index)
                if q_ready is not None:
                    main.wait_event(q_ready[li])
                timed("hca_attn", li, lambda: compressed_attn_decode(
                    q[li], L.cache, self.n_dense[li], L.n_entries, L.window, self.scale, out=self.out[li],
                    ws=self.ws[li]))
                if on_out is not None:
                    on_out(li, main)
        main.wait_stream(self.side)
        return self.out


@dataclasses.dataclass
class PrefillState:
    """One sequence's state for a chunked-prefill pass."""
    csa: KVCache                        # capacity >= (p0 + Tq) / 4
    hca: KVCache                        # capacity >= (p0 + Tq) / 128
    k_codes: torch.Tensor               # [1][Nc_csa][c/2] indexer keys of every CSA entry
    k_sf: torch.Tensor
    bias4: torch.Tensor                 # [4][d]
    bias128: torch.Tensor               # [128][d]


class PrefillRunner:
    """One prefill chunk of Tq tokens at positions p0..p0+Tq-1 (p0 a multiple
    of 128): compress the chunk's complete blocks into both caches, score
    every CSA entry for every query (causal), select top-k per query, then
    CSA (sparse) and HCA (dense causal) attention with the causal window."""

    def __init__(self, st: PrefillState, p0: int, Tq: int, H: int, k: int, W: int, softmax_scale: float,
                 device="cuda"):
        assert p0 % HCA_RATIO == 0 and Tq % HCA_RATIO == 0
        self.st, self.p0, self.Tq, self.H, self.k, self.W, self.scale = st, p0, Tq, H, k, W, softmax_scale
        dev = torch.device(device)
        self.q_pos = torch.arange(p0, p0 + Tq, dtype=torch.int32, device=dev).view(1, Tq)
        self.nc_csa = (p0 + Tq) // CSA_RATIO
        self.scores = torch.empty((1, Tq, self.nc_csa), dtype=torch.float32, device=dev)
        self.idx = torch.empty((Tq, k), dtype=torch.int32, device=dev)
        self.count = torch.empty((Tq,), dtype=torch.int32, device=dev)
        d = st.csa.layout[0]
        self.out_csa = torch.empty((Tq, H, d), dtype=torch.bfloat16, device=dev)
        self.out_hca = torch.empty((Tq, H, d), dtype=torch.bfloat16, device=dev)
        lo, hi = torch.cuda.Stream.priority_range()
        self.side = torch.cuda.Stream(device=dev, priority=hi)
        self.copy_in = torch.cuda.Stream(device=dev)     # step_host: attention queries in
        self.copy_out = torch.cuda.Stream(device=dev)    # step_host: outputs out
        self.kernels_per_step = 6

    def step(self, raw_chunk, gate_chunk, raw_window, q, iq, events: Optional[dict] = None):
        """raw_chunk, gate_chunk: [1][Tq][d] bf16 tokens p0..p0+Tq-1;
        raw_window: [(W-1)+Tq][d] bf16 tokens from p0-(W-1); q: [Tq][H][d];
        iq = (codes [1][Tq][Hi][c/2], sf, w [1][Tq][Hi]).  events: as in
        DecodeRunner.step (names compress, indexer, topk, csa_attn, hca_attn)."""
        st, p0, Tq = self.st, self.p0, self.Tq
        main = torch.cuda.current_stream()

        def timed(name, fn):
            if events is None:
                return fn()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            events[name] = (a, b)

        def compress():
            csa_compress(raw_chunk, gate_chunk, st.bias4, Tq // CSA_RATIO, st.csa, entry_begin=p0 // CSA_RATIO)
            hca_compress(raw_chunk, gate_chunk, st.bias128, Tq // HCA_RATIO, st.hca, entry_begin=p0 // HCA_RATIO)

        timed("compress", compress)
        self.side.wait_stream(main)
        with torch.cuda.stream(self.side):
            qc, qs, w = iq
            timed("indexer", lambda: lightning_index(qc, qs, w, st.k_codes, st.k_sf, self.q_pos, CSA_RATIO,
                                                     scores=self.scores))
            timed("topk", lambda: topk_select(self.scores.view(Tq, -1), self.q_pos.view(-1), CSA_RATIO, self.k,
                                              idx=self.idx, count=self.count))
            timed("csa_attn", lambda: compressed_attn_prefill(q, p0, CSA_RATIO, st.csa, raw_window, self.W,
                                                              self.scale, idx=self.idx, count=self.count,
                                                              out=self.out_csa))
        timed("hca_attn", lambda: compressed_attn_prefill(q, p0, HCA_RATIO, st.hca, raw_window, self.W, self.scale,
                                                          out=self.out_hca))
        main.wait_stream(self.side)
        return self.out_csa, self.out_hca
