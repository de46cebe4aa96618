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

import contextlib
import dataclasses
from typing import List, Optional

import torch

from . import (KVCache, compressed_attn_decode, compressed_attn_prefill, csa_compress, decode_workspace_size,
               hca_compress, lightning_index, lightning_index_topk, topk_select, topk_workspace_size,
               set_launch_budget, set_early_query, BUDGET_DENSE_DECODE, BUDGET_SPARSE_DECODE, BUDGET_DECODE_INDEX)

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


def packed_indexer_query(iq, device=None, pin: bool = False):
    """A copy of one layer's indexer query (codes, scales, weights) in one
    byte buffer, in that order, each part from a 16-byte boundary: views of
    the same shapes and dtypes.  hca_decode_step_host moves such a query with
    one copy when its host and device buffers are both packed so."""
    parts = tuple(iq)
    sizes = [t.numel() * t.element_size() for t in parts]
    offs = [0]
    for n in sizes[:-1]:
        offs.append(offs[-1] + (n + 15) // 16 * 16)
    dev = torch.device(device) if device is not None else parts[0].device
    buf = torch.zeros(offs[-1] + sizes[-1], dtype=torch.uint8, device=dev, pin_memory=pin and dev.type == "cpu")
    out = []
    for t, n, off in zip(parts, sizes, offs):
        v = buf[off:off + n].view(t.dtype).view(t.shape)
        v.copy_(t)
        out.append(v)
    return tuple(out)


def dense_beside_select(sm: int, B: int) -> int:
    """CTA cap of a decode step's dense (HCA) attention beside the top-k select of B
    rows: the SMs that the select's B * floor(sm / 2 / B) CTAs leave, at least half
    of them (the C host step's default for hca_ctas)."""
    return max(sm // 2, sm - B * max(1, (sm // 2) // max(B, 1)))


class DecodeRunner:
    """Queues one decode step over a list of layers.  Per layer: CSA ->
    lightning_index, topk_select, compressed_attn_decode(sparse); HCA ->
    compressed_attn_decode(dense).  CSA chains run on `side`, a stream of
    higher priority, and HCA on the current stream; the step ends with both
    joined.  An HCA launch waits for the indexer queued before it: the
    indexer fills every SM anyway."""

    def __init__(self, layers: List[DecodeLayer], B: int, H: int, k: int, pos: int, softmax_scale: float,
                 device="cuda", dense_budget: Optional[int] = None,
                 fused_select: bool = True, sparse_budget: int = 0, extras: Optional[list] = None,
                 index_budget: int = 0):
        """An HCA launch waits for the indexer queued before it (queued first, the
        HCA launches measured no faster).  dense_budget caps the CTAs of this
        runner's HCA launches (applied
        around its own calls only): None -- when the step is one CSA layer
        beside one HCA layer, the SMs that the top-k select's B * floor(SMs / 2
        / B) CTAs leave, at least half (the select and then the CSA attention
        keep the rest), else the library default (in a deep stack both streams
        stay busy and the HCA launches do better on every SM: 3.46 against
        3.62 ms per step for 61 layers at 32 x 256K); 0 -- the library default.
        extras: per layer,
        an AttnExtras (section 9 query RMSNorm, RoPE, sink) for its attention
        call, or None."""
        self.extras = extras if extras is not None else [None] * len(layers)
        dev = torch.device(device)
        if dense_budget is None:
            pair = len(layers) == 2 and sorted(L.ratio == CSA_RATIO for L in layers) == [False, True]
            sm = torch.cuda.get_device_properties(dev).multi_processor_count
            dense_budget = dense_beside_select(sm, B) if pair else 0
        self.dense_budget = dense_budget
        if sparse_budget:
            set_launch_budget(BUDGET_SPARSE_DECODE, sparse_budget)
        if index_budget:
            set_launch_budget(BUDGET_DECODE_INDEX, index_budget)
        self.layers, self.B, self.H, self.k, self.pos = layers, B, H, k, pos
        self.scale = softmax_scale
        d = layers[0].cache.layout[0]
        self.d = d
        self.q_pos = torch.full((B, 1), pos, dtype=torch.int32, device=dev)
        # the layers' outputs back to back (hca_decode_step_host then copies both at once)
        self.out = list(torch.empty((len(layers), B, H, d), dtype=torch.bfloat16, device=dev).unbind(0))
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
            with self._dense_scope(L.ratio != CSA_RATIO):
                nbytes = decode_workspace_size(B, H, L.cache.layout, mc, W)
            self.ws[li] = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
        lo, hi = torch.cuda.Stream.priority_range()
        self.side = torch.cuda.Stream(device=dev, priority=hi)
        self.copy_in = torch.cuda.Stream(device=dev)     # step_host: attention queries in
        self.copy_out = torch.cuda.Stream(device=dev)    # step_host: outputs out
        self.kernels_per_step = self._count_kernels()

    @contextlib.contextmanager
    def _dense_scope(self, on: bool):
        """This runner's HCA CTA budget, around its own dense calls only."""
        if not on or not self.dense_budget:
            yield
            return
        prev = set_launch_budget(BUDGET_DENSE_DECODE, self.dense_budget)
        try:
            yield
        finally:
            set_launch_budget(BUDGET_DENSE_DECODE, prev)

    @staticmethod
    @contextlib.contextmanager
    def _early_query_scope():
        """The CSA attention may load its query before it waits for the top-k: the
        side stream waited for the caller's stream before the indexer, so every
        query passed to step() is complete before the top-k starts."""
        prev = set_early_query(True)
        try:
            yield
        finally:
            set_early_query(prev)

    def _count_kernels(self) -> int:
        """Kernels of this library launched per step: attention (+ split combine) per
        layer; per CSA layer the indexer and the top-k (the select kernel, after
        a histogram kernel unless the indexer built the histogram, on the
        histogram path; one cluster kernel otherwise)."""
        n = 0
        for li, L in enumerate(self.layers):
            mc = min(self.k, L.n_entries) if L.ratio == CSA_RATIO else L.n_entries
            with self._dense_scope(L.ratio != CSA_RATIO):
                split = decode_workspace_size(self.B, self.H, L.cache.layout, mc, L.window.shape[1]) > 0
            n += 1 + int(split)
            if L.ratio == CSA_RATIO:
                wide = topk_workspace_size(self.B, L.n_entries, self.k) > 0
                n += 1 + ((1 if self.fused_select[li] else 2) if wide else 1)
        return n

    def capi_plan(self, d_q: List[torch.Tensor], d_iq: List[Optional[tuple]], packed: int = 0):
        """The hca_decode_step_plan of this runner's two layers (one CSA, one
        HCA), for hca_decode_step_host: the caches, keys and windows of the
        layers, d_q / d_iq as the staging buffers of the queries, this runner's
        scores, top-k and attention buffers, a side stream and five events.
        packed: the plan's packing bits (1: the indexer query's arrays, host
        and device, as packed_indexer_query lays them out; 2: the host outputs
        back to back in one allocation, as this runner's device outputs are)."""
        from . import CacheStruct, DecodeStepPlan, Layout
        ci = [li for li, L in enumerate(self.layers) if L.ratio == CSA_RATIO]
        hi = [li for li, L in enumerate(self.layers) if L.ratio == HCA_RATIO]
        if len(ci) != 1 or len(hi) != 1:
            raise ValueError("capi_plan: one CSA and one HCA layer")
        c_, h_ = ci[0], hi[0]
        Lc, Lh = self.layers[c_], self.layers[h_]
        qc, qs, w = d_iq[c_]
        lo, hi_prio = torch.cuda.Stream.priority_range()
        self._capi_side = torch.cuda.Stream(device=d_q[0].device, priority=hi_prio)   # the CSA chain
        self._capi_events = [torch.cuda.Event() for _ in range(5)]
        for e in self._capi_events:
            e.record(torch.cuda.current_stream())     # creates the CUDA event (outside any capture)
        torch.cuda.synchronize()
        ptr = lambda t: t.data_ptr()
        p = DecodeStepPlan()
        p.B, p.H, p.Hi, p.c, p.k, p.W = self.B, self.H, qc.shape[2], qc.shape[3] * 2, self.k, Lc.window.shape[1]
        p.softmax_scale = self.scale
        p.layout = Layout(*Lc.cache.layout)
        p.csa_cache = Lc.cache.c_struct
        p.csa_entries = Lc.n_entries
        p.k_codes, p.k_sf, p.csa_window = ptr(Lc.k_codes), ptr(Lc.k_sf), ptr(Lc.window)
        p.hca_cache = Lh.cache.c_struct
        p.hca_n, p.hca_max, p.hca_window = ptr(self.n_dense[h_]), Lh.n_entries, ptr(Lh.window)
        p.q_pos = ptr(self.q_pos)
        p.q_csa, p.q_hca = ptr(d_q[c_]), ptr(d_q[h_])
        p.iq_codes, p.iq_sf, p.iq_w = ptr(qc), ptr(qs), ptr(w)
        p.scores, p.idx, p.count = ptr(self.scores[c_]), ptr(self.idx[c_]), ptr(self.count[c_])
        p.topk_ws, p.topk_ws_bytes = ptr(self.topk_ws[c_]), self.topk_ws[c_].numel()
        p.ws_csa, p.ws_csa_bytes = ptr(self.ws[c_]), self.ws[c_].numel()
        p.ws_hca, p.ws_hca_bytes = ptr(self.ws[h_]), self.ws[h_].numel()
        p.out_csa, p.out_hca = ptr(self.out[c_]), ptr(self.out[h_])
        p.side_stream = self._capi_side.cuda_stream
        p.ev_fork, p.ev_index, p.ev_q, p.ev_join, p.ev_iq = (e.cuda_event for e in self._capi_events)
        p.hca_ctas = self.dense_budget
        p.packed = packed
        self._capi_layers = (c_, h_)
        return p

    def step_host_capi(self, plan, h_q: List[torch.Tensor], h_iq: List[Optional[tuple]], h_out: List[torch.Tensor]):
        """One decode step through hca_decode_step_host (the C ABI's host-to-host
        call): pinned host queries in, pinned host outputs out."""
        from . import decode_step_host
        c_, h_ = self._capi_layers
        decode_step_host(plan, h_q[c_], h_q[h_], h_iq[c_], h_out[c_], h_out[h_])
        return h_out

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
        for li in range(len(self.layers)):
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
                    with self._early_query_scope():
                        timed("csa_attn", li, lambda: compressed_attn_decode(
                            q[li], L.cache, self.count[li], min(self.k, L.n_entries), L.window, self.scale,
                            idx=self.idx[li], out=self.out[li], ws=self.ws[li], extras=self.extras[li]))
                    if on_out is not None:
                        on_out(li, self.side)
            else:
                if after_index is not None:
                    main.wait_event(after_index)
                if q_ready is not None:
                    main.wait_event(q_ready[li])
                with self._dense_scope(True):
                    timed("hca_attn", li, lambda: compressed_attn_decode(
                        q[li], L.cache, self.n_dense[li], L.n_entries, L.window, self.scale, out=self.out[li],
                        ws=self.ws[li], extras=self.extras[li]))
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
    entry_extras: object = None         # EntryExtras used when the chunk's entries are stored (or None)


class PrefillRunner:
    """One prefill chunk of Tq tokens at positions p0..p0+Tq-1 (p0 a multiple
    of 128): compress the chunk's complete blocks into both caches, score
    every CSA entry for every query (causal), select top-k per query, then
    CSA (sparse) and HCA (dense causal) attention with the causal window."""

    def __init__(self, st: PrefillState, p0: int, Tq: int, H: int, k: int, W: int, softmax_scale: float,
                 device="cuda", extras=None):
        """extras: an AttnExtras (section 9 query RMSNorm, RoPE, sink) for both
        attention calls, or None."""
        self.extras = extras
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
            # external events stay timing events when the step is captured into a graph
            a = torch.cuda.Event(enable_timing=True, external=True)
            b = torch.cuda.Event(enable_timing=True, external=True)
            a.record()
            fn()
            b.record()
            events[name] = (a, b)

        def compress():
            csa_compress(raw_chunk, gate_chunk, st.bias4, Tq // CSA_RATIO, st.csa, entry_begin=p0 // CSA_RATIO,
                         extras=st.entry_extras)
            hca_compress(raw_chunk, gate_chunk, st.bias128, Tq // HCA_RATIO, st.hca, entry_begin=p0 // HCA_RATIO,
                         extras=st.entry_extras)

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
                                                              out=self.out_csa, extras=self.extras))
        timed("hca_attn", lambda: compressed_attn_prefill(q, p0, HCA_RATIO, st.hca, raw_window, self.W, self.scale,
                                                          out=self.out_hca, extras=self.extras))
        main.wait_stream(self.side)
        return self.out_csa, self.out_hca


# ------------------------------------------------------------------ state-cache decode loop
@dataclasses.dataclass
class LoopLayer:
    """One layer of a state-cache decode loop: the classical cache of
    compressed entries (none for ratio 0), and the per-sequence state cache:
    the window ring of the last W tokens and the raw tail of the block not yet
    complete ("DeepSeek V4 ..." note, section 11, KV cache table)."""
    ratio: int                                  # 0 (window only), 4 (CSA) or 128 (HCA)
    window: torch.Tensor                        # [B][W][d] ring, token at position p in row p % W
    cache: Optional[KVCache] = None             # capacity = max_tokens // ratio
    tail_x: Optional[torch.Tensor] = None       # [B][ratio][d] the current block's raw tokens
    tail_gate: Optional[torch.Tensor] = None
    bias: Optional[torch.Tensor] = None         # [ratio][d]
    k_codes: Optional[torch.Tensor] = None      # CSA: indexer keys of every entry [B][cap][c/2]
    k_sf: Optional[torch.Tensor] = None
    entry_extras: object = None                 # EntryExtras (section 9) or None
    s9: Optional[dict] = None                   # section 9 attention parameters (q_norm_w, sink, inv_freq, eps)


class DecodeLoop:
    """Token-by-token decode over a state cache.  All B sequences advance in
    lockstep; step(t) takes token t of every sequence, for each layer:
      1. appends it to the window ring and the block tail (kv_state_append;
         with the section 9 extras the window keeps the token RMS-normalised
         and rotated, kv_token_prep);
      2. pools the block when t is its last token (csa_compress /
         hca_compress of the tail into entry (t+1)/m - 1);
      3. runs attention at position t: CSA layers index every eligible entry,
         select the top-k and attend to them plus the window; HCA layers
         attend to every complete entry plus the window; ratio-0 layers (the
         note's section 8 compress_ratio table: compressed branch disabled)
         attend to the window alone.  Before the window is full only its
         first t+1 rows hold tokens (win_len)."""

    def __init__(self, B: int, H: int, layout, ratios: List[int], W: int, k: int, max_tokens: int,
                 softmax_scale: float, Hi: int = 4, c: int = 128, device="cuda", s9: Optional[List[dict]] = None):
        from . import EntryExtras
        d, dr, g = layout
        dev = torch.device(device)
        self.B, self.H, self.layout, self.W, self.k, self.scale = B, H, tuple(layout), W, k, softmax_scale
        self.ratios, self.max_tokens, self.Hi, self.c = list(ratios), max_tokens, Hi, c
        self.layers: List[LoopLayer] = []
        for li, r in enumerate(ratios):
            P = s9[li] if s9 is not None else None
            L = LoopLayer(r, torch.zeros((B, W, d), dtype=torch.bfloat16, device=dev), s9=P)
            if P is not None:
                L.entry_extras = EntryExtras(P["kv_norm_w"], P["eps"], P["inv_freq"])
            if r > 0:
                L.cache = KVCache(B, max_tokens // r, layout, device=dev, zero=True)
                L.tail_x = torch.zeros((B, r, d), dtype=torch.bfloat16, device=dev)
                L.tail_gate = torch.zeros((B, r, d), dtype=torch.bfloat16, device=dev)
            self.layers.append(L)
        # a one-entry cache for window-only layers (the attention call takes a cache; it reads no entry)
        self._empty = KVCache(B, 1, layout, device=dev, zero=True)
        self.q_pos = torch.zeros((B,), dtype=torch.int32, device=dev)
        self.win_len = torch.zeros((B,), dtype=torch.int32, device=dev)
        self.n_ent = {r: torch.zeros((B,), dtype=torch.int32, device=dev) for r in set(ratios)}
        self.out = [torch.empty((B, H, d), dtype=torch.bfloat16, device=dev) for _ in ratios]
        self.scores, self.idx, self.count, self.topk_ws, self.ws = {}, {}, {}, {}, {}
        for li, L in enumerate(self.layers):
            mc = 0
            if r_is_csa(L.ratio):
                cap = L.cache.capacity
                self.scores[li] = torch.empty((B, 1, cap), dtype=torch.float32, device=dev)
                self.idx[li] = torch.empty((B, k), dtype=torch.int32, device=dev)
                self.count[li] = torch.empty((B,), dtype=torch.int32, device=dev)
                self.topk_ws[li] = torch.empty(max(topk_workspace_size(B, cap, k), 16), dtype=torch.uint8,
                                               device=dev)
                mc = min(k, cap)
            elif L.ratio > 0:
                mc = L.cache.capacity
            self.ws[li] = torch.empty(max(decode_workspace_size(B, H, layout, mc, W), 16), dtype=torch.uint8,
                                      device=dev)

    def set_indexer_keys(self, li: int, k_codes: torch.Tensor, k_sf: torch.Tensor):
        """CSA layer li: the indexer key of every entry the loop may create
        ([B][max_tokens/4][c/2], [B][max_tokens/4][c/32]; given inputs)."""
        self.layers[li].k_codes, self.layers[li].k_sf = k_codes, k_sf

    def load_prefix(self, li: int, x: torch.Tensor, gate: torch.Tensor, bias: torch.Tensor, t0: int):
        """State of layer li after tokens 0..t0-1 (x, gate: [B][>=t0][d]): every
        complete block pooled, the tail holding the incomplete block's tokens,
        the window ring holding the last min(W, t0) tokens."""
        L = self.layers[li]
        L.bias = bias
        r = L.ratio
        if r > 0:
            n_blk = t0 // r
            if n_blk:
                (csa_compress if r == CSA_RATIO else hca_compress)(x, gate, bias, n_blk, L.cache,
                                                                   extras=L.entry_extras)
            for p in range(n_blk * r, t0):
                L.tail_x[:, p % r].copy_(x[:, p])
                L.tail_gate[:, p % r].copy_(gate[:, p])
        from . import kv_token_prep
        for p in range(max(0, t0 - self.W), t0):
            tok = x[:, p].contiguous()
            if L.entry_extras is not None:
                pos = torch.full((self.B,), p, dtype=torch.int32, device=tok.device)
                tok = kv_token_prep(tok, pos, self.layout, L.entry_extras)
            L.window[:, p % self.W].copy_(tok)

    def step(self, t: int, x_new: List[torch.Tensor], gate_new: List[torch.Tensor], q: List[torch.Tensor],
             iq: List[Optional[tuple]], stream=None):
        """Token t of every sequence: x_new[li], gate_new[li] [B][d] bf16,
        q[li] [B][H][d] bf16, iq[li] (codes [B][1][Hi][c/2], sf, w [B][1][Hi])
        for CSA layers.  Returns the per-layer outputs [B][H][d]."""
        from . import AttnExtras, kv_state_append, kv_token_prep
        self.q_pos.fill_(t)
        self.win_len.fill_(min(self.W, t + 1))
        for r, n in self.n_ent.items():
            n.fill_((t + 1) // r if r > 0 else 0)
        for li, L in enumerate(self.layers):
            win_x = None
            if L.entry_extras is not None:
                win_x = kv_token_prep(x_new[li], self.q_pos, self.layout, L.entry_extras)
            kv_state_append(x_new[li], gate_new[li], t, L.window, L.tail_x, L.tail_gate, win_x=win_x,
                            stream=stream)
            r = L.ratio
            if r > 0 and (t + 1) % r == 0:
                (csa_compress if r == CSA_RATIO else hca_compress)(L.tail_x, L.tail_gate, L.bias, 1, L.cache,
                                                                   entry_begin=(t + 1) // r - 1,
                                                                   extras=L.entry_extras, stream=stream)
            P = L.s9
            ex = AttnExtras(P["q_norm_w"] if P else None, P["eps"] if P else 1e-6, P["sink"] if P else None,
                            P["inv_freq"] if P else None, self.q_pos, self.win_len)
            if r == CSA_RATIO:
                cap = L.cache.capacity
                qc, qs, w = iq[li]
                lightning_index(qc, qs, w, L.k_codes, L.k_sf, self.q_pos.view(self.B, 1), CSA_RATIO,
                                scores=self.scores[li], stream=stream)
                topk_select(self.scores[li].view(self.B, cap), self.q_pos, CSA_RATIO, self.k, idx=self.idx[li],
                            count=self.count[li], ws=self.topk_ws[li], stream=stream)
                compressed_attn_decode(q[li], L.cache, self.count[li], min(self.k, cap), L.window, self.scale,
                                       idx=self.idx[li], out=self.out[li], ws=self.ws[li], stream=stream, extras=ex)
            elif r == HCA_RATIO:
                compressed_attn_decode(q[li], L.cache, self.n_ent[r], L.cache.capacity, L.window, self.scale,
                                       out=self.out[li], ws=self.ws[li], stream=stream, extras=ex)
            else:
                compressed_attn_decode(q[li], self._empty, self.n_ent[0], 0, L.window, self.scale,
                                       out=self.out[li], ws=self.ws[li], stream=stream, extras=ex)
        return self.out


def r_is_csa(ratio: int) -> bool:
    return ratio == CSA_RATIO
