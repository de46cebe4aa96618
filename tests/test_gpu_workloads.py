"""GPU parity on the five synthetic workloads, run through the same runners
(and launch configuration) that bench.py times.

tiny_decode_1k      everything compared in full.
decode_b16_64k,     compressed entries: sampled blocks (raw rows copied to the
decode_b4_1m        host while they exist); index scores, top-k sets and both
                    attention outputs: every sequence in full.
prefill_4096_131k   the chunk's compressed entries in full, prefix entries
                    sampled; index scores / top-k / attention on sampled
                    query positions (first, last, block and tile edges).
stack61_b32_256k    layers 0, 1, 2, 59, 60 and sequences 0 and 31 sampled.
"""
import numpy as np
import pytest
import torch

import hca_inputs as inp
import oracle
from gpu_util import assert_attn_close, cache_host, host

pytestmark = pytest.mark.gpu

hca = pytest.importorskip("long_context_attention_hca_b200")
from hca_workloads import build_decode, build_prefill  # noqa: E402
from long_context_attention_hca_b200.pipeline import DecodeRunner, PrefillRunner  # noqa: E402


class RawSampler:
    """on_raw hook: copies the raw rows of chosen blocks to the host."""

    def __init__(self, picks):
        self.picks = picks            # {layer: [(b, j), ...]}  (block index j of that layer's ratio)
        self.got = {}

    def __call__(self, li, r, x, gate, bias):
        for (b, j) in self.picks.get(li, []):
            self.got[(li, b, j)] = (host(x[b:b + 1, j * r:(j + 1) * r]), host(gate[b:b + 1, j * r:(j + 1) * r]),
                                    host(bias))


def _s9_entry_kw(dw, li):
    """oracle.compress keywords of layer li's section 9 entry extras (none when off)."""
    if dw is None or dw.s9 is None:
        return {}
    P = dw.s9[li]
    return {"norm_w": host(P["kv_norm_w"]), "eps": P["eps"], "inv_freq": host(P["inv_freq"])}


def _s9_attn_kw(dw, li, t):
    if dw is None or dw.s9 is None:
        return {}
    P = dw.s9[li]
    return {"q_norm_w": host(P["q_norm_w"]), "eps": P["eps"], "sink": host(P["sink"]),
            "inv_freq": host(P["inv_freq"]), "q_pos": t}


def check_sampled_entries(wl, layers, sampler, dw=None):
    for (li, b, j), (xr, gr, br) in sampler.got.items():
        L = layers[li]
        c, s, r, _ = oracle.compress(xr, gr, br, L.ratio, 1, wl.d_rope, wl.g, pos_entry0=j, **_s9_entry_kw(dw, li))
        gc, gs, grp = host(L.cache.codes[b, j]), host(L.cache.scales[b, j]), host(L.cache.rope[b, j])
        assert np.array_equal(gc, c[0, 0]), (li, b, j)
        assert np.array_equal(gs.view(np.uint32), s[0, 0].view(np.uint32)), (li, b, j)
        assert np.array_equal(grp, r[0, 0]), (li, b, j)


def check_decode_layer(wl, dw, runner, li, seqs):
    L = dw.layers[li]
    qh = host(dw.q[li])
    out = host(runner.out[li])
    win = host(L.window)
    if dw.s9 is not None:
        # the prepared window against the oracle's preparation of the raw one
        P = dw.s9[li]
        raw = host(dw.raw_window[li])
        pos = np.arange(wl.t + 1 - wl.W, wl.t + 1, dtype=np.int64)
        for b in seqs:
            want = oracle.token_prep(raw[b], pos, wl.d_rope, norm_w=host(P["kv_norm_w"]), eps=P["eps"],
                                     inv_freq=host(P["inv_freq"]))
            assert np.array_equal(win[b], want), f"prepared window layer {li} b {b}"
    codes, scales, rope = cache_host(L.cache)
    if L.ratio == 4:
        qc, qs, w = (host(t) for t in dw.iq[li])
        kc, ks = host(L.k_codes), host(L.k_sf)
        gpu_scores = host(runner.scores[li])
        gpu_idx, gpu_cnt = host(runner.idx[li]), host(runner.count[li])
    for b in seqs:
        if L.ratio == 4:
            pos = np.array([[wl.t]], np.int32)
            s, n_inexact = oracle.index_scores(qc[b:b + 1], qs[b:b + 1], w[b:b + 1], kc[b:b + 1], ks[b:b + 1], pos, 4)
            assert n_inexact == 0
            assert np.array_equal(gpu_scores[b, 0].view(np.uint32), s[0, 0].view(np.uint32)), f"scores layer {li} b {b}"
            idx, cnt = oracle.topk(s[0], pos[0], 4, wl.k)
            assert gpu_cnt[b] == cnt[0] and np.array_equal(gpu_idx[b], idx[0]), f"top-k layer {li} b {b}"
            ent = idx[0, :cnt[0]]
        else:
            ent = np.arange(L.n_entries)
        ref, _ = oracle.attend(qh[b], codes[b], scales[b], rope[b], ent, win[b], wl.softmax_scale, wl.g,
                               **_s9_attn_kw(dw, li, wl.t))
        assert_attn_close(out[b], ref, f"layer {li} (ratio {L.ratio}) seq {b}")


def _decode_case(name, n_samples, seqs=None, layers=None, section9=False):
    wl = inp.WORKLOADS[name]
    rng = np.random.default_rng(wl.seed)
    ratios = [4, 128] if wl.layers == 1 else [128 if (i < 2 or i % 2) else 4 for i in range(wl.layers)]
    check_layers = list(range(len(ratios))) if layers is None else layers
    picks = {}
    T = wl.t + 1
    for li in check_layers:
        nb = T // ratios[li]
        js = [0, nb - 1] + list(rng.integers(0, nb, n_samples))
        picks[li] = [(int(rng.integers(0, wl.B)), int(j)) for j in js]
    sampler = RawSampler(picks)
    dw = build_decode(wl, on_raw=sampler, section9=section9)
    runner = DecodeRunner(dw.layers, wl.B, wl.H, wl.k, wl.t, wl.softmax_scale, extras=dw.extras)
    runner.step(dw.q, dw.iq)
    torch.cuda.synchronize()
    check_sampled_entries(wl, dw.layers, sampler, dw)
    for li in check_layers:
        check_decode_layer(wl, dw, runner, li, range(wl.B) if seqs is None else seqs)
    del dw, runner
    torch.cuda.empty_cache()


@pytest.mark.parametrize("section9", [False, True])
def test_tiny_decode_1k_full(section9):
    wl = inp.WORKLOADS["tiny_decode_1k"]
    raw = {}
    dw = build_decode(wl, on_raw=lambda li, r, x, g, b: raw.setdefault(li, (host(x), host(g), host(b))),
                      section9=section9)
    runner = DecodeRunner(dw.layers, wl.B, wl.H, wl.k, wl.t, wl.softmax_scale, extras=dw.extras)
    runner.step(dw.q, dw.iq)
    torch.cuda.synchronize()
    for li, L in enumerate(dw.layers):
        x, g, b = raw[li]
        c, s, r, _ = oracle.compress(x, g, b, L.ratio, L.n_entries, wl.d_rope, wl.g, **_s9_entry_kw(dw, li))
        gc, gs, gr = cache_host(L.cache)
        assert np.array_equal(gc, c) and np.array_equal(gs.view(np.uint32), s.view(np.uint32)) and np.array_equal(gr, r)
        check_decode_layer(wl, dw, runner, li, range(wl.B))


def test_step_host_matches_device_step():
    """DecodeRunner.step_host (pinned host in and out, copies overlapped with the
    kernels, captured in a CUDA graph) returns exactly what step() computes."""
    wl = inp.WORKLOADS["decode_b16_64k"]
    dw = build_decode(wl)
    runner = DecodeRunner(dw.layers, wl.B, wl.H, wl.k, wl.t, wl.softmax_scale)
    ref = [o.clone() for o in runner.step(dw.q, dw.iq)]
    torch.cuda.synchronize()
    h_q = [t.to("cpu").pin_memory() for t in dw.q]
    h_iq = [None if t is None else tuple(x.to("cpu").pin_memory() for x in t) for t in dw.iq]
    h_out = [torch.zeros_like(o, device="cpu").pin_memory() for o in runner.out]
    d_q = [torch.zeros_like(t) for t in dw.q]
    d_iq = [None if t is None else tuple(torch.zeros_like(x) for x in t) for t in dw.iq]
    for o in runner.out:
        o.zero_()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        runner.step_host(h_q, h_iq, h_out, d_q, d_iq)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    for a, b in zip(h_out, ref):
        assert torch.equal(a.view(torch.int16), b.cpu().view(torch.int16))
    # the same step captured in a graph and replayed
    for h in h_out:
        h.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        runner.step_host(h_q, h_iq, h_out, d_q, d_iq)
    g.replay()
    torch.cuda.synchronize()
    for a, b in zip(h_out, ref):
        assert torch.equal(a.view(torch.int16), b.cpu().view(torch.int16))


@pytest.mark.parametrize("section9", [False, True])
def test_decode_b16_64k(section9):
    _decode_case("decode_b16_64k", n_samples=40, section9=section9)


@pytest.mark.parametrize("section9", [False, True])
def test_decode_b4_1m(section9):
    _decode_case("decode_b4_1m", n_samples=40, section9=section9)


@pytest.mark.parametrize("section9", [False, True])
def test_stack61_b32_256k_sampled(section9):
    _decode_case("stack61_b32_256k", n_samples=6, seqs=[0, 31], layers=[0, 1, 2, 59, 60], section9=section9)


@pytest.mark.parametrize("section9", [False, True])
def test_prefill_4096_131k_sampled(section9):
    wl = inp.WORKLOADS["prefill_4096_131k"]
    pw = build_prefill(wl, keep_raw=True, section9=section9)
    st = pw.state
    P = pw.s9
    ex = hca.AttnExtras(P["q_norm_w"], P["eps"], P["sink"], P["inv_freq"]) if section9 else None
    ekw = {"norm_w": host(P["kv_norm_w"]), "eps": P["eps"], "inv_freq": host(P["inv_freq"])} if section9 else {}
    runner = PrefillRunner(st, wl.t, wl.Tq, wl.H, wl.k, wl.W, wl.softmax_scale, extras=ex)
    runner.step(pw.raw_chunk, pw.gate_chunk, pw.raw_window, pw.q, pw.iq)
    torch.cuda.synchronize()
    p0, Tq = wl.t, wl.Tq
    # chunk entries in full, a sample of the cached prefix
    xc, gc = host(pw.raw_chunk), host(pw.gate_chunk)
    for cache, m, bias in ((st.csa, 4, st.bias4), (st.hca, 128, st.bias128)):
        c, s, r, _ = oracle.compress(xc, gc, host(bias), m, Tq // m, wl.d_rope, wl.g, pos_entry0=p0 // m, **ekw)
        e0 = p0 // m
        assert np.array_equal(host(cache.codes[0, e0:]), c[0])
        assert np.array_equal(host(cache.scales[0, e0:]).view(np.uint32), s[0].view(np.uint32))
        assert np.array_equal(host(cache.rope[0, e0:]), r[0])
        for j in (0, 1, e0 // 2, e0 - 1):
            xr, gr = host(pw.x_all[:, j * m:(j + 1) * m]), host(pw.gate_all[:, j * m:(j + 1) * m])
            c1, s1, r1, _ = oracle.compress(xr, gr, host(bias), m, 1, wl.d_rope, wl.g, pos_entry0=j, **ekw)
            assert np.array_equal(host(cache.codes[0, j]), c1[0, 0])
            assert np.array_equal(host(cache.scales[0, j]).view(np.uint32), s1[0, 0].view(np.uint32))
    # sampled query positions
    rows = [0, 1, 2, 3, 4, 127, 128, 511, 2047, 2048, 4094, 4095]
    qc, qs, w = (host(t) for t in pw.iq)
    kc, ks = host(st.k_codes), host(st.k_sf)
    codes4, scales4, rope4 = (a[0] for a in cache_host(st.csa))
    codes128, scales128, rope128 = (a[0] for a in cache_host(st.hca))
    gs, gi, gcnt = host(runner.scores), host(runner.idx), host(runner.count)
    qh, rawh = host(pw.q), host(pw.raw_window)
    if section9:
        pos = np.arange(p0 - (wl.W - 1), p0 + Tq, dtype=np.int64)
        want = oracle.token_prep(host(pw.raw_window_unprepared), pos, wl.d_rope, **ekw)
        assert np.array_equal(rawh, want), "prepared window"
    akw = (lambda p: {"q_norm_w": host(P["q_norm_w"]), "eps": P["eps"], "sink": host(P["sink"]),
                      "inv_freq": host(P["inv_freq"]), "q_pos": p}) if section9 else (lambda p: {})
    oc, oh = host(runner.out_csa), host(runner.out_hca)
    for i in rows:
        p = p0 + i
        pos = np.array([[p]], np.int32)
        s, n_inexact = oracle.index_scores(qc[:, i:i + 1], qs[:, i:i + 1], w[:, i:i + 1], kc, ks, pos, 4)
        assert n_inexact == 0
        assert np.array_equal(gs[0, i].view(np.uint32), s[0, 0].view(np.uint32)), f"scores row {i}"
        idx, cnt = oracle.topk(s[0], pos[0], 4, wl.k)
        assert gcnt[i] == cnt[0] and np.array_equal(gi[i], idx[0]), f"top-k row {i}"
        ent128, w0, w1 = oracle.causal_keys(p, 128, wl.W)
        win = rawh[w0 - (p0 - (wl.W - 1)):w1 - (p0 - (wl.W - 1))]
        ref, _ = oracle.attend(qh[i], codes4, scales4, rope4, idx[0, :cnt[0]], win, wl.softmax_scale, wl.g,
                               **akw(p))
        assert_attn_close(oc[i], ref, f"CSA pos {p}")
        ref, _ = oracle.attend(qh[i], codes128, scales128, rope128, ent128, win, wl.softmax_scale, wl.g, **akw(p))
        assert_attn_close(oh[i], ref, f"HCA pos {p}")


def test_decode_b4_1m_and_prefill_run_twice_identical():
    """Determinism (no floating-point atomics, the same reduction order on
    every run): the 1M-context decode step and the prefill chunk give the
    same bytes when run again (outputs, index scores, top-k sets)."""
    wl = inp.WORKLOADS["decode_b4_1m"]
    dw = build_decode(wl)
    runner = DecodeRunner(dw.layers, wl.B, wl.H, wl.k, wl.t, wl.softmax_scale)
    first = [o.clone() for o in runner.step(dw.q, dw.iq)]
    sc1 = {li: t.clone() for li, t in runner.scores.items()}
    idx1 = {li: t.clone() for li, t in runner.idx.items()}
    second = runner.step(dw.q, dw.iq)
    torch.cuda.synchronize()
    for a, b in zip(first, second):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    for li in sc1:
        assert torch.equal(sc1[li].view(torch.int32), runner.scores[li].view(torch.int32))
        assert torch.equal(idx1[li], runner.idx[li])
    del dw, runner
    torch.cuda.empty_cache()
    wl = inp.WORKLOADS["prefill_4096_131k"]
    pw = build_prefill(wl)
    pr = PrefillRunner(pw.state, wl.t, wl.Tq, wl.H, wl.k, wl.W, wl.softmax_scale)
    a = [t.clone() for t in pr.step(pw.raw_chunk, pw.gate_chunk, pw.raw_window, pw.q, pw.iq)]
    b = pr.step(pw.raw_chunk, pw.gate_chunk, pw.raw_window, pw.q, pw.iq)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))
