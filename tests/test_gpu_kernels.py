"""GPU parity of each C-ABI call against the CPU oracle on small shapes that
still span several tiles, ragged tails and the degenerate cases.

Bit-exact: FP8 codes, fp32 scales, bf16 RoPE dims, index scores (incl. -inf),
top-k index sets and counts.  Attention outputs: max-abs 1e-2 and mean-rel
1e-3 against the oracle's fp64 result rounded to bf16.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_attn_close, cache_host, host

pytestmark = pytest.mark.gpu

hca = pytest.importorskip("long_context_attention_hca_b200")

DEV = "cuda"


def _gen(seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return g


def _bf16(shape, seed, std=1.0):
    return (torch.randn(shape, generator=_gen(seed), device=DEV) * std).to(torch.bfloat16)


# ------------------------------------------------------------------ compress
@pytest.mark.parametrize("layout", [(128, 32, 32), (512, 64, 64)])
@pytest.mark.parametrize("m", [4, 128])
def test_compress_bit_exact(layout, m):
    d, dr, g = layout
    B = 3
    n_blocks = 37 if m == 4 else 5                       # ragged against 4 / 16 entries per CTA
    T = n_blocks * m + 7
    x = _bf16((B, T, d), 1 + m)
    gate = _bf16((B, T, d), 2 + m)
    bias = torch.randn((m, d), generator=_gen(3 + m), device=DEV) * 0.5
    # edge cases: an all-zero scale group, negative zeros, saturating gates
    x[0, :m, :g] = 0.0
    x[1, :m, g:2 * g] = -0.0
    gate[2, 0, :] = 80.0
    gate[2, m:2 * m, :] = -80.0
    bias[0, :8] = 40.0
    entry_begin, cap = 5, 5 + n_blocks + 3
    cache = hca.KVCache(B, cap, layout, zero=True)
    fn = hca.csa_compress if m == 4 else hca.hca_compress
    fn(x, gate, bias, n_blocks, cache, entry_begin=entry_begin)
    torch.cuda.synchronize()
    codes, scales, rope, worst = oracle.compress(host(x), host(gate), host(bias), m, n_blocks, dr, g, cap=cap,
                                                 entry_begin=entry_begin)
    gc, gs, gr = cache_host(cache)
    assert np.array_equal(gc, codes)
    assert np.array_equal(gs.view(np.uint32), scales.view(np.uint32))
    assert np.array_equal(gr, rope)
    # fp64 cross-check of the fp32 sequence: z = gate + bias is rounded at the
    # scale of |z| (ulp 2^-17 at the |z| ~ 80 planted above)
    assert worst < 4 * 2.0 ** -17


def test_compress_rejects_bad_arguments():
    d, dr, g = 512, 64, 64
    x = _bf16((1, 8, d), 0)
    cache = hca.KVCache(1, 2, (d, dr, g))
    bias = torch.zeros((4, d), device=DEV)
    with pytest.raises(hca.HCAError):
        hca.csa_compress(x, x, bias, 3, cache)           # 3 blocks need 12 tokens, only 8
    with pytest.raises(hca.HCAError):
        hca.csa_compress(x, x, bias, 2, cache, entry_begin=1)   # past capacity
    bad = hca.KVCache(1, 2, (d, dr, g))
    bad.layout = (256, 64, 64)
    with pytest.raises(hca.HCAError):
        hca.csa_compress(x, x, bias, 2, bad)


# ------------------------------------------------------------------ indexer
def _fp4_inputs(B, Tq, Hi, c, Nc, seed):
    g = _gen(seed)
    qc = torch.randint(0, 256, (B, Tq, Hi, c // 2), generator=g, device=DEV, dtype=torch.uint8)
    qs = torch.randint(123, 128, (B, Tq, Hi, c // 32), generator=g, device=DEV, dtype=torch.uint8)
    w = torch.rand((B, Tq, Hi), generator=g, device=DEV)
    kc = torch.randint(0, 256, (B, Nc, c // 2), generator=g, device=DEV, dtype=torch.uint8)
    ks = torch.randint(123, 128, (B, Nc, c // 32), generator=g, device=DEV, dtype=torch.uint8)
    return qc, qs, w, kc, ks


@pytest.mark.parametrize("c,Hi,Nc", [(64, 4, 37), (128, 4, 1000), (128, 1, 5003), (64, 8, 4097), (128, 4, 1)])
def test_indexer_bit_exact(c, Hi, Nc):
    B, Tq, m = 2, 5, 4
    qc, qs, w, kc, ks = _fp4_inputs(B, Tq, Hi, c, Nc, c * 7 + Hi + Nc)
    pos = torch.tensor([[0, 2, 3, 4 * Nc - 2, 4 * Nc + 50], [4 * (Nc // 2) - 1, 4 * (Nc // 2), 7, 11, 1 << 30]],
                       dtype=torch.int32, device=DEV)
    s = hca.lightning_index(qc, qs, w, kc, ks, pos, m)
    torch.cuda.synchronize()
    want, n_inexact = oracle.index_scores(host(qc), host(qs), host(w), host(kc), host(ks), host(pos), m)
    assert n_inexact == 0
    assert np.array_equal(host(s).view(np.uint32), want.view(np.uint32))


def test_indexer_full_scale_range_ordered_sum():
    """Scale bytes far outside 2^-4..2^0: the dot is then the fp32 block-ordered
    sum, which the oracle and the kernel must reproduce bit for bit."""
    B, Tq, Hi, c, Nc, m = 1, 3, 4, 128, 300, 1
    qc, qs, w, kc, ks = _fp4_inputs(B, Tq, Hi, c, Nc, 99)
    g = _gen(100)
    qs = torch.randint(100, 150, qs.shape, generator=g, device=DEV, dtype=torch.uint8)
    ks = torch.randint(100, 150, ks.shape, generator=g, device=DEV, dtype=torch.uint8)
    pos = torch.full((B, Tq), 10 ** 6, dtype=torch.int32, device=DEV)
    s = hca.lightning_index(qc, qs, w, kc, ks, pos, m)
    torch.cuda.synchronize()
    want, _ = oracle.index_scores(host(qc), host(qs), host(w), host(kc), host(ks), host(pos), m)
    assert np.array_equal(host(s).view(np.uint32), want.view(np.uint32))


def _same_scores(got, want):
    """Bit-identical, except that any NaN matches any NaN (payloads differ between CPU and GPU)."""
    g, w_ = got.view(np.uint32), want.view(np.uint32)
    nan_g, nan_w = np.isnan(got), np.isnan(want)
    return np.array_equal(nan_g, nan_w) and np.array_equal(g[~nan_g], w_[~nan_w])


@pytest.mark.parametrize("Tq,Nc", [(3, 512), (3, 511), (64, 512), (64, 509)])
def test_indexer_extreme_exponents(Tq, Nc):
    """ue8m0 bytes at both ends of their range: 2^(uq+uk-254) overflows fp32 (a zero
    block must still give 0, a nonzero one inf) or lies far in the subnormal range
    (the product is rounded once).  Covers the tensor-map path (Nc a multiple of 4),
    the fallback path (Nc not), one query per CTA (Tq = 3) and 16 per CTA (Tq = 64)."""
    B, Hi, c, m = 2, 4, 128, 1
    qc, qs, w, kc, ks = _fp4_inputs(B, Tq, Hi, c, Nc, 7 * Tq + Nc)
    g = _gen(Tq + Nc)
    ends = torch.tensor([0, 1, 2, 3, 60, 127, 200, 250, 253, 254, 255], dtype=torch.uint8, device=DEV)
    qs = ends[torch.randint(0, len(ends), qs.shape, generator=g, device=DEV)]
    ks = ends[torch.randint(0, len(ends), ks.shape, generator=g, device=DEV)]
    # zero whole 32-element blocks of some keys (0 * 2^e must stay 0 when 2^e overflows)
    zero = torch.rand((B, Nc, c // 32), generator=g, device=DEV) < 0.3
    kc = kc.view(B, Nc, c // 32, 16).masked_fill(zero[..., None], 0).view(B, Nc, c // 2).contiguous()
    w[..., 0] = 0.0                                     # 0 * inf = NaN in head 0 where its dot overflows
    pos = torch.full((B, Tq), 10 ** 6, dtype=torch.int32, device=DEV)
    pos[1, 0] = Nc // 2
    s = hca.lightning_index(qc, qs, w, kc, ks, pos, m)
    torch.cuda.synchronize()
    want, _ = oracle.index_scores(host(qc), host(qs), host(w), host(kc), host(ks), host(pos), m)
    got = host(s)
    assert np.isinf(want).any() and np.isnan(want).any()          # the planted cases occur
    assert _same_scores(got, want)


@pytest.mark.parametrize("Tq,Nc", [(64, 1000), (64, 4099), (80, 2048)])
def test_indexer_sixteen_queries_per_cta(Tq, Nc):
    """Prefill-shaped calls (Tq a multiple of 16, >= 64): 16 queries share each key
    tile; causal positions cut the eligible range inside tiles."""
    B, Hi, c, m = 2, 4, 128, 4
    qc, qs, w, kc, ks = _fp4_inputs(B, Tq, Hi, c, Nc, Tq * 31 + Nc)
    base = torch.arange(Tq, dtype=torch.int32, device=DEV) * 37
    pos = torch.stack([base + 4 * Nc - 37 * Tq, base + 5]).to(torch.int32)
    s = hca.lightning_index(qc, qs, w, kc, ks, pos, m)
    torch.cuda.synchronize()
    want, n_inexact = oracle.index_scores(host(qc), host(qs), host(w), host(kc), host(ks), host(pos), m)
    assert n_inexact == 0
    assert np.array_equal(host(s).view(np.uint32), want.view(np.uint32))


# ------------------------------------------------------------------ top-k
@pytest.mark.parametrize("Nc,k", [(1, 1), (100, 7), (5000, 32), (33000, 1024), (70000, 512), (140000, 4096),
                                  (600000, 4096)])
def test_topk_bit_exact(Nc, k):
    R, m = 5, 4
    g = _gen(Nc + k)
    # few distinct values -> many ties; include signed zeros
    vals = torch.tensor([-1.0, -0.0, 0.0, 0.25, 0.5, 1.0, 1.5, 3.0], device=DEV)
    scores = vals[torch.randint(0, 8, (R, Nc), generator=g, device=DEV)]
    scores[1] = torch.randn((Nc,), generator=g, device=DEV)            # all distinct
    scores[2] = 0.0                                                      # all tied
    pos = torch.tensor([4 * Nc + 3, 4 * Nc - 1, 4 * (Nc // 3) + 2, 2, 4 * k - 1], dtype=torch.int32, device=DEV)
    idx, cnt = hca.topk_select(scores, pos, m, k)
    torch.cuda.synchronize()
    wi, wc = oracle.topk(host(scores), host(pos), m, k)
    assert np.array_equal(host(cnt), wc)
    assert np.array_equal(host(idx), wi)


@pytest.mark.parametrize("R,Nc,k", [(4, 262144, 1024), (2, 70001, 777)])
def test_topk_crowded_threshold_bin(R, Nc, k):
    """Scores packed into a narrow range (one top-11-bit histogram bin holds most of
    them), duplicated so that the k-th score is tied: the exact key and the
    lowest-index ties must be found among the candidates."""
    g = _gen(R * Nc + k)
    base = 1.0 + torch.randint(0, 3000, (R, Nc), generator=g, device=DEV).float() * 2.0 ** -13
    pos = torch.full((R,), 4 * Nc - 1, dtype=torch.int32, device=DEV)
    pos[-1] = 4 * (Nc // 2) + 1
    idx, cnt = hca.topk_select(base, pos, 4, k)
    torch.cuda.synchronize()
    wi, wc = oracle.topk(host(base), host(pos), 4, k)
    assert np.array_equal(host(cnt), wc)
    assert np.array_equal(host(idx), wi)


@pytest.mark.parametrize("R,Nc,k", [(320, 12000, 700), (300, 70001, 1024)])
def test_topk_many_rows(R, Nc, k):
    """Many rows (the prefill shape: a cluster of CTAs per row, more rows than
    SMs): random, few-valued, all-tied, crowded and tie-dominated rows, rows
    whose eligible prefix is shorter than k or empty; bit-exact against the
    oracle."""
    g = _gen(R * 7 + Nc + k)
    scores = torch.randn((R, Nc), generator=g, device=DEV)
    vals = torch.tensor([-1.0, -0.0, 0.0, 0.25, 0.5, 1.0, 1.5, 3.0], device=DEV)
    scores[0:10] = vals[torch.randint(0, 8, (10, Nc), generator=g, device=DEV)]
    scores[10] = 0.0
    scores[11] = 1.0 + torch.randint(0, 3000, (Nc,), generator=g, device=DEV).float() * 2.0 ** -13
    scores[12] = 0.5
    scores[12, torch.randperm(Nc, generator=g, device=DEV)[: k // 2]] = 2.0 + torch.rand(k // 2, generator=g, device=DEV)
    scores[13, :] = -0.0
    scores[13, ::3] = 0.0
    pos = torch.full((R,), 4 * Nc - 1, dtype=torch.int32, device=DEV)
    pos[14] = 4 * (k - 1) + 2          # fewer eligible entries than k
    pos[15] = 4 * k - 1                # exactly k eligible
    pos[16] = 2                        # none eligible
    pos[17] = 4 * (Nc // 3) + 1
    idx, cnt = hca.topk_select(scores, pos, 4, k)
    torch.cuda.synchronize()
    wi, wc = oracle.topk(host(scores), host(pos), 4, k)
    assert np.array_equal(host(cnt), wc)
    assert np.array_equal(host(idx), wi)


@pytest.mark.parametrize("Nc,k,zero_w", [(20000, 512, False), (5000, 64, False), (70001, 1024, False),
                                         (20000, 777, True)])
def test_lightning_index_topk_fused(Nc, k, zero_w):
    """The fused decode call (indexer building the top-k histogram) equals the
    oracle's scores and selection; Nc = 5000 takes the cluster top-k, Nc = 70001
    (not a multiple of 4) the separate kernels; zero weights make every score
    0, so the selection is all ties (lowest indices)."""
    B, Hi, c, m = 3, 4, 128, 4
    qc, qs, w, kc, ks = _fp4_inputs(B, 1, Hi, c, Nc, Nc + k)
    if zero_w:
        w.zero_()
    pos = torch.tensor([4 * Nc - 1, 4 * 1234 + 1, 4 * 600], dtype=torch.int32, device=DEV)
    s, idx, cnt = hca.lightning_index_topk(qc, qs, w, kc, ks, pos, m, k)
    torch.cuda.synchronize()
    want, n_inexact = oracle.index_scores(host(qc), host(qs), host(w), host(kc), host(ks), host(pos).reshape(B, 1), m)
    assert n_inexact == 0
    assert np.array_equal(host(s).view(np.uint32), want.view(np.uint32))
    wi, wc = oracle.topk(want.reshape(B, Nc), host(pos), m, k)
    assert np.array_equal(host(cnt), wc)
    assert np.array_equal(host(idx), wi)


def test_topk_from_index_scores_pipeline():
    """Index scores straight into top-k: the sets must match the oracle's."""
    B, Hi, c, Nc, m, k = 3, 4, 128, 20000, 4, 512
    qc, qs, w, kc, ks = _fp4_inputs(B, 1, Hi, c, Nc, 5)
    pos = torch.tensor([[4 * Nc - 1], [4 * 1234 + 1], [4 * 600]], dtype=torch.int32, device=DEV)
    s = hca.lightning_index(qc, qs, w, kc, ks, pos, m)
    idx, cnt = hca.topk_select(s.view(B, Nc), pos.view(B), m, k)
    torch.cuda.synchronize()
    ws, _ = oracle.index_scores(host(qc), host(qs), host(w), host(kc), host(ks), host(pos), m)
    wi, wc = oracle.topk(ws.reshape(B, Nc), host(pos).reshape(B), m, k)
    assert np.array_equal(host(idx), wi) and np.array_equal(host(cnt), wc)


# ------------------------------------------------------------------ attention
def _random_cache(B, cap, layout, seed):
    d, dr, g = layout
    gen = _gen(seed)
    cache = hca.KVCache(B, cap, layout)
    codes = torch.randint(0, 256, cache.codes.shape, generator=gen, device=DEV, dtype=torch.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x38                                  # no NaN encodings
    cache.codes.copy_(codes)
    cache.scales.copy_(torch.rand(cache.scales.shape, generator=gen, device=DEV) * 0.01 + 0.001)
    cache.rope.copy_(torch.randn(cache.rope.shape, generator=gen, device=DEV).to(torch.bfloat16))
    return cache


@pytest.mark.parametrize("layout,H", [((128, 32, 32), 8), ((512, 64, 64), 64), ((128, 32, 32), 64)])
def test_decode_dense_and_sparse(layout, H):
    d, dr, g = layout
    B, cap, W = 4, 3000, 128
    cache = _random_cache(B, cap, layout, 11)
    q = _bf16((B, H, d), 12)
    win = _bf16((B, W, d), 13)
    scale = d ** -0.5
    # dense: ragged counts, one sequence with no compressed key (window only)
    n_comp = torch.tensor([cap, 0, 517, 64], dtype=torch.int32, device=DEV)
    lse = torch.empty((B, H), dtype=torch.float32, device=DEV)
    out = hca.compressed_attn_decode(q, cache, n_comp, cap, win, scale, lse=lse)
    # sparse: sorted random subsets, count < k, -1 padding
    k = 300
    idx = torch.full((B, k), -1, dtype=torch.int32, device=DEV)
    counts = [300, 17, 0, 299]
    gen = _gen(14)
    for b in range(B):
        sel = torch.randperm(cap, generator=gen, device=DEV)[:counts[b]].sort().values
        idx[b, :counts[b]] = sel.to(torch.int32)
    cnt = torch.tensor(counts, dtype=torch.int32, device=DEV)
    out_s = hca.compressed_attn_decode(q, cache, cnt, k, win, scale, idx=idx)
    torch.cuda.synchronize()
    codes, scales, rope = cache_host(cache)
    qh, wh, oh, osh, lh = host(q), host(win), host(out), host(out_s), host(lse)
    for b in range(B):
        ref, rl = oracle.attend(qh[b], codes[b], scales[b], rope[b], np.arange(host(n_comp)[b]), wh[b], scale, g)
        assert_attn_close(oh[b], ref, f"dense b={b}")
        assert np.abs(lh[b] - rl).max() < 1e-3
        refs, _ = oracle.attend(qh[b], codes[b], scales[b], rope[b], host(idx)[b, :counts[b]], wh[b], scale, g)
        assert_attn_close(osh[b], refs, f"sparse b={b}")


def test_decode_no_keys_and_no_window():
    layout = (512, 64, 64)
    cache = _random_cache(2, 64, layout, 21)
    q = _bf16((2, 64, 512), 22)
    win = torch.zeros((2, 0, 512), dtype=torch.bfloat16, device=DEV)
    n_comp = torch.tensor([0, 10], dtype=torch.int32, device=DEV)
    lse = torch.empty((2, 64), dtype=torch.float32, device=DEV)
    out = hca.compressed_attn_decode(q, cache, n_comp, 64, win, 512 ** -0.5, lse=lse)
    torch.cuda.synchronize()
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))
    codes, scales, rope = cache_host(cache)
    ref, _ = oracle.attend(host(q)[1], codes[1], scales[1], rope[1], np.arange(10), np.zeros((0, 512), np.uint16),
                           512 ** -0.5, 64)
    assert_attn_close(host(out)[1], ref)


def test_decode_many_splits_match_single_split():
    """The split-K + log-sum-exp path against the oracle on a long dense list."""
    layout = (512, 64, 64)
    B, cap, W = 2, 20000, 128
    cache = _random_cache(B, cap, layout, 31)
    q = _bf16((B, 64, 512), 32)
    win = _bf16((B, W, 512), 33)
    n_comp = torch.tensor([cap, 12345], dtype=torch.int32, device=DEV)
    out = hca.compressed_attn_decode(q, cache, n_comp, cap, win, 512 ** -0.5)
    torch.cuda.synchronize()
    codes, scales, rope = cache_host(cache)
    for b in range(B):
        ref, _ = oracle.attend(host(q)[b], codes[b], scales[b], rope[b], np.arange(host(n_comp)[b]), host(win)[b],
                               512 ** -0.5, 64)
        assert_attn_close(host(out)[b], ref, f"b={b}")


@pytest.mark.parametrize("budget", [2, 7, 40])
def test_decode_launch_budget(budget):
    """A CTA budget changes the split plan of the dense decode attention, not its
    result (the workspace is sized for the larger of the sparse and dense plans)."""
    layout = (512, 64, 64)
    B, cap, W = 2, 9000, 128
    cache = _random_cache(B, cap, layout, 41)
    q = _bf16((B, 64, 512), 42)
    win = _bf16((B, W, 512), 43)
    n_comp = torch.tensor([cap, 4321], dtype=torch.int32, device=DEV)
    prev = hca.set_launch_budget(hca.BUDGET_DENSE_DECODE, budget)
    try:
        out = hca.compressed_attn_decode(q, cache, n_comp, cap, win, 512 ** -0.5)
        torch.cuda.synchronize()
    finally:
        hca.set_launch_budget(hca.BUDGET_DENSE_DECODE, prev)
    codes, scales, rope = cache_host(cache)
    for b in range(B):
        ref, _ = oracle.attend(host(q)[b], codes[b], scales[b], rope[b], np.arange(host(n_comp)[b]), host(win)[b],
                               512 ** -0.5, 64)
        assert_attn_close(host(out)[b], ref, f"budget={budget} b={b}")


@pytest.mark.parametrize("layout,H,p0", [((512, 64, 64), 64, 1000), ((128, 32, 32), 8, 10)])
def test_prefill_dense_and_sparse(layout, H, p0):
    d, dr, g = layout
    Tq, W, m = 150, 128, 4
    cap = (p0 + Tq) // m
    cache = _random_cache(1, cap, layout, 41)
    q = _bf16((Tq, H, d), 42)
    raw = _bf16((W - 1 + Tq, d), 43)
    scale = d ** -0.5
    out_d = hca.compressed_attn_prefill(q, p0, m, cache, raw, W, scale)
    # sparse: per position a random subset of its eligible entries
    k = 64
    idx = torch.full((Tq, k), -1, dtype=torch.int32, device=DEV)
    cnt = torch.zeros((Tq,), dtype=torch.int32, device=DEV)
    gen = _gen(44)
    for i in range(Tq):
        e = (p0 + i + 1) // m
        n = min(k, e)
        sel = torch.randperm(e, generator=gen, device=DEV)[:n].sort().values if e else torch.zeros(0, device=DEV)
        idx[i, :n] = sel.to(torch.int32)
        cnt[i] = n
    out_s = hca.compressed_attn_prefill(q, p0, m, cache, raw, W, scale, idx=idx, count=cnt)
    torch.cuda.synchronize()
    codes, scales, rope = cache_host(cache.sequence(0))
    codes, scales, rope = codes[0], scales[0], rope[0]
    qh, rh, idh, cth = host(q), host(raw), host(idx), host(cnt)
    for i in list(range(0, Tq, 7)) + [Tq - 1]:
        p = p0 + i
        ent, w0, w1 = oracle.causal_keys(p, m, W, n_cap=cap)
        win = rh[w0 - (p0 - (W - 1)):w1 - (p0 - (W - 1))]
        ref, _ = oracle.attend(qh[i], codes, scales, rope, ent, win, scale, g)
        assert_attn_close(host(out_d)[i], ref, f"dense pos {p}")
        refs, _ = oracle.attend(qh[i], codes, scales, rope, idh[i, :cth[i]], win, scale, g)
        assert_attn_close(host(out_s)[i], refs, f"sparse pos {p}")
