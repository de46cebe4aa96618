"""GPU parity of the section 9 extras ("DeepSeek V4 ..." reading note,
section 9: query and KV-entry RMSNorm, partial RoPE on the query, the entry
and the output, and the per-head attention sink) against the CPU oracle.

Bit-exact: compressed entries stored with RMSNorm and RoPE (FP8 codes, fp32
scales, bf16 RoPE dims) and prepared window tokens.  Attention outputs with
the extras: max-abs 1e-2 and mean-rel 1e-3 against the oracle's fp64 result
rounded to bf16.  With every extra off, the _ex calls give the plain calls'
outputs bit for bit.
"""
import numpy as np
import pytest
import torch

import hca_inputs as inp
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


def _params(d, dr, H, seed):
    g = _gen(seed)
    return {"kv_norm_w": 1.0 + 0.1 * torch.randn((d,), generator=g, device=DEV),
            "q_norm_w": 1.0 + 0.1 * torch.randn((d,), generator=g, device=DEV),
            "sink": torch.randn((H,), generator=g, device=DEV),
            "inv_freq": inp.rope_inv_freq(dr, device=DEV), "eps": 1e-6}


@pytest.mark.parametrize("layout", [(128, 32, 32), (512, 64, 64)])
@pytest.mark.parametrize("m", [4, 128])
@pytest.mark.parametrize("mode", ["norm", "rope", "both"])
def test_compress_ex_bit_exact(layout, m, mode):
    d, dr, g = layout
    B, n_blocks = 3, (29 if m == 4 else 3)
    T = n_blocks * m
    x = _bf16((B, T, d), 101 + m)
    gate = _bf16((B, T, d), 102 + m)
    bias = torch.randn((m, d), generator=_gen(103), device=DEV) * 0.5
    x[0, :m] = 0.0                                   # an all-zero entry: RMSNorm of zeros (eps keeps it finite)
    P = _params(d, dr, 8, 104)
    nw = P["kv_norm_w"] if mode in ("norm", "both") else None
    fq = P["inv_freq"] if mode in ("rope", "both") else None
    entry_begin = 1000 if m == 4 else 8000           # large positions for RoPE
    cap = entry_begin + n_blocks
    cache = hca.KVCache(B, cap, layout, zero=True)
    fn = hca.csa_compress if m == 4 else hca.hca_compress
    fn(x, gate, bias, n_blocks, cache, entry_begin=entry_begin, extras=hca.EntryExtras(nw, P["eps"], fq))
    torch.cuda.synchronize()
    c, s, r, _ = oracle.compress(host(x), host(gate), host(bias), m, n_blocks, dr, g, cap=n_blocks,
                                 norm_w=None if nw is None else host(nw), eps=P["eps"],
                                 inv_freq=None if fq is None else host(fq), pos_entry0=entry_begin)
    gc, gs, gr = (a[:, entry_begin:] for a in cache_host(cache))
    assert np.array_equal(gc, c)
    assert np.array_equal(gs.view(np.uint32), s.view(np.uint32))
    assert np.array_equal(gr, r)


@pytest.mark.parametrize("layout", [(128, 32, 32), (512, 64, 64)])
def test_token_prep_bit_exact(layout):
    d, dr, g = layout
    n = 301
    x = _bf16((n, d), 111)
    pos = torch.cat([torch.arange(0, 200, device=DEV), torch.randint(0, 1 << 20, (101,), generator=_gen(112),
                                                                      device=DEV)]).to(torch.int32)
    P = _params(d, dr, 8, 113)
    for nw, fq in ((P["kv_norm_w"], None), (None, P["inv_freq"]), (P["kv_norm_w"], P["inv_freq"])):
        out = hca.kv_token_prep(x, pos, layout, hca.EntryExtras(nw, P["eps"], fq))
        torch.cuda.synchronize()
        want = oracle.token_prep(host(x), host(pos).astype(np.int64), dr, norm_w=None if nw is None else host(nw),
                                 eps=P["eps"], inv_freq=None if fq is None else host(fq))
        assert np.array_equal(host(out), want)


def _random_cache(B, cap, layout, seed):
    gen = _gen(seed)
    cache = hca.KVCache(B, cap, layout)
    codes = torch.randint(0, 256, cache.codes.shape, generator=gen, device=DEV, dtype=torch.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x38
    cache.codes.copy_(codes)
    cache.scales.copy_(torch.rand(cache.scales.shape, generator=gen, device=DEV) * 0.01 + 0.001)
    cache.rope.copy_(torch.randn(cache.rope.shape, generator=gen, device=DEV).to(torch.bfloat16))
    return cache


EXTRA_SETS = [("norm",), ("sink",), ("rope",), ("norm", "sink", "rope")]


def _extras(P, which, q_pos):
    return hca.AttnExtras(P["q_norm_w"] if "norm" in which else None, P["eps"],
                          P["sink"] if "sink" in which else None,
                          P["inv_freq"] if "rope" in which else None, q_pos)


def _oracle_kw(P, which, t):
    return {"q_norm_w": host(P["q_norm_w"]) if "norm" in which else None, "eps": P["eps"],
            "sink": host(P["sink"]) if "sink" in which else None,
            "inv_freq": host(P["inv_freq"]) if "rope" in which else None, "q_pos": t}


@pytest.mark.parametrize("layout,H", [((128, 32, 32), 8), ((512, 64, 64), 64)])
@pytest.mark.parametrize("which", EXTRA_SETS)
def test_decode_extras(layout, H, which):
    d, dr, g = layout
    B, cap, W = 3, 2500, 128
    cache = _random_cache(B, cap, layout, 121)
    q = _bf16((B, H, d), 122)
    win = _bf16((B, W, d), 123)
    scale = d ** -0.5
    P = _params(d, dr, H, 124)
    qpos = torch.tensor([1048575, 77, 262143], dtype=torch.int32, device=DEV)
    ex = _extras(P, which, qpos)
    # dense over ragged counts (many splits), then a short sparse list (one split on the CSA plan)
    n_comp = torch.tensor([cap, 0, 700], dtype=torch.int32, device=DEV)
    lse = torch.empty((B, H), dtype=torch.float32, device=DEV)
    out = hca.compressed_attn_decode(q, cache, n_comp, cap, win, scale, lse=lse, extras=ex)
    k = 40
    idx = torch.stack([torch.randperm(cap, generator=_gen(125 + b), device=DEV)[:k].sort().values
                       for b in range(B)]).to(torch.int32)
    cnt = torch.tensor([40, 3, 0], dtype=torch.int32, device=DEV)
    out_s = hca.compressed_attn_decode(q, cache, cnt, k, win, scale, idx=idx, extras=ex)
    torch.cuda.synchronize()
    codes, scales, rope = cache_host(cache)
    qh, wh, lh = host(q), host(win), host(lse)
    for b in range(B):
        kw = _oracle_kw(P, which, int(host(qpos)[b]))
        ref, rl = oracle.attend(qh[b], codes[b], scales[b], rope[b], np.arange(host(n_comp)[b]), wh[b], scale, g, **kw)
        assert_attn_close(host(out)[b], ref, f"dense b={b} {which}")
        assert np.abs(lh[b] - rl).max() < 1e-3
        refs, _ = oracle.attend(qh[b], codes[b], scales[b], rope[b], host(idx)[b, :host(cnt)[b]], wh[b], scale, g,
                                **kw)
        assert_attn_close(host(out_s)[b], refs, f"sparse b={b} {which}")


@pytest.mark.parametrize("which", [(), ("norm", "sink", "rope")])
def test_early_query_is_bit_identical(which):
    """A sparse decode attention that loads its query before waiting on the top-k
    launched just before it (set_early_query) gives the same bits as one that
    loads it after the wait.  The top-k on long rows keeps the previous kernel
    running while the attention's CTAs are placed."""
    layout, H = (512, 64, 64), 64
    d, dr, g = layout
    B, cap, W, k = 3, 70001, 128, 1024
    cache = _random_cache(B, cap, layout, 141)
    q = _bf16((B, H, d), 142)
    win = _bf16((B, W, d), 143)
    P = _params(d, dr, H, 144)
    qpos = torch.tensor([4 * cap - 1, 4 * 2000 + 1, 4 * 600 + 3], dtype=torch.int32, device=DEV)
    ex = _extras(P, which, qpos) if which else None
    scores = torch.randn((B, cap), generator=_gen(145), device=DEV)
    outs = []
    for early in (False, True):
        prev = hca.set_early_query(early)
        try:
            idx, cnt = hca.topk_select(scores, qpos, 4, k)
            outs.append(hca.compressed_attn_decode(q, cache, cnt, k, win, d ** -0.5, idx=idx, extras=ex))
        finally:
            hca.set_early_query(prev)
    torch.cuda.synchronize()
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    assert torch.isfinite(outs[1].float()).all()


@pytest.mark.parametrize("layout,H", [((128, 32, 32), 8), ((512, 64, 64), 64)])
def test_extras_off_is_the_plain_call(layout, H):
    d, dr, g = layout
    B, cap, W = 2, 1500, 128
    cache = _random_cache(B, cap, layout, 131)
    q = _bf16((B, H, d), 132)
    win = _bf16((B, W, d), 133)
    n_comp = torch.tensor([cap, 333], dtype=torch.int32, device=DEV)
    a = hca.compressed_attn_decode(q, cache, n_comp, cap, win, d ** -0.5)
    b = hca.compressed_attn_decode(q, cache, n_comp, cap, win, d ** -0.5, extras=hca.AttnExtras())
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("layout,H,p0", [((512, 64, 64), 64, 1000), ((128, 32, 32), 8, 10)])
def test_prefill_extras(layout, H, p0):
    d, dr, g = layout
    Tq, W, m = 130, 128, 4
    cap = (p0 + Tq) // m
    cache = _random_cache(1, cap, layout, 141)
    q = _bf16((Tq, H, d), 142)
    raw = _bf16((W - 1 + Tq, d), 143)
    scale = d ** -0.5
    P = _params(d, dr, H, 144)
    which = ("norm", "sink", "rope")
    ex = _extras(P, which, None)
    out_d = hca.compressed_attn_prefill(q, p0, m, cache, raw, W, scale, extras=ex)
    k = 48
    idx = torch.full((Tq, k), -1, dtype=torch.int32, device=DEV)
    cnt = torch.zeros((Tq,), dtype=torch.int32, device=DEV)
    gen = _gen(145)
    for i in range(Tq):
        e = (p0 + i + 1) // m
        n = min(k, e)
        if n:
            idx[i, :n] = torch.randperm(e, generator=gen, device=DEV)[:n].sort().values.to(torch.int32)
        cnt[i] = n
    out_s = hca.compressed_attn_prefill(q, p0, m, cache, raw, W, scale, idx=idx, count=cnt, extras=ex)
    torch.cuda.synchronize()
    codes, scales, rope = (a[0] for a in cache_host(cache))
    qh, rh, idh, cth = host(q), host(raw), host(idx), host(cnt)
    for i in list(range(0, Tq, 9)) + [Tq - 1]:
        p = p0 + i
        ent, w0, w1 = oracle.causal_keys(p, m, W, n_cap=cap)
        win = rh[w0 - (p0 - (W - 1)):w1 - (p0 - (W - 1))]
        kw = _oracle_kw(P, which, p)
        ref, _ = oracle.attend(qh[i], codes, scales, rope, ent, win, scale, g, **kw)
        assert_attn_close(host(out_d)[i], ref, f"dense pos {p}")
        refs, _ = oracle.attend(qh[i], codes, scales, rope, idh[i, :cth[i]], win, scale, g, **kw)
        assert_attn_close(host(out_s)[i], refs, f"sparse pos {p}")


def test_ex_calls_reject_bad_extras():
    layout = (512, 64, 64)
    cache = _random_cache(1, 64, layout, 151)
    q = _bf16((1, 64, 512), 152)
    win = _bf16((1, 128, 512), 153)
    n = torch.tensor([64], dtype=torch.int32, device=DEV)
    f = inp.rope_inv_freq(64, device=DEV)
    with pytest.raises(hca.HCAError):                      # RoPE in decode needs the query positions
        hca.compressed_attn_decode(q, cache, n, 64, win, 0.04, extras=hca.AttnExtras(inv_freq=f))
    with pytest.raises(hca.HCAError):                      # negative epsilon
        hca.compressed_attn_decode(q, cache, n, 64, win, 0.04,
                                   extras=hca.AttnExtras(q_norm_w=torch.ones(512, device=DEV), eps=-1.0))
