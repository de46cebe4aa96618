"""The state-cache decode loop ("DeepSeek V4 ..." note, section 11 KV cache
table: compressed entries in the classical cache, the recent window and the
uncompressed tail of the incomplete block in a per-sequence state cache;
section 8 compress_ratio table: ratio 0 disables the compressed branch)
against the oracle at every step.

Three layers (ratio 0: window only; 4: CSA; 128: HCA), d = 128, H = 8, a
4 x 64 FP4 indexer, k = 32, W = 128, two sequences.  Every step appends one
token, pools a block when its last token arrives (the new entry is compared
bit for bit with the oracle's pooling of the same raw tokens), and runs the
three attention calls; index scores and top-k sets are compared bit for bit
and the outputs within the attention tolerance.  One run crosses 300 tokens
from position 1000 (CSA blocks every 4 tokens, HCA blocks at 1023, 1151,
1279); one starts from an empty state at position 0 (the window fills up,
the first blocks complete) with the section 9 extras on.
"""
import numpy as np
import pytest
import torch

import hca_inputs as inp
import oracle
from gpu_util import assert_attn_close, host

pytestmark = pytest.mark.gpu

hca = pytest.importorskip("long_context_attention_hca_b200")
from long_context_attention_hca_b200.pipeline import DecodeLoop  # noqa: E402

DEV = "cuda"
D, DR, G, H, HI, C, K, W, B = 128, 32, 32, 8, 4, 64, 32, 128, 2
RATIOS = [0, 4, 128]


def _gen(seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return g


def _run_loop(t0, t_end, section9, seed):
    scale = D ** -0.5
    g = _gen(seed)
    x = [(torch.randn((B, t_end, D), generator=g, device=DEV)).to(torch.bfloat16) for _ in RATIOS]
    gate = [(torch.randn((B, t_end, D), generator=g, device=DEV)).to(torch.bfloat16) for _ in RATIOS]
    bias = [None if r == 0 else torch.randn((r, D), generator=g, device=DEV) * 0.5 for r in RATIOS]
    ncap = t_end // 4
    kc = torch.randint(0, 256, (B, ncap, C // 2), generator=g, device=DEV, dtype=torch.uint8)
    ks = torch.randint(123, 128, (B, ncap, C // 32), generator=g, device=DEV, dtype=torch.uint8)
    s9 = None
    if section9:
        s9 = [{"kv_norm_w": 1.0 + 0.1 * torch.randn((D,), generator=g, device=DEV),
               "q_norm_w": 1.0 + 0.1 * torch.randn((D,), generator=g, device=DEV),
               "sink": torch.randn((H,), generator=g, device=DEV),
               "inv_freq": inp.rope_inv_freq(DR, device=DEV), "eps": 1e-6} for _ in RATIOS]
    loop = DecodeLoop(B, H, (D, DR, G), RATIOS, W, K, t_end, scale, Hi=HI, c=C, s9=s9)
    loop.set_indexer_keys(1, kc, ks)
    for li in range(len(RATIOS)):
        loop.load_prefix(li, x[li], gate[li], bias[li], t0)
    # the oracle's entries of every block, pooled from the same raw tokens
    ref_ent = {}
    for li, r in enumerate(RATIOS):
        if r:
            kw = {} if s9 is None else {"norm_w": host(s9[li]["kv_norm_w"]), "eps": 1e-6,
                                        "inv_freq": host(s9[li]["inv_freq"])}
            ref_ent[li] = oracle.compress(host(x[li]), host(gate[li]), host(bias[li]), r, t_end // r, DR, G, **kw)[:3]
    xh = [host(t) for t in x]
    kch, ksh = host(kc), host(ks)
    n_checked = 0
    for t in range(t0, t_end):
        q = [(torch.randn((B, H, D), generator=g, device=DEV)).to(torch.bfloat16) for _ in RATIOS]
        qc = torch.randint(0, 256, (B, 1, HI, C // 2), generator=g, device=DEV, dtype=torch.uint8)
        qs = torch.randint(123, 128, (B, 1, HI, C // 32), generator=g, device=DEV, dtype=torch.uint8)
        w = torch.rand((B, 1, HI), generator=g, device=DEV)
        iq = [None, (qc, qs, w), None]
        out = loop.step(t, [xt[:, t].contiguous() for xt in x], [gt[:, t].contiguous() for gt in gate], q, iq)
        torch.cuda.synchronize()
        qh = [host(a) for a in q]
        for li, r in enumerate(RATIOS):
            L = loop.layers[li]
            if r and (t + 1) % r == 0:                  # the entry made at this step
                e = (t + 1) // r - 1
                c_, s_, r_ = ref_ent[li]
                assert np.array_equal(host(L.cache.codes[:, e]), c_[:, e]), (t, li)
                assert np.array_equal(host(L.cache.scales[:, e]).view(np.uint32), s_[:, e].view(np.uint32)), (t, li)
                assert np.array_equal(host(L.cache.rope[:, e]), r_[:, e]), (t, li)
            # window: the raw tokens max(0, t-W+1) .. t (prepared with the section 9 extras)
            w0 = max(0, t - W + 1)
            for b in range(B):
                win = xh[li][b, w0:t + 1]
                akw = {}
                if s9 is not None:
                    P = s9[li]
                    win = oracle.token_prep(win, np.arange(w0, t + 1), DR, norm_w=host(P["kv_norm_w"]), eps=1e-6,
                                            inv_freq=host(P["inv_freq"]))
                    akw = {"q_norm_w": host(P["q_norm_w"]), "eps": 1e-6, "sink": host(P["sink"]),
                           "inv_freq": host(P["inv_freq"]), "q_pos": t}
                if r == 4:
                    c_, s_, r_ = ref_ent[li]
                    pos = np.array([[t]], np.int32)
                    sc, _ = oracle.index_scores(host(qc)[b:b + 1], host(qs)[b:b + 1], host(w)[b:b + 1],
                                                kch[b:b + 1], ksh[b:b + 1], pos, 4)
                    assert np.array_equal(host(loop.scores[li])[b, 0].view(np.uint32), sc[0, 0].view(np.uint32)), t
                    idx, cnt = oracle.topk(sc[0], pos[0], 4, K)
                    assert host(loop.count[li])[b] == cnt[0] and np.array_equal(host(loop.idx[li])[b], idx[0]), t
                    ref, _ = oracle.attend(qh[li][b], c_[b], s_[b], r_[b], idx[0, :cnt[0]], win, scale, G, **akw)
                elif r == 128:
                    c_, s_, r_ = ref_ent[li]
                    ref, _ = oracle.attend(qh[li][b], c_[b], s_[b], r_[b], np.arange((t + 1) // 128), win, scale, G,
                                           **akw)
                else:
                    empty = (np.zeros((1, D - DR), np.uint8), np.zeros((1, (D - DR) // G), np.float32),
                             np.zeros((1, DR), np.uint16))
                    ref, _ = oracle.attend(qh[li][b], *empty, np.zeros(0, np.int64), win, scale, G, **akw)
                assert_attn_close(host(out[li])[b], ref, f"t={t} layer={li} (ratio {r}) b={b}")
                n_checked += 1
    return n_checked


def test_decode_loop_300_tokens_across_blocks():
    assert _run_loop(1000, 1300, section9=False, seed=501) == 300 * 3 * B


def test_decode_loop_from_empty_state_with_section9_extras():
    assert _run_loop(0, 140, section9=True, seed=502) == 140 * 3 * B


def test_decode_loop_with_section9_extras_across_blocks():
    assert _run_loop(1020, 1160, section9=True, seed=503) == 140 * 3 * B
