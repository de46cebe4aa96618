"""Pins for the oracle's top-k selection and core attention (CPU only).

Top-k follows the "DeepSeek V4 ..." reading note, section 7
(C^SprsComp_t = entries whose I_{t,s} is in Top-k(I_{t,:})); ties go to the
lower index.  Attention follows section 7 (shared key-value MQA: the
compressed entry is both key and value; sliding-window branch over the last
n_win raw tokens) and section 8 (HCA: dense over all compressed entries).

Pins: brute-force sort on tiny inputs with many ties, a textbook fp64 torch
attention (softmax(q K^T * scale) V) over keys dequantised through torch's
float8 / bfloat16 types, exact special cases (single key, zero query) and the
log-sum-exp merge identity that split-K decoding relies on.
"""
import numpy as np
import pytest
import torch

import oracle


# ------------------------------------------------------------------ top-k
def _brute_topk(row, pos, m, k):
    n = min(len(row), (pos + 1) // m)
    order = sorted(range(n), key=lambda s: (-(float(row[s]) + 0.0), s))
    chosen = sorted(order[:k])
    return chosen + [-1] * (k - len(chosen)), len(chosen)


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(0)
    vals = np.array([-np.inf, -1.0, -0.0, 0.0, 0.5, 1.0, 2.0], np.float32)
    for trial in range(400):
        Nc = int(rng.integers(1, 13))
        m = int(rng.choice([1, 4]))
        rows = rng.choice(vals, size=(3, Nc)).astype(np.float32)
        pos = rng.integers(0, Nc * m + 3, 3).astype(np.int32)
        for k in range(1, 15):
            idx, cnt = oracle.topk(rows, pos, m, k)
            for r in range(3):
                want, wc = _brute_topk(rows[r], int(pos[r]), m, k)
                assert list(idx[r]) == want and cnt[r] == wc, (trial, k, r)


def test_topk_signed_zero_and_lower_index():
    row = np.array([[0.0, -0.0, 0.0, -0.0, 1.0]], np.float32)
    idx, cnt = oracle.topk(row, np.array([100], np.int32), 1, 3)
    assert list(idx[0]) == [0, 1, 4] and cnt[0] == 3


def test_topk_k_at_least_eligible_returns_all():
    rng = np.random.default_rng(1)
    row = rng.standard_normal((1, 50)).astype(np.float32)
    idx, cnt = oracle.topk(row, np.array([4 * 20 + 2], np.int32), 4, 64)   # 20 eligible
    assert cnt[0] == 20 and list(idx[0, :20]) == list(range(20)) and np.all(idx[0, 20:] == -1)


# ------------------------------------------------------------------ attention
def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)


def _bits(t):
    return t.view(torch.int16).numpy().view(np.uint16)


def _random_cache(rng, n, d, d_rope, g):
    dn = d - d_rope
    codes = rng.integers(0, 256, (n, dn), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3C                            # no NaN codes
    scales = rng.uniform(0.001, 0.01, (n, dn // g)).astype(np.float32)
    rope = _bits(_bf16(rng.standard_normal((n, d_rope))))
    return codes, scales, rope


def _keys_via_torch(codes, scales, rope, ent, win_bits, g):
    """Dequantise through torch's float8_e4m3fn / bfloat16 types (library)."""
    c = torch.from_numpy(codes[ent].copy()).view(torch.float8_e4m3fn).to(torch.float64)
    s = torch.from_numpy(scales[ent].astype(np.float64)).repeat_interleave(g, dim=1)
    r = torch.from_numpy(rope[ent].copy()).view(torch.bfloat16).to(torch.float64)
    comp = torch.cat([c * s, r], dim=1)
    win = torch.from_numpy(win_bits.copy()).view(torch.bfloat16).to(torch.float64)
    return torch.cat([comp, win], dim=0)


def _torch_attention(q_bits, K, scale):
    q = torch.from_numpy(q_bits.copy()).view(torch.bfloat16).to(torch.float64)
    logits = (q @ K.T) * scale
    p = torch.softmax(logits, dim=-1)
    return (p @ K).numpy(), torch.logsumexp(logits, dim=-1).numpy()


@pytest.mark.parametrize("d,d_rope,g,H", [(128, 32, 32, 8), (512, 64, 64, 16)])
def test_attention_matches_textbook_torch(d, d_rope, g, H):
    rng = np.random.default_rng(d)
    codes, scales, rope = _random_cache(rng, 300, d, d_rope, g)
    ent = rng.choice(300, 77, replace=False).astype(np.int64)
    win = _bits(_bf16(rng.standard_normal((128, d))))
    q = _bits(_bf16(rng.standard_normal((H, d))))
    scale = np.float32(1.0 / np.sqrt(d))
    out, lse = oracle.attend(q, codes, scales, rope, ent, win, scale, g)
    K = _keys_via_torch(codes, scales, rope, ent, win, g)
    want, want_lse = _torch_attention(q, K, float(scale))
    assert np.abs(out - want).max() < 1e-12
    assert np.abs(lse - want_lse).max() < 1e-12


def test_attention_reduces_to_mqa_when_m1_and_no_window():
    """Compression ratio 1 and a window of 0: pooling is the identity (m = 1),
    so attention over the compressed stream is plain MQA over the FP8-stored
    tokens."""
    rng = np.random.default_rng(2)
    d, d_rope, g, H, T = 128, 32, 32, 8, 64
    x = _bits(_bf16(rng.standard_normal((1, T, d))))
    gate = _bits(_bf16(rng.standard_normal((1, T, d))))
    bias = (rng.standard_normal((1, d)) * 0.5).astype(np.float32)
    codes, scales, rope, _ = oracle.compress(x, gate, bias, 1, T, d_rope, g)
    # independent storage of the raw tokens: torch casts of x itself
    xf = torch.from_numpy(x[0].copy()).view(torch.bfloat16).to(torch.float32)
    dn = d - d_rope
    amax = xf[:, :dn].abs().reshape(T, dn // g, g).amax(-1)
    sc = amax / 448.0
    c8 = (xf[:, :dn].reshape(T, dn // g, g) / sc[..., None]).reshape(T, dn).to(torch.float8_e4m3fn)
    assert np.array_equal(scales[0], sc.numpy())
    assert np.array_equal(codes[0], c8.view(torch.uint8).numpy())
    K = torch.cat([c8.to(torch.float64) * sc.to(torch.float64).repeat_interleave(g, 1), xf[:, dn:].to(torch.float64)], 1)
    q = _bits(_bf16(rng.standard_normal((H, d))))
    scale = np.float32(d ** -0.5)
    out, _ = oracle.attend(q, codes[0], scales[0], rope[0], np.arange(T), np.zeros((0, d), np.uint16), scale, g)
    want, _ = _torch_attention(q, K, float(scale))
    assert np.abs(out - want).max() < 1e-12


def test_attention_single_key_and_zero_query():
    rng = np.random.default_rng(3)
    d, d_rope, g = 128, 32, 32
    codes, scales, rope = _random_cache(rng, 10, d, d_rope, g)
    q = _bits(_bf16(rng.standard_normal((4, d))))
    out, lse = oracle.attend(q, codes, scales, rope, np.array([6]), np.zeros((0, d), np.uint16), 0.1, g)
    K = _keys_via_torch(codes, scales, rope, np.array([6]), np.zeros((0, d), np.uint16), g).numpy()
    assert np.array_equal(out, np.broadcast_to(K[0], out.shape))
    # zero query: every logit is 0, softmax is uniform, output is the key mean
    zq = np.zeros((2, d), np.uint16)
    win = _bits(_bf16(rng.standard_normal((5, d))))
    ent = np.array([1, 3, 8])
    out, lse = oracle.attend(zq, codes, scales, rope, ent, win, 0.1, g)
    K = _keys_via_torch(codes, scales, rope, ent, win, g).numpy()
    assert np.allclose(out, K.mean(0), rtol=0, atol=1e-14)
    assert np.allclose(lse, np.log(8.0))


def test_attention_lse_merge_identity():
    """attend(A u B) equals the log-sum-exp merge of attend(A) and attend(B)."""
    rng = np.random.default_rng(4)
    d, d_rope, g, H = 512, 64, 64, 4
    codes, scales, rope = _random_cache(rng, 200, d, d_rope, g)
    win = _bits(_bf16(rng.standard_normal((20, d))))
    q = _bits(_bf16(rng.standard_normal((H, d))))
    A, Bset = np.arange(0, 120), np.arange(120, 200)
    oa, la = oracle.attend(q, codes, scales, rope, A, np.zeros((0, d), np.uint16), 0.05, g)
    ob, lb = oracle.attend(q, codes, scales, rope, Bset, win, 0.05, g)
    o, l = oracle.attend(q, codes, scales, rope, np.arange(200), win, 0.05, g)
    M = np.maximum(la, lb)
    wa, wb = np.exp(la - M), np.exp(lb - M)
    merged = (oa * wa[:, None] + ob * wb[:, None]) / (wa + wb)[:, None]
    assert np.abs(merged - o).max() < 1e-12
    assert np.abs(M + np.log(wa + wb) - l).max() < 1e-12


def test_csa_with_k_covering_all_entries_equals_dense():
    """Top-k equal to all complete blocks: the sparse key set is every
    eligible entry, so CSA equals dense attention over the compressed stream."""
    rng = np.random.default_rng(5)
    d, d_rope, g, Nc, m = 128, 32, 32, 40, 4
    codes, scales, rope = _random_cache(rng, Nc, d, d_rope, g)
    scores = rng.standard_normal((1, Nc)).astype(np.float32)
    pos = np.array([4 * Nc - 1], np.int32)
    idx, cnt = oracle.topk(scores, pos, m, 64)
    q = _bits(_bf16(rng.standard_normal((8, d))))
    win = _bits(_bf16(rng.standard_normal((16, d))))
    o_sparse, _ = oracle.attend(q, codes, scales, rope, idx[0, :cnt[0]], win, 0.1, g)
    o_dense, _ = oracle.attend(q, codes, scales, rope, np.arange(Nc), win, 0.1, g)
    assert np.array_equal(o_sparse, o_dense)


def test_causal_key_sets_by_enumeration():
    """The causal rule of a prefill query at position p, enumerated token by
    token: entry s is visible iff all m tokens of its block are at or before
    p; the window holds the raw tokens in (p - W, p], none before 0."""
    for m in (1, 4, 128):
        for W in (1, 5, 128):
            for p in list(range(0, 300)) + [1023, 131071, 135167]:
                ent, w0, w1 = oracle.causal_keys(p, m, W)
                want = [s for s in range(p // m + 2) if all(t <= p for t in range(s * m, s * m + m))]
                assert list(ent) == want
                assert list(range(w0, w1)) == [t for t in range(max(0, p - 2 * W), p + 1) if p - W < t]
    ent, _, _ = oracle.causal_keys(1000, 4, 128, n_cap=100)
    assert len(ent) == 100
    ent, w0, w1 = oracle.causal_keys(50, 0, 128)
    assert len(ent) == 0 and (w0, w1) == (0, 51)

