"""Pins of the oracle's overlapped CSA compressor and indexer-key compressor
("DeepSeek V4 ..." reading note, section 7: two KV streams C_a, C_b and two
gate streams Z_a, Z_b; every entry pools 2m adjacent tokens with row-wise
softmax weights, neighbouring entries overlapping; the indexer keys
K^IComp come from a compressor and are FP4, section 9).

The reading (entry i = block i-1 of stream a + block i of stream b, one
softmax over the 2m tokens) is pinned by reductions to the pinned plain
compressor, a numpy fp64 softmax pooling, a mean under uniform gates, and
chunking consistency; the FP4 storage (OCP MX e2m1 rule) by the nearest-
value property over a dense grid, the shared-exponent rule on constructed
blocks and power-of-two invariance."""
import numpy as np
import torch

import oracle

MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _f(bits):
    return oracle.bf16_to_f32(bits).astype(np.float64)


# ------------------------------------------------------------------ e2m1 / FP4 blocks
def test_e2m1_is_nearest_value_ties_to_even():
    grid = np.concatenate([np.linspace(-8, 8, 6401), MAG, -MAG, MAG[1:] + 0.25, (MAG[1:] + MAG[:-1]) / 2])
    for v in grid.astype(np.float32):
        code = oracle.f32_to_e2m1(v)
        val = oracle.e2m1_value(code)
        a = min(abs(float(v)), 6.0)
        dist = np.abs(MAG - a)
        best = dist.min()
        assert abs(abs(val) - a) == best, (v, code)
        ties = np.nonzero(dist == best)[0]
        if len(ties) > 1:                                   # a midpoint: the even code
            assert (code & 7) % 2 == 0, (v, code)
        assert (code & 8) == (8 if np.signbit(v) else 0)
    for k, mval in enumerate(MAG):                          # every value round-trips
        assert oracle.f32_to_e2m1(mval) == k and oracle.f32_to_e2m1(-mval) == 8 | k


def test_fp4_block_shared_exponent_rule():
    rng = np.random.default_rng(21)
    for X in (-10, -3, 0, 1, 5, 20):
        for top in (4.0, 5.0, 6.0, 7.99):                    # amax in [4, 8) * 2^X -> exponent byte X + 127
            v = rng.uniform(-1, 1, 32).astype(np.float32) * np.float32(2.0 ** X)
            v[7] = np.float32(top * 2.0 ** X)
            codes, sf = oracle.fp4_quant_block(v)
            assert sf == X + 127
            nib = np.stack([codes & 0xF, codes >> 4], axis=1).reshape(-1)
            deq = np.array([oracle.e2m1_value(int(n)) for n in nib]) * 2.0 ** X
            assert np.all(np.abs(deq - v) <= 2.0 ** (X + 1) + 1e-30)   # half a spacing, or the 6..8 clamp
            assert abs(deq[7] - min(top, 6.0) * 2.0 ** X) <= 2.0 ** X
    zero = np.zeros(32, np.float32)
    codes, sf = oracle.fp4_quant_block(zero)
    assert sf == 0 and not codes.any()
    v = rng.standard_normal(32).astype(np.float32)
    c0, s0 = oracle.fp4_quant_block(v)
    for k in (-7, 3, 11):
        ck, sk = oracle.fp4_quant_block((v * np.float32(2.0 ** k)).astype(np.float32))
        assert np.array_equal(ck, c0) and sk == s0 + k


# ------------------------------------------------------------------ overlapped pooling
def _streams(B, T, d, seed, std_gate=1.0):
    rng = np.random.default_rng(seed)
    return [_bf16(rng.standard_normal((B, T, d)) * (std_gate if i % 2 else 1.0)) for i in range(4)]  # xa, za, xb, zb


def _np_overlap(xa, za, xb, zb, bias, m, e):
    """fp64 numpy softmax pooling of entry e of sequence 0, by the reading."""
    rows_x, rows_z, rows_b = [], [], []
    if e >= 1:
        rows_x.append(_f(xa[0, (e - 1) * m:e * m])); rows_z.append(_f(za[0, (e - 1) * m:e * m])); rows_b.append(bias[:m])
    rows_x.append(_f(xb[0, e * m:(e + 1) * m])); rows_z.append(_f(zb[0, e * m:(e + 1) * m])); rows_b.append(bias[m:])
    X = np.concatenate(rows_x); Z = np.concatenate(rows_z) + np.concatenate(rows_b).astype(np.float64)
    p = np.exp(Z - Z.max(axis=0))
    return (p * X).sum(axis=0) / p.sum(axis=0)


def test_overlap_against_numpy_fp64():
    d, m, n = 128, 4, 9
    xa, za, xb, zb = _streams(1, n * m, d, 22)
    bias = (np.random.default_rng(23).standard_normal((2 * m, d)) * 0.5).astype(np.float32)
    codes, scales, rope, worst = oracle.compress_overlap(xa, za, xb, zb, bias, m, n, 32, 32)
    assert worst < 1e-5
    for e in range(n):
        y = _np_overlap(xa, za, xb, zb, bias, m, e)
        deq = oracle.e4m3_value(codes[0, e]) * np.repeat(scales[0, e].astype(np.float64), 32)
        assert np.all(np.abs(deq - y[:96]) <= 2.0 ** -4 * np.abs(y[:96]) + np.repeat(scales[0, e], 32) * 2.0 ** -9)
        assert np.all(np.abs(_f(rope[0, e]) - y[96:]) <= 2.0 ** -8 * np.abs(y[96:]) + 1e-30)


def test_overlap_reduces_to_plain_compressor_when_stream_a_is_off():
    """Gates of stream a at -1e4 give exact zero weights: each entry is the plain
    m-token pooling of stream b (with bias rows m..2m-1), bit for bit."""
    d, m, n = 512, 4, 7
    xa, za, xb, zb = _streams(2, n * m, d, 24)
    za = _bf16(np.full(za.shape, -1e4))
    bias = (np.random.default_rng(25).standard_normal((2 * m, d)) * 0.5).astype(np.float32)
    got = oracle.compress_overlap(xa, za, xb, zb, bias, m, n, 64, 64)
    want = oracle.compress(xb, zb, bias[m:], m, n, 64, 64)
    for a, b in zip(got[:3], want[:3]):
        assert np.array_equal(a, b)


def test_overlap_uniform_gates_give_the_2m_mean_and_chunks_agree():
    d, m, n = 128, 4, 10
    rng = np.random.default_rng(26)
    xa, _, xb, _ = _streams(1, n * m, d, 27)
    z0 = _bf16(np.zeros((1, n * m, d)))
    bias = np.zeros((2 * m, d), np.float32)
    c, s, r, _ = oracle.compress_overlap(xa, z0, xb, z0, bias, m, n, 32, 32)
    for e in range(1, n):
        mean = (np.concatenate([_f(xa[0, (e - 1) * m:e * m]), _f(xb[0, e * m:(e + 1) * m])])).mean(axis=0)
        assert np.all(np.abs(_f(r[0, e]) - mean[96:]) <= 2.0 ** -8 * np.abs(mean[96:]) + 1e-6)
    # entries k.. from a chunk starting at block k, with stream a's block k-1 passed separately
    za, zb = _streams(1, n * m, d, 28)[1::2]
    bias = (rng.standard_normal((2 * m, d)) * 0.5).astype(np.float32)
    full = oracle.compress_overlap(xa, za, xb, zb, bias, m, n, 32, 32)
    k = 6
    part = oracle.compress_overlap(xa[:, k * m:], za[:, k * m:], xb[:, k * m:], zb[:, k * m:], bias, m, n - k, 32, 32,
                                   a_prev=xa[:, (k - 1) * m:][:, :(n - k) * m], za_prev=za[:, (k - 1) * m:][:, :(n - k) * m],
                                   cap=n, entry_begin=k)
    for a, b in zip(full[:3], part[:3]):
        assert np.array_equal(a[:, k:], b[:, k:])


def test_index_key_compress_dequantises_to_the_pooled_key():
    c, m, n = 128, 4, 6
    xa, za, xb, zb = _streams(2, n * m, c, 29)
    bias = (np.random.default_rng(30).standard_normal((2 * m, c)) * 0.5).astype(np.float32)
    kc, ks = oracle.index_key_compress(xa, za, xb, zb, bias, m, n)
    for b in range(2):
        for e in range(n):
            y = _np_overlap(xa[b:b + 1], za[b:b + 1], xb[b:b + 1], zb[b:b + 1], bias, m, e)
            nib = np.stack([kc[b, e] & 0xF, kc[b, e] >> 4], axis=1).reshape(-1)
            deq = np.array([oracle.e2m1_value(int(v)) for v in nib]) * np.repeat(
                [2.0 ** (int(u) - 127) for u in ks[b, e]], 32)
            for blk in range(4):
                sl = slice(32 * blk, 32 * blk + 32)
                amax = np.abs(y[sl]).max()
                assert np.all(np.abs(deq[sl] - y[sl]) <= amax / 4 + 1e-6)
                assert ks[b, e, blk] == int(np.floor(np.log2(np.float32(amax)))) - 2 + 127
