"""Pins for the oracle's pooling arithmetic (CPU only).

Pooling follows the "DeepSeek V4 ..." reading note, section 8 (HCA):
S = Softmax_row(Z_block + B), C^Comp = sum_j S_j (.) C_j, and the Hugging Face
blog's "softmax-gated pooling with a learned positional bias".  The pins below
tie the oracle's fp32 sequence to things other than itself: libm/numpy exp,
closed forms (uniform gates -> block mean, m = 1 -> identity), limits
(a dominant gate or bias selects one token) and an fp64 numpy evaluation.
"""
import math

import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.filterwarnings("ignore")


def _bits_bf16(a):
    import torch
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------------ E(z)
def test_exp_constants_are_correctly_rounded():
    mpmath = pytest.importorskip("mpmath")
    mpmath.mp.prec = 200

    def is_rn(f32, exact):
        f = np.float32(f32)
        lo, hi = np.nextafter(f, np.float32(-np.inf)), np.nextafter(f, np.float32(np.inf))
        e = abs(mpmath.mpf(float(f)) - exact)
        return e <= abs(mpmath.mpf(float(lo)) - exact) and e <= abs(mpmath.mpf(float(hi)) - exact)

    ln2 = mpmath.log(2)
    assert is_rn(oracle.constant(0), 1 / ln2)                       # log2(e)
    hi = oracle.constant(1)
    assert np.float32(hi).view(np.uint32) & 0x1FF == 0              # short head: n*hi exact
    assert abs(mpmath.mpf(float(hi)) - ln2) < 2.0 ** -15
    assert is_rn(oracle.constant(2), ln2 - mpmath.mpf(float(hi)))   # tail
    for k in range(8):
        assert is_rn(oracle.constant(10 + k), mpmath.mpf(1) / mpmath.factorial(k)), k


def test_exp_accuracy_against_libm():
    rng = np.random.default_rng(0)
    z = np.concatenate([np.linspace(-87, 0, 20001), -rng.exponential(3.0, 20000), [0.0, -1e-30, -0.5, -1.0]])
    z = z[z >= -87].astype(np.float32)
    e = oracle.exp_neg(z).astype(np.float64)
    ref = np.exp(z.astype(np.float64))
    rel = np.abs(e - ref) / ref
    assert rel.max() < 4 * 2.0 ** -24, rel.max()
    assert oracle.exp_neg(np.float32(0.0)) == np.float32(1.0)


def test_exp_flush_and_monotone():
    assert oracle.exp_neg(np.float32(-87.5)) == 0.0
    assert oracle.exp_neg(np.float32(-1000.0)) == 0.0
    z = np.sort(np.random.default_rng(1).uniform(-87, 0, 50000).astype(np.float32))
    e = oracle.exp_neg(z)
    assert np.all(np.diff(e) >= 0)


# ------------------------------------------------------------------ pooling
def _rand_block(rng, m, d):
    x = _bits_bf16(rng.standard_normal((m, d)))
    gate = _bits_bf16(rng.standard_normal((m, d)))
    bias = (rng.standard_normal((m, d)) * 0.5).astype(np.float32)
    return x, gate, bias


def _numpy_pool64(x, gate, bias):
    """Textbook pooling in fp64 with numpy's exp: softmax over tokens per channel."""
    z = oracle.bf16_to_f32(gate).astype(np.float64) + bias.astype(np.float64)
    z = z - z.max(axis=0, keepdims=True)
    p = np.exp(z)
    p /= p.sum(axis=0, keepdims=True)
    xv = oracle.bf16_to_f32(x).astype(np.float64)
    return (p * xv).sum(axis=0), (p * np.abs(xv)).sum(axis=0)


@pytest.mark.parametrize("m", [1, 4, 128])
def test_pool_matches_fp64_numpy(m):
    rng = np.random.default_rng(m)
    x, gate, bias = _rand_block(rng, m, 64)
    y, _ = oracle.pool_block(x, gate, bias)
    y64, mag = _numpy_pool64(x, gate, bias)
    err = np.abs(y.astype(np.float64) - y64)
    assert np.all(err <= (2 * m + 4) * 2.0 ** -24 * mag + 1e-37), (err / mag).max()


def test_pool_m1_is_identity():
    rng = np.random.default_rng(5)
    x, gate, bias = _rand_block(rng, 1, 256)
    y, _ = oracle.pool_block(x, gate, bias)
    assert np.array_equal(y, oracle.bf16_to_f32(x)[0])


@pytest.mark.parametrize("m", [4, 128])
def test_pool_uniform_gates_is_block_mean(m):
    rng = np.random.default_rng(10 + m)
    d = 96
    x = _bits_bf16(rng.standard_normal((m, d)))
    gate = np.tile(_bits_bf16(rng.standard_normal((1, d))), (m, 1))     # same logit for every token
    bias = np.zeros((m, d), np.float32)
    y, _ = oracle.pool_block(x, gate, bias)
    xv = oracle.bf16_to_f32(x).astype(np.float64)
    mean = xv.mean(axis=0)
    bound = m * 2.0 ** -24 * np.abs(xv).sum(axis=0) / m + 2.0 ** -24 * np.abs(mean)
    assert np.all(np.abs(y - mean) <= bound)


@pytest.mark.parametrize("m", [4, 128])
def test_pool_dominant_gate_selects_token(m):
    rng = np.random.default_rng(20 + m)
    d = 64
    x, gate, bias = _rand_block(rng, m, d)
    gate_f = oracle.bf16_to_f32(gate).copy()
    star = rng.integers(0, m, d)                     # a different winning token per channel
    gate_f[star, np.arange(d)] = 60.0
    y, _ = oracle.pool_block(x, _bits_bf16(gate_f), bias)
    want = oracle.bf16_to_f32(x)[star, np.arange(d)]
    assert np.allclose(y, want, rtol=1e-6, atol=1e-12)


@pytest.mark.parametrize("m", [4, 128])
def test_pool_bias_indexed_by_position_in_block_and_channel(m):
    rng = np.random.default_rng(30 + m)
    d = 64
    x = _bits_bf16(rng.standard_normal((m, d)))
    gate = _bits_bf16(np.zeros((m, d)))
    bias = np.zeros((m, d), np.float32)
    star = (np.arange(d) * 7 + 3) % m
    bias[star, np.arange(d)] = 60.0
    y, _ = oracle.pool_block(x, gate, bias)
    assert np.allclose(y, oracle.bf16_to_f32(x)[star, np.arange(d)], rtol=1e-6, atol=1e-12)


def test_pool_channel_permutation_equivariant():
    rng = np.random.default_rng(40)
    x, gate, bias = _rand_block(rng, 4, 128)
    perm = rng.permutation(128)
    y, _ = oracle.pool_block(x, gate, bias)
    yp, _ = oracle.pool_block(x[:, perm], gate[:, perm], bias[:, perm])
    assert np.array_equal(yp, y[perm])


def test_compress_places_entries_and_sequences():
    """compress() over [B][T][d] equals per-block pool + quantise at the right
    (sequence, entry) slot, starting at entry_begin."""
    rng = np.random.default_rng(50)
    B, m, d, d_rope, g, nb, e0 = 3, 4, 128, 32, 32, 5, 7
    x = _bits_bf16(rng.standard_normal((B, nb * m + 3, d)))
    gate = _bits_bf16(rng.standard_normal((B, nb * m + 3, d)))
    bias = (rng.standard_normal((m, d)) * 0.5).astype(np.float32)
    codes, scales, rope, worst = oracle.compress(x, gate, bias, m, nb, d_rope, g, cap=e0 + nb + 2, entry_begin=e0)
    assert worst < 2e-6
    assert not codes[:, :e0].any() and not codes[:, e0 + nb:].any()
    for b in range(B):
        for j in range(nb):
            y, y64 = oracle.pool_block(x[b, j * m:(j + 1) * m], gate[b, j * m:(j + 1) * m], bias)
            c, s, r = oracle.quant_entry(y, d_rope, g)
            assert np.array_equal(codes[b, e0 + j], c)
            assert np.array_equal(scales[b, e0 + j], s)
            assert np.array_equal(rope[b, e0 + j], r)
            # independent: numpy fp64 pooling, then the dequantised entry is within FP8 precision
            y_np, _ = _numpy_pool64(x[b, j * m:(j + 1) * m], gate[b, j * m:(j + 1) * m], bias)
            deq = oracle.e4m3_value(c) * np.repeat(s.astype(np.float64), g)
            dn = d - d_rope
            assert np.all(np.abs(deq - y_np[:dn]) <= 2.0 ** -4 * np.abs(y_np[:dn]) + np.repeat(s, g) * 2.0 ** -9 + 1e-6)
            assert np.allclose(oracle.bf16_to_f32(r), y_np[dn:], rtol=2.0 ** -8, atol=1e-30)
