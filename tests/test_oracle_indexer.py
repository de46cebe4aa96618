"""Pins for the oracle's lightning-indexer score (CPU only).

The score follows the "DeepSeek V4 ..." reading note, section 7:
I_{t,s} = sum_h w^I_{t,h} ReLU(q^I_{t,h} . K^IComp_s), with FP4 (section 9).
Pinned against: the e2m1 bit-field definition, exact fp64 numpy dots of the
decoded values, brute-force element pairs (all 16 x 16 codes x 5 x 5 scales),
the closed-form bound, the order of the head sum (constructed so that another
order gives other bits) and the causal block rule.
"""
import itertools

import numpy as np
import pytest

import oracle


def e2m1_from_bits(n):
    """Value of an e2m1 code from the format definition: sign, 2-bit exponent
    (bias 1), 1-bit mantissa, exponent 0 subnormal."""
    s = -1.0 if n & 8 else 1.0
    e = (n >> 1) & 3
    f = n & 1
    return s * (f * 0.5 if e == 0 else (1 + f / 2) * 2.0 ** (e - 1))


def test_e2m1_table_matches_bit_fields():
    for n in range(16):
        assert oracle.e2m1_value(n) == e2m1_from_bits(n)


def decode(codes, sf, c):
    """fp64 values of packed FP4 (element 2i in the low nibble) with ue8m0 per 32."""
    codes = np.asarray(codes, np.uint8)
    lo, hi = codes & 0xF, codes >> 4
    nib = np.stack([lo, hi], -1).reshape(*codes.shape[:-1], c)
    tab = np.array([e2m1_from_bits(n) for n in range(16)])
    v = tab[nib]
    scale = np.repeat(2.0 ** (np.asarray(sf, np.float64) - 127), 32, axis=-1)
    return v * scale


def test_single_element_pairs_exhaustive():
    c = 64
    for qn, kn in itertools.product(range(16), range(16)):
        for eq, ek in itertools.product(range(123, 128), range(123, 128)):
            pos = (qn * 7 + kn * 3 + eq + ek) % c               # vary the element position
            qc = np.zeros(c // 2, np.uint8)
            kc = np.zeros(c // 2, np.uint8)
            qc[pos // 2] = qn << (4 * (pos & 1))
            kc[pos // 2] = kn << (4 * (pos & 1))
            qs = np.full(c // 32, 127, np.uint8)
            ks = np.full(c // 32, 127, np.uint8)
            qs[pos // 32], ks[pos // 32] = eq, ek
            v, inexact = oracle.fp4_dot(qc, qs, kc, ks)
            assert not inexact
            assert v == e2m1_from_bits(qn) * e2m1_from_bits(kn) * 2.0 ** (eq - 127 + ek - 127)


@pytest.mark.parametrize("c", [64, 128])
def test_random_dots_equal_exact_numpy(c):
    rng = np.random.default_rng(c)
    for _ in range(300):
        qc = rng.integers(0, 256, c // 2, dtype=np.uint8)
        kc = rng.integers(0, 256, c // 2, dtype=np.uint8)
        qs = rng.integers(123, 128, c // 32, dtype=np.uint8)
        ks = rng.integers(123, 128, c // 32, dtype=np.uint8)
        v, inexact = oracle.fp4_dot(qc, qs, kc, ks)
        assert not inexact
        assert float(v) == float(np.dot(decode(qc, qs, c), decode(kc, ks, c)))


def test_closed_form_bound():
    c = 128
    six = np.full(c // 2, 0x77, np.uint8)        # every element 6.0
    neg6 = np.full(c // 2, 0xFF, np.uint8)       # every element -6.0
    one = np.full(c // 32, 127, np.uint8)
    assert oracle.fp4_dot(six, one, six, one)[0] == 4608.0
    assert oracle.fp4_dot(six, one, neg6, one)[0] == -4608.0
    # smallest scales: 2^-4 * 2^-4 -> 4608 / 256
    small = np.full(c // 32, 123, np.uint8)
    assert oracle.fp4_dot(six, small, six, small)[0] == 18.0


def _one_hot(c, pos, code):
    a = np.zeros(c // 2, np.uint8)
    a[pos // 2] = code << (4 * (pos & 1))
    return a


def test_score_head_order_relu_and_weights():
    """Four heads whose dots are 1, 1, 1, -6 with weights 1, 2^-24, 2^-24, 1:
    the defined order h = 0..3 gives exactly 1.0 (each 2^-24 add ties to even);
    summing the small terms first would give 1 + 2^-22.  The negative dot must
    contribute +0 (ReLU)."""
    c = 128
    one = 0x2                                                   # e2m1 code of 1.0
    # heads 0-2: query -1 on element 5; head 3: query +6 on element 5; key -1 on element 5
    qc2 = np.stack([_one_hot(c, 5, 0x8 | one)] * 3 + [_one_hot(c, 5, 0x7)])[None, None]
    qs = np.full((1, 1, 4, c // 32), 127, np.uint8)
    w = np.array([[[1.0, 2.0 ** -24, 2.0 ** -24, 1.0]]], np.float32)
    kc2 = _one_hot(c, 5, 0x8 | one)[None, None]
    ks = np.full((1, 1, c // 32), 127, np.uint8)
    pos = np.array([[3]], np.int32)
    s, n_inexact = oracle.index_scores(qc2, qs, w, kc2, ks, pos, m=4)
    assert n_inexact == 0
    assert s[0, 0, 0] == np.float32(1.0)
    small_first = np.float32(np.float32(np.float32(2.0 ** -24) + np.float32(2.0 ** -24)) + np.float32(1.0))
    assert small_first != np.float32(1.0)                       # the pin really distinguishes orders


def test_causal_block_rule():
    rng = np.random.default_rng(3)
    c, Hi, Nc = 64, 4, 40
    qc = rng.integers(0, 256, (1, 6, Hi, c // 2), dtype=np.uint8)
    qs = rng.integers(123, 128, (1, 6, Hi, c // 32), dtype=np.uint8)
    w = rng.uniform(0, 1, (1, 6, Hi)).astype(np.float32)
    kc = rng.integers(0, 256, (1, Nc, c // 2), dtype=np.uint8)
    ks = rng.integers(123, 128, (1, Nc, c // 32), dtype=np.uint8)
    for m in (4, 128):
        pos = np.array([[0, 2, 3, 4 * 7 + 2, 4 * 7 + 3, 1000]], np.int32) if m == 4 else \
            np.array([[0, 126, 127, 255, 256, 5000]], np.int32)
        s, _ = oracle.index_scores(qc, qs, w, kc, ks, pos, m)
        for t in range(6):
            n_elig = min(Nc, (int(pos[0, t]) + 1) // m)
            assert np.all(np.isneginf(s[0, t, n_elig:]))
            assert np.all(np.isfinite(s[0, t, :n_elig]))
            assert np.all(s[0, t, :n_elig] >= 0)


def test_scores_equal_numpy_relu_sum_for_random_inputs():
    """Independent fp64 evaluation.  With scales 2^-1..2^0 the dots are
    multiples of 2^-4 below 2^13, and with weights j/16 every product and
    partial sum fits 24 bits, so the fp32 score must equal the fp64 value."""
    rng = np.random.default_rng(9)
    B, Tq, Hi, c, Nc = 2, 3, 4, 128, 50
    qc = rng.integers(0, 256, (B, Tq, Hi, c // 2), dtype=np.uint8)
    qs = rng.integers(126, 128, (B, Tq, Hi, c // 32), dtype=np.uint8)
    w = (rng.integers(0, 17, (B, Tq, Hi)) / 16.0).astype(np.float32)
    kc = rng.integers(0, 256, (B, Nc, c // 2), dtype=np.uint8)
    ks = rng.integers(126, 128, (B, Nc, c // 32), dtype=np.uint8)
    pos = np.full((B, Tq), 10 ** 6, np.int32)
    s, _ = oracle.index_scores(qc, qs, w, kc, ks, pos, m=4)
    qv = decode(qc, qs, c)                  # [B][Tq][Hi][c]
    kv = decode(kc, ks, c)                  # [B][Nc][c]
    dots = np.einsum("bthc,bnc->btnh", qv, kv)
    want = (np.maximum(dots, 0) * w[:, :, None, :].astype(np.float64)).sum(-1)
    assert np.array_equal(s.astype(np.float64), want)
