"""Pins for the oracle's FP8 / BF16 storage rules (CPU only).

Storage follows the "DeepSeek V4 ..." reading note, section 9 (RoPE dims in
BF16, the other KV dims in FP8); the scale rule is amax/448 per group of g
channels (the e4m3fn finite maximum is 448).  The conversions are pinned
against torch's own float8_e4m3fn and bfloat16 casts (library routines), the
format's code table (round trip), constructed midpoints, and the exact
power-of-two scale invariance of the rule.
"""
import numpy as np
import pytest
import torch

import oracle


def _torch_e4m3(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_code_table_round_trip():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)   # all finite codes
    vals = oracle.e4m3_value(codes)
    # independent decode through torch's float8 type
    tv = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(vals, tv)
    assert np.array_equal(oracle.f32_to_e4m3(vals.astype(np.float32)), codes)
    assert vals.max() == 448.0


def test_e4m3_matches_torch_rn_in_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.uniform(-448, 448, 200000),
        rng.standard_normal(200000) * 0.01,            # subnormal region (< 2^-6)
        rng.standard_normal(200000) * 30,
    ]).astype(np.float32)
    x = x[np.abs(x) <= 448]
    assert np.array_equal(oracle.f32_to_e4m3(x), _torch_e4m3(x))


def test_e4m3_midpoints_round_to_even():
    codes = np.arange(0, 0x7E, dtype=np.uint8)
    lo = oracle.e4m3_value(codes)
    hi = oracle.e4m3_value(codes + 1)
    mid = ((lo + hi) / 2).astype(np.float32)
    assert np.array_equal(mid.astype(np.float64), (lo + hi) / 2)          # midpoints exact in fp32
    got = oracle.f32_to_e4m3(mid)
    want = np.where(codes % 2 == 0, codes, codes + 1)
    assert np.array_equal(got, want)
    assert np.array_equal(got, _torch_e4m3(mid))
    assert np.array_equal(oracle.f32_to_e4m3(-mid), want | 0x80)


def test_e4m3_saturates_and_keeps_sign_of_zero():
    assert oracle.f32_to_e4m3(np.float32(448.0)) == 0x7E
    assert oracle.f32_to_e4m3(np.float32(460.0)) == 0x7E
    assert oracle.f32_to_e4m3(np.float32(1e9)) == 0x7E
    assert oracle.f32_to_e4m3(np.float32(-1e9)) == 0xFE
    assert oracle.f32_to_e4m3(np.float32(-0.0)) == 0x80
    assert oracle.f32_to_e4m3(np.float32(0.0)) == 0x00
    assert oracle.f32_to_e4m3(np.float32(-1e-9)) == 0x80
    assert oracle.f32_to_e4m3(np.float32(2.0 ** -10)) == 0x00               # half of the smallest subnormal: tie -> even 0
    assert oracle.f32_to_e4m3(np.float32(1.5 * 2.0 ** -10)) == 0x01


def test_bf16_matches_torch():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(100000) * s for s in (1e-30, 1e-3, 1, 1e3, 1e30)]).astype(np.float32)
    # exact ties: low 16 bits = 0x8000
    ties = (rng.integers(0, 2**31, 20000, dtype=np.uint32) & 0xFFFF0000 | 0x8000).view(np.float32)
    ties = ties[np.isfinite(ties)]
    x = np.concatenate([x, ties])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f32_to_bf16(x), want)


@pytest.mark.parametrize("d,d_rope,g", [(128, 32, 32), (512, 64, 64)])
def test_quant_entry_rule(d, d_rope, g):
    rng = np.random.default_rng(d)
    y = (rng.standard_normal(d) * rng.uniform(0.01, 3)).astype(np.float32)
    dn = d - d_rope
    y[g:2 * g] = 0.0                                                         # an all-zero group
    codes, scales, rope = oracle.quant_entry(y, d_rope, g)
    assert scales[1] == 0.0 and not codes[g:2 * g].any()
    for G in range(dn // g):
        grp = y[G * g:(G + 1) * g]
        amax = np.abs(grp).max()
        assert scales[G] == np.float32(amax) / np.float32(448.0)
        if amax > 0:
            j = int(np.abs(grp).argmax())
            assert codes[G * g + j] & 0x7F == 0x7E                          # amax element -> +-448
    deq = oracle.e4m3_value(codes) * np.repeat(scales.astype(np.float64), g)
    s_rep = np.repeat(scales.astype(np.float64), g)
    assert np.all(np.abs(deq - y[:dn]) <= 2.0 ** -4 * np.abs(y[:dn]) + s_rep * 2.0 ** -10)
    want_rope = torch.from_numpy(y[dn:].copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(rope, want_rope)


def test_quant_power_of_two_invariance():
    rng = np.random.default_rng(7)
    y = rng.standard_normal(512).astype(np.float32)
    c0, s0, _ = oracle.quant_entry(y, 64, 64)
    for k in (-12, -5, -1, 1, 3, 9):
        ck, sk, _ = oracle.quant_entry((y * np.float32(2.0 ** k)).astype(np.float32), 64, 64)
        assert np.array_equal(ck, c0)
        assert np.array_equal(sk, (s0 * np.float32(2.0 ** k)).astype(np.float32))


def _bf16_exact(x: float) -> int:
    """bf16 bits of x rounded once to nearest-even, by exact rational arithmetic."""
    from fractions import Fraction
    import math
    if x == 0.0:
        return 0x8000 if math.copysign(1.0, x) < 0 else 0
    sign = 0x8000 if x < 0 else 0
    a = Fraction(abs(x))
    e = math.floor(math.log2(abs(x)))
    if Fraction(2) ** e > a:
        e -= 1
    if Fraction(2) ** (e + 1) <= a:
        e += 1
    sp = max(e - 7, -133)                                  # spacing of bf16 values near x
    q = a / Fraction(2) ** sp
    n = math.floor(q)
    rem = q - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    r = Fraction(n) * Fraction(2) ** sp
    if r >= Fraction(2) ** 128:
        return sign | 0x7F80
    f = np.float32(float(r))                               # exact: a bf16 value
    return sign | int(f.view(np.uint32)) >> 16


def test_round_bf16_rounds_once_from_fp64():
    """The attention tolerance compares against the fp64 result rounded to
    bf16: one rounding.  1 + 2^-8 + 2^-30 lies above the bf16 midpoint
    1 + 2^-8 but rounds to that midpoint in fp32, so a detour through fp32
    would give 1.0 instead of 1 + 2^-7."""
    x = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert int(oracle.round_bf16(np.array([x]))[0]) == 0x3F81
    assert int(oracle.round_bf16(np.array([-x]))[0]) == 0xBF81
    assert int(oracle.round_bf16(np.array([1.0 + 2.0 ** -8]))[0]) == 0x3F80          # tie to even
    assert int(oracle.round_bf16(np.array([1.0 + 3 * 2.0 ** -8]))[0]) == 0x3F82      # tie to even (up)
    rng = np.random.default_rng(11)
    xs = np.concatenate([rng.standard_normal(3000) * 10.0 ** rng.uniform(-40, 38, 3000),
                         [0.0, -0.0, 3.3895313892515355e38, 3.4e38, 1e-40, -2.0 ** -133, 2.0 ** -134 * 1.5]])
    got = oracle.round_bf16(xs)
    want = np.array([_bf16_exact(float(v)) for v in xs], np.uint16)
    assert np.array_equal(got, want)

