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
