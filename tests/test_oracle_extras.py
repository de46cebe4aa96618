"""Pins of the oracle's section-9 extras ("DeepSeek V4 ..." reading note,
section 9: query / KV entry RMSNorm, partial RoPE on the last dims of the
query, the KV entry and the attention output, and the per-head attention
sink).  Each is checked against a closed form, an invariance, or the same
computation written with torch library routines in fp64 (rms_norm, complex
rotation, softmax), chosen so that a plausible slip (a missing weight, d-1
in the mean, a wrong rotation sign or pairing, a sink in the numerator, no
de-rotation of the output) fails."""
import numpy as np
import pytest
import torch

import oracle

D, DR, G = 512, 64, 64


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _inv_freq(dr=DR, base=10000.0):
    return (base ** (-np.arange(0, dr, 2, dtype=np.float64) / dr)).astype(np.float32)


# ------------------------------------------------------------------ RMSNorm
def test_rmsnorm_closed_forms_and_fp64():
    d = 512
    w1 = np.ones(d, np.float32)
    y = np.full(d, 3.0, np.float32)
    assert np.array_equal(oracle.rmsnorm_f32(y, w1, 0.0), np.ones(d, np.float32))
    y[::2] = -3.0
    assert np.array_equal(oracle.rmsnorm_f32(y, w1, 0.0), np.sign(y))
    rng = np.random.default_rng(3)
    for eps in (0.0, 1e-6, 0.25):
        y = (rng.standard_normal(d) * rng.uniform(0.01, 10)).astype(np.float32)
        w = rng.uniform(-2, 2, d).astype(np.float32)
        got = oracle.rmsnorm_f32(y, w, eps).astype(np.float64)
        ref = torch.nn.functional.rms_norm(torch.from_numpy(y.astype(np.float64)), (d,),
                                           weight=torch.from_numpy(w.astype(np.float64)), eps=eps).numpy()
        assert np.allclose(got, ref, rtol=4e-7, atol=1e-30)


def test_rmsnorm_power_of_two_invariance():
    rng = np.random.default_rng(4)
    y = rng.standard_normal(128).astype(np.float32)
    w = rng.uniform(0.5, 1.5, 128).astype(np.float32)
    base = oracle.rmsnorm_f32(y, w, 0.0)
    for k in (-20, -3, 5, 30):
        assert np.array_equal(oracle.rmsnorm_f32((y * np.float32(2.0 ** k)).astype(np.float32), w, 0.0), base)


# ------------------------------------------------------------------ RoPE
def test_rope_against_complex_rotation():
    rng = np.random.default_rng(5)
    f = _inv_freq()
    v = rng.standard_normal(DR)
    for pos in (0, 1, 7, 1023, 131071, 1048575):
        got = oracle.rope_f64(v, pos, f)
        z = torch.view_as_complex(torch.from_numpy(v.reshape(-1, 2).copy()))
        ang = torch.from_numpy(pos * f.astype(np.float64))
        ref = torch.view_as_real(z * torch.polar(torch.ones_like(ang), ang)).reshape(-1).numpy()
        assert np.allclose(got, ref, rtol=0, atol=1e-12)
    assert np.array_equal(oracle.rope_f64(v, 0, f), v)                    # position 0: identity


def test_rope_inverse_composition_and_relative_positions():
    rng = np.random.default_rng(6)
    f = _inv_freq()
    q, k = rng.standard_normal(DR), rng.standard_normal(DR)
    r = oracle.rope_f64(q, 5000, f)
    assert np.allclose(oracle.rope_f64(r, 5000, f, sign=-1), q, atol=1e-12)
    assert np.allclose(oracle.rope_f64(oracle.rope_f64(q, 300, f), 700, f), oracle.rope_f64(q, 1000, f), atol=1e-10)
    assert np.allclose(np.hypot(r[0::2], r[1::2]), np.hypot(q[0::2], q[1::2]), atol=1e-12)
    a = oracle.rope_f64(q, 100, f) @ oracle.rope_f64(k, 40, f)
    b = oracle.rope_f64(q, 1060, f) @ oracle.rope_f64(k, 1000, f)
    assert abs(a - b) < 1e-9


def test_token_prep():
    rng = np.random.default_rng(7)
    x = _bf16(rng.standard_normal((5, D)))
    pos = np.array([0, 3, 127, 4096, 1048575])
    assert np.array_equal(oracle.token_prep(x, pos, DR), x)                # nothing to do: bf16 identity
    f = _inv_freq()
    w = rng.uniform(0.5, 1.5, D).astype(np.float32)
    got = oracle.token_prep(x, pos, DR, norm_w=w, inv_freq=f)
    xf = oracle.bf16_to_f32(x).astype(np.float64)
    for j, p in enumerate(pos):
        yn = torch.nn.functional.rms_norm(torch.from_numpy(xf[j]), (D,), weight=torch.from_numpy(w.astype(np.float64)),
                                          eps=1e-6).numpy()
        yn[D - DR:] = oracle.rope_f64(yn[D - DR:], p, f)
        g = oracle.bf16_to_f32(got[j]).astype(np.float64)
        assert np.all(np.abs(g - yn) <= 2.0 ** -8 * np.abs(yn) + 1e-30)
    # position 0 with no norm leaves the token as it is
    assert np.array_equal(oracle.token_prep(x[:1], pos[:1], DR, inv_freq=f), x[:1])


# ------------------------------------------------------------------ compressed entries
def _raw(B, T, seed):
    rng = np.random.default_rng(seed)
    return _bf16(rng.standard_normal((B, T, D))), _bf16(rng.standard_normal((B, T, D))), \
        (rng.standard_normal((4, D)) * 0.5).astype(np.float32)


def test_compress_ex_reduces_and_scales():
    x, gt, b = _raw(2, 40, 8)
    base = oracle.compress(x, gt, b, 4, 10, DR, G)
    same = oracle.compress(x, gt, b, 4, 10, DR, G, norm_w=None, inv_freq=None)
    for a_, b_ in zip(base[:3], same[:3]):
        assert np.array_equal(a_, b_)
    w = np.random.default_rng(9).uniform(0.5, 1.5, D).astype(np.float32)
    f = _inv_freq()
    c0, s0, r0, _ = oracle.compress(x, gt, b, 4, 10, DR, G, norm_w=w, eps=0.0, inv_freq=f)
    # pooling is linear in x and RMSNorm (eps = 0) undoes any power-of-two scale exactly
    xs = _bf16(oracle.bf16_to_f32(x) * np.float32(8.0))
    c1, s1, r1, _ = oracle.compress(xs, gt, b, 4, 10, DR, G, norm_w=w, eps=0.0, inv_freq=f)
    assert np.array_equal(c0, c1) and np.array_equal(s0, s1) and np.array_equal(r0, r1)
    # normalised entries: dequantised, (y / rms) has mean square 1 after dividing out w
    c2, s2, r2, _ = oracle.compress(x, gt, b, 4, 10, DR, G, norm_w=np.ones(D, np.float32), eps=0.0)
    deq = oracle.e4m3_value(c2) * np.repeat(s2.astype(np.float64), G, axis=-1)
    full = np.concatenate([deq, oracle.bf16_to_f32(r2).astype(np.float64)], axis=-1)
    ms = (full ** 2).mean(axis=-1)
    assert np.all(np.abs(ms - 1.0) < 0.05)
    # RoPE dims: rotating the stored values back by the entry position e*m gives the unrotated ones
    c3, s3, r3, _ = oracle.compress(x, gt, b, 4, 10, DR, G, norm_w=w, eps=0.0)
    assert np.array_equal(c3, c0) and np.array_equal(s3, s0)              # FP8 dims untouched by RoPE
    for bb in range(2):
        for e in range(10):
            back = oracle.rope_f64(oracle.bf16_to_f32(r0[bb, e]).astype(np.float64), 4 * e, f, sign=-1)
            ref = oracle.bf16_to_f32(r3[bb, e]).astype(np.float64)
            assert np.all(np.abs(back - ref) <= 2.0 ** -7 * (np.abs(ref).max() + 1e-30))


# ------------------------------------------------------------------ attention with the extras
def _torch_attend(q_bits, K, scale, q_norm_w=None, eps=1e-6, sink=None, inv_freq=None, q_pos=0):
    """Textbook attention with torch fp64 library routines: rms_norm, complex
    rotation, softmax over the logits with the sink as one more column whose
    value row is zero."""
    q = torch.from_numpy(oracle.bf16_to_f32(q_bits).astype(np.float64))
    H, d = q.shape
    if q_norm_w is not None:
        q = torch.nn.functional.rms_norm(q, (d,), weight=torch.from_numpy(q_norm_w.astype(np.float64)), eps=eps)
    if inv_freq is not None:
        ang = torch.from_numpy(q_pos * inv_freq.astype(np.float64))
        rot = torch.polar(torch.ones_like(ang), ang)
        qr = torch.view_as_complex(q[:, d - DR:].reshape(H, -1, 2).contiguous()) * rot
        q = torch.cat([q[:, :d - DR], torch.view_as_real(qr).reshape(H, DR)], dim=1)
    Kt = torch.from_numpy(K)
    logits = scale * q @ Kt.T
    V = Kt
    if sink is not None:
        logits = torch.cat([logits, torch.from_numpy(sink.astype(np.float64)).view(H, 1)], dim=1)
        V = torch.cat([V, torch.zeros((1, d), dtype=torch.float64)], dim=0)
    o = torch.softmax(logits, dim=1) @ V
    if inv_freq is not None:
        orot = torch.view_as_complex(o[:, d - DR:].reshape(H, -1, 2).contiguous()) * torch.conj(rot)
        o = torch.cat([o[:, :d - DR], torch.view_as_real(orot).reshape(H, DR)], dim=1)
    return o.numpy()


def _keys(seed, n_ent=40, n_win=9):
    rng = np.random.default_rng(seed)
    x, gt, b = _raw(1, 4 * n_ent, seed)
    codes, scales, rope, _ = oracle.compress(x, gt, b, 4, n_ent, DR, G)
    win = _bf16(rng.standard_normal((n_win, D)))
    ent = np.sort(rng.choice(n_ent, n_ent // 2, replace=False))
    deq = oracle.e4m3_value(codes[0, ent]) * np.repeat(scales[0, ent].astype(np.float64), G, axis=-1)
    K = np.concatenate([np.concatenate([deq, oracle.bf16_to_f32(rope[0, ent]).astype(np.float64)], axis=-1),
                        oracle.bf16_to_f32(win).astype(np.float64)], axis=0)
    q = _bf16(rng.standard_normal((8, D)))
    return q, codes[0], scales[0], rope[0], ent, win, K


def test_attend_extras_against_torch():
    q, codes, scales, rope, ent, win, K = _keys(10)
    rng = np.random.default_rng(11)
    w = rng.uniform(0.5, 1.5, D).astype(np.float32)
    sink = rng.standard_normal(8).astype(np.float32)
    f = _inv_freq()
    scale = float(np.float32(D ** -0.5))               # the oracle takes the scale as fp32
    for kw in ({}, {"q_norm_w": w}, {"sink": sink}, {"inv_freq": f, "q_pos": 123457},
               {"q_norm_w": w, "sink": sink, "inv_freq": f, "q_pos": 1048575}):
        got, lse = oracle.attend(q, codes, scales, rope, ent, win, scale, G, **kw)
        ref = _torch_attend(q, K, scale, **kw)
        assert np.allclose(got, ref, rtol=0, atol=1e-11), kw


def test_sink_closed_forms():
    q, codes, scales, rope, ent, win, K = _keys(12)
    scale = D ** -0.5
    base, lse0 = oracle.attend(q, codes, scales, rope, ent, win, scale, G)
    far, lse1 = oracle.attend(q, codes, scales, rope, ent, win, scale, G, sink=np.full(8, -1e30, np.float32))
    assert np.allclose(far, base, atol=1e-14) and np.allclose(lse1, lse0, atol=1e-12)
    big, _ = oracle.attend(q, codes, scales, rope, ent, win, scale, G, sink=np.full(8, 1e3, np.float32))
    assert np.abs(big).max() < 1e-300
    # a sink of 0 is one more key with logit 0 and value 0: an all-zero window token
    zs, lse2 = oracle.attend(q, codes, scales, rope, ent, win, scale, G, sink=np.zeros(8, np.float32))
    zk, lse3 = oracle.attend(q, codes, scales, rope, ent, np.concatenate([win, np.zeros((1, D), np.uint16)]),
                             scale, G)
    assert np.allclose(zs, zk, atol=1e-14) and np.allclose(lse2, lse3, atol=1e-12)
    assert np.allclose(lse2, np.logaddexp(lse0, 0.0), atol=1e-12)
    # no keys: output 0, lse = the sink
    o, l = oracle.attend(q, codes, scales, rope, np.zeros(0, np.int64), np.zeros((0, D), np.uint16), scale, G,
                         sink=np.arange(8, dtype=np.float32))
    assert not o.any() and np.array_equal(l, np.arange(8, dtype=np.float64))


def test_rope_cancels_when_keys_share_the_query_position():
    """Keys stored rotated to the query's own position t: the logits are those
    of the unrotated vectors and the de-rotated output is the unrotated
    attention output (up to the bf16 rounding of the stored keys)."""
    rng = np.random.default_rng(13)
    f = _inv_freq()
    t = 777777
    win = _bf16(rng.standard_normal((20, D)))
    q = _bf16(rng.standard_normal((8, D)))
    empty = (np.zeros((1, D - DR), np.uint8), np.zeros((1, (D - DR) // G), np.float32), np.zeros((1, DR), np.uint16))
    win_rot = oracle.token_prep(win, np.full(20, t), DR, inv_freq=f)
    got, _ = oracle.attend(q, *empty, np.zeros(0, np.int64), win_rot, D ** -0.5, G, inv_freq=f, q_pos=t)
    ref, _ = oracle.attend(q, *empty, np.zeros(0, np.int64), win, D ** -0.5, G)
    assert np.abs(got - ref).max() < 2e-2 and np.abs(got - ref).mean() < 2e-3
