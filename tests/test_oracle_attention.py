"""Pins of the oracle's Q4_0 KV cache and decode attention (its reading R12:
Q4_0 blocks of 32 with one fp16 scale, K/V decoded inside attention -- Bonsai
page, "先交代机器和配置" and the passage before "PQ2 会不会快很多"), checked
against closed forms, invariants and the pages' byte figures."""
import math

import numpy as np
import pytest

import oracle


def test_q4_0_error_bound_and_extreme_element():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((200, 32)) * rng.uniform(0.01, 5, (200, 1))).astype(np.float32)
    d, qs = oracle.q4_0_quantize(x)
    y = oracle.q4_0_dequantize(d, qs)
    for b in range(200):
        i = int(np.argmax(np.abs(x[b])))
        dd = -x[b, i] / 8.0  # the block scale before fp16 rounding
        d16 = float(d[b, 0])
        assert abs(d16 - dd) <= abs(dd) * 2.0 ** -11
        slack = 8 * abs(d16 - dd) + 1e-7 * abs(dd)
        r = x[b] / dd
        err = np.abs(y[b] - x[b])
        assert np.all(err[r < 7.5] <= 0.5 * abs(dd) + slack)   # rounded to the nearest level
        assert np.all(err[r >= 7.5] <= abs(dd) + slack)        # the clamped top level (code 15)
        assert abs(y[b, i] - (-8.0 * d16)) == 0.0              # the extreme value sits on code 0


def test_q4_0_closed_forms_and_nibble_layout():
    z = np.zeros((1, 32), np.float32)
    d, qs = oracle.q4_0_quantize(z)
    assert float(d[0, 0]) == 0.0 and np.all(qs == 0x88)
    x = np.zeros((1, 32), np.float32)
    x[0, 5] = 2.0
    d, qs = oracle.q4_0_quantize(x)
    assert float(d[0, 0]) == -0.25 and qs[0, 0, 5] == 0x80 and np.all(np.delete(qs[0, 0], 5) == 0x88)
    # values -8d .. 7d on codes 0 .. 15: element j low nibble, element j + 16 high nibble
    d0 = 0.5
    lv = np.arange(32) % 16
    x = ((lv - 8) * d0).astype(np.float32).reshape(1, 32)
    x[0, 0] = -8 * d0  # the extreme (first on ties), so d = +d0
    d, qs = oracle.q4_0_quantize(x)
    assert float(d[0, 0]) == d0
    np.testing.assert_array_equal(qs[0, 0] & 15, lv[:16])
    np.testing.assert_array_equal(qs[0, 0] >> 4, lv[16:])


def test_q4_0_bytes_match_the_pages_kv_figures():
    """18 bytes per 32 values.  With the KV formula of pwwt.cn/news/4940051
    (section 4.1: 2 x layers x KV heads x head dim x context x bytes per
    element), 64 layers, 2 KV heads of 128 give the Bonsai page's 18,432 B
    per token, and 65,536 tokens give its 1.125 GiB."""
    per_value = 18 / 32
    per_token = 2 * 64 * 2 * 128 * per_value
    assert per_token == 18432
    assert per_token * 65536 / 2 ** 30 == 1.125
    # the 27B shape benched here (8 KV heads of 128): 1152 B per layer and token
    assert 2 * 8 * 128 * per_value == 1152


def _cache(rng, Hkv, L, D, scale=1.0):
    k = (rng.standard_normal((Hkv, L, D)) * scale).astype(np.float32)
    v = rng.standard_normal((Hkv, L, D)).astype(np.float32)
    return oracle.q4_0_quantize(k) + oracle.q4_0_quantize(v)


def test_attention_single_token_and_uniform_weights():
    rng = np.random.default_rng(2)
    kd, kq, vd, vq = _cache(rng, 2, 1, 64)
    q = rng.standard_normal((4, 64)).astype(np.float32)
    out = oracle.attention_decode(q, kd, kq, vd, vq)
    v = oracle.q4_0_dequantize(vd, vq)
    np.testing.assert_allclose(out, np.repeat(v[:, 0], 2, axis=0), rtol=0, atol=1e-15)
    kd, kq, vd, vq = _cache(rng, 2, 37, 64)
    out = oracle.attention_decode(np.zeros((4, 64), np.float32), kd, kq, vd, vq)
    v = oracle.q4_0_dequantize(vd, vq)
    np.testing.assert_allclose(out, np.repeat(v.mean(axis=1), 2, axis=0), rtol=1e-12, atol=1e-14)


def test_attention_two_tokens_is_a_sigmoid_blend():
    """L = 2: out = v0 + sigmoid(s1 - s0) (v1 - v0), s = q.k / sqrt(D)."""
    rng = np.random.default_rng(3)
    D = 128
    kd, kq, vd, vq = _cache(rng, 1, 2, D, scale=0.3)
    q = rng.standard_normal((1, D)).astype(np.float32)
    k = oracle.q4_0_dequantize(kd, kq)[0]
    v = oracle.q4_0_dequantize(vd, vq)[0]
    s = k @ q[0].astype(np.float64) / math.sqrt(D)
    w1 = 1.0 / (1.0 + math.exp(-(s[1] - s[0])))
    np.testing.assert_allclose(oracle.attention_decode(q, kd, kq, vd, vq)[0], v[0] + w1 * (v[1] - v[0]),
                               rtol=1e-12, atol=1e-14)


def test_attention_invariants():
    rng = np.random.default_rng(4)
    Hkv, Hq, L, D = 2, 10, 50, 128
    kd, kq, vd, vq = _cache(rng, Hkv, L, D, scale=0.2)
    q = rng.standard_normal((Hq, D)).astype(np.float32)
    out = oracle.attention_decode(q, kd, kq, vd, vq)
    v = oracle.q4_0_dequantize(vd, vq)
    # a convex combination of the value rows of the head's KV group
    for h in range(Hq):
        g = h * Hkv // Hq
        assert np.all(out[h] <= v[g].max(axis=0) + 1e-12) and np.all(out[h] >= v[g].min(axis=0) - 1e-12)
    # token order does not matter; every token twice gives the same softmax
    perm = rng.permutation(L)
    np.testing.assert_allclose(oracle.attention_decode(q, kd[:, perm], kq[:, perm], vd[:, perm], vq[:, perm]),
                               out, rtol=1e-12, atol=1e-13)
    dup = np.repeat(np.arange(L), 2)
    np.testing.assert_allclose(oracle.attention_decode(q, kd[:, dup], kq[:, dup], vd[:, dup], vq[:, dup]),
                               out, rtol=1e-12, atol=1e-13)
    # grouped query heads: KV head 1 feeds query heads 5..9 only
    vd2 = vd.copy()
    vd2[1] = (vd2[1].astype(np.float32) * 3).astype(np.float16)
    out2 = oracle.attention_decode(q, kd, kq, vd2, vq)
    np.testing.assert_array_equal(out2[:5], out[:5])
    assert np.all(np.abs(out2[5:] - out[5:]).max(axis=1) > 0)


def test_attention_dominant_key():
    """A query along one cached key, scaled up, selects that token's value."""
    rng = np.random.default_rng(5)
    kd, kq, vd, vq = _cache(rng, 1, 20, 128)
    k = oracle.q4_0_dequantize(kd, kq)[0]
    v = oracle.q4_0_dequantize(vd, vq)[0]
    j = 13
    q = (k[j] / np.linalg.norm(k[j]) * 400.0).astype(np.float32).reshape(1, 128)
    s = k @ q[0].astype(np.float64)
    assert np.argmax(s) == j
    out = oracle.attention_decode(q, kd, kq, vd, vq)[0]
    np.testing.assert_allclose(out, v[j], atol=1e-3 * np.abs(v[j]).max())
