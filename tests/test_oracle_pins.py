"""Pins of the CPU oracle against things other than itself.

Each check compares the oracle with an independent source: Python's own
base-3 / base-4 integer parsing, scipy's Sylvester Hadamard matrix, numpy's
fp16 conversion and matrix product, IEEE round-half-even, or a figure printed
on the pages.  Chosen so that a dropped term, a wrong sign or index, or a
transposed operand in the oracle fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg
import scipy.special

import oracle
from ternary_weight_decode_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ formats
def test_base3_all_243_codes_match_python_base3():
    digits = list(itertools.product(range(3), repeat=5))  # (t0..t4), t0 least significant
    w = np.array(digits, dtype=np.int8) - 1               # one 5-trit row per code
    packed = oracle.pack_base3(w)
    assert packed.shape == (243, 1)
    for t, b in zip(digits, packed[:, 0]):
        assert int(b) == int("".join(str(d) for d in reversed(t)), 3)
    assert sorted(packed[:, 0].tolist()) == list(range(243))
    back = oracle.unpack_base3(packed, 5)
    np.testing.assert_array_equal(back, w)


def test_base3_rejects_invalid_bytes_and_padding():
    for b in range(243, 256):
        with pytest.raises(oracle.OracleError):
            oracle.unpack_base3(np.array([[b]], np.uint8), 5)
    # K = 3: digits 3 and 4 are padding and must be 1 (w = 0)
    ok = int("11" + "000", 3)     # t4=1, t3=1, t2..t0 = 0
    assert oracle.unpack_base3(np.array([[ok]], np.uint8), 3).tolist() == [[-1, -1, -1]]
    bad = int("21" + "000", 3)
    with pytest.raises(oracle.OracleError):
        oracle.unpack_base3(np.array([[bad]], np.uint8), 3)


def test_base3_closed_form_bytes():
    # all w = 0 -> all digits 1 -> 1+3+9+27+81 = 121; all +1 -> 242; all -1 -> 0
    for val, byte in ((0, 121), (1, 242), (-1, 0)):
        assert oracle.pack_base3(np.full((1, 5), val, np.int8))[0, 0] == byte


def test_2bit_all_81_codes_match_python_base4():
    digits = list(itertools.product(range(3), repeat=4))
    w = np.array(digits, dtype=np.int8) - 1
    packed = oracle.pack_2bit(w)
    for t, b in zip(digits, packed[:, 0]):
        assert int(b) == int("".join(str(d) for d in reversed(t)), 4)
    np.testing.assert_array_equal(oracle.unpack_2bit(packed, 4), w)
    valid = set(int(b) for b in packed[:, 0])
    for b in range(256):
        if b not in valid:
            with pytest.raises(oracle.OracleError):
                oracle.unpack_2bit(np.array([[b]], np.uint8), 4)


def test_d3_fixed_point_codes():
    codes = [oracle.d3_encode_value(V) for V in range(243)]
    assert len(set(codes)) == 243 and min(codes) >= 0 and max(codes) <= 255
    assert codes == sorted(codes)
    valid = 0
    for y in range(256):
        V = oracle.d3_decode_value(y)
        if V >= 0:
            valid += 1
            assert codes[V] == y
    assert valid == 243
    # The multiply-and-floor digit rule the kernels use gives the base-3 digits
    # (most significant first) that numpy's base_repr prints.
    for V, y in enumerate(codes):
        ref = [int(c) for c in np.base_repr(V, 3).zfill(5)]
        got = [(y * 3 ** (i + 1) // 256) % 3 for i in range(5)]
        assert got == ref, (V, y)
        assert (y * 243) // 256 == V


@pytest.mark.parametrize("fmt", [oracle.FMT_BASE3, oracle.FMT_2BIT])
def test_device_layout_positions_by_probe(fmt):
    K = 47
    used = oracle.device_row_bytes(fmt, K)
    assert used == (4 * math.ceil(K / 20) if fmt == 0 else 4 * math.ceil(K / 16))
    stride = 32
    base = oracle.pack_device(fmt, np.zeros((1, K), np.int8), stride)
    assert not base[0, used:].any()
    for k in range(K):
        w = np.zeros((1, K), np.int8)
        w[0, k] = 1
        changed = np.nonzero(oracle.pack_device(fmt, w, stride)[0] != base[0])[0].tolist()
        if fmt == 0:
            assert changed == [4 * (k // 20) + (k % 20) % 4]
        else:
            assert changed == [4 * (k // 16) + (k % 16) % 4]
            field = (k % 16) // 4
            byte = oracle.pack_device(fmt, w, stride)[0, changed[0]]
            assert (byte >> (2 * field)) & 3 == 2


@pytest.mark.parametrize("fmt", [oracle.FMT_BASE3, oracle.FMT_2BIT])
@pytest.mark.parametrize("K", [1, 5, 19, 20, 21, 127, 128, 300, 641])
def test_device_layout_round_trip_equals_canonical(fmt, K):
    w = synth.trits(7, 3, 9, K)
    stride = ((oracle.device_row_bytes(fmt, K) + 15) // 16) * 16
    dev = oracle.pack_device(fmt, w, stride)
    np.testing.assert_array_equal(oracle.unpack_device(fmt, dev, K), w)
    np.testing.assert_array_equal(oracle.unpack_base3(oracle.pack_base3(w), K), w)
    np.testing.assert_array_equal(oracle.unpack_2bit(oracle.pack_2bit(w), K), w)


def test_half_to_double_all_bit_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    finite = np.isfinite(ref)
    np.testing.assert_array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(np.isinf(got), np.isinf(ref))


# ------------------------------------------------------------------ Hadamard
def test_fwht_f64_equals_sylvester_matrix():
    H = scipy.linalg.hadamard(128).astype(np.float64)
    rng = np.random.default_rng(1)
    v = rng.integers(-50, 50, 128).astype(np.float64)
    np.testing.assert_array_equal(oracle.fwht128_f64(v), H @ v)
    v = rng.standard_normal(128)
    np.testing.assert_allclose(oracle.fwht128_f64(v), H @ v, rtol=0, atol=1e-12)


def test_fwht_involution_and_parseval():
    rng = np.random.default_rng(2)
    v = rng.integers(-1000, 1000, 128).astype(np.float64)
    np.testing.assert_array_equal(oracle.fwht128_f64(oracle.fwht128_f64(v)), 128 * v)
    x = rng.standard_normal(128)
    hx = oracle.fwht128_f64(x)
    assert abs(hx @ hx - 128 * (x @ x)) < 1e-9 * (x @ x)


def test_fwht_f32_within_rounding_bound():
    H = scipy.linalg.hadamard(128).astype(np.float64)
    rng = np.random.default_rng(3)
    x = synth.activations(5, 1, 128)[0].astype(np.float32)
    got = oracle.fwht128_f32(x).astype(np.float64)
    ref = H @ x.astype(np.float64)
    # 7 butterfly stages, one fp32 rounding each: |err| <= 7 * 2^-24 * sum|x| (loose)
    bound = 7 * 2.0 ** -24 * np.abs(x.astype(np.float64)).sum() * 1.01
    assert np.max(np.abs(got - ref)) <= bound
    xi = rng.integers(-100, 100, 128).astype(np.float32)
    np.testing.assert_array_equal(oracle.fwht128_f32(xi), (H @ xi.astype(np.float64)).astype(np.float32))


# ------------------------------------------------------------------ quantisation
def test_quant_round_half_even_and_extremes():
    x = np.array([[127.0, 2.5, 3.5, -2.5, 0.5, -127.0, 1.5, -0.5]], np.float32)
    q, s = oracle.act_quant(x)
    assert q.tolist() == [[127, 2, 4, -2, 0, -127, 2, 0]]
    assert s[0] == np.float32(1.0)


def test_quant_zero_row():
    q, s = oracle.act_quant(np.zeros((2, 64), np.float32))
    assert not q.any() and not s.any()


def test_quant_scale_invariance_and_error_bound():
    x = synth.activations(11, 3, 640).astype(np.float32)
    q, s = oracle.act_quant(x)
    for k in (-3, 1, 4):
        q2, s2 = oracle.act_quant(x * np.float32(2.0 ** k))
        np.testing.assert_array_equal(q2, q)
        np.testing.assert_array_equal(s2, s * np.float32(2.0 ** k))
    amax = np.abs(x.astype(np.float64)).max(axis=1)
    np.testing.assert_allclose(s, amax / 127, rtol=1e-7)
    assert (np.abs(q).max(axis=1) == 127).all()
    err = np.abs(s[:, None].astype(np.float64) * q - x)
    assert (err <= s[:, None] * 0.5 * (1 + 1e-5)).all()


def test_quant_fwht_dequantises_to_orthonormal_hadamard():
    H = scipy.linalg.hadamard(128).astype(np.float64) / math.sqrt(128)
    x = synth.activations(12, 2, 512).astype(np.float32)
    q, s = oracle.act_quant(x, fwht_block=128)
    ref = np.concatenate([x[:, b * 128:(b + 1) * 128].astype(np.float64) @ H.T for b in range(4)],
                         axis=1)
    amax = np.abs(ref).max(axis=1)
    np.testing.assert_allclose(s, amax / 127, rtol=1e-6)
    err = np.abs(s[:, None].astype(np.float64) * q - ref)
    assert (err <= s[:, None] * 0.5 * (1 + 1e-4) + 1e-6).all()


def test_quant_rmsnorm_scales_by_inverse_rms():
    x = synth.activations(13, 3, 640).astype(np.float32)
    q, s = oracle.act_quant(x)
    qn, sn = oracle.act_quant(x, rmsnorm=True)
    np.testing.assert_array_equal(q, qn)
    rms = np.sqrt((x.astype(np.float64) ** 2).mean(axis=1) + 1e-6)
    np.testing.assert_allclose(sn, s / rms, rtol=1e-7)
    # a constant row of value c has rms |c|: the scale becomes 1/127
    qc, sc = oracle.act_quant(np.full((1, 256), -3.0, np.float32), rmsnorm=True)
    np.testing.assert_allclose(sc[0], 1 / 127, rtol=1e-6)


def test_quant_rejects_bad_arguments():
    with pytest.raises(oracle.OracleError):
        oracle.act_quant(np.ones((1, 200), np.float32), fwht_block=128)
    with pytest.raises(oracle.OracleError):
        oracle.act_quant(np.ones((1, 256), np.float32), fwht_block=64)


# ------------------------------------------------------------------ products
@pytest.mark.parametrize("N,K", [(5, 128), (7, 300), (3, 1280), (4, 17)])
def test_group_partials_match_numpy_matmul(N, K):
    w = synth.trits(3, 0, N, K)
    q = np.random.default_rng(4).integers(-127, 128, (2, K)).astype(np.int8)
    P = oracle.group_partials(w, q)
    G = math.ceil(K / 128)
    assert P.shape == (2, N, G)
    for g in range(G):
        sl = slice(128 * g, min(K, 128 * (g + 1)))
        ref = q[:, sl].astype(np.int64) @ w[:, sl].astype(np.int64).T
        np.testing.assert_array_equal(P[:, :, g], ref)


@pytest.mark.parametrize("N,K,M", [(8, 256, 1), (16, 640, 3), (5, 1280, 2), (9, 300, 1)])
def test_gemv_matches_dense_dequantised_matmul(N, K, M):
    w = synth.trits(1, 0, N, K)
    sw = synth.scales(1, 1, N, math.ceil(K / 128))
    x = synth.activations(2, M, K)
    q, s = oracle.act_quant(x)
    y = oracle.gemv(w, sw, q, s)
    # brute force: expand the group scale to every weight, one dense product
    wdeq = w.astype(np.float64) * np.repeat(sw.astype(np.float64), 128, axis=1)[:, :K]
    ref = (s.astype(np.float64)[:, None] * q.astype(np.float64)) @ wdeq.T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_gemv_special_weights():
    K = 128
    x = synth.activations(3, 2, K)
    q, s = oracle.act_quant(x)
    sw = np.full((1, 1), 0.03125, np.float16)
    y0 = oracle.gemv(np.zeros((1, K), np.int8), sw, q, s)
    assert not y0.any()
    y1 = oracle.gemv(np.ones((1, K), np.int8), sw, q, s)
    expect = s.astype(np.float64) * 0.03125 * q.astype(np.int64).sum(axis=1)
    np.testing.assert_array_equal(y1[:, 0], expect)
    ym = oracle.gemv(-np.ones((1, K), np.int8), sw, q, s)
    np.testing.assert_array_equal(ym, -y1)


def test_swiglu_against_scipy_expit():
    rng = np.random.default_rng(5)
    g = rng.standard_normal(1000) * 5
    u = rng.standard_normal(1000)
    np.testing.assert_allclose(oracle.swiglu(g, u), g * scipy.special.expit(g) * u,
                               rtol=1e-14, atol=1e-300)
    assert oracle.swiglu(np.zeros(1), np.ones(1))[0] == 0.0
    assert not np.allclose(oracle.swiglu(g, u), oracle.swiglu(u, g))


def test_gateup_swiglu_composes_two_gemvs():
    N, K = 12, 384
    wg, wu = synth.trits(9, 4, N, K), synth.trits(9, 6, N, K)
    sg, su = synth.scales(9, 5, N, 3), synth.scales(9, 7, N, 3)
    q, s = oracle.act_quant(synth.activations(4, 2, K), fwht_block=128)
    h = oracle.gateup_swiglu(wg, sg, wu, su, q, s)
    g = oracle.gemv(wg, sg, q, s)
    u = oracle.gemv(wu, su, q, s)
    np.testing.assert_allclose(h, g * scipy.special.expit(g) * u, rtol=1e-13)


# ------------------------------------------------------------------ page figures
def _fig():
    with open(os.path.join(GOLDEN, "page_figures.json")) as f:
        return json.load(f)


def test_page_bit_widths_against_oracle_sizes():
    fig = _fig()
    assert abs(math.log2(3) - fig["log2_3_bits"]["value"]) < 5e-4
    K = 5120
    code_bits = 8 * oracle.base3_row_bytes(K) / K
    assert code_bits == 1.6 == fig["base3_bits_per_trit_approx"]["value"]
    assert 8 * oracle.device_row_bytes(oracle.FMT_BASE3, K) / K == 1.6
    assert 8 * oracle.twobit_row_bytes(K) / K == 2.0
    # codes + one fp16 scale per 128 weights
    b3 = code_bits + 16 / 128
    b2 = 2.0 + 16 / 128
    params = fig["bonsai_params"]["value"]
    # the whole published file (embeddings included) sits just above the codes + scales
    assert b3 < fig["bonsai_effective_bits"]["value"] < b3 + 0.05
    assert abs(params * fig["bonsai_effective_bits"]["value"] / 8
               - fig["bonsai_effective_bytes"]["value"]) / 5.94e9 < 0.001
    # PQ2 (2-bit codes + fp16/128 scales) at 27e9 weights ~ the quoted 7.2 GB
    assert abs(params * b2 / 8 - fig["pq2_bytes"]["value"]) / 7.2e9 < 0.01
    assert abs(params * 2 / 8 - fig["two_bit_bytes_27b"]["value"]) < 1


def test_page_bandwidth_arithmetic():
    fig = _fig()
    f = fig["ptq1_0_file_bytes"]
    assert abs(f["value"] / 2 ** 30 - f["gib"]) < 5e-4
    ws = fig["weight_stream_gibs"]
    lo, hi = ws["tok_s_low"] * f["gib"], ws["tok_s_high"] * f["gib"]
    assert abs(lo - ws["low"]) < 1 and abs(hi - ws["high"]) < 1.2
    kv = fig["q4_kv_bytes_per_token"]
    assert kv["value"] * kv["ctx"] / 2 ** 30 == kv["gib"]
