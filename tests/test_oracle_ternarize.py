"""Pins of the oracle's ternarisation (its reading R10: per group of 128 along
K, the symmetric thresholds and the one FP16 scale that minimise the
residual sum (w - alpha t)^2 -- pwwt.cn/news/5175886, section 1.2; one scale
per group, 4sapi page, section 三), each checked against something other
than the oracle itself."""
import itertools

import numpy as np
import pytest

import oracle


def _err(w, t):
    """Residual of pattern t with its own best scale, in fp64."""
    w = w.astype(np.float64)
    nz = t != 0
    if not nz.any():
        return float(np.sum(w * w))
    s = float(np.sum(np.abs(w[nz])))
    return float(np.sum(w * w) - s * s / nz.sum())


def test_float_to_half_matches_numpy():
    rng = np.random.default_rng(3)
    vals = [rng.standard_normal(5000).astype(np.float32) * np.float32(s)
            for s in (1e-9, 1e-6, 3e-5, 1e-2, 1.0, 300.0, 4e4)]
    edge = np.float32([0.0, -0.0, 65504.0, 65519.99, 65520.0, 65536.0, 1e30, -1e30,
                       2.0 ** -24, 2.0 ** -25, 1.5 * 2.0 ** -25, 2.0 ** -14, 2.0 ** -14 * 0.9999,
                       1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, np.inf, -np.inf])
    for v in np.concatenate(vals + [edge]):
        with np.errstate(over="ignore"):
            want = int(np.float32(v).astype(np.float16).view(np.uint16))
        assert oracle.float_to_half_bits(v) == want, v


@pytest.mark.parametrize("n", [1, 2, 3, 5, 8])
def test_brute_force_over_every_pattern(n):
    """On tiny groups the chosen pattern has the smallest residual of all
    3^n ternary patterns (each with its optimal scale)."""
    rng = np.random.default_rng(100 + n)
    for trial in range(40):
        w = rng.standard_normal((1, n)).astype(np.float32) * np.float32(rng.uniform(0.01, 10))
        if trial % 7 == 0:
            w[0, rng.integers(n)] = 0.0
        t, _ = oracle.ternarize(w)
        best = min(_err(w[0], np.array(p, np.int8))
                   for p in itertools.product((-1, 0, 1), repeat=n))
        got = _err(w[0], t[0])
        assert got <= best + 1e-6 * float(np.sum(w.astype(np.float64) ** 2)) + 1e-30
        # signs follow the weights on the kept entries
        kept = t[0] != 0
        assert np.all(np.sign(w[0][kept]) == t[0][kept])


def test_scale_is_the_mean_of_the_kept_magnitudes():
    rng = np.random.default_rng(7)
    w = (rng.standard_normal((40, 384)) * 0.02).astype(np.float32)
    t, s = oracle.ternarize(w)
    for n in range(40):
        for g in range(3):
            blk, tb = w[n, 128 * g:128 * g + 128], t[n, 128 * g:128 * g + 128]
            kept = tb != 0
            mean = np.abs(blk[kept]).astype(np.float64).mean()
            # fp32 sum order vs fp64: within one fp16 step
            assert abs(float(s[n, g]) - mean) <= 2.0 ** -10 * mean


def test_closed_forms_and_special_cases():
    z = np.zeros((1, 128), np.float32)
    t, s = oracle.ternarize(z)
    assert not t.any() and float(s[0, 0]) == 0.0
    one = z.copy()
    one[0, 37] = -0.75
    t, s = oracle.ternarize(one)
    assert t[0, 37] == -1 and np.count_nonzero(t) == 1 and float(s[0, 0]) == 0.75
    eq = np.where(np.arange(128) % 3 == 0, 0.5, -0.5).astype(np.float32).reshape(1, 128)
    t, s = oracle.ternarize(eq)
    assert np.array_equal(t[0], np.sign(eq[0]).astype(np.int8)) and float(s[0, 0]) == 0.5
    # two magnitude levels: keep only the large ones when they dominate
    two = np.full((1, 128), 0.01, np.float32)
    two[0, :10] = 1.0
    t, s = oracle.ternarize(two)
    assert np.count_nonzero(t) == 10 and float(s[0, 0]) == 1.0


def test_invariances():
    rng = np.random.default_rng(11)
    w = rng.standard_normal((16, 640)).astype(np.float32)
    t, s = oracle.ternarize(w)
    t2, s2 = oracle.ternarize(w * np.float32(8.0))      # power-of-two scaling: exact
    assert np.array_equal(t, t2) and np.array_equal(s2.astype(np.float32), s.astype(np.float32) * 8)
    t3, s3 = oracle.ternarize(-w)
    assert np.array_equal(t3, -t) and np.array_equal(s3, s)
    # groups are independent: a ragged K equals the groups taken one by one
    K = 300
    wr = w[:, :K].copy()
    tr, sr = oracle.ternarize(wr)
    for g, (a, b) in enumerate([(0, 128), (128, 256), (256, 300)]):
        tg, sg = oracle.ternarize(np.ascontiguousarray(wr[:, a:b]))
        assert np.array_equal(tr[:, a:b], tg) and np.array_equal(sr[:, g], sg[:, 0])


def test_gaussian_groups_zero_fraction():
    """For Gaussian weights the residual-optimal threshold is about 0.61
    sigma, so about 46% of the trits are 0 (the large-group limit)."""
    rng = np.random.default_rng(5)
    w = rng.standard_normal((200, 1280)).astype(np.float32)
    t, _ = oracle.ternarize(w)
    frac = float(np.mean(t == 0))
    assert 0.42 < frac < 0.50
    assert abs(float(np.mean(t == 1)) - float(np.mean(t == -1))) < 0.02
