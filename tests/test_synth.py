"""Pins of the seeded input generator (host side)."""
import json
import os

import numpy as np

from ternary_weight_decode_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_splitmix64_reference_outputs():
    with open(os.path.join(GOLDEN, "splitmix64_reference.json")) as f:
        ref = json.load(f)
    for case in ref["cases"]:
        outs = case.get("outputs_hex") or case.get("outputs_dec")
        expect = [int(o, 0) for o in outs]
        # the idx-th output of the generator started at `state`
        got_int = [synth.mix64_int(case["state"] + (i + 1) * synth.GAMMA) for i in range(len(expect))]
        assert got_int == expect
        got_np = synth._mix64_np(np.array([(case["state"] + (i + 1) * synth.GAMMA) & synth.MASK64
                                           for i in range(len(expect))], dtype=np.uint64))
        assert [int(v) for v in got_np] == expect


def test_hash_at_matches_scalar_definition():
    seed, stream = 17, 5
    key = synth.stream_key(seed, stream)
    idx = np.array([0, 1, 2, 1000, 2 ** 40 + 3], dtype=np.uint64)
    got = synth.hash_at(seed, stream, idx)
    for i, v in zip(idx.tolist(), got.tolist()):
        assert v == synth.mix64_int(key + (i + 1) * synth.GAMMA)


def test_trit_distribution():
    t = synth.trits(0, synth.stream_id(0, 0), 256, 4096)
    n = t.size
    for val, p in ((-1, 0.3), (0, 0.4), (1, 0.3)):
        frac = (t == val).sum() / n
        assert abs(frac - p) < 4 * np.sqrt(p * (1 - p) / n)


def test_rows_are_independent_of_matrix_size():
    a = synth.trits(3, 2, 40, 300)
    b = synth.trits_rows(3, 2, np.array([7, 39]), 300)
    np.testing.assert_array_equal(a[[7, 39]], b)
    s = synth.scales(3, 3, 40, 3)
    np.testing.assert_array_equal(s[[5]], synth.scales_rows(3, 3, np.array([5]), 3))


def test_scale_range_and_fp16():
    s = synth.scales(1, 1, 512, 40).astype(np.float64)
    assert s.min() >= 0.005 - 1e-6 and s.max() < 0.05 + 1e-5
    assert abs(s.mean() - 0.0275) < 0.001


def test_activation_outliers():
    x = synth.activations(0, 4, 25600).astype(np.float64)
    frac = (np.abs(x) > 6).mean()
    assert 0.006 < frac < 0.011
    np.testing.assert_array_equal(synth.activations(0, 4, 25600), synth.activations(0, 4, 25600))
