"""The stored single-GEMV golden file still matches the oracle (regression pin)."""
import json
import os

import numpy as np

import oracle
from ternary_weight_decode_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "single_gemv_k256_n256_seed0.json")


def test_single_gemv_golden_matches_oracle():
    with open(GOLDEN) as f:
        g = json.load(f)
    K = N = 256
    w = synth.trits(0, 0, N, K)
    assert oracle.pack_base3(w).tobytes().hex() == g["canonical_base3_hex"]
    q, s = oracle.act_quant(synth.activations(0, 1, K))
    assert q[0].tolist() == g["q"]
    assert np.float32(s[0]).tobytes().hex() == g["s_x_hex"]
    y = oracle.gemv(w, synth.scales(0, 1, N, 2), q, s)
    np.testing.assert_array_equal(y[0], np.array(g["y"]))
