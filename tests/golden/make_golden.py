"""Writes tests/golden/single_gemv_k256_n256_seed0.json from the CPU oracle.

Calls only ``oracle`` and the seeded generator; never the CUDA path.
Workload: K = 256, N = 256, M = 1, trits (seed 0, stream 0), fp16 scales
(seed 0, stream 1), fp16 activations (seed 0), no Hadamard rotation.
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from ternary_weight_decode_b200 import synth  # noqa: E402


def main():
    K = N = 256
    w = synth.trits(0, 0, N, K)
    sw = synth.scales(0, 1, N, synth.groups(K))
    x = synth.activations(0, 1, K)
    q, s = oracle.act_quant(x)
    y = oracle.gemv(w, sw, q, s)
    P = oracle.group_partials(w, q)
    out = {
        "workload": "single ternary GEMV K=256 N=256 M=1 seed 0 (trits stream 0, scales stream 1, activations seed 0)",
        "written_by": "tests/golden/make_golden.py (CPU oracle only)",
        "canonical_base3_hex": oracle.pack_base3(w).tobytes().hex(),
        "q": q[0].tolist(),
        "s_x_hex": np.float32(s[0]).tobytes().hex(),
        "partials_checksum": int((P.astype(np.int64) * np.arange(1, P.size + 1).reshape(P.shape)).sum()),
        "y": [float(v) for v in y[0]],
    }
    path = os.path.join(HERE, "single_gemv_k256_n256_seed0.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=0)
    print(path)


if __name__ == "__main__":
    main()
