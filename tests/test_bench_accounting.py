"""The bench's byte accounting and its reference arm, on the CPU.

The roofline's "achieved" figure divides the algorithmic bytes of a launch
by its time, so the bench's row-byte rule is checked here against the
lengths of the rows the oracle's canonical packers actually produce, for
every format, and the per-layer and per-step totals against the figures
the documentation quotes.  The reference arm (the oracle timed on the
host) must print one JSON line with the contract's keys."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.mark.parametrize("K", [1, 4, 5, 19, 20, 127, 128, 129, 640, 5120, 7168, 17408, 17407])
def test_row_bytes_equal_the_oracle_packers(K):
    rng = np.random.default_rng(K)
    w = rng.integers(-1, 2, size=(3, K)).astype(np.int8)
    packers = {0: oracle.pack_base3, 1: oracle.pack_2bit, 2: oracle.pack_bitplane}
    for fmt, pack in packers.items():
        assert bench.canonical_row_bytes(fmt, K) == pack(w).shape[1], (fmt, K)
    assert bench.canonical_row_bytes(0, K) == oracle.base3_row_bytes(K)
    assert bench.canonical_row_bytes(1, K) == oracle.twobit_row_bytes(K)
    assert bench.canonical_row_bytes(2, K) == oracle.bitplane_row_bytes(K)


def test_layer_and_step_bytes():
    # codes + fp16 scales of QKV (7168 x 5120), O (5120 x 5120), gate and up
    # (17408 x 5120) and down (5120 x 17408)
    assert bench.layer_bytes(0) == 71_223_296
    assert bench.layer_bytes(1) == bench.layer_bytes(2) == 87_736_320
    assert 64 * bench.layer_bytes(0) == 4_558_290_944
    assert 2 * bench.mat_bytes(0, bench.FFN, bench.HIDDEN) == 38_436_864   # the gate/up launch
    assert 2 * bench.mat_bytes(1, bench.FFN, bench.HIDDEN) == 47_349_760
    scales = 2 * bench.FFN * oracle.groups(bench.HIDDEN)
    assert bench.mat_bytes(0, bench.FFN, bench.HIDDEN) == bench.FFN * oracle.base3_row_bytes(bench.HIDDEN) + scales


def test_reference_arm_prints_the_contract_line():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "3",
                        "--warmup", "3"], capture_output=True, text=True, timeout=900, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 3
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert "workload" in line["config"]
