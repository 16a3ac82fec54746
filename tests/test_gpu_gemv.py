"""GPU parity: ternary GEMV, fused gate/up + SwiGLU and the integer partials."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from ternary_weight_decode_b200 import synth, tern
from gpu_util import make_matrix, padded_q, to_dev, tolerance

pytestmark = pytest.mark.gpu

FMTS = [tern.TERN_FMT_BASE3, tern.TERN_FMT_2BIT, tern.TERN_FMT_BITPLANE]
SHAPES = [(256, 256), (37, 300), (100, 1280), (33, 5120), (64, 641), (5, 17408), (1, 1), (32, 20)]


def inputs(N, K, M, seed=0):
    w = synth.trits(seed, 0, N, K)
    sw = synth.scales(seed, 1, N, synth.groups(K))
    x = synth.activation_rows([seed * 31 + r for r in range(M)], K)
    q, s = oracle.act_quant(x)
    return w, sw, q, s


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("M", [1, 2, 3, 8, 16])
def test_group_partials_bit_exact(fmt, N, K, M):
    w, sw, q, s = inputs(N, K, M, seed=N + K)
    W = make_matrix(fmt, w, sw)
    G = synth.groups(K)
    P = torch.full((M, N, G), -999, dtype=torch.int32, device="cuda")
    tern.tern_debug_group_partials(W, padded_q(q, ((K + 15) // 16) * 16 + 16), P)
    ref = oracle.group_partials(w, q)
    np.testing.assert_array_equal(P.cpu().numpy().astype(np.int64), ref)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("M", [1, 2, 4, 5, 16])
def test_gemv_within_tolerance(fmt, N, K, M):
    w, sw, q, s = inputs(N, K, M, seed=3 * N + K)
    W = make_matrix(fmt, w, sw)
    ldy = N + 3
    y = torch.full((M, ldy), 123.0, dtype=torch.float32, device="cuda")
    tern.tern_gemv(W, padded_q(q, ((K + 15) // 16) * 16), to_dev(s), y)
    ref = oracle.gemv(w, sw, q, s)
    got = y.cpu().numpy()
    assert np.max(np.abs(got[:, :N] - ref)) <= tolerance(ref)
    assert (got[:, N:] == 123.0).all(), "columns past N must be untouched"


@pytest.mark.parametrize("fmt", FMTS)
def test_gemv_residual_in_place(fmt):
    N, K, M = 300, 5120, 2
    w, sw, q, s = inputs(N, K, M, seed=9)
    W = make_matrix(fmt, w, sw)
    r = np.random.default_rng(0).standard_normal((M, N)).astype(np.float32)
    y = to_dev(r.copy())
    tern.tern_gemv(W, padded_q(q, K), to_dev(s), y, residual=y)
    ref = r.astype(np.float64) + oracle.gemv(w, sw, q, s)
    assert np.max(np.abs(y.cpu().numpy() - ref)) <= tolerance(ref)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K", [(256, 256), (100, 1280), (70, 5120), (8, 17408)])
@pytest.mark.parametrize("M", [1, 4, 16])
def test_gateup_swiglu(fmt, N, K, M):
    wg, wu = synth.trits(5, 4, N, K), synth.trits(5, 6, N, K)
    sg, su = synth.scales(5, 5, N, synth.groups(K)), synth.scales(5, 7, N, synth.groups(K))
    x = synth.activation_rows(range(M), K)
    fw = 128 if K % 128 == 0 else 0
    q, s = oracle.act_quant(x, fwht_block=fw)
    Wg, Wu = make_matrix(fmt, wg, sg), make_matrix(fmt, wu, su)
    h = torch.empty((M, N), dtype=torch.float32, device="cuda")
    tern.tern_gateup_swiglu(Wg, Wu, padded_q(q, ((K + 15) // 16) * 16), to_dev(s), h)
    ref = oracle.gateup_swiglu(wg, sg, wu, su, q, s)
    assert np.max(np.abs(h.cpu().numpy() - ref)) <= tolerance(ref)


def test_single_gemv_golden_file():
    path = os.path.join(os.path.dirname(__file__), "golden", "single_gemv_k256_n256_seed0.json")
    with open(path) as f:
        g = json.load(f)
    K = N = 256
    W = make_matrix(tern.TERN_FMT_BASE3, synth.trits(0, 0, N, K), synth.scales(0, 1, N, 2))
    x = to_dev(synth.activations(0, 1, K))
    q = torch.empty((1, K), dtype=torch.int8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    tern.act_quant_fwht(x, q, s)
    assert q.cpu().numpy()[0].tolist() == g["q"]
    y = torch.empty((1, N), dtype=torch.float32, device="cuda")
    tern.tern_gemv(W, q, s, y)
    ref = np.array(g["y"])
    assert np.max(np.abs(y.cpu().numpy()[0] - ref)) <= tolerance(ref)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K,M", [(7168, 5120, 1), (5120, 17408, 1), (17408, 5120, 4),
                                   (5120, 17408, 16)])
def test_full_size_sampled_rows(fmt, N, K, M):
    """Full 27B-layer shapes: every output row on the GPU, sampled rows on the oracle."""
    seed, stream = 2, 40
    wd = synth.device_trits(seed, stream, N, K)
    W = tern.TernMatrix.empty(fmt, N, K)
    tern.tern_pack(fmt, wd, W)
    del wd
    synth.device_scales(seed, stream + 1, N, synth.groups(K), out=W.scales)
    x = synth.activation_rows(range(500, 500 + M), K)
    q, s = oracle.act_quant(x)
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    tern.tern_gemv(W, padded_q(q, ((K + 15) // 16) * 16), to_dev(s), y)
    got = y.cpu().numpy()
    rows = np.unique(np.concatenate([np.arange(0, 40), np.arange(N - 40, N),
                                     np.random.default_rng(1).integers(0, N, 64)]))
    wr = synth.trits_rows(seed, stream, rows, K)
    sr = synth.scales_rows(seed, stream + 1, rows, synth.groups(K))
    ref = oracle.gemv(wr, sr, q, s)
    assert np.max(np.abs(got[:, rows] - ref)) <= tolerance(ref)
    assert np.isfinite(got).all()
