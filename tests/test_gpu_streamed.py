"""GPU parity of the streamed (persistent, evenly split) GEMV entry points:
outputs match the oracle, repeated calls are identical, and every call
leaves the workspace all zero (it clears the partials it published)."""
import numpy as np
import pytest
import torch

import oracle
from ternary_weight_decode_b200 import synth, tern
from gpu_util import make_matrix, to_dev, tolerance

pytestmark = pytest.mark.gpu
FMTS = [tern.TERN_FMT_BASE3, tern.TERN_FMT_2BIT, tern.TERN_FMT_BITPLANE]
RMS, ROT = tern.TERN_QUANT_RMSNORM, tern.TERN_QUANT_FWHT128


def tiled(fmt, w, sw):
    return make_matrix(fmt, w, sw).retile_scales()


def leftovers(ws):
    """Nonzero words left in the workspace (must be none after a call)."""
    return int(torch.count_nonzero(ws).item())


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K,M,qflags", [(256, 256, 1, 0), (7168, 5120, 1, RMS), (5120, 17408, 1, RMS),
                                          (5120, 5120, 2, ROT), (37, 300, 1, 0), (1000, 1280, 2, RMS | ROT),
                                          (33, 20, 1, 0), (4100, 17408, 2, 0),
                                          # several rounds of input blocks per warp: rotated (K % 128
                                          # == 0), a partial last block, three rounds
                                          (1000, 17408, 1, RMS | ROT), (700, 17407, 2, RMS),
                                          (600, 29952, 1, RMS | ROT), (300, 30001, 2, RMS)])
def test_streamed_gemv_matches_oracle(fmt, N, K, M, qflags):
    w = synth.trits(31, 0, N, K)
    sw = synth.scales(31, 1, N, synth.groups(K))
    W = tiled(fmt, w, sw)
    xh = synth.activation_rows(range(60, 60 + M), K).astype(np.float32) * np.float32(1.3)
    ldx = ((K + 3) // 4) * 4
    xb = np.zeros((M, ldx), np.float32)
    xb[:, :K] = xh
    x = to_dev(xb)
    ws = tern.stream_workspace(fmt, N, M, False)
    outs = []
    for _ in range(2):
        y = torch.full((M, N), 5.0, dtype=torch.float32, device="cuda")
        tern.tern_gemv_streamed(W, x[:, :K] if ldx == K else x, y, ws, qflags=qflags, M=M)
        outs.append(y.cpu().numpy())
    np.testing.assert_array_equal(outs[0], outs[1])
    assert leftovers(ws) == 0, "the workspace must be left zero"
    q, s = oracle.act_quant(xh, fwht_block=128 if qflags & ROT else 0, rmsnorm=bool(qflags & RMS))
    ref = oracle.gemv(w, sw, q, s)
    assert np.max(np.abs(outs[0] - ref)) <= tolerance(ref)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K,M", [(17408, 5120, 1), (17408, 5120, 2), (300, 640, 1),
                                   (600, 12800, 1), (260, 17408, 2)])
def test_streamed_gateup(fmt, N, K, M):
    wg, wu = synth.trits(32, 4, N, K), synth.trits(32, 6, N, K)
    G = synth.groups(K)
    sg, su = synth.scales(32, 5, N, G), synth.scales(32, 7, N, G)
    Wg, Wu = tiled(fmt, wg, sg), tiled(fmt, wu, su)
    xh = synth.activation_rows(range(70, 70 + M), K).astype(np.float32)
    ldx = ((K + 3) // 4) * 4  # rows 16-byte aligned; the columns past K are not read
    xb = np.full((M, ldx), np.nan, np.float32)
    xb[:, :K] = xh
    x = to_dev(xb)[:, :K]
    ws = tern.stream_workspace(fmt, N, M, True)
    h = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    tern.tern_gateup_swiglu_streamed(Wg, Wu, x, h, ws, qflags=RMS | ROT)
    qo, so = oracle.act_quant(xh, fwht_block=128, rmsnorm=True)
    ref = oracle.gateup_swiglu(wg, sg, wu, su, qo, so)
    assert np.max(np.abs(h.cpu().numpy() - ref)) <= tolerance(ref)
    assert leftovers(ws) == 0


@pytest.mark.parametrize("fmt", FMTS)
def test_streamed_residual_in_place_and_strided_input(fmt):
    N, K, M = 5120, 5120, 1
    w = synth.trits(33, 0, N, K)
    sw = synth.scales(33, 1, N, synth.groups(K))
    W = tiled(fmt, w, sw)
    wide = synth.activation_rows([80], 7168).astype(np.float32)
    xw = to_dev(wide)
    r = np.random.default_rng(4).standard_normal((M, N)).astype(np.float32)
    y = to_dev(r.copy())
    ws = tern.stream_workspace(fmt, N, M, False)
    tern.tern_gemv_streamed(W, xw[:, :K], y, ws, qflags=RMS, residual=y)
    q, s = oracle.act_quant(wide[:, :K], rmsnorm=True)
    ref = r.astype(np.float64) + oracle.gemv(w, sw, q, s)
    assert np.max(np.abs(y.cpu().numpy() - ref)) <= tolerance(ref)


def test_retiled_scales_layout():
    fmt, N, K = tern.TERN_FMT_BASE3, 70, 1400
    sw = synth.scales(34, 1, N, synth.groups(K))
    W = make_matrix(fmt, synth.trits(34, 0, N, K), sw).retile_scales()
    t = W.scales_tiled.cpu().numpy()
    SB = -(-(4 * -(-K // 20)) // 128)
    GPS, G = 5, synth.groups(K)
    for u in range(-(-N // 32) * SB):
        rb, sb = divmod(u, SB)
        for r in range(32):
            for g in range(GPS):
                n, gg = rb * 32 + r, sb * GPS + g
                expect = sw[n, gg] if n < N and gg < G else np.float16(0)
                assert t[(u * 32 + r) * GPS + g] == expect


@pytest.mark.parametrize("fmt", FMTS)
def test_one_workspace_serves_calls_of_different_sizes(fmt):
    """A chain QKV -> O -> gate/up -> down on one workspace sized for the
    largest call, as the decode step runs it."""
    rng = np.random.default_rng(9)
    shapes = [(7168, 5120, False), (5120, 5120, False), (17408, 5120, True), (5120, 17408, False)]
    ws = tern.stream_workspace(fmt, 17408, 1, True)
    for N, K, two in shapes * 2:
        w = synth.trits(int(rng.integers(1000)), 0, N, K)
        sw = synth.scales(int(rng.integers(1000)), 1, N, synth.groups(K))
        W = tiled(fmt, w, sw)
        xh = (rng.standard_normal((1, K)) * 2).astype(np.float32)
        y = torch.zeros((1, N), dtype=torch.float32, device="cuda")
        if two:
            tern.tern_gateup_swiglu_streamed(W, W, to_dev(xh), y, ws, qflags=RMS | ROT)
            q, s = oracle.act_quant(xh, fwht_block=128, rmsnorm=True)
            ref = oracle.gateup_swiglu(w, sw, w, sw, q, s)
        else:
            tern.tern_gemv_streamed(W, to_dev(xh), y, ws, qflags=RMS)
            q, s = oracle.act_quant(xh, rmsnorm=True)
            ref = oracle.gemv(w, sw, q, s)
        assert np.max(np.abs(y.cpu().numpy() - ref)) <= tolerance(ref)
    assert leftovers(ws) == 0
