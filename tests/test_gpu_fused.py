"""GPU parity of the fused-quantisation entry points: the in-kernel
quantisation equals act_quant_fwht bit for bit, and the block statistics a
producer writes equal tern_act_stats of its output."""
import numpy as np
import pytest
import torch

import oracle
from ternary_weight_decode_b200 import synth, tern
from gpu_util import make_matrix, to_dev, tolerance

pytestmark = pytest.mark.gpu
FMTS = [tern.TERN_FMT_BASE3, tern.TERN_FMT_2BIT, tern.TERN_FMT_BITPLANE]
RMS, ROT = tern.TERN_QUANT_RMSNORM, tern.TERN_QUANT_FWHT128


def stats_of(x: torch.Tensor, K=None):
    st = tern.stats_buffer(x.shape[0], x.shape[1] if K is None else K)
    tern.tern_act_stats(x, st, K=K)
    return st


@pytest.mark.parametrize("M,K", [(1, 128), (1, 5120), (3, 300), (16, 17408), (2, 1)])
def test_act_stats_against_oracle(M, K):
    x = (synth.activations(40 + K, M, K).astype(np.float32) * np.float32(0.731))
    ldx = ((K + 3) // 4) * 4
    xb = np.zeros((M, ldx), np.float32)
    xb[:, :K] = x
    st = stats_of(to_dev(xb), K=K).cpu().numpy()
    nb = (K + 127) // 128
    for m in range(M):
        for b in range(nb):
            blk = np.zeros(128, np.float32)
            seg = x[m, 128 * b:128 * (b + 1)]
            blk[:len(seg)] = seg
            assert st[m, b, 0] == np.abs(blk).max()
            assert st[m, b, 1] == np.abs(oracle.fwht128_f32(blk)).max()
            np.testing.assert_allclose(st[m, b, 2], (blk.astype(np.float64) ** 2).sum(), rtol=2e-6)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K,M,qflags", [(256, 256, 1, 0), (300, 1280, 2, ROT), (7168, 5120, 1, 0),
                                          (512, 5120, 4, ROT), (5120, 17408, 1, 0), (96, 300, 3, 0),
                                          (1000, 5120, 16, ROT)])
def test_fused_equals_int8_path_bitwise(fmt, N, K, M, qflags):
    w = synth.trits(7, 0, N, K)
    sw = synth.scales(7, 1, N, synth.groups(K))
    W = make_matrix(fmt, w, sw)
    x = to_dev(synth.activation_rows(range(M), K).astype(np.float32) * np.float32(1.9))
    # int8 path: separate quantisation, then tern_gemv
    ldq = ((K + 15) // 16) * 16
    q = torch.zeros((M, ldq), dtype=torch.int8, device="cuda")
    s = torch.zeros(M, dtype=torch.float32, device="cuda")
    tern.act_quant_fwht(x, q, s, fwht_block=128 if qflags & ROT else 0)
    y_ref = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    tern.tern_gemv(W, q, s, y_ref)
    # fused path
    y = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    ys = tern.stats_buffer(M, N)
    tern.tern_gemv_fused(W, x, stats_of(x), y, qflags=qflags, y_stats=ys)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(y.cpu().numpy(), y_ref.cpu().numpy())
    # the statistics the producer wrote equal those of its output
    np.testing.assert_array_equal(ys.cpu().numpy(), stats_of(y).cpu().numpy())
    # and the result is the oracle's
    qo, so = oracle.act_quant(x.cpu().numpy(), fwht_block=128 if qflags & ROT else 0)
    ref = oracle.gemv(w, sw, qo, so)
    assert np.max(np.abs(y.cpu().numpy() - ref)) <= tolerance(ref)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K,M", [(384, 5120, 1), (17408, 5120, 2), (130, 256, 4)])
def test_fused_gateup_rms_rot(fmt, N, K, M):
    wg, wu = synth.trits(8, 4, N, K), synth.trits(8, 6, N, K)
    G = synth.groups(K)
    sg, su = synth.scales(8, 5, N, G), synth.scales(8, 7, N, G)
    Wg, Wu = make_matrix(fmt, wg, sg), make_matrix(fmt, wu, su)
    xh = synth.activation_rows(range(10, 10 + M), K).astype(np.float32) * np.float32(3.0)
    x = to_dev(xh)
    ldh = ((N + 3) // 4) * 4  # rows 16-byte aligned so h can feed a fused call
    h = torch.zeros((M, ldh), dtype=torch.float32, device="cuda")
    hs = tern.stats_buffer(M, N)
    tern.tern_gateup_swiglu_fused(Wg, Wu, x, stats_of(x), h, qflags=RMS | ROT, h_stats=hs)
    qo, so = oracle.act_quant(xh, fwht_block=128, rmsnorm=True)
    ref = oracle.gateup_swiglu(wg, sg, wu, su, qo, so)
    got = h.cpu().numpy()[:, :N]
    assert np.max(np.abs(got - ref)) <= tolerance(ref)
    np.testing.assert_array_equal(hs.cpu().numpy(), stats_of(h, K=N).cpu().numpy())


@pytest.mark.parametrize("fmt", FMTS)
def test_fused_residual_and_strided_input(fmt):
    # the O projection of the decode layer: x is the first 5120 columns of a
    # 7168-wide buffer, the output accumulates into the residual stream
    N, K, M = 5120, 5120, 2
    w = synth.trits(9, 0, N, K)
    G = synth.groups(K)
    sw = synth.scales(9, 1, N, G)
    W = make_matrix(fmt, w, sw)
    wide = synth.activation_rows(range(20, 20 + M), 7168).astype(np.float32)
    xw = to_dev(wide)
    st = stats_of(xw)
    r = np.random.default_rng(3).standard_normal((M, N)).astype(np.float32)
    y = to_dev(r.copy())
    tern.tern_gemv_fused(W, xw[:, :K], st, y, qflags=RMS, residual=y)
    qo, so = oracle.act_quant(wide[:, :K], rmsnorm=True)
    ref = r.astype(np.float64) + oracle.gemv(w, sw, qo, so)
    assert np.max(np.abs(y.cpu().numpy() - ref)) <= tolerance(ref)
