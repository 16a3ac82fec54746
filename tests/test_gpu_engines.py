"""The tensor-core (tcgen05) and CUDA-core (dp4a) GEMV engines compute the
same integer group partials and accumulate them in the same order, so their
outputs agree bit for bit; both match the oracle."""
import numpy as np
import pytest
import torch

import oracle
from ternary_weight_decode_b200 import synth, tern
from gpu_util import make_matrix, padded_q, to_dev, tolerance

pytestmark = pytest.mark.gpu
FMTS = [tern.TERN_FMT_BASE3, tern.TERN_FMT_2BIT]


@pytest.fixture(autouse=True)
def restore_engine():
    yield
    tern.tern_debug_select_engine(tern.ENGINE_CUDA_CORES)


def run_both(fn):
    outs = []
    for eng in (tern.ENGINE_TENSOR_CORES, tern.ENGINE_CUDA_CORES):
        tern.tern_debug_select_engine(eng)
        outs.append(fn())
    torch.cuda.synchronize()
    return [o.cpu().numpy() for o in outs]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K", [(256, 256), (7168, 5120), (5120, 17408), (37, 300), (130, 1280),
                                 (1, 20)])
@pytest.mark.parametrize("M", [1, 2, 3, 8, 16])
def test_gemv_engines_agree(fmt, N, K, M):
    w = synth.trits(21, 0, N, K)
    sw = synth.scales(21, 1, N, synth.groups(K))
    W = make_matrix(fmt, w, sw)
    x = synth.activation_rows(range(M), K)
    q, s = oracle.act_quant(x)
    qd, sd = padded_q(q, ((K + 15) // 16) * 16), to_dev(s)

    def one():
        y = torch.full((M, N), 7.0, dtype=torch.float32, device="cuda")
        tern.tern_gemv(W, qd, sd, y)
        return y
    y_tc, y_cc = run_both(one)
    np.testing.assert_array_equal(y_tc, y_cc)
    ref = oracle.gemv(w, sw, q, s)
    assert np.max(np.abs(y_tc - ref)) <= tolerance(ref)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K,M", [(17408, 5120, 1), (384, 5120, 4), (300, 1280, 16)])
def test_fused_gateup_engines_agree(fmt, N, K, M):
    wg, wu = synth.trits(22, 4, N, K), synth.trits(22, 6, N, K)
    G = synth.groups(K)
    sg, su = synth.scales(22, 5, N, G), synth.scales(22, 7, N, G)
    Wg, Wu = make_matrix(fmt, wg, sg), make_matrix(fmt, wu, su)
    xh = synth.activation_rows(range(40, 40 + M), K).astype(np.float32)
    x = to_dev(xh)
    st = tern.stats_buffer(M, K)
    tern.tern_act_stats(x, st)
    flags = tern.TERN_QUANT_FWHT128 | tern.TERN_QUANT_RMSNORM

    def one():
        h = torch.zeros((M, N), dtype=torch.float32, device="cuda")
        tern.tern_gateup_swiglu_fused(Wg, Wu, x, st, h, qflags=flags)
        return h
    h_tc, h_cc = run_both(one)
    np.testing.assert_array_equal(h_tc, h_cc)
    qo, so = oracle.act_quant(xh, fwht_block=128, rmsnorm=True)
    ref = oracle.gateup_swiglu(wg, sg, wu, su, qo, so)
    assert np.max(np.abs(h_tc - ref)) <= tolerance(ref)
