"""GPU parity of tern_ternarize with the oracle: the trits and the fp16
group scales bit for bit (the integer decisions are taken in the fp32
arithmetic the definition fixes), then the ternarised matrix through
tern_pack and the streamed GEMV against the oracle's product."""
import numpy as np
import pytest
import torch

import oracle
from ternary_weight_decode_b200 import synth, tern
from gpu_util import to_dev, tolerance

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,K", [(37, 300), (256, 5120), (5, 20), (64, 17408), (9, 128), (300, 1)])
def test_ternarize_matches_oracle_bit_for_bit(N, K):
    w = synth.float_weights(90 + N, N, K)
    ldw = K + 3  # a row stride wider than K
    wb = np.zeros((N, ldw), np.float32)
    wb[:, :K] = w
    wb[:, K:] = np.nan  # never read
    t = torch.full((N, K), 5, dtype=torch.int8, device="cuda")
    s = torch.zeros((N, synth.groups(K)), dtype=torch.float16, device="cuda")
    tern.tern_ternarize(to_dev(wb), t, s, K=K)
    torch.cuda.synchronize()
    t_ref, s_ref = oracle.ternarize(w)
    np.testing.assert_array_equal(t.cpu().numpy(), t_ref)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint16), s_ref.view(np.uint16))


@pytest.mark.parametrize("fmt", [tern.TERN_FMT_BASE3, tern.TERN_FMT_2BIT])
def test_ternarized_matrix_through_the_decode_kernel(fmt):
    N, K = 1000, 5120
    w = synth.float_weights(7, N, K)
    wd = to_dev(w)
    W = tern.TernMatrix.empty(fmt, N, K)
    t = torch.empty((N, K), dtype=torch.int8, device="cuda")
    tern.tern_ternarize(wd, t, W.scales)
    tern.tern_pack(fmt, t, W)
    W.retile_scales()
    xh = synth.activation_rows([33], K).astype(np.float32)
    y = torch.zeros((1, N), dtype=torch.float32, device="cuda")
    ws = tern.stream_workspace(fmt, N, 1, False)
    tern.tern_gemv_streamed(W, to_dev(xh), y, ws, qflags=tern.TERN_QUANT_RMSNORM)
    t_ref, s_ref = oracle.ternarize(w)
    q, sx = oracle.act_quant(xh, rmsnorm=True)
    ref = oracle.gemv(t_ref, s_ref, q, sx)
    assert np.max(np.abs(y.cpu().numpy() - ref)) <= tolerance(ref)
    # and the ternarised product approximates the float one
    dense = (xh.astype(np.float64) @ w.astype(np.float64).T)
    rms = np.sqrt(np.mean(xh.astype(np.float64) ** 2) + 1e-6)  # folded into s_x by RMSNORM
    rel = np.linalg.norm(y.cpu().numpy() * rms - dense) / np.linalg.norm(dense)
    assert rel < 0.6  # about 0.5 for Gaussian weights at the residual-optimal cut
