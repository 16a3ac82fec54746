"""GPU parity: act_quant_fwht against the oracle, bit for bit (q and s_x)."""
import numpy as np
import pytest
import torch

import oracle
from ternary_weight_decode_b200 import synth, tern
from gpu_util import to_dev

pytestmark = pytest.mark.gpu


def run_quant(x: np.ndarray, fwht: int, ldq: int | None = None, flags: int = 0):
    M, K = x.shape
    ldq = ldq or ((K + 15) // 16) * 16
    # rows padded to a 16-byte multiple, as the ABI requires
    ldx = ((K + 7) // 8) * 8
    xb = np.zeros((M, ldx), x.dtype)
    xb[:, :K] = x
    q = torch.full((M, ldq), 55, dtype=torch.int8, device="cuda")
    s = torch.empty(M, dtype=torch.float32, device="cuda")
    tern.act_quant_fwht(to_dev(xb), q, s, fwht_block=fwht, K=K, flags=flags)
    return q.cpu().numpy(), s.cpu().numpy()


@pytest.mark.parametrize("dtype", [np.float16, np.float32])
@pytest.mark.parametrize("M,K,fwht", [(1, 256, 0), (1, 256, 128), (1, 5120, 0), (1, 5120, 128),
                                      (3, 300, 0), (16, 17408, 0), (16, 5120, 128), (2, 17408, 128),
                                      (5, 1, 0), (4, 129, 0)])
def test_quant_bit_exact(dtype, M, K, fwht):
    x = synth.activations(100 + M + K, M, K).astype(dtype)
    if dtype == np.float32:
        x = x * np.float32(1.37)  # values that are not fp16-representable
    q, s = run_quant(x, fwht, ldq=((K + 15) // 16) * 16 + 32)
    qr, sr = oracle.act_quant(x, fwht_block=fwht)
    np.testing.assert_array_equal(q[:, :K], qr)
    assert not q[:, K:].any(), "bytes past K must be zero"
    np.testing.assert_array_equal(s.view(np.uint32), sr.view(np.uint32))


def test_quant_zero_and_constant_rows():
    x = np.zeros((3, 640), np.float32)
    x[1, :] = -2.5
    x[2, 7] = 1e-30
    q, s = run_quant(x, 0)
    qr, sr = oracle.act_quant(x)
    np.testing.assert_array_equal(q[:, :640], qr)
    np.testing.assert_array_equal(s, sr)
    assert s[0] == 0 and not q[0].any()


def test_quant_fwht_rotates_before_amax():
    # one spike per block: the rotation spreads it evenly, so every |q| = 127
    x = np.zeros((1, 256), np.float32)
    x[0, 3] = 4.0
    x[0, 200] = -4.0
    q, s = run_quant(x, 128)
    assert (np.abs(q[0, :256]) == 127).all()
    np.testing.assert_allclose(s[0], 4.0 / 127 / np.sqrt(128), rtol=1e-6)


@pytest.mark.parametrize("fwht", [0, 128])
def test_quant_rmsnorm_folds_into_scale_only(fwht):
    x = synth.activations(77, 4, 5120).astype(np.float32) * np.float32(3.0)
    q0, s0 = run_quant(x, fwht)
    q1, s1 = run_quant(x, fwht, flags=tern.TERN_QUANT_RMSNORM)
    np.testing.assert_array_equal(q0, q1)
    qr, sr = oracle.act_quant(x, fwht_block=fwht, rmsnorm=True)
    np.testing.assert_array_equal(q1[:, :5120], qr)
    np.testing.assert_allclose(s1, sr, rtol=2e-6)
