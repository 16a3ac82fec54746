"""tern_gemv_streamed_noalloc: the streamed GEMV for callers that cannot
allocate device memory.

Some callers cannot call cudaMalloc: a plug-in whose host program owns all
device memory through its own pool or budget, or code on a latency-critical
path where cudaMalloc's implicit device-wide synchronisation would stall
other streams.  For them the library keeps the streamed kernel's scratch
(partial sums of the row blocks two CTAs share) in a
fixed 1 MiB array of its own.  These tests check that this entry point gives
the results of tern_gemv_streamed, which takes a caller workspace, on two
calls in a row, and that it rejects sizes whose scratch would not fit.

This file is collected last, so a run that stops at the first failure has
run every other test before it."""
import ctypes

import numpy as np
import pytest
import torch

from ternary_weight_decode_b200 import synth, tern

FMTS = [tern.TERN_FMT_BASE3, tern.TERN_FMT_2BIT]
RMS, ROT = tern.TERN_QUANT_RMSNORM, tern.TERN_QUANT_FWHT128


def _input(seed, M, K):
    x = np.zeros((M, (K + 3) // 4 * 4), np.float32)
    x[:, :K] = synth.activation_rows(range(seed, seed + M), K).astype(np.float32) * np.float32(1.7)
    return torch.from_numpy(x).cuda()


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K,M,qflags", [(5120, 5120, 1, RMS), (4100, 17408, 2, ROT),
                                          (37, 300, 1, 0), (7168, 5120, 2, RMS | ROT)])
def test_noalloc_matches_streamed_on_two_calls(fmt, N, K, M, qflags):
    """Same kernel, same fixed summation order: the results are identical
    bit for bit to tern_gemv_streamed's, and within the oracle's tolerance."""
    import oracle
    from gpu_util import make_matrix, tolerance
    w = synth.trits(77, 0, N, K)
    sw = synth.scales(77, 1, N, synth.groups(K))
    W = make_matrix(fmt, w, sw).retile_scales()
    ws = tern.stream_workspace(fmt, N, M, False)
    for call in range(2):
        x = _input(500 + 10 * call, M, K)
        residual = None
        if call == 1:
            residual = torch.from_numpy(
                synth.activation_rows(range(900, 900 + M), N).astype(np.float32)).cuda()
        y_ref = torch.full((M, N), 3.0, dtype=torch.float32, device="cuda")
        y = torch.full((M, N), -3.0, dtype=torch.float32, device="cuda")
        tern.tern_gemv_streamed(W, x, y_ref, ws, qflags=qflags, residual=residual, M=M)
        tern.tern_gemv_streamed_noalloc(W, x, y, qflags=qflags, residual=residual, M=M)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(y.cpu().numpy(), y_ref.cpu().numpy(), err_msg=f"call {call}")
        if call == 0:
            xh = x.cpu().numpy()[:, :K]
            q, s = oracle.act_quant(xh, fwht_block=128 if qflags & ROT else 0,
                                    rmsnorm=bool(qflags & RMS))
            ref = oracle.gemv(w, sw, q, s)
            assert np.max(np.abs(y.cpu().numpy() - ref)) <= tolerance(ref)
    assert tern.tern_device_error() == 0


@pytest.mark.gpu
def test_noalloc_shared_array_large_then_small_and_mixed():
    """Calls share one array: a large call (N = 129024 at M = 1, the whole
    array) leaves its words cleared, and smaller calls of the other format
    and of M = 2 that follow on the same array still give the workspace
    path's results bit for bit."""
    from gpu_util import make_matrix
    seq = [(tern.TERN_FMT_BASE3, 129024, 640, 1), (tern.TERN_FMT_2BIT, 300, 1280, 2),
           (tern.TERN_FMT_BASE3, 5120, 5120, 2), (tern.TERN_FMT_2BIT, 65024, 512, 2),
           (tern.TERN_FMT_BASE3, 33, 20, 1), (tern.TERN_FMT_2BIT, 7168, 5120, 1)]
    for i, (fmt, N, K, M) in enumerate(seq):
        w = synth.trits(78, i, N, K)
        sw = synth.scales(78, 100 + i, N, synth.groups(K))
        W = make_matrix(fmt, w, sw).retile_scales()
        x = _input(520 + 3 * i, M, K)
        ws = tern.stream_workspace(fmt, N, M, False)
        y_ref = torch.zeros((M, N), dtype=torch.float32, device="cuda")
        y = torch.ones((M, N), dtype=torch.float32, device="cuda")
        tern.tern_gemv_streamed(W, x, y_ref, ws, qflags=RMS, M=M)
        tern.tern_gemv_streamed_noalloc(W, x, y, qflags=RMS, M=M)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(y.cpu().numpy(), y_ref.cpu().numpy(), err_msg=f"call {i}")
        del W, x, ws, y, y_ref
    assert tern.tern_device_error() == 0


@pytest.mark.parametrize("N,M", [(129025, 1), (65025, 2), (1 << 30, 1)])
def test_noalloc_rejects_sizes_beyond_its_scratch(N, M):
    """Needs no GPU: the size check comes before any CUDA call."""
    L = tern.lib()
    m = tern.tern_matrix(fmt=0, N=N, K=256, group=128, row_stride=64, packed=4096, scales=8192,
                         scales_tiled=16384, flags=0, reserved=0)
    st = L.tern_gemv_streamed_noalloc(ctypes.byref(m), ctypes.c_void_p(4096), 256, 0, M, None,
                                      ctypes.c_void_p(4096), N, None)
    assert st == tern.TERN_EINVAL
    assert b"scratch" in L.tern_last_error()
    assert tern.tern_stream_workspace_bytes(0, N, M, False) > tern.NOALLOC_SCRATCH_BYTES
    # the largest accepted size fits
    n_max = 129024 if M == 1 else 65024
    assert tern.tern_stream_workspace_bytes(0, n_max, M, False) <= tern.NOALLOC_SCRATCH_BYTES
