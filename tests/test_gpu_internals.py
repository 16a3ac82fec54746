"""Bit-exact parity of the integer internals of the two hot-path kernels.

The streamed decode kernel quantises its fp32 input itself and takes integer
dot products; the prefill GEMM accumulates integer partials on the tensor
cores.  Both are instantiated here with their debug outputs (the same kernel
code, written to also store what it holds) and compared with the oracle bit
for bit:
  * the int8 input codes and the row scale of the streamed kernel against
    oracle.act_quant (and against the act_quant_fwht entry point);
  * every int32 group partial P[m][n][g] against oracle.group_partials
    (exact integers, so any dropped, doubled or misplaced product shows).
Shapes are the decode projections of the 27B-shaped layer at M = 1 and 2,
where every matrix is cut into ranges over all SMs and row blocks are split
between neighbouring CTAs, plus ragged shapes; and a ragged prefill tile."""
import numpy as np
import pytest
import torch

import oracle
from ternary_weight_decode_b200 import synth, tern
from gpu_util import make_matrix, to_dev, tolerance

pytestmark = pytest.mark.gpu
FMTS = [tern.TERN_FMT_BASE3, tern.TERN_FMT_2BIT, tern.TERN_FMT_BITPLANE]
RMS, ROT = tern.TERN_QUANT_RMSNORM, tern.TERN_QUANT_FWHT128


def _x(seed, M, K, scale=1.0):
    ldx = (K + 3) // 4 * 4
    xb = np.zeros((M, ldx), np.float32)
    xh = synth.activation_rows(range(seed, seed + M), K).astype(np.float32) * np.float32(scale)
    xb[:, :K] = xh
    return xh, to_dev(xb)


def _run_streamed(fmt, ws_list, xh, x, qflags, M):
    """ws_list: [(w, sw)] one or two matrices; returns (out, q, s_x, P)."""
    mats = [make_matrix(fmt, w, sw).retile_scales() for w, sw in ws_list]
    N, K = ws_list[0][0].shape
    G = synth.groups(K)
    nmat = len(mats)
    out = torch.full((M, N), 7.0, dtype=torch.float32, device="cuda")
    q = torch.full((M, K), 99, dtype=torch.int8, device="cuda")
    s = torch.full((M,), -1.0, dtype=torch.float32, device="cuda")
    P = torch.full((nmat, M, N, G), -(1 << 30), dtype=torch.int32, device="cuda")
    ws = tern.stream_workspace(fmt, N, M, nmat == 2)
    tern.tern_debug_streamed(mats[0], mats[1] if nmat == 2 else None, x, out, q, s, P, ws,
                             qflags=qflags, M=M)
    torch.cuda.synchronize()
    assert int(torch.count_nonzero(ws).item()) == 0, "the workspace must be left zero"
    return out.cpu().numpy(), q.cpu().numpy(), s.cpu().numpy(), P.cpu().numpy(), mats


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M", [1, 2])
@pytest.mark.parametrize("name,N,K,qflags", [("qkv", 7168, 5120, RMS), ("o", 5120, 5120, RMS),
                                             ("down", 5120, 17408, RMS), ("ragged", 37, 300, 0),
                                             ("tiny", 33, 20, 0), ("rot_only", 1000, 1280, ROT)])
def test_streamed_codes_and_partials_bit_exact(fmt, M, name, N, K, qflags):
    w = synth.trits(41, 0, N, K)
    sw = synth.scales(41, 1, N, synth.groups(K))
    xh, x = _x(600, M, K, 1.9)
    out, q, s, P, _ = _run_streamed(fmt, [(w, sw)], xh, x, qflags, M)
    q_ref, s_ref = oracle.act_quant(xh, fwht_block=128 if qflags & ROT else 0, rmsnorm=bool(qflags & RMS))
    np.testing.assert_array_equal(q, q_ref)
    if qflags & RMS:
        # the RMS factor: fp32 sum of squares in the kernel, fp64 in the oracle
        np.testing.assert_allclose(s, s_ref, rtol=2e-6, atol=0)
    else:
        np.testing.assert_array_equal(s, s_ref)
    P_ref = oracle.group_partials(w, q_ref)
    np.testing.assert_array_equal(P[0], P_ref)
    y_ref = oracle.gemv(w, sw, q_ref, s_ref)
    assert np.max(np.abs(out - y_ref)) <= tolerance(y_ref)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M", [1, 2])
def test_streamed_gateup_codes_and_partials_bit_exact(fmt, M):
    """The fused gate/up + SwiGLU launch of the 27B-shaped layer with the
    Hadamard rotation and the RMS factor: both matrices' partials."""
    N, K = 17408, 5120
    wg, wu = synth.trits(42, 0, N, K), synth.trits(42, 2, N, K)
    G = synth.groups(K)
    sg, su = synth.scales(42, 1, N, G), synth.scales(42, 3, N, G)
    xh, x = _x(610, M, K)
    h, q, s, P, _ = _run_streamed(fmt, [(wg, sg), (wu, su)], xh, x, RMS | ROT, M)
    q_ref, s_ref = oracle.act_quant(xh, fwht_block=128, rmsnorm=True)
    np.testing.assert_array_equal(q, q_ref)
    np.testing.assert_allclose(s, s_ref, rtol=2e-6, atol=0)
    np.testing.assert_array_equal(P[0], oracle.group_partials(wg, q_ref))
    np.testing.assert_array_equal(P[1], oracle.group_partials(wu, q_ref))
    h_ref = oracle.gateup_swiglu(wg, sg, wu, su, q_ref, s_ref)
    assert np.max(np.abs(h - h_ref)) <= tolerance(h_ref)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("K,qflags", [(5120, RMS | ROT), (17408, 0), (5120, 0), (1280, ROT)])
def test_streamed_codes_equal_act_quant_entry_point(fmt, K, qflags):
    """The streamed kernel's own quantisation gives act_quant_fwht's codes
    bit for bit (and its scale, bit for bit without the RMS factor)."""
    M = 2
    N = 256
    w = synth.trits(43, 0, N, K)
    sw = synth.scales(43, 1, N, synth.groups(K))
    xh, x = _x(620, M, K, 0.7)
    _, q, s, _, _ = _run_streamed(fmt, [(w, sw)], xh, x, qflags, M)
    qa = torch.zeros((M, K), dtype=torch.int8, device="cuda")
    sa = torch.zeros((M,), dtype=torch.float32, device="cuda")
    tern.act_quant_fwht(x, qa, sa, fwht_block=128 if qflags & ROT else 0, K=K,
                        flags=qflags & RMS)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(q, qa.cpu().numpy())
    if not qflags & RMS:
        np.testing.assert_array_equal(s, sa.cpu().numpy())


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,N,K", [(300, 200, 1000), (256, 512, 17408), (17, 130, 5120)])
def test_gemm_partials_bit_exact(fmt, M, N, K):
    """The tensor-core accumulator of the prefill GEMM holds the exact group
    partials: ragged token and weight-row tiles, a partial last group, and
    the down-projection K."""
    w = synth.trits(44, 0, N, K)
    sw = synth.scales(44, 1, N, synth.groups(K))
    W = make_matrix(fmt, w, sw)
    xh = synth.activation_rows(range(700, 700 + M), K).astype(np.float32)
    q, s = oracle.act_quant(xh)
    ldq = (K + 15) // 16 * 16
    qb = np.zeros((M, ldq), np.int8)
    qb[:, :K] = q
    y = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    P = torch.full((M, N, synth.groups(K)), -(1 << 30), dtype=torch.int32, device="cuda")
    tern.tern_debug_gemm_partials(W, to_dev(qb), to_dev(s), y, P, M=M)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(P.cpu().numpy(), oracle.group_partials(w, q))
    ref = oracle.gemv(w, sw, q, s)
    assert np.max(np.abs(y.cpu().numpy() - ref)) <= tolerance(ref)
    assert tern.tern_device_error() == 0


@pytest.mark.parametrize("fmt", [tern.TERN_FMT_2BIT, tern.TERN_FMT_BITPLANE])
def test_streamed_partials_stable_under_ring_reuse(fmt):
    """The 2-bit and bit-plane items hand their ring slot back as soon as the
    codes are in registers, and the producer refills it by TMA at once.  A
    missing proxy fence between the consumers' reads and that refill showed
    as a few wrong partials in about one run of ten; thirty repeats of the
    gate/up launch, every partial of both matrices bit for bit."""
    N, K, M = 17408, 5120, 1
    wg, wu = synth.trits(45, 0, N, K), synth.trits(45, 2, N, K)
    G = synth.groups(K)
    sg, su = synth.scales(45, 1, N, G), synth.scales(45, 3, N, G)
    xh, x = _x(630, M, K)
    q_ref, _ = oracle.act_quant(xh, fwht_block=128, rmsnorm=True)
    Pg, Pu = oracle.group_partials(wg, q_ref), oracle.group_partials(wu, q_ref)
    mats = [make_matrix(fmt, w, sw).retile_scales() for w, sw in ((wg, sg), (wu, su))]
    h = torch.empty((M, N), dtype=torch.float32, device="cuda")
    q = torch.empty((M, K), dtype=torch.int8, device="cuda")
    s = torch.empty((M,), dtype=torch.float32, device="cuda")
    P = torch.empty((2, M, N, G), dtype=torch.int32, device="cuda")
    ws = tern.stream_workspace(fmt, N, M, True)
    for rep in range(30):
        P.fill_(-(1 << 30))
        tern.tern_debug_streamed(mats[0], mats[1], x, h, q, s, P, ws, qflags=RMS | ROT, M=M)
        torch.cuda.synchronize()
        got = P.cpu().numpy()
        assert np.array_equal(got[0], Pg) and np.array_equal(got[1], Pu), f"repeat {rep}"
    assert tern.tern_device_error() == 0
