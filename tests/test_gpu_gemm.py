"""GPU parity of the prefill GEMM (tern_gemm, tcgen05 kind::i8) against the
oracle: element by element at sizes the oracle finishes quickly (several
128 x 128 tiles, ragged edges, garbage past K in q), and on sampled rows and
tokens at the prefill shapes (M = 512 .. 8192, K x N = 5120 x 17408 and
17408 x 5120) in the launch configuration the bench times."""
import numpy as np
import pytest
import torch

import oracle
from ternary_weight_decode_b200 import synth, tern
from gpu_util import make_matrix, padded_q, to_dev, tolerance

pytestmark = pytest.mark.gpu
FMTS = [tern.TERN_FMT_BASE3, tern.TERN_FMT_2BIT, tern.TERN_FMT_BITPLANE]


def quantised(seed, M, K):
    x = synth.activation_rows([seed * 1009 + r for r in range(M)], K)
    return oracle.act_quant(x)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K,M", [(256, 256, 128), (128, 128, 1), (300, 640, 200), (1000, 1280, 384),
                                   (130, 17408, 130), (37, 300, 5), (64, 20, 3), (129, 5120, 257)])
def test_gemm_matches_oracle(fmt, N, K, M):
    w = synth.trits(N + K, 0, N, K)
    sw = synth.scales(N + K, 1, N, synth.groups(K))
    q, s = quantised(N + M, M, K)
    W = make_matrix(fmt, w, sw)
    ldq = ((K + 15) // 16) * 16 + 16
    ldy = N + 5
    y = torch.full((M + 3, ldy), 77.0, dtype=torch.float32, device="cuda")
    tern.tern_gemm(W, padded_q(q, ldq), to_dev(s), y, M=M)
    ref = oracle.gemv(w, sw, q, s)
    got = y.cpu().numpy()
    assert np.max(np.abs(got[:M, :N] - ref)) <= tolerance(ref)
    assert (got[:M, N:] == 77.0).all(), "columns past N must be untouched"
    assert (got[M:] == 77.0).all(), "rows past M must be untouched"
    assert tern.tern_device_error() == 0


@pytest.mark.parametrize("fmt", FMTS)
def test_gemm_repeatable(fmt):
    N, K, M = 384, 1280, 256
    w = synth.trits(5, 0, N, K)
    sw = synth.scales(5, 1, N, synth.groups(K))
    q, s = quantised(6, M, K)
    W = make_matrix(fmt, w, sw)
    qd, sd = padded_q(q, K), to_dev(s)
    y1 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    y2 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    tern.tern_gemm(W, qd, sd, y1)
    tern.tern_gemm(W, qd, sd, y2)
    assert torch.equal(y1, y2)


def big_matrix(fmt, N, K, seed):
    W = tern.TernMatrix.empty(fmt, N, K)
    trits = torch.empty((N, K), dtype=torch.int8, device="cuda")
    synth.device_trits(seed, 0, N, K, out=trits)
    tern.tern_pack(fmt, trits, W)
    synth.device_scales(seed, 1, N, synth.groups(K), out=W.scales)
    del trits
    return W


@pytest.mark.parametrize("fmt,K,N,M", [(tern.TERN_FMT_BASE3, 5120, 17408, 512),
                                       (tern.TERN_FMT_BASE3, 17408, 5120, 512),
                                       (tern.TERN_FMT_2BIT, 5120, 17408, 2048),
                                       (tern.TERN_FMT_BITPLANE, 17408, 5120, 2048),
                                       (tern.TERN_FMT_BASE3, 5120, 17408, 8192)])
def test_gemm_prefill_shapes_sampled(fmt, K, N, M):
    seed = 40 + M
    W = big_matrix(fmt, N, K, seed)
    rng = np.random.default_rng(M + K)
    toks = np.unique(np.concatenate([[0, M - 1], rng.integers(0, M, 6)]))
    rows = np.unique(np.concatenate([[0, N - 1, 127, 128], rng.integers(0, N, 60)]))
    # the tokens the check reads are seeded rows; the others are filler
    # with the same statistics
    q = np.zeros((M, K), np.int8)
    s = np.ones(M, np.float32)
    qt, st = quantised(seed, len(toks), K)
    q[toks] = qt
    s[toks] = st
    filler = [t for t in range(M) if t not in set(toks.tolist())]
    if filler:
        qf, sf = quantised(seed + 1, min(len(filler), 256), K)
        for i, t in enumerate(filler):
            q[t] = qf[i % len(qf)]
            s[t] = sf[i % len(sf)]
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    tern.tern_gemm(W, to_dev(q), to_dev(s), y)
    got = y[torch.from_numpy(toks).cuda()][:, torch.from_numpy(rows).cuda()].cpu().numpy()
    w = synth.trits_rows(seed, 0, rows, K)
    sw = synth.scales_rows(seed, 1, rows, synth.groups(K))
    ref = oracle.gemv(w, sw, q[toks], s[toks])
    assert np.max(np.abs(got - ref)) <= tolerance(ref)
    assert tern.tern_device_error() == 0


# ---------------------------------------------------------------- multi-token verify
@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("N,K,M", [(300, 5120, 17), (512, 17408, 100), (1000, 1280, 64),
                                   (130, 5120, 128), (5120, 640, 65), (2000, 17408, 33)])
def test_verify_sizes_match_oracle(fmt, N, K, M):
    """Token rows 17..128 run on 64- or 128-token tiles, with a cluster split
    of K when the weight-row tiles are few (N = 300, 512, 130: up to 8 ranks)."""
    w = synth.trits(N + 3 * K, 0, N, K)
    sw = synth.scales(N + 3 * K, 1, N, synth.groups(K))
    q, s = quantised(N + 7 * M, M, K)
    W = make_matrix(fmt, w, sw)
    ldq = ((K + 15) // 16) * 16
    y = torch.full((M + 2, N + 3), 77.0, dtype=torch.float32, device="cuda")
    tern.tern_gemm(W, padded_q(q, ldq), to_dev(s), y, M=M)
    ref = oracle.gemv(w, sw, q, s)
    got = y.cpu().numpy()
    assert np.max(np.abs(got[:M, :N] - ref)) <= tolerance(ref)
    assert (got[:M, N:] == 77.0).all() and (got[M:] == 77.0).all()
    # the same launch with its partials: exact integers on every rank
    P = torch.full((M, N, synth.groups(K)), -(1 << 30), dtype=torch.int32, device="cuda")
    y2 = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    tern.tern_debug_gemm_partials(W, padded_q(q, ldq), to_dev(s), y2, P, M=M)
    np.testing.assert_array_equal(P.cpu().numpy(), oracle.group_partials(w, q))
    np.testing.assert_array_equal(y2.cpu().numpy(), got[:M, :N])
    assert tern.tern_device_error() == 0


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("K,N,M", [(5120, 17408, 64), (17408, 5120, 128), (17408, 5120, 24),
                                   (5120, 17408, 4), (17408, 5120, 8)])
def test_verify_full_shapes_sampled(fmt, K, N, M):
    """The 27B-shaped gate/up and down matrices at verify sizes, in the
    launch configuration the bench times, checked on sampled rows."""
    seed = 90 + M
    W = big_matrix(fmt, N, K, seed)
    q, s = quantised(seed, M, K)
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    tern.tern_gemm(W, to_dev(q), to_dev(s), y)
    rng = np.random.default_rng(M)
    rows = np.unique(np.concatenate([[0, N - 1, 127, 128, 4095], rng.integers(0, N, 80)]))
    got = y[:, torch.from_numpy(rows).cuda()].cpu().numpy()
    w = synth.trits_rows(seed, 0, rows, K)
    sw = synth.scales_rows(seed, 1, rows, synth.groups(K))
    ref = oracle.gemv(w, sw, q, s)
    assert np.max(np.abs(got - ref)) <= tolerance(ref)
    assert tern.tern_device_error() == 0
