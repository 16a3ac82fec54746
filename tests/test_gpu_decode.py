"""GPU parity of the decode step at the full 27B layer shapes.

The step runs as bench.py runs it (same kernels, same launch configuration;
eager here so that every projection's fp32 input can be recorded).  For
sampled layers and sampled output rows, the oracle quantises the recorded
input itself and computes those rows; the GPU output must match within the
tolerance.  Every layer's int8 decision is checked too, through the
statistics chain (each fused call's output statistics feed the next call).
"""
import numpy as np
import pytest
import torch

import oracle
from ternary_weight_decode_b200 import decode, synth, tern
from gpu_util import tolerance

pytestmark = pytest.mark.gpu

H, Q, F = decode.HIDDEN, decode.QKV, decode.FFN


def oracle_rows(layer, proj, N, K, rows, q, s):
    st = synth.stream_id(layer, proj)
    w = synth.trits_rows(layer, st, rows, K)
    sw = synth.scales_rows(layer, st + 1, rows, (K + 127) // 128)
    return oracle.gemv(w, sw, q, s)


def check_layer(rec, l, rng, nrows=48):
    qkv_in = rec[4 * l][1].cpu().numpy()
    qkv_out, x_before_o = (t.cpu().numpy() for t in rec[4 * l + 1][1:])
    x_after_o = rec[4 * l + 2][1].cpu().numpy()
    h, x_before_down = (t.cpu().numpy() for t in rec[4 * l + 3][1:])
    x_after_down = rec[4 * l + 4][1].cpu().numpy() if 4 * l + 4 < len(rec) else None

    def rows(N):
        return np.unique(np.concatenate([[0, N - 1], rng.integers(0, N, nrows)]))

    q, s = oracle.act_quant(qkv_in, rmsnorm=True)
    r = rows(Q)
    ref = oracle_rows(l, synth.PROJ_QKV, Q, H, r, q, s)
    assert np.max(np.abs(qkv_out[:, r] - ref)) <= tolerance(ref)

    q, s = oracle.act_quant(qkv_out[:, :H], rmsnorm=True)
    r = rows(H)
    ref = x_before_o[:, r] + oracle_rows(l, synth.PROJ_O, H, H, r, q, s)
    assert np.max(np.abs(x_after_o[:, r] - ref)) <= tolerance(ref)

    q, s = oracle.act_quant(x_after_o, fwht_block=128, rmsnorm=True)
    r = rows(F)
    st = synth.stream_id(l, synth.PROJ_GATE)
    su = synth.stream_id(l, synth.PROJ_UP)
    G = H // 128
    ref = oracle.gateup_swiglu(synth.trits_rows(l, st, r, H), synth.scales_rows(l, st + 1, r, G),
                               synth.trits_rows(l, su, r, H), synth.scales_rows(l, su + 1, r, G),
                               q, s)
    assert np.max(np.abs(h[:, r] - ref)) <= tolerance(ref)

    if x_after_down is not None:
        q, s = oracle.act_quant(h, rmsnorm=True)
        r = rows(H)
        ref = x_before_down[:, r] + oracle_rows(l, synth.PROJ_DOWN, H, F, r, q, s)
        assert np.max(np.abs(x_after_down[:, r] - ref)) <= tolerance(ref)


@pytest.mark.parametrize("fmt", [tern.TERN_FMT_BASE3, tern.TERN_FMT_2BIT, tern.TERN_FMT_BITPLANE])
@pytest.mark.parametrize("mode", ["streamed", "fused"])
def test_decode_step_64_layers_sampled(fmt, mode):
    model = decode.DecodeModel(fmt, 64, M=1, mode=mode).build(seed_base=0)
    model.x.copy_(torch.from_numpy(synth.activations(0, 1, H).astype(np.float32)))
    rec = []
    model.step(keep=rec)
    rec.append(("qkv_in", model.x.clone()))  # the step output closes the last layer
    torch.cuda.synchronize()
    assert len(rec) == 4 * 64 + 1
    rng = np.random.default_rng(5)
    for l in (0, 1, 17, 40, 63):
        check_layer(rec, l, rng)
    assert np.isfinite(model.x.cpu().numpy()).all()
    assert tern.tern_device_error() == 0


@pytest.mark.parametrize("fmt", [tern.TERN_FMT_BASE3, tern.TERN_FMT_BITPLANE])
@pytest.mark.parametrize("M", [2, 4, 16])
def test_decode_layers_multi_slot(fmt, M):
    mode = "streamed" if M <= 2 else "fused"
    model = decode.DecodeModel(fmt, 2, M=M, mode=mode).build(seed_base=0)
    x0 = synth.activation_rows([1000 + r for r in range(M)], H).astype(np.float32)
    model.x.copy_(torch.from_numpy(x0))
    rec = []
    model.step(keep=rec)
    rec.append(("qkv_in", model.x.clone()))
    torch.cuda.synchronize()
    rng = np.random.default_rng(6)
    for l in (0, 1):
        check_layer(rec, l, rng, nrows=24)


@pytest.mark.parametrize("mode", ["streamed", "fused"])
def test_graph_replay_matches_eager(mode):
    model = decode.DecodeModel(tern.TERN_FMT_BASE3, 3, M=1, mode=mode).build(seed_base=0)
    x0 = torch.from_numpy(synth.activations(3, 1, H).astype(np.float32)).cuda()
    model.x.copy_(x0)
    model.step()
    eager = model.x.clone()
    g = model.capture()
    model.x.copy_(x0)
    g.replay()
    torch.cuda.synchronize()
    np.testing.assert_array_equal(model.x.cpu().numpy(), eager.cpu().numpy())
