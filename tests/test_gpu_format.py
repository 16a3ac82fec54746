"""GPU parity: packing, unpacking and the load-time re-tile, bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from ternary_weight_decode_b200 import synth, tern
from gpu_util import to_dev, make_matrix

pytestmark = pytest.mark.gpu

SHAPES = [(1, 1), (3, 5), (7, 19), (9, 20), (5, 21), (33, 127), (40, 300), (17, 641), (64, 5120),
          (8, 17408)]


ALL_FMTS = [tern.TERN_FMT_BASE3, tern.TERN_FMT_2BIT, tern.TERN_FMT_BITPLANE]


def canonical(fmt, w):
    return {tern.TERN_FMT_BASE3: oracle.pack_base3, tern.TERN_FMT_2BIT: oracle.pack_2bit,
            tern.TERN_FMT_BITPLANE: oracle.pack_bitplane}[fmt](w)


@pytest.mark.parametrize("fmt", ALL_FMTS)
@pytest.mark.parametrize("N,K", SHAPES)
def test_pack_matches_oracle_device_layout(fmt, N, K):
    w = synth.trits(11, 2, N, K)
    M = tern.TernMatrix.empty(fmt, N, K)
    M.packed.fill_(0xAB)  # every byte, stride padding included, must be rewritten
    bad = torch.zeros(1, dtype=torch.int32, device="cuda")
    tern.tern_pack(fmt, to_dev(w), M, d_invalid=bad)
    ref = oracle.pack_device(fmt, w, M.row_stride)
    np.testing.assert_array_equal(M.packed.cpu().numpy(), ref)
    assert int(bad.item()) == 0
    out = torch.empty((N, K), dtype=torch.int8, device="cuda")
    tern.tern_unpack(M, out, d_invalid=bad)
    np.testing.assert_array_equal(out.cpu().numpy(), w)
    assert int(bad.item()) == 0


@pytest.mark.parametrize("fmt", ALL_FMTS)
@pytest.mark.parametrize("N,K", SHAPES)
def test_import_export_canonical(fmt, N, K):
    w = synth.trits(12, 4, N, K)
    canon = canonical(fmt, w)
    M = tern.TernMatrix.empty(fmt, N, K)
    bad = torch.zeros(1, dtype=torch.int32, device="cuda")
    tern.tern_import(fmt, to_dev(canon), K, M, d_invalid=bad)
    np.testing.assert_array_equal(M.packed.cpu().numpy(), oracle.pack_device(fmt, w, M.row_stride))
    back = torch.empty(canon.shape, dtype=torch.uint8, device="cuda")
    tern.tern_export(M, back, d_invalid=bad)
    np.testing.assert_array_equal(back.cpu().numpy(), canon)
    assert int(bad.item()) == 0


def test_invalid_codes_are_counted():
    K = 20
    w = np.zeros((1, K), np.int8)
    M = make_matrix(tern.TERN_FMT_BASE3, w, np.ones((1, 1), np.float16))
    invalid = [y for y in range(256) if oracle.d3_decode_value(y) < 0]
    assert len(invalid) == 13
    raw = M.packed.cpu().numpy()
    raw[0, 0] = invalid[0]
    raw[0, 2] = invalid[5]
    M.packed.copy_(torch.from_numpy(raw))
    bad = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty((1, K), dtype=torch.int8, device="cuda")
    tern.tern_unpack(M, out, d_invalid=bad)
    assert int(bad.item()) == 2
    # invalid trits handed to tern_pack are counted too
    w2 = np.array([[0, 1, 2, -1, -3]], np.int8)
    M2 = tern.TernMatrix.empty(tern.TERN_FMT_2BIT, 1, 5)
    bad.zero_()
    tern.tern_pack(tern.TERN_FMT_2BIT, to_dev(w2), M2, d_invalid=bad)
    assert int(bad.item()) == 2
    # canonical base-3 bytes >= 243 are counted by the import
    canon = np.array([[121, 250, 7, 243]], np.uint8)
    M3 = tern.TernMatrix.empty(tern.TERN_FMT_BASE3, 1, 20)
    bad.zero_()
    tern.tern_import(tern.TERN_FMT_BASE3, to_dev(canon), 20, M3, d_invalid=bad)
    assert int(bad.item()) >= 2


def test_device_generator_matches_host():
    N, K = 300, 1000
    for seed, stream in ((0, 0), (5, 17), (63, synth.stream_id(63, synth.PROJ_DOWN))):
        np.testing.assert_array_equal(synth.device_trits(seed, stream, N, K).cpu().numpy(),
                                      synth.trits(seed, stream, N, K))
        np.testing.assert_array_equal(
            synth.device_scales(seed, stream + 1, N, 8).cpu().numpy().view(np.uint16),
            synth.scales(seed, stream + 1, N, 8).view(np.uint16))
    rows = synth.device_trits(3, 9, 4, K, row0=150).cpu().numpy()
    np.testing.assert_array_equal(rows, synth.trits_rows(3, 9, np.arange(150, 154), K))


def test_bitplane_invalid_bits_are_counted():
    """A sign bit without its nonzero bit, in the device layout and in the
    canonical planes, and a nonzero bit past K, are counted and read as 0."""
    K = 40
    w = np.zeros((1, K), np.int8)
    M = tern.TernMatrix.empty(tern.TERN_FMT_BITPLANE, 1, K)
    tern.tern_pack(tern.TERN_FMT_BITPLANE, to_dev(w), M)
    raw = M.packed.cpu().numpy()
    raw[0, 4] |= 1           # sign word of pair 0: position 0 has no nonzero bit
    raw[0, 8 + 3] |= 0x80    # nonzero word of pair 1, bit 31: position 32 + 28 + 3 = 63 >= K
    M.packed.copy_(torch.from_numpy(raw))
    bad = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full((1, K), 9, dtype=torch.int8, device="cuda")
    tern.tern_unpack(M, out, d_invalid=bad)
    assert int(bad.item()) == 2 and not out.cpu().numpy().any()
    canon = oracle.pack_bitplane(w)
    canon[0, 5 + 1] |= 2     # sign plane, position 9, nonzero bit clear
    bad.zero_()
    tern.tern_import(tern.TERN_FMT_BITPLANE, to_dev(canon), K, M, d_invalid=bad)
    assert int(bad.item()) == 1


def test_bitplane_rejected_only_by_the_tensor_core_gemv_engine():
    N, K = 64, 256
    w = synth.trits(13, 0, N, K)
    M = make_matrix(tern.TERN_FMT_BITPLANE, w, synth.scales(13, 1, N, 2))
    q = torch.zeros((1, K), dtype=torch.int8, device="cuda")
    s = torch.ones(1, dtype=torch.float32, device="cuda")
    y = torch.zeros((1, N), dtype=torch.float32, device="cuda")
    tern.tern_debug_select_engine(tern.ENGINE_TENSOR_CORES)
    try:
        with pytest.raises(tern.TernError) as e:
            tern.tern_gemv(M, q, s, y)
        assert e.value.status == tern.TERN_EUNSUPPORTED
    finally:
        tern.tern_debug_select_engine(tern.ENGINE_CUDA_CORES)
    tern.tern_gemv(M, q, s, y)   # the CUDA-core engine and the GEMM take it
    tern.tern_gemm(M, q, s, y)
    torch.cuda.synchronize()
    assert not y.any()
