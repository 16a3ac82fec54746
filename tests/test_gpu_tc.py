"""The tcgen05 int8 MMA encodings (instruction and shared-memory descriptors,
tensor-memory operand layout) against a plain integer product."""
import numpy as np
import pytest
import torch

from ternary_weight_decode_b200 import tern
from gpu_util import to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("a_in_smem", [False, True])
@pytest.mark.parametrize("K,N", [(32, 16), (64, 16), (256, 32), (512, 16), (128, 64)])
@pytest.mark.parametrize("a_signed,b_signed", [(True, True), (False, True)])
def test_mma_i8_matches_integer_product(a_in_smem, K, N, a_signed, b_signed):
    rng = np.random.default_rng(K + N)
    lo = -128 if a_signed else 0
    A = rng.integers(lo, 128 if a_signed else 256, (128, K)).astype(np.uint8 if not a_signed else np.int8)
    B = rng.integers(-128, 128, (N, K)).astype(np.int8)
    D = torch.zeros((128, N), dtype=torch.int32, device="cuda")
    Ad = to_dev(A.view(np.int8))
    tern.tern_debug_mma_i8(Ad, to_dev(B), D, a_in_smem=a_in_smem, a_signed=a_signed, b_signed=b_signed)
    ref = A.astype(np.int64) @ B.astype(np.int64).T
    np.testing.assert_array_equal(D.cpu().numpy().astype(np.int64), ref)
    assert tern.tern_device_error() == 0


@pytest.mark.parametrize("K,N", [(128, 16), (128, 128), (256, 64), (512, 32), (384, 256)])
@pytest.mark.parametrize("a_signed", [True, False])
def test_mma_i8_swizzled_operands(K, N, a_signed):
    """Both operands in the 128-byte-swizzled K-major layout of the prefill GEMM."""
    rng = np.random.default_rng(7 * K + N)
    A = rng.integers(-128 if a_signed else 0, 128 if a_signed else 256, (128, K))
    A = A.astype(np.int8 if a_signed else np.uint8)
    B = rng.integers(-128, 128, (N, K)).astype(np.int8)
    D = torch.zeros((128, N), dtype=torch.int32, device="cuda")
    tern.tern_debug_mma_i8(to_dev(A.view(np.int8)), to_dev(B), D, a_in_smem=2, a_signed=a_signed)
    ref = A.astype(np.int64) @ B.astype(np.int64).T
    np.testing.assert_array_equal(D.cpu().numpy().astype(np.int64), ref)
    assert tern.tern_device_error() == 0
