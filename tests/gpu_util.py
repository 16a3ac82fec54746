"""Helpers for the GPU parity tests: move seeded inputs to the device."""
import numpy as np
import torch

from ternary_weight_decode_b200 import synth, tern


def to_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def make_matrix(fmt: int, w: np.ndarray, sw: np.ndarray) -> tern.TernMatrix:
    """Packs host trits with the CUDA tern_pack into a fresh device matrix."""
    N, K = w.shape
    M = tern.TernMatrix.empty(fmt, N, K)
    tern.tern_pack(fmt, to_dev(w.astype(np.int8)), M)
    M.scales.copy_(to_dev(sw.astype(np.float16)))
    return M


def padded_q(q: np.ndarray, ldq: int) -> torch.Tensor:
    M, K = q.shape
    buf = np.zeros((M, ldq), np.int8)
    buf[:, :K] = q
    # garbage past K must be ignored by the kernels
    buf[:, K:] = 77
    return to_dev(buf)


def tolerance(ref: np.ndarray) -> float:
    return 1e-3 * float(np.abs(ref).max()) + 1e-5
