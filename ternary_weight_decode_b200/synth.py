"""Seeded synthetic inputs for the ternary weight path.

This module holds input generation only: no packing, quantisation or
dot-product arithmetic lives here.  Both the CUDA path and the CPU oracle
consume what it produces.

Weights and scales come from a counter-based generator so that any single
row can be regenerated on its own, on the host or on the device:

* ``mix64`` is the SplitMix64 output function (Steele, Lea & Flood,
  "Fast splittable pseudorandom number generators", OOPSLA 2014; the
  public-domain reference code by S. Vigna).
* ``h(seed, stream, idx)`` is the ``idx``-th output (0-based) of SplitMix64
  whose state starts at ``key = mix64(seed * GAMMA + stream)``, i.e.
  ``mix64(key + (idx + 1) * GAMMA)`` modulo 2**64.

A trit is drawn from ``u = h >> 32``: -1 when ``u < T_NEG``, +1 when
``u >= T_POS``, else 0 (P(-1) = P(+1) = 0.3, P(0) = 0.4, the distribution
of the single-GEMV workload).  A group scale is drawn from ``u24 = h >> 40``
as ``fp16(fp32(fp32(u24 * 2**-24) * 0.045) + 0.005)`` with every fp32 step
rounded to nearest, giving scales in [0.005, 0.05).

The device generator in ``synth_csrc/tern_synth.cu`` implements the same definition;
a GPU test checks the two bit for bit.

Activations are drawn on the host with numpy's PCG64: N(0, 1), 1% of the
entries (``rng.random() < 0.01``) multiplied by 20, stored as fp16.
"""
from __future__ import annotations

import numpy as np

GAMMA = 0x9E3779B97F4A7C15
MASK64 = (1 << 64) - 1
T_NEG = 1288490189  # ceil(0.3 * 2**32)
T_POS = 3006477108  # ceil(0.7 * 2**32)

# Stream ids: projection p of layer l draws its trits from stream_id(l, p)
# and its scales from stream_id(l, p, scales=True).
PROJ_QKV, PROJ_O, PROJ_GATE, PROJ_UP, PROJ_DOWN = 0, 1, 2, 3, 4


def stream_id(layer: int, proj: int, scales: bool = False) -> int:
    return (layer * 16 + proj * 2 + (1 if scales else 0)) & MASK64


def mix64_int(z: int) -> int:
    """SplitMix64 output function on a Python int (mod 2**64)."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, stream: int) -> int:
    return mix64_int(((seed * GAMMA) + stream) & MASK64)


def _mix64_np(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.uint64, copy=True)
    z ^= z >> np.uint64(30)
    z *= np.uint64(0xBF58476D1CE4E5B9)
    z ^= z >> np.uint64(27)
    z *= np.uint64(0x94D049BB133111EB)
    z ^= z >> np.uint64(31)
    return z


def hash_at(seed: int, stream: int, idx: np.ndarray) -> np.ndarray:
    """h(seed, stream, idx) for an array of uint64 counters."""
    key = np.uint64(stream_key(seed, stream))
    idx = np.asarray(idx, dtype=np.uint64)
    with np.errstate(over="ignore"):
        x = key + (idx + np.uint64(1)) * np.uint64(GAMMA)
    return _mix64_np(x)


def trits_rows(seed: int, stream: int, rows: np.ndarray, K: int) -> np.ndarray:
    """Trits int8 [len(rows), K] of the matrix (seed, stream) at the given rows:
    h(seed, stream, row * K + col) as hash_at defines it, evaluated a few rows
    at a time with in-place numpy steps (the same bits, without full-size
    temporaries)."""
    rows = np.asarray(rows, dtype=np.uint64).ravel()
    out = np.empty((rows.size, K), np.int8)
    key = np.uint64(stream_key(seed, stream))
    col1 = np.arange(1, K + 1, dtype=np.uint64).reshape(1, -1)  # idx + 1
    chunk = max(1, (1 << 18) // max(K, 1))
    c1, c2 = np.uint64(0xBF58476D1CE4E5B9), np.uint64(0x94D049BB133111EB)
    tn, tp = np.uint64(T_NEG), np.uint64(T_POS)
    with np.errstate(over="ignore"):
        for r0 in range(0, rows.size, chunk):
            z = rows[r0:r0 + chunk].reshape(-1, 1) * np.uint64(K) + col1
            z *= np.uint64(GAMMA)
            z += key
            t = z >> np.uint64(30)
            z ^= t
            z *= c1
            np.right_shift(z, np.uint64(27), out=t)
            z ^= t
            z *= c2
            np.right_shift(z, np.uint64(31), out=t)
            z ^= t
            z >>= np.uint64(32)
            o = out[r0:r0 + chunk]
            np.greater_equal(z, tp, out=o, casting="unsafe")  # +1
            o -= (z < tn)                                        # -1
    return out


def trits(seed: int, stream: int, N: int, K: int) -> np.ndarray:
    """Trits int8 [N, K] in {-1, 0, +1}."""
    return trits_rows(seed, stream, np.arange(N), K)


def scales_rows(seed: int, stream: int, rows: np.ndarray, G: int) -> np.ndarray:
    """fp16 group scales [len(rows), G] as numpy float16."""
    rows = np.asarray(rows, dtype=np.uint64).reshape(-1, 1)
    idx = rows * np.uint64(G) + np.arange(G, dtype=np.uint64).reshape(1, -1)
    u24 = (hash_at(seed, stream, idx) >> np.uint64(40)).astype(np.float32)
    a = u24 * np.float32(2.0 ** -24)  # exact: u24 < 2**24
    b = a * np.float32(0.045)
    c = b + np.float32(0.005)
    return c.astype(np.float16)


def scales(seed: int, stream: int, N: int, G: int) -> np.ndarray:
    return scales_rows(seed, stream, np.arange(N), G)


def activations(seed: int, M: int, K: int) -> np.ndarray:
    """fp16 activations [M, K]: N(0,1) with 1% of entries scaled by 20."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(M * K)
    mask = rng.random(M * K) < 0.01
    x[mask] *= 20.0
    return x.astype(np.float16).reshape(M, K)


def activation_rows(seeds, K: int) -> np.ndarray:
    """One independently seeded fp16 row per seed (multi-slot decode rows)."""
    return np.concatenate([activations(int(s), 1, K) for s in seeds], axis=0)


def float_weights(seed: int, N: int, K: int) -> np.ndarray:
    """fp32 weights [N, K] for the ternariser: N(0, 0.02) with 1% of the
    entries x10, every 7th row rounded to a coarse grid (repeated magnitudes,
    so that ties occur), and row 3 (when present) all zero."""
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((N, K)) * 0.02
    w[rng.random((N, K)) < 0.01] *= 10.0
    w[::7] = np.round(w[::7] * 200.0) / 200.0
    if N > 3:
        w[3] = 0.0
    return w.astype(np.float32)


def groups(K: int, group: int = 128) -> int:
    return (K + group - 1) // group


# ---------------------------------------------------------------- device side
_synth_lib = None


def _device_lib():
    """libtern_synth.so: the same generator as above, run on the GPU."""
    global _synth_lib
    if _synth_lib is None:
        import ctypes
        import os
        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtern_synth.so")
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with "
                               "`python -m ternary_weight_decode_b200.build`")
        L = ctypes.CDLL(path)
        L.tern_synth_trits.restype = ctypes.c_int
        L.tern_synth_trits.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64,
                                       ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
        L.tern_synth_scales.restype = ctypes.c_int
        L.tern_synth_scales.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64,
                                        ctypes.c_void_p, ctypes.c_void_p]
        _synth_lib = L
    return _synth_lib


def device_trits(seed: int, stream: int, N: int, K: int, out=None, row0: int = 0):
    """Trits of rows [row0, row0+N) as a CUDA int8 tensor [N, K]."""
    import ctypes
    import torch
    if out is None:
        out = torch.empty((N, K), dtype=torch.int8, device="cuda")
    rc = _device_lib().tern_synth_trits(stream_key(seed, stream), row0, N, K,
                                        ctypes.c_void_p(out.data_ptr()),
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    if rc != 0:
        raise RuntimeError(f"tern_synth_trits failed with CUDA error {rc}")
    return out


def device_scales(seed: int, stream: int, N: int, G: int, out=None):
    """fp16 group scales as a CUDA float16 tensor [N, G]."""
    import ctypes
    import torch
    if out is None:
        out = torch.empty((N, G), dtype=torch.float16, device="cuda")
    rc = _device_lib().tern_synth_scales(stream_key(seed, stream), N, G,
                                         ctypes.c_void_p(out.data_ptr()),
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    if rc != 0:
        raise RuntimeError(f"tern_synth_scales failed with CUDA error {rc}")
    return out
