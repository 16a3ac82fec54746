"""ctypes wrapper around the plain-C oracle (``tern_oracle.c``).

TEST INFRASTRUCTURE: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code
with the CUDA library and never calls it.

Every function takes and returns numpy arrays.  Weights are passed as
unpacked trits (int8 in {-1, 0, +1}); fp16 scales as numpy float16; the
quantised activations as int8 with their fp32 per-row scale.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tern_oracle.c")
_LIB = os.path.join(_HERE, "libtern_oracle.so")
_lock = threading.Lock()
_lib = None

FMT_BASE3 = 0
FMT_2BIT = 1
FMT_BITPLANE = 2


class OracleError(ValueError):
    pass


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", "-std=c11", "-o", tmp, _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            i64, i32 = ctypes.c_int64, ctypes.c_int
            p = ctypes.c_void_p
            lib.oracle_half_to_double.restype = ctypes.c_double
            lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
            for name in ("oracle_base3_row_bytes", "oracle_2bit_row_bytes",
                         "oracle_bitplane_row_bytes"):
                getattr(lib, name).restype = i64
                getattr(lib, name).argtypes = [i64]
            lib.oracle_device_row_bytes.restype = i64
            lib.oracle_device_row_bytes.argtypes = [i32, i64]
            lib.oracle_groups.restype = i64
            lib.oracle_groups.argtypes = [i64, i64]
            for name in ("oracle_pack_base3", "oracle_unpack_base3", "oracle_pack_2bit",
                         "oracle_unpack_2bit", "oracle_pack_bitplane", "oracle_unpack_bitplane"):
                getattr(lib, name).restype = i32
                getattr(lib, name).argtypes = [p, i64, i64, p]
            for name in ("oracle_pack_device", "oracle_unpack_device"):
                getattr(lib, name).restype = i32
                getattr(lib, name).argtypes = [i32, p, i64, i64, i64, p]
            lib.oracle_d3_encode_value.restype = i32
            lib.oracle_d3_encode_value.argtypes = [i32]
            lib.oracle_d3_decode_value.restype = i32
            lib.oracle_d3_decode_value.argtypes = [i32]
            lib.oracle_act_quant.restype = i32
            lib.oracle_act_quant.argtypes = [p, i64, i64, i32, i32, p, p]
            lib.oracle_fwht128_f32.restype = None
            lib.oracle_fwht128_f32.argtypes = [p]
            lib.oracle_fwht128_f64.restype = None
            lib.oracle_fwht128_f64.argtypes = [p]
            lib.oracle_group_partials.restype = i32
            lib.oracle_group_partials.argtypes = [p, i64, i64, i64, p, i64, p]
            lib.oracle_gemv.restype = i32
            lib.oracle_gemv.argtypes = [p, p, i64, i64, i64, p, p, i64, p]
            lib.oracle_swiglu.restype = None
            lib.oracle_swiglu.argtypes = [p, p, i64, p]
            lib.oracle_gateup_swiglu.restype = i32
            lib.oracle_gateup_swiglu.argtypes = [p, p, p, p, i64, i64, i64, p, p, i64, p]
            lib.oracle_float_to_half.restype = ctypes.c_uint16
            lib.oracle_float_to_half.argtypes = [ctypes.c_float]
            lib.oracle_ternarize.restype = i32
            lib.oracle_ternarize.argtypes = [p, i64, i64, i64, i64, p, p]
            lib.oracle_q4_0_quantize.restype = i32
            lib.oracle_q4_0_quantize.argtypes = [p, i64, p, p]
            lib.oracle_q4_0_dequantize.restype = None
            lib.oracle_q4_0_dequantize.argtypes = [p, p, i64, p]
            lib.oracle_attention_decode.restype = i32
            lib.oracle_attention_decode.argtypes = [p, p, p, p, p, i64, i64, i64, i64, p]
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc: int, what: str):
    if rc != 0:
        raise OracleError(f"{what}: invalid input (oracle status {rc})")


def set_threads(n: int) -> None:
    """Thread count of the OpenMP loop over output rows in ``gemv``."""
    os.environ["OMP_NUM_THREADS"] = str(int(n))
    try:
        libgomp = ctypes.CDLL("libgomp.so.1")
        libgomp.omp_set_num_threads(ctypes.c_int(int(n)))
    except OSError:
        pass


# ---------------------------------------------------------------- formats
def half_to_double(bits: int) -> float:
    return _load().oracle_half_to_double(int(bits))


def base3_row_bytes(K: int) -> int:
    return int(_load().oracle_base3_row_bytes(K))


def twobit_row_bytes(K: int) -> int:
    return int(_load().oracle_2bit_row_bytes(K))


def device_row_bytes(fmt: int, K: int) -> int:
    return int(_load().oracle_device_row_bytes(fmt, K))


def groups(K: int, group: int = 128) -> int:
    return int(_load().oracle_groups(K, group))


def pack_base3(w: np.ndarray) -> np.ndarray:
    w = _c(w, np.int8)
    N, K = w.shape
    out = np.zeros((N, base3_row_bytes(K)), np.uint8)
    _check(_load().oracle_pack_base3(_ptr(w), N, K, _ptr(out)), "pack_base3")
    return out


def unpack_base3(b: np.ndarray, K: int) -> np.ndarray:
    b = _c(b, np.uint8)
    N = b.shape[0]
    w = np.zeros((N, K), np.int8)
    _check(_load().oracle_unpack_base3(_ptr(b), N, K, _ptr(w)), "unpack_base3")
    return w


def pack_2bit(w: np.ndarray) -> np.ndarray:
    w = _c(w, np.int8)
    N, K = w.shape
    out = np.zeros((N, twobit_row_bytes(K)), np.uint8)
    _check(_load().oracle_pack_2bit(_ptr(w), N, K, _ptr(out)), "pack_2bit")
    return out


def unpack_2bit(b: np.ndarray, K: int) -> np.ndarray:
    b = _c(b, np.uint8)
    N = b.shape[0]
    w = np.zeros((N, K), np.int8)
    _check(_load().oracle_unpack_2bit(_ptr(b), N, K, _ptr(w)), "unpack_2bit")
    return w


def bitplane_row_bytes(K: int) -> int:
    return int(_load().oracle_bitplane_row_bytes(K))


def pack_bitplane(w: np.ndarray) -> np.ndarray:
    """Canonical bit planes [N, 2 * ceil(K/8)]: the nonzero plane, then the sign plane."""
    w = _c(w, np.int8)
    N, K = w.shape
    out = np.zeros((N, bitplane_row_bytes(K)), np.uint8)
    _check(_load().oracle_pack_bitplane(_ptr(w), N, K, _ptr(out)), "pack_bitplane")
    return out


def unpack_bitplane(b: np.ndarray, K: int) -> np.ndarray:
    b = _c(b, np.uint8)
    N = b.shape[0]
    w = np.zeros((N, K), np.int8)
    _check(_load().oracle_unpack_bitplane(_ptr(b), N, K, _ptr(w)), "unpack_bitplane")
    return w


def d3_encode_value(V: int) -> int:
    return int(_load().oracle_d3_encode_value(V))


def d3_decode_value(y: int) -> int:
    return int(_load().oracle_d3_decode_value(y))


def pack_device(fmt: int, w: np.ndarray, row_stride: int) -> np.ndarray:
    w = _c(w, np.int8)
    N, K = w.shape
    out = np.zeros((N, row_stride), np.uint8)
    _check(_load().oracle_pack_device(fmt, _ptr(w), N, K, row_stride, _ptr(out)), "pack_device")
    return out


def unpack_device(fmt: int, b: np.ndarray, K: int) -> np.ndarray:
    b = _c(b, np.uint8)
    N, stride = b.shape
    w = np.zeros((N, K), np.int8)
    _check(_load().oracle_unpack_device(fmt, _ptr(b), N, K, stride, _ptr(w)), "unpack_device")
    return w


# ---------------------------------------------------------------- activations
def fwht128_f32(v: np.ndarray) -> np.ndarray:
    v = _c(v, np.float32).copy()
    assert v.shape == (128,)
    _load().oracle_fwht128_f32(_ptr(v))
    return v


def fwht128_f64(v: np.ndarray) -> np.ndarray:
    v = _c(v, np.float64).copy()
    assert v.shape == (128,)
    _load().oracle_fwht128_f64(_ptr(v))
    return v


def act_quant(x: np.ndarray, fwht_block: int = 0, rmsnorm: bool = False):
    """Returns (q int8 [M, K], s_x fp32 [M]) for fp16 or fp32 input x [M, K]."""
    x = _c(np.asarray(x).astype(np.float32), np.float32)
    M, K = x.shape
    q = np.zeros((M, K), np.int8)
    s = np.zeros((M,), np.float32)
    _check(_load().oracle_act_quant(_ptr(x), M, K, fwht_block, 1 if rmsnorm else 0, _ptr(q),
                                   _ptr(s)), "act_quant")
    return q, s


# ---------------------------------------------------------------- products
def group_partials(w: np.ndarray, q: np.ndarray, group: int = 128) -> np.ndarray:
    """Exact integer partials P int64 [M, N, G]."""
    w = _c(w, np.int8)
    q = _c(q, np.int8)
    N, K = w.shape
    M = q.shape[0]
    assert q.shape[1] == K
    G = groups(K, group)
    P = np.zeros((M, N, G), np.int64)
    _check(_load().oracle_group_partials(_ptr(w), N, K, group, _ptr(q), M, _ptr(P)),
           "group_partials")
    return P


def gemv(w: np.ndarray, scales: np.ndarray, q: np.ndarray, s_x: np.ndarray,
         group: int = 128) -> np.ndarray:
    """y fp64 [M, N] = s_x[m] * sum_g s_w[n, g] * P[m, n, g]."""
    w = _c(w, np.int8)
    sc = _c(np.asarray(scales, dtype=np.float16).view(np.uint16), np.uint16)
    q = _c(q, np.int8)
    s_x = _c(s_x, np.float32)
    N, K = w.shape
    M = q.shape[0]
    assert q.shape[1] == K and sc.shape == (N, groups(K, group)) and s_x.shape == (M,)
    y = np.zeros((M, N), np.float64)
    _check(_load().oracle_gemv(_ptr(w), _ptr(sc), N, K, group, _ptr(q), _ptr(s_x), M, _ptr(y)),
           "gemv")
    return y


def swiglu(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    g = _c(g, np.float64)
    u = _c(u, np.float64)
    h = np.zeros_like(g)
    _load().oracle_swiglu(_ptr(g), _ptr(u), g.size, _ptr(h))
    return h


def gateup_swiglu(wg, sg, wu, su, q, s_x, group: int = 128) -> np.ndarray:
    wg = _c(wg, np.int8)
    wu = _c(wu, np.int8)
    sg = _c(np.asarray(sg, dtype=np.float16).view(np.uint16), np.uint16)
    su = _c(np.asarray(su, dtype=np.float16).view(np.uint16), np.uint16)
    q = _c(q, np.int8)
    s_x = _c(s_x, np.float32)
    N, K = wg.shape
    M = q.shape[0]
    h = np.zeros((M, N), np.float64)
    _check(_load().oracle_gateup_swiglu(_ptr(wg), _ptr(sg), _ptr(wu), _ptr(su), N, K, group,
                                        _ptr(q), _ptr(s_x), M, _ptr(h)), "gateup_swiglu")
    return h


# ---------------------------------------------------------------- ternarisation
def float_to_half_bits(f: float) -> int:
    """IEEE binary16 bits of fp32 f, round to nearest even."""
    return int(_load().oracle_float_to_half(float(np.float32(f))))


def ternarize(w: np.ndarray, group: int = 128):
    """(trits int8 [N, K], scales float16 [N, G]) of fp32 weights w [N, K]:
    per group the MSE-optimal symmetric thresholds and scale, in the fp32
    arithmetic the C file states (its reading R10)."""
    w = _c(w, np.float32)
    N, K = w.shape
    G = groups(K, group)
    t = np.zeros((N, K), np.int8)
    sc = np.zeros((N, G), np.uint16)
    _check(_load().oracle_ternarize(_ptr(w), N, K, K, group, _ptr(t), _ptr(sc)), "ternarize")
    return t, sc.view(np.float16)


# ---------------------------------------------------------------- Q4_0 KV attention
def q4_0_quantize(x: np.ndarray):
    """(d float16 [..., n/32], qs uint8 [..., n/32, 16]) of fp32 x [..., n], n % 32 == 0."""
    x = _c(x, np.float32)
    n = x.size
    d = np.zeros(n // 32, np.uint16)
    qs = np.zeros((n // 32, 16), np.uint8)
    _check(_load().oracle_q4_0_quantize(_ptr(x), n, _ptr(d), _ptr(qs)), "q4_0_quantize")
    lead = x.shape[:-1] + (x.shape[-1] // 32,)
    return d.view(np.float16).reshape(lead), qs.reshape(lead + (16,))


def q4_0_dequantize(d: np.ndarray, qs: np.ndarray) -> np.ndarray:
    d = _c(np.asarray(d, np.float16).view(np.uint16), np.uint16)
    qs = _c(qs, np.uint8)
    n = d.size * 32
    out = np.zeros(n, np.float64)
    _load().oracle_q4_0_dequantize(_ptr(d), _ptr(qs), n, _ptr(out))
    return out.reshape(d.shape[:-1] + (d.shape[-1] * 32,))


def attention_decode(q, kd, kq, vd, vq):
    """out fp64 [Hq, D] for q fp32 [Hq, D] and a Q4_0 cache: kd/vd float16
    [Hkv, L, D/32], kq/vq uint8 [Hkv, L, D/32, 16]."""
    q = _c(q, np.float32)
    Hq, D = q.shape
    Hkv, L = kd.shape[0], kd.shape[1]
    args = [_c(np.asarray(a, np.float16).view(np.uint16), np.uint16) if i % 2 == 0 else _c(a, np.uint8)
            for i, a in enumerate((kd, kq, vd, vq))]
    out = np.zeros((Hq, D), np.float64)
    _check(_load().oracle_attention_decode(_ptr(q), *[_ptr(a) for a in args], L, Hkv, Hq, D,
                                          _ptr(out)), "attention_decode")
    return out
