"""The C-ABI library loads and exports every entry point of include/*.h; host
validation rejects bad arguments without touching a GPU."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _lib():
    from ternary_weight_decode_b200 import build, tern
    if not os.path.exists(tern.LIB_PATH):
        build.build()
    return tern.lib()


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported():
    lib = _lib()
    names = declared_functions()
    assert "tern_gemv" in names and "act_quant_fwht" in names and len(names) >= 12
    for n in names:
        assert hasattr(lib, n), f"libtern.so does not export {n}"


def test_status_strings():
    lib = _lib()
    for s in range(5):
        assert lib.tern_status_string(s)


def _matrix(**kw):
    from ternary_weight_decode_b200.tern import tern_matrix
    base = dict(fmt=0, N=4, K=256, group=128, row_stride=64, packed=4096, scales=8192,
                scales_tiled=None, flags=0, reserved=0)
    base.update(kw)
    return tern_matrix(**base)


@pytest.mark.parametrize("kw", [dict(fmt=7), dict(N=0), dict(K=0), dict(row_stride=48),
                                dict(row_stride=72), dict(packed=4097), dict(packed=0),
                                dict(scales=0), dict(flags=2), dict(reserved=1)])
def test_gemv_rejects_bad_matrix(kw):
    lib = _lib()
    m = _matrix(**kw)
    st = lib.tern_gemv(ctypes.byref(m), ctypes.c_void_p(4096), 256, ctypes.c_void_p(4096), 1, None,
                       ctypes.c_void_p(4096), 4, None)
    assert st == 1, lib.tern_last_error()
    assert lib.tern_last_error()


def test_gemv_rejects_group_other_than_128():
    lib = _lib()
    m = _matrix(group=64)
    st = lib.tern_gemv(ctypes.byref(m), ctypes.c_void_p(4096), 256, ctypes.c_void_p(4096), 1, None,
                       ctypes.c_void_p(4096), 4, None)
    assert st == 3


@pytest.mark.parametrize("q,ldq,M,ldy", [(4097, 256, 1, 4), (4096, 250, 1, 4), (4096, 240, 1, 4),
                                         (4096, 256, 0, 4), (4096, 256, 17, 4), (4096, 256, 1, 3)])
def test_gemv_rejects_bad_activations(q, ldq, M, ldy):
    lib = _lib()
    m = _matrix()
    st = lib.tern_gemv(ctypes.byref(m), ctypes.c_void_p(q), ldq, ctypes.c_void_p(4096), M, None,
                       ctypes.c_void_p(4096), ldy, None)
    assert st == 1


@pytest.mark.parametrize("args", [
    (4096, 1, 1, 200, 200, 128, 4096, 208, 4096),   # rotation needs K % 128 == 0
    (4096, 1, 1, 256, 256, 64, 4096, 256, 4096),    # block other than 128
    (4098, 1, 1, 256, 256, 0, 4096, 256, 4096),     # misaligned x
    (4096, 1, 1, 256, 250, 0, 4096, 256, 4096),     # ldx < K
    (4096, 1, 1, 256, 256, 0, 4096, 264, 4096),     # ldq not a multiple of 16
    (4096, 1, 0, 256, 256, 0, 4096, 256, 4096),     # M = 0
])
def test_act_quant_rejects(args):
    lib = _lib()
    x, fp16, M, K, ldx, fw, q, ldq, s = args
    st = lib.act_quant_fwht(ctypes.c_void_p(x), fp16, M, K, ldx, fw, 0, ctypes.c_void_p(q), ldq,
                            ctypes.c_void_p(s), None)
    assert st == 1


def test_pack_rejects_bad_stride_and_sizes():
    lib = _lib()
    assert lib.tern_pack(0, ctypes.c_void_p(4096), 4, 256, ctypes.c_void_p(4096), 48, None, None) == 1
    assert lib.tern_pack(0, ctypes.c_void_p(4096), 0, 256, ctypes.c_void_p(4096), 64, None, None) == 1
    assert lib.tern_pack(3, ctypes.c_void_p(4096), 4, 256, ctypes.c_void_p(4096), 64, None, None) == 1


def test_packed_size_matches_layout():
    lib = _lib()
    rs = ctypes.c_int64()
    pb = ctypes.c_size_t()
    sb = ctypes.c_size_t()
    assert lib.tern_packed_size(0, 5120, 17408, 128, ctypes.byref(rs), ctypes.byref(pb),
                                ctypes.byref(sb)) == 0
    assert rs.value == 3488 and pb.value == 5120 * 3488 and sb.value == 2 * 5120 * 136
    assert lib.tern_packed_size(1, 7168, 5120, 128, ctypes.byref(rs), None, None) == 0
    assert rs.value == 1280


def test_act_quant_rejects_unknown_flags():
    lib = _lib()
    st = lib.act_quant_fwht(ctypes.c_void_p(4096), 1, 1, 256, 256, 0, 2, ctypes.c_void_p(4096), 256,
                            ctypes.c_void_p(4096), None)
    assert st == 1


@pytest.mark.parametrize("ldq,M,ldy,q,y", [(250, 4, 8, 4096, 8192), (256, 0, 8, 4096, 8192),
                                          (256, 4, 3, 4096, 8192), (256, 4, 8, 4097, 8192),
                                          (256, 4, 8, 4096, 0)])
def test_gemm_rejects_bad_arguments(ldq, M, ldy, q, y):
    lib = _lib()
    m = _matrix()
    st = lib.tern_gemm(ctypes.byref(m), ctypes.c_void_p(q), ldq, ctypes.c_void_p(4096), M,
                       ctypes.c_void_p(y) if y else None, ldy, None)
    assert st == 1, lib.tern_last_error()
    assert b"tern_gemm" in lib.tern_last_error()


@pytest.mark.parametrize("kind,budget", [(2, 1000), (-1, 1000), (0, 0), (1, 200000001)])
def test_bounded_wait_hook_rejects_bad_arguments(kind, budget):
    """Host validation only: no kernel is launched."""
    lib = _lib()
    assert lib.tern_debug_bounded_wait(kind, budget, None) == 1
    assert b"tern_debug_bounded_wait" in lib.tern_last_error()


def test_debug_streamed_requires_its_outputs():
    lib = _lib()
    m = _matrix(scales_tiled=16384)
    st = lib.tern_debug_streamed(ctypes.byref(m), None, ctypes.c_void_p(4096), 256, 0, 1,
                                 ctypes.c_void_p(4096), 4, None, 256, ctypes.c_void_p(4096),
                                 ctypes.c_void_p(4096), ctypes.c_void_p(4096), 1 << 20, None)
    assert st == 1 and b"q_out" in lib.tern_last_error()


def test_noalloc_validates_before_touching_its_array():
    """A call rejected on its arguments fails before any CUDA call (no GPU is
    needed to see the error), so it cannot have cleared the shared array."""
    lib = _lib()
    m = _matrix(scales_tiled=16384)
    # x misaligned
    st = lib.tern_gemv_streamed_noalloc(ctypes.byref(m), ctypes.c_void_p(4100), 256, 0, 1, None,
                                        ctypes.c_void_p(4096), 4, None)
    assert st == 1 and b"x must be" in lib.tern_last_error()
    # unknown qflags
    st = lib.tern_gemv_streamed_noalloc(ctypes.byref(m), ctypes.c_void_p(4096), 256, 8, 1, None,
                                        ctypes.c_void_p(4096), 4, None)
    assert st == 1 and b"qflags" in lib.tern_last_error()

