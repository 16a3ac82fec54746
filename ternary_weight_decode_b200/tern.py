"""Python binding of libtern.so (include/tern.h): argument marshalling only.

Every function has the name of its C entry point, takes torch CUDA tensors
for device buffers, passes their pointers and the current torch stream, and
raises ``TernError`` on a non-OK status.  All arithmetic runs in the CUDA
kernels of libtern.so; there is no CPU fallback and no other backend: when
the library is missing this module raises instead of computing anything.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtern.so")

TERN_OK, TERN_EINVAL, TERN_ECUDA, TERN_EUNSUPPORTED, TERN_ETIMEOUT = 0, 1, 2, 3, 4
TERN_FMT_BASE3, TERN_FMT_2BIT, TERN_FMT_BITPLANE = 0, 1, 2
TERN_MATRIX_STATIC = 1
TERN_QUANT_RMSNORM = 1
TERN_QUANT_FWHT128 = 2
GROUP = 128


class TernError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: status {status}: {message}")
        self.status = status


class tern_matrix(ctypes.Structure):
    _fields_ = [
        ("fmt", ctypes.c_int32),
        ("N", ctypes.c_int32),
        ("K", ctypes.c_int32),
        ("group", ctypes.c_int32),
        ("row_stride", ctypes.c_int64),
        ("packed", ctypes.c_void_p),
        ("scales", ctypes.c_void_p),
        ("scales_tiled", ctypes.c_void_p),
        ("flags", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


class tern_kv_cache(ctypes.Structure):
    _fields_ = [
        ("Hkv", ctypes.c_int32),
        ("D", ctypes.c_int32),
        ("capacity", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
        ("k_codes", ctypes.c_void_p),
        ("k_scales", ctypes.c_void_p),
        ("v_codes", ctypes.c_void_p),
        ("v_scales", ctypes.c_void_p),
    ]


_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """The loaded libtern.so; raises when it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m ternary_weight_decode_b200.build` (no CPU fallback exists)")
            L = ctypes.CDLL(LIB_PATH)
            i32, i64, p, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t
            pm = ctypes.POINTER(tern_matrix)
            sig = {
                "tern_status_string": (ctypes.c_char_p, [ctypes.c_int]),
                "tern_last_error": (ctypes.c_char_p, []),
                "tern_packed_size": (ctypes.c_int, [i32, i32, i32, i32, ctypes.POINTER(i64),
                                                    ctypes.POINTER(sz), ctypes.POINTER(sz)]),
                "tern_canonical_row_bytes": (ctypes.c_int, [i32, i32, ctypes.POINTER(i64)]),
                "tern_tiled_scales_bytes": (ctypes.c_int, [i32, i32, i32, ctypes.POINTER(sz)]),
                "tern_retile_scales": (ctypes.c_int, [pm, p, p]),
                "tern_pack": (ctypes.c_int, [i32, p, i32, i32, p, i64, p, p]),
                "tern_unpack": (ctypes.c_int, [pm, p, p, p]),
                "tern_import": (ctypes.c_int, [i32, p, i32, i32, p, i64, p, p]),
                "tern_export": (ctypes.c_int, [pm, p, p, p]),
                "act_quant_fwht": (ctypes.c_int, [p, i32, i32, i32, i32, i32, i32, p, i32, p, p]),
                "tern_ternarize": (ctypes.c_int, [p, i32, i32, i32, i32, p, p, p]),
                "tern_gemv": (ctypes.c_int, [pm, p, i32, p, i32, p, p, i32, p]),
                "tern_gateup_swiglu": (ctypes.c_int, [pm, pm, p, i32, p, i32, p, i32, p]),
                "tern_debug_group_partials": (ctypes.c_int, [pm, p, i32, i32, p, p]),
                "tern_device_error": (ctypes.c_int, [ctypes.POINTER(i32), p]),
                "tern_act_stats": (ctypes.c_int, [p, i32, i32, i32, p, i32, p]),
                "tern_debug_mma_i8": (ctypes.c_int, [i32, p, i32, p, i32, p, i32, i32, p]),
                "tern_debug_select_engine": (ctypes.c_int, [i32]),
                "tern_stream_workspace_bytes": (ctypes.c_int, [i32, i32, i32, i32, ctypes.POINTER(sz)]),
                "tern_gemv_streamed": (ctypes.c_int, [pm, p, i32, i32, i32, p, p, i32, p, sz, p]),
                "tern_gateup_swiglu_streamed": (ctypes.c_int, [pm, pm, p, i32, i32, i32, p, i32, p, sz,
                                                               p]),
                "tern_gemv_streamed_noalloc": (ctypes.c_int, [pm, p, i32, i32, i32, p, p, i32, p]),
                "tern_gemm": (ctypes.c_int, [pm, p, i32, p, i32, p, i32, p]),
                "tern_debug_streamed": (ctypes.c_int, [pm, pm, p, i32, i32, i32, p, i32, p, i32, p, p,
                                                       p, sz, p]),
                "tern_debug_gemm_partials": (ctypes.c_int, [pm, p, i32, p, i32, p, i32, p, p]),
                "tern_debug_bounded_wait": (ctypes.c_int, [i32, i64, p]),
                "tern_kv_append_q4_0": (ctypes.c_int, [p, p, i32, ctypes.POINTER(tern_kv_cache), p]),
                "tern_attention_workspace_bytes": (ctypes.c_int, [i32, i32, ctypes.POINTER(tern_kv_cache),
                                                                  ctypes.POINTER(sz)]),
                "tern_attention_decode_q4_0": (ctypes.c_int, [p, i32, ctypes.POINTER(tern_kv_cache), i32, p,
                                                              p, sz, p]),
                "tern_gemv_fused": (ctypes.c_int, [pm, p, i32, p, i32, i32, i32, p, p, i32, p, i32, p]),
                "tern_gateup_swiglu_fused": (ctypes.c_int, [pm, pm, p, i32, p, i32, i32, i32, p, i32,
                                                            p, i32, p]),
            }
            for name, (res, args) in sig.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
    return _lib


def _check(status: int, where: str) -> None:
    if status != TERN_OK:
        msg = lib().tern_last_error().decode(errors="replace")
        raise TernError(status, where, msg)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("device buffers must be CUDA tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


# ------------------------------------------------------------------ sizes
def tern_packed_size(fmt: int, N: int, K: int, group: int = GROUP):
    rs = ctypes.c_int64()
    pb = ctypes.c_size_t()
    sb = ctypes.c_size_t()
    _check(lib().tern_packed_size(fmt, N, K, group, ctypes.byref(rs), ctypes.byref(pb),
                                  ctypes.byref(sb)), "tern_packed_size")
    return rs.value, pb.value, sb.value


def tern_canonical_row_bytes(fmt: int, K: int) -> int:
    b = ctypes.c_int64()
    _check(lib().tern_canonical_row_bytes(fmt, K, ctypes.byref(b)), "tern_canonical_row_bytes")
    return b.value


def tern_tiled_scales_bytes(fmt: int, N: int, K: int) -> int:
    b = ctypes.c_size_t()
    _check(lib().tern_tiled_scales_bytes(fmt, N, K, ctypes.byref(b)), "tern_tiled_scales_bytes")
    return b.value


def tern_retile_scales(W, out: torch.Tensor, stream=None):
    s = W.struct()
    _check(lib().tern_retile_scales(ctypes.byref(s), _ptr(out), _stream(stream)),
           "tern_retile_scales")


# ------------------------------------------------------------------ matrices
@dataclass
class TernMatrix:
    """A packed device matrix: `packed` uint8 [N, row_stride], `scales` fp16 [N, G]."""
    fmt: int
    N: int
    K: int
    row_stride: int
    packed: torch.Tensor
    scales: torch.Tensor
    static: bool = True
    scales_tiled: torch.Tensor | None = None

    def struct(self) -> tern_matrix:
        return tern_matrix(self.fmt, self.N, self.K, GROUP, self.row_stride,
                           self.packed.data_ptr(), self.scales.data_ptr(),
                           None if self.scales_tiled is None else self.scales_tiled.data_ptr(),
                           TERN_MATRIX_STATIC if self.static else 0, 0)

    def retile_scales(self, stream=None) -> "TernMatrix":
        """Writes the unit-major copy of the scales the streamed kernels read."""
        nbytes = tern_tiled_scales_bytes(self.fmt, self.N, self.K)
        self.scales_tiled = torch.zeros(nbytes // 2, dtype=torch.float16, device=self.packed.device)
        tern_retile_scales(self, self.scales_tiled, stream)
        return self

    @staticmethod
    def empty(fmt: int, N: int, K: int, device="cuda") -> "TernMatrix":
        rs, pb, sb = tern_packed_size(fmt, N, K)
        packed = torch.empty((N, rs), dtype=torch.uint8, device=device)
        scales = torch.empty((N, (K + GROUP - 1) // GROUP), dtype=torch.float16, device=device)
        return TernMatrix(fmt, N, K, rs, packed, scales)


def tern_pack(fmt: int, trits: torch.Tensor, out: TernMatrix, d_invalid=None, stream=None):
    N, K = trits.shape
    assert trits.dtype == torch.int8 and trits.is_contiguous()
    assert out.packed.dtype == torch.uint8 and out.packed.shape == (N, out.row_stride)
    _check(lib().tern_pack(fmt, _ptr(trits), N, K, _ptr(out.packed), out.row_stride,
                           _ptr(d_invalid), _stream(stream)), "tern_pack")


def tern_unpack(W: TernMatrix, trits_out: torch.Tensor, d_invalid=None, stream=None):
    assert trits_out.dtype == torch.int8 and trits_out.shape == (W.N, W.K)
    s = W.struct()
    _check(lib().tern_unpack(ctypes.byref(s), _ptr(trits_out), _ptr(d_invalid), _stream(stream)),
           "tern_unpack")


def tern_import(fmt: int, canonical: torch.Tensor, K: int, out: TernMatrix, d_invalid=None,
                stream=None):
    N = canonical.shape[0]
    assert canonical.dtype == torch.uint8 and canonical.is_contiguous()
    assert canonical.shape[1] == tern_canonical_row_bytes(fmt, K)
    _check(lib().tern_import(fmt, _ptr(canonical), N, K, _ptr(out.packed), out.row_stride,
                             _ptr(d_invalid), _stream(stream)), "tern_import")


def tern_export(W: TernMatrix, canonical_out: torch.Tensor, d_invalid=None, stream=None):
    assert canonical_out.dtype == torch.uint8
    assert canonical_out.shape == (W.N, tern_canonical_row_bytes(W.fmt, W.K))
    s = W.struct()
    _check(lib().tern_export(ctypes.byref(s), _ptr(canonical_out), _ptr(d_invalid),
                             _stream(stream)), "tern_export")


def tern_ternarize(w: torch.Tensor, trits: torch.Tensor, scales: torch.Tensor, K: int | None = None,
                   stream=None):
    """fp32 weights w [N, >=K] -> trits int8 [N, K] and fp16 group scales [N, G]."""
    assert w.dtype == torch.float32 and w.stride(1) == 1
    N = w.shape[0]
    K = w.shape[1] if K is None else K
    assert trits.dtype == torch.int8 and trits.is_contiguous() and trits.shape == (N, K)
    assert scales.dtype == torch.float16 and scales.is_contiguous()
    _check(lib().tern_ternarize(_ptr(w), N, K, w.stride(0), GROUP, _ptr(trits), _ptr(scales),
                                _stream(stream)), "tern_ternarize")


# ------------------------------------------------------------------ compute
def act_quant_fwht(x: torch.Tensor, q: torch.Tensor, s_x: torch.Tensor, fwht_block: int = 0,
                   K: int | None = None, flags: int = 0, stream=None):
    """x fp16/fp32 [M, ldx] -> q int8 [M, ldq], s_x fp32 [M] (first K columns of x)."""
    assert x.dtype in (torch.float16, torch.float32) and x.stride(1) == 1
    M = x.shape[0]
    K = x.shape[1] if K is None else K
    assert q.dtype == torch.int8 and q.stride(1) == 1 and q.shape[0] == M
    assert s_x.dtype == torch.float32 and s_x.numel() >= M
    _check(lib().act_quant_fwht(_ptr(x), 1 if x.dtype == torch.float16 else 0, M, K, x.stride(0),
                                fwht_block, flags, _ptr(q), q.stride(0), _ptr(s_x),
                                _stream(stream)),
           "act_quant_fwht")


def tern_gemv(W: TernMatrix, q: torch.Tensor, s_x: torch.Tensor, y: torch.Tensor,
              residual: torch.Tensor | None = None, M: int | None = None, stream=None):
    M = q.shape[0] if M is None else M
    assert q.dtype == torch.int8 and y.dtype == torch.float32 and y.stride(1) == 1
    if residual is not None:
        assert residual.dtype == torch.float32 and residual.stride(0) == y.stride(0)
    s = W.struct()
    _check(lib().tern_gemv(ctypes.byref(s), _ptr(q), q.stride(0), _ptr(s_x), M, _ptr(residual),
                           _ptr(y), y.stride(0), _stream(stream)), "tern_gemv")


def tern_gemm(W: TernMatrix, q: torch.Tensor, s_x: torch.Tensor, y: torch.Tensor, M: int | None = None,
              stream=None):
    """Prefill GEMM: y [M, N] = s_x * (group-scaled W q) on the tensor cores."""
    M = q.shape[0] if M is None else M
    assert q.dtype == torch.int8 and q.stride(1) == 1 and y.dtype == torch.float32
    s = W.struct()
    _check(lib().tern_gemm(ctypes.byref(s), _ptr(q), q.stride(0), _ptr(s_x), M, _ptr(y), y.stride(0),
                           _stream(stream)),
           "tern_gemm")


def tern_gateup_swiglu(Wg: TernMatrix, Wu: TernMatrix, q: torch.Tensor, s_x: torch.Tensor,
                       h: torch.Tensor, M: int | None = None, stream=None):
    M = q.shape[0] if M is None else M
    assert q.dtype == torch.int8 and h.dtype == torch.float32 and h.stride(1) == 1
    sg, su = Wg.struct(), Wu.struct()
    _check(lib().tern_gateup_swiglu(ctypes.byref(sg), ctypes.byref(su), _ptr(q), q.stride(0),
                                    _ptr(s_x), M, _ptr(h), h.stride(0), _stream(stream)),
           "tern_gateup_swiglu")


def tern_debug_group_partials(W: TernMatrix, q: torch.Tensor, P: torch.Tensor,
                              M: int | None = None, stream=None):
    M = q.shape[0] if M is None else M
    assert P.dtype == torch.int32 and P.is_contiguous()
    s = W.struct()
    _check(lib().tern_debug_group_partials(ctypes.byref(s), _ptr(q), q.stride(0), M, _ptr(P),
                                           _stream(stream)), "tern_debug_group_partials")


def stats_buffer(M: int, length: int, device="cuda") -> torch.Tensor:
    """A statistics buffer fp32 [M, ceil(length/128), 4] for the fused calls."""
    return torch.zeros((M, (length + 127) // 128, 4), dtype=torch.float32, device=device)


def tern_act_stats(x: torch.Tensor, stats: torch.Tensor, K: int | None = None, stream=None):
    assert x.dtype == torch.float32 and x.stride(1) == 1 and stats.dtype == torch.float32
    M = x.shape[0]
    K = x.shape[1] if K is None else K
    _check(lib().tern_act_stats(_ptr(x), M, K, x.stride(0), _ptr(stats), stats.shape[1],
                                _stream(stream)), "tern_act_stats")


def tern_gemv_fused(W: TernMatrix, x: torch.Tensor, x_stats: torch.Tensor, y: torch.Tensor,
                    qflags: int = 0, residual: torch.Tensor | None = None,
                    y_stats: torch.Tensor | None = None, M: int | None = None, stream=None):
    """y = [residual +] W . quant(x); x fp32 [M, >=K] with block statistics x_stats."""
    M = x.shape[0] if M is None else M
    assert x.dtype == torch.float32 and x.stride(1) == 1 and y.dtype == torch.float32
    if residual is not None:
        assert residual.dtype == torch.float32 and residual.stride(0) == y.stride(0)
    s = W.struct()
    _check(lib().tern_gemv_fused(ctypes.byref(s), _ptr(x), x.stride(0), _ptr(x_stats),
                                 x_stats.shape[1], qflags, M, _ptr(residual), _ptr(y), y.stride(0),
                                 _ptr(y_stats), 0 if y_stats is None else y_stats.shape[1],
                                 _stream(stream)), "tern_gemv_fused")


def tern_gateup_swiglu_fused(Wg: TernMatrix, Wu: TernMatrix, x: torch.Tensor,
                             x_stats: torch.Tensor, h: torch.Tensor, qflags: int = 0,
                             h_stats: torch.Tensor | None = None, M: int | None = None,
                             stream=None):
    M = x.shape[0] if M is None else M
    assert x.dtype == torch.float32 and x.stride(1) == 1 and h.dtype == torch.float32
    sg, su = Wg.struct(), Wu.struct()
    _check(lib().tern_gateup_swiglu_fused(ctypes.byref(sg), ctypes.byref(su), _ptr(x), x.stride(0),
                                          _ptr(x_stats), x_stats.shape[1], qflags, M, _ptr(h),
                                          h.stride(0), _ptr(h_stats),
                                          0 if h_stats is None else h_stats.shape[1],
                                          _stream(stream)), "tern_gateup_swiglu_fused")


def tern_debug_mma_i8(A: torch.Tensor, B: torch.Tensor, D: torch.Tensor, a_in_smem: int = 0,
                      a_signed: bool = True, b_signed: bool = True, stream=None):
    """D int32 [128, N] = A [128, K] . B [N, K]^T on the tensor cores (test hook).
    a_in_smem: 0 A in tensor memory, 1 A in shared memory, 2 both operands in
    the 128-byte-swizzled layout."""
    K = A.shape[1]
    N = B.shape[0]
    _check(lib().tern_debug_mma_i8(int(a_in_smem), _ptr(A), 1 if a_signed else 0, _ptr(B),
                                   1 if b_signed else 0, _ptr(D), K, N, _stream(stream)),
           "tern_debug_mma_i8")


def tern_stream_workspace_bytes(fmt: int, N: int, M: int, two_matrices: bool) -> int:
    b = ctypes.c_size_t()
    _check(lib().tern_stream_workspace_bytes(fmt, N, M, 1 if two_matrices else 0, ctypes.byref(b)),
           "tern_stream_workspace_bytes")
    return b.value


def stream_workspace(fmt: int, N: int, M: int, two_matrices: bool, device="cuda") -> torch.Tensor:
    """A zeroed workspace for the streamed calls (kept zero by every call)."""
    n = tern_stream_workspace_bytes(fmt, N, M, two_matrices)
    return torch.zeros((n + 15) // 16 * 4, dtype=torch.int32, device=device)


def tern_gemv_streamed(W: TernMatrix, x: torch.Tensor, y: torch.Tensor, workspace: torch.Tensor,
                       qflags: int = 0, residual: torch.Tensor | None = None, M: int | None = None,
                       stream=None):
    M = x.shape[0] if M is None else M
    assert x.dtype == torch.float32 and x.stride(1) == 1 and y.dtype == torch.float32
    s = W.struct()
    _check(lib().tern_gemv_streamed(ctypes.byref(s), _ptr(x), x.stride(0), qflags, M,
                                    _ptr(residual), _ptr(y), y.stride(0), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream)),
           "tern_gemv_streamed")


# Size of the scratch array tern_gemv_streamed_noalloc uses (include/tern.h).
NOALLOC_SCRATCH_BYTES = 1 << 20


def tern_gemv_streamed_noalloc(W: TernMatrix, x: torch.Tensor, y: torch.Tensor, qflags: int = 0,
                               residual: torch.Tensor | None = None, M: int | None = None,
                               stream=None):
    """tern_gemv_streamed with the library's own scratch array in place of a
    caller workspace: for callers that cannot allocate device memory."""
    M = x.shape[0] if M is None else M
    assert x.dtype == torch.float32 and x.stride(1) == 1 and y.dtype == torch.float32
    s = W.struct()
    _check(lib().tern_gemv_streamed_noalloc(ctypes.byref(s), _ptr(x), x.stride(0), qflags, M,
                                            _ptr(residual), _ptr(y), y.stride(0), _stream(stream)),
           "tern_gemv_streamed_noalloc")


def tern_gateup_swiglu_streamed(Wg: TernMatrix, Wu: TernMatrix, x: torch.Tensor, h: torch.Tensor,
                                workspace: torch.Tensor, qflags: int = 0, M: int | None = None,
                                stream=None):
    M = x.shape[0] if M is None else M
    assert x.dtype == torch.float32 and x.stride(1) == 1 and h.dtype == torch.float32
    sg, su = Wg.struct(), Wu.struct()
    _check(lib().tern_gateup_swiglu_streamed(ctypes.byref(sg), ctypes.byref(su), _ptr(x),
                                             x.stride(0), qflags, M, _ptr(h), h.stride(0),
                                             _ptr(workspace),
                                             workspace.numel() * workspace.element_size(),
                                             _stream(stream)), "tern_gateup_swiglu_streamed")


def tern_debug_streamed(W0: TernMatrix, W1: TernMatrix | None, x: torch.Tensor, out: torch.Tensor,
                        q_out: torch.Tensor, s_x_out: torch.Tensor, P_out: torch.Tensor,
                        workspace: torch.Tensor, qflags: int = 0, M: int | None = None, stream=None):
    """Test hook: the streamed kernel (GEMV, or SwiGLU when W1 is given) also
    writes its int8 input q_out [M, >=K], row scales s_x_out [M] and exact
    group partials P_out int32 [NMAT, M, N, G]."""
    M = x.shape[0] if M is None else M
    assert x.dtype == torch.float32 and x.stride(1) == 1 and out.dtype == torch.float32
    assert q_out.dtype == torch.int8 and s_x_out.dtype == torch.float32
    assert P_out.dtype == torch.int32 and P_out.is_contiguous()
    s0 = W0.struct()
    s1 = None if W1 is None else ctypes.byref(W1.struct())
    _check(lib().tern_debug_streamed(ctypes.byref(s0), s1, _ptr(x), x.stride(0), qflags, M, _ptr(out),
                                     out.stride(0), _ptr(q_out), q_out.stride(0), _ptr(s_x_out),
                                     _ptr(P_out), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(stream)),
           "tern_debug_streamed")


def tern_debug_gemm_partials(W: TernMatrix, q: torch.Tensor, s_x: torch.Tensor, y: torch.Tensor,
                             P: torch.Tensor, M: int | None = None, stream=None):
    """Test hook: tern_gemm that also writes its exact group partials P int32 [M, N, G]."""
    M = q.shape[0] if M is None else M
    assert q.dtype == torch.int8 and q.stride(1) == 1 and y.dtype == torch.float32
    assert P.dtype == torch.int32 and P.is_contiguous()
    s = W.struct()
    _check(lib().tern_debug_gemm_partials(ctypes.byref(s), _ptr(q), q.stride(0), _ptr(s_x), M, _ptr(y),
                                          y.stride(0), _ptr(P), _stream(stream)),
           "tern_debug_gemm_partials")


def tern_debug_bounded_wait(kind: int, budget_cycles: int, stream=None):
    """Test hook: a kernel whose bounded wait (0: mbarrier, 1: tagged word) runs out."""
    _check(lib().tern_debug_bounded_wait(kind, budget_cycles, _stream(stream)),
           "tern_debug_bounded_wait")


@dataclass
class KVCache:
    """A Q4_0 KV cache of one layer: codes uint8 [Hkv, capacity, D/2] and
    fp16 scales [Hkv, capacity, D/32] for K and for V."""
    Hkv: int
    D: int
    capacity: int
    k_codes: torch.Tensor
    k_scales: torch.Tensor
    v_codes: torch.Tensor
    v_scales: torch.Tensor

    @staticmethod
    def empty(Hkv: int, D: int, capacity: int, device="cuda") -> "KVCache":
        def codes():
            return torch.zeros((Hkv, capacity, D // 2), dtype=torch.uint8, device=device)

        def scales():
            return torch.zeros((Hkv, capacity, D // 32), dtype=torch.float16, device=device)
        return KVCache(Hkv, D, capacity, codes(), scales(), codes(), scales())

    def struct(self) -> tern_kv_cache:
        return tern_kv_cache(self.Hkv, self.D, self.capacity, 0, self.k_codes.data_ptr(),
                             self.k_scales.data_ptr(), self.v_codes.data_ptr(), self.v_scales.data_ptr())


def tern_kv_append_q4_0(k: torch.Tensor, v: torch.Tensor, pos: int, cache: KVCache, stream=None):
    """Quantises one token's k and v (fp32 [Hkv, D]) into the cache at pos."""
    assert k.dtype == torch.float32 and v.dtype == torch.float32 and k.is_contiguous() and v.is_contiguous()
    c = cache.struct()
    _check(lib().tern_kv_append_q4_0(_ptr(k), _ptr(v), pos, ctypes.byref(c), _stream(stream)),
           "tern_kv_append_q4_0")


def tern_attention_workspace_bytes(Hq: int, L: int, cache: KVCache) -> int:
    b = ctypes.c_size_t()
    c = cache.struct()
    _check(lib().tern_attention_workspace_bytes(Hq, L, ctypes.byref(c), ctypes.byref(b)),
           "tern_attention_workspace_bytes")
    return b.value


def attention_workspace(Hq: int, L: int, cache: KVCache) -> torch.Tensor:
    n = tern_attention_workspace_bytes(Hq, L, cache)
    return torch.empty(((n + 15) // 16) * 4, dtype=torch.float32, device=cache.k_codes.device)


def tern_attention_decode_q4_0(q: torch.Tensor, cache: KVCache, L: int, out: torch.Tensor,
                               workspace: torch.Tensor, stream=None):
    """out fp32 [Hq, D] = attention of q fp32 [Hq, D] over the first L cached tokens."""
    assert q.dtype == torch.float32 and q.is_contiguous() and out.dtype == torch.float32
    Hq = q.shape[0]
    c = cache.struct()
    _check(lib().tern_attention_decode_q4_0(_ptr(q), Hq, ctypes.byref(c), L, _ptr(out), _ptr(workspace),
                                            workspace.numel() * workspace.element_size(),
                                            _stream(stream)), "tern_attention_decode_q4_0")


ENGINE_TENSOR_CORES, ENGINE_CUDA_CORES = 0, 1


def tern_debug_select_engine(engine: int):
    """Test hook: 0 = tensor-core GEMV engine, 1 = CUDA-core engine (default)."""
    _check(lib().tern_debug_select_engine(engine), "tern_debug_select_engine")


def tern_device_error(stream=None) -> int:
    code = ctypes.c_int32()
    _check(lib().tern_device_error(ctypes.byref(code), _stream(stream)), "tern_device_error")
    return code.value


def loaded_library_path() -> str:
    lib()
    return LIB_PATH
