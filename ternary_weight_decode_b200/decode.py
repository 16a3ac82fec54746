"""Batch-1 (and skinny multi-slot) decode step over a 27B-shaped ternary
layer stack, run through the C ABI and replayed as one CUDA graph.

The weight path of one decoder layer (Bonsai page, "Decode 为什么只能算一般":
per layer the Q/K/V/O projections, then the Hadamard-rotated FFN input shared
by the fused gate/up + SwiGLU kernel, then down; CUDA Graph replay).  Each
projection quantises its own fp32 input inside the kernel, from the block
statistics its producer wrote (4 launches per layer, 1 per step for the
statistics of the step input):

  1. tern_gemv_fused(Wqkv, x)                   -> qkv   (N = 7168 = q 5120 + k 1024 + v 1024)
  2. tern_gemv_fused(Wo, qkv[:, :5120], +x)     -> x     (attention stand-in: the q output)
  3. tern_gateup_swiglu_fused(Wg, Wu, H x)      -> h     (N = 17408, Hadamard-rotated input)
  4. tern_gemv_fused(Wd, h, +x)                 -> x     (K = 17408)

By default (M = 1 or 2) the projections run as the streamed kernels, which
need no statistics (each CTA quantises the input itself) and split every
matrix evenly over the SMs.  The fused form with statistics ("fused") and
the unfused form with separate act_quant_fwht launches ("unfused", 8 per
layer) are kept for comparison and for M > 2.

Attention and norms are not on this path (the pages give no detail); the
attention output is stood in by the q projection, and a weightless RMSNorm
before each block is folded into s_x only (TERN_QUANT_RMSNORM), which leaves
every int8 code unchanged and keeps the residual stream bounded over 64
layers.  Every step above runs in libtern's kernels.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

from . import synth, tern

HIDDEN = 5120
QKV = 7168
FFN = 17408


def layer_bytes(fmt: int, hidden: int = HIDDEN, qkv: int = QKV, ffn: int = FFN) -> int:
    """Algorithmic bytes of one layer: packed codes (canonical bytes per row)
    plus fp16 group scales, for the four projections."""
    def mat(N, K):
        return N * tern.tern_canonical_row_bytes(fmt, K) + 2 * N * ((K + 127) // 128)
    return mat(qkv, hidden) + mat(hidden, hidden) + 2 * mat(ffn, hidden) + mat(hidden, ffn)


@dataclass
class Layer:
    wqkv: tern.TernMatrix
    wo: tern.TernMatrix
    wg: tern.TernMatrix
    wu: tern.TernMatrix
    wd: tern.TernMatrix


def make_matrix(fmt: int, N: int, K: int, seed: int, stream: int, scratch: torch.Tensor):
    """Generates trits and scales on the device and packs them with tern_pack."""
    W = tern.TernMatrix.empty(fmt, N, K)
    trits = scratch[: N * K].view(N, K)
    synth.device_trits(seed, stream, N, K, out=trits)
    tern.tern_pack(fmt, trits, W)
    synth.device_scales(seed, stream + 1, N, (K + 127) // 128, out=W.scales)
    return W


@dataclass
class DecodeModel:
    fmt: int
    n_layers: int
    M: int = 1
    hidden: int = HIDDEN
    qkv: int = QKV
    ffn: int = FFN
    mode: str = "streamed"  # "streamed" (M <= 2), "fused" or "unfused"
    layers: list = field(default_factory=list)

    @property
    def fused(self) -> bool:
        return self.mode != "unfused"

    def build(self, seed_base: int = 0):
        scratch = torch.empty(max(self.qkv, self.ffn) * max(self.hidden, self.ffn),
                              dtype=torch.int8, device="cuda")
        for l in range(self.n_layers):
            s = seed_base + l
            self.layers.append(Layer(
                make_matrix(self.fmt, self.qkv, self.hidden, s, synth.stream_id(l, synth.PROJ_QKV), scratch),
                make_matrix(self.fmt, self.hidden, self.hidden, s, synth.stream_id(l, synth.PROJ_O), scratch),
                make_matrix(self.fmt, self.ffn, self.hidden, s, synth.stream_id(l, synth.PROJ_GATE), scratch),
                make_matrix(self.fmt, self.ffn, self.hidden, s, synth.stream_id(l, synth.PROJ_UP), scratch),
                make_matrix(self.fmt, self.hidden, self.ffn, s, synth.stream_id(l, synth.PROJ_DOWN), scratch),
            ))
        del scratch
        if self.mode == "streamed":
            assert self.M <= 2, "the streamed kernels take M = 1 or 2"
            for L in self.layers:
                for W in (L.wqkv, L.wo, L.wg, L.wu, L.wd):
                    W.retile_scales()
            self.ws = tern.stream_workspace(self.fmt, max(self.qkv, self.ffn, self.hidden), self.M, True)
        torch.cuda.synchronize()
        M = self.M
        ld_h = ((self.hidden + 15) // 16) * 16
        ld_f = ((self.ffn + 15) // 16) * 16
        self.x = torch.zeros((M, self.hidden), dtype=torch.float32, device="cuda")
        self.qkv_out = torch.zeros((M, self.qkv), dtype=torch.float32, device="cuda")
        self.h = torch.zeros((M, self.ffn), dtype=torch.float32, device="cuda")
        self.q_h = torch.zeros((M, ld_h), dtype=torch.int8, device="cuda")
        self.q_f = torch.zeros((M, ld_f), dtype=torch.int8, device="cuda")
        self.s = torch.zeros((4, M), dtype=torch.float32, device="cuda")
        self.st_x = tern.stats_buffer(M, self.hidden)
        self.st_qkv = tern.stats_buffer(M, self.qkv)
        self.st_x1 = tern.stats_buffer(M, self.hidden)
        self.st_h = tern.stats_buffer(M, self.ffn)
        return self

    def bytes_per_step(self) -> int:
        return self.n_layers * layer_bytes(self.fmt, self.hidden, self.qkv, self.ffn)

    def launches_per_step(self) -> int:
        if self.mode == "streamed":
            return 4 * self.n_layers
        return 4 * self.n_layers + 1 if self.mode == "fused" else 8 * self.n_layers

    def layer_step_streamed(self, L: Layer, keep=None):
        M = self.M
        rms, rot = tern.TERN_QUANT_RMSNORM, tern.TERN_QUANT_FWHT128
        if keep is not None:
            keep.append(("qkv_in", self.x.clone()))
        tern.tern_gemv_streamed(L.wqkv, self.x, self.qkv_out, self.ws, qflags=rms, M=M)
        if keep is not None:
            keep.append(("o_in", self.qkv_out.clone(), self.x.clone()))
        tern.tern_gemv_streamed(L.wo, self.qkv_out[:, : self.hidden], self.x, self.ws, qflags=rms,
                                residual=self.x, M=M)
        if keep is not None:
            keep.append(("ffn_in", self.x.clone()))
        tern.tern_gateup_swiglu_streamed(L.wg, L.wu, self.x, self.h, self.ws, qflags=rms | rot, M=M)
        if keep is not None:
            keep.append(("down_in", self.h.clone(), self.x.clone()))
        tern.tern_gemv_streamed(L.wd, self.h, self.x, self.ws, qflags=rms, residual=self.x, M=M)

    def layer_step_fused(self, L: Layer, keep=None):
        M = self.M
        rms, rot = tern.TERN_QUANT_RMSNORM, tern.TERN_QUANT_FWHT128
        if keep is not None:
            keep.append(("qkv_in", self.x.clone()))
        tern.tern_gemv_fused(L.wqkv, self.x, self.st_x, self.qkv_out, qflags=rms,
                             y_stats=self.st_qkv, M=M)
        if keep is not None:
            keep.append(("o_in", self.qkv_out.clone(), self.x.clone()))
        tern.tern_gemv_fused(L.wo, self.qkv_out[:, : self.hidden], self.st_qkv, self.x, qflags=rms,
                             residual=self.x, y_stats=self.st_x1, M=M)
        if keep is not None:
            keep.append(("ffn_in", self.x.clone()))
        tern.tern_gateup_swiglu_fused(L.wg, L.wu, self.x, self.st_x1, self.h, qflags=rms | rot,
                                      h_stats=self.st_h, M=M)
        if keep is not None:
            keep.append(("down_in", self.h.clone(), self.x.clone()))
        tern.tern_gemv_fused(L.wd, self.h, self.st_h, self.x, qflags=rms, residual=self.x,
                             y_stats=self.st_x, M=M)

    def layer_step(self, L: Layer, keep=None):
        M = self.M
        norm = tern.TERN_QUANT_RMSNORM
        tern.act_quant_fwht(self.x, self.q_h, self.s[0], 0, flags=norm)
        tern.tern_gemv(L.wqkv, self.q_h, self.s[0], self.qkv_out, M=M)
        tern.act_quant_fwht(self.qkv_out, self.q_h, self.s[1], 0, K=self.hidden, flags=norm)
        if keep is not None:
            keep.append(("o_in", self.q_h.clone(), self.s[1].clone(), self.x.clone()))
        tern.tern_gemv(L.wo, self.q_h, self.s[1], self.x, residual=self.x, M=M)
        tern.act_quant_fwht(self.x, self.q_h, self.s[2], 128, flags=norm)
        if keep is not None:
            keep.append(("ffn_in", self.q_h.clone(), self.s[2].clone()))
        tern.tern_gateup_swiglu(L.wg, L.wu, self.q_h, self.s[2], self.h, M=M)
        tern.act_quant_fwht(self.h, self.q_f, self.s[3], 0, flags=norm)
        if keep is not None:
            keep.append(("down_in", self.q_f.clone(), self.s[3].clone(), self.x.clone(), self.h.clone()))
        tern.tern_gemv(L.wd, self.q_f, self.s[3], self.x, residual=self.x, M=M)

    def step(self, keep=None):
        if self.mode == "streamed":
            for L in self.layers:
                self.layer_step_streamed(L, keep)
        elif self.mode == "fused":
            tern.tern_act_stats(self.x, self.st_x)
            for L in self.layers:
                self.layer_step_fused(L, keep)
        else:
            for L in self.layers:
                self.layer_step(L, keep)

    def capture(self) -> torch.cuda.CUDAGraph:
        """One CUDA graph holding the whole step."""
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.step()  # warm: sets kernel attributes outside capture
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.step()
        return g
