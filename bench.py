#!/usr/bin/env python3
"""Benchmark of the ternary decode weight stream on B200.

Headline step = one batch-1 decode step of a 64-layer 27B-shaped ternary
layer stack, replayed as one CUDA graph.  Per layer four kernels (the
streamed GEMV entry points, which quantise their fp32 input themselves): QKV
GEMV, O GEMV + residual, fused gate/up + SwiGLU with the 128-point Hadamard
rotation, down GEMV + residual.  The metric is the weight stream's
algorithmic bytes (canonical packed codes + fp16 group scales) per second,
with the decode-step rate (tok/s-equivalent) beside it.

The same JSON line carries the other workloads under "configs":
  c1  single GEMV K = N = 256, M = 1 (microseconds per call);
  c2  one 27B-shaped layer, base-3, 2-bit and bit-plane, rotating 8
      independent layers so the weights never sit in L2, with the
      per-projection split;
  c3_2bit, c3_bitplane  the 64-layer step in the other two formats;
  c4  gate/up + SwiGLU and down at M = 1, 2, 4, 8, 16 token rows (GB/s, TOPS),
      each format;
  c5  prefill GEMM, (K, N) = (5120, 17408) and (17408, 5120), M = 512 / 2048 / 8192,
      each format;
  c6  multi-token verify: the gate and down GEMMs at M = 16 .. 128 on the tensor cores;
  c7  decode attention over a Q4_0 KV cache at 4K / 16K / 64K tokens;
each with a bounded sample of the CPU oracle timed on this host.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--fmt base3|2bit|bitplane] [--layers 64] [--M 1] [--quick]
    python bench.py --attention 4096 65536      # c7 alone

N > 1 runs N independent replicas (one process per GPU, launched by
torch.distributed.run): the path has no cross-GPU exchange step.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ternary GEMV HBM GB/s (% of 8 TB/s) & decode tok/s-equiv, 27B-shape, batch 1"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
HIDDEN, QKV, FFN = 5120, 7168, 17408
ROT_COPIES = 8  # independent layers cycled through so that weights never sit in L2


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--fmt", choices=["base3", "2bit", "bitplane"], default="base3")
    ap.add_argument("--layers", type=int, default=64)
    ap.add_argument("--M", type=int, default=1)
    ap.add_argument("--mode", choices=["auto", "streamed", "fused", "unfused"], default="auto",
                    help="decode-step kernels (auto: streamed for M <= 2, else fused)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle sample of the headline workload")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill GEMM (c5)")
    ap.add_argument("--quick", action="store_true", help="headline step only (no c1..c5)")
    ap.add_argument("--attention", type=int, nargs="+", default=None, metavar="L",
                    help="decode attention (c7) alone at these context lengths, one GPU; "
                         "prints its JSON and no decode step")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def int8_peak():
    """Dense int8 tensor peak: the measured bf16 burst figure x the nominal
    int8 / bf16 ratio (4.5 / 2.25 PFLOP/s), else the recipe's fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return 2.0 * float(json.load(f)["bf16_tflops"]), "measured bf16 x 2"
    except Exception:
        return 2.0 * 1590.0, "fallback bf16 x 2"


FMT_NAMES = {"base3": 0, "2bit": 1, "bitplane": 2}


def fmt_id_of(name: str) -> int:
    return FMT_NAMES[name]


def fmt_label(fmt: int) -> str:
    return {0: "base-3", 1: "2-bit", 2: "bit-plane"}[fmt]


def canonical_row_bytes(fmt: int, K: int) -> int:
    """Bytes per row of the canonical encodings: 5 trits a byte (base-3), 4
    (2-bit), or a nonzero and a sign plane of ceil(K/8) bytes each
    (bit-plane); the same rule as the oracle's and the library's row-byte
    calls."""
    return {0: (K + 4) // 5, 1: (K + 3) // 4, 2: 2 * ((K + 7) // 8)}[fmt]


def mat_bytes(fmt: int, N: int, K: int) -> int:
    """Algorithmic bytes of one matrix: canonical codes + fp16 group scales."""
    return N * canonical_row_bytes(fmt, K) + 2 * N * ((K + 127) // 128)


def layer_bytes(fmt: int) -> int:
    return (mat_bytes(fmt, QKV, HIDDEN) + mat_bytes(fmt, HIDDEN, HIDDEN) +
            2 * mat_bytes(fmt, FFN, HIDDEN) + mat_bytes(fmt, HIDDEN, FFN))


def ffn_bytes(fmt: int) -> int:
    return 2 * mat_bytes(fmt, FFN, HIDDEN) + mat_bytes(fmt, HIDDEN, FFN)


FFN_MACS = 3 * FFN * HIDDEN  # gate, up, down: multiply-accumulates per token row


def dist_setup(n_gpus, backend="nccl"):
    """One process per GPU (torch.distributed.run sets RANK / WORLD_SIZE /
    LOCAL_RANK / MASTER_*).  The replicas share no data-path collective; the
    process group only carries the barrier and the max-over-ranks timing.
    A short timeout makes ranks that wait for a missing peer fail."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(values, world, device="cuda"):
    """Element-wise max of per-rank timings (every rank calls it, in the same
    order); a single process returns them unchanged."""
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def replica_value(bytes_per_step, ms_per_step, world):
    """Whole-job throughput of N weak-scaled replicas: every rank streams
    bytes_per_step per step; the step time is the slowest rank's."""
    return world * bytes_per_step / (ms_per_step * 1e-3) / 1e9


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def source_digest() -> str:
    h = hashlib.sha256()
    for rel in ("ternary_weight_decode_b200/csrc/tern_gemv_stream.cuh",
                "ternary_weight_decode_b200/csrc/tern_gemv_common.cuh",
                "ternary_weight_decode_b200/csrc/tern_common.cuh"):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_record(kernel: str, fmt: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source; otherwise None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        r = rec[f"{kernel}/{fmt}"]
        if r.get("source_digest") == source_digest():
            return r["dram_bytes_per_launch"]
    except Exception:
        pass
    return None


# ---------------------------------------------------------------- CPU oracle samples
def _weights(fmt_dev_ok: bool, seed: int, stream: int, N: int, K: int, rows=None):
    """(trits, scales) of one synthetic matrix on the host.  Our arm draws the
    trits with the device generator (the same definition as the host one,
    checked bit for bit by the tests); the reference arm with the host one."""
    import numpy as np
    from ternary_weight_decode_b200 import synth
    G = (K + 127) // 128
    if rows is None:
        rows = np.arange(N)
    if fmt_dev_ok:
        w = synth.device_trits(seed, stream, N, K).cpu().numpy()[rows]
    else:
        w = synth.trits_rows(seed, stream, rows, K)
    return w, synth.scales_rows(seed, stream + 1, rows, G)


def oracle_layer(W, x0):
    """One decode layer through the CPU oracle (the chain the step runs).
    W: dict of (trits, scales).  Returns (seconds of oracle time, x out)."""
    import numpy as np
    import oracle
    t0 = time.perf_counter()
    x = x0.astype(np.float64)
    q, s = oracle.act_quant(x.astype(np.float32), rmsnorm=True)
    qkv = oracle.gemv(*W["qkv"], q, s)
    q, s = oracle.act_quant(qkv[:, :HIDDEN].astype(np.float32), rmsnorm=True)
    x = x + oracle.gemv(*W["o"], q, s)
    q, s = oracle.act_quant(x.astype(np.float32), fwht_block=128, rmsnorm=True)
    h = oracle.gateup_swiglu(W["g"][0], W["g"][1], W["u"][0], W["u"][1], q, s)
    q, s = oracle.act_quant(h.astype(np.float32), rmsnorm=True)
    x = x + oracle.gemv(*W["d"], q, s)
    return time.perf_counter() - t0, x


def layer_weights(layer: int, device_gen: bool):
    from ternary_weight_decode_b200 import synth
    def one(N, K, proj):
        return _weights(device_gen, layer, synth.stream_id(layer, proj), N, K)
    return {"qkv": one(QKV, HIDDEN, synth.PROJ_QKV), "o": one(HIDDEN, HIDDEN, synth.PROJ_O),
            "g": one(FFN, HIDDEN, synth.PROJ_GATE), "u": one(FFN, HIDDEN, synth.PROJ_UP),
            "d": one(HIDDEN, FFN, synth.PROJ_DOWN)}


def cpu_threads():
    import oracle
    cores = len(os.sched_getaffinity(0))
    oracle.set_threads(cores)
    return cores


def cpu_decode_sample(fmt: int, M: int, target_s: float, device_gen: bool):
    """Decode layers of the headline workload through the oracle until about
    target_s seconds of oracle time (at most 64 layers)."""
    import numpy as np
    from ternary_weight_decode_b200 import synth
    cores = cpu_threads()
    x = synth.activations(0, M, HIDDEN).astype(np.float32)
    tb, tt, layers = 0, 0.0, 0
    while tt < target_s and layers < 64:
        dt, x = oracle_layer(layer_weights(layers, device_gen), x)
        tb += layer_bytes(fmt)
        tt += dt
        layers += 1
    return {"value": tb / tt / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "ms_per_layer": 1e3 * tt / layers,
            "sample": f"{layers} of 64 decode layers (M={M}), all 4 projections, plain-C fp64 "
                      f"oracle with OpenMP over output rows; {tt:.1f} s of oracle time"}


def cpu_single_gemv():
    """Config 1 through the oracle: act_quant + gemv, K = N = 256, repeated."""
    import numpy as np
    import oracle
    from ternary_weight_decode_b200 import synth
    cores = cpu_threads()
    w, sw = synth.trits(0, 0, 256, 256), synth.scales(0, 1, 256, 2)
    x = synth.activations(0, 1, 256).astype(np.float32)
    n, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < 0.5:
        q, s = oracle.act_quant(x)
        oracle.gemv(w, sw, q, s)
        n += 1
    dt = (time.perf_counter() - t0) / n
    return {"us_per_call": dt * 1e6, "GB/s": mat_bytes(0, 256, 256) / dt / 1e9, "cores": cores,
            "kind": "oracle", "sample": f"{n} calls of act_quant + gemv"}


def cpu_ffn_sweep(fmt: int, Ms):
    """Config 4 through the oracle: gate/up + SwiGLU and down of one layer."""
    import numpy as np
    import oracle
    from ternary_weight_decode_b200 import synth
    cores = cpu_threads()
    W = layer_weights(0, True)
    out = []
    for M in Ms:
        x = synth.activation_rows(range(1000, 1000 + M), HIDDEN).astype(np.float32)
        t0 = time.perf_counter()
        q, s = oracle.act_quant(x, fwht_block=128, rmsnorm=True)
        h = oracle.gateup_swiglu(W["g"][0], W["g"][1], W["u"][0], W["u"][1], q, s)
        q, s = oracle.act_quant(h.astype(np.float32), rmsnorm=True)
        oracle.gemv(*W["d"], q, s)
        dt = time.perf_counter() - t0
        out.append({"M": M, "ms": dt * 1e3, "GB/s": ffn_bytes(fmt) / dt / 1e9,
                    "TOPS": 2.0 * M * FFN_MACS / dt / 1e12})
    return {"cores": cores, "kind": "oracle", "results": out,
            "sample": "one layer's gate/up + SwiGLU + down per M"}


def cpu_prefill(M=512, rows=512):
    """Config 5 at M = 512 through the oracle, on a sample of weight rows."""
    import numpy as np
    import oracle
    from ternary_weight_decode_b200 import synth
    cores = cpu_threads()
    out = []
    for K, N in ((HIDDEN, FFN), (FFN, HIDDEN)):
        w, sw = _weights(True, 977, 5, N, K, rows=np.arange(rows))
        x = synth.activation_rows(range(2000, 2000 + M), K).astype(np.float32)
        q, s = oracle.act_quant(x)
        t0 = time.perf_counter()
        oracle.gemv(w, sw, q, s)
        dt = time.perf_counter() - t0
        out.append({"K": K, "N": N, "M": M, "rows_sampled": rows,
                    "TOPS": 2.0 * M * rows * K / dt / 1e12})
    return {"cores": cores, "kind": "oracle", "results": out,
            "sample": f"M={M} tokens x {rows} of the N weight rows, plain-C fp64 gemv"}


def cpu_attention(L=4096, Hq=40, Hkv=8, D=128):
    """Config 7 through the oracle: one token's attention over a Q4_0 cache
    of L tokens (40 query heads over 8 KV heads), repeated for about a second."""
    import numpy as np
    import oracle
    cores = cpu_threads()
    rng = np.random.default_rng(L)
    kd, kq = oracle.q4_0_quantize(rng.standard_normal((Hkv, L, D)).astype(np.float32))
    vd, vq = oracle.q4_0_quantize(rng.standard_normal((Hkv, L, D)).astype(np.float32))
    q = rng.standard_normal((Hq, D)).astype(np.float32)
    n, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < 1.0:
        oracle.attention_decode(q, kd, kq, vd, vq)
        n += 1
    dt = (time.perf_counter() - t0) / n
    nbytes = 2 * Hkv * L * (D // 2 + 2 * (D // 32))
    return {"L": L, "us_per_call": dt * 1e6, "GB/s": nbytes / dt / 1e9, "cores": cores, "kind": "oracle",
            "sample": f"{n} calls of the fp64 oracle at L = {L}"}


# ---------------------------------------------------------------- reference arm
def run_reference(args, world, rank):
    """The oracle timed on this host's cores, on the headline workload: each
    step is one decode layer (M = args.M) of the 64-layer stream, weights
    drawn by the host generator.  Loads nothing of the CUDA library."""
    if rank != 0:
        return 0
    import numpy as np
    from ternary_weight_decode_b200 import synth
    fmt = fmt_id_of(args.fmt)
    cores = cpu_threads()
    pool = [layer_weights(i, False) for i in range(min(2, max(1, args.steps + args.warmup)))]
    x = synth.activations(0, args.M, HIDDEN).astype(np.float32)
    for i in range(args.warmup):
        _, x = oracle_layer(pool[i % len(pool)], x)
    tt = 0.0
    for i in range(args.steps):
        dt, x = oracle_layer(pool[(args.warmup + i) % len(pool)], x)
        tt += dt
    value = args.steps * layer_bytes(fmt) / tt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 64e3 * tt / args.steps,
        "step_unit": "one 64-layer decode step, extrapolated from the per-layer oracle time "
                     "(each timed step runs one layer)",
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(args),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step = one of the 64 decode layers (M={args.M}) through "
                                   f"the plain-C fp64 oracle, OpenMP over output rows"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(args):
    return {"workload": f"64-layer 27B-shape ternary decode weight stream, {args.fmt} codes + fp16/128 "
                        f"scales, hidden 5120, qkv 7168, ffn 17408, batch {args.M}, one CUDA graph"
                        if args.layers == 64 else
                        f"{args.layers}-layer 27B-shape ternary decode stream ({args.fmt}), batch {args.M}",
            "layers": args.layers, "format": args.fmt, "batch": args.M,
            "kernels": args.mode if args.mode != "auto" else ("streamed" if args.M <= 2 else "fused"),
            "l2": "inputs larger than L2: each step streams every layer's weights once"}


# ---------------------------------------------------------------- GPU timing helpers
def graph_ms(fn, reps=20):
    """fn captured once into a CUDA graph, replayed reps times after 3
    warm-up replays; CUDA events on the replay stream.  Returns ms per replay."""
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # sets kernel attributes outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    e1.synchronize()
    del g
    return e0.elapsed_time(e1) / reps


def single_gemv(fmt):
    """c1: K = N = 256, M = 1, seed 0, the streamed decode kernel."""
    import numpy as np
    import torch
    from ternary_weight_decode_b200 import decode, synth, tern
    scratch = torch.empty(256 * 256, dtype=torch.int8, device="cuda")
    W = decode.make_matrix(fmt, 256, 256, seed=0, stream=0, scratch=scratch).retile_scales()
    x = torch.from_numpy(synth.activations(0, 1, 256).astype(np.float32)).cuda()
    y = torch.empty((1, 256), dtype=torch.float32, device="cuda")
    ws = tern.stream_workspace(fmt, 256, 1, False)
    calls = 200
    ms = graph_ms(lambda: [tern.tern_gemv_streamed(W, x, y, ws) for _ in range(calls)], reps=10)
    us = ms * 1e3 / calls
    return {"workload": "single ternary GEMV, K=256, N=256, M=1, base-3, seed 0, streamed kernel, "
                        f"{calls} back-to-back calls in one graph",
            "us_per_call": us, "GB/s": mat_bytes(fmt, 256, 256) / (us * 1e-6) / 1e9,
            "bound": "launch latency (14,336 algorithmic bytes per call)"}


def layer_configs(model, fmt, peak):
    """c2: one layer, rotating ROT_COPIES layers of the built model, whole
    layer and per projection (8 launches of one kind per graph)."""
    from ternary_weight_decode_b200 import tern
    L8 = model.layers[:ROT_COPIES]
    M = model.M
    rms, rot = tern.TERN_QUANT_RMSNORM, tern.TERN_QUANT_FWHT128

    def whole():
        for L in L8:
            model.layer_step_streamed(L)
    per_layer = graph_ms(whole) / len(L8)
    projs = {
        "qkv": (lambda L: tern.tern_gemv_streamed(L.wqkv, model.x, model.qkv_out, model.ws, qflags=rms, M=M),
                mat_bytes(fmt, QKV, HIDDEN)),
        "o": (lambda L: tern.tern_gemv_streamed(L.wo, model.qkv_out[:, :HIDDEN], model.x, model.ws,
                                                qflags=rms, residual=model.x, M=M),
              mat_bytes(fmt, HIDDEN, HIDDEN)),
        "gateup_swiglu": (lambda L: tern.tern_gateup_swiglu_streamed(L.wg, L.wu, model.x, model.h, model.ws,
                                                                     qflags=rms | rot, M=M),
                          2 * mat_bytes(fmt, FFN, HIDDEN)),
        "down": (lambda L: tern.tern_gemv_streamed(L.wd, model.h, model.x, model.ws, qflags=rms,
                                                   residual=model.x, M=M),
                 mat_bytes(fmt, HIDDEN, FFN)),
    }
    split = {}
    for name, (call, nbytes) in projs.items():
        ms = graph_ms(lambda: [call(L) for L in L8]) / len(L8)
        gbs = nbytes / (ms * 1e-3) / 1e9
        split[name] = {"us": ms * 1e3, "GB/s": gbs, "frac": gbs / peak}
    lb = layer_bytes(fmt)
    return {"workload": f"one 27B-shaped decode layer ({fmt_label(fmt)}), M={M}, "
                        f"{ROT_COPIES} independent layers cycled (weights never in L2)",
            "us_per_layer": per_layer * 1e3, "bytes_per_layer": lb,
            "GB/s": lb / (per_layer * 1e-3) / 1e9, "frac": lb / (per_layer * 1e-3) / 1e9 / peak,
            "per_projection": split}


def ffn_sweep(model, fmt, peak, Ms=(1, 2, 4, 8, 16)):
    """c4: gate/up + SwiGLU and down of ROT_COPIES layers at M token rows:
    the streamed kernels at M <= 2, the fused kernels (quantisation from the
    producer's block statistics) at every M."""
    import numpy as np
    import torch
    from ternary_weight_decode_b200 import synth, tern
    rms, rot = tern.TERN_QUANT_RMSNORM, tern.TERN_QUANT_FWHT128
    L8 = model.layers[:ROT_COPIES]
    fb = ffn_bytes(fmt)
    res = []
    for M in Ms:
        x = torch.from_numpy(synth.activation_rows(range(1000, 1000 + M), HIDDEN)
                             .astype(np.float32)).cuda()
        h = torch.zeros((M, FFN), dtype=torch.float32, device="cuda")
        kinds = {}
        if M <= 2:
            ws = tern.stream_workspace(fmt, FFN, M, True)

            def streamed():
                for L in L8:
                    tern.tern_gateup_swiglu_streamed(L.wg, L.wu, x, h, ws, qflags=rms | rot, M=M)
                    tern.tern_gemv_streamed(L.wd, h, x, ws, qflags=rms, residual=x, M=M)
            kinds["streamed"] = streamed
        st_x, st_h = tern.stats_buffer(M, HIDDEN), tern.stats_buffer(M, FFN)

        def fused():
            tern.tern_act_stats(x, st_x)
            for L in L8:
                tern.tern_gateup_swiglu_fused(L.wg, L.wu, x, st_x, h, qflags=rms | rot, h_stats=st_h, M=M)
                tern.tern_gemv_fused(L.wd, h, st_h, x, qflags=rms, residual=x, y_stats=st_x, M=M)
        kinds["fused"] = fused
        for kind, fn in kinds.items():
            x.copy_(torch.from_numpy(synth.activation_rows(range(1000, 1000 + M), HIDDEN)
                                     .astype(np.float32)))
            ms = graph_ms(fn) / len(L8)
            gbs = fb / (ms * 1e-3) / 1e9
            res.append({"M": M, "kernels": kind, "us_per_layer_slice": ms * 1e3, "GB/s": gbs,
                        "frac": gbs / peak, "TOPS": 2.0 * M * FFN_MACS / (ms * 1e-3) / 1e12})
    best = {}
    for r in res:
        if r["M"] not in best or r["GB/s"] > best[r["M"]]["GB/s"]:
            best[r["M"]] = r
    return {"workload": f"gate/up + SwiGLU and down of the 27B-shaped layer "
                        f"({fmt_label(fmt)}), {ROT_COPIES} layers cycled, "
                        f"independent per-row quantisation",
            "bytes_per_layer_slice": fb, "results": res,
            "faster_kernels_by_M": {str(M): r["kernels"] for M, r in sorted(best.items())}}


def verify_sweep(model, fmt, Ms=(4, 8, 16, 32, 64, 128)):
    """c6: multi-token verify on the tensor cores -- tern_gemm of the gate
    (K = 5120, N = 17408) and down (K = 17408, N = 5120) matrices of
    ROT_COPIES layers (weights never in L2) at M token rows (64- or
    128-token tiles, a cluster split of K for down).  M = 4 and 8 place the
    crossover with the CUDA-core kernels of c4 (GB/s of weights)."""
    import torch
    from ternary_weight_decode_b200 import tern
    L8 = model.layers[:ROT_COPIES]
    peak8, _ = int8_peak()
    hbm, _ = peaks()
    nbytes = mat_bytes(fmt, FFN, HIDDEN) + mat_bytes(fmt, HIDDEN, FFN)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(99)
    res = []
    for M in Ms:
        qg = torch.randint(-127, 128, (M, HIDDEN), dtype=torch.int8, device="cuda", generator=gen)
        qd = torch.randint(-127, 128, (M, FFN), dtype=torch.int8, device="cuda", generator=gen)
        s = torch.rand(M, device="cuda", generator=gen) * 0.01 + 0.001
        yg = torch.empty((M, FFN), dtype=torch.float32, device="cuda")
        yd = torch.empty((M, HIDDEN), dtype=torch.float32, device="cuda")

        def run():
            for L in L8:
                tern.tern_gemm(L.wg, qg, s, yg)
                tern.tern_gemm(L.wd, qd, s, yd)
        ms = graph_ms(run) / len(L8)
        gbs = nbytes / (ms * 1e-3) / 1e9
        tops = 2.0 * M * 2 * FFN * HIDDEN / (ms * 1e-3) / 1e12
        res.append({"M": M, "us_gate_plus_down": ms * 1e3, "GB/s": gbs, "frac_hbm": gbs / hbm,
                    "TOPS": tops, "frac_int8": tops / peak8})
    return {"workload": f"tern_gemm on the gate (5120 -> 17408) and down (17408 -> 5120) matrices "
                        f"({fmt_label(fmt)}), {ROT_COPIES} layers cycled, int8 "
                        f"activations, M token rows (64/128-token tiles)",
            "bytes_per_pair": nbytes, "results": res}


def attention_sweep(Ls=(4096, 16384, 65536), Hq=40, Hkv=8, D=128):
    """c7: decode attention of one token over a Q4_0 KV cache of L tokens,
    the 27B layer's 40 query heads over 8 KV heads of 128 (the cache
    filled by tern_kv_append_q4_0).  Bytes = the cache read once (codes +
    scales of K and V).  One graph holds one call per cache over enough
    independent caches (about 160 MB) that none is still in L2 when it is
    read again; time per call = graph time / calls."""
    import torch
    from ternary_weight_decode_b200 import tern
    hbm, _ = peaks()
    res = []
    for L in Ls:
        nbytes = 2 * Hkv * L * (D // 2 + 2 * (D // 32))
        ncache = max(2, -(-160_000_000 // nbytes))
        cache = tern.KVCache.empty(Hkv, D, L)
        g = torch.Generator(device="cuda")
        g.manual_seed(L)
        kv = torch.randn((2, min(L, 64), Hkv, D), device="cuda", generator=g)
        for t in range(min(L, 64)):
            tern.tern_kv_append_q4_0(kv[0, t], kv[1, t], t, cache)
        # the rest of the cache: copies of the appended rows (the kernel's cost does not depend on values)
        reps = (L + 63) // 64
        for arr in (cache.k_codes, cache.k_scales, cache.v_codes, cache.v_scales):
            arr.copy_(arr[:, :64].repeat(1, reps, 1)[:, :L])
        caches = [cache] + [tern.KVCache(cache.Hkv, cache.D, cache.capacity, cache.k_codes.clone(),
                                         cache.k_scales.clone(), cache.v_codes.clone(), cache.v_scales.clone())
                            for _ in range(ncache - 1)]
        q = torch.randn((Hq, D), device="cuda", generator=g)
        out = torch.empty((Hq, D), dtype=torch.float32, device="cuda")
        ws = tern.attention_workspace(Hq, L, cache)
        ms = graph_ms(lambda: [tern.tern_attention_decode_q4_0(q, c, L, out, ws) for c in caches], reps=10)
        ms /= ncache
        res.append({"L": L, "us": ms * 1e3, "GB/s": nbytes / (ms * 1e-3) / 1e9,
                    "frac_hbm": nbytes / (ms * 1e-3) / 1e9 / hbm, "cache_bytes": nbytes,
                    "caches_cycled": ncache})
        del cache, caches, kv
    return {"workload": f"decode attention over a Q4_0 KV cache, {Hq} query heads / {Hkv} KV heads of {D}, "
                        f"one token, split-context flash decoding + ordered merge (2 launches), "
                        f"caches cycled so that none is in L2",
            "results": res}


def prefill_gemm(fmt, K, N, Ms=(512, 2048, 8192), reps=10):
    """c5: tern_gemm at prefill batch sizes; TOPS = 2 M N K / device time
    (CUDA events, after warm-up).  W (17.8 MB base-3) stays L2-resident
    across the token tiles, as in any prefill; the kernel is bound by the
    tensor cores and its CUDA-core epilogue, not by HBM."""
    import torch
    from ternary_weight_decode_b200 import decode, tern
    scratch = torch.empty(N * K, dtype=torch.int8, device="cuda")
    W = decode.make_matrix(fmt, N, K, seed=977, stream=5, scratch=scratch)
    del scratch
    peak, kind = int8_peak()
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1234)
    res = []
    for M in Ms:
        q = torch.randint(-127, 128, (M, K), dtype=torch.int8, device="cuda", generator=gen)
        s = torch.rand(M, device="cuda", generator=gen) * 0.01 + 0.001
        y = torch.empty((M, N), dtype=torch.float32, device="cuda")
        for _ in range(3):
            tern.tern_gemm(W, q, s, y)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            tern.tern_gemm(W, q, s, y)
        e1.record()
        e1.synchronize()
        t = e0.elapsed_time(e1) / reps * 1e-3
        tops = 2.0 * M * N * K / t / 1e12
        res.append({"M": M, "ms": t * 1e3, "TOPS": tops, "frac": tops / peak})
        del q, s, y
    return {"workload": f"tern_gemm, K={K}, N={N}, {fmt_label(fmt)}, int8 activations, "
                        f"fp16/128 group scales",
            "unit": "TOPS", "peak": peak, "peak_kind": kind, "results": res}


def other_format(name, x0, steps, peak, stream):
    """c3 (the 64-layer step), c2 and c4 in another weight format: the A/B
    of base-3, 2-bit and bit-plane on the same box and kernels."""
    import torch
    from ternary_weight_decode_b200 import decode
    fmt = fmt_id_of(name)
    om = decode.DecodeModel(fmt, 64, M=1, mode="streamed").build(seed_base=0)
    om.x.copy_(x0)
    g2 = om.capture()
    for _ in range(3):
        g2.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        g2.replay()
    e1.record(stream)
    e1.synchronize()
    oms = e0.elapsed_time(e1) / steps
    del g2
    ob = om.bytes_per_step()
    out = {"c3_" + name: {"workload": f"64-layer 27B-shape decode step, {fmt_label(fmt)}, batch 1, one CUDA graph",
                          "ms_per_step": oms, "GB/s": ob / (oms * 1e-3) / 1e9,
                          "frac": ob / (oms * 1e-3) / 1e9 / peak, "tok_s_equiv": 1e3 / oms,
                          "bytes_per_step": ob},
           "c2_" + name: layer_configs(om, fmt, peak)}
    out["c4_" + name] = ffn_sweep(om, fmt, peak)
    del om
    return out


# ---------------------------------------------------------------- our arm
def main():
    args = parse()
    world, rank, local = dist_setup(args.gpus)
    if args.impl == "reference":
        rc = run_reference(args, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return rc

    import numpy as np
    import torch
    from ternary_weight_decode_b200 import decode, synth, tern

    torch.cuda.set_device(local)
    if args.attention:
        if world > 1:
            raise SystemExit("--attention runs on one GPU")
        print(json.dumps({"config": "c7_attention", **attention_sweep(Ls=tuple(args.attention))}))
        return 0
    fmt_id = fmt_id_of(args.fmt)
    mode = args.mode if args.mode != "auto" else ("streamed" if args.M <= 2 else "fused")
    model = decode.DecodeModel(fmt_id, args.layers, M=args.M, mode=mode).build(seed_base=0)
    x0 = torch.from_numpy(synth.activations(0, args.M, decode.HIDDEN).astype(np.float32))
    x0_host = x0.pin_memory()
    out_host = torch.empty_like(x0_host).pin_memory()
    model.x.copy_(x0)
    graph = model.capture()
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    # ---- dominant kernel alone: fused gate/up + SwiGLU over every layer
    gu_bytes = 2 * mat_bytes(fmt_id, FFN, HIDDEN)
    rms, rot = tern.TERN_QUANT_RMSNORM, tern.TERN_QUANT_FWHT128

    def gateup_all():
        for L in model.layers:
            if mode == "streamed":
                tern.tern_gateup_swiglu_streamed(L.wg, L.wu, model.x, model.h, model.ws,
                                                 qflags=rms | rot, M=args.M)
            elif mode == "fused":
                tern.tern_gateup_swiglu_fused(L.wg, L.wu, model.x, model.st_x1, model.h,
                                              qflags=rms | rot, M=args.M)
            else:
                tern.tern_gateup_swiglu(L.wg, L.wu, model.q_h, model.s[2], model.h, M=args.M)
    if mode == "fused":
        tern.tern_act_stats(model.x, model.st_x1)
    gu_ms = graph_ms(gateup_all, reps=5) / len(model.layers)
    model.x.copy_(x0)

    # ---- warm-up
    for _ in range(max(args.warmup, 3)):
        graph.replay()
    torch.cuda.synchronize()

    # ---- timed region (device time, max over ranks)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        graph.replay()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = t0.elapsed_time(t1) / args.steps

    # ---- end to end through the public API: host input in, host result out, every step
    h2d = x0_host.numel() * 4
    d2h = out_host.numel() * 4
    torch.cuda.synchronize()
    barrier()
    t2, t3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t2.record(stream)
    for _ in range(args.steps):
        model.x.copy_(x0_host, non_blocking=True)
        graph.replay()
        out_host.copy_(model.x, non_blocking=True)
    t3.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = t2.elapsed_time(t3) / args.steps
    clk = clocks.stop()

    ms, e2e_ms, gu_ms = max_over_ranks([ms, e2e_ms, gu_ms], world)

    err = tern.tern_device_error()
    step_bytes = model.bytes_per_step()
    assert step_bytes == args.layers * layer_bytes(fmt_id)
    value = replica_value(step_bytes, ms, world)
    e2e_val = replica_value(step_bytes, e2e_ms, world)
    peak, peak_kind = peaks()
    gu_achieved = gu_bytes / (gu_ms * 1e-3) / 1e9
    out_ok = bool(torch.isfinite(model.x).all().item())
    del graph

    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return 0

    configs = {}
    cpu = None
    if world == 1 and not args.quick:
        if mode == "streamed" and args.M == 1 and args.layers >= ROT_COPIES:
            configs["c2_" + args.fmt] = layer_configs(model, fmt_id, peak)
            configs["c4_" + args.fmt] = ffn_sweep(model, fmt_id, peak)
            configs["c6_verify_" + args.fmt] = verify_sweep(model, fmt_id)
        configs["c1"] = single_gemv(0)
        del model
        torch.cuda.empty_cache()
        if mode == "streamed" and args.M == 1 and args.layers == 64:
            for other in [f for f in FMT_NAMES if f != args.fmt]:
                configs.update(other_format(other, x0, args.steps, peak, stream))
                torch.cuda.empty_cache()
        if not args.no_prefill:
            configs["c5"] = [prefill_gemm(f, K, N) for f in (0, 1, 2)
                             for K, N in ((HIDDEN, FFN), (FFN, HIDDEN))]
        configs["c7_attention"] = attention_sweep()
        if not args.no_cpu_baseline:
            configs["cpu_oracle"] = {"c1": cpu_single_gemv(), "c4": cpu_ffn_sweep(fmt_id, (1, 2, 4, 8, 16)),
                                     "c5": cpu_prefill(), "c7": cpu_attention()}
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_decode_sample(fmt_id, args.M, args.cpu_seconds, device_gen=True)

    line = {
        "metric": METRIC,
        "value": value,
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": max(args.warmup, 3),
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "u8",
        "data": "synthetic",
        "config": workload_config(args),
        "pct_of_8TBs": 100.0 * value / world / NOMINAL_HBM_GBS,
        "pct_of_measured_hbm": 100.0 * value / world / peak,
        "tok_s_equiv": world * 1e3 / ms,
        "bytes_per_step": step_bytes,
        "e2e": {"value": e2e_val, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "tok_s_equiv": world * 1e3 / e2e_ms},
        "roofline": {"bound": "hbm",
                     "kernel": f"tern_gateup_swiglu{'_streamed' if mode == 'streamed' else '_fused' if mode == 'fused' else ''}"
                               " (gate/up + SwiGLU, K=5120, N=17408, 2 matrices)",
                     "achieved": gu_achieved, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": gu_achieved / peak, "traffic": traffic_record("gateup_swiglu", args.fmt),
                     "algorithmic_bytes_per_launch": gu_bytes, "avg_launch_us": gu_ms * 1e3},
        "gpu_launches": (4 * args.layers if mode == "streamed" else
                         4 * args.layers + 1 if mode == "fused" else 8 * args.layers) * args.steps,
        "clocks": clk,
        "cpu_baseline": cpu,
        "configs": configs,
        "device_error": err,
        "output_finite": out_ok,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
