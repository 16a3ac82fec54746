#!/usr/bin/env python3
"""Benchmark of the ternary decode weight stream on B200.

One step = one batch-1 decode step of a 64-layer 27B-shaped ternary layer
stack, replayed as one CUDA graph.  Per layer four kernels (the streamed
GEMV entry points, which quantise their fp32 input themselves): QKV GEMV,
O GEMV + residual, fused gate/up + SwiGLU with the 128-point Hadamard
rotation, down GEMV + residual.  The metric is the weight stream's
algorithmic bytes (packed codes + fp16 group scales) per second, with the
decode-step rate (tok/s-equivalent) beside it.  The line also carries the
prefill GEMM (tern_gemm on the tensor cores) at M = 512 / 2048 / 8192.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--fmt base3|2bit] [--layers 64] [--M 1] [--no-prefill]

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


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--fmt", choices=["base3", "2bit"], default="base3")
    ap.add_argument("--layers", type=int, default=64)
    ap.add_argument("--M", type=int, default=1)
    ap.add_argument("--mode", choices=["auto", "streamed", "fused", "unfused"], default="auto",
                    help="decode-step kernels (auto: streamed for M <= 2, else fused)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill GEMM measurement")
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


def prefill_gemm(fmt_id, Ms=(512, 2048, 8192), K=5120, N=17408, reps=10):
    """tern_gemm on the gate/up shape (K = 5120, N = 17408) at prefill batch
    sizes; TOPS = 2 M N K / device time (CUDA events, after warm-up).  W
    (17.8 MB base-3) stays L2-resident across the token tiles, as in any
    prefill; the kernel is tensor-core and epilogue bound, not HBM bound."""
    import torch
    from ternary_weight_decode_b200 import decode, tern
    scratch = torch.empty(N * K, dtype=torch.int8, device="cuda")
    W = decode.make_matrix(fmt_id, N, K, seed=977, stream=5, scratch=scratch)
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
    return {"workload": f"tern_gemm, K={K}, N={N}, int8 activations, fp16/128 group scales",
            "unit": "TOPS", "peak": peak, "peak_kind": kind, "results": res}


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
    for rel in ("ternary_weight_decode_b200/csrc/tern_gemv_stream.cu",
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


# ---------------------------------------------------------------- CPU oracle sample
def oracle_layer_sample(fmt_id: int, layer: int, M: int, x0):
    """Runs one decode layer of the same workload through the CPU oracle.
    Returns (algorithmic bytes processed, seconds of oracle time)."""
    import numpy as np
    import oracle
    from ternary_weight_decode_b200 import decode, synth
    H, Q, F = decode.HIDDEN, decode.QKV, decode.FFN

    def weights(N, K, proj):
        st = synth.stream_id(layer, proj)
        return (_host_trits(layer, st, N, K), synth.scales(layer, st + 1, N, (K + 127) // 128))

    Wqkv, Wo = weights(Q, H, synth.PROJ_QKV), weights(H, H, synth.PROJ_O)
    Wg, Wu = weights(F, H, synth.PROJ_GATE), weights(F, H, synth.PROJ_UP)
    Wd = weights(H, F, synth.PROJ_DOWN)
    t0 = time.perf_counter()
    x = x0.astype(np.float64)
    q, s = oracle.act_quant(x.astype(np.float32), rmsnorm=True)
    qkv = oracle.gemv(*Wqkv, q, s)
    q, s = oracle.act_quant(qkv[:, :H].astype(np.float32), rmsnorm=True)
    x = x + oracle.gemv(*Wo, q, s)
    q, s = oracle.act_quant(x.astype(np.float32), fwht_block=128, rmsnorm=True)
    h = oracle.gateup_swiglu(Wg[0], Wg[1], Wu[0], Wu[1], q, s)
    q, s = oracle.act_quant(h.astype(np.float32), rmsnorm=True)
    x = x + oracle.gemv(*Wd, q, s)
    dt = time.perf_counter() - t0
    return decode_layer_bytes(fmt_id), dt, x


def decode_layer_bytes(fmt_id: int) -> int:
    from ternary_weight_decode_b200 import decode
    return decode.layer_bytes(fmt_id)


def _host_trits(seed, stream, N, K):
    """Trits for the CPU sample, from the device generator when a GPU is
    present (same definition as the host generator, checked bit for bit)."""
    import torch
    from ternary_weight_decode_b200 import synth
    if torch.cuda.is_available():
        return synth.device_trits(seed, stream, N, K).cpu().numpy()
    return synth.trits(seed, stream, N, K)


def cpu_baseline(fmt_id: int, M: int, target_s: float, unit_scale=1e9):
    import numpy as np
    import oracle
    from ternary_weight_decode_b200 import synth
    cores = len(os.sched_getaffinity(0))
    oracle.set_threads(cores)
    x0 = synth.activations(0, M, 5120).astype(np.float32)
    total_b, total_t, layers = 0, 0.0, 0
    x = x0
    while total_t < target_s and layers < 64:
        b, dt, x = oracle_layer_sample(fmt_id, layers, M, x)
        total_b += b
        total_t += dt
        layers += 1
    return {"value": total_b / total_t / unit_scale, "unit": "GB/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{layers} of 64 decode layers (M={M}), all 4 projections, plain-C fp64 "
                      f"oracle with OpenMP over output rows; {total_t:.1f} s of oracle time"}


# ---------------------------------------------------------------- reference arm
def run_reference(args, world, rank):
    if rank != 0:
        return 0
    import numpy as np
    from ternary_weight_decode_b200 import synth, tern
    fmt_id = tern.TERN_FMT_BASE3 if args.fmt == "base3" else tern.TERN_FMT_2BIT
    cores = len(os.sched_getaffinity(0))
    import oracle
    oracle.set_threads(cores)
    x = synth.activations(0, args.M, 5120).astype(np.float32)
    for i in range(args.warmup):
        _, _, x = oracle_layer_sample(fmt_id, i % 64, args.M, x)
    tb, tt = 0, 0.0
    for i in range(args.steps):
        b, dt, x = oracle_layer_sample(fmt_id, (args.warmup + i) % 64, args.M, x)
        tb += b
        tt += dt
    value = tb / tt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tt / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step = one of the 64 decode layers (M={args.M}) through "
                                   f"the plain-C fp64 oracle"},
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
    fmt_id = tern.TERN_FMT_BASE3 if args.fmt == "base3" else tern.TERN_FMT_2BIT
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
    gu_bytes = 2 * (decode.FFN * tern.tern_canonical_row_bytes(fmt_id, decode.HIDDEN)
                    + 2 * decode.FFN * (decode.HIDDEN // 128))
    def gateup_all():
        rms, rot = tern.TERN_QUANT_RMSNORM, tern.TERN_QUANT_FWHT128
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
    gateup_all()
    torch.cuda.synchronize()
    gu_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gu_graph):
        gateup_all()
    for _ in range(3):
        gu_graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 5
    e0.record(stream)
    for _ in range(reps):
        gu_graph.replay()
    e1.record(stream)
    e1.synchronize()
    gu_ms = e0.elapsed_time(e1) / (reps * len(model.layers))
    del gu_graph

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
    value = replica_value(step_bytes, ms, world)
    e2e_val = replica_value(step_bytes, e2e_ms, world)
    peak, peak_kind = peaks()
    gu_achieved = gu_bytes / (gu_ms * 1e-3) / 1e9
    out_ok = bool(torch.isfinite(model.x).all().item())

    if rank != 0:
        del graph
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return 0

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(fmt_id, args.M, args.cpu_seconds)
    prefill = None
    if world == 1 and not args.no_prefill:
        del graph
        graph = None
        prefill = prefill_gemm(fmt_id)

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
        "gpu_launches": model.launches_per_step() * args.steps,
        "clocks": clk,
        "cpu_baseline": cpu,
        "prefill_gemm": prefill,
        "device_error": err,
        "output_finite": out_ok,
    }
    print(json.dumps(line), flush=True)
    del graph
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
