"""Benchmark of the INT8 ConvRot hot path on B200.

One step = one pass of the whole path over one batch of synthetic tokens: the
FFN block (rotate + per-token quantize x, int8 GEMM against the [gate; up]
weight with the fused SwiGLU epilogue, re-rotate + requantize h, int8 GEMM
against the down weight with the fused rescale epilogue), i.e. every step of
the method. Default workload: M = 16384 tokens, hidden K = 5376, FFN width
F = 14336, activations N(0,1) with 1% outlier channels x50, weights N(0, 0.02)
prepared on the device by the library's own weight preparation.

Headline value: int8 GEMM operations of the step (2*M*2F*K + 2*M*K*F) per
second of device time, in TOPS. Also reported: FFN tokens/s, the
rotate+quantize bandwidth, the dominant kernel's roofline fraction, an
end-to-end number through host buffers, and the CPU oracle's rate on a bounded
sample of the same workload.

Multi-GPU (torchrun): every rank runs its own batch with replicated weights
(the rows are independent; there is no data-path collective). Times are the
max over ranks; the value is the work of all ranks over that time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_FLUSH_BYTES = 256 << 20
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")
GEMM_SRC = os.path.join(ROOT, "w8a8_rotation_quantized_b200", "csrc", "gemm_sm100.cuh")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="h3q", choices=["h3q", "reference"])
    ap.add_argument("--M", type=int, default=16384)
    ap.add_argument("--K", type=int, default=5376)
    ap.add_argument("--F", type=int, default=14336)
    ap.add_argument("--kernel-reps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


def gemm_ops(M, K, F):
    return 2.0 * M * (2 * F) * K + 2.0 * M * K * F


def workload_config(args, world):
    return {
        "workload": f"FFN block M={args.M} K={args.K} F={args.F}: rotquant(x) -> int8 GEMM [gate;up] + SwiGLU "
                    f"-> rotquant(h) -> int8 GEMM down",
        "tokens_per_gpu": args.M, "hidden": args.K, "ffn_width": args.F,
        "global_batch_tokens": args.M * world, "parallelism": f"replicas x{world} (rows independent)",
        "activations": "bf16 N(0,1), 1% outlier channels x50, seed 0",
        "weights": "fp32 N(0,0.02) -> rotated per-row int8 on device, seed 0",
        "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write); inputs also exceed L2",
    }


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index, self.proc, self.path = index, None, None

    def start(self):
        try:
            self.path = f"/tmp/h3q_clocks_{os.getpid()}.csv"
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        load = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- oracle rate
def oracle_rate(M, K, F, target_s, threads_note=True):
    """Times the CPU oracle's FFN on a bounded sample of rows of the same workload."""
    import numpy as np

    import oracle
    import synth

    wl_ids = synth.tensor_ids()
    factors = synth.column_factors(K, synth.outlier_columns(0, wl_ids["outlier"], K, int(round(0.01 * K))), 50.0)
    wgu = synth.weight_host(0, wl_ids["w_gu"], np.arange(2 * F), K)
    wd = synth.weight_host(0, wl_ids["w_down"], np.arange(K), F)
    qgu, sgu = oracle.prepare_weight(wgu)
    qd, sd = oracle.prepare_weight(wd)
    del wgu, wd
    rows = 8
    while True:
        x = synth.activation_host(0, wl_ids["x"], np.arange(rows), K, factors)
        t0 = time.perf_counter()
        oracle.ffn(x, qgu, sgu, qd, sd)
        dt = time.perf_counter() - t0
        if dt >= target_s or rows >= M:
            break
        rows = min(M, max(rows * 2, int(rows * target_s / max(dt, 1e-3) * 1.1)))
    return {"value": gemm_ops(rows, K, F) / dt / 1e12, "unit": "TOPS", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{rows} of {M} token rows of the same FFN workload (full weights), {dt:.1f} s"}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    import numpy as np

    import oracle
    import synth

    K, F = args.K, args.F
    ids = synth.tensor_ids()
    factors = synth.column_factors(K, synth.outlier_columns(0, ids["outlier"], K, int(round(0.01 * K))), 50.0)
    qgu, sgu = oracle.prepare_weight(synth.weight_host(0, ids["w_gu"], np.arange(2 * F), K))
    qd, sd = oracle.prepare_weight(synth.weight_host(0, ids["w_down"], np.arange(K), F))
    # rows per step: sized so that warmup + steps finish in about a minute of CPU time
    x = synth.activation_host(0, ids["x"], np.arange(8), K, factors)
    t0 = time.perf_counter()
    oracle.ffn(x, qgu, sgu, qd, sd)
    per_row = (time.perf_counter() - t0) / 8
    rows = max(1, min(args.M, int(60.0 / max(1, args.steps + args.warmup) / per_row)))
    x = synth.activation_host(0, ids["x"], np.arange(rows), K, factors)
    for _ in range(args.warmup):
        oracle.ffn(x, qgu, sgu, qd, sd)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.ffn(x, qgu, sgu, qd, sd)
        times.append(time.perf_counter() - t0)
    dt = sum(times)
    value = gemm_ops(rows, K, F) * args.steps / dt / 1e12
    cfg = workload_config(args, world)
    line = {"impl": "reference", "metric": "INT8 ConvRot linear TOPS", "value": value, "unit": "TOPS",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic",
            "config": cfg,
            "cpu_baseline": {"value": value, "unit": "TOPS", "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"{rows} of {args.M} token rows per step, full weights"},
            "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
def traffic_from_profile(kernel_tag):
    try:
        prof = json.load(open(PROFILE_TRAFFIC))
        src_hash = hashlib.sha256(open(GEMM_SRC, "rb").read()).hexdigest()
        ent = prof.get(kernel_tag)
        if ent and ent.get("source_sha256") == src_hash:
            return ent.get("bytes_per_launch")
    except Exception:
        pass
    return None


def measured_peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def run_gpu(args):
    import torch
    import torch.distributed as dist

    import synth
    import w8a8_rotation_quantized_b200 as h3q

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    M, K, F = args.M, args.K, args.F
    ids = synth.tensor_ids()
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream

    # ---- inputs, generated on the device; the weights prepared by the library
    factors = synth.column_factors(K, synth.outlier_columns(0, ids["outlier"], K, int(round(0.01 * K))), 50.0)
    fdev = torch.from_numpy(factors).to(dev)
    x = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    # each rank takes its own rows of one long token stream
    synth.fill_device(0, ids["x"], rank * M, M, K, x.data_ptr(), sp, factors_ptr=fdev.data_ptr(), bf16=True)
    qgu = torch.empty((2 * F, K), dtype=torch.int8, device=dev)
    sgu = torch.empty(2 * F, dtype=torch.float32, device=dev)
    qd = torch.empty((K, F), dtype=torch.int8, device=dev)
    sd = torch.empty(K, dtype=torch.float32, device=dev)
    w = torch.empty((2 * F, K), dtype=torch.float32, device=dev)
    synth.fill_device(0, ids["w_gu"], 0, 2 * F, K, w.data_ptr(), sp, scale=float(synth.SIGMA_W), bf16=False)
    h3q.h3q_prepare_weight(w, qgu, sgu)
    w = torch.empty((K, F), dtype=torch.float32, device=dev)
    synth.fill_device(0, ids["w_down"], 0, K, F, w.data_ptr(), sp, scale=float(synth.SIGMA_W), bf16=False)
    h3q.h3q_prepare_weight(w, qd, sd)
    del w
    ws = torch.empty(h3q.h3q_ffn_workspace_size(M, K, F), dtype=torch.uint8, device=dev)
    y = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()

    def step():
        h3q.h3q_ffn(x, qgu, sgu, qd, sd, y, ws)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(v):
        if world == 1:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    for _ in range(args.warmup):
        step()
    barrier()

    clocks = ClockSampler(local)
    clocks.start()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    barrier()
    clk = clocks.stop()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(sum(step_ms))
    st = h3q.h3q_get_device_status()
    if st != h3q.H3Q_OK:
        raise RuntimeError(f"device status after the timed region: {h3q.h3q_status_string(st)}")

    # ---- per-kernel device times (same stream, events around each launch, L2 flushed)
    L = h3q.h3q_ffn_workspace_size  # noqa: F841
    off = 0
    def carve(nbytes, dtype, shape):
        nonlocal off
        t = ws[off:off + nbytes].view(dtype).view(*shape)
        off = (off + nbytes + 255) // 256 * 256
        return t
    xq = carve(M * K, torch.int8, (M, K))
    sx = carve(M * 4, torch.float32, (M,))
    hbuf = carve(M * F * 2, torch.bfloat16, (M, F))
    hq = carve(M * F, torch.int8, (M, F))
    sh = carve(M * 4, torch.float32, (M,))

    def time_kernel(fn):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.kernel_reps)]
        fn()
        for a, b in ev:
            flush.fill_(1)
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in ev) / len(ev)

    t_rq_x = time_kernel(lambda: h3q.h3q_rotate_quant(x, xq, sx))
    t_gu = time_kernel(lambda: h3q.h3q_linear_w8a8(xq, sx, qgu, sgu, hbuf, epilogue=h3q.H3Q_EPI_SWIGLU))
    t_rq_h = time_kernel(lambda: h3q.h3q_rotate_quant(hbuf, hq, sh))
    t_down = time_kernel(lambda: h3q.h3q_linear_w8a8(hq, sh, qd, sd, y))

    # ---- end to end through host buffers: H2D of x, the C-ABI call, D2H of y
    e2e = None
    if not args.no_e2e:
        x_host = torch.empty((M, K), dtype=torch.bfloat16, pin_memory=True)
        x_host.copy_(x)
        y_host = torch.empty((M, K), dtype=torch.bfloat16, pin_memory=True)
        x_dev = torch.empty_like(x)
        e_steps = max(3, min(args.steps, 10))
        def e2e_step():
            x_dev.copy_(x_host, non_blocking=True)
            h3q.h3q_ffn(x_dev, qgu, sgu, qd, sd, y, ws)
            y_host.copy_(y, non_blocking=True)
        e2e_step()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(e_steps):
            e2e_step()
        b.record(stream)
        barrier()
        e_ms = max_over_ranks(a.elapsed_time(b) / e_steps)
        e2e = {"value": gemm_ops(M, K, F) * world / (e_ms * 1e-3) / 1e12, "unit": "TOPS",
               "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * K * 2, "ms_per_step": e_ms}

    if rank == 0:
        ms = total_ms / args.steps
        value = gemm_ops(M, K, F) * world / (ms * 1e-3) / 1e12
        peaks, peak_src = measured_peaks()
        # int8 dense tensor rate on B200 is twice the bf16 rate (4.5 vs 2.25 PFLOP/s nominal)
        i8_peak = 2.0 * peaks["bf16_tflops"]
        gu_ops = 2.0 * M * (2 * F) * K
        achieved = gu_ops / (t_gu * 1e-3) / 1e12
        traffic = traffic_from_profile("gemm_i8_swiglu_ffn")
        rq_bytes = M * K * 3 + M * 4
        line = {
            "metric": "INT8 ConvRot linear TOPS", "value": value, "unit": "TOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic",
            "config": workload_config(args, world),
            "ffn_tokens_per_s": M * world / (ms * 1e-3),
            "int8_peak_tops": i8_peak,
            "frac_of_int8_peak": value / i8_peak,
            "kernels_ms": {"rotate_quant_x": t_rq_x, "gemm_gate_up_swiglu": t_gu, "rotate_quant_h": t_rq_h,
                           "gemm_down": t_down},
            "rotquant_gbs": {"x": rq_bytes / (t_rq_x * 1e-3) / 1e9,
                             "h": (M * F * 3 + M * 4) / (t_rq_h * 1e-3) / 1e9,
                             "peak": peaks["hbm_gbs"]},
            "roofline": {"bound": "tensor", "kernel": "gemm_i8_kernel<SwiGLU> (gate/up)",
                         "achieved": achieved, "peak": i8_peak, "unit": "TOPS",
                         "frac": achieved / i8_peak, "traffic": traffic,
                         "peak_source": f"{peak_src}: 2 x bf16 burst {peaks['bf16_tflops']} TFLOP/s "
                                        "(int8 dense rate = 2 x bf16 on B200)"},
            "gpu_launches": 4 * args.steps,
            "clocks": clk,
            "e2e": e2e,
        }
        if not args.no_cpu_baseline:
            try:
                line["cpu_baseline"] = oracle_rate(M, K, F, args.cpu_seconds)
            except Exception as exc:  # the line still prints; the reason is kept
                line["cpu_baseline"] = {"value": None, "error": repr(exc)}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
