"""Benchmark of the INT8 ConvRot hot path on B200.

One step = one pass of the whole path over one batch of synthetic tokens. The
default workload is the FFN block (every step of the method: rotate + per-token
quantize x, int8 GEMM against the [gate; up] weight with the fused SwiGLU
epilogue, re-rotate + requantize h, int8 GEMM against the down weight with the
fused rescale epilogue) at M = 16384 tokens, hidden K = 5376, FFN width
F = 14336; activations N(0,1) with 1% outlier channels x50, weights N(0, 0.02)
prepared on the device by the library's own weight preparation.

Headline value: int8 GEMM operations of the step per second of device time, in
TOPS. Also reported: FFN tokens/s, the rotate+quantize bandwidth, the dominant
kernel's roofline fraction, an end-to-end number through host buffers, and the
CPU oracle's rate on a bounded sample of the same workload.

Other workloads (--workload): qkv (4096 x 5376 -> 16128 with bias), out
(32768 x 5376 -> 5376 with bias), tiny (64 x 512 -> 256), sweep (one denoising
step's linear sweep: 50 blocks x (QKV, out, FFN) at 32768 tokens, about 17 GB of
int8 weights resident, per-block activations generated before timing).

Workload lora: merging a rank-64 LoRA at load into one FFN block's int8
weights (gate/up [28672, 5376] and down [5376, 14336]); value in fp32 TFLOP/s of
the merge's low-rank product, bound by the fp32 FMA pipe.

Workload nvfp4: the hybrid checkpoints' four linear operations of one block at
16000 tokens (QKV and FFN input in NVFP4, attention output and FFN output in
INT8 ConvRot, each with the quantization of its input), next to the same four
operations all in INT8 ConvRot; value in TOPS of the four GEMMs.

Workload attention: the DiT attention call at 16384 tokens, 42 heads of 128
(int8 Q.K^T, bf16 P.V), from a QKV projection output; value in TFLOP/s of the
two products (4 S^2 D H); the library's bf16 scaled-dot-product attention on
the same tensors is timed beside it as context.

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
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_FLUSH_BYTES = 256 << 20
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")
GEMM_SRC = os.path.join(ROOT, "w8a8_rotation_quantized_b200", "csrc", "gemm_sm100.cuh")
METRIC = "INT8 ConvRot linear TOPS"
# NVIDIA's published dense int8 rate for one B200 (HGX figure; the doubled figure assumes 2:4
# sparsity). The roofline fraction uses the measured rate; this one is reported beside it.
I8_NOMINAL_TOPS = 4500.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="h3q", choices=["h3q", "reference"])
    ap.add_argument("--workload", default="ffn", choices=["ffn", "qkv", "out", "tiny", "sweep", "lora", "nvfp4", "attention"])
    ap.add_argument("--M", type=int, default=None, help="tokens per GPU (default: the workload's)")
    ap.add_argument("--F", type=int, default=None, help="FFN width (default 14336)")
    ap.add_argument("--kernel-reps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


# ----------------------------------------------------------------------------- workloads
class Spec:
    """Shapes of one workload; ops() is the int8 GEMM work of one step."""

    def __init__(self, name, M, K, N=None, F=None, bias=False, blocks=1):
        self.name, self.M, self.K, self.N, self.F, self.bias, self.blocks = name, M, K, N, F, bias, blocks

    def ops(self, M=None):
        M = self.M if M is None else M
        if self.name == "ffn":
            return 2.0 * M * (2 * self.F) * self.K + 2.0 * M * self.K * self.F
        if self.name == "sweep":
            per_block = 2.0 * M * self.K * (16128 + 5376) + 2.0 * M * (2 * self.F) * self.K + 2.0 * M * self.K * self.F
            return per_block * self.blocks
        return 2.0 * M * self.N * self.K

    def describe(self, world):
        d = {"ffn": f"FFN block M={self.M} K={self.K} F={self.F}: rotquant(x) -> int8 GEMM [gate;up] + SwiGLU "
                    f"-> rotquant(h) -> int8 GEMM down",
             "qkv": f"QKV projection M={self.M} K={self.K} N={self.N} with bias: rotquant(x) -> int8 GEMM + rescale",
             "out": f"attention-output projection M={self.M} K={self.K} N={self.N} with bias: rotquant(x) -> "
                    f"int8 GEMM + rescale",
             "tiny": f"tiny linear M={self.M} K={self.K} N={self.N}: rotquant(x) -> int8 GEMM + rescale",
             "sweep": f"one denoising step's linear sweep: {self.blocks} blocks x (QKV {self.K}->16128, out "
                      f"{self.K}->{self.K}, FFN {self.K}->2x{self.F}->{self.K}) at M={self.M}"}[self.name]
        return {
            "workload": d, "tokens_per_gpu": self.M, "hidden": self.K,
            "global_batch_tokens": self.M * world, "parallelism": f"replicas x{world} (rows independent)",
            "activations": "bf16 N(0,1), 1% outlier channels x50 (tiny: 4 channels x40), seed 0",
            "weights": "fp32 N(0,0.02) -> rotated per-row int8 on device, seed 0",
            "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write); inputs also exceed L2",
        }


def make_spec(args):
    F = args.F or 14336
    table = {
        "ffn": Spec("ffn", 16384, 5376, F=F),
        "qkv": Spec("qkv", 4096, 5376, N=16128, bias=True),
        "out": Spec("out", 32768, 5376, N=5376, bias=True),
        "tiny": Spec("tiny", 64, 512, N=256),
        "sweep": Spec("sweep", 32768, 5376, F=F, bias=True, blocks=50),
    }
    s = table[args.workload]
    if args.M is not None:
        s.M = args.M
    return s


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index, self.proc, self.path = index, None, None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="h3q_clocks_", suffix=".csv")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=os.fdopen(fd, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, t0=None, t1=None):
        """Summary of the samples taken between host times t0 and t1 (seconds)."""
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        from datetime import datetime
        samples = []
        with open(self.path) as f:
            lines = f.readlines()
        try:
            os.unlink(self.path)
        except OSError:
            pass
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                continue
            samples.append((ts, parts[1:]))
        window = "timed region"
        rows = [r for ts, r in samples if t0 is None or t0 <= ts <= t1]
        if not rows and t0 is not None:
            # a timed region shorter than the sampling interval: the samples just around it
            rows = [r for ts, r in samples if t0 - 0.15 <= ts <= t1 + 0.15]
            window = "nearest samples (timed region shorter than the 100 ms sampling interval)"
        if not rows:
            return None

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        pw = [num(r[3]) for r in rows if num(r[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        load = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None, "reasons": reasons, "samples": len(rows), "window": window}


# ----------------------------------------------------------------------------- oracle rate
def _oracle_ffn_setup(K, F):
    import numpy as np

    import oracle
    import synth

    ids = synth.tensor_ids()
    factors = synth.column_factors(K, synth.outlier_columns(0, ids["outlier"], K, int(round(0.01 * K))), 50.0)
    qgu, sgu = oracle.prepare_weight(synth.weight_host(0, ids["w_gu"], np.arange(2 * F), K))
    qd, sd = oracle.prepare_weight(synth.weight_host(0, ids["w_down"], np.arange(K), F))
    return ids, factors, qgu, sgu, qd, sd


def oracle_rate(spec, target_s):
    """Times the CPU oracle's FFN (or linear layer) on a bounded sample of rows of the workload."""
    import numpy as np

    import oracle
    import synth

    K = spec.K
    if spec.name in ("ffn", "sweep"):
        ids, factors, qgu, sgu, qd, sd = _oracle_ffn_setup(K, spec.F)

        def run(rows):
            x = synth.activation_host(0, ids["x"], np.arange(rows), K, factors)
            t0 = time.perf_counter()
            oracle.ffn(x, qgu, sgu, qd, sd)
            return time.perf_counter() - t0

        def ops(rows):
            return 2.0 * rows * (2 * spec.F) * K + 2.0 * rows * K * spec.F
        what = "FFN"
    else:
        ids = synth.tensor_ids()
        nout = 4 if spec.name == "tiny" else int(round(0.01 * K))
        factors = synth.column_factors(K, synth.outlier_columns(0, ids["outlier"], K, nout),
                                       40.0 if spec.name == "tiny" else 50.0)
        wq, sw = oracle.prepare_weight(synth.weight_host(0, ids["w"], np.arange(spec.N), K))
        b = synth.bias_host(0, ids["bias"], spec.N) if spec.bias else None

        def run(rows):
            x = synth.activation_host(0, ids["x"], np.arange(rows), K, factors)
            t0 = time.perf_counter()
            oracle.linear(x, wq, sw, bias_bits=b)
            return time.perf_counter() - t0

        def ops(rows):
            return 2.0 * rows * spec.N * K
        what = "linear layer"
    rows = 8
    while True:
        dt = run(rows)
        if dt >= target_s or rows >= spec.M:
            break
        rows = min(spec.M, max(rows * 2, int(rows * target_s / max(dt, 1e-3) * 1.1)))
    return {"value": ops(rows) / dt / 1e12, "unit": "TOPS", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{rows} of {spec.M} token rows of the same {what} workload (full weights), {dt:.1f} s"}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    """The oracle itself, timed on the host cores: there is no other reference
    implementation (the reference is a set of pages, not code)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    import numpy as np

    import oracle
    import synth

    if args.workload == "attention":
        per_step = 60.0 / max(1, args.steps + args.warmup)
        S = args.M or 16384
        for _ in range(args.warmup):
            oracle_attention_rate(S, 42, per_step)
        vals = [oracle_attention_rate(S, 42, per_step) for _ in range(args.steps)]
        secs = sum(v["seconds"] for v in vals)
        value = sum(v["value"] * v["seconds"] for v in vals) / secs
        line = {"impl": "reference", "metric": "int8 attention TFLOP/s", "value": value, "unit": "TFLOP/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "i8+bf16",
                "data": "synthetic", "config": {"workload": f"DiT attention S={S}, 42 heads, sampled query rows"},
                "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                                 "sample": vals[-1]["sample"]},
                "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0
    if args.workload == "nvfp4":
        per_step = 60.0 / max(1, args.steps + args.warmup)
        for _ in range(args.warmup):
            oracle_nvfp4_rate(per_step)
        vals = [oracle_nvfp4_rate(per_step) for _ in range(args.steps)]
        secs = sum(v["seconds"] for v in vals)
        value = sum(v["value"] * v["seconds"] for v in vals) / secs
        line = {"impl": "reference", "metric": "hybrid NVFP4/INT8 linear TOPS", "value": value, "unit": "TOPS",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp4+i8",
                "data": "synthetic", "config": {"workload": "NVFP4 QKV projection, sampled rows"},
                "cpu_baseline": {"value": value, "unit": "TOPS", "cores": oracle.num_threads(), "kind": "oracle",
                                 "sample": vals[-1]["sample"]},
                "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0
    if args.workload == "lora":
        per_step = 60.0 / max(1, args.steps + args.warmup)
        for _ in range(args.warmup):
            oracle_lora_rate(per_step)
        vals = [oracle_lora_rate(per_step) for _ in range(args.steps)]
        value = sum(v["rows"] for v in vals) * 2.0 * 5376 * synth.WORKLOADS["lora"].rank / \
            sum(v["seconds"] for v in vals) / 1e12
        line = {"impl": "reference", "metric": "LoRA merge TFLOP/s", "value": value, "unit": "TFLOP/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1e3 * sum(v["seconds"] for v in vals) / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": {"workload": "LoRA merge at load into the gate/up weight, sampled rows"},
                "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                                 "sample": vals[-1]["sample"]},
                "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0
    spec = make_spec(args)
    if spec.name == "sweep":
        spec = Spec("ffn", spec.M, spec.K, F=spec.F)  # the sweep's dominant layer
    K = spec.K
    if spec.name == "ffn":
        ids, factors, qgu, sgu, qd, sd = _oracle_ffn_setup(K, spec.F)

        def run(x):
            oracle.ffn(x, qgu, sgu, qd, sd)
    else:
        ids = synth.tensor_ids()
        factors = synth.column_factors(K, synth.outlier_columns(0, ids["outlier"], K, int(round(0.01 * K))), 50.0)
        wq, sw = oracle.prepare_weight(synth.weight_host(0, ids["w"], np.arange(spec.N), K))
        b = synth.bias_host(0, ids["bias"], spec.N) if spec.bias else None

        def run(x):
            oracle.linear(x, wq, sw, bias_bits=b)
    # rows per step: sized so that warmup + steps finish in about a minute of CPU time
    x = synth.activation_host(0, ids["x"], np.arange(8), K, factors)
    t0 = time.perf_counter()
    run(x)
    per_row = (time.perf_counter() - t0) / 8
    rows = max(1, min(spec.M, int(60.0 / max(1, args.steps + args.warmup) / per_row)))
    x = synth.activation_host(0, ids["x"], np.arange(rows), K, factors)
    for _ in range(args.warmup):
        run(x)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        run(x)
        times.append(time.perf_counter() - t0)
    dt = sum(times)
    value = spec.ops(rows) * args.steps / dt / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic",
            "config": make_spec(args).describe(world),
            "cpu_baseline": {"value": value, "unit": "TOPS", "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"{rows} of {spec.M} token rows per step, full weights"},
            "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- multi-rank plumbing
def shard_rows(rank, world, M):
    """First row and row count of this rank's slice of one long token stream: every
    rank processes M rows of its own (weak scaling); the slices are disjoint."""
    assert 0 <= rank < world
    return rank * M, M


def max_over_ranks(value, device=None):
    """The largest value over all ranks (the job's time is the slowest rank's)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tops(ops_per_rank_step, world, ms_per_step):
    """Whole-job throughput: the work of all ranks over the (max-over-ranks) step time."""
    return ops_per_rank_step * world / (ms_per_step * 1e-3) / 1e12


# ----------------------------------------------------------------------------- GPU arm
def traffic_from_profile(kernel_tag):
    """DRAM bytes per launch of a kernel from a committed ncu summary, or None
    once the kernel's source file has changed since the counters were taken."""
    try:
        prof = json.load(open(PROFILE_TRAFFIC))
        ent = prof.get(kernel_tag)
        if not ent:
            return None
        src = os.path.join(ROOT, ent.get("source_file", os.path.relpath(GEMM_SRC, ROOT)))
        if ent.get("source_sha256") == hashlib.sha256(open(src, "rb").read()).hexdigest():
            return ent.get("bytes_per_launch")
    except Exception:
        pass
    return None


def measured_peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class Layer:
    """Device tensors of one linear layer (x, prepared weight, bias); the codes,
    scales and output may be shared between layers (`bufs`)."""

    def __init__(self, h3q, synth, torch, dev, sp, M, K, N, tid_x, tid_w, tid_b, factors_dev, x_row0, bias,
                 bufs=None):
        self.M, self.K, self.N = M, K, N
        self.x = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
        synth.fill_device(0, tid_x, x_row0, M, K, self.x.data_ptr(), sp,
                          factors_ptr=None if factors_dev is None else factors_dev.data_ptr(), bf16=True)
        w = torch.empty((N, K), dtype=torch.float32, device=dev)
        synth.fill_device(0, tid_w, 0, N, K, w.data_ptr(), sp, scale=float(synth.SIGMA_W), bf16=False)
        self.wq = torch.empty((N, K), dtype=torch.int8, device=dev)
        self.sw = torch.empty(N, dtype=torch.float32, device=dev)
        h3q.h3q_prepare_weight(w, self.wq, self.sw)
        del w
        self.bias = None
        if bias:
            self.bias = torch.from_numpy(synth.bias_host(0, tid_b, N).view("int16")).to(dev).view(torch.bfloat16)
        if bufs is None:
            bufs = {"xq": torch.empty(M * K, dtype=torch.int8, device=dev),
                    "sx": torch.empty(M, dtype=torch.float32, device=dev),
                    "y": torch.empty(M * N, dtype=torch.bfloat16, device=dev)}
        self.xq = bufs["xq"][:M * K].view(M, K)
        self.sx = bufs["sx"][:M]
        self.y = bufs["y"][:M * N].view(M, N)

    def run(self, h3q, x=None):
        h3q.h3q_rotate_quant(self.x if x is None else x, self.xq, self.sx)
        h3q.h3q_linear_w8a8(self.xq, self.sx, self.wq, self.sw, self.y, bias=self.bias)


class FFN:
    """Device tensors of one FFN block."""

    def __init__(self, h3q, synth, torch, dev, sp, M, K, F, tid_x, tid_gu, tid_d, factors_dev, x_row0, y=None):
        self.M, self.K, self.F = M, K, F
        self.x = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
        synth.fill_device(0, tid_x, x_row0, M, K, self.x.data_ptr(), sp,
                          factors_ptr=None if factors_dev is None else factors_dev.data_ptr(), bf16=True)
        self.qgu = torch.empty((2 * F, K), dtype=torch.int8, device=dev)
        self.sgu = torch.empty(2 * F, dtype=torch.float32, device=dev)
        self.qd = torch.empty((K, F), dtype=torch.int8, device=dev)
        self.sd = torch.empty(K, dtype=torch.float32, device=dev)
        w = torch.empty((2 * F, K), dtype=torch.float32, device=dev)
        synth.fill_device(0, tid_gu, 0, 2 * F, K, w.data_ptr(), sp, scale=float(synth.SIGMA_W), bf16=False)
        h3q.h3q_prepare_weight(w, self.qgu, self.sgu)
        w = torch.empty((K, F), dtype=torch.float32, device=dev)
        synth.fill_device(0, tid_d, 0, K, F, w.data_ptr(), sp, scale=float(synth.SIGMA_W), bf16=False)
        h3q.h3q_prepare_weight(w, self.qd, self.sd)
        del w
        self.y = torch.empty((M, K), dtype=torch.bfloat16, device=dev) if y is None else y

    def run(self, h3q, ws, x=None):
        h3q.h3q_ffn(self.x if x is None else x, self.qgu, self.sgu, self.qd, self.sd, self.y, ws)


def fp32_fma_peak_tflops(sms, sm_mhz):
    """fp32 peak of the CUDA cores: 128 FMA lanes per SM, 2 flops per FMA."""
    return sms * 128 * 2 * sm_mhz * 1e6 / 1e12


def _lora_shapes(wl):
    """(name, N, K) of the weights one LoRA step merges into."""
    return [("gate_up", 2 * wl.F, wl.K), ("down", wl.K, wl.F)]


def run_lora(args):
    """LoRA merge at load: one step merges a rank-r LoRA into both int8 weights of
    an FFN block, in place (rotate A, then the merge kernel, per weight)."""
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
    wl = synth.WORKLOADS["lora"]
    r, alpha = wl.rank, wl.alpha
    ids = synth.tensor_ids()
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    mats = []
    for (name, N, K), (ta, tb, tw) in zip(_lora_shapes(wl), [("lora_a", "lora_b", "w_gu"),
                                                           ("lora_a_down", "lora_b_down", "w_down")]):
        w = torch.empty((N, K), dtype=torch.float32, device=dev)
        synth.fill_device(wl.seed, ids[tw], 0, N, K, w.data_ptr(), sp, scale=float(synth.SIGMA_W), bf16=False)
        wq = torch.empty((N, K), dtype=torch.int8, device=dev)
        sw = torch.empty(N, dtype=torch.float32, device=dev)
        h3q.h3q_prepare_weight(w, wq, sw)
        del w
        a = torch.empty((r, K), dtype=torch.float32, device=dev)
        b = torch.empty((N, r), dtype=torch.float32, device=dev)
        synth.fill_device(wl.seed, ids[ta], 0, r, K, a.data_ptr(), sp, scale=float(synth.SIGMA_W), bf16=False)
        synth.fill_device(wl.seed, ids[tb], 0, N, r, b.data_ptr(), sp, scale=float(synth.SIGMA_W), bf16=False)
        ws = torch.empty(h3q.h3q_lora_workspace_size(r, K), dtype=torch.uint8, device=dev)
        mats.append(dict(name=name, N=N, K=K, wq=wq, sw=sw, a=a, b=b, ws=ws))
    flops = sum(2.0 * m["N"] * m["K"] * r for m in mats)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()

    def merge(m, a=None, b=None):
        h3q.h3q_lora_merge(m["wq"], m["sw"], m["a"] if a is None else a, m["b"] if b is None else b, alpha, m["ws"])

    def step():
        for m in mats:
            merge(m)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    steps = max(1, min(args.steps, 50))
    for _ in range(args.warmup):
        step()
    barrier()
    clocks = ClockSampler(local)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier()
    clocks.start()
    time.sleep(0.5)
    t_host0 = time.time()
    for i in range(steps):
        flush.fill_(i & 0xFF)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    barrier()
    clk = clocks.stop(t_host0, time.time())
    total_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(starts, ends)), dev)
    st = h3q.h3q_get_device_status()
    if st != h3q.H3Q_OK:
        raise RuntimeError(f"device status after the timed region: {h3q.h3q_status_string(st)}")

    kernels = {}
    for m in mats:
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.kernel_reps)]
        for e0, e1 in ev:
            flush.fill_(1)
            e0.record(stream)
            merge(m)
            e1.record(stream)
        torch.cuda.synchronize()
        kernels["merge_" + m["name"]] = sum(e0.elapsed_time(e1) for e0, e1 in ev) / len(ev)

    # end to end: the factors come from pinned host memory each step and the new
    # scales go back; the weights stay resident (they are the model's).
    e2e = None
    if not args.no_e2e:
        host = [(torch.empty(m["a"].shape, dtype=torch.float32, pin_memory=True).copy_(m["a"]),
                 torch.empty(m["b"].shape, dtype=torch.float32, pin_memory=True).copy_(m["b"]),
                 torch.empty(m["sw"].shape, dtype=torch.float32, pin_memory=True)) for m in mats]
        dev_ab = [(torch.empty_like(m["a"]), torch.empty_like(m["b"])) for m in mats]
        e_steps = max(4, min(steps, 12))
        barrier()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(e_steps):
            for m, (ha, hb, hs), (da, db) in zip(mats, host, dev_ab):
                da.copy_(ha, non_blocking=True)
                db.copy_(hb, non_blocking=True)
                merge(m, da, db)
                hs.copy_(m["sw"], non_blocking=True)
        t1.record(stream)
        barrier()
        e_ms = max_over_ranks(t0.elapsed_time(t1) / e_steps, dev)
        e2e = {"value": flops * world / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": sum(m["a"].numel() * 4 + m["b"].numel() * 4 for m in mats),
               "d2h_bytes_per_step": sum(m["sw"].numel() * 4 for m in mats), "ms_per_step": e_ms,
               "steps": e_steps, "how": "factors copied from pinned host memory, scales read back, one stream"}

    if rank == 0:
        ms = total_ms / steps
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        sm_mhz = (clk or {}).get("sm_max_mhz") or 1965.0
        peak = fp32_fma_peak_tflops(sms, sm_mhz)
        dom = max(mats, key=lambda m: m["N"] * m["K"])
        dom_ms = kernels["merge_" + dom["name"]]
        achieved = 2.0 * dom["N"] * dom["K"] * r / (dom_ms * 1e-3) / 1e12
        line = {
            "metric": "LoRA merge TFLOP/s", "value": flops * world / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "n_gpus": world, "steps": steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"LoRA merge at load, rank {r}, alpha {alpha}, into one FFN block's int8 "
                                   f"weights: " + ", ".join(f"{m['name']} [{m['N']}, {m['K']}]" for m in mats),
                       "factors": "A [r, K] and B [N, r] fp32 N(0, 0.02), seed 0; weights fp32 N(0, 0.02) "
                                  "prepared on device",
                       "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write)",
                       "parallelism": f"replicas x{world}"},
            "kernels_ms": kernels,
            "hbm_bytes_per_step": sum(2 * m["N"] * m["K"] + 8 * m["N"] + 8 * r * m["K"] + 4 * m["N"] * r
                                      for m in mats),
            "roofline": {"bound": "alu", "kernel": f"lora_merge_kernel ({dom['name']})", "achieved": achieved,
                         "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                         "traffic": traffic_from_profile("lora_merge_" + dom["name"]),
                         "peak_source": f"derived: {sms} SMs x 128 fp32 FMA lanes x 2 flops x {sm_mhz} MHz "
                                        "(max SM clock)"},
            "gpu_launches": 2 * len(mats) * steps,
            "clocks": clk,
            "e2e": e2e,
        }
        if not args.no_cpu_baseline:
            try:
                line["cpu_baseline"] = oracle_lora_rate(args.cpu_seconds)
            except Exception as exc:
                line["cpu_baseline"] = {"value": None, "error": repr(exc)}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


NVFP4_OPS = [  # (name, K, N, SwiGLU, NVFP4 in the hybrid)
    ("qkv", 5376, 16128, False, True),
    ("attn_out", 5376, 5376, False, False),
    ("ffn_in", 5376, 28672, True, True),
    ("ffn_out", 14336, 5376, False, False),
]


def run_nvfp4(args):
    """The hybrid block's four linear operations (NVFP4 for QKV and FFN input,
    INT8 ConvRot for the output projections) against all-INT8 ConvRot."""
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
    M = args.M or 16000
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    ids = synth.tensor_ids()
    K0 = 5376
    factors = torch.from_numpy(synth.column_factors(K0, synth.outlier_columns(0, ids["outlier"], K0, 54), 50.0)).to(dev)
    row0, _ = shard_rows(rank, world, M)
    x = {}
    for name, tid in (("qkv", ids["x_qkv"]), ("attn_out", ids["x_out"]), ("ffn_in", ids["x_ffn"])):
        t = torch.empty((M, K0), dtype=torch.bfloat16, device=dev)
        synth.fill_device(0, tid, row0, M, K0, t.data_ptr(), sp, factors_ptr=factors.data_ptr(), bf16=True)
        x[name] = t
    ops = {}
    for name, K, N, swiglu, fp4 in NVFP4_OPS:
        tid = {"qkv": ids["w_qkv"], "attn_out": ids["w_out"], "ffn_in": ids["w_gu"], "ffn_out": ids["w_down"]}[name]
        w = torch.empty((N, K), dtype=torch.float32, device=dev)
        synth.fill_device(0, tid, 0, N, K, w.data_ptr(), sp, scale=float(synth.SIGMA_W), bf16=False)
        o = dict(K=K, N=N, swiglu=swiglu, fp4=fp4, epi=h3q.H3Q_EPI_SWIGLU if swiglu else h3q.H3Q_EPI_NONE)
        o["wq"] = torch.empty((N, K), dtype=torch.int8, device=dev)
        o["sw"] = torch.empty(N, dtype=torch.float32, device=dev)
        h3q.h3q_prepare_weight(w, o["wq"], o["sw"])
        if True:  # NVFP4 weights for every op: the hybrid uses two, the per-op table all four
            o["wc"] = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
            o["wsf"] = torch.empty(h3q.h3q_nvfp4_sf_bytes(N, K), dtype=torch.uint8, device=dev)
            o["ws"] = torch.empty(2, dtype=torch.float32, device=dev)
            h3q.h3q_nvfp4_quantize(w, o["wc"], o["wsf"], o["ws"])
            o["xc"] = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
            o["xsf"] = torch.empty(h3q.h3q_nvfp4_sf_bytes(M, K), dtype=torch.uint8, device=dev)
            o["xs"] = torch.empty(2, dtype=torch.float32, device=dev)
        del w
        o["xq"] = torch.empty((M, K), dtype=torch.int8, device=dev)
        o["sx"] = torch.empty(M, dtype=torch.float32, device=dev)
        o["y"] = torch.empty((M, N // 2 if swiglu else N), dtype=torch.bfloat16, device=dev)
        ops[name] = o
    x["ffn_out"] = ops["ffn_in"]["y"]  # h, produced by the FFN input projection within the step

    def run_op(name, use_fp4):
        o = ops[name]
        if use_fp4:
            h3q.h3q_nvfp4_quantize(x[name], o["xc"], o["xsf"], o["xs"])
            h3q.h3q_linear_nvfp4(o["xc"], o["xsf"], o["xs"], o["wc"], o["wsf"], o["ws"], o["y"], epilogue=o["epi"])
        else:
            h3q.h3q_rotate_quant(x[name], o["xq"], o["sx"])
            h3q.h3q_linear_w8a8(o["xq"], o["sx"], o["wq"], o["sw"], o["y"], epilogue=o["epi"])

    def step(hybrid=True):
        for name, _, _, _, fp4 in NVFP4_OPS:
            run_op(name, hybrid and fp4)

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def timed(fn, n):
        st = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        en = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for i in range(n):
            flush.fill_(i & 0xFF)
            st[i].record(stream)
            fn()
            en[i].record(stream)
        barrier()
        return sum(a.elapsed_time(b) for a, b in zip(st, en))

    steps = max(1, min(args.steps, 50))
    for _ in range(args.warmup):
        step(True)
        step(False)
    barrier()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.5)
    t_host0 = time.time()
    total_ms = max_over_ranks(timed(lambda: step(True), steps), dev)
    clk = clocks.stop(t_host0, time.time())
    int8_ms = max_over_ranks(timed(lambda: step(False), steps), dev) / steps
    st = h3q.h3q_get_device_status()
    if st != h3q.H3Q_OK:
        raise RuntimeError(f"device status after the timed region: {h3q.h3q_status_string(st)}")
    per_op = {}
    for name, K, N, swiglu, fp4 in NVFP4_OPS:
        reps = max(3, args.kernel_reps)
        t8 = max_over_ranks(timed(lambda: run_op(name, False), reps), dev) / reps
        t4 = max_over_ranks(timed(lambda: run_op(name, True), reps), dev) / reps
        per_op[name] = {"int8_convrot_ms": t8, "nvfp4_ms": t4, "change": t4 / t8 - 1.0, "nvfp4_in_hybrid": fp4}
    o = ops["ffn_in"]
    reps = max(3, args.kernel_reps)
    dom_ms = max_over_ranks(timed(lambda: h3q.h3q_linear_nvfp4(o["xc"], o["xsf"], o["xs"], o["wc"], o["wsf"], o["ws"],
                                                                o["y"], epilogue=o["epi"]), reps), dev) / reps
    if rank == 0:
        ms = total_ms / steps
        flops = sum(2.0 * M * N * K for _, K, N, _, _ in NVFP4_OPS)
        peaks, peak_src = measured_peaks()
        fp4_peak = 4.0 * peaks["bf16_tflops"]
        achieved = 2.0 * M * 28672 * 5376 / (dom_ms * 1e-3) / 1e12
        line = {
            "metric": "hybrid NVFP4/INT8 linear TOPS", "value": job_tops(flops, world, ms), "unit": "TOPS",
            "n_gpus": world, "steps": steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "fp4+i8", "data": "synthetic",
            "config": {"workload": f"one block's four linear operations at M={M}: QKV {K0}->16128 and FFN input "
                                   f"{K0}->2x14336+SwiGLU in NVFP4, attention output {K0}->{K0} and FFN output "
                                   f"14336->{K0} in INT8 ConvRot, each with its input's quantization",
                       "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write)",
                       "parallelism": f"replicas x{world}"},
            "all_int8_convrot_ms_per_step": int8_ms,
            "hybrid_vs_int8": int8_ms / ms,
            "per_op_ms": per_op,
            "roofline": {"bound": "tensor", "kernel": "gemm_fp4_kernel<SwiGLU> (FFN input)", "achieved": achieved,
                         "peak": fp4_peak, "unit": "TFLOP/s", "frac": achieved / fp4_peak,
                         "traffic": traffic_from_profile("gemm_fp4_swiglu_ffn_in"),
                         "peak_source": f"{peak_src} bf16 burst {peaks['bf16_tflops']} TFLOP/s x 4 "
                                        "(dense fp4/bf16 nominal ratio 9/2.25)"},
            "gpu_launches": 10 * steps,
            "clocks": clk,
            "e2e": None,
        }
        if not args.no_cpu_baseline:
            try:
                line["cpu_baseline"] = oracle_nvfp4_rate(args.cpu_seconds)
            except Exception as exc:
                line["cpu_baseline"] = {"value": None, "error": repr(exc)}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def oracle_rotquant_rate(K, target_s):
    """The oracle's rotate+quantize of bf16 activation rows of width K on a bounded sample
    of rows, on all host cores and on one core; GB/s of 2 B read + 1 B written per element
    + 4 B per row, as the GPU kernel's figure."""
    import numpy as np

    import oracle
    import synth
    ids = synth.tensor_ids()
    factors = synth.column_factors(K, synth.outlier_columns(0, ids["outlier"], K, int(round(0.01 * K))), 50.0)
    x = synth.activation_host(0, ids["x"], np.arange(4096), K, factors)
    cores = oracle.num_threads()

    def rate(threads, budget):
        oracle.set_num_threads(threads)
        rows = 16
        while True:
            t0 = time.perf_counter()
            oracle.rotate_quant_bf16(x[:rows])
            dt = time.perf_counter() - t0
            if dt >= budget or rows >= x.shape[0]:
                break
            rows = min(x.shape[0], max(rows * 2, int(rows * budget / max(dt, 1e-4) * 1.1)))
        return (3.0 * rows * K + 4.0 * rows) / dt / 1e9, rows, dt
    try:
        all_gbs, all_rows, all_dt = rate(cores, target_s)
        one_gbs, one_rows, one_dt = rate(1, target_s)
    finally:
        oracle.set_num_threads(cores)
    return {"unit": "GB/s", "kind": "oracle", "K": K,
            "all_cores": {"value": all_gbs, "cores": cores, "sample": f"{all_rows} rows, {all_dt:.1f} s"},
            "one_core": {"value": one_gbs, "cores": 1, "sample": f"{one_rows} rows, {one_dt:.1f} s"}}


def oracle_nvfp4_rate(target_s):
    """The oracle's NVFP4 layer on a bounded sample of rows of the QKV projection
    (full weight); GEMM flops per second."""
    import numpy as np

    import oracle
    import synth
    ids = synth.tensor_ids()
    K, N = 5376, 16128
    cw, sfw, ew = oracle.nvfp4_quantize(synth.weight_host(0, ids["w_qkv"], np.arange(N), K))

    def run(rows):
        ca, sfa, ea = oracle.nvfp4_quantize(synth.activation_host(0, ids["x_qkv"], np.arange(rows), K))
        t0 = time.perf_counter()
        oracle.nvfp4_linear(ca, sfa, ea, cw, sfw, ew)
        return time.perf_counter() - t0
    rows = 2
    while True:
        dt = run(rows)
        if dt >= target_s or rows >= 4096:
            break
        rows = min(4096, max(rows * 2, int(rows * target_s / max(dt, 1e-3) * 1.1)))
    return {"value": 2.0 * rows * N * K / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle", "rows": rows, "seconds": dt,
            "sample": f"{rows} token rows of the QKV projection in NVFP4 (full weight), {dt:.1f} s"}


def run_attention(args):
    """int8 attention of one DiT block (S tokens, 42 heads of 128) from a QKV output."""
    import torch
    import torch.distributed as dist

    import w8a8_rotation_quantized_b200 as h3q

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    S = args.M or 16384
    H, D = 42, 128
    gen = torch.Generator(device=dev)
    gen.manual_seed(1000 + rank)
    qkv = torch.randn((S, 3 * H * D), device=dev, dtype=torch.float32, generator=gen).to(torch.bfloat16)
    q, k, v = qkv[:, :H * D], qkv[:, H * D:2 * H * D], qkv[:, 2 * H * D:]
    out = torch.empty((S, H * D), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(h3q.h3q_attention_workspace_size(S, H), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        h3q.h3q_attention_int8(q, k, v, H, out, ws)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def timed(fn, n):
        st = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        en = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for i in range(n):
            flush.fill_(i & 0xFF)
            st[i].record(stream)
            fn()
            en[i].record(stream)
        barrier()
        return sum(a.elapsed_time(b) for a, b in zip(st, en))

    steps = max(1, min(args.steps, 20))
    for _ in range(args.warmup):
        step()
    barrier()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.5)
    t_host0 = time.time()
    total_ms = max_over_ranks(timed(step, steps), dev)
    clk = clocks.stop(t_host0, time.time())
    st = h3q.h3q_get_device_status()
    if st != h3q.H3Q_OK:
        raise RuntimeError(f"device status after the timed region: {h3q.h3q_status_string(st)}")
    qh, kh, vh = (t.reshape(S, H, D).transpose(0, 1)[None].contiguous() for t in (q, k, v))
    sdpa_ms, sdpa_backend = None, None
    from torch.nn.attention import SDPBackend, sdpa_kernel
    for backend in (SDPBackend.CUDNN_ATTENTION, SDPBackend.FLASH_ATTENTION, SDPBackend.EFFICIENT_ATTENTION):
        try:
            with sdpa_kernel([backend]):
                torch.nn.functional.scaled_dot_product_attention(qh, kh, vh)
                torch.cuda.synchronize()
                sdpa_ms = max_over_ranks(
                    timed(lambda: torch.nn.functional.scaled_dot_product_attention(qh, kh, vh), 3), dev) / 3
            sdpa_backend = str(backend).split(".")[-1]
            break
        except RuntimeError:
            continue
    if rank == 0:
        ms = total_ms / steps
        flops = 4.0 * S * S * D * H
        peaks, peak_src = measured_peaks()
        p8, p16 = 2.0 * peaks["bf16_tflops"], peaks["bf16_tflops"]
        mixed = 2.0 / (1.0 / p8 + 1.0 / p16)  # half the work int8, half bf16
        achieved = flops / (ms * 1e-3) / 1e12
        line = {
            "metric": "int8 attention TFLOP/s", "value": achieved * world, "unit": "TFLOP/s", "n_gpus": world,
            "steps": steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "i8+bf16", "data": "synthetic",
            "config": {"workload": f"DiT attention, S={S} tokens, {H} heads x {D} (int8 Q.K^T, bf16 P.V), "
                                   "q/k/v column slices of one [S, 3*5376] bf16 QKV output, N(0,1)",
                       "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write)",
                       "parallelism": f"replicas x{world}"},
            "context_library_bf16_sdpa": {"ms": sdpa_ms, "backend": sdpa_backend,
                                          "note": "library bf16 attention on the same tensors; context, not a target"},
            "roofline": {"bound": "tensor", "kernel": "attn_kernel (+ attn_prep_kernel)", "achieved": achieved,
                         "peak": mixed, "unit": "TFLOP/s", "frac": achieved / mixed,
                         "traffic": traffic_from_profile("attn_kernel_attention"),
                         "peak_source": f"{peak_src}: half the flops at the int8 rate (2 x bf16 burst) and half at "
                                        f"the bf16 burst rate {peaks['bf16_tflops']} TFLOP/s"},
            "gpu_launches": 2 * steps,
            "clocks": clk,
            "e2e": None,
        }
        if not args.no_cpu_baseline:
            try:
                line["cpu_baseline"] = oracle_attention_rate(S, H, args.cpu_seconds)
            except Exception as exc:
                line["cpu_baseline"] = {"value": None, "error": repr(exc)}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def oracle_attention_rate(S, H, target_s):
    """The oracle's int8 attention for a bounded sample of query rows of every head
    (all S keys); flops of the two products per second."""
    import numpy as np

    import oracle
    D = 128
    rng = np.random.default_rng(0)
    bits = np.ascontiguousarray(
        (rng.standard_normal((S, 3 * H * D), dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16))
    q, k, v = bits[:, :H * D], bits[:, H * D:2 * H * D], bits[:, 2 * H * D:]
    n = 1
    while True:
        t0 = time.perf_counter()
        oracle.attention_int8(q, k, v, H, rows=np.arange(n))
        dt = time.perf_counter() - t0
        if dt >= target_s or n >= S:
            break
        n = min(S, max(2 * n, int(n * target_s / max(dt, 1e-3) * 1.1)))
    return {"value": 4.0 * n * S * D * H / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle", "rows": n, "seconds": dt,
            "sample": f"{n} query rows x {H} heads against all {S} keys (includes quantizing all Q/K rows), {dt:.1f} s"}


def oracle_lora_rate(target_s, steps=None):
    """The oracle's LoRA merge on a bounded sample of the gate/up weight's rows
    (full K and rank); flops of the low-rank product per second."""
    import numpy as np

    import oracle
    import synth
    wl = synth.WORKLOADS["lora"]
    ids = synth.tensor_ids()
    N, K = _lora_shapes(wl)[0][1:]
    r = wl.rank
    a = synth.weight_host(wl.seed, ids["lora_a"], np.arange(r), K)

    def run(rows):
        wq, sw = oracle.prepare_weight(synth.weight_host(wl.seed, ids["w_gu"], np.arange(rows), K))
        b = synth.weight_host(wl.seed, ids["lora_b"], np.arange(rows), r)
        t0 = time.perf_counter()
        oracle.lora_merge(wq, sw, a, b, wl.alpha)
        return time.perf_counter() - t0
    rows = 64
    while True:
        dt = run(rows)
        if dt >= target_s or rows >= N:
            break
        rows = min(N, max(rows * 2, int(rows * target_s / max(dt, 1e-3) * 1.1)))
    return {"value": 2.0 * rows * K * r / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle", "rows": rows, "seconds": dt,
            "sample": f"{rows} of {N} rows of the gate/up weight (K={K}, rank {r}), {dt:.1f} s"}


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

    spec = make_spec(args)
    M, K = spec.M, spec.K
    row0, _ = shard_rows(rank, world, M)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    ids = synth.tensor_ids()
    nout = 4 if spec.name == "tiny" else int(round(0.01 * K))
    factors = synth.column_factors(K, synth.outlier_columns(0, ids["outlier"], K, nout),
                                   40.0 if spec.name == "tiny" else 50.0)
    fdev = torch.from_numpy(factors).to(dev)
    ws_bytes = 0

    # ---- inputs generated on the device; weights prepared by the library. Each
    # rank takes its own rows of one long token stream.
    if spec.name == "ffn":
        ffn = FFN(h3q, synth, torch, dev, sp, M, K, spec.F, ids["x"], ids["w_gu"], ids["w_down"], fdev, row0)
        ws_bytes = h3q.h3q_ffn_workspace_size(M, K, spec.F)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

        def step():
            ffn.run(h3q, ws)
        launches_per_step = 4
        in_tensor, out_tensor = ffn.x, ffn.y
    elif spec.name == "sweep":
        # per block: its weights and its three input activations; codes, scales
        # and outputs are shared by all blocks
        bufs = {"xq": torch.empty(M * K, dtype=torch.int8, device=dev),
                "sx": torch.empty(M, dtype=torch.float32, device=dev),
                "y": torch.empty(M * 16128, dtype=torch.bfloat16, device=dev)}
        y_ffn = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
        blocks = []
        for b in range(spec.blocks):
            t = synth.tensor_ids(b)
            fb = torch.from_numpy(synth.column_factors(K, synth.outlier_columns(0, t["outlier"], K, nout), 50.0)).to(dev)
            qkv = Layer(h3q, synth, torch, dev, sp, M, K, 16128, t["x_qkv"], t["w_qkv"], t["b_qkv"], fb, row0,
                        True, bufs)
            out = Layer(h3q, synth, torch, dev, sp, M, K, K, t["x_out"], t["w_out"], t["b_out"], fb, row0,
                        True, bufs)
            ffn_b = FFN(h3q, synth, torch, dev, sp, M, K, spec.F, t["x_ffn"], t["w_gu"], t["w_down"], fb, row0,
                        y_ffn)
            blocks.append((qkv, out, ffn_b))
            torch.cuda.synchronize()
        ws_bytes = h3q.h3q_ffn_workspace_size(M, K, spec.F)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

        def step():
            for qkv, out, ffn_b in blocks:
                qkv.run(h3q)
                out.run(h3q)
                ffn_b.run(h3q, ws)
        launches_per_step = 8 * spec.blocks
        in_tensor, out_tensor = blocks[0][0].x, blocks[0][0].y
    else:
        layer = Layer(h3q, synth, torch, dev, sp, M, K, spec.N, ids["x"], ids["w"], ids["bias"], fdev, row0,
                      spec.bias)

        def step():
            layer.run(h3q)
        launches_per_step = 2
        in_tensor, out_tensor = layer.x, layer.y
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    steps = args.steps if spec.name != "sweep" else max(1, min(args.steps, 5))
    for _ in range(args.warmup):
        step()
    barrier()

    clocks = ClockSampler(local)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier()
    clocks.start()
    time.sleep(0.5)  # the sampler is running before the timed region starts
    t_host0 = time.time()
    for i in range(steps):
        flush.fill_(i & 0xFF)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    barrier()
    clk = clocks.stop(t_host0, time.time())
    total_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(starts, ends)), dev)
    st = h3q.h3q_get_device_status()
    if st != h3q.H3Q_OK:
        raise RuntimeError(f"device status after the timed region: {h3q.h3q_status_string(st)}")

    # ---- per-kernel device times (same stream, events around each launch, L2 flushed)
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

    peaks, peak_src = measured_peaks()
    # int8 dense tensor rate on B200 is twice the bf16 rate (4.5 vs 2.25 PFLOP/s nominal)
    i8_peak = 2.0 * peaks["bf16_tflops"]
    kernels = {}
    if spec.name in ("ffn", "sweep"):
        f = ffn if spec.name == "ffn" else blocks[0][2]
        F = spec.F
        off = [0]

        def carve(nbytes, dtype, shape):
            t = ws[off[0]:off[0] + nbytes].view(dtype).view(*shape)
            off[0] = (off[0] + nbytes + 255) // 256 * 256
            return t
        xq = carve(M * K, torch.int8, (M, K))
        sx = carve(M * 4, torch.float32, (M,))
        hbuf = carve(M * F * 2, torch.bfloat16, (M, F))
        hq = carve(M * F, torch.int8, (M, F))
        sh = carve(M * 4, torch.float32, (M,))
        kernels["rotate_quant_x"] = time_kernel(lambda: h3q.h3q_rotate_quant(f.x, xq, sx))
        kernels["gemm_gate_up_swiglu"] = time_kernel(
            lambda: h3q.h3q_linear_w8a8(xq, sx, f.qgu, f.sgu, hbuf, epilogue=h3q.H3Q_EPI_SWIGLU))
        kernels["rotate_quant_h"] = time_kernel(lambda: h3q.h3q_rotate_quant(hbuf, hq, sh))
        kernels["gemm_down"] = time_kernel(lambda: h3q.h3q_linear_w8a8(hq, sh, f.qd, f.sd, f.y))
        dom_ops = 2.0 * M * (2 * F) * K
        dom_ms = kernels["gemm_gate_up_swiglu"]
        dom_name, dom_tag = "gemm_i8_kernel<SwiGLU> (FFN gate/up)", "gemm_i8_swiglu_ffn"
        rq = {"x": (M * K * 3 + M * 4) / (kernels["rotate_quant_x"] * 1e-3) / 1e9,
              "h": (M * F * 3 + M * 4) / (kernels["rotate_quant_h"] * 1e-3) / 1e9}
    else:
        kernels["rotate_quant_x"] = time_kernel(lambda: h3q.h3q_rotate_quant(layer.x, layer.xq, layer.sx))
        kernels["gemm"] = time_kernel(
            lambda: h3q.h3q_linear_w8a8(layer.xq, layer.sx, layer.wq, layer.sw, layer.y, bias=layer.bias))
        dom_ops = 2.0 * M * spec.N * K
        dom_ms = kernels["gemm"]
        dom_name, dom_tag = "gemm_i8_kernel<BF16> (linear)", f"gemm_i8_bf16_{spec.name}"
        rq = {"x": (M * K * 3 + M * 4) / (kernels["rotate_quant_x"] * 1e-3) / 1e9}

    # ---- end to end through host buffers: every step copies its input from pinned
    # host memory and its output back, through the library's public calls. Copies
    # run on their own streams and overlap the compute of the neighbouring steps
    # (double-buffered device input and output).
    e2e = None
    if not args.no_e2e and spec.name != "sweep":
        e_steps = max(4, steps)  # the same K steps as the device-timed region
        copy_in, copy_out = torch.cuda.Stream(), torch.cuda.Stream()
        x_host = [torch.empty(in_tensor.shape, dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
        for hbuf in x_host:
            hbuf.copy_(in_tensor)
        y_host = [torch.empty(out_tensor.shape, dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
        x_dev = [torch.empty_like(in_tensor) for _ in range(2)]
        y_dev = [torch.empty_like(out_tensor) for _ in range(2)]

        def compute(xd, yd):
            if spec.name == "ffn":
                h3q.h3q_ffn(xd, ffn.qgu, ffn.sgu, ffn.qd, ffn.sd, yd, ws)
            else:
                h3q.h3q_rotate_quant(xd, layer.xq, layer.sx)
                h3q.h3q_linear_w8a8(layer.xq, layer.sx, layer.wq, layer.sw, yd, bias=layer.bias)

        def pipeline(n):
            ev_in = [torch.cuda.Event() for _ in range(n)]
            ev_comp = [torch.cuda.Event() for _ in range(n)]
            ev_out = [torch.cuda.Event() for _ in range(n)]
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            for i in range(n):
                j = i % 2
                copy_in.wait_event(t0)
                if i >= 2:
                    copy_in.wait_event(ev_comp[i - 2])   # x_dev[j] free again
                with torch.cuda.stream(copy_in):
                    x_dev[j].copy_(x_host[j], non_blocking=True)
                    ev_in[i].record(copy_in)
                stream.wait_event(ev_in[i])
                if i >= 2:
                    stream.wait_event(ev_out[i - 2])     # y_dev[j] drained
                compute(x_dev[j], y_dev[j])
                ev_comp[i].record(stream)
                copy_out.wait_event(ev_comp[i])
                with torch.cuda.stream(copy_out):
                    y_host[j].copy_(y_dev[j], non_blocking=True)
                    ev_out[i].record(copy_out)
            stream.wait_event(ev_out[n - 1])
            t1.record(stream)
            return t0, t1
        pipeline(2)
        barrier()
        t0, t1 = pipeline(e_steps)
        barrier()
        e_ms = max_over_ranks(t0.elapsed_time(t1) / e_steps, dev)
        e2e = {"value": job_tops(spec.ops(), world, e_ms), "unit": "TOPS",
               "h2d_bytes_per_step": in_tensor.numel() * 2, "d2h_bytes_per_step": out_tensor.numel() * 2,
               "ms_per_step": e_ms, "steps": e_steps,
               "how": "pinned host buffers; H2D, compute and D2H on separate streams, double-buffered; "
                      "the pipeline's fill (first H2D) and drain (last D2H) are inside the timed region"}

    if rank == 0:
        ms = total_ms / steps
        value = job_tops(spec.ops(), world, ms)
        achieved = dom_ops / (dom_ms * 1e-3) / 1e12
        line = {
            "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
            "steps": steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic",
            "config": spec.describe(world),
            "int8_peak_tops": i8_peak,
            "frac_of_int8_peak": value / i8_peak,
            "frac_of_nominal_int8_peak": value / I8_NOMINAL_TOPS,
            "kernels_ms": kernels,
            "rotquant_gbs": dict(rq, peak=peaks["hbm_gbs"]),
            "roofline": {"bound": "tensor", "kernel": dom_name,
                         "achieved": achieved, "peak": i8_peak, "unit": "TOPS",
                         "frac": achieved / i8_peak, "traffic": traffic_from_profile(dom_tag),
                         "frac_of_nominal": achieved / I8_NOMINAL_TOPS,
                         "nominal_peak": I8_NOMINAL_TOPS,
                         "peak_source": f"{peak_src}: 2 x bf16 burst {peaks['bf16_tflops']} TFLOP/s "
                                        "(int8 dense rate = 2 x bf16 on B200)"},
            "gpu_launches": launches_per_step * steps,
            "clocks": clk,
            "e2e": e2e,
        }
        if spec.name in ("ffn", "sweep"):
            line["ffn_tokens_per_s"] = M * world / (ms * 1e-3) * (1 if spec.name == "ffn" else 1.0 / spec.blocks)
        if not args.no_cpu_baseline:
            try:
                line["cpu_baseline"] = oracle_rate(spec if spec.name != "sweep" else Spec("ffn", M, K, F=spec.F),
                                                   args.cpu_seconds)
            except Exception as exc:  # the line still prints; the reason is kept
                line["cpu_baseline"] = {"value": None, "error": repr(exc)}
            if spec.name in ("ffn", "qkv", "out"):  # the rotate+quantize oracle alone, all cores and one
                try:
                    line["cpu_baseline_rotquant"] = oracle_rotquant_rate(K, min(2.0, args.cpu_seconds))
                except Exception as exc:
                    line["cpu_baseline_rotquant"] = {"value": None, "error": repr(exc)}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "lora":
        return run_lora(args)
    if args.workload == "nvfp4":
        return run_nvfp4(args)
    if args.workload == "attention":
        return run_attention(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
