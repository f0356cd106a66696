"""Seeded synthetic inputs for the INT8 ConvRot linear layer.

This module is the one piece of code that both the CPU oracle tests and the
CUDA path consume. It draws random numbers and lays out tensors; it performs no
step of the method itself (no rotation, no quantization, no product).

Generator (integer-only until the last scaling, so every implementation that
follows this definition produces the same bits):

* ``mix64`` is the splitmix64 output function (Steele, Lea and Flood, "Fast
  splittable pseudorandom number generators", OOPSLA 2014): xor-shift 30,
  multiply by 0xBF58476D1CE4E5B9, xor-shift 27, multiply by 0x94D049BB133111EB,
  xor-shift 31, all modulo 2**64.
* ``word(key, c) = mix64(key + (c + 1) * GAMMA)`` with GAMMA = 0x9E3779B97F4A7C15
  is the c-th output of a splitmix64 stream whose state starts at ``key``.
* A tensor's stream key is ``word(seed, tensor_id)``.
* Element ``i`` (row-major linear index) of a tensor takes the three words
  ``word(key, 3i)``, ``word(key, 3i+1)``, ``word(key, 3i+2)``, splits them into
  twelve 16-bit integers and sums them to ``S``.  ``z = (2S - 12*65535) / 2**17``
  is an Irwin-Hall approximation of N(0, 1) (mean 0, variance 1) and is exact
  in fp32.
* Activations: ``v = z`` (sigma 1); on an outlier column ``v = fp32(v * factor)``;
  the stored value is ``bf16_rne(v)``.
* Weights: ``fp32(z * sigma_w)`` with sigma_w = fp32(0.02).
* Biases: ``bf16_rne(fp32(z * 0.01f))``.
* Outlier columns: a partial Fisher-Yates shuffle of ``range(K)`` drawn from the
  stream of ``outlier_tensor_id``: for t = 0, 1, ...: ``j = t + word(key, t) mod
  (K - t)``, swap entries t and j; the first ``n`` entries are the outliers.

The workloads are synthetic stand-ins for MiniMax H3 DiT activations and
weights (hidden 5376, 50 blocks), which are not available.
"""
from __future__ import annotations

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_C1 = np.uint64(0xBF58476D1CE4E5B9)
_C2 = np.uint64(0x94D049BB133111EB)
_MASK16 = np.uint64(0xFFFF)

SIGMA_W = np.float32(0.02)
SIGMA_BIAS = np.float32(0.01)

__all__ = [
    "mix64", "word", "stream_key", "normal_fp32", "bf16_rne_bits", "bf16_bits_to_fp32",
    "outlier_columns", "activation_bf16", "weight_fp32", "bias_bf16", "column_factors",
    "WORKLOADS", "Workload", "tensor_ids",
]


def mix64(z):
    """splitmix64 output function on uint64 numpy values (wrapping arithmetic)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _C1
        z = (z ^ (z >> np.uint64(27))) * _C2
    return z ^ (z >> np.uint64(31))


def word(key, c):
    """c-th output of the splitmix64 stream whose state starts at ``key``."""
    key = np.asarray(key, dtype=np.uint64)
    c = np.asarray(c, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return mix64(key + (c + np.uint64(1)) * GAMMA)


def stream_key(seed: int, tensor_id: int) -> np.uint64:
    return np.uint64(word(np.uint64(seed), np.uint64(tensor_id)))


def normal_fp32(seed: int, tensor_id: int, index) -> np.ndarray:
    """Irwin-Hall N(0,1) draws (fp32, exact) for the given linear element indices."""
    key = stream_key(seed, tensor_id)
    idx = np.asarray(index, dtype=np.uint64)
    s = np.zeros(idx.shape, dtype=np.int64)
    with np.errstate(over="ignore"):
        base = idx * np.uint64(3)
        for j in range(3):
            w = word(key, base + np.uint64(j))
            for b in range(4):
                s += ((w >> np.uint64(16 * b)) & _MASK16).astype(np.int64)
    # 2S - 12*65535 is an integer below 2**21 in magnitude: exact in fp32, and the
    # power-of-two scale keeps it exact.
    return (2 * s - 12 * 65535).astype(np.float32) * np.float32(2.0 ** -17)


def bf16_rne_bits(x) -> np.ndarray:
    """fp32 -> bf16 bit pattern (uint16) with round-to-nearest-even. Inputs are finite."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return (u >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_fp32(b) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def outlier_columns(seed: int, tensor_id: int, K: int, n: int) -> np.ndarray:
    """First n entries of a seeded partial Fisher-Yates shuffle of range(K)."""
    if n <= 0:
        return np.zeros(0, dtype=np.int64)
    key = stream_key(seed, tensor_id)
    perm = np.arange(K, dtype=np.int64)
    for t in range(n):
        j = t + int(word(key, np.uint64(t)) % np.uint64(K - t))
        perm[t], perm[j] = perm[j], perm[t]
    return np.sort(perm[:n])


def column_factors(K: int, cols, factor: float) -> np.ndarray:
    f = np.ones(K, dtype=np.float32)
    f[np.asarray(cols, dtype=np.int64)] = np.float32(factor)
    return f


def _rows_cols_index(rows, K):
    rows = np.asarray(rows, dtype=np.int64)
    return (rows[:, None] * K + np.arange(K, dtype=np.int64)[None, :]).astype(np.uint64)


def activation_bf16(seed: int, tensor_id: int, rows, K: int, factors: np.ndarray | None = None,
                    chunk_rows: int = 2048) -> np.ndarray:
    """bf16 bit patterns (uint16 [len(rows), K]) of the activation rows ``rows``."""
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((rows.shape[0], K), dtype=np.uint16)
    for r0 in range(0, rows.shape[0], chunk_rows):
        sel = rows[r0:r0 + chunk_rows]
        v = normal_fp32(seed, tensor_id, _rows_cols_index(sel, K))
        if factors is not None:
            v = (v * factors[None, :]).astype(np.float32)
        out[r0:r0 + chunk_rows] = bf16_rne_bits(v)
    return out


def weight_fp32(seed: int, tensor_id: int, rows, K: int, sigma=SIGMA_W, chunk_rows: int = 2048) -> np.ndarray:
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((rows.shape[0], K), dtype=np.float32)
    for r0 in range(0, rows.shape[0], chunk_rows):
        sel = rows[r0:r0 + chunk_rows]
        out[r0:r0 + chunk_rows] = normal_fp32(seed, tensor_id, _rows_cols_index(sel, K)) * np.float32(sigma)
    return out


def bias_bf16(seed: int, tensor_id: int, N: int, sigma=SIGMA_BIAS) -> np.ndarray:
    return bf16_rne_bits(normal_fp32(seed, tensor_id, np.arange(N, dtype=np.uint64)) * np.float32(sigma))


# Tensor ids within one workload.  Per-block tensors of the 50-block sweep use
# tensor_id = 256 * (block + 1) + local id.
TID_X, TID_W, TID_BIAS, TID_OUTLIER, TID_WGU, TID_WDOWN = 1, 2, 3, 4, 5, 6
TID_WQKV, TID_BQKV, TID_WOUT, TID_BOUT, TID_XQKV, TID_XOUT, TID_XFFN = 7, 8, 9, 10, 11, 12, 13
TID_LORA_A, TID_LORA_B, TID_LORA_A_DOWN, TID_LORA_B_DOWN = 14, 15, 16, 17


def tensor_ids(block: int | None = None) -> dict:
    base = 0 if block is None else 256 * (block + 1)
    names = dict(x=TID_X, w=TID_W, bias=TID_BIAS, outlier=TID_OUTLIER, w_gu=TID_WGU, w_down=TID_WDOWN,
                 w_qkv=TID_WQKV, b_qkv=TID_BQKV, w_out=TID_WOUT, b_out=TID_BOUT,
                 x_qkv=TID_XQKV, x_out=TID_XOUT, x_ffn=TID_XFFN, lora_a=TID_LORA_A, lora_b=TID_LORA_B,
                 lora_a_down=TID_LORA_A_DOWN, lora_b_down=TID_LORA_B_DOWN)
    return {k: base + v for k, v in names.items()}


class Workload:
    """Shapes and distributions of one synthetic workload."""

    def __init__(self, name, kind, M, K, N=None, F=None, bias=False, n_outliers=0, outlier_factor=1.0,
                 blocks=1, seed=0, rank=None, alpha=None):
        self.name, self.kind, self.M, self.K, self.N, self.F = name, kind, M, K, N, F
        self.bias, self.n_outliers, self.outlier_factor = bias, n_outliers, outlier_factor
        self.blocks, self.seed = blocks, seed
        self.rank, self.alpha = rank, alpha

    def factors(self, block=None, K=None):
        K = self.K if K is None else K
        if self.n_outliers == 0:
            return None
        cols = outlier_columns(self.seed, tensor_ids(block)["outlier"], K, self.n_outliers)
        return column_factors(K, cols, self.outlier_factor)

    def as_dict(self):
        return {k: getattr(self, k) for k in ("name", "kind", "M", "K", "N", "F", "bias", "n_outliers",
                                                "outlier_factor", "blocks", "seed", "rank", "alpha")
                if getattr(self, k) is not None}


def _pct_outliers(K):
    return int(round(0.01 * K))


WORKLOADS = {
    # 64x512 activations, 4 outlier channels x40; 256x512 weights; seed 0.
    "tiny": Workload("tiny", "linear", M=64, K=512, N=256, n_outliers=4, outlier_factor=40.0),
    # QKV projection at H3 width: 1% outlier channels x50, bf16 bias.
    "qkv": Workload("qkv", "linear", M=4096, K=5376, N=16128, bias=True,
                    n_outliers=_pct_outliers(5376), outlier_factor=50.0),
    # attention output projection at a full clip's token count.
    "out": Workload("out", "linear", M=32768, K=5376, N=5376, bias=True,
                    n_outliers=_pct_outliers(5376), outlier_factor=50.0),
    # fused FFN block with FFN width 14336 (56 Hadamard groups).
    "ffn": Workload("ffn", "ffn", M=16384, K=5376, F=14336,
                    n_outliers=_pct_outliers(5376), outlier_factor=50.0),
    # one denoising step's linear sweep: 50 blocks of QKV, out and FFN at 32768 tokens.
    "sweep": Workload("sweep", "sweep", M=32768, K=5376, N=16128, F=14336, bias=True,
                      n_outliers=_pct_outliers(5376), outlier_factor=50.0, blocks=50),
    # LoRA merge at load into one FFN block's int8 weights (gate/up [28672, 5376]
    # and down [5376, 14336]): rank-64 factors A [r, K] and B [N, r], both
    # N(0, 0.02^2), merged with alpha = 1. M is unused (no activations).
    "lora": Workload("lora", "lora", M=0, K=5376, F=14336, rank=64, alpha=1.0),
}


# ---------------------------------------------------------------------------
# Fast implementations of the same definition: C on the host (OpenMP) and CUDA
# on the device. Both are checked against the numpy functions above.
# ---------------------------------------------------------------------------
import ctypes as _ct
import os as _os
import subprocess as _sp

_HERE = _os.path.dirname(_os.path.abspath(__file__))
_CPU_SRC = _os.path.join(_HERE, "synth.c")
_CPU_LIB = _os.path.join(_HERE, "libh3q_synth_cpu.so")
_GPU_SRC = _os.path.join(_HERE, "synth_gpu.cu")
_GPU_LIB = _os.path.join(_HERE, "libh3q_synth_gpu.so")
_cpu = None
_gpu = None


def _stale(lib, src):
    return not _os.path.exists(lib) or _os.path.getmtime(lib) < _os.path.getmtime(src)


def build(force: bool = False, gpu: bool = True) -> None:
    """Compile the host (gcc) and device (nvcc, sm_100a) generator libraries in place."""
    if force or _stale(_CPU_LIB, _CPU_SRC):
        tmp = _CPU_LIB + f".tmp{_os.getpid()}"
        _sp.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-shared", "-fPIC", "-o", tmp, _CPU_SRC])
        _os.replace(tmp, _CPU_LIB)
    if gpu and (force or _stale(_GPU_LIB, _GPU_SRC)):
        tmp = _GPU_LIB + f".tmp{_os.getpid()}"
        _sp.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-fmad=false",
                        "-Xcompiler", "-fPIC", "-shared", "-o", tmp, _GPU_SRC])
        _os.replace(tmp, _GPU_LIB)


def _cpu_lib():
    global _cpu
    if _cpu is None:
        build(gpu=False)
        lib = _ct.CDLL(_CPU_LIB)
        lib.synth_fill.restype = None
        lib.synth_fill.argtypes = [_ct.c_uint64, _ct.c_uint64, _ct.c_void_p, _ct.c_int64, _ct.c_int64, _ct.c_int64,
                                   _ct.c_float, _ct.c_void_p, _ct.c_int, _ct.c_void_p]
        _cpu = lib
    return _cpu


def _gpu_lib():
    global _gpu
    if _gpu is None:
        if not _os.path.exists(_GPU_LIB):
            raise RuntimeError(f"{_GPU_LIB} is not built; run synth.build()")
        lib = _ct.CDLL(_GPU_LIB)
        lib.synth_fill_device.restype = _ct.c_int
        lib.synth_fill_device.argtypes = [_ct.c_uint64, _ct.c_uint64, _ct.c_int64, _ct.c_int64, _ct.c_int64,
                                          _ct.c_float, _ct.c_void_p, _ct.c_int, _ct.c_void_p, _ct.c_void_p]
        _gpu = lib
    return _gpu


def fill_host(seed, tensor_id, rows, K, scale=1.0, factors=None, bf16=True):
    """C implementation: rows (array of row indices) of a [*, K] tensor."""
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.empty((rows.shape[0], K), dtype=np.uint16 if bf16 else np.float32)
    f = None if factors is None else np.ascontiguousarray(factors, dtype=np.float32)
    _cpu_lib().synth_fill(int(seed), int(tensor_id), rows.ctypes.data, 0, rows.shape[0], K, float(scale),
                          None if f is None else f.ctypes.data, 1 if bf16 else 0, out.ctypes.data)
    return out


def fill_device(seed, tensor_id, row0, nrows, K, out_ptr, stream_ptr=0, scale=1.0, factors_ptr=None, bf16=True):
    """CUDA implementation: writes rows row0 .. row0+nrows-1 into device memory at out_ptr."""
    err = _gpu_lib().synth_fill_device(int(seed), int(tensor_id), int(row0), int(nrows), int(K), float(scale),
                                       factors_ptr, 1 if bf16 else 0, out_ptr, stream_ptr)
    if err != 0:
        raise RuntimeError(f"synth_fill_device failed with CUDA error {err}")


def activation_host(seed, tensor_id, rows, K, factors=None):
    return fill_host(seed, tensor_id, rows, K, 1.0, factors, bf16=True)


def weight_host(seed, tensor_id, rows, K, sigma=SIGMA_W):
    return fill_host(seed, tensor_id, rows, K, float(sigma), None, bf16=False)


def bias_host(seed, tensor_id, N, sigma=SIGMA_BIAS):
    return fill_host(seed, tensor_id, np.zeros(1, dtype=np.int64), N, float(sigma), None, bf16=True)[0]
