"""CPU oracle for the INT8 ConvRot linear layer: numpy front end over ``h3q_oracle.cpp``.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers. The product path neither
imports this package nor shares code with it.

Every function follows the step of the same number in ``h3q_oracle.cpp``,
whose header cites the passages of the pages each step comes from. Arrays are
numpy; bf16 tensors travel as their uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "h3q_oracle.cpp")
_LIB = os.path.join(_HERE, "libh3q_oracle.so")
_FLAGS = ["-O2", "-std=c++17", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC"]

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle library in place (gcc), if missing or older than its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", *_FLAGS, "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P, I64, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float
        sig = {
            "orc_hadamard256": (None, [P]),
            "orc_rotate_f32": (None, [P, I64, I64, P]),
            "orc_rotate_f64": (None, [P, I64, I64, P]),
            "orc_quantize_rows": (None, [P, I64, I64, P, P]),
            "orc_rotate_quant_bf16": (None, [P, I64, I64, P, P]),
            "orc_prepare_weight": (None, [P, I64, I64, P, P]),
            "orc_gemm_s32": (I64, [P, P, I64, I64, I64, P]),
            "orc_epilogue": (None, [P, P, P, P, I64, I64, P, P]),
            "orc_exp_f32": (F, [F]),
            "orc_silu_f32": (F, [F]),
            "orc_exp_f32_array": (None, [P, I64, P]),
            "orc_silu_f32_array": (None, [P, I64, P]),
            "orc_swiglu": (None, [P, I64, I64, P, P]),
            "orc_linear": (I64, [P, I64, I64, P, P, I64, P, ctypes.c_int, P, P, P, P, P]),
            "orc_ffn": (I64, [P, I64, I64, P, P, P, I64, P, P, P, P, P, P, P]),
            "orc_num_threads": (ctypes.c_int, []),
            "orc_set_num_threads": (None, [ctypes.c_int]),
            "orc_lora_merge": (None, [P, P, I64, I64, P, P, I64, F]),
            "orc_f32_to_bf16": (ctypes.c_uint16, [F]),
            "orc_bf16_to_f32": (F, [ctypes.c_uint16]),
            "orc_e2m1_value": (F, [ctypes.c_uint8]),
            "orc_e2m1_rne": (ctypes.c_uint8, [F]),
            "orc_e4m3_value": (F, [ctypes.c_uint8]),
            "orc_e4m3_rne_sat": (ctypes.c_uint8, [F]),
            "orc_nvfp4_encode_scale": (F, [P, I64]),
            "orc_nvfp4_quantize": (None, [P, I64, I64, F, P, P]),
            "orc_nvfp4_linear": (None, [P, P, F, I64, I64, P, P, F, I64, P, ctypes.c_int, P, P, P]),
            "orc_nvfp4_epilogue": (None, [P, I64, I64, F, F, P, ctypes.c_int, P]),
            "orc_attention_int8": (None, [P, P, P, I64, I64, I64, I64, P, P, P, P, P, I64, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype, fn.argtypes = res, args
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(_load().orc_num_threads())


def set_num_threads(n: int) -> None:
    """Thread count of the oracle's parallel loops from now on (for timing on one core)."""
    _load().orc_set_num_threads(int(n))


def f32_to_bf16(v: float) -> int:
    """bf16 bits of an fp32 value, round to nearest even."""
    return int(_load().orc_f32_to_bf16(float(v)))


def hadamard256() -> np.ndarray:
    """Step 1: H[i, j] = (-1)^popcount(i & j), int8 [256, 256]."""
    H = np.empty((256, 256), dtype=np.int8)
    _load().orc_hadamard256(_p(H))
    return H


def rotate_f32(v) -> np.ndarray:
    """Step 2: block-diagonal H/16 rotation of fp32 rows, pinned pairwise summation."""
    v = _c(v, np.float32)
    rows, K = v.shape
    assert K % 256 == 0
    y = np.empty_like(v)
    _load().orc_rotate_f32(_p(v), rows, K, _p(y))
    return y


def rotate_f64(v) -> np.ndarray:
    v = _c(v, np.float64)
    rows, K = v.shape
    assert K % 256 == 0
    y = np.empty_like(v)
    _load().orc_rotate_f64(_p(v), rows, K, _p(y))
    return y


def quantize_rows(y):
    """Steps 3-4: per-row absmax/127 scale and clamp(rne(y/s)) codes."""
    y = _c(y, np.float32)
    rows, K = y.shape
    q = np.empty((rows, K), dtype=np.int8)
    s = np.empty(rows, dtype=np.float32)
    _load().orc_quantize_rows(_p(y), rows, K, _p(q), _p(s))
    return q, s


def rotate_quant_bf16(x_bits):
    """Activations: bf16 bits [M, K] -> (int8 [M, K], fp32 [M])."""
    x = _c(x_bits, np.uint16)
    rows, K = x.shape
    assert K % 256 == 0
    q = np.empty((rows, K), dtype=np.int8)
    s = np.empty(rows, dtype=np.float32)
    _load().orc_rotate_quant_bf16(_p(x), rows, K, _p(q), _p(s))
    return q, s


def prepare_weight(w):
    """Step 5: fp32 weights [N, K] -> rotated per-row int8 codes and fp32 scales."""
    w = _c(w, np.float32)
    N, K = w.shape
    assert K % 256 == 0
    q = np.empty((N, K), dtype=np.int8)
    s = np.empty(N, dtype=np.float32)
    _load().orc_prepare_weight(_p(w), N, K, _p(q), _p(s))
    return q, s


def gemm_s32(xq, wq) -> np.ndarray:
    """Step 6: exact integer GEMM xq [M,K] x wq [N,K]^T -> int32 [M,N]."""
    xq = _c(xq, np.int8)
    wq = _c(wq, np.int8)
    M, K = xq.shape
    N, K2 = wq.shape
    assert K == K2
    acc = np.empty((M, N), dtype=np.int32)
    ovf = _load().orc_gemm_s32(_p(xq), _p(wq), M, N, K, _p(acc))
    if ovf:
        raise OverflowError(f"{ovf} accumulators outside the int32 range")
    return acc


def epilogue(acc, sx, sw, bias_bits=None):
    """Step 7: v = ((float)acc * sx) * sw (+ bias); returns (v fp32, bf16 bits)."""
    acc = _c(acc, np.int32)
    M, N = acc.shape
    sx = _c(sx, np.float32)
    sw = _c(sw, np.float32)
    b = None if bias_bits is None else _c(bias_bits, np.uint16)
    v = np.empty((M, N), dtype=np.float32)
    out = np.empty((M, N), dtype=np.uint16)
    _load().orc_epilogue(_p(acc), _p(sx), _p(sw), _p(b), M, N, _p(v), _p(out))
    return v, out


def exp_f32(t: float) -> float:
    return float(_load().orc_exp_f32(float(t)))


def silu_f32(g: float) -> float:
    return float(_load().orc_silu_f32(float(g)))


def exp_f32_array(t: np.ndarray) -> np.ndarray:
    t = np.ascontiguousarray(t, dtype=np.float32)
    out = np.empty_like(t)
    _load().orc_exp_f32_array(t.ctypes.data, t.size, out.ctypes.data)
    return out


def silu_f32_array(g: np.ndarray) -> np.ndarray:
    g = np.ascontiguousarray(g, dtype=np.float32)
    out = np.empty_like(g)
    _load().orc_silu_f32_array(g.ctypes.data, g.size, out.ctypes.data)
    return out


def swiglu(v):
    """Step 8: v [M, 2F] -> (h fp32 [M, F], bf16 bits [M, F])."""
    v = _c(v, np.float32)
    M, N2 = v.shape
    F = N2 // 2
    h = np.empty((M, F), dtype=np.float32)
    out = np.empty((M, F), dtype=np.uint16)
    _load().orc_swiglu(_p(v), M, F, _p(h), _p(out))
    return h, out


def linear(x_bits, wq, sw, bias_bits=None, swiglu_epilogue=False, want=()):
    """The layer: rotate+quant x, GEMM with wq, epilogue (optionally SwiGLU).

    Returns the bf16 bits of y, plus a dict with any of "xq", "sx", "acc", "v"
    named in ``want``.
    """
    x = _c(x_bits, np.uint16)
    wq = _c(wq, np.int8)
    sw = _c(sw, np.float32)
    M, K = x.shape
    N = wq.shape[0]
    b = None if bias_bits is None else _c(bias_bits, np.uint16)
    y = np.empty((M, N // 2 if swiglu_epilogue else N), dtype=np.uint16)
    extra = {}
    xq = np.empty((M, K), dtype=np.int8) if "xq" in want else None
    sx = np.empty(M, dtype=np.float32) if "sx" in want else None
    acc = np.empty((M, N), dtype=np.int32) if "acc" in want else None
    v = np.empty((M, N), dtype=np.float32) if "v" in want else None
    ovf = _load().orc_linear(_p(x), M, K, _p(wq), _p(sw), N, _p(b), 1 if swiglu_epilogue else 0, _p(y),
                             _p(xq), _p(sx), _p(acc), _p(v))
    if ovf:
        raise OverflowError(f"{ovf} accumulators outside the int32 range")
    for name, arr in (("xq", xq), ("sx", sx), ("acc", acc), ("v", v)):
        if arr is not None:
            extra[name] = arr
    return y, extra


def lora_merge(wq, sw, lora_a, lora_b, alpha):
    """LoRA merge: (wq, sw) rotated int8 rows plus alpha * B A, A rotated along K,
    requantized per row. Returns new (wq, sw); the inputs are not modified."""
    q = np.array(wq, dtype=np.int8, copy=True, order="C")
    s = np.array(sw, dtype=np.float32, copy=True, order="C")
    a = _c(lora_a, np.float32)
    b = _c(lora_b, np.float32)
    N, K = q.shape
    r = a.shape[0]
    assert a.shape == (r, K) and b.shape == (N, r) and K % 256 == 0
    _load().orc_lora_merge(_p(q), _p(s), N, K, _p(a), _p(b), r, float(alpha))
    return q, s


def ffn(x_bits, w_gu, s_gu, w_down, s_down, b_gu=None, b_down=None):
    """Step 9: y = down(rotquant(swiglu(gate_up(rotquant(x))))).

    Returns (y bits [M, K], h bits [M, F], hq [M, F], sh [M]).
    """
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    w_gu = _c(w_gu, np.int8)
    F = w_gu.shape[0] // 2
    w_down = _c(w_down, np.int8)
    assert w_down.shape == (K, F)
    y = np.empty((M, K), dtype=np.uint16)
    h = np.empty((M, F), dtype=np.uint16)
    hq = np.empty((M, F), dtype=np.int8)
    sh = np.empty(M, dtype=np.float32)
    bg = None if b_gu is None else _c(b_gu, np.uint16)
    bd = None if b_down is None else _c(b_down, np.uint16)
    ovf = _load().orc_ffn(_p(x), M, K, _p(w_gu), _p(_c(s_gu, np.float32)), _p(bg), F,
                          _p(w_down), _p(_c(s_down, np.float32)), _p(bd), _p(y), _p(h), _p(hq), _p(sh))
    if ovf:
        raise OverflowError(f"{ovf} accumulators outside the int32 range")
    return y, h, hq, sh


# ----------------------------------------------------------------------- NVFP4
def e2m1_value(c: int) -> float:
    return float(_load().orc_e2m1_value(int(c)))


def e2m1_rne(x: float) -> int:
    return int(_load().orc_e2m1_rne(float(x)))


def e4m3_value(c: int) -> float:
    return float(_load().orc_e4m3_value(int(c)))


def e4m3_rne_sat(u: float) -> int:
    return int(_load().orc_e4m3_rne_sat(float(u)))


def nvfp4_encode_scale(x) -> float:
    """Per-tensor encode scale 2688 / max|x| (x: fp32 values, or bf16 bits as uint16)."""
    x = _values_f32(x)
    return float(_load().orc_nvfp4_encode_scale(_p(x), x.size))


def _values_f32(x):
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return np.ascontiguousarray((x.astype(np.uint32) << 16).view(np.float32))
    return _c(x, np.float32)


def nvfp4_quantize(x, s_enc=None):
    """NVFP4 of rows x [rows, K] (fp32, or bf16 bits as uint16). Returns
    (codes uint8 [rows, K/2], sf uint8 [rows, K/16], s_enc)."""
    x = _values_f32(x)
    rows, K = x.shape
    assert K % 16 == 0
    if s_enc is None:
        s_enc = nvfp4_encode_scale(x)
    codes = np.empty((rows, K // 2), dtype=np.uint8)
    sf = np.empty((rows, K // 16), dtype=np.uint8)
    _load().orc_nvfp4_quantize(_p(x), rows, K, float(s_enc), _p(codes), _p(sf))
    return codes, sf, float(s_enc)


def nvfp4_linear(ca, sfa, s_enc_a, cw, sfw, s_enc_w, bias_bits=None, swiglu_epilogue=False):
    """The NVFP4 layer. Returns (y bf16 bits, acc fp64 [M, N], mag fp64 [M, N])."""
    ca, sfa, cw, sfw = (_c(a, np.uint8) for a in (ca, sfa, cw, sfw))
    M, K2 = ca.shape
    N = cw.shape[0]
    K = 2 * K2
    b = None if bias_bits is None else _c(bias_bits, np.uint16)
    y = np.empty((M, N // 2 if swiglu_epilogue else N), dtype=np.uint16)
    acc = np.empty((M, N), dtype=np.float64)
    mag = np.empty((M, N), dtype=np.float64)
    _load().orc_nvfp4_linear(_p(ca), _p(sfa), float(s_enc_a), M, K, _p(cw), _p(sfw), float(s_enc_w), N, _p(b),
                             1 if swiglu_epilogue else 0, _p(y), _p(acc), _p(mag))
    return y, acc, mag


def nvfp4_epilogue(acc32, s_enc_a, s_enc_w, bias_bits=None, swiglu_epilogue=False):
    """The NVFP4 layer's epilogue on given fp32 accumulators [M, N]: bf16 bits."""
    acc = _c(acc32, np.float32)
    M, N = acc.shape
    b = None if bias_bits is None else _c(bias_bits, np.uint16)
    y = np.empty((M, N // 2 if swiglu_epilogue else N), dtype=np.uint16)
    _load().orc_nvfp4_epilogue(_p(acc), M, N, float(s_enc_a), float(s_enc_w), _p(b), 1 if swiglu_epilogue else 0,
                               _p(y))
    return y


# ------------------------------------------------------------ int8 attention
def attention_int8(q_bits, k_bits, v_bits, H, D=128, rows=None):
    """int8 Q.K^T / softmax / P.V per head. q, k, v: bf16 bits [S, ld], head h at
    columns h*D .. h*D+D-1. Q is quantized per token, K per block of 128 keys.
    Returns (o float64 [n, H*D] for the query rows `rows` (all rows if None),
    qq int8 [H, S, D], qs fp32 [H, S], kq int8 [H, S, D], ks fp32 [H, ceil(S/128)])."""
    q, k, v = (_c(a, np.uint16) for a in (q_bits, k_bits, v_bits))
    assert q.shape == k.shape == v.shape and q.shape[1] >= H * D
    S, ld = q.shape
    qq = np.empty((H, S, D), dtype=np.int8)
    kq = np.empty((H, S, D), dtype=np.int8)
    qs = np.empty((H, S), dtype=np.float32)
    ks = np.empty((H, (S + 127) // 128), dtype=np.float32)
    r = None if rows is None else _c(rows, np.int64)
    n = S if r is None else r.size
    o = np.empty((n, H * D), dtype=np.float64)
    _load().orc_attention_int8(_p(q), _p(k), _p(v), S, D, H, ld, _p(qq), _p(qs), _p(kq), _p(ks), _p(r), n, _p(o))
    return o, qq, qs, kq, ks
