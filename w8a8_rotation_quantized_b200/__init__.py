"""INT8 ConvRot (W8A8, Hadamard-256) linear layer on B200: Python binding of libh3q.so.

The functions carry the C ABI's names (include/h3q.h) and only marshal
arguments: torch tensors in device memory become pointers, the current CUDA
stream becomes the stream argument, and a non-OK status raises H3QError. Every
step of the computation runs in the library's kernels. There is no fallback:
if the library is missing or cannot be loaded, importing this package fails.
"""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libh3q.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "h3q.h")

H3Q_OK, H3Q_ERR_INVALID_ARG, H3Q_ERR_UNSUPPORTED, H3Q_ERR_CUDA, H3Q_ERR_TIMEOUT = range(5)
H3Q_EPI_NONE, H3Q_EPI_SWIGLU = 0, 1
H3Q_DTYPE_BF16, H3Q_DTYPE_F32 = 0, 1
H3Q_MAX_K = 16384

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python w8a8_rotation_quantized_b200/build.py` "
                      "(or __graft_entry__.build())")

lib = ctypes.CDLL(LIB_PATH)

_P, _I64, _SZ, _INT, _U64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int, ctypes.c_uint64
_SIGS = {
    "h3q_rotate_quant": (_INT, [_P, _I64, _I64, _P, _P, _P]),
    "h3q_prepare_weight": (_INT, [_P, _I64, _I64, _P, _P, _P]),
    "h3q_linear_w8a8": (_INT, [_P, _P, _I64, _I64, _P, _P, _I64, _P, _INT, _P, _P]),
    "h3q_ffn_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "h3q_ffn": (_INT, [_P, _I64, _I64, _P, _P, _P, _I64, _P, _P, _P, _P, _P, _SZ, _P]),
    "h3q_ffn_static_scratch": (_INT, [_P, _I64, _I64, _P, _P, _P, _I64, _P, _P, _P, _P, _P]),
    "h3q_lora_workspace_size": (_SZ, [_I64, _I64]),
    "h3q_lora_merge": (_INT, [_P, _P, _I64, _I64, _P, _P, _I64, ctypes.c_float, _P, _SZ, _P]),
    "h3q_nvfp4_sf_bytes": (_SZ, [_I64, _I64]),
    "h3q_nvfp4_quantize": (_INT, [_P, _INT, _I64, _I64, _P, _P, _P, _P]),
    "h3q_linear_nvfp4": (_INT, [_P, _P, _P, _I64, _I64, _P, _P, _P, _I64, _P, _INT, _P, _P]),
    "h3q_gemm_nvfp4_f32": (_INT, [_P, _P, _I64, _I64, _P, _P, _I64, _P, _P]),
    "h3q_attention_workspace_size": (_SZ, [_I64, _I64]),
    "h3q_attention_int8": (_INT, [_P, _P, _P, _I64, _I64, _I64, _P, _I64, _P, _SZ, _P]),
    "h3q_attention_prep": (_INT, [_P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P]),
    "h3q_gemm_s32": (_INT, [_P, _P, _I64, _I64, _I64, _P, _P]),
    "h3q_get_device_status": (_INT, [_P]),
    "h3q_set_wait_limit_ns": (None, [_U64]),
    "h3q_test_stalled_wait": (_INT, [_U64, _P]),
    "h3q_status_string": (ctypes.c_char_p, [_INT]),
    "h3q_version": (ctypes.c_char_p, []),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype, _fn.argtypes = _res, _args


class H3QError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lib.h3q_status_string(status).decode()} (status {status})")


def header_functions() -> list[str]:
    """Names of the functions include/h3q.h declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]*?\b(h3q_\w+)\s*\(", text, flags=re.M)))


def _check(status: int, where: str) -> None:
    if status != H3Q_OK:
        raise H3QError(status, where)


def _dtypes():
    import torch
    return {"bf16": torch.bfloat16, "f32": torch.float32, "i8": torch.int8, "u8": torch.uint8,
            "i32": torch.int32}


def _need(where: str, name: str, t, dtype: str, shape, device=None, dense: bool = True):
    """Raises ValueError unless t is a CUDA tensor of `dtype` and `shape` (None entries
    match any size), dense (or, with dense=False, with unit column stride) and, when
    given, on `device`. The kernels index their operands from the sizes alone, so a
    tensor of another shape or layout would be read or written out of bounds."""
    if t is None:
        raise ValueError(f"{where}: {name} is required")
    want = _dtypes()[dtype]
    if t.dtype != want:
        raise ValueError(f"{where}: {name} must be {want}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{where}: {name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{where}: {name} is on {t.device}, the other operands on {device}")
    if len(t.shape) != len(shape) or any(w is not None and int(g) != int(w) for g, w in zip(t.shape, shape)):
        raise ValueError(f"{where}: {name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if dense and not t.is_contiguous():
        raise ValueError(f"{where}: {name} must be contiguous (row-major, dense)")
    if not dense and t.dim() == 2 and t.shape[1] > 1 and t.stride(1) != 1:
        raise ValueError(f"{where}: {name} must have unit column stride")
    return t


def _nbytes(where: str, name: str, t, device) -> int:
    """Byte size of a caller-owned scratch tensor (any dtype, contiguous, on `device`)."""
    if t is None or not t.is_cuda or t.device != device or not t.is_contiguous():
        raise ValueError(f"{where}: {name} must be a contiguous CUDA tensor on {device}")
    return t.numel() * t.element_size()


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is not None:
        return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    import torch
    return torch.cuda.current_stream().cuda_stream


def h3q_rotate_quant(x, xq, sx, stream=None) -> None:
    """x bf16 [M, K] -> xq int8 [M, K] (rotated codes), sx fp32 [M]."""
    w = "h3q_rotate_quant"
    M, K = _need(w, "x", x, "bf16", (None, None)).shape
    _need(w, "xq", xq, "i8", (M, K), x.device)
    _need(w, "sx", sx, "f32", (M,), x.device)
    _check(lib.h3q_rotate_quant(_ptr(x), M, K, _ptr(xq), _ptr(sx), _stream(stream)), "h3q_rotate_quant")


def h3q_prepare_weight(w, wq, sw, stream=None) -> None:
    """w fp32 [N, K] -> wq int8 [N, K] (rotated along K), sw fp32 [N]."""
    wh = "h3q_prepare_weight"
    N, K = _need(wh, "w", w, "f32", (None, None)).shape
    _need(wh, "wq", wq, "i8", (N, K), w.device)
    _need(wh, "sw", sw, "f32", (N,), w.device)
    _check(lib.h3q_prepare_weight(_ptr(w), N, K, _ptr(wq), _ptr(sw), _stream(stream)), "h3q_prepare_weight")


def h3q_linear_w8a8(xq, sx, wq, sw, y, bias=None, epilogue=H3Q_EPI_NONE, stream=None) -> None:
    """y bf16 = rescale(xq @ wq^T) (+ bias); SwiGLU epilogue: y [M, N/2]."""
    w = "h3q_linear_w8a8"
    M, K = _need(w, "xq", xq, "i8", (None, None)).shape
    dev = xq.device
    N = _need(w, "wq", wq, "i8", (None, K), dev).shape[0]
    _need(w, "sx", sx, "f32", (M,), dev)
    _need(w, "sw", sw, "f32", (N,), dev)
    if bias is not None:
        _need(w, "bias", bias, "bf16", (N,), dev)
    _need(w, "y", y, "bf16", (M, N // 2 if int(epilogue) == H3Q_EPI_SWIGLU else N), dev)
    _check(lib.h3q_linear_w8a8(_ptr(xq), _ptr(sx), M, K, _ptr(wq), _ptr(sw), N, _ptr(bias), int(epilogue),
                               _ptr(y), _stream(stream)), "h3q_linear_w8a8")


def h3q_ffn_workspace_size(M: int, K: int, F: int) -> int:
    return int(lib.h3q_ffn_workspace_size(M, K, F))


def _ffn_operands(w, x, w_gu, s_gu, w_down, s_down, y, b_gu, b_down):
    M, K = _need(w, "x", x, "bf16", (None, None)).shape
    dev = x.device
    F2 = _need(w, "w_gu", w_gu, "i8", (None, K), dev).shape[0]
    if F2 % 2:
        raise ValueError(f"{w}: w_gu must have an even row count (gate rows, then up rows), got {F2}")
    F = F2 // 2
    _need(w, "s_gu", s_gu, "f32", (2 * F,), dev)
    _need(w, "w_down", w_down, "i8", (K, F), dev)
    _need(w, "s_down", s_down, "f32", (K,), dev)
    _need(w, "y", y, "bf16", (M, K), dev)
    if b_gu is not None:
        _need(w, "b_gu", b_gu, "bf16", (2 * F,), dev)
    if b_down is not None:
        _need(w, "b_down", b_down, "bf16", (K,), dev)
    return M, K, F


def h3q_ffn(x, w_gu, s_gu, w_down, s_down, y, workspace, b_gu=None, b_down=None, stream=None) -> None:
    """y [M, K] = down(rotquant(swiglu(gate_up(rotquant(x)))))."""
    w = "h3q_ffn"
    M, K, F = _ffn_operands(w, x, w_gu, s_gu, w_down, s_down, y, b_gu, b_down)
    nbytes = _nbytes(w, "workspace", workspace, x.device)
    _check(lib.h3q_ffn(_ptr(x), M, K, _ptr(w_gu), _ptr(s_gu), _ptr(b_gu), F, _ptr(w_down), _ptr(s_down),
                       _ptr(b_down), _ptr(y), _ptr(workspace), nbytes, _stream(stream)), "h3q_ffn")


H3Q_STATIC_SCRATCH_BYTES = 64 << 20


def h3q_ffn_static_scratch(x, w_gu, s_gu, w_down, s_down, y, b_gu=None, b_down=None, stream=None) -> None:
    """h3q_ffn without a workspace, for callers that cannot allocate device memory:
    the intermediates live in the library's fixed 64 MiB device array, shared by
    all calls (calls that may overlap on the GPU must be serialized)."""
    M, K, F = _ffn_operands("h3q_ffn_static_scratch", x, w_gu, s_gu, w_down, s_down, y, b_gu, b_down)
    _check(lib.h3q_ffn_static_scratch(_ptr(x), M, K, _ptr(w_gu), _ptr(s_gu), _ptr(b_gu), F, _ptr(w_down),
                                      _ptr(s_down), _ptr(b_down), _ptr(y), _stream(stream)),
           "h3q_ffn_static_scratch")


H3Q_LORA_MAX_RANK = 512


def h3q_lora_workspace_size(r: int, K: int) -> int:
    return int(lib.h3q_lora_workspace_size(r, K))


def h3q_lora_merge(wq, sw, lora_a, lora_b, alpha: float, workspace, stream=None) -> None:
    """Merge alpha * lora_b @ lora_a (rotated along K) into the int8 weights
    wq [N, K] / sw [N], in place. lora_a [r, K], lora_b [N, r] fp32."""
    w = "h3q_lora_merge"
    N, K = _need(w, "wq", wq, "i8", (None, None)).shape
    dev = wq.device
    _need(w, "sw", sw, "f32", (N,), dev)
    r = _need(w, "lora_a", lora_a, "f32", (None, K), dev).shape[0]
    _need(w, "lora_b", lora_b, "f32", (N, r), dev)
    nbytes = _nbytes(w, "workspace", workspace, dev)
    _check(lib.h3q_lora_merge(_ptr(wq), _ptr(sw), N, K, _ptr(lora_a), _ptr(lora_b), r, float(alpha),
                              _ptr(workspace), nbytes, _stream(stream)), "h3q_lora_merge")


def h3q_nvfp4_sf_bytes(rows: int, K: int) -> int:
    return int(lib.h3q_nvfp4_sf_bytes(rows, K))


def h3q_nvfp4_quantize(x, codes, sf, scale, stream=None) -> None:
    """x [rows, K] bf16 or fp32 -> codes uint8 [rows, K/2], sf uint8 [h3q_nvfp4_sf_bytes],
    scale fp32 [2] (max|x|, s_enc)."""
    import torch
    w = "h3q_nvfp4_quantize"
    rows, K = _need(w, "x", x, "bf16" if x.dtype == torch.bfloat16 else "f32", (None, None)).shape
    dt = H3Q_DTYPE_BF16 if x.dtype == torch.bfloat16 else H3Q_DTYPE_F32
    _need(w, "codes", codes, "u8", (rows, K // 2), x.device)
    _need(w, "sf", sf, "u8", (h3q_nvfp4_sf_bytes(rows, K),), x.device)
    _need(w, "scale", scale, "f32", (2,), x.device)
    _check(lib.h3q_nvfp4_quantize(_ptr(x), dt, rows, K, _ptr(codes), _ptr(sf), _ptr(scale), _stream(stream)),
           "h3q_nvfp4_quantize")


def _nvfp4_operands(w, xc, xsf, wc, wsf):
    M, K2 = _need(w, "xc", xc, "u8", (None, None)).shape
    dev = xc.device
    N = _need(w, "wc", wc, "u8", (None, K2), dev).shape[0]
    _need(w, "xsf", xsf, "u8", (h3q_nvfp4_sf_bytes(M, 2 * K2),), dev)
    _need(w, "wsf", wsf, "u8", (h3q_nvfp4_sf_bytes(N, 2 * K2),), dev)
    return M, N, K2


def h3q_linear_nvfp4(xc, xsf, x_scale, wc, wsf, w_scale, y, bias=None, epilogue=H3Q_EPI_NONE, stream=None) -> None:
    """y bf16 = NVFP4 linear of x (codes xc [M, K/2]) with w (codes wc [N, K/2])."""
    w = "h3q_linear_nvfp4"
    M, N, K2 = _nvfp4_operands(w, xc, xsf, wc, wsf)
    _need(w, "x_scale", x_scale, "f32", (2,), xc.device)
    _need(w, "w_scale", w_scale, "f32", (2,), xc.device)
    if bias is not None:
        _need(w, "bias", bias, "bf16", (N,), xc.device)
    _need(w, "y", y, "bf16", (M, N // 2 if int(epilogue) == H3Q_EPI_SWIGLU else N), xc.device)
    _check(lib.h3q_linear_nvfp4(_ptr(xc), _ptr(xsf), _ptr(x_scale), M, 2 * K2, _ptr(wc), _ptr(wsf), _ptr(w_scale), N,
                                _ptr(bias), int(epilogue), _ptr(y), _stream(stream)), "h3q_linear_nvfp4")


def h3q_gemm_nvfp4_f32(xc, xsf, wc, wsf, acc, stream=None) -> None:
    """acc fp32 [M, N]: the raw NVFP4 accumulators (test hook)."""
    w = "h3q_gemm_nvfp4_f32"
    M, N, K2 = _nvfp4_operands(w, xc, xsf, wc, wsf)
    _need(w, "acc", acc, "f32", (M, N), xc.device)
    _check(lib.h3q_gemm_nvfp4_f32(_ptr(xc), _ptr(xsf), M, 2 * K2, _ptr(wc), _ptr(wsf), N, _ptr(acc),
                                  _stream(stream)), "h3q_gemm_nvfp4_f32")


def h3q_attention_workspace_size(S: int, H: int) -> int:
    return int(lib.h3q_attention_workspace_size(S, H))


def _ld(t):
    return t.stride(0)


def _attention_inputs(w, q, k, v, H):
    """q, k, v: [S, >= 128 H] bf16 views with unit column stride and one common row stride."""
    S = _need(w, "q", q, "bf16", (None, None), dense=False).shape[0]
    for name, t in (("k", k), ("v", v)):
        _need(w, name, t, "bf16", (S, None), q.device, dense=False)
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.shape[1] < 128 * H:
            raise ValueError(f"{w}: {name} must have at least {128 * H} columns, got {t.shape[1]}")
        if t.stride(0) != q.stride(0):
            raise ValueError(f"{w}: q, k and v must share one row stride")
    return S


def h3q_attention_int8(q, k, v, H, out, workspace, stream=None) -> None:
    """out [S, >= 128 H] bf16 = int8 attention of q, k, v ([S, ld] bf16 views, head h
    at columns h*128; q, k, v may be column slices of one matrix)."""
    w = "h3q_attention_int8"
    S = _attention_inputs(w, q, k, v, H)
    _need(w, "out", out, "bf16", (S, None), q.device, dense=False)
    if out.shape[1] < 128 * H:
        raise ValueError(f"{w}: out must have at least {128 * H} columns, got {out.shape[1]}")
    nbytes = _nbytes(w, "workspace", workspace, q.device)
    _check(lib.h3q_attention_int8(_ptr(q), _ptr(k), _ptr(v), S, H, _ld(q), _ptr(out), _ld(out), _ptr(workspace),
                                  nbytes, _stream(stream)), "h3q_attention_int8")


def h3q_attention_prep(q, k, v, H, qq, qs, kq, ks, vt, stream=None) -> None:
    """The attention's input pass: int8 Q codes and scales per token and head, K codes per
    head with one scale per block of 128 keys (ks [H, ceil(S/128)]), V^T per head."""
    w = "h3q_attention_prep"
    S = _attention_inputs(w, q, k, v, H)
    dev = q.device
    _need(w, "qq", qq, "i8", (H, S, 128), dev)
    _need(w, "kq", kq, "i8", (H, S, 128), dev)
    _need(w, "qs", qs, "f32", (H, S), dev)
    _need(w, "ks", ks, "f32", (H, (S + 127) // 128), dev)
    _need(w, "vt", vt, "bf16", (H * 128, S), dev)
    _check(lib.h3q_attention_prep(_ptr(q), _ptr(k), _ptr(v), S, H, _ld(q), _ptr(qq), _ptr(qs), _ptr(kq), _ptr(ks),
                                  _ptr(vt), _stream(stream)), "h3q_attention_prep")


def h3q_gemm_s32(xq, wq, acc, stream=None) -> None:
    """acc int32 [M, N] = xq [M, K] @ wq [N, K]^T."""
    w = "h3q_gemm_s32"
    M, K = _need(w, "xq", xq, "i8", (None, None)).shape
    N = _need(w, "wq", wq, "i8", (None, K), xq.device).shape[0]
    _need(w, "acc", acc, "i32", (M, N), xq.device)
    _check(lib.h3q_gemm_s32(_ptr(xq), _ptr(wq), M, N, K, _ptr(acc), _stream(stream)), "h3q_gemm_s32")


def h3q_get_device_status(stream=None) -> int:
    return int(lib.h3q_get_device_status(_stream(stream)))


def h3q_set_wait_limit_ns(ns: int) -> None:
    lib.h3q_set_wait_limit_ns(int(ns))


def h3q_test_stalled_wait(limit_ns: int, stream=None) -> None:
    _check(lib.h3q_test_stalled_wait(int(limit_ns), _stream(stream)), "h3q_test_stalled_wait")


def h3q_status_string(status: int) -> str:
    return lib.h3q_status_string(int(status)).decode()


def h3q_version() -> str:
    return lib.h3q_version().decode()
