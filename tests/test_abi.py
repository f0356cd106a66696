"""The C-ABI library on the host: it loads, exports every function the header
declares, and rejects bad arguments before launching anything. No call here
reaches the GPU (each one fails its host-side checks first)."""
import ctypes
import subprocess

import pytest

import w8a8_rotation_quantized_b200 as h3q

INV = h3q.H3Q_ERR_INVALID_ARG


def test_exports_every_header_function():
    names = h3q.header_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(h3q.lib, n), n
    # and nothing but the header's entry points is exported with the h3q_ prefix
    out = subprocess.run(["nm", "-D", "--defined-only", h3q.LIB_PATH], capture_output=True, text=True).stdout
    exported = sorted({ln.split()[-1] for ln in out.splitlines() if ln.split()[-1].startswith("h3q_")})
    assert exported == names


def test_status_strings_and_version():
    assert h3q.h3q_status_string(0) == "ok"
    assert "invalid" in h3q.h3q_status_string(1)
    assert "timed out" in h3q.h3q_status_string(4)
    assert "sm_100a" in h3q.h3q_version()


def test_workspace_size():
    M, K, F = 16384, 5376, 14336
    ws = h3q.h3q_ffn_workspace_size(M, K, F)
    assert ws >= M * K + 4 * M + 2 * M * F + M * F + 4 * M
    assert ws % 256 == 0
    assert h3q.h3q_ffn_workspace_size(-1, K, F) == 0


P = ctypes.c_void_p
FAKE = 0x10000  # never dereferenced: every call below fails a host-side check first


@pytest.mark.parametrize("args", [
    (FAKE, -1, 512, FAKE, FAKE),        # negative M
    (FAKE, 4, 500, FAKE, FAKE),         # K not a multiple of 256
    (FAKE, 4, 0, FAKE, FAKE),           # K = 0
    (None, 4, 512, FAKE, FAKE),         # null input
    (FAKE + 8, 4, 512, FAKE, FAKE),     # misaligned input
    (FAKE, 4, 512, None, FAKE),         # null output
])
def test_rotate_quant_rejects(args):
    assert h3q.lib.h3q_rotate_quant(*args, None) == INV
    assert h3q.lib.h3q_prepare_weight(*args, None) == INV


def test_rotate_quant_too_wide_is_unsupported():
    assert h3q.lib.h3q_rotate_quant(FAKE, 4, 16384 + 256, FAKE, FAKE, None) == h3q.H3Q_ERR_UNSUPPORTED


def test_zero_rows_is_a_noop():
    assert h3q.lib.h3q_rotate_quant(None, 0, 512, None, None, None) == h3q.H3Q_OK
    assert h3q.lib.h3q_linear_w8a8(None, None, 0, 512, None, None, 256, None, 0, None, None) == h3q.H3Q_OK


@pytest.mark.parametrize("M,K,N,epi,bias", [
    (4, 512, 250, 0, None),     # N not a multiple of 8
    (4, 500, 256, 0, None),     # K not a multiple of 256
    (4, 512, 0, 0, None),       # N = 0
    (4, 512, 384, 1, None),     # SwiGLU with F = 192, not a multiple of 128
    (4, 512, 256, 7, None),     # unknown epilogue
    (4, 512, 256, 0, FAKE + 2), # misaligned bias
])
def test_linear_rejects(M, K, N, epi, bias):
    assert h3q.lib.h3q_linear_w8a8(FAKE, FAKE, M, K, FAKE, FAKE, N, bias, epi, FAKE, None) == INV


def test_linear_rejects_null_and_misaligned():
    assert h3q.lib.h3q_linear_w8a8(None, FAKE, 4, 512, FAKE, FAKE, 256, None, 0, FAKE, None) == INV
    assert h3q.lib.h3q_linear_w8a8(FAKE, FAKE, 4, 512, FAKE + 4, FAKE, 256, None, 0, FAKE, None) == INV
    assert h3q.lib.h3q_gemm_s32(FAKE, FAKE, 4, 12, 256, FAKE, None) == INV
    assert h3q.lib.h3q_gemm_s32(FAKE, FAKE, 4, 16, 100, FAKE, None) == INV


def test_ffn_rejects_short_workspace_and_bad_shapes():
    ws = h3q.h3q_ffn_workspace_size(8, 512, 768)
    args = [FAKE, 8, 512, FAKE, FAKE, None, 768, FAKE, FAKE, None, FAKE, FAKE, ws - 1, None]
    assert h3q.lib.h3q_ffn(*args) == INV
    args[12] = ws
    args[11] = FAKE + 16  # workspace must be 256-byte aligned
    assert h3q.lib.h3q_ffn(*args) == INV
    args[11] = FAKE
    args[6] = 640         # F not a multiple of 256
    assert h3q.lib.h3q_ffn(*args) == INV


def test_stalled_wait_rejects_huge_limit():
    assert h3q.lib.h3q_test_stalled_wait(10**12, None) == INV


def test_lora_workspace_size():
    assert h3q.h3q_lora_workspace_size(64, 5376) == 64 * 5376 * 4
    assert h3q.h3q_lora_workspace_size(0, 5376) == 0


def test_lora_merge_rejects():
    ws = h3q.h3q_lora_workspace_size(8, 512)
    f = h3q.lib.h3q_lora_merge
    ok = [FAKE, FAKE, 16, 512, FAKE, FAKE, 8, 1.0, FAKE, ws, None]
    for i, bad in [(3, 500), (3, 0), (2, -1), (6, 0), (9, ws - 1), (0, None), (4, None), (8, None),
                   (5, FAKE + 4), (1, FAKE + 8)]:
        args = list(ok)
        args[i] = bad
        assert f(*args) == INV, (i, bad)
    args = list(ok)
    args[6] = h3q.H3Q_LORA_MAX_RANK + 1
    assert f(*args) == h3q.H3Q_ERR_UNSUPPORTED
    args = list(ok)
    args[3] = 16384 + 256
    assert f(*args) == h3q.H3Q_ERR_UNSUPPORTED
    # N = 0 launches nothing, whatever the pointers
    assert f(None, None, 0, 512, None, None, 8, 1.0, None, 0, None) == h3q.H3Q_OK


def test_nvfp4_sizes_and_rejects():
    assert h3q.h3q_nvfp4_sf_bytes(300, 512) == 384 * 32
    assert h3q.h3q_nvfp4_sf_bytes(128, 5376) == 128 * 336
    q = h3q.lib.h3q_nvfp4_quantize
    assert q(FAKE, 0, 4, 500, FAKE, FAKE, FAKE, None) == INV     # K not a multiple of 256
    assert q(FAKE, 2, 4, 512, FAKE, FAKE, FAKE, None) == INV     # unknown dtype
    assert q(FAKE, 0, 4, 512, FAKE, FAKE, None, None) == INV     # no scale
    assert q(FAKE + 8, 0, 4, 512, FAKE, FAKE, FAKE, None) == INV  # misaligned
    assert q(None, 0, 0, 512, None, None, None, None) == h3q.H3Q_OK
    lin = h3q.lib.h3q_linear_nvfp4
    ok = [FAKE, FAKE, FAKE, 4, 512, FAKE, FAKE, FAKE, 512, None, 0, FAKE, None]
    for i, bad in [(8, 384), (4, 500), (10, 3), (11, None), (0, None), (2, FAKE + 4)]:
        args = list(ok)
        args[i] = bad
        assert lin(*args) == INV, (i, bad)
    assert h3q.lib.h3q_gemm_nvfp4_f32(FAKE, FAKE, 4, 512, FAKE, FAKE, 100, FAKE, None) == INV


def test_attention_rejects():
    f = h3q.lib.h3q_attention_int8
    ws = h3q.h3q_attention_workspace_size(64, 2)
    assert ws >= 2 * 64 * 128 * 4 + 2 * 64 * 4 + 2 * 4  # codes, V^T, qs [H, S], ks [H, S / 128]
    ok = [FAKE, FAKE, FAKE, 64, 2, 256, FAKE, 256, FAKE, ws, None]
    for i, bad in [(3, 60), (4, 0), (5, 200), (5, 260), (7, 100), (9, ws - 1), (8, FAKE + 16), (0, None),
                   (6, FAKE + 8)]:
        args = list(ok)
        args[i] = bad
        assert f(*args) == INV, (i, bad)
    assert f(None, None, None, 0, 2, 256, None, 256, None, 0, None) == h3q.H3Q_OK


def test_binding_rejects_host_tensors_and_wrong_dtypes():
    """The Python binding checks each operand's dtype, device, shape and layout before it
    builds a pointer: a tensor the kernels would index past its end never reaches them."""
    torch = pytest.importorskip("torch")
    x = torch.zeros((4, 256), dtype=torch.bfloat16)
    xq = torch.zeros((4, 256), dtype=torch.int8)
    sx = torch.zeros(4, dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        h3q.h3q_rotate_quant(x, xq, sx)
    with pytest.raises(ValueError, match="must be torch.bfloat16"):
        h3q.h3q_rotate_quant(x.float(), xq, sx)
    with pytest.raises(ValueError, match="must be torch.int8"):
        h3q.h3q_gemm_s32(x, xq, sx)
    with pytest.raises(ValueError, match="is required"):
        h3q.h3q_linear_w8a8(None, sx, xq, sx, x)
