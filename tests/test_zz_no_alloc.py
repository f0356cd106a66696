"""h3q_ffn_static_scratch: the FFN block for callers that cannot allocate.

Some users of the library have no device allocator of their own (they reach it
through plain pointers only, or run inside a host framework that owns all device
memory), and some must not allocate while serving because cudaMalloc/cudaFree can
synchronize the device. For them the library offers an FFN call that takes no
workspace and keeps its intermediates in a fixed device array of the library.

This test calls that entry point through the C ABI twice in a row, on different
shapes and inputs, and checks each result against the workspace-taking h3q_ffn
on the same inputs (within 1 bf16 ulp, the tolerance of the other parity tests;
both run the same kernels, so the outputs are expected to be identical). It also
checks that a request larger than the array is refused without a launch. The
file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import synth  # noqa: E402

pytestmark = pytest.mark.gpu


def _to_dev_bf16(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _ulp_diff(a_bits, b_bits):
    a = synth.bf16_bits_to_fp32(a_bits).astype(np.float64)
    b = synth.bf16_bits_to_fp32(b_bits).astype(np.float64)
    mag = np.maximum(np.abs(a), np.abs(b)).astype(np.float32)
    ulp = np.maximum(np.spacing(mag).astype(np.float64) * 65536.0, 2.0 ** -133)
    return np.abs(a - b) / ulp


def _case(h3q, dev, M, K, F, seed, with_bias):
    f = synth.column_factors(K, synth.outlier_columns(seed, 4, K, max(1, K // 100)), 50.0)
    x = _to_dev_bf16(synth.activation_host(seed, 1, np.arange(M), K, f), dev)
    qgu = torch.empty((2 * F, K), dtype=torch.int8, device=dev)
    sgu = torch.empty(2 * F, dtype=torch.float32, device=dev)
    qd = torch.empty((K, F), dtype=torch.int8, device=dev)
    sd = torch.empty(K, dtype=torch.float32, device=dev)
    h3q.h3q_prepare_weight(torch.from_numpy(synth.weight_host(seed, 5, np.arange(2 * F), K)).to(dev), qgu, sgu)
    h3q.h3q_prepare_weight(torch.from_numpy(synth.weight_host(seed, 6, np.arange(K), F)).to(dev), qd, sd)
    bgu = _to_dev_bf16(synth.bias_host(seed, 8, 2 * F), dev) if with_bias else None
    bd = _to_dev_bf16(synth.bias_host(seed, 10, K), dev) if with_bias else None
    return x, qgu, sgu, qd, sd, bgu, bd


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def test_static_scratch_ffn_matches_workspace_ffn_twice(cuda_device):
    import w8a8_rotation_quantized_b200 as h3q
    dev = cuda_device
    stream = torch.cuda.current_stream().cuda_stream
    for M, K, F, seed, with_bias in [(300, 5376, 14336, 0, False), (64, 512, 768, 1, True)]:
        x, qgu, sgu, qd, sd, bgu, bd = _case(h3q, dev, M, K, F, seed, with_bias)
        y_static = torch.full((M, K), float("nan"), dtype=torch.bfloat16, device=dev)
        st = h3q.lib.h3q_ffn_static_scratch(_p(x), M, K, _p(qgu), _p(sgu), _p(bgu), F, _p(qd), _p(sd), _p(bd),
                                            _p(y_static), stream)
        assert st == h3q.H3Q_OK, h3q.h3q_status_string(st)
        ws = torch.empty(h3q.h3q_ffn_workspace_size(M, K, F), dtype=torch.uint8, device=dev)
        y_ws = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
        h3q.h3q_ffn(x, qgu, sgu, qd, sd, y_ws, ws, b_gu=bgu, b_down=bd)
        torch.cuda.synchronize()
        assert h3q.h3q_get_device_status() == h3q.H3Q_OK
        a, b = _bits(y_static), _bits(y_ws)
        assert _ulp_diff(a, b).max() <= 1.0
        assert np.array_equal(a, b), f"{(a != b).sum()} of {a.size} outputs differ (within 1 ulp)"


def test_static_scratch_ffn_refuses_requests_beyond_its_array(cuda_device):
    import w8a8_rotation_quantized_b200 as h3q
    K, F = 5376, 14336
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the size check fails first
    st = h3q.lib.h3q_ffn_static_scratch(fake, 1387, K, fake, fake, None, F, fake, fake, None, fake, None)
    assert st == h3q.H3Q_ERR_UNSUPPORTED
    assert h3q.h3q_ffn_workspace_size(1386, K, F) <= h3q.H3Q_STATIC_SCRATCH_BYTES
