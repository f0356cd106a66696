"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Integer outputs (rotated int8 codes, scales as fp32 bits, int32 accumulators)
must match bit for bit. bf16 outputs must be within 1 bf16 ulp of the oracle's
value (the benchmark spec's tolerance); both sides fix the order of every fp32
operation, so they are expected to agree exactly, and the tests also report
the count of differing elements. Small cases are compared in full; the
full-size workloads, in the launch configuration the benchmark times, are
compared on sampled rows and columns the oracle computes one by one.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import synth  # noqa: E402

pytestmark = pytest.mark.gpu

RNG = np.random.default_rng(7)


@pytest.fixture(scope="module")
def h3q(cuda_device):
    import w8a8_rotation_quantized_b200 as mod
    return mod


def _u(dev):
    from _gpu_util import bits, to_dev_bf16
    return bits, to_dev_bf16


def bf16_ulp_diff(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """|difference| in units of the bf16 spacing at the larger magnitude."""
    a = synth.bf16_bits_to_fp32(a_bits).astype(np.float64)
    b = synth.bf16_bits_to_fp32(b_bits).astype(np.float64)
    mag = np.maximum(np.abs(a), np.abs(b))
    ulp = np.spacing(mag.astype(np.float32)).astype(np.float64) * 65536.0
    ulp = np.maximum(ulp, 2.0 ** -133)
    return np.abs(a - b) / ulp


def assert_bf16_close(got, want, where):
    d = bf16_ulp_diff(got, want)
    assert d.max() <= 1.0, f"{where}: max {d.max()} bf16 ulp, {(d > 0).sum()} of {d.size} differ"


# ---------------------------------------------------------------- rotate + quantize
@pytest.mark.parametrize("M,K", [(1, 256), (7, 512), (64, 512), (129, 768), (300, 5376), (33, 14336),
                                 (5, 16384), (130, 1280), (17, 256),
                                 # more rows than SMs, so blocks cycle their ring and the row buffers
                                 (300, 14336), (20, 7168), (1000, 5376), (601, 10752),
                                 # K = 5376 takes two rows per work item: an odd M leaves the last
                                 # item one real row (the other reads as zeros and is not written)
                                 (301, 5376), (1, 5376),
                                 # 8192 rows or more at up to 42 groups run the tensor-memory kernel
                                 # (values parked in tensor memory, two work items in flight, row
                                 # maxima in tagged buffers): 3 rows per item at K = 5376, so 8194
                                 # leaves a last item of one row; K = 10752 takes the searched shape
                                 (8192, 5376), (8194, 5376), (8195, 10752),
                                 # the searched shapes of that kernel for other row lengths: one group
                                 # (64 rows per item), five groups, 28 groups
                                 (8200, 256), (8193, 1280), (8192, 7168)])
def test_rotate_quant_bitexact(h3q, cuda_device, M, K):
    bits, to_dev = _u(cuda_device)
    f = synth.column_factors(K, synth.outlier_columns(0, 4, K, max(1, K // 100)), 50.0)
    x_h = synth.activation_host(0, 1, np.arange(M), K, f)
    if M >= 7:
        x_h[3] = 0                      # all-zero row: s = 0, q = 0
        x_h[5] = 0
        x_h[5, K // 2] = 0x3F80          # a single 1.0: flat rotated group
        x_h[6] = 0xC2C8                  # constant -100 row
        # tiny row (|x| ~ 2^-109): its scale is below 2^-100
        x_h[4] = (0x0900 | (x_h[4] & 0x807F)).astype(np.uint16)
    x = to_dev(x_h, cuda_device)
    xq = torch.empty((M, K), dtype=torch.int8, device=cuda_device)
    sx = torch.empty(M, dtype=torch.float32, device=cuda_device)
    h3q.h3q_rotate_quant(x, xq, sx)
    torch.cuda.synchronize()
    oq, os_ = oracle.rotate_quant_bf16(x_h)
    assert np.array_equal(sx.cpu().numpy().view(np.uint32), os_.view(np.uint32))
    assert np.array_equal(xq.cpu().numpy(), oq)


# fp32 rows longer than 8192 are copied as two boxes per row (a box holds at most
# 256 units of 128 bytes); K = 8448 splits a group across the two boxes.
@pytest.mark.parametrize("N,K", [(256, 512), (264, 5376), (8, 14336), (3, 256), (5, 8448), (3, 16384)])
def test_prepare_weight_bitexact(h3q, cuda_device, N, K):
    w_h = synth.weight_host(0, 2, np.arange(N), K)
    w_h[N // 2, 7] = 3.0  # an outlier weight
    w = torch.from_numpy(w_h).to(cuda_device)
    wq = torch.empty((N, K), dtype=torch.int8, device=cuda_device)
    sw = torch.empty(N, dtype=torch.float32, device=cuda_device)
    h3q.h3q_prepare_weight(w, wq, sw)
    torch.cuda.synchronize()
    oq, os_ = oracle.prepare_weight(w_h)
    assert np.array_equal(sw.cpu().numpy().view(np.uint32), os_.view(np.uint32))
    assert np.array_equal(wq.cpu().numpy(), oq)


def test_prepare_weight_half_integer_quotients(h3q, cuda_device):
    """Weight rows a e0 + b e1 with a + b = 254 and a - b = m odd: the first group
    rotates to values (a + b)/16 and (a - b)/16, so s = 0.125 and the smaller values
    give the quotient m/2, exactly half-integer; with b moved by 1 or 4 ulps the
    quotients sit a few ulps from the half-integers. There the kernel's candidate
    code fails its residual check and the exactly rounded quotient decides."""
    K = 512
    rows = []
    for m in range(1, 254, 2):
        a = np.float32((254 + m) / 2)
        for db in (0, 1, -1, 4, -4):
            b = np.float32((254 - m) / 2)
            for _ in range(abs(db)):
                b = np.nextafter(b, np.float32(np.inf if db > 0 else -np.inf), dtype=np.float32)
            w = np.zeros(K, dtype=np.float32)
            w[0], w[1] = a, b
            w[300] = np.float32(0.001 * m)  # second group: ordinary values
            rows.append(w)
    w_h = np.stack(rows)
    N = w_h.shape[0]
    w = torch.from_numpy(w_h).to(cuda_device)
    wq = torch.empty((N, K), dtype=torch.int8, device=cuda_device)
    sw = torch.empty(N, dtype=torch.float32, device=cuda_device)
    h3q.h3q_prepare_weight(w, wq, sw)
    torch.cuda.synchronize()
    oq, os_ = oracle.prepare_weight(w_h)
    assert np.array_equal(sw.cpu().numpy().view(np.uint32), os_.view(np.uint32))
    got = wq.cpu().numpy()
    assert np.array_equal(got, oq)
    # the exact ties round half to even: m/2 -> the even neighbour
    ties = got[0::5, :256]
    assert set(np.unique(np.abs(ties[:, 1::2]) % 2)) <= {0}


# ---------------------------------------------------------------- int8 GEMM
@pytest.mark.parametrize("M,N,K", [(1, 8, 128), (64, 256, 512), (129, 264, 640), (300, 520, 1024),
                                   (257, 1000, 5376), (128, 256, 128), (640, 512, 256)])
def test_gemm_s32_bitexact(h3q, cuda_device, M, N, K):
    a = RNG.integers(-128, 128, size=(M, K), dtype=np.int64).astype(np.int8)
    b = RNG.integers(-128, 128, size=(N, K), dtype=np.int64).astype(np.int8)
    a[0, :] = -128
    b[0, :] = -128
    acc = torch.empty((M, N), dtype=torch.int32, device=cuda_device)
    h3q.h3q_gemm_s32(torch.from_numpy(a).to(cuda_device), torch.from_numpy(b).to(cuda_device), acc)
    torch.cuda.synchronize()
    assert h3q.h3q_get_device_status() == h3q.H3Q_OK
    want = oracle.gemm_s32(a, b)
    got = acc.cpu().numpy()
    assert np.array_equal(got, want), f"{(got != want).sum()} of {got.size} differ"


def test_gemm_s32_extreme_accumulators(h3q, cuda_device):
    K = 14336
    a = np.full((130, K), 127, dtype=np.int8)
    a[1] = -127
    b = np.full((16, K), 127, dtype=np.int8)
    acc = torch.empty((130, 16), dtype=torch.int32, device=cuda_device)
    h3q.h3q_gemm_s32(torch.from_numpy(a).to(cuda_device), torch.from_numpy(b).to(cuda_device), acc)
    got = acc.cpu().numpy()
    assert got[0, 0] == 127 * 127 * K and got[1, 0] == -127 * 127 * K
    assert np.array_equal(got, oracle.gemm_s32(a, b))


# ---------------------------------------------------------------- linear (bf16, bias, SwiGLU)
def _linear_case(h3q, dev, M, K, N, with_bias, swiglu, outliers=4, factor=40.0):
    bits, to_dev = _u(dev)
    f = synth.column_factors(K, synth.outlier_columns(0, 4, K, outliers), factor)
    x_h = synth.activation_host(0, 1, np.arange(M), K, f)
    w_h = synth.weight_host(0, 2, np.arange(N), K)
    b_h = synth.bias_host(0, 3, N) if with_bias else None
    x = to_dev(x_h, dev)
    w = torch.from_numpy(w_h).to(dev)
    xq = torch.empty((M, K), dtype=torch.int8, device=dev)
    sx = torch.empty(M, dtype=torch.float32, device=dev)
    wq = torch.empty((N, K), dtype=torch.int8, device=dev)
    sw = torch.empty(N, dtype=torch.float32, device=dev)
    y = torch.empty((M, N // 2 if swiglu else N), dtype=torch.bfloat16, device=dev)
    h3q.h3q_rotate_quant(x, xq, sx)
    h3q.h3q_prepare_weight(w, wq, sw)
    h3q.h3q_linear_w8a8(xq, sx, wq, sw, y, bias=None if b_h is None else to_dev(b_h, dev),
                        epilogue=h3q.H3Q_EPI_SWIGLU if swiglu else h3q.H3Q_EPI_NONE)
    torch.cuda.synchronize()
    assert h3q.h3q_get_device_status() == h3q.H3Q_OK
    owq, osw = oracle.prepare_weight(w_h)
    oy, _ = oracle.linear(x_h, owq, osw, bias_bits=b_h, swiglu_epilogue=swiglu)
    return bits(y), oy, x_h, w_h, b_h


@pytest.mark.parametrize("M,K,N,with_bias", [(64, 512, 256, False), (64, 512, 256, True), (77, 768, 392, True),
                                             (1, 256, 8, True), (129, 5376, 520, True), (256, 1024, 768, False)])
def test_linear_bitexact(h3q, cuda_device, M, K, N, with_bias):
    got, want, x_h, w_h, b_h = _linear_case(h3q, cuda_device, M, K, N, with_bias, False)
    assert_bf16_close(got, want, "linear")
    assert np.array_equal(got, want), f"{(got != want).sum()} of {got.size} differ (within 1 ulp)"
    ref = synth.bf16_bits_to_fp32(x_h).astype(np.float64) @ w_h.astype(np.float64).T
    if b_h is not None:
        ref += synth.bf16_bits_to_fp32(b_h)[None, :]
    rel = np.linalg.norm(synth.bf16_bits_to_fp32(got) - ref) / np.linalg.norm(ref)
    assert rel <= 2e-2


@pytest.mark.parametrize("M,K,F,with_bias", [(64, 512, 128, False), (100, 512, 256, True), (129, 768, 384, True),
                                             (3, 256, 128, True)])
def test_linear_swiglu_bitexact(h3q, cuda_device, M, K, F, with_bias):
    got, want, _, _, _ = _linear_case(h3q, cuda_device, M, K, 2 * F, with_bias, True)
    assert got.shape == (M, F)
    assert_bf16_close(got, want, "swiglu")
    assert np.array_equal(got, want), f"{(got != want).sum()} of {got.size} differ (within 1 ulp)"


def test_swiglu_gate_values_past_fp32_exp_overflow(h3q, cuda_device):
    """Gate values over [-400, 400]: silu's e^-g runs past 2^64 (g < -44.4, the quotient
    taken with the power of two on the numerator), past fp32 overflow (g < -88.72, silu still
    a nonzero value near g e^g) and past silu's own underflow (g < -104). Bit-exact."""
    dev = cuda_device
    M, K, F = 128, 256, 128
    rng = np.random.default_rng(11)
    xq_h = rng.integers(-127, 128, size=(M, K), dtype=np.int8)
    wq_h = rng.integers(-127, 128, size=(2 * F, K), dtype=np.int8)
    acc = oracle.gemm_s32(xq_h, wq_h)
    sw_h = np.full(2 * F, 1.0 / float(np.abs(acc).max()), dtype=np.float32)
    sx_h = np.linspace(1.0, 400.0, M, dtype=np.float32)
    sw_h[F:] = sw_h[F:] * np.float32(1e30)         # up values large, so h = silu(g) u stays visible
    v, _ = oracle.epilogue(acc, sx_h, sw_h)
    g = v[:, :F]
    assert (g < -120).any() and ((g < -88.8) & (g > -103)).any() and ((g < -44.5) & (g > -88)).any()
    _, want = oracle.swiglu(v)
    y = torch.empty((M, F), dtype=torch.bfloat16, device=dev)
    h3q.h3q_linear_w8a8(torch.from_numpy(xq_h).to(dev), torch.from_numpy(sx_h).to(dev),
                        torch.from_numpy(wq_h).to(dev), torch.from_numpy(sw_h).to(dev), y,
                        epilogue=h3q.H3Q_EPI_SWIGLU)
    torch.cuda.synchronize()
    got = _u(dev)[0](y)
    deep = (g < -88.8) & (g > -100)
    assert np.all(synth.bf16_bits_to_fp32(want)[deep] != 0.0)
    assert np.array_equal(got, want), f"{(got != want).sum()} of {got.size} differ"


# ---------------------------------------------------------------- FFN
@pytest.mark.parametrize("M,K,F,with_bias", [(70, 512, 768, False), (64, 512, 256, True), (129, 256, 512, True)])
def test_ffn_bitexact(h3q, cuda_device, M, K, F, with_bias):
    bits, to_dev = _u(cuda_device)
    f = synth.column_factors(K, synth.outlier_columns(0, 4, K, 4), 50.0)
    x_h = synth.activation_host(0, 1, np.arange(M), K, f)
    wgu_h = synth.weight_host(0, 5, np.arange(2 * F), K)
    wd_h = synth.weight_host(0, 6, np.arange(K), F)
    bgu_h = synth.bias_host(0, 8, 2 * F) if with_bias else None
    bd_h = synth.bias_host(0, 10, K) if with_bias else None
    dev = cuda_device
    qgu = torch.empty((2 * F, K), dtype=torch.int8, device=dev)
    sgu = torch.empty(2 * F, dtype=torch.float32, device=dev)
    qd = torch.empty((K, F), dtype=torch.int8, device=dev)
    sd = torch.empty(K, dtype=torch.float32, device=dev)
    h3q.h3q_prepare_weight(torch.from_numpy(wgu_h).to(dev), qgu, sgu)
    h3q.h3q_prepare_weight(torch.from_numpy(wd_h).to(dev), qd, sd)
    ws = torch.empty(h3q.h3q_ffn_workspace_size(M, K, F), dtype=torch.uint8, device=dev)
    y = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    h3q.h3q_ffn(to_dev(x_h, dev), qgu, sgu, qd, sd, y, ws,
                b_gu=None if bgu_h is None else to_dev(bgu_h, dev),
                b_down=None if bd_h is None else to_dev(bd_h, dev))
    torch.cuda.synchronize()
    assert h3q.h3q_get_device_status() == h3q.H3Q_OK
    ogu, osgu = oracle.prepare_weight(wgu_h)
    od, osd = oracle.prepare_weight(wd_h)
    oy, oh, ohq, osh = oracle.ffn(x_h, ogu, osgu, od, osd, b_gu=bgu_h, b_down=bd_h)
    got = bits(y)
    assert_bf16_close(got, oy, "ffn")
    assert np.array_equal(got, oy), f"{(got != oy).sum()} of {got.size} differ (within 1 ulp)"


# ---------------------------------------------------------------- bounded waits
def test_stalled_wait_reports_timeout_and_context_survives(h3q, cuda_device):
    assert h3q.h3q_get_device_status() == h3q.H3Q_OK
    h3q.h3q_test_stalled_wait(20_000_000)  # 20 ms on a barrier nothing arrives on
    assert h3q.h3q_get_device_status() == h3q.H3Q_ERR_TIMEOUT
    assert h3q.h3q_get_device_status() == h3q.H3Q_OK  # cleared
    a = torch.ones((4, 256), dtype=torch.int8, device=cuda_device)
    b = torch.ones((8, 256), dtype=torch.int8, device=cuda_device)
    acc = torch.empty((4, 8), dtype=torch.int32, device=cuda_device)
    h3q.h3q_gemm_s32(a, b, acc)
    torch.cuda.synchronize()
    assert (acc.cpu().numpy() == 256).all()


def test_runs_on_a_side_stream(h3q, cuda_device):
    bits, to_dev = _u(cuda_device)
    s = torch.cuda.Stream()
    x_h = synth.activation_host(0, 1, np.arange(40), 512)
    with torch.cuda.stream(s):
        x = to_dev(x_h, cuda_device)
        xq = torch.empty((40, 512), dtype=torch.int8, device=cuda_device)
        sx = torch.empty(40, dtype=torch.float32, device=cuda_device)
        h3q.h3q_rotate_quant(x, xq, sx, stream=s)
    s.synchronize()
    oq, _ = oracle.rotate_quant_bf16(x_h)
    assert np.array_equal(xq.cpu().numpy(), oq)


def test_binding_rejects_wrong_shapes_and_layouts(h3q, cuda_device):
    """Operands of the wrong shape, a transposed or strided view, or on another device are
    refused by the binding before any pointer reaches the library."""
    dev = cuda_device
    M, K, N, F = 8, 256, 16, 512
    x = torch.zeros((M, K), dtype=torch.bfloat16, device=dev)
    xq = torch.zeros((M, K), dtype=torch.int8, device=dev)
    sx = torch.zeros(M, dtype=torch.float32, device=dev)
    wq = torch.zeros((N, K), dtype=torch.int8, device=dev)
    sw = torch.zeros(N, dtype=torch.float32, device=dev)
    with pytest.raises(ValueError, match="shape"):
        h3q.h3q_linear_w8a8(xq, sx, wq, sw, torch.zeros((M, N + 8), dtype=torch.bfloat16, device=dev))
    with pytest.raises(ValueError, match="shape"):
        h3q.h3q_linear_w8a8(xq, sx, wq, sw, torch.zeros((M, N), dtype=torch.bfloat16, device=dev),
                            epilogue=h3q.H3Q_EPI_SWIGLU)
    with pytest.raises(ValueError, match="contiguous"):
        h3q.h3q_rotate_quant(torch.zeros((K, M), dtype=torch.bfloat16, device=dev).t(), xq, sx)
    with pytest.raises(ValueError, match="CUDA tensor"):
        h3q.h3q_rotate_quant(x, xq, sx.cpu())
    w_gu = torch.zeros((2 * F, K), dtype=torch.int8, device=dev)
    s_gu = torch.zeros(2 * F, dtype=torch.float32, device=dev)
    w_down_t = torch.zeros((F, K), dtype=torch.int8, device=dev)     # [F, K] instead of [K, F]
    s_down = torch.zeros(K, dtype=torch.float32, device=dev)
    ws = torch.empty(h3q.h3q_ffn_workspace_size(M, K, F), dtype=torch.uint8, device=dev)
    y = torch.zeros((M, K), dtype=torch.bfloat16, device=dev)
    with pytest.raises(ValueError, match="w_down"):
        h3q.h3q_ffn(x, w_gu, s_gu, w_down_t, s_down, y, ws)
    with pytest.raises(ValueError, match="s_down"):
        h3q.h3q_ffn(x, w_gu, s_gu, torch.zeros((K, F), dtype=torch.int8, device=dev), s_down[:8], y, ws)
    assert h3q.h3q_get_device_status() == h3q.H3Q_OK
