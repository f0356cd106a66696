"""NVFP4 projections on the GPU against the oracle.

* Quantizer: codes, block scales (read back through the documented atom
  layout) and the tensor scale bit-exact, for bf16 activations with outlier
  channels, fp32 weights, ragged row counts and all-zero blocks.
* GEMM: the tensor cores accumulate the K/16 exact block terms in fp32 in their
  own order, so the raw accumulators are compared with the oracle's float64
  sum within the fp32 accumulation bound (K/16) * 2^-22 * sum|terms| (four
  times the worst case of a sequential fp32 sum).
* Epilogue: given the GPU's own accumulators, the bf16 (bias) and SwiGLU
  outputs are bit-exact against the oracle's epilogue.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import synth  # noqa: E402

pytestmark = pytest.mark.gpu


def _sf_offset(r, j, K):
    return ((r // 128) * (K // 64) + j // 4) * 512 + 16 * (r % 32) + 4 * ((r % 128) // 32) + (j % 4)


def _sf_plain(sf_swz, rows, K):
    r = np.arange(rows)[:, None]
    j = np.arange(K // 16)[None, :]
    return sf_swz[_sf_offset(r, j, K)]


def _quantize_gpu(h3q, x):
    rows, K = x.shape
    codes = torch.empty((rows, K // 2), dtype=torch.uint8, device=x.device)
    sf = torch.full((h3q.h3q_nvfp4_sf_bytes(rows, K),), 0xAB, dtype=torch.uint8, device=x.device)
    scale = torch.empty(2, dtype=torch.float32, device=x.device)
    h3q.h3q_nvfp4_quantize(x, codes, sf, scale)
    torch.cuda.synchronize()
    return codes, sf, scale


def _act(seed, M, K, dev):
    f = synth.column_factors(K, synth.outlier_columns(seed, synth.TID_OUTLIER, K, max(1, K // 100)), 50.0)
    bits = synth.activation_host(seed, synth.TID_X, np.arange(M), K, f)
    return bits, torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)


@pytest.mark.parametrize("M,K,seed", [(300, 512, 0), (128, 5376, 1), (1, 256, 2)])
def test_quantize_bf16_matches_oracle(cuda_device, M, K, seed):
    import w8a8_rotation_quantized_b200 as h3q
    bits, x = _act(seed, M, K, cuda_device)
    if M > 2:
        bits[2, 32:48] = 0  # an all-zero block
        x[2, 32:48] = 0
    codes, sf, scale = _quantize_gpu(h3q, x)
    c_ref, sf_ref, e_ref = oracle.nvfp4_quantize(bits)
    sc = scale.cpu().numpy()
    assert sc[1] == np.float32(e_ref)
    assert sc[0] == np.abs(synth.bf16_bits_to_fp32(bits)).max()
    sf_h = sf.cpu().numpy()
    assert np.array_equal(_sf_plain(sf_h, M, K), sf_ref)
    pad = np.arange(M, (M + 127) // 128 * 128)
    assert not _sf_plain(sf_h, (M + 127) // 128 * 128, K)[pad].any()
    c_gpu = codes.cpu().numpy()
    assert np.array_equal(c_gpu, c_ref), f"{(c_gpu != c_ref).sum()} code bytes differ"


def test_quantize_fp32_weights_and_zero_tensor(cuda_device):
    import w8a8_rotation_quantized_b200 as h3q
    w = synth.weight_host(3, synth.TID_W, np.arange(384), 768)
    codes, sf, scale = _quantize_gpu(h3q, torch.from_numpy(w).to(cuda_device))
    c_ref, sf_ref, e_ref = oracle.nvfp4_quantize(w)
    assert scale.cpu().numpy()[1] == np.float32(e_ref)
    assert np.array_equal(_sf_plain(sf.cpu().numpy(), 384, 768), sf_ref)
    assert np.array_equal(codes.cpu().numpy(), c_ref)
    codes, sf, scale = _quantize_gpu(h3q, torch.zeros((64, 256), dtype=torch.bfloat16, device=cuda_device))
    assert scale.cpu().numpy()[1] == 1.0 and not codes.any().item() and not sf.any().item()


def _setup(h3q, dev, M, K, N, seed):
    bits, x = _act(seed, M, K, dev)
    w = synth.weight_host(seed, synth.TID_W, np.arange(N), K)
    xc, xsf, xs = _quantize_gpu(h3q, x)
    wc, wsf, ws = _quantize_gpu(h3q, torch.from_numpy(w).to(dev))
    ca, sfa, ea = oracle.nvfp4_quantize(bits)
    cw, sfw, ew = oracle.nvfp4_quantize(w)
    return (xc, xsf, xs, wc, wsf, ws), (ca, sfa, ea, cw, sfw, ew)


def _acc_gpu(h3q, g):
    xc, xsf, xs, wc, wsf, ws = g
    acc = torch.empty((xc.shape[0], wc.shape[0]), dtype=torch.float32, device=xc.device)
    h3q.h3q_gemm_nvfp4_f32(xc, xsf, wc, wsf, acc)
    torch.cuda.synchronize()
    assert h3q.h3q_get_device_status() == h3q.H3Q_OK
    return acc


def _check_acc(acc_gpu, acc_ref, mag, K):
    bound = (K / 16) * 2.0 ** -22 * mag + 2.0 ** -120
    err = np.abs(acc_gpu.astype(np.float64) - acc_ref)
    assert np.all(err <= bound), f"max err / bound {np.max(err / bound):.3g}"
    return float(np.max(err / bound))


@pytest.mark.parametrize("M,K,N,seed", [(300, 768, 512, 4), (256, 256, 256, 5), (40, 5376, 768, 6)])
def test_gemm_accumulators_within_fp32_bound(cuda_device, M, K, N, seed):
    import w8a8_rotation_quantized_b200 as h3q
    g, o = _setup(h3q, cuda_device, M, K, N, seed)
    acc = _acc_gpu(h3q, g).cpu().numpy()
    _, acc_ref, mag = oracle.nvfp4_linear(*o)
    _check_acc(acc, acc_ref, mag, K)


@pytest.mark.parametrize("swiglu", [False, True])
def test_linear_epilogue_bit_exact_given_accumulators(cuda_device, swiglu):
    import w8a8_rotation_quantized_b200 as h3q
    M, K, N = 300, 512, 512
    g, o = _setup(h3q, cuda_device, M, K, N, 7)
    xc, xsf, xs, wc, wsf, ws = g
    bias_bits = synth.bias_host(7, synth.TID_BIAS, N)
    bias = torch.from_numpy(bias_bits.view(np.int16)).to(cuda_device).view(torch.bfloat16)
    y = torch.empty((M, N // 2 if swiglu else N), dtype=torch.bfloat16, device=cuda_device)
    h3q.h3q_linear_nvfp4(xc, xsf, xs, wc, wsf, ws, y, bias=bias,
                         epilogue=h3q.H3Q_EPI_SWIGLU if swiglu else h3q.H3Q_EPI_NONE)
    acc = _acc_gpu(h3q, g).cpu().numpy()
    sx, sw = xs.cpu().numpy()[1], ws.cpu().numpy()[1]
    want = oracle.nvfp4_epilogue(acc, sx, sw, bias_bits=bias_bits, swiglu_epilogue=swiglu)
    got = y.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, want), f"{(got != want).sum()} of {got.size} outputs differ"
    # and the layer as a whole is the oracle's layer up to the accumulation order
    y_ref, _, _ = oracle.nvfp4_linear(*o, bias_bits=bias_bits, swiglu_epilogue=swiglu)
    a = synth.bf16_bits_to_fp32(got).astype(np.float64)
    b = synth.bf16_bits_to_fp32(y_ref).astype(np.float64)
    assert np.abs(a - b).max() <= 2.0 ** -6 * np.abs(b).max()


def test_qkv_full_size_sampled_rows(cuda_device):
    """QKV shape (4096 x 5376 -> 16128), all rows on the GPU; 12 sampled rows of
    the accumulators against the oracle (rows are independent; the activation
    tensor scale comes from the whole tensor)."""
    import w8a8_rotation_quantized_b200 as h3q
    from _gpu_util import dev_activation, dev_weight, sample_indices
    M, K, N = 4096, 5376, 16128
    dev = cuda_device
    ids = synth.tensor_ids()
    f = synth.column_factors(K, synth.outlier_columns(0, ids["outlier"], K, 54), 50.0)
    x = dev_activation(0, ids["x_qkv"], M, K, f, dev)
    w = dev_weight(0, ids["w_qkv"], N, K, dev)
    g = _quantize_gpu(h3q, x) + _quantize_gpu(h3q, w)
    acc = _acc_gpu(h3q, g)
    rows = sample_indices(M, 12, np.random.default_rng(8), must=(255, 256))
    xb = x.view(torch.int16).cpu().numpy().view(np.uint16)
    e_a = oracle.nvfp4_encode_scale(xb)
    assert g[2].cpu().numpy()[1] == np.float32(e_a)
    ca, sfa, _ = oracle.nvfp4_quantize(xb[rows], s_enc=e_a)
    cw, sfw, ew = oracle.nvfp4_quantize(w.cpu().numpy())
    assert np.array_equal(g[0].cpu().numpy()[rows], ca)
    _, acc_ref, mag = oracle.nvfp4_linear(ca, sfa, e_a, cw, sfw, ew)
    _check_acc(acc.cpu().numpy()[rows], acc_ref, mag, K)
