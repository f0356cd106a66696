"""Full-size workloads on the GPU, in the launch configuration the benchmark
uses, checked against the CPU oracle on sampled rows and columns that the
oracle computes one by one (its inputs come from the seeded generator on the
host, never from the GPU). Integer outputs bit-exact; bf16 outputs within 1
bf16 ulp (expected: identical)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import synth  # noqa: E402

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def h3q(cuda_device):
    import w8a8_rotation_quantized_b200 as mod
    return mod


def _linear_fullsize(h3q, dev, M, K, N, seed=0, block=None, rows=24, cols=48):
    from _gpu_util import bits, dev_activation, dev_bias, dev_weight, sample_indices
    ids = synth.tensor_ids(block)
    rng = np.random.default_rng(M + N)
    f = synth.column_factors(K, synth.outlier_columns(seed, ids["outlier"], K, int(round(0.01 * K))), 50.0)
    x = dev_activation(seed, ids["x"], M, K, f, dev)
    w = dev_weight(seed, ids["w"], N, K, dev)
    bias = dev_bias(seed, ids["bias"], N, dev)
    xq = torch.empty((M, K), dtype=torch.int8, device=dev)
    sx = torch.empty(M, dtype=torch.float32, device=dev)
    wq = torch.empty((N, K), dtype=torch.int8, device=dev)
    sw = torch.empty(N, dtype=torch.float32, device=dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    h3q.h3q_prepare_weight(w, wq, sw)
    del w
    h3q.h3q_rotate_quant(x, xq, sx)
    h3q.h3q_linear_w8a8(xq, sx, wq, sw, y, bias=bias)
    torch.cuda.synchronize()
    assert h3q.h3q_get_device_status() == h3q.H3Q_OK

    ms = sample_indices(M, rows, rng, must=(127, 128, 129, M - 129, M - 128))
    ns = sample_indices(N, cols, rng, must=(255, 256, 257, N - 257, N - 8))
    x_h = synth.activation_host(seed, ids["x"], ms, K, f)
    w_h = synth.weight_host(seed, ids["w"], ns, K)
    b_h = synth.bias_host(seed, ids["bias"], N)[ns]
    owq, osw = oracle.prepare_weight(w_h)
    assert np.array_equal(wq[torch.from_numpy(ns).to(dev)].cpu().numpy(), owq)
    assert np.array_equal(sw.cpu().numpy()[ns].view(np.uint32), osw.view(np.uint32))
    oq, osx = oracle.rotate_quant_bf16(x_h)
    msd = torch.from_numpy(ms).to(dev)
    assert np.array_equal(xq[msd].cpu().numpy(), oq)
    assert np.array_equal(sx.cpu().numpy()[ms].view(np.uint32), osx.view(np.uint32))
    oy, _ = oracle.linear(x_h, owq, osw, bias_bits=b_h)
    got = bits(y[msd][:, torch.from_numpy(ns).to(dev)])
    assert np.array_equal(got, oy), f"{(got != oy).sum()} of {got.size} sampled outputs differ"
    # a property of every row: the largest code of a nonzero row is +-127
    assert int(xq.abs().amax(dim=1).min()) == 127


def test_qkv_projection_fullsize(h3q, cuda_device):
    _linear_fullsize(h3q, cuda_device, 4096, 5376, 16128)


def test_out_projection_fullsize(h3q, cuda_device):
    _linear_fullsize(h3q, cuda_device, 32768, 5376, 5376)


def test_ffn_fullsize(h3q, cuda_device):
    from _gpu_util import bits, dev_activation, dev_weight, sample_indices
    dev = cuda_device
    M, K, F = 16384, 5376, 14336
    ids = synth.tensor_ids()
    f = synth.column_factors(K, synth.outlier_columns(0, ids["outlier"], K, int(round(0.01 * K))), 50.0)
    x = dev_activation(0, ids["x"], M, K, f, dev)
    qgu = torch.empty((2 * F, K), dtype=torch.int8, device=dev)
    sgu = torch.empty(2 * F, dtype=torch.float32, device=dev)
    qd = torch.empty((K, F), dtype=torch.int8, device=dev)
    sd = torch.empty(K, dtype=torch.float32, device=dev)
    w = dev_weight(0, ids["w_gu"], 2 * F, K, dev)
    h3q.h3q_prepare_weight(w, qgu, sgu)
    w = dev_weight(0, ids["w_down"], K, F, dev)
    h3q.h3q_prepare_weight(w, qd, sd)
    del w
    nbytes = h3q.h3q_ffn_workspace_size(M, K, F)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    y = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    h3q.h3q_ffn(x, qgu, sgu, qd, sd, y, ws)
    torch.cuda.synchronize()
    assert h3q.h3q_get_device_status() == h3q.H3Q_OK

    rng = np.random.default_rng(3)
    ms = sample_indices(M, 6, rng, must=(128,))
    wgu_h = synth.weight_host(0, ids["w_gu"], np.arange(2 * F), K)
    ogu, osgu = oracle.prepare_weight(wgu_h)
    del wgu_h
    assert np.array_equal(sgu.cpu().numpy().view(np.uint32), osgu.view(np.uint32))
    wd_h = synth.weight_host(0, ids["w_down"], np.arange(K), F)
    od, osd = oracle.prepare_weight(wd_h)
    del wd_h
    assert np.array_equal(sd.cpu().numpy().view(np.uint32), osd.view(np.uint32))
    rows_check = torch.from_numpy(np.array([0, 77, 5000, 28671])).to(dev)
    assert np.array_equal(qgu[rows_check].cpu().numpy(), ogu[[0, 77, 5000, 28671]])
    x_h = synth.activation_host(0, ids["x"], ms, K, f)
    oy, oh, ohq, osh = oracle.ffn(x_h, ogu, osgu, od, osd)
    msd = torch.from_numpy(ms).to(dev)
    # the SwiGLU output and its codes, read back from the workspace (layout of h3q_ffn)
    off_sx = (M * K + 255) // 256 * 256
    off_h = (off_sx + M * 4 + 255) // 256 * 256
    off_hq = (off_h + M * F * 2 + 255) // 256 * 256
    off_sh = (off_hq + M * F + 255) // 256 * 256
    h = ws[off_h:off_h + M * F * 2].view(torch.bfloat16).view(M, F)
    hq = ws[off_hq:off_hq + M * F].view(torch.int8).view(M, F)
    sh = ws[off_sh:off_sh + M * 4].view(torch.float32)
    assert np.array_equal(bits(h[msd]), oh), "SwiGLU output"
    assert np.array_equal(hq[msd].cpu().numpy(), ohq), "re-rotated codes of h"
    assert np.array_equal(sh[msd].cpu().numpy().view(np.uint32), osh.view(np.uint32))
    got = bits(y[msd])
    assert np.array_equal(got, oy), f"{(got != oy).sum()} of {got.size} outputs differ"


@pytest.mark.parametrize("block", [0, 49])
def test_sweep_block_fullsize(h3q, cuda_device, block):
    """One block of a denoising step's linear sweep at 32768 tokens: QKV and out
    projections with bias and the FFN, each with its own per-block tensors."""
    from _gpu_util import bits, dev_activation, dev_bias, dev_weight, sample_indices
    dev = cuda_device
    M, K, F = 32768, 5376, 14336
    t = synth.tensor_ids(block)
    f = synth.column_factors(K, synth.outlier_columns(0, t["outlier"], K, int(round(0.01 * K))), 50.0)
    rng = np.random.default_rng(100 + block)
    ms = sample_indices(M, 4, rng, must=(M - 1,))
    xq = torch.empty((M, K), dtype=torch.int8, device=dev)
    sx = torch.empty(M, dtype=torch.float32, device=dev)
    for name, N in (("qkv", 16128), ("out", K)):
        x = dev_activation(0, t["x_" + name], M, K, f, dev)
        w = dev_weight(0, t["w_" + name], N, K, dev)
        wq = torch.empty((N, K), dtype=torch.int8, device=dev)
        sw = torch.empty(N, dtype=torch.float32, device=dev)
        h3q.h3q_prepare_weight(w, wq, sw)
        del w
        bias = dev_bias(0, t["b_" + name], N, dev)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        h3q.h3q_rotate_quant(x, xq, sx)
        h3q.h3q_linear_w8a8(xq, sx, wq, sw, y, bias=bias)
        torch.cuda.synchronize()
        ns = sample_indices(N, 32, rng)
        owq, osw = oracle.prepare_weight(synth.weight_host(0, t["w_" + name], ns, K))
        oy, _ = oracle.linear(synth.activation_host(0, t["x_" + name], ms, K, f), owq, osw,
                              bias_bits=synth.bias_host(0, t["b_" + name], N)[ns])
        got = bits(y[torch.from_numpy(ms).to(dev)][:, torch.from_numpy(ns).to(dev)])
        assert np.array_equal(got, oy), f"block {block} {name}: {(got != oy).sum()} of {got.size} differ"
        del x, wq, y
    x = dev_activation(0, t["x_ffn"], M, K, f, dev)
    qgu = torch.empty((2 * F, K), dtype=torch.int8, device=dev)
    sgu = torch.empty(2 * F, dtype=torch.float32, device=dev)
    qd = torch.empty((K, F), dtype=torch.int8, device=dev)
    sd = torch.empty(K, dtype=torch.float32, device=dev)
    h3q.h3q_prepare_weight(dev_weight(0, t["w_gu"], 2 * F, K, dev), qgu, sgu)
    h3q.h3q_prepare_weight(dev_weight(0, t["w_down"], K, F, dev), qd, sd)
    ws = torch.empty(h3q.h3q_ffn_workspace_size(M, K, F), dtype=torch.uint8, device=dev)
    y = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    h3q.h3q_ffn(x, qgu, sgu, qd, sd, y, ws)
    torch.cuda.synchronize()
    assert h3q.h3q_get_device_status() == h3q.H3Q_OK
    ogu, osgu = oracle.prepare_weight(synth.weight_host(0, t["w_gu"], np.arange(2 * F), K))
    od, osd = oracle.prepare_weight(synth.weight_host(0, t["w_down"], np.arange(K), F))
    oy, _, _, _ = oracle.ffn(synth.activation_host(0, t["x_ffn"], ms, K, f), ogu, osgu, od, osd)
    got = bits(y[torch.from_numpy(ms).to(dev)])
    assert np.array_equal(got, oy), f"block {block} ffn: {(got != oy).sum()} of {got.size} differ"
