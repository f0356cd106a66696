"""The seeded input generator: determinism, distribution, and agreement of its
numpy, C and CUDA implementations (the CUDA one under the gpu marker)."""
import numpy as np
import pytest

import synth


def test_splitmix64_reference_values():
    # splitmix64 seeded with 0: the first outputs published with the algorithm
    # (Vigna's reference implementation, splitmix64.c, state starting at 0).
    got = [int(synth.word(np.uint64(0), np.uint64(c))) for c in range(3)]
    assert got == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_normal_moments_and_exactness():
    z = synth.normal_fp32(0, 1, np.arange(2_000_000, dtype=np.uint64))
    assert abs(z.mean()) < 3e-3 and abs(z.var() - 1.0) < 5e-3
    # every draw is an integer multiple of 2^-17
    assert np.all((z * np.float32(2 ** 17)) == np.round(z * np.float32(2 ** 17)))
    assert np.array_equal(z, synth.normal_fp32(0, 1, np.arange(2_000_000, dtype=np.uint64)))
    assert not np.array_equal(z[:1000], synth.normal_fp32(0, 2, np.arange(1000, dtype=np.uint64)))


def test_outlier_columns():
    cols = synth.outlier_columns(0, 4, 5376, 54)
    assert cols.size == 54 and np.unique(cols).size == 54 and cols.min() >= 0 and cols.max() < 5376
    assert synth.WORKLOADS["qkv"].n_outliers == 54
    f = synth.WORKLOADS["tiny"].factors()
    assert (f == 40.0).sum() == 4 and (f == 1.0).sum() == 508


@pytest.mark.parametrize("bf16", [True, False])
def test_c_matches_numpy(bf16):
    rows = np.array([0, 3, 64, 1000, 4095])
    if bf16:
        f = synth.WORKLOADS["qkv"].factors()
        a = synth.activation_bf16(0, 11, rows, 5376, f)
        b = synth.activation_host(0, 11, rows, 5376, f)
        assert np.array_equal(a, b)
    else:
        a = synth.weight_fp32(0, 7, rows, 5376)
        b = synth.weight_host(0, 7, rows, 5376)
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    assert np.array_equal(synth.bias_bf16(0, 8, 16128), synth.bias_host(0, 8, 16128))


@pytest.mark.gpu
def test_cuda_matches_c(cuda_device):
    import torch
    synth.build()
    wl = synth.WORKLOADS["qkv"]
    f = wl.factors()
    fd = torch.from_numpy(f).to(cuda_device)
    x = torch.empty((300, wl.K), dtype=torch.bfloat16, device=cuda_device)
    synth.fill_device(0, 11, 100, 300, wl.K, x.data_ptr(), factors_ptr=fd.data_ptr(), bf16=True)
    w = torch.empty((257, wl.K), dtype=torch.float32, device=cuda_device)
    synth.fill_device(0, 7, 0, 257, wl.K, w.data_ptr(), scale=float(synth.SIGMA_W), bf16=False)
    torch.cuda.synchronize()
    xh = x.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(xh, synth.activation_host(0, 11, np.arange(100, 400), wl.K, f))
    wh = w.cpu().numpy()
    assert np.array_equal(wh.view(np.uint32), synth.weight_host(0, 7, np.arange(257), wl.K).view(np.uint32))
