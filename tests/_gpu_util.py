"""Helpers shared by the GPU tests: moving bf16 bit patterns between numpy and
torch, and building seeded device tensors with the CUDA generator."""
import numpy as np
import torch

import synth


def to_dev_bf16(a: np.ndarray, dev) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)


def bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def dev_activation(seed, tid, M, K, factors, dev):
    x = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    f = None if factors is None else torch.from_numpy(factors).to(dev)
    synth.fill_device(seed, tid, 0, M, K, x.data_ptr(), torch.cuda.current_stream().cuda_stream,
                      factors_ptr=None if f is None else f.data_ptr(), bf16=True)
    torch.cuda.current_stream().synchronize()
    return x


def dev_weight(seed, tid, N, K, dev):
    w = torch.empty((N, K), dtype=torch.float32, device=dev)
    synth.fill_device(seed, tid, 0, N, K, w.data_ptr(), torch.cuda.current_stream().cuda_stream,
                      scale=float(synth.SIGMA_W), bf16=False)
    torch.cuda.current_stream().synchronize()
    return w


def dev_bias(seed, tid, N, dev):
    return to_dev_bf16(synth.bias_host(seed, tid, N), dev)


def sample_indices(n, k, rng, must=()):
    """k distinct indices in [0, n) including the first, the last and `must`."""
    picks = set(i for i in must if 0 <= i < n) | {0, n - 1}
    while len(picks) < min(k, n):
        picks.add(int(rng.integers(0, n)))
    return np.array(sorted(picks), dtype=np.int64)
