"""LoRA merge into rotated int8 weights on the GPU, element by element against
the oracle: codes bit-exact, scales bit-exact.

The merge (h3-rs README, "Speed", "What makes it fast": a LoRA is folded into
the int8 weights once, at model load, by dequantizing, adding and requantizing) rotates A
along K, forms alpha * B A_rot in fp32 in a fixed order and requantizes each
row; both sides take every rounding in the same order, so nothing differs.
Cases cover ragged row blocks, every cluster width the launch picks (one CTA
per row block at K = 512, four at K = 5376, five at K = 14336 with a short last
slice, six at K = 16384), rank 1 and the maximum rank, alpha = 0, rows that are
zero before and after, and in-place use on the ffn workload's full-size
gate/up weight (sampled rows).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import synth  # noqa: E402

pytestmark = pytest.mark.gpu


def _factors(seed, N, K, r):
    a = synth.weight_host(seed, synth.TID_LORA_A, np.arange(r), K)
    b = synth.weight_host(seed, synth.TID_LORA_B, np.arange(N), r)
    return a, b


def _merge_gpu(h3q, dev, wq, sw, a, b, alpha):
    tq = torch.from_numpy(np.ascontiguousarray(wq)).to(dev)
    ts = torch.from_numpy(np.ascontiguousarray(sw)).to(dev)
    ta = torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    tb = torch.from_numpy(np.ascontiguousarray(b)).to(dev)
    ws = torch.empty(h3q.h3q_lora_workspace_size(a.shape[0], wq.shape[1]), dtype=torch.uint8, device=dev)
    h3q.h3q_lora_merge(tq, ts, ta, tb, alpha, ws)
    torch.cuda.synchronize()
    assert h3q.h3q_get_device_status() == h3q.H3Q_OK
    return tq.cpu().numpy(), ts.cpu().numpy()


@pytest.mark.parametrize("N,K,r,alpha,seed", [
    (100, 512, 8, 0.75, 0),        # R = 16 with a ragged last row block, one CTA per block
    (69, 5376, 64, 1.0, 1),        # four CTAs per row block
    (37, 14336, 16, 0.5, 2),       # R = 8, five CTAs, short last slice
    (9, 16384, 512, 0.125, 3),     # widest K, maximum rank
    (3, 256, 1, -2.0, 4),          # one group, rank 1, negative alpha
])
def test_lora_merge_matches_oracle(cuda_device, N, K, r, alpha, seed):
    import w8a8_rotation_quantized_b200 as h3q
    w = synth.weight_host(seed, synth.TID_W, np.arange(N), K)
    wq, sw = oracle.prepare_weight(w)
    a, b = _factors(seed, N, K, r)
    q_ref, s_ref = oracle.lora_merge(wq, sw, a, b, alpha)
    q_gpu, s_gpu = _merge_gpu(h3q, cuda_device, wq, sw, a, b, alpha)
    assert np.array_equal(s_gpu.view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(q_gpu, q_ref), f"{(q_gpu != q_ref).sum()} codes differ"


def test_lora_merge_degenerate_rows(cuda_device):
    import w8a8_rotation_quantized_b200 as h3q
    N, K, r = 20, 768, 4
    w = synth.weight_host(5, synth.TID_W, np.arange(N), K)
    w[3] = 0.0                    # zero weight row, zero LoRA row -> stays zero, scale 0
    wq, sw = oracle.prepare_weight(w)
    a, b = _factors(5, N, K, r)
    b[3] = 0.0
    b[7] = 0.0                    # no delta: the row's codes and scale stay as they were
    for alpha in (0.0, 3.0):
        q_ref, s_ref = oracle.lora_merge(wq, sw, a, b, alpha)
        q_gpu, s_gpu = _merge_gpu(h3q, cuda_device, wq, sw, a, b, alpha)
        assert np.array_equal(s_gpu.view(np.uint32), s_ref.view(np.uint32))
        assert np.array_equal(q_gpu, q_ref)
        assert s_gpu[3] == 0.0 and not q_gpu[3].any()
        assert np.array_equal(q_gpu[7], wq[7]) and s_gpu[7] == sw[7]
    assert np.array_equal(q_gpu, q_ref)


@pytest.mark.slow
def test_lora_merge_full_size_gate_up_sampled(cuda_device):
    """The lora workload's gate/up weight [28672, 5376], rank 64, merged in place
    on the device; 48 sampled rows (first, last, both sides of the gate/up
    boundary) compared with the oracle run on those rows alone (rows are
    independent)."""
    import w8a8_rotation_quantized_b200 as h3q
    from _gpu_util import dev_weight, sample_indices
    wl = synth.WORKLOADS["lora"]
    N, K, r, alpha = 2 * wl.F, wl.K, wl.rank, wl.alpha
    dev = cuda_device
    w = dev_weight(wl.seed, synth.TID_WGU, N, K, dev)
    wq = torch.empty((N, K), dtype=torch.int8, device=dev)
    sw = torch.empty(N, dtype=torch.float32, device=dev)
    h3q.h3q_prepare_weight(w, wq, sw)
    del w
    a = torch.from_numpy(synth.weight_host(wl.seed, synth.TID_LORA_A, np.arange(r), K)).to(dev)
    b = torch.empty((N, r), dtype=torch.float32, device=dev)
    synth.fill_device(wl.seed, synth.TID_LORA_B, 0, N, r, b.data_ptr(), torch.cuda.current_stream().cuda_stream,
                      scale=float(synth.SIGMA_W), bf16=False)
    rows = sample_indices(N, 48, np.random.default_rng(7), must=(wl.F - 1, wl.F))
    wq0 = wq[torch.from_numpy(rows).to(dev)].cpu().numpy()
    sw0 = sw[torch.from_numpy(rows).to(dev)].cpu().numpy()
    ws = torch.empty(h3q.h3q_lora_workspace_size(r, K), dtype=torch.uint8, device=dev)
    h3q.h3q_lora_merge(wq, sw, a, b, alpha, ws)
    torch.cuda.synchronize()
    assert h3q.h3q_get_device_status() == h3q.H3Q_OK
    q_ref, s_ref = oracle.lora_merge(wq0, sw0, a.cpu().numpy(), b[torch.from_numpy(rows).to(dev)].cpu().numpy(),
                                     alpha)
    idx = torch.from_numpy(rows).to(dev)
    assert np.array_equal(sw[idx].cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(wq[idx].cpu().numpy(), q_ref)
