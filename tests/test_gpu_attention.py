"""int8 attention on the GPU against the oracle.

* The input pass (int8 codes of Q per token and of K per block of 128 keys, their
  scales, V^T per head) is bit-exact.
* The attention output is compared with the oracle's float64 attention of the
  same int8 codes within a bound from the arithmetic: P is rounded to bf16
  (relative 2^-9 per weight, the row sum uses the same rounded weights, so the
  output moves by at most 2 * 2^-9 * max|V| from the reweighting), 2^x is the
  hardware approximation (relative ~2^-22), sums are fp32 (S * 2^-24), and the
  output is rounded to bf16 (2^-9 relative): |o - ref| <= 2^-7 max|V_h| +
  2^-8 |ref|.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import synth  # noqa: E402

pytestmark = pytest.mark.gpu
D = 128


def _qkv(S, H, seed, dev, growing=False, zero_q_rows=()):
    """One [S, 3 H D] bf16 matrix (a QKV projection output); q, k, v column slices."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((S, 3 * H * D), dtype=np.float32)
    x[:, :H * D] *= 1.5
    for i in zero_q_rows:  # a query row of zeros: its scale is 0, all its scores 0, uniform weights
        x[i, :D] = 0.0
    if growing:  # keys grow along the sequence: the running maximum keeps moving
        x[:, H * D:2 * H * D] *= np.linspace(0.2, 4.0, S, dtype=np.float32)[:, None]
    t = torch.from_numpy(x).to(dev).bfloat16()
    bits = t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t, bits


def _run(h3q, t, S, H):
    q, k, v = t[:, :H * D], t[:, H * D:2 * H * D], t[:, 2 * H * D:]
    out = torch.full((S, H * D), float("nan"), dtype=torch.bfloat16, device=t.device)
    ws = torch.empty(h3q.h3q_attention_workspace_size(S, H), dtype=torch.uint8, device=t.device)
    h3q.h3q_attention_int8(q, k, v, H, out, ws)
    torch.cuda.synchronize()
    assert h3q.h3q_get_device_status() == h3q.H3Q_OK
    return out


def _check(out, bits, S, H, rows=None):
    q, k, v = bits[:, :H * D], bits[:, H * D:2 * H * D], bits[:, 2 * H * D:]
    ref, *_ = oracle.attention_int8(q, k, v, H, rows=rows)
    got = out.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        got = got[rows]
    vmax = np.abs(synth.bf16_bits_to_fp32(v).astype(np.float64)).reshape(S, H, D).max(axis=(0, 2))
    bound = 2.0 ** -7 * np.repeat(vmax, D)[None, :] + 2.0 ** -8 * np.abs(ref)
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got))
    assert np.all(err <= bound), f"max err/bound {np.max(err / bound):.3g}"
    return float(np.max(err / bound))


def test_prep_is_bit_exact(cuda_device):
    import w8a8_rotation_quantized_b200 as h3q
    S, H = 200, 3
    t, bits = _qkv(S, H, 0, cuda_device)
    q, k, v = t[:, :H * D], t[:, H * D:2 * H * D], t[:, 2 * H * D:]
    qq = torch.empty((H, S, D), dtype=torch.int8, device=cuda_device)
    kq = torch.empty_like(qq)
    qs = torch.empty((H, S), dtype=torch.float32, device=cuda_device)
    ks = torch.empty((H, (S + 127) // 128), dtype=torch.float32, device=cuda_device)
    vt = torch.empty((H * D, S), dtype=torch.bfloat16, device=cuda_device)
    h3q.h3q_attention_prep(q, k, v, H, qq, qs, kq, ks, vt)
    torch.cuda.synchronize()
    _, rq, rqs, rk, rks = oracle.attention_int8(bits[:, :H * D], bits[:, H * D:2 * H * D], bits[:, 2 * H * D:], H,
                                                 rows=np.arange(1))
    assert np.array_equal(qq.cpu().numpy(), rq) and np.array_equal(kq.cpu().numpy(), rk)
    assert np.array_equal(qs.cpu().numpy(), rqs) and np.array_equal(ks.cpu().numpy(), rks)
    want_vt = bits[:, 2 * H * D:].reshape(S, H, D).transpose(1, 2, 0).reshape(H * D, S)
    assert np.array_equal(vt.view(torch.int16).cpu().numpy().view(np.uint16), want_vt)


@pytest.mark.parametrize("S,H,seed", [(128, 1, 1), (264, 2, 2), (8, 1, 3), (1024, 2, 4)])
def test_attention_matches_oracle(cuda_device, S, H, seed):
    import w8a8_rotation_quantized_b200 as h3q
    t, bits = _qkv(S, H, seed, cuda_device)
    out = _run(h3q, t, S, H)
    _check(out, bits, S, H)


def test_zero_query_row_with_ragged_last_block(cuda_device):
    import w8a8_rotation_quantized_b200 as h3q
    S, H = 200, 1
    t, bits = _qkv(S, H, 7, cuda_device, zero_q_rows=(5, 150))
    out = _run(h3q, t, S, H)
    _check(out, bits, S, H)
    mean_v = synth.bf16_bits_to_fp32(bits[:, 2 * D:3 * D]).astype(np.float64).mean(axis=0)
    assert np.abs(out[5].float().cpu().numpy() - mean_v).max() < 2e-2


def test_attention_with_moving_maximum(cuda_device):
    """Keys grow along the sequence, so every row's maximum keeps rising and the
    output accumulator is rescaled in tensor memory."""
    import w8a8_rotation_quantized_b200 as h3q
    S, H = 1536, 1
    t, bits = _qkv(S, H, 5, cuda_device, growing=True)
    out = _run(h3q, t, S, H)
    _check(out, bits, S, H)


def test_attention_full_size_sampled_rows(cuda_device):
    """16384 tokens, 42 heads (hidden 5376): 6 sampled query rows of every head
    against the oracle."""
    import w8a8_rotation_quantized_b200 as h3q
    from _gpu_util import sample_indices
    S, H = 16384, 42
    t, bits = _qkv(S, H, 6, cuda_device)
    out = _run(h3q, t, S, H)
    rows = sample_indices(S, 6, np.random.default_rng(9), must=(127, 128))
    _check(out, bits, S, H, rows=rows)


@pytest.mark.parametrize("S,H,seed", [(392, 3, 11), (136, 2, 12)])
def test_attention_strided_views_leave_padding_untouched(cuda_device, S, H, seed):
    """q, k, v are column slices of a matrix with padding columns past the three
    blocks (row stride 3 H D + 64), the output a column slice of a wider NaN-filled
    matrix: every written value is within the bound and the padding is untouched;
    S leaves a ragged last key block of 8 keys (136) or of 8 past three blocks (392)."""
    import w8a8_rotation_quantized_b200 as h3q
    t, bits = _qkv(S, H, seed, cuda_device)
    pad = 64
    wide = torch.zeros((S, 3 * H * D + pad), dtype=torch.bfloat16, device=cuda_device)
    wide[:, :3 * H * D] = t
    q, k, v = wide[:, :H * D], wide[:, H * D:2 * H * D], wide[:, 2 * H * D:3 * H * D]
    big = torch.full((S, H * D + 3 * D), float("nan"), dtype=torch.bfloat16, device=cuda_device)
    out = big[:, D:D + H * D]  # columns before and after the written block stay NaN
    ws = torch.empty(h3q.h3q_attention_workspace_size(S, H), dtype=torch.uint8, device=cuda_device)
    h3q.h3q_attention_int8(q, k, v, H, out, ws)
    torch.cuda.synchronize()
    assert h3q.h3q_get_device_status() == h3q.H3Q_OK
    assert torch.isnan(big[:, :D]).all() and torch.isnan(big[:, D + H * D:]).all()
    _check(out.contiguous(), bits, S, H)
