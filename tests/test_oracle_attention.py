"""Pins of the oracle's int8 attention (int8 Q.K^T, softmax, P.V per head):
closed forms, torch's float64 scaled-dot-product attention on the dequantized
inputs, the quantizer it shares with the weight path, and its accuracy against
unquantized attention."""
import numpy as np
import torch

import oracle
import synth

D = 128


def _bits(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).bfloat16().view(torch.int16).numpy().view(np.uint16)


def _vals(b):
    return synth.bf16_bits_to_fp32(b).astype(np.float64)


def _inputs(S, H, seed, outlier=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((S, H * D)) * 1.5
    k = rng.standard_normal((S, H * D))
    if outlier:
        k[:, 5] *= 20.0  # an outlier channel
    v = rng.standard_normal((S, H * D))
    return _bits(q), _bits(k), _bits(v)


def test_codes_q_per_token_k_per_block_of_128_keys():
    """Q rows use the weight-row quantizer per token; K uses it per block of 128 keys
    of a head (the block read as one vector), the last block taking the keys left."""
    S, H = 300, 2  # key blocks of 128, 128 and 44
    q, k, v = _inputs(S, H, 0)
    _, qq, qs, kq, ks = oracle.attention_int8(q, k, v, H)
    assert ks.shape == (H, 3)
    for h in range(H):
        cq, sq = oracle.quantize_rows(_vals(q[:, h * D:(h + 1) * D]).astype(np.float32))
        assert np.array_equal(qq[h], cq) and np.array_equal(qs[h], sq)
        kh = _vals(k[:, h * D:(h + 1) * D]).astype(np.float32)
        for b, (j0, j1) in enumerate(((0, 128), (128, 256), (256, 300))):
            ck, sk = oracle.quantize_rows(kh[j0:j1].reshape(1, -1))
            assert np.array_equal(kq[h, j0:j1], ck.reshape(j1 - j0, D)) and ks[h, b] == sk[0]


def test_key_block_scale_covers_its_own_block_only():
    """Doubling the keys of block 1 (exact in bf16) doubles its scale and keeps its
    codes; block 0 is untouched; one large key coarsens only its own block."""
    S = 256
    q, k, v = _inputs(S, 1, 5, outlier=False)
    _, _, _, kq, ks = oracle.attention_int8(q, k, v, 1)
    k2 = k.copy()
    k2[128:] = _bits(_vals(k[128:]) * 2.0)
    _, _, _, kq2, ks2 = oracle.attention_int8(q, k2, v, 1)
    assert ks2[0, 0] == ks[0, 0] and ks2[0, 1] == 2 * ks[0, 1]
    assert np.array_equal(kq2, kq)
    k3 = k.copy()
    k3[200, 3] = _bits(np.array([[1000.0]]))[0, 0]
    _, _, _, kq3, ks3 = oracle.attention_int8(q, k3, v, 1)
    assert ks3[0, 0] == ks[0, 0] and np.array_equal(kq3[0, :128], kq[0, :128])
    assert ks3[0, 1] > 100 * ks[0, 1] and kq3[0, 200, 3] == 127


def test_identical_keys_give_the_mean_of_v():
    q, k, v = _inputs(33, 1, 1)
    k[:] = k[0]
    o, *_ = oracle.attention_int8(q, k, v, 1)
    assert np.allclose(o, _vals(v).mean(axis=0, keepdims=True), rtol=0, atol=1e-12)


def test_matches_torch_sdpa_on_dequantized_inputs():
    S, H = 200, 3
    q, k, v = _inputs(S, H, 2)
    o, qq, qs, kq, ks = oracle.attention_int8(q, k, v, H)
    qd = torch.from_numpy(qq.astype(np.float64) * qs[:, :, None].astype(np.float64))
    ks_key = np.repeat(ks.astype(np.float64), 128, axis=1)[:, :S]  # each key's block scale
    kd = torch.from_numpy(kq.astype(np.float64) * ks_key[:, :, None])
    vd = torch.from_numpy(_vals(v).reshape(S, H, D).transpose(1, 0, 2).copy())
    ref = torch.nn.functional.scaled_dot_product_attention(qd[None], kd[None], vd[None])[0]
    ref = ref.numpy().transpose(1, 0, 2).reshape(S, H * D)
    assert np.abs(o - ref).max() <= 1e-10


def test_dominant_key_selects_its_value_and_accuracy():
    S = 64
    q, k, v = _inputs(S, 1, 3)
    qv = _vals(q)
    k[7] = _bits(qv[0:1] * 8.0)[0]  # key 7 strongly aligned with query 0
    o, *_ = oracle.attention_int8(q, k, v, 1)
    assert np.abs(o[0] - _vals(v)[7]).max() < 1e-6
    # int8 Q and K against unquantized attention (Gaussian, no outlier channel:
    # per-token int8 of K loses the other channels next to a x20 channel)
    q, k, v = _inputs(256, 2, 4, outlier=False)
    o, *_ = oracle.attention_int8(q, k, v, 2)
    qt = torch.from_numpy(_vals(q).reshape(256, 2, D).transpose(1, 0, 2).copy())
    kt = torch.from_numpy(_vals(k).reshape(256, 2, D).transpose(1, 0, 2).copy())
    vt = torch.from_numpy(_vals(v).reshape(256, 2, D).transpose(1, 0, 2).copy())
    ref = torch.nn.functional.scaled_dot_product_attention(qt[None], kt[None], vt[None])[0]
    ref = ref.numpy().transpose(1, 0, 2).reshape(256, 2 * D)
    assert np.linalg.norm(o - ref) / np.linalg.norm(ref) < 0.03
