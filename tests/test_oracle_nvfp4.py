"""Pins of the oracle's NVFP4 functions (the hybrid checkpoints' format for the
QKV and FFN-input projections) against what the format's definition and the
mathematics fix, independently of the oracle's own code:

* e2m1 values from the sign/exponent/mantissa fields; e2m1 rounding against
  numpy's round-half-even at the format's quantum for each binade;
* e4m3 values and rounding against torch's float8_e4m3fn conversion;
* the quantizer: power-of-two invariance (the tensor scale absorbs it exactly),
  exact round trip of tensors that are representable, the zero tensor, an
  error bound;
* the layer: exact result on representable inputs against a float64 matmul,
  accuracy on Gaussian data, gate-first SwiGLU, the magnitude sum.
"""
import numpy as np
import pytest
import torch

import oracle


def _e2m1_from_fields(c):
    s, e, m = (c >> 3) & 1, (c >> 1) & 3, c & 1
    mag = m * 0.5 if e == 0 else (1.0 + m / 2.0) * 2.0 ** (e - 1)
    return -mag if s else mag


def test_e2m1_values_from_fields():
    for c in range(16):
        assert oracle.e2m1_value(c) == _e2m1_from_fields(c)
        assert np.signbit(oracle.e2m1_value(c)) == bool(c & 8)


def _e2m1_round_numpy(x):
    a = abs(x)
    if a >= 6.0:
        mag = 6.0
    else:
        q = 0.5 if a < 2.0 else (1.0 if a < 4.0 else 2.0)  # spacing of the binade
        mag = min(6.0, float(np.rint(a / q)) * q)
    return -mag if np.signbit(x) else mag


def test_e2m1_rounding_matches_round_half_even_per_binade():
    xs = np.concatenate([np.linspace(-8, 8, 4097), [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, 1e30, -1e-30]])
    for x in xs.astype(np.float32):
        got = oracle.e2m1_value(oracle.e2m1_rne(float(x)))
        want = _e2m1_round_numpy(float(x))
        assert got == want and np.signbit(got) == np.signbit(want), (x, got, want)
    # the ties, explicitly
    for x, v in [(0.25, 0.0), (0.75, 1.0), (1.25, 1.0), (1.75, 2.0), (2.5, 2.0), (3.5, 4.0), (5.0, 4.0)]:
        assert oracle.e2m1_value(oracle.e2m1_rne(x)) == v


def test_e4m3_values_match_torch():
    codes = np.arange(0x7F, dtype=np.uint8)  # every non-negative finite code
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    for c in codes:
        assert oracle.e4m3_value(int(c)) == ref[c]
    assert oracle.e4m3_value(0x7E) == 448.0


def test_e4m3_rounding_matches_torch_and_saturates():
    rng = np.random.default_rng(1)
    us = np.concatenate([np.exp(rng.uniform(np.log(1e-4), np.log(448.0), 3000)),
                         [oracle.e4m3_value(c) for c in range(0x7F)],
                         [(oracle.e4m3_value(c) + oracle.e4m3_value(c + 1)) / 2 for c in range(0x7E)]]).astype(np.float32)
    ref = torch.from_numpy(us).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for u, r in zip(us, ref):
        assert oracle.e4m3_rne_sat(float(u)) == r, u
    assert oracle.e4m3_rne_sat(449.0) == 0x7E and oracle.e4m3_rne_sat(1e9) == 0x7E
    assert oracle.e4m3_rne_sat(0.0) == 0


def _dequant(codes, sf, s_enc):
    rows, k2 = codes.shape
    q = np.empty((rows, 2 * k2), dtype=np.float64)
    q[:, 0::2] = np.vectorize(oracle.e2m1_value)(codes & 15)
    q[:, 1::2] = np.vectorize(oracle.e2m1_value)(codes >> 4)
    s = np.vectorize(oracle.e4m3_value)(sf).astype(np.float64)
    return q * np.repeat(s, 16, axis=1) / np.float64(s_enc)


def test_quantize_is_invariant_under_powers_of_two():
    x = (np.random.default_rng(2).standard_normal((6, 128)) * 3).astype(np.float32)
    c0, s0, e0 = oracle.nvfp4_quantize(x)
    for j in (-3, 5):
        c1, s1, e1 = oracle.nvfp4_quantize(x * np.float32(2.0 ** j))
        assert np.array_equal(c0, c1) and np.array_equal(s0, s1)
        assert e1 == e0 * 2.0 ** -j


def _representable(rng, rows, K):
    """Rows whose blocks are e2m1 values times 2^-j with one element at +-6 * 2^-j,
    and a tensor max of 6: NVFP4 represents them exactly (s_enc = 448)."""
    grid = np.array([oracle.e2m1_value(c) for c in range(16)])
    x = rng.choice(grid, size=(rows, K))
    j = rng.integers(0, 6, size=(rows, K // 16))
    j[0, 0] = 0
    x = x.reshape(rows, K // 16, 16)
    x[:, :, 0] = np.where(rng.integers(0, 2, size=(rows, K // 16)) == 1, 6.0, -6.0)
    return (x * 2.0 ** -j[:, :, None]).reshape(rows, K).astype(np.float32)


def test_quantize_round_trips_representable_tensors():
    x = _representable(np.random.default_rng(3), 8, 256)
    codes, sf, s_enc = oracle.nvfp4_quantize(x)
    assert s_enc == 448.0
    assert np.array_equal(_dequant(codes, sf, s_enc), x.astype(np.float64))


def test_quantize_zero_tensor_and_error_bound():
    codes, sf, s_enc = oracle.nvfp4_quantize(np.zeros((2, 64), np.float32))
    assert s_enc == 1.0 and not codes.any() and not sf.any()
    x = np.random.default_rng(4).standard_normal((16, 512)).astype(np.float32)
    x[3, :16] = 0.0  # an all-zero block keeps scale 0 and codes 0
    codes, sf, s_enc = oracle.nvfp4_quantize(x)
    assert sf[3, 0] == 0 and not codes[3, :8].any()
    err = np.abs(_dequant(codes, sf, s_enc) - x)
    bmax = np.repeat(np.abs(x).reshape(16, -1, 16).max(axis=2), 16, axis=1)
    # half the widest e2m1 spacing (1 of 6) of a block scale within 1/16 of bmax/6
    assert np.all(err <= bmax / 6.0 * (1 + 1 / 16) + 1e-30)
    assert np.abs(_dequant(codes, sf, s_enc)).max() <= np.abs(x).max() * (1 + 1 / 16)


def test_linear_exact_on_representable_inputs():
    rng = np.random.default_rng(5)
    x, w = _representable(rng, 12, 256), _representable(rng, 40, 256)
    ca, sfa, ea = oracle.nvfp4_quantize(x)
    cw, sfw, ew = oracle.nvfp4_quantize(w)
    y, acc, mag = oracle.nvfp4_linear(ca, sfa, ea, cw, sfw, ew)
    ref = x.astype(np.float64) @ w.astype(np.float64).T * (448.0 * 448.0)
    assert np.array_equal(acc, ref)
    assert np.all(mag >= np.abs(acc))
    yv = torch.from_numpy(y.view(np.int16)).view(torch.bfloat16).double().numpy()
    want = torch.from_numpy((x.astype(np.float64) @ w.astype(np.float64).T).astype(np.float32)).bfloat16().double().numpy()
    assert np.abs(yv - want).max() <= np.abs(want).max() * 2.0 ** -7


def test_linear_accuracy_and_gate_first_swiglu():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((32, 512)).astype(np.float32)
    w = (rng.standard_normal((64, 512)) * 0.02).astype(np.float32)
    ca, sfa, ea = oracle.nvfp4_quantize(x)
    cw, sfw, ew = oracle.nvfp4_quantize(w)
    y, _, _ = oracle.nvfp4_linear(ca, sfa, ea, cw, sfw, ew)
    yv = torch.from_numpy(y.view(np.int16)).view(torch.bfloat16).double().numpy()
    ref = x.astype(np.float64) @ w.astype(np.float64).T
    rel = np.linalg.norm(yv - ref) / np.linalg.norm(ref)
    assert 0.02 < rel < 0.2  # 4-bit elements: well above int8's error, well below noise
    h, _, _ = oracle.nvfp4_linear(ca, sfa, ea, cw, sfw, ew, swiglu_epilogue=True)
    hv = torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).double().numpy()
    g, u = yv[:, :32], yv[:, 32:]
    assert np.abs(hv - g / (1 + np.exp(-g)) * u).max() <= 0.02 * np.abs(hv).max() + 1e-3
    h2, _, _ = oracle.nvfp4_linear(ca, sfa, ea, np.concatenate([cw[32:], cw[:32]]),
                                   np.concatenate([sfw[32:], sfw[:32]]), ew, swiglu_epilogue=True)
    assert not np.array_equal(h, h2)


def test_epilogue_closed_form_and_agreement_with_the_layer():
    rng = np.random.default_rng(7)
    # power-of-two tensor scales make alpha exact: v = acc * 2^-16 + bias
    acc = (rng.integers(-2 ** 20, 2 ** 20, size=(5, 64)) * 0.25).astype(np.float32)
    bias = torch.from_numpy(rng.standard_normal(64).astype(np.float32)).bfloat16()
    bb = bias.view(torch.int16).numpy().view(np.uint16)
    y = oracle.nvfp4_epilogue(acc, 256.0, 256.0, bias_bits=bb)
    want = (torch.from_numpy(acc.astype(np.float64) * 2.0 ** -16).float() + bias.float()).bfloat16()
    assert np.array_equal(y, want.view(torch.int16).numpy().view(np.uint16))
    # the layer's output is its epilogue applied to RN(acc)
    x = rng.standard_normal((8, 256)).astype(np.float32)
    w = (rng.standard_normal((32, 256)) * 0.02).astype(np.float32)
    ca, sfa, ea = oracle.nvfp4_quantize(x)
    cw, sfw, ew = oracle.nvfp4_quantize(w)
    for sw in (False, True):
        y1, a64, _ = oracle.nvfp4_linear(ca, sfa, ea, cw, sfw, ew, swiglu_epilogue=sw)
        assert np.array_equal(y1, oracle.nvfp4_epilogue(a64.astype(np.float32), ea, ew, swiglu_epilogue=sw))
