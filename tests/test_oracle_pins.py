"""Pins for the CPU oracle: each test checks it against something other than itself.

Closed forms, invariants, brute force on tiny shapes, library routines (numpy
fp64 matmul, torch's bf16 conversion, Python's round-half-even, math.exp) and
error bounds. Each test names the oracle step it pins; a plausible slip in that
step (a dropped term, a wrong sign or index, a transposed operand, a swapped
gate/up) fails at least one of them.
"""
import math
import os
import subprocess

import numpy as np
import pytest

import oracle
import synth

RNG = np.random.default_rng(1234)


def kron_hadamard(n_levels=8):
    h = np.array([[1]], dtype=np.int64)
    for _ in range(n_levels):
        h = np.kron(np.array([[1, 1], [1, -1]], dtype=np.int64), h)
    return h


def popcount_sign(i, j):
    return -1 if bin(i & j).count("1") % 2 else 1


def fwht_ascending_f32(v):
    """Independent restatement of the pinned order: radix-2 butterflies over each
    256-group, index bit 0 first up to bit 7, fp32 adds, then the 1/16 scale."""
    a = np.array(v, dtype=np.float32).reshape(v.shape[0], -1, 256).copy()
    for b in range(8):
        s = 1 << b
        a = a.reshape(a.shape[0], a.shape[1], 256 // (2 * s), 2, s)
        lo = a[:, :, :, 0, :].copy()
        hi = a[:, :, :, 1, :].copy()
        a[:, :, :, 0, :] = lo + hi
        a[:, :, :, 1, :] = lo - hi
        a = a.reshape(a.shape[0], a.shape[1], 256)
    return (a * np.float32(1.0 / 16.0)).reshape(v.shape[0], -1)


def bf16_rows(rows, K, outliers=0, factor=50.0, seed=0, tid=1):
    f = None
    if outliers:
        f = synth.column_factors(K, synth.outlier_columns(seed, 99, K, outliers), factor)
    return synth.activation_bf16(seed, tid, np.arange(rows), K, f)


def f32(bits):
    return synth.bf16_bits_to_fp32(bits)


# --------------------------------------------------------------------------- H
def test_hadamard_orthogonal_and_kronecker():
    H = oracle.hadamard256().astype(np.int64)
    assert np.array_equal(H @ H.T, 256 * np.eye(256, dtype=np.int64))
    assert np.array_equal(H, kron_hadamard())
    assert np.array_equal(H, H.T)
    for i, j in [(0, 0), (1, 1), (3, 5), (255, 255), (128, 127), (200, 77)]:
        assert H[i, j] == popcount_sign(i, j)


# ------------------------------------------------------------------- rotation
def test_rotate_one_hot_closed_form():
    K = 512
    for g, j in [(0, 0), (0, 7), (1, 200), (1, 255)]:
        v = np.zeros((1, K), dtype=np.float32)
        v[0, g * 256 + j] = 1.0
        y = oracle.rotate_f32(v)
        expect = np.zeros(K, dtype=np.float32)
        expect[g * 256:(g + 1) * 256] = [popcount_sign(i, j) / 16.0 for i in range(256)]
        assert np.array_equal(y[0], expect)
        q, s = oracle.quantize_rows(y)
        assert s[0] == np.float32(np.float32(1 / 16) / np.float32(127))
        grp = q[0, g * 256:(g + 1) * 256]
        assert np.array_equal(grp, np.array([127 * popcount_sign(i, j) for i in range(256)], dtype=np.int8))
        assert not q[0, (1 - g) * 256:(2 - g) * 256].any()


def test_rotate_constant_and_walsh_rows():
    c = np.float32(0.375)
    v = np.full((1, 256), c, dtype=np.float32)
    y = oracle.rotate_f32(v)
    expect = np.zeros(256, dtype=np.float32)
    expect[0] = 16 * c
    assert np.array_equal(y[0], expect)
    q, _ = oracle.quantize_rows(y)
    assert q[0, 0] == 127 and not q[0, 1:].any()
    H = kron_hadamard().astype(np.float32)
    for i in [0, 1, 37, 128, 255]:
        y = oracle.rotate_f32(H[i:i + 1])
        e = np.zeros(256, dtype=np.float32)
        e[i] = 16.0
        assert np.array_equal(y[0], e)


def test_rotate_f32_matches_ascending_fwht_bitwise():
    x = f32(bf16_rows(16, 1024, outliers=10))
    y = oracle.rotate_f32(x)
    assert np.array_equal(y.view(np.uint32), fwht_ascending_f32(x).view(np.uint32))


def test_rotate_f32_within_bound_of_exact():
    x = f32(bf16_rows(8, 768, outliers=8))
    H = kron_hadamard().astype(np.float64) / 16.0
    x64 = x.astype(np.float64).reshape(8, 3, 256)
    exact = np.einsum("rgj,ij->rgi", x64, H).reshape(8, 768)   # exact for these inputs
    y = oracle.rotate_f32(x).astype(np.float64)
    bound = 8 * 2.0 ** -24 * (np.abs(x64).sum(axis=2, keepdims=True) / 16.0)
    bound = np.repeat(bound, 256, axis=2).reshape(8, 768)
    assert np.all(np.abs(y - exact) <= bound)
    assert np.allclose(oracle.rotate_f64(x), exact, rtol=0, atol=1e-12)


def test_rotation_involution_and_invariance_fp64():
    x = RNG.standard_normal((6, 512))
    w = RNG.standard_normal((5, 512))
    xx = oracle.rotate_f64(oracle.rotate_f64(x))
    assert np.max(np.abs(xx - x)) <= 1e-12 * np.max(np.abs(x))
    lhs = oracle.rotate_f64(x) @ oracle.rotate_f64(w).T
    rhs = x @ w.T
    assert np.max(np.abs(lhs - rhs)) <= 1e-12 * np.max(np.abs(rhs))


def test_rotation_spreads_outliers():
    # the purpose of the rotation: a row with one huge channel gets a flat absmax
    x = f32(bf16_rows(4, 512))
    x[:, 3] = 400.0
    y = oracle.rotate_f32(x)
    assert np.max(np.abs(y[:, :256])) < 0.2 * 400.0


# ------------------------------------------------------------------ quantizer
def test_quantizer_round_half_even_ties():
    # absmax = 127 * 2^-3 makes s = 2^-3 exactly, so y/s = n + 1/2 exactly.
    s = 2.0 ** -3
    ns = np.arange(-126, 126, dtype=np.float64)
    y = np.zeros((1, 512), dtype=np.float32)
    y[0, 0] = 127 * s
    y[0, 1:1 + ns.size] = ((ns + 0.5) * s).astype(np.float32)
    q, sc = oracle.quantize_rows(y)
    assert sc[0] == np.float32(s)
    expect = [round(n + 0.5) for n in ns]   # Python rounds half to even
    assert list(q[0, 1:1 + ns.size]) == expect


def test_quantizer_properties():
    y = oracle.rotate_f32(f32(bf16_rows(32, 768, outliers=8)))
    q, s = oracle.quantize_rows(y)
    qn, sn = oracle.quantize_rows(-y)
    assert np.array_equal(qn, -q) and np.array_equal(sn, s)
    for k in (-5, 3):
        qk, sk = oracle.quantize_rows(y * np.float32(2.0 ** k))
        assert np.array_equal(qk, q) and np.array_equal(sk, s * np.float32(2.0 ** k))
    assert np.all(np.abs(q).max(axis=1) == 127)
    assert q.min() >= -127
    err = np.abs(q.astype(np.float64) * s[:, None] - y)
    assert np.all(err <= s[:, None] * (0.5 + 1e-5))
    q0, s0 = oracle.quantize_rows(np.zeros((2, 256), dtype=np.float32))
    assert not q0.any() and not s0.any()


def test_quantizer_scale_is_fp32_division():
    y = np.zeros((1, 256), dtype=np.float32)
    y[0, 5] = np.float32(3.3)
    _, s = oracle.quantize_rows(y)
    # absmax/127 correctly rounded to fp32 (Python float division is exact to fp64, then fp32)
    assert s[0] == np.float32(np.float64(np.float32(3.3)) / 127.0)


# ----------------------------------------------------------------------- GEMM
def test_gemm_brute_force_tiny():
    for M, N in [(1, 1), (3, 4), (4, 2)]:
        xq = RNG.integers(-127, 128, size=(M, 256), dtype=np.int64).astype(np.int8)
        wq = RNG.integers(-127, 128, size=(N, 256), dtype=np.int64).astype(np.int8)
        acc = oracle.gemm_s32(xq, wq)
        assert acc.shape == (M, N)
        for m in range(M):
            for n in range(N):
                assert acc[m, n] == sum(int(xq[m, k]) * int(wq[n, k]) for k in range(256))


def test_gemm_matches_fp64_matmul_and_extremes():
    xq = RNG.integers(-127, 128, size=(37, 1024), dtype=np.int64).astype(np.int8)
    wq = RNG.integers(-127, 128, size=(29, 1024), dtype=np.int64).astype(np.int8)
    acc = oracle.gemm_s32(xq, wq)
    assert np.array_equal(acc.astype(np.float64), xq.astype(np.float64) @ wq.astype(np.float64).T)
    K = 14336
    a = np.full((1, K), 127, dtype=np.int8)
    b = np.full((2, K), -127, dtype=np.int8)
    b[1] = 127
    acc = oracle.gemm_s32(a, b)
    assert acc[0, 0] == -127 * 127 * K and acc[0, 1] == 127 * 127 * K


# ------------------------------------------------------------------- epilogue
def test_epilogue_closed_form_indices():
    M, N = 3, 5
    acc = np.arange(M * N, dtype=np.int32).reshape(M, N) * 8 - 40
    sx = np.array([0.5, 2.0, 0.25], dtype=np.float32)
    sw = np.array([1.0, 4.0, 0.125, 2.0, 0.5], dtype=np.float32)
    bias = synth.bf16_rne_bits(np.array([1.0, -2.0, 0.5, 3.0, -0.25], dtype=np.float32))
    v, out = oracle.epilogue(acc, sx, sw, bias)
    expect = np.array([[acc[m, n] * float(sx[m]) * float(sw[n]) + [1.0, -2.0, 0.5, 3.0, -0.25][n]
                        for n in range(N)] for m in range(M)])
    assert np.array_equal(v.astype(np.float64), expect)
    assert np.array_equal(f32(out).astype(np.float64), expect)   # all representable in bf16
    v2, _ = oracle.epilogue(acc, sx, sw, None)
    assert np.array_equal(v2.astype(np.float64), expect - np.array([1.0, -2.0, 0.5, 3.0, -0.25])[None, :])


def test_epilogue_within_ulps_of_fp64():
    acc = RNG.integers(-2 ** 27, 2 ** 27, size=(16, 24)).astype(np.int32)
    sx = RNG.random(16).astype(np.float32) * 0.1
    sw = RNG.random(24).astype(np.float32) * 1e-4
    bias = synth.bf16_rne_bits(RNG.standard_normal(24).astype(np.float32) * 0.01)
    v, out = oracle.epilogue(acc, sx, sw, bias)
    exact = acc.astype(np.float64) * sx[:, None] * sw[None, :] + f32(bias)[None, :]
    ulp = np.spacing(np.maximum(np.abs(exact), np.abs(acc * sx[:, None].astype(np.float64) * sw[None, :]))
                     .astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(v - exact) <= 3 * ulp)


def test_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    vals = np.concatenate([
        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 3.0e38, 1e-30, 0.0, -0.0], dtype=np.float32),
        RNG.standard_normal(1000).astype(np.float32) * 100])
    theirs = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    mine = np.array([oracle.f32_to_bf16(v) for v in vals], dtype=np.uint16)
    assert np.array_equal(mine, theirs)


# --------------------------------------------------------------------- SwiGLU
def test_exp_and_silu_against_math():
    ts = np.linspace(-19.9, 88.7, 4001, dtype=np.float32)
    for t in ts:
        e = oracle.exp_f32(float(t))
        ref = math.exp(float(t))
        assert abs(e - ref) <= 2 * np.spacing(np.float32(ref)), (t, e, ref)
    for g in np.linspace(-100, 100, 2001, dtype=np.float32):
        s = oracle.silu_f32(float(g))
        ref = float(g) / (1.0 + math.exp(-float(g)))
        assert abs(s - ref) <= 4 * np.spacing(np.float32(abs(ref))) + 2.0 ** -149, (g, s, ref)
    assert oracle.silu_f32(0.0) == 0.0
    assert oracle.silu_f32(30.0) == 30.0
    assert oracle.silu_f32(-130.0) == 0.0 and math.copysign(1.0, oracle.silu_f32(-130.0)) == -1.0


def test_exp_finite_up_to_fp32_overflow():
    """e^t is finite for every fp32 t whose true exponential is at most FLT_MAX (ln FLT_MAX
    is about 88.7228) and +inf above; silu(g) for g just below -88 (where e^-g is finite
    but above 2^127) and below -88.72 (where it overflows) is a nonzero value near g e^g."""
    fmax = float(np.finfo(np.float32).max)
    t = np.float32(88.0)
    while math.exp(float(np.nextafter(t, np.float32(np.inf)))) <= fmax:
        t = np.nextafter(t, np.float32(np.inf))
    assert math.exp(float(t)) <= fmax < math.exp(float(np.nextafter(t, np.float32(np.inf))))
    assert math.isfinite(oracle.exp_f32(float(t)))
    top_ulp = 2.0 ** 104  # the spacing of fp32 values in [2^127, 2^128), where e^t lies here
    assert abs(oracle.exp_f32(float(t)) - math.exp(float(t))) <= 2 * top_ulp
    assert math.isfinite(oracle.exp_f32(88.3)) and oracle.exp_f32(89.5) == math.inf
    for g in (-88.3, -88.9, -95.0):
        g32 = float(np.float32(g))
        s = oracle.silu_f32(g32)
        ref = g32 / (1.0 + math.exp(-g32))
        assert s < 0.0 and abs(s - ref) <= 4 * np.spacing(np.float32(abs(ref))) + 2.0 ** -149, (g, s, ref)
    assert abs(oracle.silu_f32(-88.3)) >= np.finfo(np.float32).tiny          # a normal number


def _exp_silu_check(tmp_path):
    exe = tmp_path / "exp_silu_check"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-o", str(exe),
                           os.path.join(os.path.dirname(__file__), "csrc", "exp_silu_check.c"), "-lm", "-ldl"])

    def run(*args):
        out = subprocess.run([str(exe), oracle.build(), *map(str, args)], capture_output=True, text=True,
                             check=True)
        checked, bad, worst_milli_ulp = map(int, out.stdout.split())
        return checked, bad, worst_milli_ulp / 1000.0
    return run


def test_exp_and_silu_over_every_float_against_libm(tmp_path):
    """Against the C library's double exp, over fp32 arguments: e^t on [-20, 89] within 2 ulps
    (+inf or FLT_MAX where the true value is above FLT_MAX), silu on [-100, 100] within 4 ulps.
    Every float in the windows where the cut-offs sit ([87.5, 89] for e^t; [-100, -80] and
    [-21, -19] for silu, [-20, -19] for e^t, below which it is taken as 0); elsewhere every 13th bit pattern, or every float
    with H3Q_FULL_EXP_SWEEP=1 (about a minute on 8 cores)."""
    run = _exp_silu_check(tmp_path)
    stride = 1 if os.environ.get("H3Q_FULL_EXP_SWEEP") == "1" else 13
    for args in (("exp", stride), ("exp", 1, 87.5, 89.0), ("exp", 1, -20.0, -19.0),
                 ("silu", stride), ("silu", 1, -100.0, -80.0), ("silu", 1, -21.0, -19.0)):
        checked, bad, worst = run(*args)
        assert checked > 100_000 and bad == 0, (args, checked, bad, worst)


def test_swiglu_gate_is_first_half():
    g = np.array([[1.5, -2.0, 0.25]], dtype=np.float32)
    u = np.array([[3.0, 0.5, -4.0]], dtype=np.float32)
    h, out = oracle.swiglu(np.concatenate([g, u], axis=1))
    ref = g.astype(np.float64) / (1 + np.exp(-g.astype(np.float64))) * u
    assert np.allclose(h, ref, rtol=1e-6, atol=0)
    swapped = u.astype(np.float64) / (1 + np.exp(-u.astype(np.float64))) * g
    assert not np.allclose(h, swapped, rtol=1e-3)


# ------------------------------------------------------------ whole layer
def _tiny_layer():
    wl = synth.WORKLOADS["tiny"]
    ids = synth.tensor_ids()
    x = synth.activation_bf16(wl.seed, ids["x"], np.arange(wl.M), wl.K, wl.factors())
    w = synth.weight_fp32(wl.seed, ids["w"], np.arange(wl.N), wl.K)
    return wl, x, w


def test_linear_accuracy_vs_unquantized_and_rotation_ablation():
    wl, x, w = _tiny_layer()
    wq, sw = oracle.prepare_weight(w)
    y, extra = oracle.linear(x, wq, sw, want=("acc", "xq", "sx"))
    ref = f32(x).astype(np.float64) @ w.astype(np.float64).T
    rel = np.linalg.norm(f32(y) - ref) / np.linalg.norm(ref)
    assert rel <= 2e-2, rel
    cos = np.sum(f32(y) * ref) / (np.linalg.norm(f32(y)) * np.linalg.norm(ref))
    assert cos > 0.999
    # ablation: the same per-row absmax int8 quantizer without the rotation
    def plain_q(a):
        s = np.abs(a).max(axis=1, keepdims=True) / 127.0
        return np.clip(np.rint(a / s), -127, 127), s
    xq0, sx0 = plain_q(f32(x).astype(np.float64))
    wq0, sw0 = plain_q(w.astype(np.float64))
    y0 = (xq0 @ wq0.T) * sx0 * sw0.T
    rel0 = np.linalg.norm(y0 - ref) / np.linalg.norm(ref)
    assert rel0 > 2 * rel, (rel0, rel)
    # the rotated int8 GEMM approximates the fp64 product of the rotated operands
    assert np.array_equal(extra["acc"], oracle.gemm_s32(extra["xq"], wq))


def test_linear_bias_and_swiglu_paths():
    wl, x, w = _tiny_layer()
    wq, sw = oracle.prepare_weight(w)
    bias = synth.bias_bf16(0, 3, wl.N)
    y, _ = oracle.linear(x, wq, sw, bias_bits=bias)
    ref = f32(x).astype(np.float64) @ w.astype(np.float64).T + f32(bias)[None, :]
    assert np.linalg.norm(f32(y) - ref) / np.linalg.norm(ref) <= 2e-2
    h, _ = oracle.linear(x, wq, sw, swiglu_epilogue=True)
    F = wl.N // 2
    g, u = ref[:, :F] - f32(bias)[None, :F], ref[:, F:] - f32(bias)[None, F:]
    href = g / (1 + np.exp(-g)) * u
    assert h.shape == (wl.M, F)
    assert np.linalg.norm(f32(h) - href) / np.linalg.norm(href) <= 3e-2


def test_ffn_accuracy_vs_unquantized():
    M, K, F = 48, 512, 768
    f = synth.column_factors(K, synth.outlier_columns(0, 4, K, 5), 50.0)
    x = synth.activation_bf16(0, 1, np.arange(M), K, f)
    wgu = synth.weight_fp32(0, 5, np.arange(2 * F), K)
    wd = synth.weight_fp32(0, 6, np.arange(K), F)
    qgu, sgu = oracle.prepare_weight(wgu)
    qd, sd = oracle.prepare_weight(wd)
    y, h, hq, sh = oracle.ffn(x, qgu, sgu, qd, sd)
    xf = f32(x).astype(np.float64)
    g = xf @ wgu[:F].astype(np.float64).T
    u = xf @ wgu[F:].astype(np.float64).T
    href = g / (1 + np.exp(-g)) * u
    yref = href @ wd.astype(np.float64).T
    assert np.linalg.norm(f32(y) - yref) / np.linalg.norm(yref) <= 3e-2
    # h's codes are its own rotation + quantization
    q2, s2 = oracle.rotate_quant_bf16(h)
    assert np.array_equal(q2, hq) and np.array_equal(s2, sh)


# ------------------------------------------------------------------- LoRA merge
def _lora(N, K, r, seed=3):
    rng = np.random.default_rng(seed)
    a = (rng.standard_normal((r, K)) * 0.05).astype(np.float32)
    b = (rng.standard_normal((N, r)) * 0.05).astype(np.float32)
    return a, b


def test_lora_merge_zero_delta_keeps_codes():
    w = synth.weight_fp32(0, 2, np.arange(64), 512)
    wq, sw = oracle.prepare_weight(w)
    a, b = _lora(64, 512, 8)
    q2, s2 = oracle.lora_merge(wq, sw, a, b, 0.0)
    assert np.array_equal(q2, wq)
    assert np.array_equal(s2, sw)
    q3, s3 = oracle.lora_merge(wq, sw, a, np.zeros_like(b), 1.5)
    assert np.array_equal(q3, wq) and np.array_equal(s3, sw)


def test_lora_merge_matches_rotated_sum_within_quantization_error():
    N, K, r, alpha = 96, 768, 16, 0.75
    w = synth.weight_fp32(0, 2, np.arange(N), K)
    wq, sw = oracle.prepare_weight(w)
    a, b = _lora(N, K, r)
    q2, s2 = oracle.lora_merge(wq, sw, a, b, alpha)
    H = kron_hadamard().astype(np.float64) / 16.0
    rot = lambda m: np.einsum("rgj,ij->rgi", m.reshape(m.shape[0], -1, 256), H).reshape(m.shape)
    target = wq.astype(np.float64) * sw[:, None] + alpha * (b.astype(np.float64) @ rot(a.astype(np.float64)))
    err = np.abs(q2.astype(np.float64) * s2[:, None] - target)
    assert np.all(err <= s2[:, None] * (0.5 + 1e-4))
    assert np.all(np.abs(q2).max(axis=1) == 127)
    # the delta is applied in the rotated basis: the unrotated sum is far off
    wrong = wq.astype(np.float64) * sw[:, None] + alpha * (b.astype(np.float64) @ a.astype(np.float64))
    assert np.abs(q2.astype(np.float64) * s2[:, None] - wrong).max() > 10 * s2.max()


def test_lora_merged_layer_matches_fp64_model():
    N, K, r, alpha = 128, 512, 8, 1.0
    x = synth.activation_bf16(0, 1, np.arange(48), K)
    w = synth.weight_fp32(0, 2, np.arange(N), K)
    wq, sw = oracle.prepare_weight(w)
    a, b = _lora(N, K, r)
    q2, s2 = oracle.lora_merge(wq, sw, a, b, alpha)
    y, _ = oracle.linear(x, q2, s2)
    ref = f32(x).astype(np.float64) @ (w.astype(np.float64) + alpha * b.astype(np.float64) @ a.astype(np.float64)).T
    assert np.linalg.norm(f32(y) - ref) / np.linalg.norm(ref) <= 2e-2
