// Plain CPU oracle for the INT8 ConvRot (W8A8, Hadamard-256) linear layer.
//
// TEST INFRASTRUCTURE ONLY. Only the tests, the package smoke check and the
// benchmark's CPU-baseline leg may load this library. The product path never
// calls it and shares no code with it.
//
// What it computes, and where the pages state it:
//  * ConvRot: a group-wise Hadamard rotation along K, expressed as a conv with
//    kernel = stride = 256, i.e. a block-diagonal product with a 256x256
//    Hadamard matrix (cloud-worker "MiniMax H3 - research findings", section
//    "Weight families"; h3-rs README, model-file table: "int8 per-row + ConvRot
//    (Hadamard-256)").
//  * Weights stored pre-rotated as per-row int8 with one scale per output row
//    (h3-rs README, model-file table).
//  * Activations rotated inside the quantizer and quantized per row (per
//    token); int8 GEMM; bf16 written directly; SwiGLU fused into fc1's epilogue
//    (h3-rs README, "Speed", "What makes it fast").
//  * The FFN-output projection stays INT8 ConvRot, so the SwiGLU output is
//    rotated and quantized again before it (Minimax_h3_hybrid model card,
//    "Checkpoints").
//  * LoRA deltas are merged into the stored int8 weights at load by
//    dequantizing, adding and requantizing (h3-rs README, "Speed", "What makes
//    it fast"); the delta is rotated along K like the weights it joins.
//
// Readings where the pages are silent (each one is listed with its reason in
// the design notes): H is the natural-order Sylvester matrix scaled by 1/16; the
// fp32 sum of each rotated element is a pairwise tree over j in natural order;
// scale = absmax / 127 (fp32 division); q = clamp(rne(y / scale), -127, 127);
// one scale per token over the whole row; epilogue order
// ((float)acc * sx) * sw + bias without fused multiply-add; SwiGLU takes the
// first half of the fc1 outputs as gate and the second half as up; e^-g is
// evaluated by Cody-Waite reduction and a degree-7 Taylor polynomial in fp32,
// with the power of two moved onto the numerator where e^-g >= 2^64;
// the LoRA delta B A_rot is a fused multiply-add chain over the rank index in
// ascending order, scaled by alpha and added to q * s as two rounded products
// and one rounded add.
//
// Plain loops, no blocking or fusion beyond what the definition states.
// Build: g++ -O2 -std=c++17 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

extern "C" {

// ---------------------------------------------------------------------------
// bf16 helpers (bit patterns in uint16_t).
// ---------------------------------------------------------------------------
static inline float bf16_to_f32(uint16_t b) {
  uint32_t u = uint32_t(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7f800000u) == 0x7f800000u) {            // inf / nan: keep, quiet nan
    return uint16_t((u >> 16) | ((u & 0xffffu) ? 0x40u : 0u));
  }
  u += 0x7fffu + ((u >> 16) & 1u);
  return uint16_t(u >> 16);
}

float orc_bf16_to_f32(uint16_t b) { return bf16_to_f32(b); }
uint16_t orc_f32_to_bf16(float f) { return f32_to_bf16_rne(f); }

// ---------------------------------------------------------------------------
// Step 1: the 256x256 Hadamard matrix, natural (Sylvester) ordering,
// H[i][j] = (-1)^popcount(i & j).
// ---------------------------------------------------------------------------
static const int kG = 256;

void orc_hadamard256(int8_t* H) {
  for (int i = 0; i < kG; ++i)
    for (int j = 0; j < kG; ++j)
      H[i * kG + j] = (__builtin_popcount(unsigned(i & j)) & 1) ? -1 : 1;
}

static const std::vector<int8_t>& hadamard() {
  static std::vector<int8_t> H = [] {
    std::vector<int8_t> h(kG * kG);
    orc_hadamard256(h.data());
    return h;
  }();
  return H;
}

// ---------------------------------------------------------------------------
// Step 2: rotate each 256-wide group of a row by H/16.
// y[g*256+i] = sum_j v[g*256+j] * H[i][j] / 16, in fp32. Every term is exact
// (a sign and a power-of-two scale of the input); the sum is a pairwise tree
// over j in natural order: level 0 adds terms (2t, 2t+1), level 1 adds those
// pairs, and so on through level 7.
// ---------------------------------------------------------------------------
static void rotate_group_f32(const float* v, float* y) {
  const std::vector<int8_t>& H = hadamard();
  float t[kG];
  for (int i = 0; i < kG; ++i) {
    for (int j = 0; j < kG; ++j) t[j] = v[j] * (float(H[i * kG + j]) / 16.0f);
    for (int width = kG; width > 1; width /= 2)
      for (int p = 0; p < width / 2; ++p) t[p] = t[2 * p] + t[2 * p + 1];
    y[i] = t[0];
  }
}

void orc_rotate_f32(const float* v, int64_t rows, int64_t K, float* y) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t g = 0; g < K / kG; ++g)
      rotate_group_f32(v + r * K + g * kG, y + r * K + g * kG);
}

// Same rotation in fp64 (plain left-to-right sum), used to check the fp32 one.
void orc_rotate_f64(const double* v, int64_t rows, int64_t K, double* y) {
  const std::vector<int8_t>& H = hadamard();
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t g = 0; g < K / kG; ++g)
      for (int i = 0; i < kG; ++i) {
        double acc = 0.0;
        for (int j = 0; j < kG; ++j) acc += v[r * K + g * kG + j] * double(H[i * kG + j]);
        y[r * K + g * kG + i] = acc / 16.0;
      }
}

// ---------------------------------------------------------------------------
// Steps 3-4: per-row symmetric int8 quantization of rotated values.
// a = max |y| over the whole row; s = a / 127 (fp32); q = clamp(rne(y / s)).
// A zero row gives s = 0 and q = 0.
// ---------------------------------------------------------------------------
static void quantize_row(const float* y, int64_t K, int8_t* q, float* s_out) {
  float a = 0.0f;
  for (int64_t k = 0; k < K; ++k) a = std::fmax(a, std::fabs(y[k]));
  const float s = a / 127.0f;
  *s_out = s;
  for (int64_t k = 0; k < K; ++k) {
    if (s == 0.0f) { q[k] = 0; continue; }
    float r = std::nearbyint(y[k] / s);   // FE_TONEAREST: ties to even
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    q[k] = int8_t(r);
  }
}

void orc_quantize_rows(const float* y, int64_t rows, int64_t K, int8_t* q, float* s) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) quantize_row(y + r * K, K, q + r * K, s + r);
}

// Activations: bf16 [rows, K] -> rotated int8 [rows, K] + fp32 scale per row.
void orc_rotate_quant_bf16(const uint16_t* x, int64_t rows, int64_t K, int8_t* q, float* s) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    std::vector<float> v(K), y(K);
    for (int64_t k = 0; k < K; ++k) v[k] = bf16_to_f32(x[r * K + k]);
    for (int64_t g = 0; g < K / kG; ++g) rotate_group_f32(v.data() + g * kG, y.data() + g * kG);
    quantize_row(y.data(), K, q + r * K, s + r);
  }
}

// Step 5: weights fp32 [N, K] -> rotated per-row int8 + fp32 scale per row.
void orc_prepare_weight(const float* w, int64_t N, int64_t K, int8_t* q, float* s) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    std::vector<float> y(K);
    for (int64_t g = 0; g < K / kG; ++g) rotate_group_f32(w + n * K + g * kG, y.data() + g * kG);
    quantize_row(y.data(), K, q + n * K, s + n);
  }
}

// ---------------------------------------------------------------------------
// Step 6: integer GEMM, acc[m][n] = sum_k xq[m][k] * wq[n][k], exact in int64.
// Returns the number of entries outside the int32 range (0 expected).
// ---------------------------------------------------------------------------
int64_t orc_gemm_s32(const int8_t* xq, const int8_t* wq, int64_t M, int64_t N, int64_t K, int32_t* acc) {
  int64_t overflow = 0;
#pragma omp parallel for schedule(static) reduction(+ : overflow)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      int64_t a = 0;
      for (int64_t k = 0; k < K; ++k) a += int64_t(xq[m * K + k]) * int64_t(wq[n * K + k]);
      if (a > INT32_MAX || a < INT32_MIN) ++overflow;
      acc[m * N + n] = int32_t(a);
    }
  return overflow;
}

// ---------------------------------------------------------------------------
// Step 7: epilogue, v = ((float)acc * sx[m]) * sw[n] (+ bias[n]); out = bf16(v).
// No fused multiply-add (the build disables contraction).
// ---------------------------------------------------------------------------
static inline float epilogue_value(int32_t acc, float sx, float sw, const uint16_t* bias, int64_t n) {
  float v = float(acc);
  v = v * sx;
  v = v * sw;
  if (bias) v = v + bf16_to_f32(bias[n]);
  return v;
}

void orc_epilogue(const int32_t* acc, const float* sx, const float* sw, const uint16_t* bias,
                  int64_t M, int64_t N, float* v, uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      const float x = epilogue_value(acc[m * N + n], sx[m], sw[n], bias, n);
      if (v) v[m * N + n] = x;
      if (out) out[m * N + n] = f32_to_bf16_rne(x);
    }
}

// ---------------------------------------------------------------------------
// Step 8: SwiGLU, h = silu(g) * u with silu(g) = g / (1 + e^-g) (h3-rs README,
// "Speed", "What makes it fast": SwiGLU in fc1's epilogue).
// e^t is evaluated in fp32 as p * 2^n: Cody-Waite reduction t = n ln2 + r with
// n = rne(t log2 e) and the two-part ln2 of fdlibm's expf (0x3f317200 and
// 0x35bfbe8e), then p = e^r by the degree-7 Taylor polynomial in Horner form
// with fused multiply-adds. e^t itself is p scaled by 2^n (ldexp: exact, +inf
// only where the scaled value overflows fp32, i.e. t above ln(FLT_MAX) ~ 88.72).
// For t < -20, 1 + e^t rounds to 1 in fp32 whatever e^t is, so e^t is taken as 0.
// ---------------------------------------------------------------------------
static void exp_parts(float t, float* p_out, int* n_out) {
  const float n = std::nearbyint(t * 1.44269502f);   // log2(e) rounded to fp32
  float r = std::fma(n, -0.693145751953125f, t);     // ln2 high part (0x3f317200)
  r = std::fma(n, -1.42860677e-06f, r);              // ln2 low part  (0x35bfbe8e)
  float p = 1.0f / 5040.0f;
  p = std::fma(p, r, 1.0f / 720.0f);
  p = std::fma(p, r, 1.0f / 120.0f);
  p = std::fma(p, r, 1.0f / 24.0f);
  p = std::fma(p, r, 1.0f / 6.0f);
  p = std::fma(p, r, 0.5f);
  p = std::fma(p, r, 1.0f);
  p = std::fma(p, r, 1.0f);
  *p_out = p;
  *n_out = int(n);
}

float orc_exp_f32(float t) {
  if (t < -20.0f) return 0.0f;
  if (t > 89.0f) return INFINITY;                    // e^t > FLT_MAX for t > 88.73
  float p;
  int n;
  exp_parts(t, &p, &n);
  return std::ldexp(p, n);
}

// silu(g) = RN(g / RN(1 + e^-g)). Where e^-g is at least 2^64 (g below about
// -44.4), 1 + e^-g rounds to e^-g = p * 2^n, and the quotient g / (p * 2^n) is
// formed as (g * 2^(64-n)) / (p * 2^64): both operands are exact, so this is the
// same correctly rounded quotient, and it stays right where e^-g itself
// overflows fp32 (g < -88.72) down to where silu underflows. For g < -120,
// |silu(g)| < 2^-160 and the result is -0.
float orc_silu_f32(float g) {
  const float t = -g;
  if (t < -20.0f) return g;
  if (t > 120.0f) return -0.0f;
  float p;
  int n;
  exp_parts(t, &p, &n);
  if (n <= 64) return g / (1.0f + std::ldexp(p, n));
  return std::ldexp(g, 64 - n) / std::ldexp(p, 64);
}

// Element-wise forms of the two functions above, for checking them over many arguments.
void orc_exp_f32_array(const float* t, int64_t n, float* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = orc_exp_f32(t[i]);
}

void orc_silu_f32_array(const float* g, int64_t n, float* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = orc_silu_f32(g[i]);
}

// v [M, 2F] (epilogue values of the fc1 rows: gate = [0,F), up = [F,2F)).
void orc_swiglu(const float* v, int64_t M, int64_t F, float* h, uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t j = 0; j < F; ++j) {
      const float g = v[m * 2 * F + j];
      const float u = v[m * 2 * F + F + j];
      const float x = orc_silu_f32(g) * u;
      if (h) h[m * F + j] = x;
      if (out) out[m * F + j] = f32_to_bf16_rne(x);
    }
}

// ---------------------------------------------------------------------------
// The layer: x bf16 [M,K] -> rotate+quant -> GEMM with wq [N,K] -> epilogue.
// epilogue 0: y [M,N]; epilogue 1 (SwiGLU): N = 2F, y [M,F].
// Optional outputs (nullable): xq, sx, acc, v (fp32 values before bf16).
// Returns the number of int32 overflows (0 expected).
// ---------------------------------------------------------------------------
int64_t orc_linear(const uint16_t* x, int64_t M, int64_t K, const int8_t* wq, const float* sw, int64_t N,
                   const uint16_t* bias, int epilogue, uint16_t* y,
                   int8_t* xq_out, float* sx_out, int32_t* acc_out, float* v_out) {
  std::vector<int8_t> xq(size_t(M) * K);
  std::vector<float> sx(M);
  std::vector<int32_t> acc(size_t(M) * N);
  std::vector<float> v(size_t(M) * N);
  orc_rotate_quant_bf16(x, M, K, xq.data(), sx.data());
  const int64_t overflow = orc_gemm_s32(xq.data(), wq, M, N, K, acc.data());
  orc_epilogue(acc.data(), sx.data(), sw, bias, M, N, v.data(), epilogue == 0 ? y : nullptr);
  if (epilogue == 1) orc_swiglu(v.data(), M, N / 2, nullptr, y);
  if (xq_out) std::memcpy(xq_out, xq.data(), xq.size());
  if (sx_out) std::memcpy(sx_out, sx.data(), sx.size() * 4);
  if (acc_out) std::memcpy(acc_out, acc.data(), acc.size() * 4);
  if (v_out) std::memcpy(v_out, v.data(), v.size() * 4);
  return overflow;
}

// ---------------------------------------------------------------------------
// Step 9: FFN, y = down(rotquant(swiglu(gate_up(rotquant(x))))).
// w_gu [2F, K] (gate rows then up rows), w_down [K, F]. Optional outputs:
// h (bf16 SwiGLU output [M,F]), hq/sh (its rotated int8 codes and scales).
// ---------------------------------------------------------------------------
int64_t orc_ffn(const uint16_t* x, int64_t M, int64_t K, const int8_t* w_gu, const float* s_gu,
                const uint16_t* b_gu, int64_t F, const int8_t* w_down, const float* s_down,
                const uint16_t* b_down, uint16_t* y, uint16_t* h_out, int8_t* hq_out, float* sh_out) {
  std::vector<uint16_t> h(size_t(M) * F);
  int64_t overflow = orc_linear(x, M, K, w_gu, s_gu, 2 * F, b_gu, 1, h.data(),
                                nullptr, nullptr, nullptr, nullptr);
  std::vector<int8_t> hq(size_t(M) * F);
  std::vector<float> sh(M);
  overflow += orc_linear(h.data(), M, F, w_down, s_down, K, b_down, 0, y,
                         hq.data(), sh.data(), nullptr, nullptr);
  if (h_out) std::memcpy(h_out, h.data(), h.size() * 2);
  if (hq_out) std::memcpy(hq_out, hq.data(), hq.size());
  if (sh_out) std::memcpy(sh_out, sh.data(), sh.size() * 4);
  return overflow;
}

// ---------------------------------------------------------------------------
// LoRA merge into stored rotated int8 weights (h3-rs README, "What makes it
// fast": a LoRA is folded into the int8 weights once, at model load, by
// dequantizing, adding and requantizing). The stored codes are in the rotated basis, so the low-rank delta
// alpha * B A (B [N, r], A [r, K] in the model's basis) is rotated along K the
// same way: A_rot = A blockdiag(H/16), delta = alpha * B A_rot. Per element, in
// fp32 and in this order: d = sum over j ascending of B[n][j] * A_rot[j][k] as a
// fused multiply-add chain from 0; w = (float)q * s + alpha * d (two rounded
// products, one rounded add); then each row is requantized like a weight row
// (step 5 without the rotation). Updates q and s in place.
// ---------------------------------------------------------------------------
void orc_lora_merge(int8_t* q, float* s, int64_t N, int64_t K, const float* lora_a, const float* lora_b,
                    int64_t r, float alpha) {
  std::vector<float> a_rot(size_t(r) * K);
  orc_rotate_f32(lora_a, r, K, a_rot.data());
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    std::vector<float> w(K);
    for (int64_t k = 0; k < K; ++k) {
      float d = 0.0f;
      for (int64_t j = 0; j < r; ++j) d = std::fma(lora_b[n * r + j], a_rot[j * K + k], d);
      const float base = float(q[n * K + k]) * s[n];
      const float delta = alpha * d;
      w[k] = base + delta;
    }
    quantize_row(w.data(), K, q + n * K, s + n);
  }
}

// ---------------------------------------------------------------------------
// NVFP4, the hybrid checkpoints' native Blackwell format for the QKV and
// FFN-input projections (Minimax_h3_hybrid model card, "Checkpoints" and
// "Native NVFP4 projection benchmarks"; h3-rs README, model-file table:
// "NVFP4 (swizzled fp8 block scales)"). The pages do not spell the format out;
// this follows the public NVFP4 definition: e2m1 elements, one e4m3 scale per
// 16 consecutive elements along K, one fp32 scale per tensor. No rotation.
// ---------------------------------------------------------------------------

// e2m1: sign bit 3, two exponent bits (bias 1) and one mantissa bit;
// magnitudes of codes 0..7: 0, 0.5, 1, 1.5, 2, 3, 4, 6.
static const float kE2m1Mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

float orc_e2m1_value(uint8_t c) {
  const float v = kE2m1Mag[c & 7];
  return (c & 8) ? -v : v;
}

// Round to the nearest e2m1 magnitude, ties to the even code, saturating at 6;
// the sign is kept (a negative value that rounds to zero gives -0, code 8).
uint8_t orc_e2m1_rne(float x) {
  const float a = std::fabs(x);
  if (a >= 6.0f) return uint8_t(7 | (std::signbit(x) ? 8 : 0));  // saturate (the search would lose the
                                                                    // distances of huge values to rounding)
  int best = 0;
  float best_d = a;
  for (int c = 1; c < 8; ++c) {
    const float d = std::fabs(a - kE2m1Mag[c]);
    if (d < best_d || (d == best_d && (c & 1) == 0)) {
      best = c;
      best_d = d;
    }
  }
  return uint8_t(best | (std::signbit(x) ? 8 : 0));
}

// e4m3 (OCP FP8 E4M3, as the unsigned block scale): exponent bits 3-6 (bias
// 7), mantissa bits 0-2; exponent 0 is subnormal (m/8 * 2^-6); code 0x7f is NaN.
float orc_e4m3_value(uint8_t c) {
  const int e = (c >> 3) & 15, m = c & 7;
  const float mag = e == 0 ? std::ldexp(float(m) / 8.0f, -6) : std::ldexp(1.0f + float(m) / 8.0f, e - 7);
  return (c & 0x80) ? -mag : mag;
}

// Round a non-negative value to the nearest e4m3 value (ties to the even code),
// saturating at 448 (the largest finite value).
uint8_t orc_e4m3_rne_sat(float u) {
  if (u >= 448.0f) return 0x7e;  // saturate
  int best = 0;
  float best_d = std::fabs(u);
  for (int c = 1; c <= 0x7e; ++c) {
    const float d = std::fabs(u - orc_e4m3_value(uint8_t(c)));
    if (d < best_d || (d == best_d && (c & 1) == 0)) {
      best = c;
      best_d = d;
    }
  }
  return uint8_t(best);
}

// The tensor's encode scale: s_enc = RN(2688 / amax) (2688 = 448 * 6: the
// largest block scale times the largest element), 1 for an all-zero tensor,
// the largest finite float if the quotient overflows.
float orc_nvfp4_encode_scale(const float* x, int64_t n) {
  float amax = 0.0f;
  for (int64_t i = 0; i < n; ++i) amax = std::fmax(amax, std::fabs(x[i]));
  if (amax == 0.0f) return 1.0f;
  const float s = 2688.0f / amax;
  return std::isinf(s) ? 3.40282347e38f : s;
}

// Rows [rows, K] (K % 16 == 0) to NVFP4 with encode scale s_enc. Per block of 16
// consecutive elements of a row, in fp32 and in this order:
//   S   = e4m3_rne_sat(RN(RN(max|x| / 6) * s_enc))     (the block scale code)
//   enc = RN(s_enc / value(S))
//   q   = e2m1_rne(RN(x * enc))                        (0 for every element if S = 0)
// codes [rows, K/2]: element 2i in the low nibble of byte i; sf [rows, K/16].
void orc_nvfp4_quantize(const float* x, int64_t rows, int64_t K, float s_enc, uint8_t* codes, uint8_t* sf) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < K / 16; ++b) {
      const float* v = x + r * K + 16 * b;
      float bmax = 0.0f;
      for (int i = 0; i < 16; ++i) bmax = std::fmax(bmax, std::fabs(v[i]));
      const float t = bmax / 6.0f;
      const float u = t * s_enc;
      const uint8_t S = orc_e4m3_rne_sat(u);
      sf[r * (K / 16) + b] = S;
      const float Sv = orc_e4m3_value(S);
      uint8_t q[16];
      for (int i = 0; i < 16; ++i) {
        if (S == 0) {
          q[i] = 0;
          continue;
        }
        const float enc = s_enc / Sv;
        const float y = v[i] * enc;
        q[i] = orc_e2m1_rne(y);
      }
      for (int i = 0; i < 8; ++i) codes[r * (K / 2) + 8 * b + i] = uint8_t(q[2 * i] | (q[2 * i + 1] << 4));
    }
}

// The NVFP4 layer. acc[m][n] = sum over k of e2m1(a) S_a(block of k) e2m1(w)
// S_w(block of k), summed in fp64 (each block's 16 products are exact, so the
// sum is exact up to fp64 rounding of the block terms); mag[m][n] = the sum of
// the block terms' magnitudes (for the error bound of an fp32 accumulation).
// The output follows the int8 layer's epilogue with the per-tensor factor
// alpha = RN(1 / RN(s_enc_a * s_enc_w)) in place of sx * sw:
//   v = RN(RN((float)acc * alpha) + bias);  swiglu: h = silu(v_gate) * v_up.
// Rows [0, F) of w are the gate and [F, 2F) the up projection when swiglu is set.
// The NVFP4 epilogue on given fp32 accumulators acc32 [M, N] (v as above; with
// swiglu, N = 2F and the output is [M, F]).
void orc_nvfp4_epilogue(const float* acc32, int64_t M, int64_t N, float s_enc_a, float s_enc_w,
                        const uint16_t* bias, int swiglu, uint16_t* y) {
  const float alpha = 1.0f / (s_enc_a * s_enc_w);
  const int64_t NO = swiglu ? N / 2 : N;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    std::vector<float> v(N);
    for (int64_t n = 0; n < N; ++n) {
      float x = acc32[m * N + n] * alpha;
      if (bias) x = x + bf16_to_f32(bias[n]);
      v[n] = x;
    }
    for (int64_t j = 0; j < NO; ++j) y[m * NO + j] = f32_to_bf16_rne(swiglu ? orc_silu_f32(v[j]) * v[NO + j] : v[j]);
  }
}

void orc_nvfp4_linear(const uint8_t* ca, const uint8_t* sfa, float s_enc_a, int64_t M, int64_t K,
                      const uint8_t* cw, const uint8_t* sfw, float s_enc_w, int64_t N, const uint16_t* bias,
                      int swiglu, uint16_t* y, double* acc, double* mag) {
  const float alpha = 1.0f / (s_enc_a * s_enc_w);
  const int64_t KB = K / 16;
  const int64_t NO = swiglu ? N / 2 : N;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    std::vector<float> v(N);
    for (int64_t n = 0; n < N; ++n) {
      double total = 0.0, total_mag = 0.0;
      for (int64_t b = 0; b < KB; ++b) {
        double blk = 0.0;
        for (int i = 0; i < 16; ++i) {
          const int64_t k = 16 * b + i;
          const uint8_t qa = (ca[m * (K / 2) + k / 2] >> (4 * (k & 1))) & 15;
          const uint8_t qw = (cw[n * (K / 2) + k / 2] >> (4 * (k & 1))) & 15;
          blk += double(orc_e2m1_value(qa)) * double(orc_e2m1_value(qw));
        }
        const double term = blk * double(orc_e4m3_value(sfa[m * KB + b])) * double(orc_e4m3_value(sfw[n * KB + b]));
        total += term;
        total_mag += std::fabs(term);
      }
      if (acc) acc[m * N + n] = total;
      if (mag) mag[m * N + n] = total_mag;
      float x = float(total) * alpha;
      if (bias) x = x + bf16_to_f32(bias[n]);
      v[n] = x;
    }
    for (int64_t j = 0; j < NO; ++j) {
      const float out = swiglu ? orc_silu_f32(v[j]) * v[NO + j] : v[j];
      if (y) y[m * NO + j] = f32_to_bf16_rne(out);
    }
  }
}

// ---------------------------------------------------------------------------
// int8 attention (h3-rs README, "What makes it fast": the DiT attention runs an
// int8 Q.K^T / 16-bit P.V flash kernel). Per head h (columns h*D .. h*D+D-1 of
// the [S, ld] q, k, v matrices, bf16 bit patterns):
//   Q rows (one token of one head) are quantized like weight rows (steps 3-4:
//   s = max|x| / 127 in fp32, codes clamp(rne(x / s)));
//   K is quantized in blocks of 128 consecutive keys of a head: one scale per
//   block, s = max|x| / 127 over the block's keys and dimensions, codes
//   clamp(rne(x / s)) (steps 3-4 on the block read as one vector; the last
//   block of a sequence takes the keys that remain);
//   s_ij = (sum_d Qq_id Kq_jd) * qs_i * ks_b(j) / sqrt(D)   (exact integer dot product)
//   O_i  = sum_j softmax_j(s_i)_j V_j                        (float64)
// qq, kq [H, S, D] int8, qs [H, S], ks [H, ceil(S / 128)]; o [n, H*D] float64 for
// the query rows rows[0..n) (all S rows in order when rows is null).
// ---------------------------------------------------------------------------
void orc_attention_int8(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t S, int64_t D, int64_t H,
                        int64_t ld, int8_t* qq, float* qs, int8_t* kq, float* ks, const int64_t* rows, int64_t n,
                        double* o) {
  if (!rows) n = S;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < H * S; ++t) {
    const int64_t h = t / S, i = t % S;
    std::vector<float> row(D);
    for (int64_t d = 0; d < D; ++d) row[d] = bf16_to_f32(q[i * ld + h * D + d]);
    quantize_row(row.data(), D, qq + t * D, qs + t);
  }
  const int64_t kb = 128, nblk = (S + kb - 1) / kb;
#pragma omp parallel for schedule(static)
  for (int64_t u = 0; u < H * nblk; ++u) {
    const int64_t h = u / nblk, b = u % nblk, j0 = b * kb, nk = std::min(kb, S - j0);
    std::vector<float> blk(nk * D);
    for (int64_t j = 0; j < nk; ++j)
      for (int64_t d = 0; d < D; ++d) blk[j * D + d] = bf16_to_f32(k[(j0 + j) * ld + h * D + d]);
    quantize_row(blk.data(), nk * D, kq + (h * S + j0) * D, ks + u);
  }
  const double inv_sqrt_d = 1.0 / std::sqrt(double(D));
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t u = 0; u < H * n; ++u) {
    const int64_t h = u / n, r = u % n;
    const int64_t i = rows ? rows[r] : r;
    const int64_t t = h * S + i;
    std::vector<double> sc(S);
    double mx = -INFINITY;
    for (int64_t j = 0; j < S; ++j) {
      int64_t dot = 0;
      for (int64_t d = 0; d < D; ++d) dot += int64_t(qq[t * D + d]) * int64_t(kq[(h * S + j) * D + d]);
      sc[j] = double(dot) * double(qs[t]) * double(ks[h * nblk + j / kb]) * inv_sqrt_d;
      mx = std::fmax(mx, sc[j]);
    }
    double l = 0.0;
    for (int64_t j = 0; j < S; ++j) {
      sc[j] = std::exp(sc[j] - mx);
      l += sc[j];
    }
    for (int64_t d = 0; d < D; ++d) {
      double acc = 0.0;
      for (int64_t j = 0; j < S; ++j) acc += sc[j] * double(bf16_to_f32(v[j * ld + h * D + d]));
      o[r * H * D + h * D + d] = acc / l;
    }
  }
}

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

// Thread count of the following parallel loops (timing on one core); n <= 0 is ignored.
void orc_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

}  // extern "C"
