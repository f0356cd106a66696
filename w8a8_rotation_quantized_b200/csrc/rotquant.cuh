// Rotate + per-row quantize: the ConvRot Hadamard-256 rotation done inside the
// quantizer (h3-rs README, "What makes it fast"), followed by per-row
// (per-token) absmax int8 quantization.
//
// Layout: a half-warp (16 lanes) owns one 256-group; lane l of the half holds
// elements 16l .. 16l+15, loaded with 16-byte accesses (one half-warp reads 512
// contiguous bytes of bf16). Index bits 0-3 live in registers, bits 4-7 are the
// lane bits. The Walsh-Hadamard butterflies run in ascending bit order: bits
// 0-2 on packed fp32 pairs (v[r], v[r+8]) with the sm_100 two-wide fp32 adds,
// bit 3 inside each pair, bits 4-7 across lanes by shuffles. Every butterfly is
// one correctly rounded fp32 add or subtract, so each rotated value has the same
// bits as the pairwise-tree sum of the explicit H/16 product. The 1/16 moves to
// the scale: y16 = 16 y and s16 = max|y16| / 127 = 16 s exactly, and
// y16 / s16 = y / s, so the codes are unchanged.
//
// Quantization needs rne(RN(y / s)) for every element. Instead of a division per
// element, each row gets rs = RN(1 / s) once, and each quotient is formed by
// q0 = RN(y rs) refined twice with exact FMA residuals, e = y - q s,
// q <- RN(q + e rs) (Markstein, "Computation of elementary functions on the IBM
// RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990): after the first
// step q is within one ulp of y/s, and then the second step returns the
// correctly rounded quotient. Rows whose scale is below 2^-100 (never met in
// practice) fall back to IEEE division. The integer is read from the bits of
// q + 1.5*2^23, whose add rounds half to even; its low byte is the int8 code.
// |y| <= max|y| bounds y/s by 127 (1 + 2^-23), so no clamp is needed.
//
// Work item = R whole rows (all their groups), held on chip until each row's
// absmax is known: one pass over HBM. The grid is persistent and each block
// loads its next item while it finishes the current one.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace h3q {

constexpr int kRqMaxRows = 16;

template <typename T>
struct Raw;  // raw 16-byte words holding one lane's 16 input values

template <>
struct Raw<__nv_bfloat16> {
  static constexpr int kWords = 2;
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, uint4 (&w)[kWords]) {
    const uint4* s = reinterpret_cast<const uint4*>(p);
    w[0] = __ldcs(s);
    w[1] = __ldcs(s + 1);
  }
  // element 2i of a word is its low half, 2i+1 its high half
  static __device__ __forceinline__ void unpack(const uint4 (&w)[kWords], float2 (&p)[8]) {
    const uint32_t u[8] = {w[0].x, w[0].y, w[0].z, w[0].w, w[1].x, w[1].y, w[1].z, w[1].w};
    float v[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[2 * i] = __uint_as_float(u[i] << 16);
      v[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) p[r] = make_float2(v[r], v[r + 8]);
  }
};

template <>
struct Raw<float> {
  static constexpr int kWords = 4;
  static __device__ __forceinline__ void load(const float* p, uint4 (&w)[kWords]) {
    const uint4* s = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int i = 0; i < kWords; ++i) w[i] = __ldcs(s + i);
  }
  static __device__ __forceinline__ void unpack(const uint4 (&w)[kWords], float2 (&p)[8]) {
    float v[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[4 * i] = __uint_as_float(w[i].x);
      v[4 * i + 1] = __uint_as_float(w[i].y);
      v[4 * i + 2] = __uint_as_float(w[i].z);
      v[4 * i + 3] = __uint_as_float(w[i].w);
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) p[r] = make_float2(v[r], v[r + 8]);
  }
};

// Unnormalized Walsh-Hadamard transform of one 256-group; p[r] = (v[r], v[r+8])
// of lane hl's 16 elements 16 hl + r.
__device__ __forceinline__ void fwht256_halfwarp(float2 (&p)[8], int hl) {
  const float2 minus1 = make_float2(-1.0f, -1.0f);
#pragma unroll
  for (int b = 0; b < 3; ++b) {  // index bits 0, 1, 2: pairs (r, r + 2^b) of packed registers
    const int s = 1 << b;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      if ((r & s) == 0) {
        const float2 lo = p[r], hi = p[r + s];
        p[r] = __fadd2_rn(lo, hi);
        p[r + s] = __ffma2_rn(hi, minus1, lo);  // lo - hi, one rounding
      }
    }
  }
#pragma unroll
  for (int r = 0; r < 8; ++r) {  // index bit 3: inside each pair
    const float lo = p[r].x, hi = p[r].y;
    p[r] = make_float2(__fadd_rn(lo, hi), __fsub_rn(lo, hi));
  }
#pragma unroll
  for (int b = 0; b < 4; ++b) {  // index bits 4-7 = lane bits 0-3 of the half-warp
    const int m = 1 << b;
    const float sg = (hl & m) ? -1.0f : 1.0f;
    const float2 sign = make_float2(sg, sg);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const float2 other = make_float2(__shfl_xor_sync(0xFFFFFFFFu, p[r].x, m),
                                       __shfl_xor_sync(0xFFFFFFFFu, p[r].y, m));
      // lower partner: own + other; upper partner: other - own
      p[r] = __ffma2_rn(p[r], sign, other);
    }
  }
}

__device__ __forceinline__ uint32_t low_bytes4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  const uint32_t ab = __byte_perm(a, b, 0x0040);  // [a.b0, b.b0, -, -]
  const uint32_t cd = __byte_perm(c, d, 0x0040);
  return __byte_perm(ab, cd, 0x5410);
}

// Codes of one lane's 16 rotated values, as 4 words in natural element order.
__device__ __forceinline__ uint4 quantize16(const float2 (&p)[8], float s16, float rs, bool exact_div) {
  const float2 magic = make_float2(12582912.0f, 12582912.0f);
  uint32_t ux[8], uy[8];
  if (!exact_div) {
    const float2 r2 = make_float2(rs, rs), ns2 = make_float2(-s16, -s16);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      float2 q = __fmul2_rn(p[r], r2);
      float2 e = __ffma2_rn(q, ns2, p[r]);
      q = __ffma2_rn(e, r2, q);
      e = __ffma2_rn(q, ns2, p[r]);
      q = __ffma2_rn(e, r2, q);
      const float2 u = __fadd2_rn(q, magic);
      ux[r] = __float_as_uint(u.x);
      uy[r] = __float_as_uint(u.y);
    }
  } else {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const float qx = s16 != 0.0f ? __fdiv_rn(p[r].x, s16) : 0.0f;
      const float qy = s16 != 0.0f ? __fdiv_rn(p[r].y, s16) : 0.0f;
      ux[r] = __float_as_uint(__fadd_rn(qx, 12582912.0f));
      uy[r] = __float_as_uint(__fadd_rn(qy, 12582912.0f));
    }
  }
  return make_uint4(low_bytes4(ux[0], ux[1], ux[2], ux[3]), low_bytes4(ux[4], ux[5], ux[6], ux[7]),
                    low_bytes4(uy[0], uy[1], uy[2], uy[3]), low_bytes4(uy[4], uy[5], uy[6], uy[7]));
}

// GPS = groups per half-warp slot and item. The host picks R rows per item and
// W <= 32 / GPS warps so that R * G <= 2 * W * GPS.
template <typename T, int GPS>
__global__ void __launch_bounds__(1024 / GPS) rotquant_kernel(const T* __restrict__ x, int64_t M, int K, int R,
                                                        int64_t items, int8_t* __restrict__ q,
                                                        float* __restrict__ s_out) {
  using L = Raw<T>;
  __shared__ uint32_t row_amax[3][kRqMaxRows];
  __shared__ float row_s16[kRqMaxRows], row_rs[kRqMaxRows];
  const int hl = threadIdx.x & 15;
  const int slot = threadIdx.x >> 4;
  const int HW = blockDim.x >> 4;
  const int G = K >> 8;

  int rr[GPS], gg[GPS];
  bool act[GPS];
#pragma unroll
  for (int t = 0; t < GPS; ++t) {
    const int i = t * HW + slot;
    act[t] = i < R * G;
    rr[t] = act[t] ? i / G : 0;
    gg[t] = act[t] ? i - rr[t] * G : 0;
  }
  if (threadIdx.x < 3 * kRqMaxRows) (&row_amax[0][0])[threadIdx.x] = 0u;
  __syncthreads();

  auto load_item = [&](int64_t item, uint4 (&raw)[GPS][L::kWords]) {
#pragma unroll
    for (int t = 0; t < GPS; ++t) {
      const int64_t row = item * R + rr[t];
      if (act[t] && row < M) {
        L::load(x + row * K + gg[t] * 256 + hl * 16, raw[t]);
      } else {
#pragma unroll
        for (int w = 0; w < L::kWords; ++w) raw[t][w] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  };

  uint4 raw[GPS][L::kWords];
  int64_t item = blockIdx.x;
  if (item < items) load_item(item, raw);
  for (int it = 0; item < items; item += gridDim.x, ++it) {
    float2 p[GPS][8];
#pragma unroll
    for (int t = 0; t < GPS; ++t) L::unpack(raw[t], p[t]);
    const int64_t next = item + gridDim.x;
    if (next < items) load_item(next, raw);  // in flight while this item is finished
    const int buf = it % 3;
    if (threadIdx.x < kRqMaxRows) row_amax[(it + 1) % 3][threadIdx.x] = 0u;

#pragma unroll
    for (int t = 0; t < GPS; ++t) {
      fwht256_halfwarp(p[t], hl);
      float m = 0.0f;
#pragma unroll
      for (int r = 0; r < 8; ++r) m = fmaxf(m, fmaxf(fabsf(p[t][r].x), fabsf(p[t][r].y)));
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
      const int64_t row = item * R + rr[t];
      if (hl == 0 && act[t] && row < M) atomicMax(&row_amax[buf][rr[t]], __float_as_uint(m));
    }
    __syncthreads();
    if (threadIdx.x < R) {
      const int64_t row = item * R + threadIdx.x;
      const float a = __uint_as_float(row_amax[buf][threadIdx.x]);
      const float s16 = __fdiv_rn(a, 127.0f);
      row_s16[threadIdx.x] = s16;
      row_rs[threadIdx.x] = s16 >= 0x1p-100f ? __frcp_rn(s16) : 0.0f;
      if (row < M) s_out[row] = __fmul_rn(s16, 0.0625f);
    }
    __syncthreads();
#pragma unroll
    for (int t = 0; t < GPS; ++t) {
      const int64_t row = item * R + rr[t];
      const float s16 = row_s16[rr[t]];
      const float rs = row_rs[rr[t]];
      const uint4 codes = quantize16(p[t], s16, rs, rs == 0.0f);
      if (act[t] && row < M)
        *reinterpret_cast<uint4*>(q + row * K + gg[t] * 256 + hl * 16) = codes;
    }
  }
}

struct RqShape {
  int gps, warps, rows;
};

// Rows per item, warps and groups per slot for a row of G groups: no idle slots
// where possible, 256-1024 threads, fewest groups per slot.
inline RqShape rotquant_shape(int G) {
  RqShape best{0, 0, 0};
  double best_score = 1e30;
  for (int gps = 1; gps <= 4; ++gps)
    for (int R = 1; R <= kRqMaxRows; ++R) {
      const int slots = R * G;
      const int W = (slots + 2 * gps - 1) / (2 * gps);
      if (W > 32 / gps) continue;  // the kernel is built for at most 1024 / gps threads
      const double waste = double(2 * W * gps - slots) / slots;
      const int threads = 32 * W;
      const double score = waste * 10.0 + (threads < 256 ? (256 - threads) / 256.0 : 0.0) + 0.05 * gps +
                           0.001 * R;
      if (score < best_score) {
        best_score = score;
        best = {gps, W, R};
      }
    }
  return best;
}

template <typename T, int GPS>
cudaError_t launch_rotquant_t(const T* x, int64_t rows, int64_t K, int8_t* q, float* s, const RqShape& sh,
                              cudaStream_t stream) {
  // blocks per SM for each block size, queried once (device 0 .. 15)
  static int occ_cache[16][33] = {};
  static int sm_cache[16] = {};
  const int threads = 32 * sh.warps;
  int dev = 0;
  cudaGetDevice(&dev);
  dev &= 15;
  if (sm_cache[dev] == 0) cudaDeviceGetAttribute(&sm_cache[dev], cudaDevAttrMultiProcessorCount, dev);
  if (occ_cache[dev][sh.warps] == 0) {
    int occ = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, rotquant_kernel<T, GPS>, threads, 0);
    occ_cache[dev][sh.warps] = occ < 1 ? 1 : occ;
  }
  const int sms = sm_cache[dev], occ = occ_cache[dev][sh.warps];
  const int64_t items = (rows + sh.rows - 1) / sh.rows;
  const int64_t cap = int64_t(sms) * occ;
  const unsigned grid = static_cast<unsigned>(items < cap ? items : cap);
  rotquant_kernel<T, GPS><<<grid, threads, 0, stream>>>(x, rows, static_cast<int>(K), sh.rows, items, q, s);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_rotquant(const T* x, int64_t rows, int64_t K, int8_t* q, float* s, cudaStream_t stream) {
  const RqShape sh = rotquant_shape(static_cast<int>(K / 256));
  switch (sh.gps) {
    case 1: return launch_rotquant_t<T, 1>(x, rows, K, q, s, sh, stream);
    case 2: return launch_rotquant_t<T, 2>(x, rows, K, q, s, sh, stream);
    case 3: return launch_rotquant_t<T, 3>(x, rows, K, q, s, sh, stream);
    default: return launch_rotquant_t<T, 4>(x, rows, K, q, s, sh, stream);
  }
}

}  // namespace h3q
