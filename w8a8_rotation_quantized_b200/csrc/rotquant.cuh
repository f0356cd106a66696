// Rotate + per-row quantize: the ConvRot Hadamard-256 rotation done warp-level
// inside the quantizer (h3-rs README, "What makes it fast"), followed by the
// per-row (per-token) absmax int8 quantization.
//
// One CTA per row. Warp w of W owns groups w, w + W, ... (GPW of them at most);
// in each group lane l holds elements 8l .. 8l+7 in registers, loaded with one
// 16-byte access (bf16) or two (fp32). The Walsh-Hadamard butterflies run in
// ascending index-bit order: bits 0-2 inside the lane, bits 3-7 across lanes
// through shuffles. Each butterfly is one fp32 add or subtract, so every
// rotated value has the same bits as the pairwise-tree sum of the explicit
// H/16 product. The 1/16 is applied to the scale instead of to every element:
// y16 = 16 y exactly, s16 = max|y16| / 127 = 16 s exactly, and y16 / s16 equals
// y / s, so the codes are identical. The whole row stays on chip until its
// absmax is known: one pass over HBM.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace h3q {

template <typename T>
struct RowLoader;

template <>
struct RowLoader<__nv_bfloat16> {
  static __device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 u = __ldcs(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};

template <>
struct RowLoader<float> {
  static __device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
    const float4 a = __ldcs(reinterpret_cast<const float4*>(p));
    const float4 b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
};

// Unnormalized Walsh-Hadamard transform of one 256-group held as 8 values per
// lane (element 8 * lane + r in v[r]); butterflies on index bits 0..7 in order.
__device__ __forceinline__ void fwht256_warp(float (&v)[8], int lane) {
#pragma unroll
  for (int b = 0; b < 3; ++b) {
    const int s = 1 << b;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      if ((r & s) == 0) {
        const float lo = v[r], hi = v[r + s];
        v[r] = __fadd_rn(lo, hi);
        v[r + s] = __fsub_rn(lo, hi);
      }
    }
  }
#pragma unroll
  for (int b = 0; b < 5; ++b) {
    const int m = 1 << b;
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const float p = __shfl_xor_sync(0xFFFFFFFFu, v[r], m);
      // lower partner: own + other; upper partner: other - own
      v[r] = upper ? __fsub_rn(p, v[r]) : __fadd_rn(v[r], p);
    }
  }
}

// Round-half-even of |t| < 2^22 to an integer, exactly: adding 1.5 * 2^23 lands
// in [2^23, 2^24) where the fp32 spacing is 1, so the add itself rounds t to the
// nearest integer, ties to even; the integer is read back from the bits.
__device__ __forceinline__ int rne_small(float t) {
  const float u = __fadd_rn(t, 12582912.0f);
  return __float_as_int(u) - 0x4B400000;
}

template <typename T, int GPW>
__global__ void __launch_bounds__(512) rotquant_kernel(const T* __restrict__ x, int64_t K, int8_t* __restrict__ q,
                                                       float* __restrict__ s_out) {
  const int64_t row = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int W = blockDim.x >> 5;
  const int G = static_cast<int>(K >> 8);
  const T* xr = x + row * K;
  int8_t* qr = q + row * K;

  float v[GPW][8];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < GPW; ++i) {
    const int g = warp + i * W;
    if (g < G) RowLoader<T>::load8(xr + g * 256 + lane * 8, v[i]);
  }
#pragma unroll
  for (int i = 0; i < GPW; ++i) {
    const int g = warp + i * W;
    if (g < G) {
      fwht256_warp(v[i], lane);
#pragma unroll
      for (int r = 0; r < 8; ++r) amax = fmaxf(amax, fabsf(v[i][r]));
    }
  }
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, m));

  __shared__ float warp_max[16];
  __shared__ float row_scale16;
  if (lane == 0) warp_max[warp] = amax;
  __syncthreads();
  if (threadIdx.x == 0) {
    float a = 0.0f;
    for (int w = 0; w < W; ++w) a = fmaxf(a, warp_max[w]);
    const float s16 = __fdiv_rn(a, 127.0f);
    row_scale16 = s16;
    s_out[row] = __fmul_rn(s16, 0.0625f);
  }
  __syncthreads();
  const float s16 = row_scale16;

#pragma unroll
  for (int i = 0; i < GPW; ++i) {
    const int g = warp + i * W;
    if (g < G) {
      uint32_t packed[2] = {0u, 0u};
      if (s16 != 0.0f) {
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          int c = rne_small(__fdiv_rn(v[i][r], s16));
          c = max(-127, min(127, c));
          packed[r >> 2] |= (static_cast<uint32_t>(c) & 0xFFu) << (8 * (r & 3));
        }
      }
      *reinterpret_cast<uint2*>(qr + g * 256 + lane * 8) = make_uint2(packed[0], packed[1]);
    }
  }
}

// Picks groups-per-warp (1..8) and warps-per-row (<= 16) with the least idle
// warp slots, preferring fewer groups per warp on ties.
inline void rotquant_shape(int G, int* gpw, int* warps) {
  int best_g = 8, best_w = (G + 7) / 8, best_waste = 1 << 30;
  for (int g = 1; g <= 8; ++g) {
    const int w = (G + g - 1) / g;
    if (w > 16) continue;
    const int waste = w * g - G;
    if (waste < best_waste) {
      best_waste = waste;
      best_g = g;
      best_w = w;
    }
  }
  *gpw = best_g;
  *warps = best_w;
}

template <typename T>
cudaError_t launch_rotquant(const T* x, int64_t rows, int64_t K, int8_t* q, float* s, cudaStream_t stream) {
  const int G = static_cast<int>(K / 256);
  int gpw, warps;
  rotquant_shape(G, &gpw, &warps);
  const dim3 grid(static_cast<unsigned>(rows)), block(32 * warps);
  switch (gpw) {
    case 1: rotquant_kernel<T, 1><<<grid, block, 0, stream>>>(x, K, q, s); break;
    case 2: rotquant_kernel<T, 2><<<grid, block, 0, stream>>>(x, K, q, s); break;
    case 3: rotquant_kernel<T, 3><<<grid, block, 0, stream>>>(x, K, q, s); break;
    case 4: rotquant_kernel<T, 4><<<grid, block, 0, stream>>>(x, K, q, s); break;
    case 5: rotquant_kernel<T, 5><<<grid, block, 0, stream>>>(x, K, q, s); break;
    case 6: rotquant_kernel<T, 6><<<grid, block, 0, stream>>>(x, K, q, s); break;
    case 7: rotquant_kernel<T, 7><<<grid, block, 0, stream>>>(x, K, q, s); break;
    default: rotquant_kernel<T, 8><<<grid, block, 0, stream>>>(x, K, q, s); break;
  }
  return cudaGetLastError();
}

}  // namespace h3q
