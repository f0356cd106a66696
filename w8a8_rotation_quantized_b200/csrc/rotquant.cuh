// Rotate + per-row quantize: the ConvRot Hadamard-256 rotation done inside the
// quantizer (h3-rs README, "What makes it fast"), followed by per-row
// (per-token) absmax int8 quantization.
//
// Data movement: a persistent grid; in each block one producer thread streams
// work items (R whole rows, contiguous in memory) into a ring of shared-memory
// stages with 1D bulk copies (cp.async.bulk, completion on an mbarrier), so
// several items are in flight per block while the consumer warps work. Each row
// is read from HBM once and its codes written once.
//
// Work split: a half-warp (16 lanes) of the consumers owns one 256-group of a
// row. Lane l of the half reads two 16-byte runs of the group from shared
// memory: elements 8l .. 8l+7 and 128+8l .. 128+8l+7 (bank-conflict free), kept
// as packed pairs p[r] = (v[r], v[r+8]) of element 8l+r and 128+8l+r. Index bits
// 0-2 are register bits, bits 3-6 the lane bits, bit 7 the pair half.
//
// Rotation: the unnormalized Walsh-Hadamard butterflies in ascending index-bit
// order: bits 0-2 on packed pairs with the sm_100 two-wide fp32 add, bits 3-6
// across lanes by shuffles (a fused multiply by +-1 and add, one rounding),
// bit 7 inside each pair. Every butterfly is one correctly rounded fp32 add or
// subtract, so each rotated value has the same bits as the pairwise-tree sum of
// the explicit H/16 product. The 1/16 moves to the scale: y16 = 16 y and
// s16 = max|y16| / 127 = 16 s exactly, and y16 / s16 = y / s, so the codes are
// unchanged.
//
// Quantization needs rne(RN(y / s)) per element. Each row gets rs = RN(1/s)
// once; each quotient is q0 = RN(y rs) refined twice with exact FMA residuals,
// e = y - q s, q <- RN(q + e rs) (Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1),
// 1990): after the first step q is within one ulp of y/s, and the second step
// returns the correctly rounded quotient. Rows whose scale is below 2^-100
// (never met in practice) use IEEE division. The integer is read from the bits
// of q + 1.5*2^23, whose add rounds half to even; its low byte is the int8 code.
// |y| <= max|y| bounds y/s by 127 (1 + 2^-23), so no clamp is needed.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "ptx_sm100.cuh"

namespace h3q {

constexpr int kRqMaxRows = 16;

template <typename T>
struct Lane16;  // one lane's 16 values of a group: runs [8l, 8l+8) and [128+8l, 128+8l+8)

template <>
struct Lane16<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* grp, int hl, float2 (&p)[8]) {
    const uint4 a = *reinterpret_cast<const uint4*>(grp + 8 * hl);
    const uint4 b = *reinterpret_cast<const uint4*>(grp + 128 + 8 * hl);
    const uint32_t ua[4] = {a.x, a.y, a.z, a.w}, ub[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // element 2i of a word is its low half
      p[2 * i] = make_float2(__uint_as_float(ua[i] << 16), __uint_as_float(ub[i] << 16));
      p[2 * i + 1] = make_float2(__uint_as_float(ua[i] & 0xFFFF0000u), __uint_as_float(ub[i] & 0xFFFF0000u));
    }
  }
};

template <>
struct Lane16<float> {
  static __device__ __forceinline__ void load(const float* grp, int hl, float2 (&p)[8]) {
    const float4* a = reinterpret_cast<const float4*>(grp + 8 * hl);
    const float4* b = reinterpret_cast<const float4*>(grp + 128 + 8 * hl);
    const float4 a0 = a[0], a1 = a[1], b0 = b[0], b1 = b[1];
    p[0] = make_float2(a0.x, b0.x); p[1] = make_float2(a0.y, b0.y);
    p[2] = make_float2(a0.z, b0.z); p[3] = make_float2(a0.w, b0.w);
    p[4] = make_float2(a1.x, b1.x); p[5] = make_float2(a1.y, b1.y);
    p[6] = make_float2(a1.z, b1.z); p[7] = make_float2(a1.w, b1.w);
  }
};

// Unnormalized Walsh-Hadamard transform of one 256-group held by a half-warp.
__device__ __forceinline__ void fwht256_halfwarp(float2 (&p)[8], int hl) {
  const float2 minus1 = make_float2(-1.0f, -1.0f);
#pragma unroll
  for (int b = 0; b < 3; ++b) {  // index bits 0, 1, 2: packed registers r and r + 2^b
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
  for (int b = 0; b < 4; ++b) {  // index bits 3-6 = lane bits 0-3 of the half-warp
    const int m = 1 << b;
    const float sg = (hl & m) ? -1.0f : 1.0f;
    const float2 sign = make_float2(sg, sg);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const float2 other = make_float2(__shfl_xor_sync(0xFFFFFFFFu, p[r].x, m),
                                       __shfl_xor_sync(0xFFFFFFFFu, p[r].y, m));
      p[r] = __ffma2_rn(p[r], sign, other);  // lower lane: own + other; upper lane: other - own
    }
  }
#pragma unroll
  for (int r = 0; r < 8; ++r) {  // index bit 7: the two halves of each pair
    const float lo = p[r].x, hi = p[r].y;
    p[r] = make_float2(__fadd_rn(lo, hi), __fsub_rn(lo, hi));
  }
}

// max of three fp32 values (sm_100 three-input max).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint32_t low_bytes4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  const uint32_t ab = __byte_perm(a, b, 0x0040);  // [a.b0, b.b0, -, -]
  const uint32_t cd = __byte_perm(c, d, 0x0040);
  return __byte_perm(ab, cd, 0x5410);
}

// Codes of one lane's 16 rotated values: .x/.y = elements 8l..8l+7,
// .z/.w = elements 128+8l .. 128+8l+7.
__device__ __forceinline__ uint4 quantize16(const float2 (&p)[8], float s16, float rs) {
  const float2 magic = make_float2(12582912.0f, 12582912.0f);
  uint32_t ux[8], uy[8];
  if (rs != 0.0f) {
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

struct RqArgs {
  int64_t M;          // rows
  int K;              // row length (multiple of 256)
  int R;              // rows per work item
  int64_t items;      // ceil(M / R)
  int stages;         // shared-memory ring depth
  uint32_t stage_bytes;
  int8_t* q;
  float* s_out;
  uint64_t wait_limit_ns;
};

// Warp 0 is the producer; warps 1..W are consumers, W * 2 * GPS >= R * (K / 256).
// MINB = 2 builds the kernel for blocks of at most 736 threads, two per SM.
template <typename T, int GPS, int MINB>
__global__ void __launch_bounds__(MINB == 2 ? 736 : 1024 / GPS + 32, MINB)
    rotquant_kernel(const T* __restrict__ x, const RqArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + size_t(a.stages) * a.stage_bytes);
  uint64_t* empty = full + a.stages;
  uint32_t* row_amax = reinterpret_cast<uint32_t*>(empty + a.stages);  // [3][kRqMaxRows]
  float* row_s16 = reinterpret_cast<float*>(row_amax + 3 * kRqMaxRows);
  float* row_rs = row_s16 + kRqMaxRows;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(row_rs + kRqMaxRows);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_cons = blockDim.x - 32;
  const int G = a.K >> 8;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], n_cons);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (threadIdx.x < 3 * kRqMaxRows) row_amax[threadIdx.x] = 0u;
  __syncthreads();

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int64_t item = blockIdx.x; item < a.items; item += gridDim.x) {
        if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, a.wait_limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        const int64_t row0 = item * a.R;
        const int64_t nrows = (a.M - row0) < a.R ? (a.M - row0) : a.R;
        const uint32_t bytes = static_cast<uint32_t>(nrows * a.K * int64_t(sizeof(T)));
        mbar_arrive_expect_tx(&full[stage], bytes);
        bulk_load(smem + size_t(stage) * a.stage_bytes, x + row0 * a.K, bytes, &full[stage], pol);
        ++issued;
        if (++stage == a.stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {  // drain this block's own copies still in flight (bounded)
        for (int s = 0; s < a.stages; ++s) {
          if (issued <= s) continue;
          const long last = ((issued - 1 - s) / a.stages) * a.stages + s;
          mbar_wait_bounded(&full[s], static_cast<uint32_t>((last / a.stages) & 1), a.wait_limit_ns, nullptr);
        }
      }
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int c = threadIdx.x - 32;
  const int hl = c & 15;
  const int slot = c >> 4;
  const int HW = n_cons >> 4;
  int rr[GPS], gg[GPS];
  bool act[GPS];
#pragma unroll
  for (int t = 0; t < GPS; ++t) {
    const int i = t * HW + slot;
    act[t] = i < a.R * G;
    rr[t] = act[t] ? i / G : 0;
    gg[t] = act[t] ? i - rr[t] * G : 0;
  }

  int stage = 0;
  uint32_t phase = 0;
  for (int64_t item = blockIdx.x, it = 0; item < a.items; item += gridDim.x, ++it) {
    mbar_wait_bounded(&full[stage], phase, a.wait_limit_ns, abort_flag);  // on expiry: garbage, no hang
    const T* tile = reinterpret_cast<const T*>(smem + size_t(stage) * a.stage_bytes);
    float2 p[GPS][8];
#pragma unroll
    for (int t = 0; t < GPS; ++t) Lane16<T>::load(tile + rr[t] * a.K + gg[t] * 256, hl, p[t]);
    mbar_arrive(&empty[stage]);  // this thread's reads of the stage are done
    if (++stage == a.stages) {
      stage = 0;
      phase ^= 1u;
    }
    const int buf = static_cast<int>(it % 3);
    if (c < kRqMaxRows) row_amax[((it + 1) % 3) * kRqMaxRows + c] = 0u;

    const int64_t row0 = item * a.R;
#pragma unroll
    for (int t = 0; t < GPS; ++t) {
      fwht256_halfwarp(p[t], hl);
      float m = 0.0f;
#pragma unroll
      for (int r = 0; r < 8; ++r) m = fmax3(m, fabsf(p[t][r].x), fabsf(p[t][r].y));
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
      if (hl == 0 && act[t] && row0 + rr[t] < a.M)
        atomicMax(&row_amax[buf * kRqMaxRows + rr[t]], __float_as_uint(m));
    }
    named_barrier(1, n_cons);
    if (c < a.R) {
      const float am = __uint_as_float(row_amax[buf * kRqMaxRows + c]);
      const float s16 = __fdiv_rn(am, 127.0f);
      row_s16[c] = s16;
      row_rs[c] = s16 >= 0x1p-100f ? __frcp_rn(s16) : 0.0f;
      if (row0 + c < a.M) a.s_out[row0 + c] = __fmul_rn(s16, 0.0625f);
    }
    named_barrier(1, n_cons);
#pragma unroll
    for (int t = 0; t < GPS; ++t) {
      const int64_t row = row0 + rr[t];
      const uint4 codes = quantize16(p[t], row_s16[rr[t]], row_rs[rr[t]]);
      if (act[t] && row < a.M) {
        int8_t* dst = a.q + row * a.K + gg[t] * 256 + 8 * hl;
        *reinterpret_cast<uint2*>(dst) = make_uint2(codes.x, codes.y);
        *reinterpret_cast<uint2*>(dst + 128) = make_uint2(codes.z, codes.w);
      }
    }
  }
}

struct RqShape {
  int gps, warps, rows;  // groups per half-warp slot, consumer warps, rows per item
};

// Rows per item, consumer warps and groups per slot for a row of G groups: no
// idle slots where possible, at least 256 consumer threads, fewest groups per
// slot.
inline RqShape rotquant_shape(int G) {
  RqShape best{0, 0, 0};
  double best_score = 1e30;
  for (int gps = 1; gps <= 4; ++gps)
    for (int R = 1; R <= kRqMaxRows; ++R) {
      const int slots = R * G;
      const int W = (slots + 2 * gps - 1) / (2 * gps);
      // consumers of a block built for 1024 / gps + 32 threads, at most 1024 with the producer
      if (W > 32 / gps || W > 31) continue;
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

inline size_t rotquant_smem_bytes(int stages, uint32_t stage_bytes) {
  return size_t(stages) * stage_bytes + 2 * sizeof(uint64_t) * stages + (3 * kRqMaxRows + 2 * kRqMaxRows) * 4 +
         16;
}

template <typename T, int GPS, int MINB>
cudaError_t launch_rotquant_t(const T* x, int64_t rows, int64_t K, int8_t* q, float* s, const RqShape& sh,
                              uint64_t wait_limit_ns, cudaStream_t stream) {
  RqArgs a;
  a.M = rows;
  a.K = static_cast<int>(K);
  a.R = sh.rows;
  a.items = (rows + sh.rows - 1) / sh.rows;
  a.stage_bytes = static_cast<uint32_t>(int64_t(sh.rows) * K * int64_t(sizeof(T)));
  // about 64 KB of loads in flight per block, 2 to 8 stages, under 110 KB so two blocks fit an SM
  int stages = static_cast<int>((65536 + a.stage_bytes - 1) / a.stage_bytes);
  stages = stages < 2 ? 2 : (stages > 8 ? 8 : stages);
  while (stages > 2 && rotquant_smem_bytes(stages, a.stage_bytes) > 110 * 1024) --stages;
  a.stages = stages;
  a.q = q;
  a.s_out = s;
  a.wait_limit_ns = wait_limit_ns;
  const size_t smem = rotquant_smem_bytes(stages, a.stage_bytes);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  const int threads = 32 * (sh.warps + 1);

  static int sm_count[16] = {};
  static bool attr_set[16] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  dev &= 15;
  if (sm_count[dev] == 0) cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
  if (!attr_set[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(rotquant_kernel<T, GPS, MINB>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  int occ = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, rotquant_kernel<T, GPS, MINB>, threads, smem);
  if (occ < 1) occ = 1;
  const int64_t cap = int64_t(sm_count[dev]) * occ;
  const unsigned grid = static_cast<unsigned>(a.items < cap ? a.items : cap);
  rotquant_kernel<T, GPS, MINB><<<grid, threads, smem, stream>>>(x, a);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_rotquant(const T* x, int64_t rows, int64_t K, int8_t* q, float* s, uint64_t wait_limit_ns,
                            cudaStream_t stream) {
  const RqShape sh = rotquant_shape(static_cast<int>(K / 256));
  const bool two_per_sm = 32 * (sh.warps + 1) <= 736;
  switch (sh.gps) {
    case 1:
      return two_per_sm ? launch_rotquant_t<T, 1, 2>(x, rows, K, q, s, sh, wait_limit_ns, stream)
                        : launch_rotquant_t<T, 1, 1>(x, rows, K, q, s, sh, wait_limit_ns, stream);
    case 2: return launch_rotquant_t<T, 2, 1>(x, rows, K, q, s, sh, wait_limit_ns, stream);
    case 3: return launch_rotquant_t<T, 3, 1>(x, rows, K, q, s, sh, wait_limit_ns, stream);
    default: return launch_rotquant_t<T, 4, 1>(x, rows, K, q, s, sh, wait_limit_ns, stream);
  }
}

}  // namespace h3q
