// Rotate + per-row quantize: the ConvRot Hadamard-256 rotation done inside the
// quantizer (h3-rs README, "What makes it fast"), followed by per-row
// (per-token) absmax int8 quantization.
//
// Data movement: a persistent grid; in each block one producer thread streams
// work items (R whole rows, contiguous in memory) into a ring of shared-memory
// stages with 1D bulk copies (cp.async.bulk, completion on an mbarrier), so
// several items are in flight per block while the consumer warps work. Each row
// is read from HBM once and its codes are written once.
//
// Rotation of one 256-group by a half-warp (16 lanes), seen as a 16 x 16 matrix
// X[a][b] = x[16a + b]:
//   phase A  lane a holds row a (16 contiguous elements) and applies the
//            butterflies of index bits 0-3 in registers;
//   transpose through a per-half-warp shared-memory scratch (fp32, chunks
//            swizzled so both the row writes and the column reads are free of
//            bank conflicts);
//   phase B  lane b holds column b and applies the butterflies of bits 4-7.
// Each phase keeps its 16 values as packed pairs (v[r], v[r+8]) and runs three
// stages on the sm_100 two-wide fp32 add and the fourth inside each pair. The
// bits are processed in ascending order and every butterfly is one correctly
// rounded fp32 add or subtract, so each rotated value has the same bits as the
// pairwise-tree sum of the explicit H/16 product. No shuffle is needed. The
// 1/16 moves to the scale: y16 = 16 y and s16 = max|y16| / 127 = 16 s exactly,
// and y16 / s16 = y / s, so the codes are unchanged.
//
// Quantization needs rne(RN(y / s)) per element. Each row gets rs = RN(1/s)
// once; each quotient is q0 = RN(y rs) refined twice with exact FMA residuals,
// e = y - q s, q <- RN(q + e rs) (Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1),
// 1990): after the first step q is within one ulp of y/s, and the second step
// returns the correctly rounded quotient. Rows whose scale is below 2^-100 are
// first rescaled by 2^64 (exact). The integer is read from the bits
// of q + 1.5*2^23, whose add rounds half to even; its low byte is the int8 code.
// |y| <= max|y| bounds y/s by 127 (1 + 2^-23), so no clamp is needed. The codes
// of a column are scattered bytes of the group; they pass through the slot's
// shared buffer and leave as one 16-byte store per lane.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "ptx_sm100.cuh"

namespace h3q {

constexpr int kRqMaxRows = 16;
constexpr int kRqSlotBytes = 1024 + 64;  // per half-warp: 16 x 16 fp32 scratch + 64 B so slots shift banks by 16

template <typename T>
struct Row16;  // lane a's 16 contiguous elements 16a .. 16a+15 of a group, as pairs (v[r], v[r+8])

template <>
struct Row16<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* grp, int a, float2 (&p)[8]) {
    const uint4* row = reinterpret_cast<const uint4*>(grp + 16 * a);
    const uint4 lo = row[0], hi = row[1];  // elements 0-7 and 8-15
    const uint32_t ul[4] = {lo.x, lo.y, lo.z, lo.w}, uh[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // element 2i of a word is its low half
      p[2 * i] = make_float2(__uint_as_float(ul[i] << 16), __uint_as_float(uh[i] << 16));
      p[2 * i + 1] = make_float2(__uint_as_float(ul[i] & 0xFFFF0000u), __uint_as_float(uh[i] & 0xFFFF0000u));
    }
  }
};

template <>
struct Row16<float> {
  static __device__ __forceinline__ void load(const float* grp, int a, float2 (&p)[8]) {
    const float4* row = reinterpret_cast<const float4*>(grp + 16 * a);
    const float4 c0 = row[0], c1 = row[1], c2 = row[2], c3 = row[3];
    p[0] = make_float2(c0.x, c2.x); p[1] = make_float2(c0.y, c2.y);
    p[2] = make_float2(c0.z, c2.z); p[3] = make_float2(c0.w, c2.w);
    p[4] = make_float2(c1.x, c3.x); p[5] = make_float2(c1.y, c3.y);
    p[6] = make_float2(c1.z, c3.z); p[7] = make_float2(c1.w, c3.w);
  }
};

// Unnormalized 16-point Walsh-Hadamard transform of v[0..15] held as
// p[r] = (v[r], v[r+8]): bits 0-2 on packed pairs, then bit 3 inside each pair.
__device__ __forceinline__ void fwht16(float2 (&p)[8]) {
  const float2 minus1 = make_float2(-1.0f, -1.0f);
#pragma unroll
  for (int b = 0; b < 3; ++b) {
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
  for (int r = 0; r < 8; ++r) {
    const float lo = p[r].x, hi = p[r].y;
    p[r] = make_float2(__fadd_rn(lo, hi), __fsub_rn(lo, hi));
  }
}

// Scratch layout: row a holds 16 fp32 values; its 16-byte chunk k sits at chunk
// position k ^ ((a >> 1) & 3) of the row.
// Rotates one group: on return, p[r] = (y16[16 r + b], y16[16 (r + 8) + b]) for
// this lane's column b = hl. `scratch` is the half-warp's private fp32 area.
template <typename T>
__device__ __forceinline__ void rotate_group(const T* grp, int hl, float* scratch, float2 (&p)[8]) {
  Row16<T>::load(grp, hl, p);
  fwht16(p);  // index bits 0-3
  const int sw = (hl >> 1) & 3;
#pragma unroll
  for (int k = 0; k < 4; ++k) {  // row hl, chunk k = elements 4k .. 4k+3
    const float4 c = k < 2 ? make_float4(p[4 * k].x, p[4 * k + 1].x, p[4 * k + 2].x, p[4 * k + 3].x)
                           : make_float4(p[4 * k - 8].y, p[4 * k - 7].y, p[4 * k - 6].y, p[4 * k - 5].y);
    *reinterpret_cast<float4*>(scratch + 16 * hl + 4 * (k ^ sw)) = c;
  }
  __syncwarp();
  // column hl: row r's element sits at 16 r + 4 ((hl >> 2) ^ (r >> 1) & 3) + (hl & 3);
  // four base pointers (one per value of r >> 1 & 3) leave an immediate offset per row
  const float* col = scratch + (hl & 3);
  const int x = hl >> 2;
  const float* b0 = col + 4 * (x & 3);
  const float* b1 = col + 4 * ((x ^ 1) & 3);
  const float* b2 = col + 4 * ((x ^ 2) & 3);
  const float* b3 = col + 4 * ((x ^ 3) & 3);
  const float* base[4] = {b0, b1, b2, b3};
#pragma unroll
  for (int r = 0; r < 8; ++r) p[r] = make_float2(base[(r >> 1) & 3][16 * r], base[((r + 8) >> 1) & 3][16 * (r + 8)]);
  __syncwarp();  // the scratch is rewritten next (codes or the next group)
  fwht16(p);     // index bits 4-7
}

// max of three fp32 values (sm_100 three-input max).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Per-row quotient constants: y / s is formed as (y f) / (s f) with f = 2^64 for
// rows whose scale is below 2^-100 (an exact rescaling that keeps 1 / (s f) in
// range), f = 1 otherwise; rs = RN(1 / (s f)), and rs = 0 for an all-zero row
// (whose codes are then 0).
struct RowQuot {
  float f, sf, rs;
};

// s = RN(a / 127) for a >= 0: RN(a RN(1/127)) and one FMA correction step, which
// returns the IEEE quotient for every non-negative float (an exhaustive host check
// over all 2^31 - 2^23 finite positive patterns), in three dependent operations.
__device__ __forceinline__ float div127(float a) {
  constexpr float c = 1.0f / 127.0f;
  const float q0 = __fmul_rn(a, c);
  return __fmaf_rn(__fmaf_rn(-q0, 127.0f, a), c, q0);
}

__device__ __forceinline__ RowQuot row_quotient(float s16) {
  RowQuot r;
  r.f = s16 < 0x1p-100f ? 0x1p64f : 1.0f;
  r.sf = __fmul_rn(s16, r.f);
  r.rs = s16 != 0.0f ? __frcp_rn(r.sf) : 0.0f;
  return r;
}

// int8 codes rne(y16 / s16) of this lane's column hl, written as bytes into the
// group's 256-byte code buffer at element positions 16 r + hl and 16 (r + 8) + hl.
// kRescaled: the row's f is 2^64 (scale below 2^-100); otherwise f = 1 and the exact
// rescaling is skipped.
template <bool kRescaled>
__device__ __forceinline__ void quantize_column(const float2 (&p)[8], const RowQuot& rq, int hl,
                                                uint8_t* codes) {
  const float2 magic = make_float2(12582912.0f, 12582912.0f);
  const float2 f2 = make_float2(rq.f, rq.f), r2 = make_float2(rq.rs, rq.rs), ns2 = make_float2(-rq.sf, -rq.sf);
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const float2 y = kRescaled ? __fmul2_rn(p[r], f2) : p[r];  // exact
    float2 q = __fmul2_rn(y, r2);
    float2 e = __ffma2_rn(q, ns2, y);
    q = __ffma2_rn(e, r2, q);
    e = __ffma2_rn(q, ns2, y);
    q = __ffma2_rn(e, r2, q);
    const float2 u = __fadd2_rn(q, magic);
    codes[16 * r + hl] = static_cast<uint8_t>(__float_as_uint(u.x));
    codes[16 * (r + 8) + hl] = static_cast<uint8_t>(__float_as_uint(u.y));
  }
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

struct RqShape {
  int gps, warps, rows, stages;  // groups per half-warp slot, consumer warps, rows per item, ring depth
  bool small;                    // built for three blocks per SM
};

inline size_t rotquant_smem_bytes(int stages, uint32_t stage_bytes, int warps) {
  return size_t(stages) * stage_bytes + size_t(2 * warps) * kRqSlotBytes + 2 * sizeof(uint64_t) * stages +
         3 * kRqMaxRows * 4 + 16;
}

// Warp 0 is the producer; warps 1..W are consumers with 2W half-warp slots, each
// taking GPS groups per item: 2 * W * GPS >= R * (K / 256). SMALL builds for
// blocks of at most 16 warps, three per SM (40 registers); otherwise up to 32
// warps, one per SM.
template <typename T, int GPS, bool SMALL>
__global__ void __launch_bounds__(SMALL ? 512 : (GPS == 1 ? 1024 : 544), SMALL ? 3 : 1)
    rotquant_kernel(const T* __restrict__ x, const RqArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int n_cons = blockDim.x - 32;
  const int HW = n_cons >> 4;
  uint8_t* scratch_base = smem + size_t(a.stages) * a.stage_bytes;  // HW slots of kRqSlotBytes
  uint64_t* full = reinterpret_cast<uint64_t*>(scratch_base + size_t(HW) * kRqSlotBytes);
  uint64_t* empty = full + a.stages;
  uint32_t* row_amax = reinterpret_cast<uint32_t*>(empty + a.stages);  // [3][kRqMaxRows]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(row_amax + 3 * kRqMaxRows);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
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
  float* scratch = reinterpret_cast<float*>(scratch_base + size_t(slot) * kRqSlotBytes);
  uint8_t* codes_buf = reinterpret_cast<uint8_t*>(scratch);  // reused once the group is rotated
  int rr[GPS], gg[GPS];
  bool act[GPS];
#pragma unroll
  for (int t = 0; t < GPS; ++t) {
    const int i = t * HW + slot;
    act[t] = i < a.R * G;
    rr[t] = act[t] ? i / G : 0;
    gg[t] = act[t] ? i - rr[t] * G : 0;
  }

  // Row slot buffers of the absmax: item k uses buffer k % 3; buffer (k + 1) % 3,
  // last read before barrier k - 1, is cleared before barrier k, ahead of item
  // k + 1's atomics.
  int stage = 0;
  uint32_t phase = 0;
  for (int64_t item = blockIdx.x, it = 0; item < a.items; item += gridDim.x, ++it) {
    mbar_wait_bounded(&full[stage], phase, a.wait_limit_ns, abort_flag);  // on expiry: garbage, no hang
    const T* tile = reinterpret_cast<const T*>(smem + size_t(stage) * a.stage_bytes);
    const int buf = static_cast<int>(it % 3);
    if (c < kRqMaxRows) row_amax[((it + 1) % 3) * kRqMaxRows + c] = 0u;
    const int64_t row0 = item * a.R;

    float2 p[GPS][8];
#pragma unroll
    for (int t = 0; t < GPS; ++t) {
      rotate_group(tile + rr[t] * a.K + gg[t] * 256, hl, scratch, p[t]);
      float m = 0.0f;
#pragma unroll
      for (int r = 0; r < 8; ++r) m = fmax3(m, fabsf(p[t][r].x), fabsf(p[t][r].y));
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
      if (hl == 0 && act[t] && row0 + rr[t] < a.M)
        atomicMax(&row_amax[buf * kRqMaxRows + rr[t]], __float_as_uint(m));
    }
    mbar_arrive(&empty[stage]);  // this thread's reads of the stage are done
    if (++stage == a.stages) {
      stage = 0;
      phase ^= 1u;
    }
    named_barrier(1, n_cons);
#pragma unroll
    for (int t = 0; t < GPS; ++t) {
      const int64_t row = row0 + rr[t];
      const float am = __uint_as_float(row_amax[buf * kRqMaxRows + rr[t]]);
      const float s16 = div127(am);
      if (hl == 0 && gg[t] == 0 && act[t] && row < a.M) a.s_out[row] = __fmul_rn(s16, 0.0625f);
      const RowQuot rq = row_quotient(s16);
      if (rq.f == 1.0f)
        quantize_column<false>(p[t], rq, hl, codes_buf);
      else
        quantize_column<true>(p[t], rq, hl, codes_buf);
      __syncwarp();
      const uint4 out = *reinterpret_cast<const uint4*>(codes_buf + 16 * hl);  // elements 16 hl .. 16 hl + 15
      __syncwarp();  // before the buffer is reused
      if (act[t] && row < a.M) *reinterpret_cast<uint4*>(a.q + row * a.K + gg[t] * 256 + 16 * hl) = out;
    }
  }
}

// ----------------------------------------------------------------------------
// Host side: shape choice and launch.

template <typename T, int GPS, bool SMALL>
cudaError_t rotquant_prepare_attr(int dev) {
  static bool done[16] = {};
  if (dev < 0 || dev >= 16) return cudaErrorInvalidDevice;
  if (done[dev]) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(rotquant_kernel<T, GPS, SMALL>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  if (e == cudaSuccess) done[dev] = true;
  return e;
}

template <typename T, int GPS, bool SMALL>
int rotquant_occupancy_t(int threads, size_t smem, int dev) {
  if (rotquant_prepare_attr<T, GPS, SMALL>(dev) != cudaSuccess) return 0;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, rotquant_kernel<T, GPS, SMALL>, threads, smem) !=
      cudaSuccess)
    return 0;
  return occ;
}

template <typename T>
int rotquant_occupancy(int gps, bool small, int threads, size_t smem, int dev) {
  if (gps == 1) return small ? rotquant_occupancy_t<T, 1, true>(threads, smem, dev)
                             : rotquant_occupancy_t<T, 1, false>(threads, smem, dev);
  return small ? rotquant_occupancy_t<T, 2, true>(threads, smem, dev)
               : rotquant_occupancy_t<T, 2, false>(threads, smem, dev);
}

// For a row of G groups: among shapes with 1 or 2 groups per slot, up to 8 rows
// per item and 2 to 6 stages, keep the one with the most consumer warps doing
// useful work per SM (occupancy times the share of busy slots), then the most
// loads in flight per SM (up to 128 KB).
template <typename T>
RqShape rotquant_plan(int K, int dev, int* blocks_per_sm) {
  static RqShape cache[16][65] = {};
  static int cache_occ[16][65] = {};
  const int G = K / 256;
  if (dev >= 0 && dev < 16 && G <= 64 && cache[dev][G].gps != 0) {
    *blocks_per_sm = cache_occ[dev][G];
    return cache[dev][G];
  }
  RqShape best{0, 0, 0, 0, false};
  int best_occ = 0;
  double best_score = -1.0;
  // Shapes measured fastest on B200 (bf16 rows, M = 16384): K = 5376: 2 groups per
  // slot, 3 rows per item, 16 consumer warps, 4 stages (2.92 TB/s, against 2.57 for
  // the best one-group shape); rows of 32 to 62 groups: one group per slot, one row
  // per item, ceil(G / 2) consumer warps, 4 stages (K = 14336: 28 warps, 2.95 TB/s;
  // K = 10752: 21 warps, 2.56 TB/s against 2.05 for the planner's choice).
  if (sizeof(T) == 2 && (K == 5376 || (G >= 32 && G <= 62))) {
    const RqShape pick = K == 5376 ? RqShape{2, 16, 3, 4, false} : RqShape{1, (G + 1) / 2, 1, 4, false};
    const uint32_t stage_bytes = static_cast<uint32_t>(int64_t(pick.rows) * K * int64_t(sizeof(T)));
    const int occ = rotquant_occupancy<T>(pick.gps, pick.small, 32 * (pick.warps + 1),
                                          rotquant_smem_bytes(pick.stages, stage_bytes, pick.warps), dev);
    if (occ >= 1) {
      best = pick;
      best_occ = occ;
      best_score = 1e30;  // keep it
    }
  }
  for (int gps = 1; gps <= 2 && best_score < 1e29; ++gps)
    for (int R = 1; R <= 8 && R <= kRqMaxRows; ++R)
      for (int small = 1; small >= 0; --small) {
        const int slots = R * G;
        const int W = (slots + 2 * gps - 1) / (2 * gps);
        const int threads = 32 * (W + 1);
        if (threads > (small ? 512 : (gps == 1 ? 1024 : 544))) continue;
        const uint32_t stage_bytes = static_cast<uint32_t>(int64_t(R) * K * int64_t(sizeof(T)));
        for (int stages = 2; stages <= 6; ++stages) {
          const size_t smem = rotquant_smem_bytes(stages, stage_bytes, W);
          if (smem > 227 * 1024) break;
          const int occ = rotquant_occupancy<T>(gps, small != 0, threads, smem, dev);
          if (occ < 1) break;
          // useful consumer warps per SM, then loads in flight per SM (capped)
          const double busy = double(slots) / double(2 * W * gps);
          const double inflight = double(occ) * stages * stage_bytes;
          const double score = occ * W * busy + 4.0 * (inflight < 131072.0 ? inflight : 131072.0) / 131072.0 -
                               0.01 * gps - 0.001 * R;
          if (score > best_score) {
            best_score = score;
            best = {gps, W, R, stages, small != 0};
            best_occ = occ;
          }
        }
      }
  if (dev >= 0 && dev < 16 && G <= 64 && best.gps != 0) {
    cache[dev][G] = best;
    cache_occ[dev][G] = best_occ;
  }
  *blocks_per_sm = best_occ;
  return best;
}

template <typename T>
cudaError_t launch_rotquant(const T* x, int64_t rows, int64_t K, int8_t* q, float* s, uint64_t wait_limit_ns,
                            cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static int sm_count[16] = {};
  if (dev < 0 || dev >= 16) return cudaErrorInvalidDevice;
  if (sm_count[dev] == 0) cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
  int occ = 0;
  const RqShape sh = rotquant_plan<T>(static_cast<int>(K), dev, &occ);
  if (sh.gps == 0) return cudaErrorInvalidConfiguration;
  RqArgs a;
  a.M = rows;
  a.K = static_cast<int>(K);
  a.R = sh.rows;
  a.items = (rows + sh.rows - 1) / sh.rows;
  a.stage_bytes = static_cast<uint32_t>(int64_t(sh.rows) * K * int64_t(sizeof(T)));
  a.stages = sh.stages;
  a.q = q;
  a.s_out = s;
  a.wait_limit_ns = wait_limit_ns;
  const size_t smem = rotquant_smem_bytes(sh.stages, a.stage_bytes, sh.warps);
  const int threads = 32 * (sh.warps + 1);
  const int64_t cap = int64_t(sm_count[dev]) * occ;
  const unsigned grid = static_cast<unsigned>(a.items < cap ? a.items : cap);
  if (sh.gps == 1) {
    if (sh.small) rotquant_kernel<T, 1, true><<<grid, threads, smem, stream>>>(x, a);
    else rotquant_kernel<T, 1, false><<<grid, threads, smem, stream>>>(x, a);
  } else {
    if (sh.small) rotquant_kernel<T, 2, true><<<grid, threads, smem, stream>>>(x, a);
    else rotquant_kernel<T, 2, false><<<grid, threads, smem, stream>>>(x, a);
  }
  return cudaGetLastError();
}

}  // namespace h3q
