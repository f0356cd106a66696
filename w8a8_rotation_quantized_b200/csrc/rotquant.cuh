// Rotate + per-row quantize: the ConvRot Hadamard-256 rotation done inside the
// quantizer (h3-rs README, "What makes it fast"), followed by per-row
// (per-token) absmax int8 quantization.
//
// Data movement: a persistent grid; in each block one producer thread streams
// work items (R whole rows) into a ring of shared-memory stages with TMA tensor
// copies (a 3D view of the rows as 128-byte units, 128-byte swizzle, completion
// on an mbarrier), so several items are in flight per block while the consumer
// warps work. Each row is read from HBM once and its codes are written once.
//
// Rotation of one 256-group by a quarter-warp (8 lanes), seen as an 8 x 32
// matrix X[j][m] = x[32 j + m]:
//   phase A  lane j holds row j (32 contiguous elements) and applies the
//            butterflies of index bits 0-4 in registers. Its 16-byte chunks are
//            read from the swizzled stage, so the 8 lanes of a quarter hit 8
//            different bank quads;
//   transpose through a per-quarter fp32 scratch of 8 rows with a 144-byte pitch
//            (each row shifted by one bank quad), written in 8-byte pairs (in
//            odd quarters with the two pairs of each 16-byte slot swapped) and
//            read in 16-byte pieces, without bank conflicts;
//   phase B  lane l holds elements 32 j + 4 l + i (j = 0..7, i = 0..3) and
//            applies the butterflies of bits 5-7.
// Values are kept as pairs (v[2i], v[2i+1]): bit 0 is one scalar add and one
// scalar subtract per pair (for bf16 the mixed-precision add reads the low
// element straight from the packed word), every other bit runs
// on the sm_100 two-wide fp32 add and FMA. The bits are processed in ascending
// order and every butterfly is one correctly rounded fp32 add or subtract, so
// each rotated value has the same bits as the pairwise-tree sum of the explicit
// H/16 product. The 1/16 moves to the scale: y16 = 16 y and s16 = max|y16| / 127
// = 16 s exactly, and y16 / s16 = y / s, so the codes are unchanged.
//
// Quantization needs rne(RN(y / s)) per element. Each row gets rs = RN(1/s)
// once. A candidate integer n = rne(y rs) and its exact-sign residual y - n s
// decide the code for all values but those within about 2^-16 of a half-integer
// quotient; for those the quotient is q0 = RN(y rs) refined twice with exact FMA
// residuals, e = y - q s, q <- RN(q + e rs) (Markstein, "Computation of
// elementary functions on the IBM RISC System/6000 processor", IBM J. Res. Dev.
// 34(1), 1990): after the first step q is within one ulp of y/s, and the second
// step returns the correctly rounded quotient, then rounded half to even. Rows
// whose scale is below 2^-100 are first rescaled by 2^64 (exact). Integers are
// read from the bits of a value plus 1.5*2^23, whose low byte is the int8 code.
// |y| <= max|y| bounds y/s by 127 (1 + 2^-23), so no clamp is needed. In phase B
// a lane's codes for j come from four consecutive elements: three byte permutes
// make one 32-bit word, stored straight to the row (a quarter writes 32
// contiguous bytes per j).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "ptx_sm100.cuh"

namespace h3q {

constexpr int kRqMaxRows = 16;
constexpr int kRqRowPitch = 144;                  // scratch row: 32 fp32 + 16 bytes
constexpr int kRqScratchBytes = 8 * kRqRowPitch;  // per quarter-warp
constexpr int kRqMaxWarps = 31;                   // consumer warps per block

// 16-byte shared-memory load at a shared-window address (ordered after the
// stage's mbarrier wait, which is also a volatile asm statement).
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// 3D tiled load of one box, completion counted on `bar`.
__device__ __forceinline__ void tma_load_3d(uint32_t smem_dst, const CUtensorMap* map, uint64_t* bar, int32_t x,
                                            int32_t y, int32_t z, uint64_t cache_policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)), "l"(cache_policy)
      : "memory");
}

// Phase A input: lane's 32 elements (32 j .. 32 j + 31 of its group) from the
// swizzled stage, chunk k at address a ^ (16 k), with the bit-0 butterfly:
// on return p[i] = (v[2i] + v[2i+1], v[2i] - v[2i+1]).
template <typename T>
struct LaneLoad;

template <>
struct LaneLoad<__nv_bfloat16> {  // four chunks of 8 elements
  static __device__ __forceinline__ void load(uint32_t a, float2 (&p)[16]) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint4 w = lds128(a ^ (16u * k));
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {  // element 2i of a word is its low half
        // lo + hi and lo - hi, each one rounding: the sm_100 mixed-precision add
        // takes the bf16 low half as it is and the high half masked to fp32
        const float hi = __uint_as_float(u[i] & 0xFFFF0000u);
        float sum, dif;
        asm("{\n\t.reg .b16 l16, h16;\n\tmov.b32 {l16, h16}, %2;\n\t"
            "add.rn.f32.bf16 %0, l16, %3;\n\tsub.rn.f32.bf16 %1, l16, %3;\n\t}"
            : "=f"(sum), "=f"(dif)
            : "r"(u[i]), "f"(hi));
        p[4 * k + i] = make_float2(sum, dif);
      }
    }
  }
};

template <>
struct LaneLoad<float> {  // eight chunks of 4 elements
  static __device__ __forceinline__ void load(uint32_t a, float2 (&p)[16]) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint4 w = lds128(a ^ (16u * k));
      const float v0 = __uint_as_float(w.x), v1 = __uint_as_float(w.y), v2 = __uint_as_float(w.z),
                  v3 = __uint_as_float(w.w);
      p[2 * k] = make_float2(__fadd_rn(v0, v1), __fsub_rn(v0, v1));
      p[2 * k + 1] = make_float2(__fadd_rn(v2, v3), __fsub_rn(v2, v3));
    }
  }
};

// The same loads in two steps: the lane's raw 16-byte chunks first (so a stage
// can be released before any arithmetic), then the unpack with the bit-0
// butterfly.
template <typename T>
struct LaneChunks {
  static constexpr int kN = 64 / int(sizeof(T)) / 2;  // bf16: 4 chunks, fp32: 8
  uint4 w[kN];
  __device__ __forceinline__ void load(uint32_t a) {
#pragma unroll
    for (int k = 0; k < kN; ++k) w[k] = lds128(a ^ (16u * k));
  }
  __device__ __forceinline__ void unpack(float2 (&p)[16]) const;
};

template <>
__device__ __forceinline__ void LaneChunks<__nv_bfloat16>::unpack(float2 (&p)[16]) const {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t u[4] = {w[k].x, w[k].y, w[k].z, w[k].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float hi = __uint_as_float(u[i] & 0xFFFF0000u);
      float sum, dif;
      asm("{\n\t.reg .b16 l16, h16;\n\tmov.b32 {l16, h16}, %2;\n\t"
          "add.rn.f32.bf16 %0, l16, %3;\n\tsub.rn.f32.bf16 %1, l16, %3;\n\t}"
          : "=f"(sum), "=f"(dif)
          : "r"(u[i]), "f"(hi));
      p[4 * k + i] = make_float2(sum, dif);
    }
  }
}

template <>
__device__ __forceinline__ void LaneChunks<float>::unpack(float2 (&p)[16]) const {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float v0 = __uint_as_float(w[k].x), v1 = __uint_as_float(w[k].y), v2 = __uint_as_float(w[k].z),
                v3 = __uint_as_float(w[k].w);
    p[2 * k] = make_float2(__fadd_rn(v0, v1), __fsub_rn(v0, v1));
    p[2 * k + 1] = make_float2(__fadd_rn(v2, v3), __fsub_rn(v2, v3));
  }
}

// Butterflies over pair indices: for every i with bit b clear,
// (p[i], p[i + 2^b]) <- (p[i] + p[i + 2^b], p[i] - p[i + 2^b]), bits B0..B1-1 in
// ascending order, each a two-wide correctly rounded add or subtract. `stride`
// maps a butterfly index to the pair index (phase B interleaves two pairs per j).
template <int N, int B0, int B1, int STRIDE>
__device__ __forceinline__ void butterflies(float2 (&p)[N]) {
  const float2 minus1 = make_float2(-1.0f, -1.0f);
#pragma unroll
  for (int b = B0; b < B1; ++b) {
    const int s = 1 << b;
#pragma unroll
    for (int i = 0; i < N / STRIDE; ++i) {
      if ((i & s) == 0) {
#pragma unroll
        for (int h = 0; h < STRIDE; ++h) {
          const float2 lo = p[STRIDE * i + h], hi = p[STRIDE * (i + s) + h];
          p[STRIDE * i + h] = __fadd2_rn(lo, hi);
          p[STRIDE * (i + s) + h] = __ffma2_rn(hi, minus1, lo);  // lo - hi, one rounding
        }
      }
    }
  }
}

// Rotates one group whose lane values (after the bit-0 butterfly, as loaded by
// LaneLoad) are in p; `scr` is the quarter's scratch, `l` the lane within the
// quarter and `odd` the quarter's parity. Phase A's pairs go to the scratch as
// 8-byte stores, each pair from its own aligned register pair (a 16-byte store
// would need two pairs moved into one aligned quad first). In an odd quarter pair
// k goes to slot k ^ 1: the two quarters of a half-warp then write disjoint bank
// sets (slots 2k, 2k+1 mod 4 against 2k+2, 2k+3 mod 4 words), so each 8-byte store
// of the warp takes the minimum two wavefronts. Phase B reads 16 bytes per row;
// in an odd quarter the two halves of each read are swapped, which the
// butterflies of bits 5-7 (across rows) do not see and the code packing undoes.
// On return p[2j + h] = (y16[32 j + 4 l + 2 (h ^ odd)], y16[32 j + 4 l + 2 (h ^ odd) + 1]).
__device__ __forceinline__ void rotate_group(float* scr, int l, int odd, float2 (&p)[16]) {
  butterflies<16, 0, 4, 1>(p);  // index bits 1-4
  float* row = scr + (kRqRowPitch / 4) * l;
  float* even_base = row + 2 * odd;  // pair k (k even) at slot k + odd
  float* odd_base = row - 2 * odd;   // pair k (k odd) at slot k - odd
#pragma unroll
  for (int k = 0; k < 16; k += 2) {
    *reinterpret_cast<float2*>(even_base + 2 * k) = p[k];
    *reinterpret_cast<float2*>(odd_base + 2 * k + 2) = p[k + 1];
  }
  __syncwarp();
#pragma unroll
  for (int j = 0; j < 8; ++j) {  // slots 2l, 2l+1 of row j
    const float4 c = *reinterpret_cast<const float4*>(scr + (kRqRowPitch / 4) * j + 4 * l);
    p[2 * j] = make_float2(c.x, c.y);
    p[2 * j + 1] = make_float2(c.z, c.w);
  }
  __syncwarp();                 // the scratch is rewritten by the next group
  butterflies<16, 0, 3, 2>(p);  // index bits 5-7
}

// max(m, |a|, |b|) (sm_100 three-input max; the absolute values are taken in
// the same asm block so they fold into the max's operands).
__device__ __forceinline__ float fmax_abs2(float m, float a, float b) {
  float r;
  asm("{\n\t.reg .f32 aa, ab;\n\tabs.f32 aa, %2;\n\tabs.f32 ab, %3;\n\tmax.f32 %0, %1, aa, ab;\n\t}"
      : "=f"(r)
      : "f"(m), "f"(a), "f"(b));
  return r;
}

__device__ __forceinline__ float group_lane_absmax(const float2 (&p)[16]) {
  float m0 = 0.0f, m1 = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    m0 = fmax_abs2(m0, p[i].x, p[i].y);
    m1 = fmax_abs2(m1, p[i + 1].x, p[i + 1].y);
  }
  return fmaxf(m0, m1);
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

// int8 codes rne(RN(y16 / s16)) of this lane's 32 values, stored as one 32-bit
// word per j at out + 32 j (out = the row's codes + 256 g + 4 l). `sel` orders the
// word's two code pairs: 0x5410 when p[2j] holds elements 4l, 4l+1 of row j, 0x1054
// when it holds 4l+2, 4l+3 (an odd quarter, see rotate_group).
//
// Fast path, three fp32 operations per value: the candidate n = rne(y rs) comes
// from one FMA onto 1.5*2^23 (whose bits then hold n in the low byte), and the
// residual r = RN(y - n s) from another. With t = RN(s (1/2 - 2^-16)), |r| <= t
// bounds |y/s - n| below 1/2 - 2^-16 + 2^-24; RN(y/s) moves y/s by at most 2^-18
// (|y/s| < 128), so n is the integer nearest RN(y/s) and the code is exact. A lane
// whose largest |r| exceeds t (y/s within about 2^-16 of a half-integer, some
// 3e-5 of the values) recomputes its 32 quotients as correctly rounded IEEE
// quotients (two Markstein steps) and rounds those. kRescaled: the row's f is
// 2^64 (scale below 2^-100); otherwise f = 1 and the exact rescaling is skipped.
// An all-zero row has s = 0, rs = 0, t = 0 and residuals 0: codes 0.
template <bool kRescaled>
__device__ __forceinline__ void quantize_store(const float2 (&p)[16], const RowQuot& rq, uint32_t sel,
                                               int8_t* out) {
  const float2 magic = make_float2(12582912.0f, 12582912.0f), nmagic = make_float2(-12582912.0f, -12582912.0f);
  const float2 f2 = make_float2(rq.f, rq.f), r2 = make_float2(rq.rs, rq.rs), ns2 = make_float2(-rq.sf, -rq.sf);
  const float t = __fmul_rn(rq.sf, 0.4999847412109375f);  // 1/2 - 2^-16
  float2 u[16];
  float m0 = 0.0f, m1 = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float2 y = kRescaled ? __fmul2_rn(p[i], f2) : p[i];  // exact
    u[i] = __ffma2_rn(y, r2, magic);
    const float2 r = __ffma2_rn(__fadd2_rn(u[i], nmagic), ns2, y);
    if (i & 1)
      m1 = fmax_abs2(m1, r.x, r.y);
    else
      m0 = fmax_abs2(m0, r.x, r.y);
  }
  if (fmaxf(m0, m1) > t) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float2 y = kRescaled ? __fmul2_rn(p[i], f2) : p[i];
      float2 q = __fmul2_rn(y, r2);
      float2 e = __ffma2_rn(q, ns2, y);
      q = __ffma2_rn(e, r2, q);
      e = __ffma2_rn(q, ns2, y);
      q = __ffma2_rn(e, r2, q);
      u[i] = __fadd2_rn(q, magic);
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t lo = __byte_perm(__float_as_uint(u[2 * j].x), __float_as_uint(u[2 * j].y), 0x0040);
    const uint32_t hi = __byte_perm(__float_as_uint(u[2 * j + 1].x), __float_as_uint(u[2 * j + 1].y), 0x0040);
    *reinterpret_cast<uint32_t*>(out + 32 * j) = __byte_perm(lo, hi, sel);
  }
}

struct RqArgs {
  int64_t M;             // rows
  int K;                 // row length (multiple of 256)
  int R;                 // rows per work item
  int items;             // ceil(M / R) (M < 2^31)
  int stages;            // shared-memory ring depth
  uint32_t stage_bytes;  // copies * copy_bytes
  uint32_t copy_bytes;   // shared-memory room of one TMA box, its bytes rounded up to 1024
  uint32_t tx_bytes;     // bytes the item's boxes deliver: copies x R x units_per_copy x 128
  int copies;            // TMA boxes per item (the row split along K)
  int units_per_copy;    // 128-byte units of a row in one box
  int8_t* q;
  float* s_out;
  uint64_t wait_limit_ns;
  uint32_t tmem_cols;    // tensor-memory columns a block allocates (tensor-memory variant)
};

struct RqShape {
  int gps, warps, rows, stages;  // groups per quarter-warp, consumer warps, rows per item, ring depth
};

// Tensor-memory columns a block of `warps` consumer warps with `gps` groups per
// quarter-warp allocates (a power of two, at least 32).
inline uint32_t rotquant_tm_cols(int warps, int gps) {
  const uint32_t need = uint32_t((warps + 3) / 4) * 64u * uint32_t(gps);
  uint32_t c = 32;
  while (c < need) c <<= 1;
  return c;
}

inline size_t rotquant_smem_bytes(int stages, uint32_t stage_bytes, int warps) {
  return 1024 + size_t(stages) * stage_bytes + size_t(4 * warps) * kRqScratchBytes + 2 * sizeof(uint64_t) * stages +
         3 * kRqMaxRows * 4 + 16;
}

// Byte offset, inside a stage, of the first 16-byte chunk of the 32 elements
// 32 l .. 32 l + 31 of group g in row r of the item: the stage holds `copies`
// boxes of copy_bytes; box c covers the units [c U, (c + 1) U) of every row as
// [rows][U][128 bytes], chunk x of unit n stored at chunk x ^ (n & 7).
template <typename T>
__device__ __forceinline__ uint32_t lane_tile_offset(const RqArgs& a, int r, int g, int l) {
  constexpr int kPerUnit = 128 / int(sizeof(T));
  const int e0 = 256 * g + 32 * l;
  const int unit = e0 / kPerUnit;
  const int chunk = (e0 % kPerUnit) * int(sizeof(T)) / 16;
  const int c = unit / a.units_per_copy, un = unit - c * a.units_per_copy;
  const int n = r * a.units_per_copy + un;
  return uint32_t(c) * a.copy_bytes + 128u * uint32_t(n) + 16u * uint32_t(chunk ^ (n & 7));
}

// Warp 0 is the producer; warps 1..W are consumers with 4W quarter-warps, each
// taking GPS groups per item: 4 W GPS >= R (K / 256).
template <typename T, int GPS>
__global__ void __launch_bounds__(GPS == 1 ? 768 : 512, 1)
    rotquant_kernel(const __grid_constant__ CUtensorMap tmap, const RqArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
  uint8_t* smem = smem_raw + pad;  // 1024-byte aligned: stages, then scratch
  const uint32_t stage0 = raw + pad;
  const int n_cons = blockDim.x - 32;
  const int NQ = n_cons >> 3;
  float* scratch_base = reinterpret_cast<float*>(smem + size_t(a.stages) * a.stage_bytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(scratch_base) +
                                               size_t(NQ) * kRqScratchBytes);
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
      tma_prefetch_desc(&tmap);
      const uint64_t pol = policy_evict_first();
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < a.items; item += gridDim.x) {
        if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, a.wait_limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[stage], a.tx_bytes);
        const uint32_t dst = stage0 + uint32_t(stage) * a.stage_bytes;
        for (int c = 0; c < a.copies; ++c)
          tma_load_3d(dst + uint32_t(c) * a.copy_bytes, &tmap, &full[stage], 0, c * a.units_per_copy,
                      item * a.R, pol);
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
  const int l = c & 7;
  const int qd = c >> 3;
  const int odd = qd & 1;
  const uint32_t sel = odd ? 0x1054u : 0x5410u;
  float* scr = scratch_base + size_t(qd) * (kRqScratchBytes / 4);
  int rr[GPS], gg[GPS];
  bool act[GPS];
  uint32_t toff[GPS];
#pragma unroll
  for (int t = 0; t < GPS; ++t) {
    const int i = t * NQ + qd;
    act[t] = i < a.R * G;
    rr[t] = act[t] ? i / G : 0;
    gg[t] = act[t] ? i - rr[t] * G : 0;
    toff[t] = lane_tile_offset<T>(a, rr[t], gg[t], l);
  }

  // Row slot buffers of the absmax: item k uses buffer k % 3; buffer (k + 1) % 3,
  // last read before barrier k - 1, is cleared before barrier k, ahead of item
  // k + 1's atomics.
  int stage = 0;
  uint32_t phase = 0;
  int buf = 0, next = kRqMaxRows;  // offsets of buffers it % 3 and (it + 1) % 3
  for (int item = blockIdx.x; item < a.items; item += gridDim.x) {
    mbar_wait_bounded_lazy(&full[stage], phase, a.wait_limit_ns, abort_flag);  // on expiry: garbage, no hang
    const uint32_t tile = stage0 + uint32_t(stage) * a.stage_bytes;
    if (c < kRqMaxRows) row_amax[next + c] = 0u;
    const int64_t row0 = int64_t(item) * a.R;
    const int rows_here = a.M - row0 < a.R ? static_cast<int>(a.M - row0) : a.R;  // the item's rows inside M

    float2 p[GPS][16];
#pragma unroll
    for (int t = 0; t < GPS; ++t) LaneLoad<T>::load(tile + toff[t], p[t]);
    mbar_arrive(&empty[stage]);  // this thread's reads of the stage are done: the producer may refill it
    if (++stage == a.stages) {
      stage = 0;
      phase ^= 1u;
    }
#pragma unroll
    for (int t = 0; t < GPS; ++t) {
      rotate_group(scr, l, odd, p[t]);
      float m = group_lane_absmax(p[t]);
#pragma unroll
      for (int o = 1; o <= 4; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
      if (l == 0 && act[t] && rr[t] < rows_here) atomicMax(&row_amax[buf + rr[t]], __float_as_uint(m));
    }
    named_barrier(1, n_cons);
    if (c < rows_here)  // one thread per row stores its scale s = s16 / 16
      a.s_out[row0 + c] = __fmul_rn(div127(__uint_as_float(row_amax[buf + c])), 0.0625f);
#pragma unroll
    for (int t = 0; t < GPS; ++t) {
      const float s16 = div127(__uint_as_float(row_amax[buf + rr[t]]));
      if (act[t] && rr[t] < rows_here) {
        const RowQuot rq = row_quotient(s16);
        int8_t* out = a.q + (row0 + rr[t]) * a.K + 256 * gg[t] + 4 * l;
        if (rq.f == 1.0f)
          quantize_store<false>(p[t], rq, sel, out);
        else
          quantize_store<true>(p[t], rq, sel, out);
      }
    }
    buf = next;
    next = next == 2 * kRqMaxRows ? 0 : next + kRqMaxRows;
  }
}

// ----------------------------------------------------------------------------
// Tensor-memory variant. The consumers keep each rotated group in tensor memory
// (tcgen05.st, 32 columns of the thread's own lane) instead of registers until
// the row's scale is known, and run two work items at once: in iteration i a
// thread loads and rotates its groups of item i, posts their maxima and parks
// the values in tensor-memory slot i % 2, then waits for item i - 1's row maxima
// (usually complete by then), reads that item's values back (tcgen05.ld) and
// quantizes them. The row maxima of item i go to buffer i % 4 as 64-bit words
// (i + 1) << 32 | bits(max) through an atomic max, so a buffer needs no clearing:
// a newer item's tag exceeds every older value. Completion of an item's maxima
// is an mbarrier per buffer that each quarter-warp's first lane arrives on after
// its posts (release), waited on with acquire before the reads. Four buffers
// suffice: a thread posts item i + 4 only after waiting for item i + 2, which
// every warp posts only after it has read item i's maxima.
//
// Tensor memory: warp w reaches lanes 32 (w % 4) .. 32 (w % 4) + 31; consumer
// warp w (1..W) takes columns ((w - 1) / 4) 64 GPS .. + 64 GPS of them, two
// slots of GPS groups of 32 columns.
constexpr int kRqtMaxRows = 64;
constexpr int kRqtMaxWarps = 16;

inline size_t rotquant_tm_smem_bytes(int stages, uint32_t stage_bytes, int warps) {
  return 1024 + size_t(stages) * stage_bytes + size_t(4 * warps) * kRqScratchBytes +
         sizeof(uint64_t) * (2 * stages + 4) + sizeof(unsigned long long) * 4 * kRqtMaxRows + 16;
}

template <typename T, int GPS>
__global__ void __launch_bounds__(32 * (kRqtMaxWarps + 1), 1)
    rotquant_tm_kernel(const __grid_constant__ CUtensorMap tmap, const RqArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
  uint8_t* smem = smem_raw + pad;  // 1024-byte aligned: stages, then scratch
  const uint32_t stage0 = raw + pad;
  const int n_cons = blockDim.x - 32;
  const int NQ = n_cons >> 3;
  float* scratch_base = reinterpret_cast<float*>(smem + size_t(a.stages) * a.stage_bytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(scratch_base) +
                                               size_t(NQ) * kRqScratchBytes);
  uint64_t* empty = full + a.stages;
  uint64_t* rowbar = empty + a.stages;                                                // [4]
  unsigned long long* rowmax = reinterpret_cast<unsigned long long*>(rowbar + 4);    // [4][kRqtMaxRows]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(rowmax + 4 * kRqtMaxRows);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.K >> 8;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], n_cons);
    }
    for (int b = 0; b < 4; ++b) mbar_init(&rowbar[b], NQ);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  for (int i = threadIdx.x; i < 4 * kRqtMaxRows; i += blockDim.x) rowmax[i] = 0ull;
  if (warp == 0) {
    tmem_alloc(tmem_slot, a.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap);
      const uint64_t pol = policy_evict_first();
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < a.items; item += gridDim.x) {
        if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, a.wait_limit_ns, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[stage], a.tx_bytes);
        const uint32_t dst = stage0 + uint32_t(stage) * a.stage_bytes;
        for (int c = 0; c < a.copies; ++c)
          tma_load_3d(dst + uint32_t(c) * a.copy_bytes, &tmap, &full[stage], 0, c * a.units_per_copy,
                      item * a.R, pol);
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
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- consumers
    const int c = threadIdx.x - 32;
    const int l = c & 7;
    const int qd = c >> 3;
    const int odd = qd & 1;
    const uint32_t sel = odd ? 0x1054u : 0x5410u;
    float* scr = scratch_base + size_t(qd) * (kRqScratchBytes / 4);
    int rr[GPS], gg[GPS];
    bool act[GPS];
    uint32_t toff[GPS];
#pragma unroll
    for (int t = 0; t < GPS; ++t) {
      const int i = t * NQ + qd;
      act[t] = i < a.R * G;
      rr[t] = act[t] ? i / G : 0;
      gg[t] = act[t] ? i - rr[t] * G : 0;
      toff[t] = lane_tile_offset<T>(a, rr[t], gg[t], l);
    }
    const uint32_t tm = tmem_base + (static_cast<uint32_t>(32 * (warp & 3)) << 16) +
                        static_cast<uint32_t>(((warp - 1) >> 2) * 64 * GPS);
    const int n_items = blockIdx.x < a.items ? (a.items - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;

    int stage = 0;
    uint32_t phase = 0;
    for (int it = 0; it <= n_items; ++it) {
      if (it < n_items) {  // load, rotate, post and park item it
        const int item = int(blockIdx.x) + it * int(gridDim.x);
        const int64_t row0 = int64_t(item) * a.R;
        const int rows_here = a.M - row0 < a.R ? static_cast<int>(a.M - row0) : a.R;
        const unsigned long long tag = static_cast<unsigned long long>(it + 1) << 32;
        unsigned long long* rmax = rowmax + (it & 3) * kRqtMaxRows;
        mbar_wait_bounded_lazy(&full[stage], phase, a.wait_limit_ns, abort_flag);  // on expiry: garbage, no hang
        const uint32_t tile = stage0 + uint32_t(stage) * a.stage_bytes;
        LaneChunks<T> raw[GPS];
#pragma unroll
        for (int t = 0; t < GPS; ++t) raw[t].load(tile + toff[t]);
        mbar_arrive(&empty[stage]);  // this thread's reads of the stage are done
        if (++stage == a.stages) {
          stage = 0;
          phase ^= 1u;
        }
#pragma unroll
        for (int t = 0; t < GPS; ++t) {
          float2 p[16];
          raw[t].unpack(p);
          rotate_group(scr, l, odd, p);
          float m = group_lane_absmax(p);
#pragma unroll
          for (int o = 1; o <= 4; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
          if (l == 0 && act[t] && rr[t] < rows_here) atomicMax(&rmax[rr[t]], tag | __float_as_uint(m));
          uint32_t v[32];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            v[2 * i] = __float_as_uint(p[i].x);
            v[2 * i + 1] = __float_as_uint(p[i].y);
          }
          tmem_st32(tm + static_cast<uint32_t>(((it & 1) * GPS + t) * 32), v);
        }
        __syncwarp();  // every lane of the warp is past its reads of item it - 4's buffer
        if (l == 0) mbar_arrive(&rowbar[it & 3]);
      }
      if (it >= 1) {  // quantize item it - 1
        const int pit = it - 1;
        const int item = int(blockIdx.x) + pit * int(gridDim.x);
        const int64_t row0 = int64_t(item) * a.R;
        const int rows_here = a.M - row0 < a.R ? static_cast<int>(a.M - row0) : a.R;
        const unsigned long long* rmax = rowmax + (pit & 3) * kRqtMaxRows;
        mbar_wait_bounded_lazy(&rowbar[pit & 3], static_cast<uint32_t>((pit >> 2) & 1), a.wait_limit_ns,
                               abort_flag);
        if (c < rows_here)  // one thread per row stores its scale s = s16 / 16
          a.s_out[row0 + c] = __fmul_rn(div127(__uint_as_float(static_cast<uint32_t>(rmax[c]))), 0.0625f);
        tmem_st_wait();
#pragma unroll
        for (int t = 0; t < GPS; ++t) {
          uint32_t v[32];
          tmem_ld32(tm + static_cast<uint32_t>(((pit & 1) * GPS + t) * 32), v);
          tmem_ld_wait();
          float2 u[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) u[i] = make_float2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
          const float s16 = div127(__uint_as_float(static_cast<uint32_t>(rmax[rr[t]])));
          if (act[t] && rr[t] < rows_here) {
            const RowQuot rq = row_quotient(s16);
            int8_t* out = a.q + (row0 + rr[t]) * a.K + 256 * gg[t] + 4 * l;
            if (rq.f == 1.0f)
              quantize_store<false>(u, rq, sel, out);
            else
              quantize_store<true>(u, rq, sel, out);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, a.tmem_cols);
  }
}

// ----------------------------------------------------------------------------
// Host side: shape choice and launch. The per-device host caches below (kernel
// attributes set, chosen shape and occupancy per row length, SM count) are
// read and written only under this mutex, which rotquant_plan holds.

inline std::mutex& rotquant_host_mutex() {
  static std::mutex m;
  return m;
}

template <typename T, int GPS>
cudaError_t rotquant_prepare_attr(int dev) {
  static bool done[16] = {};
  if (dev < 0 || dev >= 16) return cudaErrorInvalidDevice;
  if (done[dev]) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(rotquant_kernel<T, GPS>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  if (e == cudaSuccess) done[dev] = true;
  return e;
}

template <typename T>
int rotquant_occupancy(int gps, int threads, size_t smem, int dev) {
  int occ = 0;
  if (gps == 1) {
    if (rotquant_prepare_attr<T, 1>(dev) != cudaSuccess) return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, rotquant_kernel<T, 1>, threads, smem) != cudaSuccess)
      return 0;
  } else {
    if (rotquant_prepare_attr<T, 2>(dev) != cudaSuccess) return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, rotquant_kernel<T, 2>, threads, smem) != cudaSuccess)
      return 0;
  }
  return occ;
}

// TMA boxes per item and 128-byte units per box for rows of K elements of T: a
// box dimension holds at most 256 units.
template <typename T>
inline void rotquant_copies(int K, int* copies, int* units_per_copy) {
  const int units = K * int(sizeof(T)) / 128;
  int n = (units + 255) / 256;
  while (units % n != 0) ++n;
  *copies = n;
  *units_per_copy = units / n;
}

inline uint32_t align1024(uint64_t x) { return static_cast<uint32_t>((x + 1023u) & ~uint64_t(1023u)); }

template <typename T>
inline uint32_t rotquant_copy_bytes(int K, int R) {
  int n = 0, u = 0;
  rotquant_copies<T>(K, &n, &u);
  return align1024(uint64_t(R) * u * 128u);
}

// For a row of G groups: among shapes with 1 or 2 groups per quarter-warp, up to
// 8 rows per item and 2 to 6 stages, keep the one with the most consumer warps
// doing useful work per SM (occupancy times the share of busy quarters), then the
// most loads in flight per SM (up to 128 KB). bf16 rows of the model's widths use
// the shapes measured fastest on B200 at 16384 rows (two blocks per SM, two
// stages each): K = 5376: one group per quarter, 11 consumer warps, 2 rows per
// item (3.28 TB/s); K = 10752: one group per quarter, 11 warps, one row per item
// (3.5 TB/s); K = 14336: two groups per quarter, 7 warps, one row per item
// (3.7 TB/s).
template <typename T>
RqShape rotquant_plan(int K, int dev, int* blocks_per_sm, int* sms) {
  std::lock_guard<std::mutex> lock(rotquant_host_mutex());
  static RqShape cache[16][65] = {};
  static int cache_occ[16][65] = {};
  static int sm_count[16] = {};
  *blocks_per_sm = 0;
  *sms = 0;
  if (dev < 0 || dev >= 16) return RqShape{0, 0, 0, 0};
  if (sm_count[dev] == 0 &&
      cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return RqShape{0, 0, 0, 0};
  *sms = sm_count[dev];
  const int G = K / 256;
  if (G <= 64 && cache[dev][G].gps != 0) {
    *blocks_per_sm = cache_occ[dev][G];
    return cache[dev][G];
  }
  RqShape best{0, 0, 0, 0};
  int best_occ = 0;
  double best_score = -1.0;
  if (sizeof(T) == 2 && (G == 21 || G == 42 || G == 56)) {
    const RqShape pick = G == 21 ? RqShape{1, 11, 2, 2} : G == 42 ? RqShape{1, 11, 1, 2} : RqShape{2, 7, 1, 2};
    int n = 0, u = 0;
    rotquant_copies<T>(K, &n, &u);
    const uint32_t stage_bytes = uint32_t(n) * rotquant_copy_bytes<T>(K, pick.rows);
    const int occ = rotquant_occupancy<T>(pick.gps, 32 * (pick.warps + 1),
                                          rotquant_smem_bytes(pick.stages, stage_bytes, pick.warps), dev);
    if (occ >= 1) {
      best = pick;
      best_occ = occ;
      best_score = 1e30;  // keep it
    }
  }
  for (int gps = 1; gps <= 2 && best_score < 1e29; ++gps)
    for (int R = 1; R <= 8 && R <= kRqMaxRows; ++R) {
      const int slots = R * G;
      const int W = (slots + 4 * gps - 1) / (4 * gps);
      const int threads = 32 * (W + 1);
      if (W > kRqMaxWarps || threads > (gps == 1 ? 768 : 512)) continue;
      int n = 0, u = 0;
      rotquant_copies<T>(K, &n, &u);
      const uint32_t stage_bytes = uint32_t(n) * rotquant_copy_bytes<T>(K, R);
      for (int stages = 2; stages <= 6; ++stages) {
        const size_t smem = rotquant_smem_bytes(stages, stage_bytes, W);
        if (smem > 227 * 1024) break;
        const int occ = rotquant_occupancy<T>(gps, threads, smem, dev);
        if (occ < 1) break;
        const double busy = double(slots) / double(4 * W * gps);
        const double inflight = double(occ) * stages * stage_bytes;
        const double score = occ * W * busy + 4.0 * (inflight < 131072.0 ? inflight : 131072.0) / 131072.0 -
                             0.01 * gps - 0.001 * R;
        if (score > best_score) {
          best_score = score;
          best = {gps, W, R, stages};
          best_occ = occ;
        }
      }
    }
  if (G <= 64 && best.gps != 0) {
    cache[dev][G] = best;
    cache_occ[dev][G] = best_occ;
  }
  *blocks_per_sm = best_occ;
  return best;
}

// Fills the kernel arguments for a plan; the tensor map for x is built by the
// caller with the box {128 / sizeof(T), units_per_copy, R}.
template <typename T>
RqArgs rotquant_args(const RqShape& sh, int64_t rows, int64_t K, int8_t* q, float* s, uint64_t wait_limit_ns) {
  RqArgs a;
  a.M = rows;
  a.K = static_cast<int>(K);
  a.R = sh.rows;
  a.items = static_cast<int>((rows + sh.rows - 1) / sh.rows);
  rotquant_copies<T>(a.K, &a.copies, &a.units_per_copy);
  a.copy_bytes = rotquant_copy_bytes<T>(a.K, sh.rows);
  a.stage_bytes = uint32_t(a.copies) * a.copy_bytes;
  a.tx_bytes = uint32_t(a.copies) * uint32_t(sh.rows) * uint32_t(a.units_per_copy) * 128u;
  a.stages = sh.stages;
  a.q = q;
  a.s_out = s;
  a.wait_limit_ns = wait_limit_ns;
  a.tmem_cols = rotquant_tm_cols(sh.warps, sh.gps);
  return a;
}

// Launches a plan: a persistent grid of min(items, SMs x blocks per SM) blocks.
template <typename T>
cudaError_t launch_rotquant(const CUtensorMap& tmap, const RqShape& sh, int occ, int sms, const RqArgs& a,
                            cudaStream_t stream) {
  const size_t smem = rotquant_smem_bytes(sh.stages, a.stage_bytes, sh.warps);
  const int threads = 32 * (sh.warps + 1);
  const int64_t cap = int64_t(sms) * occ;
  const unsigned grid = static_cast<unsigned>(a.items < cap ? a.items : cap);
  if (sh.gps == 1)
    rotquant_kernel<T, 1><<<grid, threads, smem, stream>>>(tmap, a);
  else
    rotquant_kernel<T, 2><<<grid, threads, smem, stream>>>(tmap, a);
  return cudaGetLastError();
}

// ---- host side of the tensor-memory variant
template <typename T, int GPS>
cudaError_t rotquant_tm_prepare_attr(int dev) {
  static bool done[16] = {};
  if (dev < 0 || dev >= 16) return cudaErrorInvalidDevice;
  if (done[dev]) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(rotquant_tm_kernel<T, GPS>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  if (e == cudaSuccess) done[dev] = true;
  return e;
}

// Blocks per SM of a kernel by registers, shared memory, threads and the block
// limit, from its attributes and the device's. The runtime's occupancy query
// reports one block per SM for these kernels, which allocate tensor memory, where
// two fit and run (measured: both resident, x 80 -> 76 us at 16384 rows), so the
// count is made here; the tensor-memory limit is applied by the caller.
inline int blocks_per_sm_by_resources(const void* kernel, int threads, size_t dyn_smem, int dev) {
  cudaFuncAttributes fa{};
  if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return 0;
  int regs_sm = 0, smem_sm = 0, reserved = 0, threads_sm = 0, blocks_sm = 0;
  if (cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&threads_sm, cudaDevAttrMaxThreadsPerMultiProcessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&blocks_sm, cudaDevAttrMaxBlocksPerMultiprocessor, dev) != cudaSuccess)
    return 0;
  const int warps = (threads + 31) / 32;
  const int regs_warp = ((fa.numRegs * 32 + 255) / 256) * 256;  // allocated per warp in units of 256
  int n = blocks_sm;
  if (regs_warp > 0) n = std::min(n, regs_sm / (regs_warp * warps));
  n = std::min(n, threads_sm / (warps * 32));
  const size_t smem_block = dyn_smem + fa.sharedSizeBytes + size_t(reserved);
  n = std::min(n, int(size_t(smem_sm) / smem_block));
  return n;
}

template <typename T>
int rotquant_tm_occupancy(int gps, int threads, size_t smem, int dev) {
  if (gps == 1) {
    if (rotquant_tm_prepare_attr<T, 1>(dev) != cudaSuccess) return 0;
    return blocks_per_sm_by_resources(reinterpret_cast<const void*>(rotquant_tm_kernel<T, 1>), threads, smem, dev);
  }
  if (rotquant_tm_prepare_attr<T, 2>(dev) != cudaSuccess) return 0;
  return blocks_per_sm_by_resources(reinterpret_cast<const void*>(rotquant_tm_kernel<T, 2>), threads, smem, dev);
}

// Shape of the tensor-memory variant for rows of G = K / 256 groups: 1 or 2
// groups per quarter-warp, up to 16 consumer warps, as many rows per item as the
// quarters hold, 2 to 4 stages; blocks per SM limited by registers, shared memory
// and the 512 tensor-memory columns of an SM. Kept: the most consumer warps doing
// useful work per SM (two groups per quarter preferred: half the per-item work
// per element), then the most bytes in flight. bf16 rows of K = 5376 use the shape
// measured fastest (two groups per quarter, 8 consumer warps, 3 rows per item, 2
// stages, two blocks per SM: 75.8 us at 16384 rows).
// *smem_bytes: the dynamic shared memory to launch with. Where registers and
// shared memory would let more blocks share an SM than its tensor memory holds,
// the request is raised until they do not, so no block waits in tcgen05.alloc for
// another block on its SM to finish.
template <typename T>
RqShape rotquant_tm_plan(int K, int dev, int* blocks_per_sm, int* sms, size_t* smem_bytes) {
  std::lock_guard<std::mutex> lock(rotquant_host_mutex());
  static RqShape cache[16][65] = {};
  static int cache_occ[16][65] = {};
  static size_t cache_smem[16][65] = {};
  static int sm_count[16] = {};
  *blocks_per_sm = 0;
  *sms = 0;
  *smem_bytes = 0;
  if (dev < 0 || dev >= 16) return RqShape{0, 0, 0, 0};
  if (sm_count[dev] == 0 &&
      cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return RqShape{0, 0, 0, 0};
  *sms = sm_count[dev];
  const int G = K / 256;
  if (G <= 64 && cache[dev][G].gps != 0) {
    *blocks_per_sm = cache_occ[dev][G];
    *smem_bytes = cache_smem[dev][G];
    return cache[dev][G];
  }
  int n = 0, u = 0;
  rotquant_copies<T>(K, &n, &u);
  // blocks per SM (0 if the shape does not fit) and the shared memory to request
  auto evaluate = [&](const RqShape& sh, size_t* launch_smem) -> int {
    const uint32_t stage_bytes = uint32_t(n) * rotquant_copy_bytes<T>(K, sh.rows);
    size_t smem = rotquant_tm_smem_bytes(sh.stages, stage_bytes, sh.warps);
    if (smem > 227 * 1024) return 0;
    const int threads = 32 * (sh.warps + 1);
    const int by_tmem = int(512u / rotquant_tm_cols(sh.warps, sh.gps));
    int occ = rotquant_tm_occupancy<T>(sh.gps, threads, smem, dev);
    while (occ > by_tmem && smem + 1024 <= 227 * 1024) {
      smem += 1024;
      occ = rotquant_tm_occupancy<T>(sh.gps, threads, smem, dev);
    }
    if (occ > by_tmem) return 0;
    *launch_smem = smem;
    return occ;
  };
  RqShape best{0, 0, 0, 0};
  int best_occ = 0;
  size_t best_smem = 0;
  if (sizeof(T) == 2 && G == 21) {
    const RqShape pick{2, 8, 3, 2};
    size_t sm = 0;
    const int occ = evaluate(pick, &sm);
    if (occ >= 1) {
      best = pick;
      best_occ = occ;
      best_smem = sm;
    }
  }
  double best_score = best.gps != 0 ? 1e30 : -1.0;
  for (int gps = 2; gps >= 1 && best_score < 1e29; --gps)
    for (int W = 1; W <= kRqtMaxWarps; ++W) {
      const int slots = 4 * W * gps;
      int R = slots / G;
      if (R < 1) continue;
      if (R > kRqtMaxRows) R = kRqtMaxRows;
      if (rotquant_tm_cols(W, gps) > 512) continue;
      const uint32_t stage_bytes = uint32_t(n) * rotquant_copy_bytes<T>(K, R);
      for (int stages = 2; stages <= 4; ++stages) {
        const RqShape sh{gps, W, R, stages};
        size_t sm = 0;
        const int occ = evaluate(sh, &sm);
        if (occ < 1) break;
        const double busy = double(R * G) / double(slots);
        const double inflight = double(occ) * stages * stage_bytes;
        const double score = occ * W * busy * (gps == 2 ? 1.1 : 1.0) +
                             4.0 * (inflight < 131072.0 ? inflight : 131072.0) / 131072.0 - 0.001 * R;
        if (score > best_score) {
          best_score = score;
          best = sh;
          best_occ = occ;
          best_smem = sm;
        }
      }
    }
  if (G <= 64 && best.gps != 0) {
    cache[dev][G] = best;
    cache_occ[dev][G] = best_occ;
    cache_smem[dev][G] = best_smem;
  }
  *blocks_per_sm = best_occ;
  *smem_bytes = best_smem;
  return best;
}

// Launches a tensor-memory plan: a persistent grid of min(items, SMs x blocks per SM) blocks.
template <typename T>
cudaError_t launch_rotquant_tm(const CUtensorMap& tmap, const RqShape& sh, int occ, int sms, size_t smem,
                               const RqArgs& a, cudaStream_t stream) {
  const int threads = 32 * (sh.warps + 1);
  const int64_t cap = int64_t(sms) * occ;
  const unsigned grid = static_cast<unsigned>(a.items < cap ? a.items : cap);
  if (sh.gps == 1)
    rotquant_tm_kernel<T, 1><<<grid, threads, smem, stream>>>(tmap, a);
  else
    rotquant_tm_kernel<T, 2><<<grid, threads, smem, stream>>>(tmap, a);
  return cudaGetLastError();
}

}  // namespace h3q
