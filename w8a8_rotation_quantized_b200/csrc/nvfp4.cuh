// NVFP4 projections: the hybrid checkpoints run the QKV and FFN-input
// projections in NVFP4 on Blackwell and keep the attention-output and
// FFN-output projections INT8 ConvRot (Minimax_h3_hybrid model card,
// "Checkpoints" and "Native NVFP4 projection benchmarks"; h3-rs README,
// model-file table: "NVFP4 (swizzled fp8 block scales)").
//
// Format (the public NVFP4 definition; the pages do not spell it out): e2m1
// element codes, two per byte (element 2i in the low nibble), one e4m3 scale per
// 16 consecutive elements along K, one fp32 scale per tensor. No rotation.
//   s_enc = RN(2688 / max|x|)                   (1 for an all-zero tensor)
//   S     = e4m3_rne_sat(RN(RN(max|block| / 6) * s_enc))
//   q     = e2m1_rne_sat(RN(x * RN(s_enc / S)))  (0 where S = 0)
// Block scales are stored in the tensor cores' scale-factor layout: 512-byte
// atoms of 128 rows x 4 scales, byte 16 (r % 32) + 4 ((r % 128) / 32) + (j % 4)
// for row r and scale column j, atoms ordered by K first (atom index
// (r / 128) (K / 64) + j / 4); rows are padded to a multiple of 128 with zero
// scales.
//
// Kernels:
//  * nvfp4_amax_kernel: max|x| over the tensor into a device word (atomic max of
//    the bits of non-negative floats).
//  * nvfp4_quantize_kernel: one thread per 16-element block; the format's fp32
//    steps in the order above, with the hardware's e4m3 and e2m1 conversions
//    (round to nearest even, saturating).
//  * gemm_fp4_kernel: tcgen05.mma kind::mxf4nvf4 block16 (fp32 accumulation in
//    tensor memory, block scales from tensor memory), CTA pairs with 256 x 256
//    tiles as in the int8 GEMM, epilogue v = RN(RN(acc * alpha) + bias) with
//    alpha = RN(1 / RN(s_enc_x * s_enc_w)), bf16 or SwiGLU.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "gemm_sm100.cuh"
#include "ptx_sm100.cuh"

namespace h3q {

// ---------------------------------------------------------------- format helpers
__host__ __device__ constexpr int64_t nvfp4_sf_offset(int64_t r, int64_t j, int64_t K) {
  return ((r / 128) * (K / 64) + j / 4) * 512 + 16 * (r % 32) + 4 * ((r % 128) / 32) + (j % 4);
}

__host__ __device__ constexpr int64_t nvfp4_sf_bytes(int64_t rows, int64_t K) {
  return ((rows + 127) / 128) * 128 * (K / 16);
}

// e4m3 code (saturating at 448, round to nearest even) of a non-negative fp32.
__device__ __forceinline__ uint32_t f32_to_e4m3_sat(float u) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(u));
  return r & 0xFFu;
}

// Value of an e4m3 code (exact through f16).
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  uint32_t h2;
  const uint16_t c = static_cast<uint16_t>(code & 0xFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// Two e2m1 codes (round to nearest even, saturating at 6) in one byte: lo in
// bits 0-3, hi in bits 4-7.
__device__ __forceinline__ uint32_t f32x2_to_e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// ---------------------------------------------------------------- tensor max
template <typename T>
struct Vec16;  // 16 consecutive elements as fp32

template <>
struct Vec16<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[16]) {
    const uint4* q = reinterpret_cast<const uint4*>(p);
    const uint4 a = q[0], b = q[1];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};

template <>
struct Vec16<float> {
  static __device__ __forceinline__ void load(const float* p, float (&v)[16]) {
    const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 t = q[i];
      v[4 * i] = t.x;
      v[4 * i + 1] = t.y;
      v[4 * i + 2] = t.z;
      v[4 * i + 3] = t.w;
    }
  }
};

// scale[0] (as uint32 bits, zeroed by the caller) <- max |x| over n16 blocks of 16.
template <typename T>
__global__ void __launch_bounds__(256) nvfp4_amax_kernel(const T* __restrict__ x, int64_t n16,
                                                         uint32_t* __restrict__ amax_bits) {
  float m = 0.0f;
  for (int64_t b = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; b < n16; b += int64_t(gridDim.x) * blockDim.x) {
    float v[16];
    Vec16<T>::load(x + 16 * b, v);
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(m));
}

// ---------------------------------------------------------------- quantize
// One thread per 16-element block of rows [0, rows_pad): codes [rows, K/2],
// scales in the atom layout (zero for the padding rows rows .. rows_pad-1).
// scale[0] holds max|x| (bits); block (0,0)'s thread 0 stores s_enc in scale[1].
template <typename T>
__global__ void __launch_bounds__(256) nvfp4_quantize_kernel(const T* __restrict__ x, int64_t rows,
                                                             int64_t rows_pad, int K, float* __restrict__ scale,
                                                             uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
  const float amax = __uint_as_float(*reinterpret_cast<const uint32_t*>(scale));
  float s_enc = 1.0f;
  if (amax != 0.0f) {
    s_enc = __fdiv_rn(2688.0f, amax);
    if (isinf(s_enc)) s_enc = 3.40282347e38f;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) scale[1] = s_enc;
  const int bpr = K / 16;
  const int64_t total = rows_pad * bpr;
  for (int64_t t = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; t < total; t += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = t / bpr;
    const int j = static_cast<int>(t - r * bpr);
    uint32_t S = 0;
    if (r < rows) {
      float v[16];
      Vec16<T>::load(x + r * K + 16 * j, v);
      float bmax = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) bmax = fmaxf(bmax, fabsf(v[i]));
      const float u = __fmul_rn(__fdiv_rn(bmax, 6.0f), s_enc);
      S = f32_to_e4m3_sat(u);
      uint32_t w[4] = {0u, 0u, 0u, 0u};
      if (S != 0) {
        const float enc = __fdiv_rn(s_enc, e4m3_to_f32(S));
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t b = f32x2_to_e2m1x2(__fmul_rn(v[2 * i], enc), __fmul_rn(v[2 * i + 1], enc));
          w[i >> 2] |= b << (8 * (i & 3));
        }
      }
      *reinterpret_cast<uint2*>(codes + r * (K / 2) + 8 * j) = make_uint2(w[0], w[1]);
    }
    sf[nvfp4_sf_offset(r, j, K)] = static_cast<uint8_t>(S);
  }
}

// ---------------------------------------------------------------- tcgen05 block-scaled forms
// D[tmem] (+)= (A * SFA) x (B * SFB)^T for e2m1 A and B with one e4m3 scale per
// 16 elements (scales read from tensor memory), fp32 accumulation; CTA pair.
__device__ __forceinline__ void mma_fp4_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
      : "memory");
}

// Shared memory (32 rows x 16 bytes, rows contiguous) -> tensor memory lanes
// 0-31 and copies in lanes 32-63, 64-95, 96-127, four 32-bit columns; in both
// CTAs of the pair, each from its own shared memory at the same offset.
__device__ __forceinline__ void tmem_cp_32x128b_x4_pair(uint32_t taddr, uint64_t src_desc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(src_desc) : "memory");
}

// Descriptor of a 32 x 16-byte scale-factor atom: K-major, no swizzle; 8-row
// core matrices of 128 bytes stacked at a stride of 128 bytes (stride byte
// offset); one 16-byte column, so the leading byte offset is unused (0).
__device__ __forceinline__ uint64_t smem_desc_sf_atom(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(128u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  return d;
}

// Instruction descriptor for kind::mxf4nvf4: e2m1 A and B (format 1), e4m3
// scales (bit 23 = 0), both K-major, scale-factor byte ids 0, K = 64.
__host__ __device__ constexpr uint32_t idesc_fp4(uint32_t M, uint32_t N) {
  return (1u << 7)             // A format: e2m1
         | (1u << 10)          // B format: e2m1
         | ((N >> 3) << 17)    // N / 8
         | ((M >> 4) << 24);   // M / 16
}

// ---------------------------------------------------------------- GEMM
constexpr int kF4Stages = 5;
constexpr int kF4AStage = 128 * 128;   // 128 rows x 128 bytes (256 fp4) of A
constexpr int kF4BStage = 128 * 128;   // this CTA's 128 rows of the B tile
constexpr int kF4SfaStage = 4 * 512;   // 4 atoms: 128 rows x 16 scales
constexpr int kF4SfbStage = 8 * 512;   // 8 atoms: the whole B tile's 256 rows x 16 scales
constexpr int kF4StageBytes = kF4AStage + kF4BStage + kF4SfaStage + kF4SfbStage;
constexpr int kF4SfSlots = 4;          // tensor-memory scale-factor slots (48 columns each)
constexpr int kF4SfCols = 48;          // per slot: SFA 16 columns, SFB 32 columns
constexpr size_t kF4Smem = size_t(kF4Stages) * kF4StageBytes + 1024 + 256 + 2 * kBN * 4;
constexpr int kF4Threads = kGemmThreads + 32;  // producer, MMA, 8 epilogue warps, scale copier

struct Fp4Params {
  int M, N, K;              // N: output columns (SwiGLU: F); K in elements
  int num_m, num_n, num_tiles, group_m;
  int b_row_up;             // SwiGLU: first up row of B (= F)
  const float* x_scale;     // device [2]; [1] = s_enc of the activations
  const float* w_scale;     // device [2]; [1] = s_enc of the weights
  const __nv_bfloat16* bias;
  void* out;
  uint64_t wait_limit_ns;
};

__device__ __forceinline__ void fp4_tile_coords(int tile, const Fp4Params& p, int& mb, int& nb) {
  const int per_group = p.group_m * p.num_n;
  const int gid = tile / per_group;
  const int first_m = gid * p.group_m;
  const int gm = min(p.num_m - first_m, p.group_m);
  const int r = tile - gid * per_group;
  mb = first_m + r % gm;
  nb = r / gm;
}

// EPI: kEpiS32 = raw fp32 accumulators (test hook), kEpiBF16, kEpiSwiGLU.
template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kF4Threads, 1)
    gemm_fp4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                    const Fp4Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + kF4Stages * kF4AStage;
  uint8_t* sSFA = sB + kF4Stages * kF4BStage;
  uint8_t* sSFB = sSFA + kF4Stages * kF4SfaStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(sSFB + kF4Stages * kF4SfbStage);
  uint64_t* empty = full + kF4Stages;
  uint64_t* tfull = empty + kF4Stages;
  uint64_t* tempty = tfull + 1;
  uint64_t* drain = tempty + 1;
  uint64_t* sf_full = drain + 1;              // [slot] (leader): a stage's scales are in tensor memory
  uint64_t* sf_empty = sf_full + kF4SfSlots;  // [slot] (leader): the MMAs that read the slot are done
  uint64_t* drain_cp = sf_empty + kF4SfSlots;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_cp + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* col_bias = reinterpret_cast<float*>(smem + kF4Stages * kF4StageBytes + 256);  // [2][kBN]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int KB = p.K / 256;     // stages per tile
  const int katoms = p.K / 64;  // scale atoms per 128-row block
  const uint64_t limit = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kF4Stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, 16);
    mbar_init(drain, 1);
    for (int s = 0; s < kF4SfSlots; ++s) {
      mbar_init(&sf_full[s], 1);
      mbar_init(&sf_empty[s], 1);
    }
    mbar_init(drain_cp, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmSFA);
    tma_prefetch_desc(&tmSFB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer (both CTAs)
      const uint64_t pol = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < p.num_tiles; tile += npairs) {
        int mb, nb;
        fp4_tile_coords(tile, p, mb, nb);
        const int a_blk = mb * 2 + static_cast<int>(rank);  // this CTA's 128-row block of A
        const int b_blk0 = (EPI == kEpiSwiGLU) ? nb : 2 * nb;
        const int b_blk1 = (EPI == kEpiSwiGLU) ? p.b_row_up / 128 + nb : 2 * nb + 1;
        const int b_row = rank == 0 ? b_blk0 * 128 : b_blk1 * 128;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, limit, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t full_leader = cluster_map(&full[stage], 0);
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * kF4StageBytes);
          tma_load_2d_pair(sA + stage * kF4AStage, &tmA, full_leader, kb * 128, a_blk * 128, pol);
          tma_load_2d_pair(sB + stage * kF4BStage, &tmB, full_leader, kb * 128, b_row, pol);
          // scale atoms: 128-byte rows of the atom array, 4 rows per atom
          tma_load_2d_pair(sSFA + stage * kF4SfaStage, &tmSFA, full_leader, 0, 4 * (a_blk * katoms + 4 * kb), pol);
          tma_load_2d_pair(sSFB + stage * kF4SfbStage, &tmSFB, full_leader, 0, 4 * (b_blk0 * katoms + 4 * kb), pol);
          tma_load_2d_pair(sSFB + stage * kF4SfbStage + 2048, &tmSFB, full_leader, 0,
                           4 * (b_blk1 * katoms + 4 * kb), pol);
          ++issued;
          if (++stage == kF4Stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && rank == 0) {
        for (int s = 0; s < kF4Stages; ++s) {
          if (issued <= s) continue;
          const long last = ((issued - 1 - s) / kF4Stages) * kF4Stages + s;
          mbar_wait_bounded(&full[s], static_cast<uint32_t>((last / kF4Stages) & 1), limit, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------------ MMA issuer (leader only)
      constexpr uint32_t idesc = idesc_fp4(2 * kBM, kBN);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_phase = 0;
      long nk = 0;  // stages consumed, across tiles: scale slot nk % kF4SfSlots
      bool ok = true;
      for (int tile = pair; ok && tile < p.num_tiles; tile += npairs) {
        if (!mbar_wait_bounded_cluster(tempty, acc_phase ^ 1u, limit, abort_flag)) break;
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, limit, abort_flag)) {
            ok = false;
            break;
          }
          const int slot = static_cast<int>(nk % kF4SfSlots);
          if (!mbar_wait_bounded(&sf_full[slot], static_cast<uint32_t>((nk / kF4SfSlots) & 1), limit, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sf_col = tmem + static_cast<uint32_t>(kBN + slot * kF4SfCols);
          const uint64_t ad = smem_desc_sw128(smem_u32(sA + stage * kF4AStage));
          const uint64_t bd = smem_desc_sw128(smem_u32(sB + stage * kF4BStage));
#pragma unroll
          for (int k = 0; k < 4; ++k)  // 64 fp4 = 32 bytes per K step
            mma_fp4_pair(tmem, ad + 2u * k, bd + 2u * k, idesc, sf_col + 4 * k, sf_col + 16 + 8 * k,
                         (kb | k) != 0 ? 1u : 0u);
          mma_commit_pair(cluster_map(&empty[stage], 0));
          mma_commit_pair(cluster_map(&empty[stage], 1));
          mma_commit_pair(cluster_map(&sf_empty[slot], 0));
          ++nk;
          if (++stage == kF4Stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair(cluster_map(tfull, 0));
        mma_commit_pair(cluster_map(tfull, 1));
        acc_phase ^= 1u;
      }
      mma_commit_pair(cluster_map(drain, 0));
      mbar_wait_bounded(drain, 0, limit, nullptr);
    }
  } else if (warp == kF4Threads / 32 - 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------------ scale copier (leader only)
      // Copies each stage's block scales into tensor-memory slot n % kF4SfSlots (12
      // tcgen05.cp per stage, into both CTAs) once the stage has landed and the MMAs
      // that last read the slot are done, and signals the MMA issuer through sf_full.
      // A thread of its own: the copies no longer queue in the MMA issuer's stream.
      int stage = 0;
      uint32_t phase = 0;
      long n = 0;
      for (int tile = pair; tile < p.num_tiles; tile += npairs) {
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
          const int slot = static_cast<int>(n % kF4SfSlots);
          if (!mbar_wait_bounded(&full[stage], phase, limit, abort_flag) ||
              !mbar_wait_bounded(&sf_empty[slot], static_cast<uint32_t>(((n / kF4SfSlots) & 1) ^ 1), limit,
                                 abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sf_col = tmem + static_cast<uint32_t>(kBN + slot * kF4SfCols);
          const uint32_t sfa_base = smem_u32(sSFA + stage * kF4SfaStage);
          const uint32_t sfb_base = smem_u32(sSFB + stage * kF4SfbStage);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            tmem_cp_32x128b_x4_pair(sf_col + 4 * j, smem_desc_sf_atom(sfa_base + 512 * j));
            tmem_cp_32x128b_x4_pair(sf_col + 16 + 8 * j, smem_desc_sf_atom(sfb_base + 512 * j));
            tmem_cp_32x128b_x4_pair(sf_col + 16 + 8 * j + 4, smem_desc_sf_atom(sfb_base + 2048 + 512 * j));
          }
          mma_commit_pair(cluster_map(&sf_full[slot], 0));
          ++n;
          if (++stage == kF4Stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      mma_commit_pair(cluster_map(drain_cp, 0));
      mbar_wait_bounded(drain_cp, 0, limit, nullptr);
    }
  } else {
    // -------------------------------------------------------------- epilogue (both CTAs)
    // Warps 2..9: warp w owns TMEM lanes 32*(w%4) .. +31 and half of the tile's
    // columns. The accumulator is single-buffered (the scale-factor slots take
    // the rest of tensor memory), so each warp first pulls all of its 128
    // columns into registers and frees the accumulator, and the next tile's
    // MMAs overlap its rescale and stores.
    const int quarter = warp & 3;
    const int chalf = (warp - 2) >> 2;
    const int et = threadIdx.x - 64;  // 0 .. 255
    const int row_in_tile = static_cast<int>(rank) * kBM + quarter * 32 + lane;
    const uint32_t tempty_leader = cluster_map(tempty, 0);
    const bool has_bias = p.bias != nullptr;
    float alpha = 1.0f;
    if constexpr (EPI != kEpiS32) alpha = __fdiv_rn(1.0f, __fmul_rn(__ldg(p.x_scale + 1), __ldg(p.w_scale + 1)));
    uint32_t acc_phase = 0;
    int iter = 0;
    for (int tile = pair; tile < p.num_tiles; tile += npairs, ++iter) {
      int mb, nb;
      fp4_tile_coords(tile, p, mb, nb);
      float* cb = col_bias + (iter & 1) * kBN;
      if constexpr (EPI != kEpiS32) {
        int n;
        bool valid;
        if constexpr (EPI == kEpiSwiGLU) {
          n = et < 128 ? nb * 128 + et : p.b_row_up + nb * 128 + (et - 128);
          valid = true;
        } else {
          n = nb * kBN + et;
          valid = n < p.N;
        }
        cb[et] = (valid && has_bias) ? __bfloat162float(p.bias[n]) : 0.0f;
        named_barrier(1, 256);
      }
      if (!mbar_wait_bounded_cluster(tfull, acc_phase, limit, abort_flag)) break;
      tc_fence_after();
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
      uint32_t r[4][32];
      if constexpr (EPI == kEpiSwiGLU) {  // gate columns [64 chalf, +64), up columns 128 + the same
        tmem_ld32(taddr + (2 * chalf) * 32, r[0]);
        tmem_ld32(taddr + (2 * chalf + 1) * 32, r[1]);
        tmem_ld32(taddr + 128 + (2 * chalf) * 32, r[2]);
        tmem_ld32(taddr + 128 + (2 * chalf + 1) * 32, r[3]);
      } else {  // columns [128 chalf, +128)
#pragma unroll
        for (int i = 0; i < 4; ++i) tmem_ld32(taddr + (4 * chalf + i) * 32, r[i]);
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader);
      acc_phase ^= 1u;
      const int row = mb * (2 * kBM) + row_in_tile;
      const bool row_ok = row < p.M;
      if constexpr (EPI == kEpiS32) {
        float* out = static_cast<float*>(p.out) + static_cast<int64_t>(row) * p.N;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int n0 = nb * kBN + (4 * chalf + i) * 32;
#pragma unroll
          for (int g = 0; g < 4; ++g)
            if (row_ok && n0 + 8 * g < p.N) {
              uint4* dst = reinterpret_cast<uint4*>(out + n0 + 8 * g);
              dst[0] = make_uint4(r[i][8 * g], r[i][8 * g + 1], r[i][8 * g + 2], r[i][8 * g + 3]);
              dst[1] = make_uint4(r[i][8 * g + 4], r[i][8 * g + 5], r[i][8 * g + 6], r[i][8 * g + 7]);
            }
        }
      } else if constexpr (EPI == kEpiBF16) {
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + static_cast<int64_t>(row) * p.N;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int i0 = (4 * chalf + i) * 32 + 8 * g;  // column within the tile
            const int n = nb * kBN + i0;
            if (n < p.N) {
              uint32_t o[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                float v0 = __fmul_rn(__uint_as_float(r[i][8 * g + 2 * e]), alpha);
                float v1 = __fmul_rn(__uint_as_float(r[i][8 * g + 2 * e + 1]), alpha);
                if (has_bias) {
                  v0 = __fadd_rn(v0, cb[i0 + 2 * e]);
                  v1 = __fadd_rn(v1, cb[i0 + 2 * e + 1]);
                }
                o[e] = pack_bf16x2(v0, v1);
              }
              if (row_ok) *reinterpret_cast<uint4*>(out + n) = make_uint4(o[0], o[1], o[2], o[3]);
            }
          }
        }
      } else {  // SwiGLU
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + static_cast<int64_t>(row) * p.N;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int i0 = (2 * chalf + cc) * 32 + 8 * g;  // gate column within the tile; up is 128 + i0
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float h[2];
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                const int k = i0 + 2 * e + q;
                float gv = __fmul_rn(__uint_as_float(r[cc][8 * g + 2 * e + q]), alpha);
                float uv = __fmul_rn(__uint_as_float(r[2 + cc][8 * g + 2 * e + q]), alpha);
                if (has_bias) {
                  gv = __fadd_rn(gv, cb[k]);
                  uv = __fadd_rn(uv, cb[128 + k]);
                }
                h[q] = __fmul_rn(silu_f32(gv), uv);
              }
              o[e] = pack_bf16x2(h[0], h[1]);
            }
            if (row_ok) *reinterpret_cast<uint4*>(out + nb * 128 + i0) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, kTmemCols);
}

}  // namespace h3q
