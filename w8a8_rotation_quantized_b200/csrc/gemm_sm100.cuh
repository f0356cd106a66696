// INT8 GEMM with int32 accumulation on the 5th-generation tensor cores
// (tcgen05.mma kind::i8, accumulators in tensor memory), fed by TMA, with the
// dequantize / bias / bf16 / SwiGLU epilogue fused (h3-rs README, "What makes it
// fast": a fused int8 GEMM that writes bf16 directly, SwiGLU fused into fc1's
// epilogue).
//
//   acc[m][n] = sum_k A[m][k] * B[n][k]     A = xq [M, K], B = wq [N, K], both K-major
//
// Design (one CTA per SM, persistent):
//   warp 0      TMA producer: one 128x128 int8 box of A and two of B per stage
//               into a STAGES-deep ring of 128-byte-swizzled shared memory.
//   warp 1      allocates 512 TMEM columns; one lane issues 4 MMAs of
//               128 x 256 x 32 per stage and commits each stage back to the
//               producer and each finished tile to the epilogue.
//   warps 2-5   epilogue: tcgen05.ld of their 32-lane quarter of the
//               accumulator, fp32 rescale, bias, bf16 (or SwiGLU), stores.
// Two 256-column accumulators let the epilogue of tile i overlap the main loop
// of tile i+1. Tiles are walked in groups of GROUP_M row blocks so the weight
// blocks in flight stay in L2.
//
// SwiGLU: the B tile of an output tile holding h columns [j0, j0+128) stacks
// gate rows [j0, j0+128) over up rows [F+j0, F+j0+128) of the plain [gate; up]
// weight, so one 128 x 256 accumulator holds both halves and silu(g) * u is
// formed per element in the epilogue. This gives the locality that the pages get
// by interleaving gate/up rows at load, without repacking the weight.
//
// Every wait is bounded (see mbar_wait_bounded); past the limit the block
// records a timeout, drains its own copies and MMAs (bounded again), frees its
// tensor memory and exits.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "ptx_sm100.cuh"

namespace h3q {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 128;  // int8 elements = 128 bytes = one swizzle row
constexpr int kStages = 4;
constexpr int kAStage = kBM * kBK;  // 16 KB
constexpr int kBStage = kBN * kBK;  // 32 KB
constexpr int kTmemCols = 512;
constexpr int kGemmThreads = 192;
constexpr int kGroupM = 16;
constexpr size_t kGemmSmem = size_t(kStages) * (kAStage + kBStage) + 1024 /*align*/ + 256 /*barriers*/;

enum EpiKind : int { kEpiS32 = 0, kEpiBF16 = 1, kEpiSwiGLU = 2 };

struct GemmParams {
  int M;            // rows of A / output
  int N;            // output columns (SwiGLU: F)
  int K;
  int num_m, num_n, num_tiles;
  int b_row_up;     // SwiGLU: first up row of B (= F)
  const float* sx;  // [M]
  const float* sw;  // [N] (SwiGLU: [2F])
  const __nv_bfloat16* bias;  // nullable, [N] (SwiGLU: [2F])
  void* out;        // [M, N] int32 or bf16 (SwiGLU: [M, F] bf16)
  uint64_t wait_limit_ns;
};

__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int& mb, int& nb) {
  const int per_group = kGroupM * num_n;
  const int gid = tile / per_group;
  const int first_m = gid * kGroupM;
  const int gm = min(num_m - first_m, kGroupM);
  const int r = tile - gid * per_group;
  mb = first_m + r % gm;
  nb = r / gm;
}

// e^t in fp32: Cody-Waite reduction t = n ln2 + r with fdlibm's two-part ln2
// (0x3f317200, 0x35bfbe8e), e^r by the degree-7 Taylor polynomial in Horner form
// with fused multiply-adds, then an exact scale by 2^n. t > 88 gives +inf; for
// t < -20, 1 + e^t is 1 in fp32, so e^t is taken as 0.
__device__ __forceinline__ float exp_f32(float t) {
  if (t > 88.0f) return __int_as_float(0x7F800000);
  if (t < -20.0f) return 0.0f;
  const float n = rintf(__fmul_rn(t, 1.44269502f));
  float r = __fmaf_rn(n, -0.693145751953125f, t);
  r = __fmaf_rn(n, -1.42860677e-06f, r);
  float p = 1.0f / 5040.0f;
  p = __fmaf_rn(p, r, 1.0f / 720.0f);
  p = __fmaf_rn(p, r, 1.0f / 120.0f);
  p = __fmaf_rn(p, r, 1.0f / 24.0f);
  p = __fmaf_rn(p, r, 1.0f / 6.0f);
  p = __fmaf_rn(p, r, 0.5f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  return __fmul_rn(p, __int_as_float((static_cast<int>(n) + 127) << 23));
}

__device__ __forceinline__ float silu_f32(float g) { return __fdiv_rn(g, __fadd_rn(1.0f, exp_f32(-g))); }

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Loads 8 consecutive fp32 values and 8 bf16 values (as fp32) starting at n.
__device__ __forceinline__ void load_col8(const float* sw, const __nv_bfloat16* bias, int n, float (&s)[8],
                                          float (&b)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(sw + n));
  const float4 c = __ldg(reinterpret_cast<const float4*>(sw + n) + 1);
  s[0] = a.x; s[1] = a.y; s[2] = a.z; s[3] = a.w; s[4] = c.x; s[5] = c.y; s[6] = c.z; s[7] = c.w;
  if (bias != nullptr) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(bias + n));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      b[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
      b[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
    }
  }
}

// v = ((float)acc * sx) * sw (+ bias), no fused multiply-add.
__device__ __forceinline__ float rescale(uint32_t acc_bits, float sxr, float swn, float bn, bool has_bias) {
  float v = __int2float_rn(static_cast<int>(acc_bits));
  v = __fmul_rn(v, sxr);
  v = __fmul_rn(v, swn);
  if (has_bias) v = __fadd_rn(v, bn);
  return v;
}

template <int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_i8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kAStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kStages * kBStage);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = p.K / kBK;
  const uint64_t limit = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      const uint64_t pol = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        int mb, nb;
        tile_coords(tile, p.num_m, p.num_n, mb, nb);
        const int b_row0 = (EPI == kEpiSwiGLU) ? nb * 128 : nb * kBN;
        const int b_row1 = (EPI == kEpiSwiGLU) ? p.b_row_up + nb * 128 : nb * kBN + 128;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, limit, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], kAStage + kBStage);
          tma_load_2d(sA + stage * kAStage, &tmA, &full[stage], kb * kBK, mb * kBM, pol);
          tma_load_2d(sB + stage * kBStage, &tmB, &full[stage], kb * kBK, b_row0, pol);
          tma_load_2d(sB + stage * kBStage + kBStage / 2, &tmB, &full[stage], kb * kBK, b_row1, pol);
          ++issued;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // drain this block's own copies still in flight (bounded, ignores abort)
        for (int s = 0; s < kStages; ++s) {
          if (issued <= s) continue;
          const long last = ((issued - 1 - s) / kStages) * kStages + s;
          mbar_wait_bounded(&full[s], static_cast<uint32_t>((last / kStages) & 1), limit, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = idesc_i8(kBM, kBN);
      int stage = 0;
      uint32_t phase = 0;
      int buf = 0;
      uint32_t buf_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        if (!mbar_wait_bounded(&tempty[buf], buf_phase ^ 1u, limit, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(buf * kBN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, limit, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = smem_desc_sw128(smem_u32(sA + stage * kAStage));
          const uint64_t bd = smem_desc_sw128(smem_u32(sB + stage * kBStage));
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k) {
            // advance the start address by 32 bytes (= 2 in 16-byte units) per K step
            mma_i8(d, ad + 2u * k, bd + 2u * k, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          mma_commit(&empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&tfull[buf]);
        buf ^= 1;
        if (buf == 0) buf_phase ^= 1u;
      }
      // every MMA this block issued has completed once `drain` fires
      mma_commit(drain);
      mbar_wait_bounded(drain, 0, limit, nullptr);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31 belong to this warp
    const int row_in_tile = quarter * 32 + lane;
    int buf = 0;
    uint32_t buf_phase = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
      int mb, nb;
      tile_coords(tile, p.num_m, p.num_n, mb, nb);
      if (!mbar_wait_bounded(&tfull[buf], buf_phase, limit, abort_flag)) break;
      tc_fence_after();
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(buf * kBN);
      const int row = mb * kBM + row_in_tile;
      const bool row_ok = row < p.M;

      if constexpr (EPI == kEpiS32) {
        int32_t* out = static_cast<int32_t*>(p.out) + static_cast<int64_t>(row) * p.N;
#pragma unroll 1
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(taddr + c * 32, r);
          tmem_ld_wait();
          const int n0 = nb * kBN + c * 32;
          if (row_ok) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              if (n0 + 8 * g < p.N) {
                uint4* dst = reinterpret_cast<uint4*>(out + n0 + 8 * g);
                dst[0] = make_uint4(r[8 * g], r[8 * g + 1], r[8 * g + 2], r[8 * g + 3]);
                dst[1] = make_uint4(r[8 * g + 4], r[8 * g + 5], r[8 * g + 6], r[8 * g + 7]);
              }
            }
          }
        }
      } else if constexpr (EPI == kEpiBF16) {
        const float sxr = row_ok ? __ldg(p.sx + row) : 0.0f;
        const bool has_bias = p.bias != nullptr;
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + static_cast<int64_t>(row) * p.N;
#pragma unroll 1
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(taddr + c * 32, r);
          tmem_ld_wait();
          const int n0 = nb * kBN + c * 32;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int n = n0 + 8 * g;
            if (n < p.N) {
              float s[8], b[8];
              load_col8(p.sw, p.bias, n, s, b);
              uint32_t o[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float v0 = rescale(r[8 * g + 2 * i], sxr, s[2 * i], b[2 * i], has_bias);
                const float v1 = rescale(r[8 * g + 2 * i + 1], sxr, s[2 * i + 1], b[2 * i + 1], has_bias);
                o[i] = pack_bf16x2(v0, v1);
              }
              if (row_ok) *reinterpret_cast<uint4*>(out + n) = make_uint4(o[0], o[1], o[2], o[3]);
            }
          }
        }
      } else {  // SwiGLU: accumulator columns [0,128) gate, [128,256) up
        const float sxr = row_ok ? __ldg(p.sx + row) : 0.0f;
        const bool has_bias = p.bias != nullptr;
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + static_cast<int64_t>(row) * p.N;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t rg[32], ru[32];
          tmem_ld32(taddr + c * 32, rg);
          tmem_ld32(taddr + 128 + c * 32, ru);
          tmem_ld_wait();
          const int j0 = nb * 128 + c * 32;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int j = j0 + 8 * g;
            float sg[8], bg[8], su[8], bu[8];
            load_col8(p.sw, p.bias, j, sg, bg);
            load_col8(p.sw, p.bias, p.b_row_up + j, su, bu);
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              float h[2];
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int k = 2 * i + e;
                const float gv = rescale(rg[8 * g + k], sxr, sg[k], bg[k], has_bias);
                const float uv = rescale(ru[8 * g + k], sxr, su[k], bu[k], has_bias);
                h[e] = __fmul_rn(silu_f32(gv), uv);
              }
              o[i] = pack_bf16x2(h[0], h[1]);
            }
            if (row_ok) *reinterpret_cast<uint4*>(out + j) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
      buf ^= 1;
      if (buf == 0) buf_phase ^= 1u;
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// Test kernel for the bounded-wait path: waits on an mbarrier that nothing ever
// arrives on; the wait gives up after limit_ns and records the timeout.
__global__ void stalled_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, limit_ns, &abort_flag);
  __syncthreads();
}

}  // namespace h3q
