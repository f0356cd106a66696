// INT8 GEMM with int32 accumulation on the 5th-generation tensor cores
// (tcgen05.mma kind::i8, accumulators in tensor memory), fed by TMA, with the
// dequantize / bias / bf16 / SwiGLU epilogue fused (h3-rs README, "What makes it
// fast": a fused int8 GEMM that writes bf16 directly, SwiGLU fused into fc1's
// epilogue).
//
//   acc[m][n] = sum_k A[m][k] * B[n][k]     A = xq [M, K], B = wq [N, K], both K-major
//
// Design (persistent; CTA pairs, one CTA per SM; cta_group::2 MMAs):
//   A pair computes 256 x 256 output tiles: CTA r holds rows 128r .. 128r+127
//   of the A tile and rows 128r .. 128r+127 of the B tile, and the pair's
//   M=256 MMA (issued by the leader, rank 0) reads both CTAs' shared memory, so
//   each SM stages half the operand bytes a one-SM 128 x 256 tile would need.
//   warp 0      TMA producer (both CTAs): one 128x128 int8 box of A and one of B
//               per stage into a STAGES-deep ring of 128-byte-swizzled shared
//               memory; both CTAs' boxes complete on the leader's full barrier.
//   warp 1      allocates 512 TMEM columns (pair allocation); in the leader one
//               lane issues 4 MMAs of 256 x 256 x 32 per stage and commits each
//               stage back to both producers and each finished tile to both
//               epilogues.
//   warps 2-9   epilogue (both CTAs): each warp takes a 32-lane quarter of the
//               CTA's 128 accumulator rows and half of the columns; the tile's
//               column scales and biases are staged in shared memory first;
//               tcgen05.ld, fp32 rescale, bias, bf16 (or SwiGLU), stores; then
//               they free the accumulator on the leader's barrier.
// Two 256-column accumulators let the epilogue of tile i overlap the main loop
// of tile i+1. Tiles are walked in groups of row blocks (the group's A tiles are
// reused from L2 by every N block; each B tile is read once per group). No load
// uses cluster multicast.
//
// SwiGLU: the B tile of an output tile holding h columns [j0, j0+128) stacks
// gate rows [j0, j0+128) (in the leader) over up rows [F+j0, F+j0+128) (in the
// peer) of the plain [gate; up] weight, so each CTA's 128 x 256 accumulator
// holds both halves and silu(g) * u is formed per element in the epilogue. This gives the locality that the pages get
// by interleaving gate/up rows at load, without repacking the weight.
//
// Every wait is bounded (see mbar_wait_bounded); past the limit the pair
// records a timeout, drains its copies and MMAs (bounded again), frees its
// tensor memory and exits.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "ptx_sm100.cuh"

namespace h3q {

constexpr int kBM = 128;  // rows per CTA; a CTA pair computes 256-row tiles
constexpr int kBN = 256;  // output columns per tile; each CTA holds 128 rows of B
constexpr int kBK = 128;  // int8 elements = 128 bytes = one swizzle row
constexpr int kStages = 6;
constexpr int kAStage = kBM * kBK;  // 16 KB
constexpr int kBStage = 128 * kBK;  // 16 KB: this CTA's half of the B tile
constexpr int kTmemCols = 512;
constexpr int kGemmThreads = 320;  // producer, MMA, 8 epilogue warps
constexpr size_t kGemmSmem =
    size_t(kStages) * (kAStage + kBStage) + 1024 /*align*/ + 256 /*barriers*/ + 4 * kBN * 4 /*column scales, biases*/;

enum EpiKind : int { kEpiS32 = 0, kEpiBF16 = 1, kEpiSwiGLU = 2 };

struct GemmParams {
  int M;            // rows of A / output
  int N;            // output columns (SwiGLU: F)
  int K;
  int num_m, num_n, num_tiles;
  int raster;       // tile order: see tile_coords
  int group_m;      // pair-row blocks per group (raster 0)
  int pol_a, pol_b; // L2 policy of the A and B tile loads: 0 evict-first, 1 evict-last, 2 evict-normal
  int b_row_up;     // SwiGLU: first up row of B (= F)
  const float* sx;  // [M]
  const float* sw;  // [N] (SwiGLU: [2F])
  const __nv_bfloat16* bias;  // nullable, [N] (SwiGLU: [2F])
  void* out;        // [M, N] int32 or bf16 (SwiGLU: [M, F] bf16)
  uint64_t wait_limit_ns;
};

// Tile order. raster 0: groups of group_m pair-row blocks; within a group the
// row blocks vary fastest, so the group's A tiles are reused from L2 by every N
// block and each B tile is read once per group. raster 1: all row blocks of one
// N block before the next N block.
__device__ __forceinline__ void tile_coords(int tile, const GemmParams& p, int& mb, int& nb) {
  if (p.raster == 1) {
    mb = tile % p.num_m;
    nb = tile / p.num_m;
    return;
  }
  const int per_group = p.group_m * p.num_n;
  const int gid = tile / per_group;
  const int first_m = gid * p.group_m;
  const int gm = min(p.num_m - first_m, p.group_m);
  const int r = tile - gid * per_group;
  mb = first_m + r % gm;
  nb = r / gm;
}

// silu(g) = g / (1 + e^-g) in fp32 (SwiGLU, h3-rs README, "What makes it fast").
// e^t = p * 2^n: Cody-Waite reduction t = n ln2 + r with n = rne(t log2 e) and
// fdlibm's two-part ln2 (0x3f317200, 0x35bfbe8e), p = e^r by the degree-7 Taylor
// polynomial in Horner form with fused multiply-adds. For t < -20, 1 + e^t is 1
// in fp32 (silu(g) = g). For n <= 64 the quotient is g / (1 + p 2^n), with 2^n
// applied by one exact multiply. For n > 64, 1 + e^t rounds to p 2^n, and the
// quotient is formed as (g 2^(64-n)) / (p 2^64): both operands exact, so it is
// the same correctly rounded quotient, and it stays right where e^t overflows
// fp32 (g < -88.72) down to where silu underflows. g < -120 gives -0.
__device__ __forceinline__ float silu_f32(float g) {
  const float t = -g;
  if (t < -20.0f) return g;
  if (t > 120.0f) return -0.0f;
  // n = rne(t log2 e): adding 1.5 * 2^23 rounds to an integer (ties to even) and
  // leaves it in the low mantissa bits
  const float nm = __fadd_rn(__fmul_rn(t, 1.44269502f), 12582912.0f);
  const float n = __fsub_rn(nm, 12582912.0f);
  const int ni = __float_as_int(nm) - 0x4B400000;
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
  if (__builtin_expect(ni > 64, 0))
    return __fdiv_rn(__fmul_rn(g, __int_as_float((191 - ni) << 23)), __fmul_rn(p, 18446744073709551616.0f));
  return __fdiv_rn(g, __fadd_rn(1.0f, __fmul_rn(p, __int_as_float((ni + 127) << 23))));
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
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
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_i8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  // identical offsets in both CTAs of the pair: the leader's MMA addresses the
  // peer's operand tiles through the same shared-memory offsets
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
  float* col_scale = reinterpret_cast<float*>(smem + kStages * (kAStage + kBStage) + 256);  // [2][kBN]
  float* col_bias = col_scale + 2 * kBN;                                                      // [2][kBN]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0 = leader: issues the pair's MMAs
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int KB = p.K / kBK;
  const uint64_t limit = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);   // leader's: its expect_tx; both CTAs' boxes complete on it
      mbar_init(&empty[s], 1);  // the leader's MMA commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);   // the leader's MMA commit
      mbar_init(&tempty[b], 16);  // leader's: 8 epilogue warps of each CTA
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
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any cross-CTA use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer (both CTAs)
      auto policy = [](int k) {
        return k == 0 ? policy_evict_first() : (k == 1 ? policy_evict_last() : policy_evict_normal());
      };
      const uint64_t pol_a = policy(p.pol_a);
      const uint64_t pol_b = policy(p.pol_b);
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < p.num_tiles; tile += npairs) {
        int mb, nb;
        tile_coords(tile, p, mb, nb);
        const int a_row = mb * (2 * kBM) + static_cast<int>(rank) * kBM;
        const int b_row = (EPI == kEpiSwiGLU) ? (rank == 0 ? nb * 128 : p.b_row_up + nb * 128)
                                              : nb * kBN + static_cast<int>(rank) * 128;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, limit, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t full_leader = cluster_map(&full[stage], 0);
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * (kAStage + kBStage));
          tma_load_2d_pair(sA + stage * kAStage, &tmA, full_leader, kb * kBK, a_row, pol_a);
          tma_load_2d_pair(sB + stage * kBStage, &tmB, full_leader, kb * kBK, b_row, pol_b);
          ++issued;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && rank == 0) {
        // drain the pair's copies still in flight (bounded, ignores abort)
        for (int s = 0; s < kStages; ++s) {
          if (issued <= s) continue;
          const long last = ((issued - 1 - s) / kStages) * kStages + s;
          mbar_wait_bounded(&full[s], static_cast<uint32_t>((last / kStages) & 1), limit, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------------ MMA issuer (leader only)
      constexpr uint32_t idesc = idesc_i8(2 * kBM, kBN);
      int stage = 0;
      uint32_t phase = 0;
      int buf = 0;
      uint32_t buf_phase = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < p.num_tiles; tile += npairs) {
        if (!mbar_wait_bounded_cluster(&tempty[buf], buf_phase ^ 1u, limit, abort_flag)) break;
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
            mma_i8_pair(d, ad + 2u * k, bd + 2u * k, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          mma_commit_pair(cluster_map(&empty[stage], 0));
          mma_commit_pair(cluster_map(&empty[stage], 1));
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair(cluster_map(&tfull[buf], 0));
        mma_commit_pair(cluster_map(&tfull[buf], 1));
        buf ^= 1;
        if (buf == 0) buf_phase ^= 1u;
      }
      // every MMA this pair issued has completed once `drain` fires
      mma_commit_pair(cluster_map(drain, 0));
      mbar_wait_bounded(drain, 0, limit, nullptr);
    }
  } else {
    // -------------------------------------------------------------- epilogue (both CTAs)
    // Warps 2..9: warp w reads TMEM lanes 32*(w%4) .. +31 (its quarter of the
    // CTA's 128 rows) and one half of the tile's columns.
    const int quarter = warp & 3;
    const int chalf = (warp - 2) >> 2;
    const int et = threadIdx.x - 64;  // 0 .. 255
    const int row_in_tile = static_cast<int>(rank) * kBM + quarter * 32 + lane;
    const uint32_t tempty_leader0 = cluster_map(&tempty[0], 0);
    const uint32_t tempty_leader1 = cluster_map(&tempty[1], 0);
    const bool has_bias = p.bias != nullptr;
    int buf = 0;
    uint32_t buf_phase = 0;
    int iter = 0;
    for (int tile = pair; tile < p.num_tiles; tile += npairs, ++iter) {
      int mb, nb;
      tile_coords(tile, p, mb, nb);
      float* cs = col_scale + (iter & 1) * kBN;  // this tile's 256 column scales ...
      float* cb = col_bias + (iter & 1) * kBN;   // ... and biases, staged once per tile
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
        cs[et] = valid ? __ldg(p.sw + n) : 0.0f;
        cb[et] = (valid && has_bias) ? __bfloat162float(p.bias[n]) : 0.0f;
        named_barrier(1, 256);
      }
      if (!mbar_wait_bounded_cluster(&tfull[buf], buf_phase, limit, abort_flag)) break;
      tc_fence_after();
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(buf * kBN);
      const int row = mb * (2 * kBM) + row_in_tile;
      const bool row_ok = row < p.M;
      if constexpr (EPI == kEpiS32) {
        int32_t* out = static_cast<int32_t*>(p.out) + static_cast<int64_t>(row) * p.N;
#pragma unroll 1
        for (int c = 4 * chalf; c < 4 * chalf + 4; ++c) {
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
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + static_cast<int64_t>(row) * p.N;
#pragma unroll 1
        for (int c = 4 * chalf; c < 4 * chalf + 4; ++c) {
          uint32_t r[32];
          tmem_ld32(taddr + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int i0 = c * 32 + 8 * g;  // column within the tile
            const int n = nb * kBN + i0;
            if (n < p.N) {
              uint32_t o[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int k = i0 + 2 * i;
                const float v0 = rescale(r[8 * g + 2 * i], sxr, cs[k], cb[k], has_bias);
                const float v1 = rescale(r[8 * g + 2 * i + 1], sxr, cs[k + 1], cb[k + 1], has_bias);
                o[i] = pack_bf16x2(v0, v1);
              }
              if (row_ok) *reinterpret_cast<uint4*>(out + n) = make_uint4(o[0], o[1], o[2], o[3]);
            }
          }
        }
      } else {  // SwiGLU: accumulator columns [0,128) gate, [128,256) up
        const float sxr = row_ok ? __ldg(p.sx + row) : 0.0f;
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + static_cast<int64_t>(row) * p.N;
#pragma unroll 1
        for (int c = 2 * chalf; c < 2 * chalf + 2; ++c) {
          uint32_t rg[32], ru[32];
          tmem_ld32(taddr + c * 32, rg);
          tmem_ld32(taddr + 128 + c * 32, ru);
          tmem_ld_wait();
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int i0 = c * 32 + 8 * g;  // gate column within the tile; up column is 128 + i0
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              float h[2];
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int k = i0 + 2 * i + e;
                const float gv = rescale(rg[8 * g + 2 * i + e], sxr, cs[k], cb[k], has_bias);
                const float uv = rescale(ru[8 * g + 2 * i + e], sxr, cs[128 + k], cb[128 + k], has_bias);
                h[e] = __fmul_rn(silu_f32(gv), uv);
              }
              o[i] = pack_bf16x2(h[0], h[1]);
            }
            if (row_ok) *reinterpret_cast<uint4*>(out + nb * 128 + i0) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(buf == 0 ? tempty_leader0 : tempty_leader1);
      buf ^= 1;
      if (buf == 0) buf_phase ^= 1u;
    }
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync();  // the leader's MMAs read the peer's shared memory: both stay until all are done
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, kTmemCols);
}

// Test kernel for the bounded-wait path: waits on an mbarrier that nothing ever
// arrives on; the wait gives up after limit_ns and records the timeout.
__global__ void stalled_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag[2];
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag[0] = 0;
    abort_flag[1] = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  // thread 0 through the issuing-thread helper, warp 1 through the ring-consumer
  // helper, each with its own abort flag so that each runs into its own limit
  if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, limit_ns, &abort_flag[0]);
  if (threadIdx.x >= 32) mbar_wait_bounded_lazy(&bar, 0, limit_ns, &abort_flag[1]);
  __syncthreads();
}

}  // namespace h3q
