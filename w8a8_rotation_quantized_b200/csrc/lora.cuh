// LoRA merge into stored rotated int8 weights: the low-rank delta alpha * B A of a
// LoRA is folded into the int8 weights once, at load, by dequantizing, adding and
// requantizing (h3-rs README, "Speed", "What makes it fast"), so it costs nothing
// per step. The stored codes live in the rotated basis (W R_K), so A is rotated
// along K first: W' R_K = W R_K + alpha B (A R_K).
//
// Two kernels:
//  * lora_rotate_kernel: A [r, K] fp32 -> A R_K [r, K] fp32. One warp per
//    256-group, lane l holding elements 8l..8l+7; every element is scaled by
//    1/16 first, then the radix-2 butterflies of index bits 0-2 run in
//    registers and those of bits 3-7 across lanes (shuffle). Ascending bit order
//    with one rounded add or subtract per butterfly gives the bits of the
//    pairwise-tree sum of the explicit (H/16) product.
//  * lora_merge_kernel<R>: a cluster of CS CTAs owns R weight rows; each CTA
//    owns a contiguous slice of the K columns of those rows. Per element, in fp32:
//    d = fma chain over the rank index j ascending (from 0) of B[n][j] A_rot[j][k];
//    w = q s + alpha d (two rounded products, one rounded add). The CTA keeps its
//    slice of w in shared memory, reduces max |w| per row, and the cluster
//    combines the CTAs' maxima through distributed shared memory; then every CTA
//    requantizes its slice: s' = max / 127, q' = clamp(rne(w / s'), +-127), with
//    s' = 0 giving q' = 0. The codes and scales are updated in place.
//
// Cost: 2 N K r fp32 flops against N K bytes read and N K bytes written, so for
// ranks above a few the kernel is bound by the fp32 FMA pipe, not by HBM. The
// accumulators hold pairs of rows so each FMA instruction is the sm_100 two-wide
// fp32 FMA; A_rot (r K 4 bytes) stays in L2 and every row block streams it once.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "ptx_sm100.cuh"

namespace h3q {

constexpr int kLoraMaxRank = 512;
#ifndef H3Q_LORA_UNROLL
#define H3Q_LORA_UNROLL 1
#endif
#ifndef H3Q_LORA_THREADS
#define H3Q_LORA_THREADS 256
#endif
constexpr int kLoraUnroll = H3Q_LORA_UNROLL;  // rank steps unrolled in the product loop
constexpr int kLoraMaxThreads = 512;          // launch bound of the merge kernel
constexpr int kLoraPlanThreads = H3Q_LORA_THREADS;  // threads per CTA the plan aims for
constexpr int kLoraMaxCluster = 8;
#ifndef H3Q_LORA_RING
#define H3Q_LORA_RING 8
#endif
#ifndef H3Q_LORA_SLICE_KB
#define H3Q_LORA_SLICE_KB 64
#endif
#ifndef H3Q_LORA_MAX_ROWS
#define H3Q_LORA_MAX_ROWS 16
#endif
constexpr int kLoraRing = H3Q_LORA_RING;  // A_rot rows in flight per thread (a power of two)
static_assert((kLoraRing & (kLoraRing - 1)) == 0, "ring depth must be a power of two");

// 16-byte global -> shared copy through L2 only (the per-thread async copy of
// sm_80 and later), its commit and its bounded-depth wait.
__device__ __forceinline__ void cp_async_16(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ float ld_shared_cluster_f32(uint32_t cluster_addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(cluster_addr) : "memory");
  return v;
}

// A [rows, K] -> A R_K, where `groups` = rows * K / 256.
__global__ void __launch_bounds__(256) lora_rotate_kernel(const float* __restrict__ a, int64_t groups,
                                                          float* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t g = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (g >= groups) return;
  const float4* src = reinterpret_cast<const float4*>(a + g * 256 + lane * 8);
  const float4 lo = src[0], hi = src[1];
  float v[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(v[i], 0.0625f);
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i & h) continue;
      const float x = v[i], y = v[i | h];
      v[i] = __fadd_rn(x, y);
      v[i | h] = __fsub_rn(x, y);
    }
  }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, v[i], m);
      v[i] = upper ? __fsub_rn(o, v[i]) : __fadd_rn(v[i], o);
    }
  }
  float4* dst = reinterpret_cast<float4*>(out + g * 256 + lane * 8);
  dst[0] = make_float4(v[0], v[1], v[2], v[3]);
  dst[1] = make_float4(v[4], v[5], v[6], v[7]);
}

struct LoraArgs {
  int64_t N;      // weight rows
  int K;          // columns (multiple of 256)
  int r;          // rank
  float alpha;
  int cs;         // CTAs per cluster (the K slices of one row block)
  int qpc;        // column quads per CTA slice
};

// 4-byte global -> shared async copy (through L1), for the code bytes a thread
// dequantizes itself.
__device__ __forceinline__ void cp_async_4(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}

// Byte k of `codes` (an int8) as an exact float: the byte, offset by 128, is
// placed in the low mantissa bits of 1.5 * 2^23 and the offset subtracted.
template <int k>
__device__ __forceinline__ float code_to_float(uint32_t codes_x80) {
  return __fsub_rn(__uint_as_float(__byte_perm(codes_x80, 0x4B400000u, 0x7650u | k)), 12583040.0f);
}

template <int R>
__global__ void __launch_bounds__(kLoraMaxThreads, 1)
    lora_merge_kernel(int8_t* __restrict__ wq, float* __restrict__ sw, const float* __restrict__ a_rot,
                      const float* __restrict__ b, LoraArgs p) {
  static_assert(R % 4 == 0, "rows come in float4 loads of B");
  extern __shared__ __align__(16) float lora_smem[];
  const int nthreads = blockDim.x;
  const int cols = 4 * p.qpc;
  float* bt = lora_smem;                                             // [r][R]: B transposed, 0 past row N
  float* wbuf = bt + p.r * R;                                        // [R][cols]: merged fp32 weights
  float4* ring = reinterpret_cast<float4*>(wbuf + R * cols);         // [kLoraRing][threads]: A_rot rows
  uint32_t* qbuf = reinterpret_cast<uint32_t*>(ring + kLoraRing * nthreads);  // [R][threads]: old codes
  __shared__ float amax_part[R];
  __shared__ float s_old[R];
  __shared__ float4 quot[R];  // per row: f, s f, 1 / (s f), s

  const int tid = threadIdx.x;
  const uint32_t rank = cluster_ctarank();
  const int64_t row0 = int64_t(blockIdx.x / p.cs) * R;
  const int Q = p.K >> 2;
  const int q0 = int(rank) * p.qpc;
  const int q1 = min(Q, q0 + p.qpc);
  const int64_t K = p.K;

  for (int i = tid; i < p.r * R; i += nthreads) {
    const int rr = i / p.r, j = i - rr * p.r;
    const int64_t n = row0 + rr;
    bt[j * R + rr] = n < p.N ? b[n * p.r + j] : 0.0f;
  }
  if (tid < R) s_old[tid] = row0 + tid < p.N ? sw[row0 + tid] : 0.0f;
  __syncthreads();

  const float4* a4 = reinterpret_cast<const float4*>(a_rot);
  for (int qd = q0 + tid; qd < q1; qd += nthreads) {
    // The codes this thread dequantizes, fetched now so HBM latency overlaps
    // the products (the oldest commit group, complete at the first ring wait).
#pragma unroll
    for (int rr = 0; rr < R; ++rr)
      if (row0 + rr < p.N) cp_async_4(qbuf + rr * nthreads + tid, wq + (row0 + rr) * K + 4 * int64_t(qd));
    cp_async_commit();

    float2 acc[R / 2][4];
#pragma unroll
    for (int rp = 0; rp < R / 2; ++rp)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[rp][c] = make_float2(0.0f, 0.0f);
    // Each thread streams its own column quad of A_rot rows j through a ring of
    // kLoraRing shared-memory slots; one commit group per row keeps the count
    // uniform, so waiting until at most kLoraRing - 1 groups are pending means
    // row j has landed. A slot is refilled only after its value was consumed.
#pragma unroll
    for (int j = 0; j < kLoraRing - 1; ++j) {
      if (j < p.r) cp_async_16(ring + j * nthreads + tid, a4 + int64_t(j) * Q + qd);
      cp_async_commit();
    }
#pragma unroll kLoraUnroll
    for (int j = 0; j < p.r; ++j) {
      const int jn = j + kLoraRing - 1;
      if (jn < p.r) cp_async_16(ring + (jn & (kLoraRing - 1)) * nthreads + tid, a4 + int64_t(jn) * Q + qd);
      cp_async_commit();
      cp_async_wait<kLoraRing - 1>();
      const float4 av = ring[(j & (kLoraRing - 1)) * nthreads + tid];
      const float4* bj = reinterpret_cast<const float4*>(bt + j * R);
      const float2 ac[4] = {make_float2(av.x, av.x), make_float2(av.y, av.y), make_float2(av.z, av.z),
                            make_float2(av.w, av.w)};
#pragma unroll
      for (int r4 = 0; r4 < R / 4; ++r4) {
        const float4 bv = bj[r4];
        const float2 b01 = make_float2(bv.x, bv.y), b23 = make_float2(bv.z, bv.w);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          acc[2 * r4][c] = __ffma2_rn(b01, ac[c], acc[2 * r4][c]);
          acc[2 * r4 + 1][c] = __ffma2_rn(b23, ac[c], acc[2 * r4 + 1][c]);
        }
      }
    }
#pragma unroll
    for (int rr = 0; rr < R; ++rr) {
      float4 wv = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      if (row0 + rr < p.N) {
        // w = q s + alpha d: two rounded products and one rounded add, each a
        // separate scalar op so that nothing contracts into a fused multiply-add.
        const uint32_t c = qbuf[rr * nthreads + tid] ^ 0x80808080u;
        const float s = s_old[rr];
        const float d0 = (rr & 1) ? acc[rr >> 1][0].y : acc[rr >> 1][0].x;
        const float d1 = (rr & 1) ? acc[rr >> 1][1].y : acc[rr >> 1][1].x;
        const float d2 = (rr & 1) ? acc[rr >> 1][2].y : acc[rr >> 1][2].x;
        const float d3 = (rr & 1) ? acc[rr >> 1][3].y : acc[rr >> 1][3].x;
        wv.x = __fadd_rn(__fmul_rn(code_to_float<0>(c), s), __fmul_rn(p.alpha, d0));
        wv.y = __fadd_rn(__fmul_rn(code_to_float<1>(c), s), __fmul_rn(p.alpha, d1));
        wv.z = __fadd_rn(__fmul_rn(code_to_float<2>(c), s), __fmul_rn(p.alpha, d2));
        wv.w = __fadd_rn(__fmul_rn(code_to_float<3>(c), s), __fmul_rn(p.alpha, d3));
      }
      *reinterpret_cast<float4*>(wbuf + rr * cols + 4 * (qd - q0)) = wv;
    }
  }
  __syncthreads();

  // max |w| of each row over this CTA's slice: one warp per row, round robin.
  const int warp = tid >> 5, lane = tid & 31, nwarps = nthreads >> 5;
  const int slice_quads = q1 > q0 ? q1 - q0 : 0;
  for (int rr = warp; rr < R; rr += nwarps) {
    const float4* row = reinterpret_cast<const float4*>(wbuf + rr * cols);
    float m = 0.0f;
    for (int i = lane; i < slice_quads; i += 32) {
      const float4 v = row[i];
      m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) amax_part[rr] = m;
  }
  cluster_sync();  // every CTA's slice maxima are visible cluster-wide
  if (tid < R) {
    float m = 0.0f;
    for (int c = 0; c < p.cs; ++c) m = fmaxf(m, ld_shared_cluster_f32(cluster_map(&amax_part[tid], uint32_t(c))));
    const float s = __fdiv_rn(m, 127.0f);
    // w / s is formed as (w f) / (s f), f = 2^64 when s < 2^-100 (exact), from
    // rs = RN(1 / (s f)) and two exact-residual refinements (Markstein): the
    // correctly rounded quotient. rs = 0 for an all-zero row.
    const float f = s < 0x1p-100f ? 0x1p64f : 1.0f;
    const float sf = __fmul_rn(s, f);
    quot[tid] = make_float4(f, sf, s != 0.0f ? __frcp_rn(sf) : 0.0f, s);
    if (rank == 0 && row0 + tid < p.N) sw[row0 + tid] = s;
  }
  __syncthreads();

  const float2 magic = make_float2(12582912.0f, 12582912.0f);
  const float2 hi = make_float2(127.0f, 127.0f), lo = make_float2(-127.0f, -127.0f);
  for (int qd = q0 + tid; qd < q1; qd += nthreads) {
#pragma unroll 4
    for (int rr = 0; rr < R; ++rr) {
      const int64_t n = row0 + rr;
      if (n >= p.N) continue;
      const float4 qt = quot[rr];
      const float2 f2 = make_float2(qt.x, qt.x), ns2 = make_float2(-qt.y, -qt.y), r2 = make_float2(qt.z, qt.z);
      const float4 wv = *reinterpret_cast<const float4*>(wbuf + rr * cols + 4 * (qd - q0));
      uint32_t code[4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float2 y = __fmul2_rn(h ? make_float2(wv.z, wv.w) : make_float2(wv.x, wv.y), f2);
        float2 q = __fmul2_rn(y, r2);
        float2 e = __ffma2_rn(q, ns2, y);
        q = __ffma2_rn(e, r2, q);
        e = __ffma2_rn(q, ns2, y);
        q = __ffma2_rn(e, r2, q);
        q = make_float2(fminf(fmaxf(q.x, lo.x), hi.x), fminf(fmaxf(q.y, lo.y), hi.y));
        const float2 u = __fadd2_rn(q, magic);  // round half to even; the low byte is the code
        code[2 * h] = __float_as_uint(u.x);
        code[2 * h + 1] = __float_as_uint(u.y);
      }
      const uint32_t packed = __byte_perm(__byte_perm(code[0], code[1], 0x0040u), __byte_perm(code[2], code[3], 0x0040u),
                                          0x5410u);
      *reinterpret_cast<uint32_t*>(wq + n * K + 4 * int64_t(qd)) = packed;
    }
  }
  cluster_sync();  // no CTA leaves while a peer may still read its amax_part
}

// ----------------------------------------------------------------------------
// Host side.

struct LoraShape {
  int rows;     // R
  int cs;       // CTAs per cluster
  int qpc;      // column quads per CTA
  int threads;
  size_t smem;  // dynamic shared memory bytes
};

// Dynamic shared memory of one CTA: B^T, the fp32 slice, the A_rot ring and the
// prefetched codes.
inline size_t lora_smem_bytes(int rows, int r, int qpc, int threads) {
  return size_t(r) * rows * 4 + size_t(rows) * 4 * qpc * 4 + size_t(kLoraRing) * threads * 16 +
         size_t(rows) * threads * 4;
}

// Shape for [N, K] weights and rank r: R = 16 rows per cluster when the row
// block fits in at most 8 CTAs, else 8 rows; the fewest CTAs per cluster whose
// fp32 slice stays within the slice budget (64 KiB by default) and whose whole
// footprint fits in shared memory; about 256 threads per CTA, each owning whole
// column quads. At K = 5376 that is 6 CTAs of 224 threads and ~100 KiB each, two
// per SM, so one CTA's row-max and requantize phases overlap the other's
// products. Returns rows = 0 if nothing fits (not reached for K <= 16384 and
// r <= 512).
inline LoraShape lora_plan(int64_t K, int r) {
  const int64_t slice_budget = int64_t(H3Q_LORA_SLICE_KB) * 1024;
  const size_t limit = 227 * 1024 - 1024;  // dynamic limit, less the static arrays
  const int Q = int(K / 4);
  for (int rows : {16, 8}) {
    if (rows > H3Q_LORA_MAX_ROWS) continue;
    const int64_t bytes = int64_t(rows) * K * 4;
    int cs = int((bytes + slice_budget - 1) / slice_budget);
    if (rows == 8 && cs > kLoraMaxCluster) cs = kLoraMaxCluster;  // last option: over budget, 8 CTAs
    for (cs = cs < 1 ? 1 : cs; cs <= kLoraMaxCluster; ++cs) {
      LoraShape sh{};
      sh.rows = rows;
      sh.cs = cs;
      sh.qpc = (Q + cs - 1) / cs;
      const int iters = (sh.qpc + kLoraPlanThreads - 1) / kLoraPlanThreads;
      const int per = (sh.qpc + iters - 1) / iters;
      sh.threads = ((per + 31) / 32) * 32;
      sh.smem = lora_smem_bytes(rows, r, sh.qpc, sh.threads);
      if (sh.smem <= limit) return sh;
    }
  }
  return LoraShape{};
}

template <int R>
cudaError_t launch_lora_merge_t(const LoraShape& sh, int8_t* wq, float* sw, const float* a_rot, const float* b,
                                const LoraArgs& a, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(lora_merge_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(sh.smem));
  if (e != cudaSuccess) return e;
  const int64_t blocks = (a.N + R - 1) / R;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks * sh.cs), 1, 1);
  cfg.blockDim = dim3(static_cast<unsigned>(sh.threads), 1, 1);
  cfg.dynamicSmemBytes = sh.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(sh.cs);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, lora_merge_kernel<R>, wq, sw, a_rot, b, a);
}

// a_rot_ws receives A R_K ([r, K] fp32) and is then read by the merge.
inline cudaError_t launch_lora_merge(int8_t* wq, float* sw, int64_t N, int64_t K, const float* lora_a,
                                     const float* lora_b, int r, float alpha, float* a_rot_ws, cudaStream_t stream) {
  const int64_t groups = int64_t(r) * K / 256;
  const unsigned rot_blocks = static_cast<unsigned>((groups + 7) / 8);
  lora_rotate_kernel<<<rot_blocks, 256, 0, stream>>>(lora_a, groups, a_rot_ws);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const LoraShape sh = lora_plan(K, r);
  if (sh.rows == 0) return cudaErrorInvalidConfiguration;
  LoraArgs a;
  a.N = N;
  a.K = static_cast<int>(K);
  a.r = r;
  a.alpha = alpha;
  a.cs = sh.cs;
  a.qpc = sh.qpc;
  if (sh.rows == 16) return launch_lora_merge_t<16>(sh, wq, sw, a_rot_ws, lora_b, a, stream);
  return launch_lora_merge_t<8>(sh, wq, sw, a_rot_ws, lora_b, a, stream);
}

}  // namespace h3q
