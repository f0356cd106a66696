// int8 attention for the DiT blocks (h3-rs README, "What makes it fast": an
// int8 Q.K^T / 16-bit P.V flash kernel). Per head (head dim 128, columns
// h*128 .. h*128+127 of the [S, ld] q, k, v and out matrices):
//   Q and K rows are quantized per token (s = max|x| / 127 in fp32, codes
//   clamp(rne(x / s)), as the weight rows of the linear layers);
//   s_ij = acc_ij * qs_i * ks_j / sqrt(128) with acc the exact int32 dot product;
//   O_i = softmax_j(s_i) V, with P in bf16 and fp32 accumulation.
//
// attn_prep_kernel: one block per (64-token tile, head): Q and K codes and
// scales, and V transposed per head (V^T [H*128, S]) so both products read
// K-major operands.
//
// attn_kernel: one CTA per (head, 128-query block); warp roles:
//   warp 0   TMA: the Q tile once, then per block of 128 keys the K tile (a
//            three-stage ring, released once S_j = Q K_j^T is done) and the
//            V^T tile with the key scales (a two-stage ring, released once
//            P_j V_j is done);
//   warp 1   tensor memory (512 columns: two 128-column score buffers and the
//            128-column output accumulator O); one lane issues S_j = Q K_j^T
//            (kind::i8, 128 x 128 x 128) into score buffer j % 2, then
//            O += P_{j-1} V_{j-1} (kind::f16, bf16 in, fp32 accumulation),
//            so S_j is computed while the softmax works on block j-1;
//   warps 2-17 softmax, four threads per query row (tensor-memory lane), each
//            with 32 keys of the block: reads its score slice, scales it with
//            the key scales, exchanges the part-row maxima through shared
//            memory and a bounded mbarrier, keeps a running maximum m and sum l
//            (fp32, of the unrounded weights), writes P = 2^(s - m) as bf16
//            into its four 16-byte chunks of the 128-byte swizzled P tile
//            (double-buffered), and at the end writes its 32 columns of O / l.
//            The maximum used for the exponent is raised only when a row's
//            maximum grows by more than 2^8 (P stays below 256); O is then
//            rescaled in tensor memory after the previous P.V has completed.
// Every wait is bounded (the kernel records a timeout and drains).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "gemm_sm100.cuh"
#include "ptx_sm100.cuh"

namespace h3q {

constexpr int kAttD = 128;                 // head dimension
constexpr int kAttBlk = 128;               // queries per CTA, keys per block
constexpr int kAttQBytes = 128 * 128;      // int8 Q tile
constexpr int kAttKBytes = 128 * 128;      // int8 K tile
constexpr int kAttVBytes = 2 * 128 * 128;  // bf16 V^T tile (128 d rows x 128 keys), two 64-key boxes
constexpr int kAttPBytes = 2 * 128 * 128;  // bf16 P tile (128 rows x 128 keys), two 64-key halves
constexpr int kAttKStages = 3;  // K ring: K_{j+3} loads once S_j = Q K_j^T is done
constexpr int kAttVStages = 2;  // V^T ring (with the key scales): V_{j+2} loads once P_j V_j is done
constexpr int kAttParts = 4;      // softmax threads per query row (32 keys of a block each)
constexpr int kAttThreads = 64 + 128 * kAttParts;  // producer, MMA, 16 softmax warps
constexpr int kAttKsBytes = 128 * 4;  // the key block's scales
constexpr size_t kAttSmem = size_t(kAttQBytes) + kAttKStages * kAttKBytes + kAttVStages * (kAttVBytes + kAttKsBytes) +
                            2 * kAttPBytes + 2 * kAttParts * 128 * 4 /*row max exchange*/ +
                            kAttParts * 128 * 4 /*row sums*/ + 1024 + 256;

struct AttParams {
  int S, H;
  const float* qs;       // [H, S]
  const float* ks;       // [H, S]
  __nv_bfloat16* out;    // [S, ld_out], head h at columns h*128
  int64_t ld_out;
  float c;               // log2(e) / sqrt(128)
  uint64_t wait_limit_ns;
};

// Each lane of the warp writes 32 consecutive 32-bit columns of its own TMEM lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 x bf16 -> fp32, one CTA.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// kind::f16 with bf16 A and B, fp32 accumulator, K-major operands.
__host__ __device__ constexpr uint32_t idesc_bf16(uint32_t M, uint32_t N) {
  return (1u << 4)             // D format: f32
         | (1u << 7)           // A format: bf16
         | (1u << 10)          // B format: bf16
         | ((N >> 3) << 17)
         | ((M >> 4) << 24);
}

// max of three fp32 values (sm_100 three-input max).
__device__ __forceinline__ float att_max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------- prep
// Block (tile of 64 tokens, head h), 256 threads. Q/K rows: one warp per token
// (4 elements per lane); V: staged in shared memory and written transposed.
__global__ void __launch_bounds__(256) attn_prep_kernel(const __nv_bfloat16* __restrict__ q,
                                                        const __nv_bfloat16* __restrict__ k,
                                                        const __nv_bfloat16* __restrict__ v, int S, int64_t ld,
                                                        int8_t* __restrict__ qq, float* __restrict__ qs,
                                                        int8_t* __restrict__ kq, float* __restrict__ ks,
                                                        __nv_bfloat16* __restrict__ vt) {
  __shared__ uint16_t tile[64][kAttD + 2];  // +2 halves: column reads spread over banks
  const int h = blockIdx.y;
  const int t0 = blockIdx.x * 64;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int t = warp; t < 64; t += 8) {
    const int i = t0 + t;
    if (i >= S) break;
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const __nv_bfloat16* src = (which == 0 ? q : k) + int64_t(i) * ld + h * kAttD + 4 * lane;
      const uint2 w = *reinterpret_cast<const uint2*>(src);
      const float x[4] = {__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u),
                          __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xFFFF0000u)};
      float a = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
      const float s = __fdiv_rn(a, 127.0f);
      uint32_t packed = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float r = 0.0f;
        if (s != 0.0f) r = fminf(fmaxf(rintf(__fdiv_rn(x[e], s)), -127.0f), 127.0f);
        packed |= (static_cast<uint32_t>(static_cast<int>(r)) & 0xFFu) << (8 * e);
      }
      const int64_t row = int64_t(h) * S + i;
      *reinterpret_cast<uint32_t*>((which == 0 ? qq : kq) + row * kAttD + 4 * lane) = packed;
      if (lane == 0) (which == 0 ? qs : ks)[row] = s;
    }
  }
  // V tile [64 tokens][128 d] -> V^T rows h*128 + d, columns t0 .. t0+63
  for (int e = threadIdx.x; e < 64 * (kAttD / 2); e += 256) {
    const int t = e / (kAttD / 2), d2 = e % (kAttD / 2);
    const int i = t0 + t;
    uint32_t w = 0;
    if (i < S) w = *reinterpret_cast<const uint32_t*>(v + int64_t(i) * ld + h * kAttD + 2 * d2);
    tile[t][2 * d2] = static_cast<uint16_t>(w & 0xFFFFu);
    tile[t][2 * d2 + 1] = static_cast<uint16_t>(w >> 16);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kAttD * 32; e += 256) {
    const int d = e / 32, t2 = e % 32;  // tokens 2 t2, 2 t2 + 1
    const int i = t0 + 2 * t2;
    if (i >= S) continue;
    const uint32_t w = uint32_t(tile[2 * t2][d]) | (uint32_t(tile[2 * t2 + 1][d]) << 16);
    *reinterpret_cast<uint32_t*>(vt + (int64_t(h) * kAttD + d) * S + i) = w;
  }
}

// ---------------------------------------------------------------- attention
__global__ void __launch_bounds__(kAttThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const AttParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kAttQBytes;                   // [K stage][128 keys x 128 B]
  uint8_t* sV = sK + kAttKStages * kAttKBytes;     // [V stage][2 boxes: 128 d rows x 64 keys (128 B)]
  uint8_t* sP = sV + kAttVStages * kAttVBytes;     // [buffer][2 halves: 128 rows x 64 keys (128 B)]
  float* sKs = reinterpret_cast<float*>(sP + 2 * kAttPBytes);  // [V stage][128] key scales
  float* xmax = sKs + kAttVStages * 128;           // [block parity][part][128 rows]: part-row maxima
  float* xsum = xmax + 2 * kAttParts * 128;        // [part][128 rows]: part-row sums at the end
  uint64_t* bars = reinterpret_cast<uint64_t*>(xsum + kAttParts * 128);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;    // [K stage]
  uint64_t* k_empty = bars + 4;   // [K stage]
  uint64_t* v_full = bars + 7;    // [V stage]: V^T and the key scales
  uint64_t* v_empty = bars + 9;   // [V stage]
  uint64_t* s_full = bars + 11;   // [2]
  uint64_t* s_empty = bars + 13;  // [2]
  uint64_t* p_full = bars + 15;   // [2]
  uint64_t* pv_done = bars + 17;  // [2]
  uint64_t* drain = bars + 19;
  uint64_t* xchg = bars + 20;     // [2]: the softmax threads exchanged their part-row maxima
  uint64_t* xsum_bar = bars + 22; // the softmax threads stored their part-row sums
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 23);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, qb = blockIdx.x;
  const int S = p.S;
  const int nb = (S + kAttBlk - 1) / kAttBlk;
  const uint64_t limit = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int st = 0; st < kAttKStages; ++st) {
      mbar_init(&k_full[st], 1);
      mbar_init(&k_empty[st], 1);
    }
    for (int st = 0; st < kAttVStages; ++st) {
      mbar_init(&v_full[st], 1);
      mbar_init(&v_empty[st], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_empty[b], 4 * kAttParts);
      mbar_init(&p_full[b], 4 * kAttParts);
      mbar_init(&pv_done[b], 1);
      mbar_init(&xchg[b], 128 * kAttParts);
    }
    mbar_init(drain, 1);
    mbar_init(xsum_bar, 128 * kAttParts);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      const uint64_t pol_q = policy_evict_first();
      const uint64_t pol_kv = policy_evict_last();  // every query block of the head re-reads K and V
      mbar_arrive_expect_tx(q_full, kAttQBytes);
      tma_load_2d(sQ, &tmQ, q_full, 0, h * S + qb * kAttBlk, pol_q);
      for (int j = 0; j < nb; ++j) {
        const int kst = j % kAttKStages, vst = j % kAttVStages;
        if (!mbar_wait_bounded(&k_empty[kst], static_cast<uint32_t>(((j / kAttKStages) & 1) ^ 1), limit,
                               abort_flag))
          break;
        mbar_arrive_expect_tx(&k_full[kst], kAttKBytes);
        tma_load_2d(sK + kst * kAttKBytes, &tmK, &k_full[kst], 0, h * S + j * kAttBlk, pol_kv);
        if (!mbar_wait_bounded(&v_empty[vst], static_cast<uint32_t>(((j / kAttVStages) & 1) ^ 1), limit,
                               abort_flag))
          break;
        const uint32_t ks_bytes = static_cast<uint32_t>(min(kAttBlk, S - j * kAttBlk) * 4);  // S % 8 == 0
        mbar_arrive_expect_tx(&v_full[vst], kAttVBytes + ks_bytes);
        bulk_load(sKs + vst * 128, p.ks + int64_t(h) * S + j * kAttBlk, ks_bytes, &v_full[vst], pol_kv);
        tma_load_2d(sV + vst * kAttVBytes, &tmV, &v_full[vst], j * kAttBlk, h * kAttD, pol_kv);
        tma_load_2d(sV + vst * kAttVBytes + kAttVBytes / 2, &tmV, &v_full[vst], j * kAttBlk + 64, h * kAttD, pol_kv);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_s = idesc_i8(kAttBlk, kAttBlk);
      constexpr uint32_t idesc_o = idesc_bf16(kAttBlk, kAttD);
      bool ok = mbar_wait_bounded(q_full, 0, limit, abort_flag);
      const uint64_t qd = smem_desc_sw128(smem_u32(sQ));
      for (int j = 0; ok && j <= nb; ++j) {
        if (j < nb) {  // S_j = Q K_j^T into score buffer j % 2
          const int st = j % kAttKStages, b = j & 1;
          if (!mbar_wait_bounded(&k_full[st], static_cast<uint32_t>((j / kAttKStages) & 1), limit, abort_flag) ||
              !mbar_wait_bounded(&s_empty[b], static_cast<uint32_t>(((j >> 1) & 1) ^ 1), limit, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t kd = smem_desc_sw128(smem_u32(sK + st * kAttKBytes));
#pragma unroll
          for (int k = 0; k < 4; ++k) mma_i8(tmem + b * kAttBlk, qd + 2u * k, kd + 2u * k, idesc_s, k > 0 ? 1u : 0u);
          mma_commit(&s_full[b]);
          mma_commit(&k_empty[st]);
        }
        if (j >= 1) {  // O += P_{j-1} V_{j-1}
          const int t = j - 1, bt = t & 1, stt = t % kAttVStages;
          if (!mbar_wait_bounded(&v_full[stt], static_cast<uint32_t>((t / kAttVStages) & 1), limit, abort_flag) ||
              !mbar_wait_bounded(&p_full[bt], static_cast<uint32_t>((t >> 1) & 1), limit, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 8; ++k) {  // 16 keys = 32 bytes per K step; halves of 64 keys
            const int half = k >> 2;
            const uint64_t pd = smem_desc_sw128(smem_u32(sP + bt * kAttPBytes + half * (kAttPBytes / 2)));
            const uint64_t vd = smem_desc_sw128(smem_u32(sV + stt * kAttVBytes + half * (kAttVBytes / 2)));
            mma_bf16(tmem + 2 * kAttBlk, pd + 2u * (k & 3), vd + 2u * (k & 3), idesc_o, (t > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit(&pv_done[bt]);
          mma_commit(&v_empty[stt]);
        }
      }
      mma_commit(drain);
      mbar_wait_bounded(drain, 0, limit, nullptr);
    }
  } else {
    // -------------------------------------------------------------- softmax (warps 2..17)
    // Four threads per query row (TMEM lane): part q = (warp - 2) / 4 takes keys
    // [32 q, 32 q + 32) of each block and columns [32 q, 32 q + 32) of O. The parts
    // exchange their row maxima through shared memory and a bounded mbarrier per
    // block, so all four take the same rescale decisions.
    const int quarter = warp & 3;                     // TMEM lanes 32*quarter .. +31
    const int part = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;                // query row within the block
    const int i = qb * kAttBlk + r;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t o_cols = tmem + lane_base + 2 * kAttBlk + 32 * part;
    const float cq = __fmul_rn(i < S ? __ldg(p.qs + int64_t(h) * S + i) : 0.0f, p.c);
    float m_used = -INFINITY;
    float2 l2 = make_float2(0.0f, 0.0f);  // running sum of the weights, two partial sums
    bool ok = true;
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xFFFFFFFFu, mbar_wait_bounded(bar, parity, limit, abort_flag));
    };
    for (int j = 0; j < nb; ++j) {
      const int b = j & 1, st = j % kAttVStages;
      if (!(ok = wait_all(&s_full[b], static_cast<uint32_t>((j >> 1) & 1)))) break;
      tc_fence_after();
      uint32_t sr[32];
      tmem_ld32(tmem + lane_base + b * kAttBlk + 32 * part, sr);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[b]);
      // Raw scores s' = (float)acc * ks_j (|acc| <= 127^2 * 128 < 2^22, so the bits of
      // acc + 1.5 * 2^23 read as a float, minus 1.5 * 2^23, are (float)acc without the
      // conversion unit); the log2-domain score is s' * cq, cq = qs_i log2(e) / sqrt(128) >= 0,
      // so maxima can be taken on s'. Keys past the end (last block only) are masked.
      const int key0 = j * kAttBlk + 32 * part;
      const bool partial = key0 + 32 > S;
      // the key scales travel with V_j (that stage is released only after P_j V_j)
      if (!(ok = wait_all(&v_full[st], static_cast<uint32_t>((j / kAttVStages) & 1)))) break;
      const float* ksb = sKs + st * 128 + 32 * part;
      float mx = -INFINITY;
#pragma unroll
      for (int e4 = 0; e4 < 8; ++e4) {
        const float4 kv = *reinterpret_cast<const float4*>(ksb + 4 * e4);
        const float kk[4] = {kv.x, kv.y, kv.z, kv.w};
        float sc[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = 4 * e4 + e;
          sc[e] = __fmul_rn(__fsub_rn(__uint_as_float(sr[c] + 0x4B400000u), 12582912.0f), kk[e]);
          if (partial && key0 + c >= S) sc[e] = -INFINITY;
          sr[c] = __float_as_uint(sc[e]);
        }
        mx = att_max3(mx, att_max3(sc[0], sc[1], sc[2]), sc[3]);
      }
      float* xm = xmax + b * (kAttParts * 128);
      xm[part * 128 + r] = mx;
      mbar_arrive(&xchg[b]);
      if (!(ok = wait_all(&xchg[b], static_cast<uint32_t>((j >> 1) & 1)))) break;
      mx = att_max3(att_max3(xm[r], xm[128 + r], xm[256 + r]), xm[384 + r], -INFINITY);
      // raise the exponent's maximum when the row maximum grew by more than 2^8 (log2 units)
      const bool need = j == 0 || __fmul_rn(mx - m_used, cq) > 8.0f;
      if (__ballot_sync(0xFFFFFFFFu, need) != 0u && j > 0) {
        // O holds P.V of blocks < j with the old maximum: rescale after P_{j-1} V_{j-1} has landed
        if (!(ok = wait_all(&pv_done[(j - 1) & 1], static_cast<uint32_t>(((j - 1) >> 1) & 1)))) break;
        tc_fence_after();
        const float f = need ? ex2_approx(__fmul_rn(m_used - mx, cq)) : 1.0f;
        uint32_t o[32];
        tmem_ld32(o_cols, o);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__fmul_rn(__uint_as_float(o[e]), f));
        tmem_st32(o_cols, o);
        tmem_st_wait();
        l2 = __fmul2_rn(l2, make_float2(f, f));
      }
      if (need) m_used = mx;
      if (j >= 2) {  // P buffer b was last read by P_{j-2} V_{j-2}
        if (!(ok = wait_all(&pv_done[b], static_cast<uint32_t>(((j - 2) >> 1) & 1)))) break;
      }
      // P = 2^(s' cq - m cq) as bf16: this part's 32 keys are chunks 4 (part % 2) .. +3 of row r
      // of half-tile part / 2 (16-byte chunk c at position c ^ (r % 8) of the 128-byte row)
      const float nm = -__fmul_rn(m_used, cq);
      uint8_t* prow = sP + b * kAttPBytes + (part >> 1) * (kAttPBytes / 2) + r * 128;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c0 = 8 * cc + 2 * e;
          float p0 = ex2_approx(__fmaf_rn(__uint_as_float(sr[c0]), cq, nm));
          float p1 = ex2_approx(__fmaf_rn(__uint_as_float(sr[c0 + 1]), cq, nm));
          if (partial) {  // masked keys weigh 0 (also when cq = 0, where -inf * cq is not a number)
            if (key0 + c0 >= S) p0 = 0.0f;
            if (key0 + c0 + 1 >= S) p1 = 0.0f;
          }
          w[e] = pack_bf16x2(p0, p1);
          l2 = __fadd2_rn(l2, make_float2(p0, p1));
        }
        const int ch = 4 * (part & 1) + cc;
        *reinterpret_cast<uint4*>(prow + 16 * (ch ^ (r & 7))) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_smem();  // the tensor core reads P through the async proxy
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[b]);
    }
    if (ok) {
      const int t = nb - 1;
      ok = wait_all(&pv_done[t & 1], static_cast<uint32_t>((t >> 1) & 1));
    }
    if (ok) {
      xsum[part * 128 + r] = __fadd_rn(l2.x, l2.y);
      mbar_arrive(xsum_bar);
      ok = wait_all(xsum_bar, 0);
    }
    if (ok) {
      tc_fence_after();
      const float lsum = __fadd_rn(__fadd_rn(xsum[r], xsum[128 + r]), __fadd_rn(xsum[256 + r], xsum[384 + r]));
      const float inv_l = __fdiv_rn(1.0f, lsum);
      __nv_bfloat16* orow = p.out + int64_t(i) * p.ld_out + h * kAttD + 32 * part;
      uint32_t o[32];
      tmem_ld32(o_cols, o);
      tmem_ld_wait();
      if (i < S) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w[e] = pack_bf16x2(__fmul_rn(__uint_as_float(o[8 * g + 2 * e]), inv_l),
                               __fmul_rn(__uint_as_float(o[8 * g + 2 * e + 1]), inv_l));
          *reinterpret_cast<uint4*>(orow + 8 * g) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace h3q
