// int8 attention for the DiT blocks (h3-rs README, "What makes it fast": an
// int8 Q.K^T / 16-bit P.V flash kernel). Per head (head dim 128, columns
// h*128 .. h*128+127 of the [S, ld] q, k, v and out matrices):
//   Q rows are quantized per token (s = max|x| / 127 in fp32, codes
//   clamp(rne(x / s)), as the weight rows of the linear layers), K per block of
//   128 consecutive keys (one scale over the block's keys and dimensions), so the
//   key scale is one constant per key tile;
//   s_ij = acc_ij * qs_i * ks_b(j) / sqrt(128) with acc the exact int32 dot product;
//   O_i = softmax_j(s_i) V, with P in bf16 and fp32 accumulation.
//
// attn_prep_kernel: one block per (128-token tile, head): Q codes and scales per
// token, the tile's K codes with its one scale, and V transposed per head (V^T
// [H*128, S]) so both products read K-major operands.
//
// attn_kernel: one CTA per (head, 128-query block); warp roles:
//   warp 0   TMA: the Q tile once, then per block of 128 keys the K tile (a
//            three-stage ring, released once S_j = Q K_j^T is done) and the
//            V^T tile (a three-stage ring, released once P_j V_j is done);
//   warp 1   tensor memory (512 columns: two 128-column score buffers, the
//            128-column output accumulator O and two 64-column P buffers);
//            one lane issues O += P_j V_j (kind::f16, A = P_j from tensor
//            memory, B = V_j^T from shared memory, fp32 accumulation) once P_j
//            is written;
//   warp 3   one lane issues S_j = Q K_j^T (kind::i8, 128 x 128 x 128) into
//            score buffer j % 2 as soon as block j-2's scores have been read;
//   warp 2   idle;
//   warps 4-11 softmax, two sets of four warps, one thread per query row
//            (tensor-memory lane): set 0 takes the even key blocks, set 1 the
//            odd ones, so one set's exponentials overlap the other's score
//            loads. For its block a thread reads the whole score row, takes
//            its maximum, and writes P = 2^(s - m) as bf16 into P buffer j % 2,
//            the block's key scale folded into one multiply-add per key. The
//            maximum m used in
//            the exponent is handed from block to block through shared memory
//            (the set of block j publishes it, the set of block j+1 waits for
//            it); it is raised only when a row's maximum grows by more than
//            2^8 (P stays below 256), and O is then rescaled in tensor memory
//            after P_{j-1} V_{j-1} has completed. Each set keeps the sum of its
//            own weights; at the end the two sums are added, and set s writes
//            columns [64 s, 64 s + 64) of O / l.
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
constexpr int kAttKStages = 3;  // K ring: K_{j+3} loads once S_j = Q K_j^T is done
constexpr int kAttVStages = 3;  // V^T ring: V_{j+3} loads once P_j V_j is done
constexpr int kAttThreads = 128 + 2 * 128;  // producer, MMA (and two idle warps), two softmax sets
// Register split (setmaxnreg): the first warpgroup gives registers back, the two
// softmax warpgroups take them. The kernel is launched with at least
// kAttRegsLaunch registers per thread (the host checks the compiled count), so
// the split never asks for more than the block holds.
constexpr uint32_t kAttRegsCtl = 40, kAttRegsSoftmax = 232, kAttRegsLaunch = 168;
static_assert(128 * kAttRegsCtl + 256 * kAttRegsSoftmax <= kAttThreads * kAttRegsLaunch, "register split");
// tensor-memory columns
constexpr uint32_t kAttColS = 0;    // score buffers b at b * 128 (int32)
constexpr uint32_t kAttColO = 256;  // output accumulator (fp32)
constexpr uint32_t kAttColP = 384;  // P buffers b at 384 + b * 64 (bf16 pairs)
constexpr int kAttBiasBytes = 2 * 128 * 128;  // the bias product's two bf16 operands (128 x 64, swizzled)
constexpr size_t kAttSmem = size_t(kAttBiasBytes) + kAttQBytes + kAttKStages * kAttKBytes +
                            kAttVStages * size_t(kAttVBytes) + 2 * 128 * 4 /*maxima*/ +
                            2 * 128 * 4 /*row sums*/ + 1024 + 256;

struct AttParams {
  int S, H;
  const float* qs;       // [H, S]
  const float* ks;       // [H, ceil(S / 128)]: one scale per block of 128 keys
  __nv_bfloat16* out;    // [S, ld_out], head h at columns h*128
  int64_t ld_out;
  float c;               // log2(e) / sqrt(128)
  uint64_t wait_limit_ns;
};

// D[tmem] (+)= A[tmem] * B[smem]^T, bf16 x bf16 -> fp32, one CTA. A (M = 128
// rows in lanes 0-127) holds two bf16 per 32-bit column, the lower-indexed K
// element in the low half; one instruction reads 16 K elements (8 columns).
__device__ __forceinline__ void mma_bf16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 x bf16 -> fp32, one CTA.
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
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

template <uint32_t N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// The block's raw scores: the score products accumulate onto the bits of the fp32
// value 1.5 * 2^23 (written first by one bf16 product), and |acc| <= 127^2 * 128 <
// 2^22, so each column read as a float is F = 1.5 * 2^23 + acc exactly. Keys past
// the end (last block only) are set to -inf. Folds the 32-column chunks C0 .. C1-1
// into the running maxima mx (one chain per chunk; the caller combines the four).
template <bool kMasked, int C0, int C1>
__device__ __forceinline__ void att_raw_max(uint32_t (&sr)[4][32], int nvalid, float (&mx)[4]) {
#pragma unroll
  for (int c = C0; c < C1; ++c) {
#pragma unroll
    for (int e4 = 0; e4 < 8; ++e4) {
      const int k0 = 4 * e4;
      float sc[4] = {__uint_as_float(sr[c][k0]), __uint_as_float(sr[c][k0 + 1]), __uint_as_float(sr[c][k0 + 2]),
                     __uint_as_float(sr[c][k0 + 3])};
      if (kMasked) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (32 * c + k0 + e >= nvalid) {
            sc[e] = -INFINITY;
            sr[c][k0 + e] = __float_as_uint(-INFINITY);
          }
      }
      mx[c] = att_max3(mx[c], att_max3(sc[0], sc[1], sc[2]), sc[3]);
    }
  }
}

// P_k = 2^(F_k c - b) as bf16 pairs (lower key in the low half) into the 64 P
// columns at p_cols, F_k the raw scores of att_raw_max, c = RN(ks cq) and b =
// RN(RN(1.5 * 2^23 c) + RN(m cq)): the exponent (acc_k ks - m) cq in one fused
// multiply-add per key (F_k c is exact inside it; b differs from the exact bias by
// about one unit of acc_k c, well below the bf16 rounding of P). Returns the sum
// of the (unrounded) weights. With kMasked, keys k >= nvalid weigh 0 (also when
// c = 0, where -inf * c is not a number).
template <bool kMasked>
__device__ __forceinline__ float2 att_weights(const uint32_t (&sr)[4][32], float2 c2, float2 nb2, int nvalid,
                                              uint32_t p_cols) {
  float2 bs[4] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f),
                  make_float2(0.0f, 0.0f)};  // four partial sums, so the additions do not form one chain
#pragma unroll
  for (int hh = 0; hh < 4; ++hh) {  // 32 keys (16 P columns) per store, so each store overlaps the next keys
    uint32_t w[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int k0 = 32 * hh + 2 * e;
      const float2 t = __ffma2_rn(
          make_float2(__uint_as_float(sr[k0 >> 5][k0 & 31]), __uint_as_float(sr[k0 >> 5][(k0 & 31) + 1])), c2, nb2);
      float p0 = ex2_approx(t.x), p1 = ex2_approx(t.y);
      if (kMasked) {
        if (k0 >= nvalid) p0 = 0.0f;
        if (k0 + 1 >= nvalid) p1 = 0.0f;
      }
      w[e] = pack_bf16x2(p0, p1);
      bs[e & 3] = __fadd2_rn(bs[e & 3], make_float2(p0, p1));
    }
    tmem_st16(p_cols + 16 * hh, w);
  }
  return __fadd2_rn(__fadd2_rn(bs[0], bs[1]), __fadd2_rn(bs[2], bs[3]));
}

// ---------------------------------------------------------------- prep
// Block (tile of 128 tokens = one key block, head h), 256 threads. Every row of the
// tile (a token's 128 values of q, k or v for head h, 256 bytes) is read as sixteen
// 16-byte chunks, thread t taking chunks t + 256 n (n = 0..7): row (t + 256 n) / 16,
// chunk t % 16, so a row's chunks sit in sixteen consecutive lanes. Q: the row's
// max|x| by a 16-lane reduction, a scale per token. K: the tile's max|x| over its keys
// and dimensions gives the block's one scale. V: the chunks go to shared memory and
// leave transposed, each thread writing 16-byte runs of 8 tokens of one V^T row.
__device__ __forceinline__ void att_unpack8(const uint4& w, float (&x)[8]) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(u[i] << 16);
    x[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
  }
}

// Eight int8 codes clamp(rne(x / s)) in two words, element 0 in the low byte (0 where
// s = 0); s = RN(max|x| / 127) over a set that holds these x, so |x / s| < 128.
// rs = RN(1 / s). Fast path, as in the rotate+quantize kernel: the candidate n =
// rne(x rs) from one FMA onto 1.5 * 2^23 (the code is then the low byte of its bits)
// and the residual r = RN(x - n s) from another; |r| <= RN(s (1/2 - 2^-16)) puts x / s
// within 1/2 - 2^-16 + 2^-24 of n while RN(x / s) is within 2^-18 of x / s, so n is the
// code of the IEEE quotient. Otherwise (x / s near a half-integer), and for scales
// below 2^-100 (whose reciprocal leaves the fp32 range), the eight codes come from the
// IEEE quotients themselves.
__device__ __forceinline__ uint2 att_codes8(const float (&x)[8], float s, float rs) {
  uint32_t u[8];
  float worst = 0.0f;
  const float t = __fmul_rn(s, 0.4999847412109375f);  // 1/2 - 2^-16
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float c = __fmaf_rn(x[e], rs, 12582912.0f);
    const float n = __fsub_rn(c, 12582912.0f);
    worst = fmaxf(worst, fabsf(__fmaf_rn(-n, s, x[e])));
    u[e] = __float_as_uint(c);
  }
  if (worst > t || s < 0x1p-100f) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float r = s != 0.0f ? fminf(fmaxf(rintf(__fdiv_rn(x[e], s)), -127.0f), 127.0f) : 0.0f;
      u[e] = static_cast<uint32_t>(static_cast<int>(r));
    }
  }
  return make_uint2(__byte_perm(__byte_perm(u[0], u[1], 0x0040), __byte_perm(u[2], u[3], 0x0040), 0x5410),
                    __byte_perm(__byte_perm(u[4], u[5], 0x0040), __byte_perm(u[6], u[7], 0x0040), 0x5410));
}

__device__ __forceinline__ float att_absmax8(const float (&x)[8]) {
  float a = 0.0f;
#pragma unroll
  for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(x[e]));
  return a;
}

constexpr int kAttPrepPitch = kAttD / 2 + 1;  // words per staged V row (128 bf16 + one pad word)

__global__ void __launch_bounds__(256, 2) attn_prep_kernel(const __nv_bfloat16* __restrict__ q,
                                                        const __nv_bfloat16* __restrict__ k,
                                                        const __nv_bfloat16* __restrict__ v, int S, int64_t ld,
                                                        int8_t* __restrict__ qq, float* __restrict__ qs,
                                                        int8_t* __restrict__ kq, float* __restrict__ ks,
                                                        __nv_bfloat16* __restrict__ vt) {
  __shared__ uint32_t tile[kAttBlk * kAttPrepPitch];  // V rows (token-major), bf16 pairs
  __shared__ float warp_max[8];
  const int h = blockIdx.y;
  const int t0 = blockIdx.x * kAttBlk;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cc = threadIdx.x & 15;  // 16-byte chunk of the row: dimensions 8 cc .. 8 cc + 7
  uint4 wq[8], wk[8];  // raw bf16 chunks: every load of Q and K in flight at once
#pragma unroll
  for (int n = 0; n < 8; ++n) {
    const int row = (threadIdx.x >> 4) + 16 * n;
    const int i = t0 + row;
    wq[n] = wk[n] = make_uint4(0u, 0u, 0u, 0u);
    if (i < S) {
      const int64_t off = int64_t(i) * ld + h * kAttD + 8 * cc;
      wq[n] = *reinterpret_cast<const uint4*>(q + off);
      wk[n] = *reinterpret_cast<const uint4*>(k + off);
    }
  }
  // Q: a scale per token
#pragma unroll
  for (int n = 0; n < 8; ++n) {
    const int row = (threadIdx.x >> 4) + 16 * n;
    const int i = t0 + row;
    float x[8];
    att_unpack8(wq[n], x);
    float a = att_absmax8(x);
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
    const float sq = __fdiv_rn(a, 127.0f);
    const float rq = sq != 0.0f ? __frcp_rn(sq) : 0.0f;
    if (i < S) {
      const int64_t r = int64_t(h) * S + i;
      *reinterpret_cast<uint2*>(qq + r * kAttD + 8 * cc) = att_codes8(x, sq, rq);
      if (cc == 0) qs[r] = sq;
    }
  }
  // K: one scale for the tile's keys
  float a = 0.0f;
#pragma unroll
  for (int n = 0; n < 8; ++n) {
    float x[8];
    att_unpack8(wk[n], x);
    a = fmaxf(a, att_absmax8(x));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
  if (lane == 0) warp_max[warp] = a;
  // V rows into shared memory (loaded while the K maximum is combined)
#pragma unroll
  for (int n = 0; n < 8; ++n) {
    const int row = (threadIdx.x >> 4) + 16 * n;
    const int i = t0 + row;
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (i < S) w = *reinterpret_cast<const uint4*>(v + int64_t(i) * ld + h * kAttD + 8 * cc);
    uint32_t* dst = tile + row * kAttPrepPitch + 4 * cc;
    dst[0] = w.x;
    dst[1] = w.y;
    dst[2] = w.z;
    dst[3] = w.w;
  }
  __syncthreads();
#pragma unroll
  for (int w = 0; w < 8; ++w) a = fmaxf(a, warp_max[w]);
  const float sk = __fdiv_rn(a, 127.0f);
  const float rk = sk != 0.0f ? __frcp_rn(sk) : 0.0f;
  if (threadIdx.x == 0) ks[int64_t(h) * gridDim.x + blockIdx.x] = sk;
#pragma unroll
  for (int n = 0; n < 8; ++n) {
    const int row = (threadIdx.x >> 4) + 16 * n;
    const int i = t0 + row;
    float x[8];
    att_unpack8(wk[n], x);
    if (i < S) *reinterpret_cast<uint2*>(kq + (int64_t(h) * S + i) * kAttD + 8 * cc) = att_codes8(x, sk, rk);
  }
  // V^T: lane l takes dimension pair p = 32 (u % 2) + l (dimensions 2p, 2p + 1) and the
  // 8-token group g = 2 warp + u / 2 (u = 0..3); it reads word p of rows 8 g .. 8 g + 7
  // (consecutive lanes, consecutive words: no bank conflict) and writes 8 tokens of V^T
  // rows h*128 + 2p and h*128 + 2p + 1 as two 16-byte stores.
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int p = 32 * (u & 1) + lane;
    const int g = 2 * warp + (u >> 1);
    const int i0 = t0 + 8 * g;
    if (i0 >= S) continue;  // S % 8 == 0: a group is wholly inside or outside
    uint32_t wv[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) wv[m] = tile[(8 * g + m) * kAttPrepPitch + p];
    uint4 lo, hi;  // dimension 2p (low halves) and 2p + 1 (high halves) of tokens i0 .. i0 + 7
    lo.x = __byte_perm(wv[0], wv[1], 0x5410);
    lo.y = __byte_perm(wv[2], wv[3], 0x5410);
    lo.z = __byte_perm(wv[4], wv[5], 0x5410);
    lo.w = __byte_perm(wv[6], wv[7], 0x5410);
    hi.x = __byte_perm(wv[0], wv[1], 0x7632);
    hi.y = __byte_perm(wv[2], wv[3], 0x7632);
    hi.z = __byte_perm(wv[4], wv[5], 0x7632);
    hi.w = __byte_perm(wv[6], wv[7], 0x7632);
    *reinterpret_cast<uint4*>(vt + (int64_t(h) * kAttD + 2 * p) * S + i0) = lo;
    *reinterpret_cast<uint4*>(vt + (int64_t(h) * kAttD + 2 * p + 1) * S + i0) = hi;
  }
}

// ---------------------------------------------------------------- attention
__global__ void __launch_bounds__(kAttThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const AttParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sBias = smem;                           // [2][128 rows x 128 B]: A = e_0, B = 1.5 * 2^23 e_0
  uint8_t* sQ = sBias + kAttBiasBytes;
  uint8_t* sK = sQ + kAttQBytes;                   // [K stage][128 keys x 128 B]
  uint8_t* sV = sK + kAttKStages * kAttKBytes;     // [V stage][2 boxes: 128 d rows x 64 keys (128 B)]
  float* sMx = reinterpret_cast<float*>(sV + kAttVStages * kAttVBytes);  // [block parity][128 rows]:
                                                                         // the maximum after a block
  float* sL = sMx + 2 * 128;                       // [set][128 rows]: the sets' row sums at the end
  uint64_t* bars = reinterpret_cast<uint64_t*>(sL + 2 * 128);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;    // [K stage]
  uint64_t* k_empty = bars + 4;   // [K stage]
  uint64_t* v_full = bars + 7;    // [V stage]: V^T
  uint64_t* v_empty = bars + 10;  // [V stage]
  uint64_t* s_full = bars + 13;   // [score buffer]
  uint64_t* s_empty = bars + 15;  // [score buffer]: its scores are in the softmax threads' registers
  uint64_t* p_full = bars + 17;   // [P buffer]
  uint64_t* pv_done = bars + 19;  // [P buffer]: P_j V_j has completed
  uint64_t* mx_full = bars + 21;  // [block parity]: the maximum after the block is published
  uint64_t* l_full = bars + 23;   // both sets stored their row sums
  uint64_t* drain = bars + 24;     // the P.V issuer's products have completed
  uint64_t* drain_s = bars + 25;   // the score issuer's products have completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 26);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, qb = blockIdx.x;
  const int S = p.S;
  const int nb = (S + kAttBlk - 1) / kAttBlk;
  const uint64_t limit = p.wait_limit_ns;

  // The bias product: A = e_0 (bf16 1.0 in column 0 of every row), B = 1.5 * 2^23 e_0, so
  // A B^T writes the fp32 value 1.5 * 2^23 (bits 0x4B400000) into every score element; the
  // int8 products then accumulate onto those bits as int32 (128-byte swizzle: element 0 of
  // row m sits in 16-byte chunk m % 8).
  for (int e = threadIdx.x; e < kAttBiasBytes / 16; e += blockDim.x) {
    const int op = e / 1024, row = (e >> 3) & 127, chunk = e & 7;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (chunk == (row & 7)) v.x = op == 0 ? 0x3F80u : 0x4B40u;
    reinterpret_cast<uint4*>(sBias)[e] = v;
  }
  fence_proxy_async_smem();  // the tensor core reads them through the async proxy
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
      mbar_init(&s_empty[b], 4);   // one arrival per warp of the set
      mbar_init(&p_full[b], 4);
      mbar_init(&pv_done[b], 1);
      mbar_init(&mx_full[b], 4);
    }
    mbar_init(l_full, 8);
    mbar_init(drain, 1);
    mbar_init(drain_s, 1);
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

  if (warp < 4) {
    regs_dec<kAttRegsCtl>();  // inside the role's branch: the compiler's register limit follows it
    if (warp == 0) {
      if (lane == 0) {
        // ------------------------------------------------------------ producer
        const uint64_t pol_q = policy_evict_first();
        const uint64_t pol_kv = policy_evict_last();  // every query block of the head re-reads K and V
        mbar_arrive_expect_tx(q_full, kAttQBytes);
        tma_load_2d(sQ, &tmQ, q_full, 0, h * S + qb * kAttBlk, pol_q);
        int nk = 0, nv = 0;  // loads issued
        for (int j = 0; j < nb; ++j) {
          const int kst = j % kAttKStages, vst = j % kAttVStages;
          if (!mbar_wait_bounded(&k_empty[kst], static_cast<uint32_t>(((j / kAttKStages) & 1) ^ 1), limit,
                                 abort_flag))
            break;
          mbar_arrive_expect_tx(&k_full[kst], kAttKBytes);
          tma_load_2d(sK + kst * kAttKBytes, &tmK, &k_full[kst], 0, h * S + j * kAttBlk, pol_kv);
          ++nk;
          if (!mbar_wait_bounded(&v_empty[vst], static_cast<uint32_t>(((j / kAttVStages) & 1) ^ 1), limit,
                                 abort_flag))
            break;
          mbar_arrive_expect_tx(&v_full[vst], kAttVBytes);
          tma_load_2d(sV + vst * kAttVBytes, &tmV, &v_full[vst], j * kAttBlk, h * kAttD, pol_kv);
          tma_load_2d(sV + vst * kAttVBytes + kAttVBytes / 2, &tmV, &v_full[vst], j * kAttBlk + 64, h * kAttD, pol_kv);
          ++nv;
        }
        // the copies still in flight land before the block exits (already done on the normal path)
        mbar_wait_bounded(q_full, 0, limit, nullptr);
        for (int t = max(0, nk - kAttKStages); t < nk; ++t)
          mbar_wait_bounded(&k_full[t % kAttKStages], static_cast<uint32_t>((t / kAttKStages) & 1), limit, nullptr);
        for (int t = max(0, nv - kAttVStages); t < nv; ++t)
          mbar_wait_bounded(&v_full[t % kAttVStages], static_cast<uint32_t>((t / kAttVStages) & 1), limit, nullptr);
      }
    } else if (warp == 3) {
      if (lane == 0) {
        // ------------------------------------------------------------ score issuer
        // S_j = Q K_j^T into score buffer j % 2 once K_j has landed and S_{j-2} has been
        // read. A thread of its own, so a score product never queues behind the issue of
        // a P.V product.
        constexpr uint32_t idesc_s = idesc_i8(kAttBlk, kAttBlk);
        constexpr uint32_t idesc_bias = idesc_bf16(kAttBlk, kAttBlk);
        const uint64_t bias_a = smem_desc_sw128(smem_u32(sBias));
        const uint64_t bias_b = smem_desc_sw128(smem_u32(sBias + kAttBiasBytes / 2));
        bool ok = mbar_wait_bounded(q_full, 0, limit, abort_flag);
        const uint64_t qd = smem_desc_sw128(smem_u32(sQ));
        for (int j = 0; ok && j < nb; ++j) {
          const int st = j % kAttKStages, b = j & 1;
          if (!mbar_wait_bounded(&k_full[st], static_cast<uint32_t>((j / kAttKStages) & 1), limit, abort_flag) ||
              !mbar_wait_bounded(&s_empty[b], static_cast<uint32_t>(((j >> 1) & 1) ^ 1), limit, abort_flag))
            break;
          tc_fence_after();
          const uint64_t kd = smem_desc_sw128(smem_u32(sK + st * kAttKBytes));
          // bias 1.5 * 2^23 (fp32 bits 0x4B400000), then the int8 products on top of it
          mma_bf16_ss(tmem + kAttColS + b * kAttBlk, bias_a, bias_b, idesc_bias, 0u);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_i8(tmem + kAttColS + b * kAttBlk, qd + 2u * k, kd + 2u * k, idesc_s, 1u);
          mma_commit(&s_full[b]);
          mma_commit(&k_empty[st]);
        }
        mma_commit(drain_s);
        mbar_wait_bounded(drain_s, 0, limit, nullptr);
      }
    } else if (warp == 1) {
      if (lane == 0) {
        // ------------------------------------------------------------ P.V issuer
        // O += P_t V_t (kind::f16, A = P_t from tensor memory) once P_t is written and
        // V_t has landed.
        constexpr uint32_t idesc_o = idesc_bf16(kAttBlk, kAttD);
        for (int t = 0; t < nb; ++t) {
          const int bt = t & 1, vst = t % kAttVStages;
          if (!mbar_wait_bounded(&v_full[vst], static_cast<uint32_t>((t / kAttVStages) & 1), limit, abort_flag) ||
              !mbar_wait_bounded(&p_full[bt], static_cast<uint32_t>((t >> 1) & 1), limit, abort_flag))
            break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 8; ++k) {  // 16 keys = 8 P columns = 32 bytes of a V^T row per K step
            const int half = k >> 2;
            const uint64_t vd = smem_desc_sw128(smem_u32(sV + vst * kAttVBytes + half * (kAttVBytes / 2)));
            mma_bf16_tmem_a(tmem + kAttColO, tmem + kAttColP + bt * 64 + 8 * k, vd + 2u * (k & 3), idesc_o,
                            (t > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit(&pv_done[bt]);
          mma_commit(&v_empty[vst]);
        }
        mma_commit(drain);
        mbar_wait_bounded(drain, 0, limit, nullptr);
      }
    }
  } else {
    // -------------------------------------------------------------- softmax (warps 4..11)
    regs_inc<kAttRegsSoftmax>();
    const int set = (warp - 4) >> 2;                  // 0: even key blocks, 1: odd key blocks
    const int quarter = warp & 3;                     // TMEM lanes 32*quarter .. +31
    const int r = quarter * 32 + lane;                // query row within the block
    const int i = qb * kAttBlk + r;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const float cq = __fmul_rn(i < S ? __ldg(p.qs + int64_t(h) * S + i) : 0.0f, p.c);
    float m_used = -INFINITY;             // the maximum this set's weights are relative to
    float2 l2 = make_float2(0.0f, 0.0f);  // this set's sum of weights, two partial sums
    bool ok = true;
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xFFFFFFFFu, mbar_wait_bounded(bar, parity, limit, abort_flag));
    };
    auto adopt = [&](float mp) {  // move this set's sum to the (larger) maximum mp
      if (mp != m_used) {
        if (m_used != -INFINITY) {
          const float f = ex2_approx(__fmul_rn(m_used - mp, cq));
          l2 = __fmul2_rn(l2, make_float2(f, f));
        }
        m_used = mp;
      }
    };
    float ks_next = set < nb ? __ldg(p.ks + int64_t(h) * nb + set) : 0.0f;
    for (int j = set; j < nb; j += 2) {
      const int b = j & 1;
      const float ksj = ks_next;  // loaded one block ahead: its latency stays off the score path
      if (j + 2 < nb) ks_next = __ldg(p.ks + int64_t(h) * nb + j + 2);
      if (!(ok = wait_all(&s_full[b], static_cast<uint32_t>((j >> 1) & 1)))) break;
      tc_fence_after();
      // Scores s' = acc * ks_j (ks_j the key block's scale); the log2-domain score is
      // s' * cq, cq = qs_i log2(e) / sqrt(128) >= 0, so maxima can be taken on s', and
      // on the raw scores F = 1.5 * 2^23 + acc (ks_j >= 0). Keys past the end (last
      // block only) are masked. The row is read in two halves: the maximum of the first
      // runs while the second is in flight.
      const int key0 = j * kAttBlk;
      const bool partial = key0 + kAttBlk > S;
      const int nvalid = S - key0;  // keys of the block inside the sequence (>= 8)
      uint32_t sr[4][32];
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      tmem_ld32(tmem + lane_base + kAttColS + b * kAttBlk, sr[0]);
      tmem_ld32(tmem + lane_base + kAttColS + b * kAttBlk + 32, sr[1]);
      tmem_ld_wait();
      tmem_ld32(tmem + lane_base + kAttColS + b * kAttBlk + 64, sr[2]);
      tmem_ld32(tmem + lane_base + kAttColS + b * kAttBlk + 96, sr[3]);
      if (partial)
        att_raw_max<true, 0, 2>(sr, nvalid, mx4);
      else
        att_raw_max<false, 0, 2>(sr, nvalid, mx4);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[b]);  // S_{j+2} may now be written into buffer b
      if (partial)
        att_raw_max<true, 2, 4>(sr, nvalid, mx4);
      else
        att_raw_max<false, 2, 4>(sr, nvalid, mx4);
      const float f_max = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      const float mx = __fmul_rn(__fsub_rn(f_max, 12582912.0f), ksj);
      if (j > 0) {  // the maximum after block j-1, published by the other set
        if (!(ok = wait_all(&mx_full[(j - 1) & 1], static_cast<uint32_t>(((j - 1) >> 1) & 1)))) break;
        adopt(sMx[((j - 1) & 1) * 128 + r]);
      }
      // raise the exponent's maximum when the row maximum grew by more than 2^8 (log2 units)
      const bool need = j == 0 || __fmul_rn(mx - m_used, cq) > 8.0f;
      const float m_new = need ? mx : m_used;
      sMx[(j & 1) * 128 + r] = m_new;  // slot j % 2 was last read before the other set published m_{j-1}
      __syncwarp();
      if (lane == 0) mbar_arrive(&mx_full[j & 1]);
      if (j >= 2) {  // P buffer b was last read by P_{j-2} V_{j-2}
        if (!(ok = wait_all(&pv_done[b], static_cast<uint32_t>(((j >> 1) & 1) ^ 1)))) break;
      }
      tc_fence_after();
      // P = 2^(s' cq - m cq) as bf16 pairs (lower key in the low half), 64 keys per store
      const float c = __fmul_rn(ksj, cq);
      const float nbias = -__fadd_rn(__fmul_rn(12582912.0f, c), __fmul_rn(m_new, cq));
      const float2 c2 = make_float2(c, c), nb2 = make_float2(nbias, nbias);
      const uint32_t p_cols = tmem + lane_base + kAttColP + b * 64;
      const float2 bs2 = partial ? att_weights<true>(sr, c2, nb2, nvalid, p_cols)
                                 : att_weights<false>(sr, c2, nb2, nvalid, p_cols);
      if (__ballot_sync(0xFFFFFFFFu, need) != 0u && j > 0) {
        // O holds P.V of blocks < j relative to m_used: rescale it once P_{j-1} V_{j-1} has
        // landed (P_j V_j waits for this block's P)
        if (!(ok = wait_all(&pv_done[(j - 1) & 1], static_cast<uint32_t>(((j - 1) >> 1) & 1)))) break;
        tc_fence_after();
        const float f = need ? ex2_approx(__fmul_rn(m_used - m_new, cq)) : 1.0f;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + kAttColO + 32 * c, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__fmul_rn(__uint_as_float(o[e]), f));
          tmem_st32(tmem + lane_base + kAttColO + 32 * c, o);
        }
        l2 = __fmul2_rn(l2, make_float2(f, f));
      }
      m_used = m_new;
      l2 = __fadd2_rn(l2, bs2);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[b]);
    }
    // the final maximum is the other set's when it took the last block
    if (ok && ((nb - 1) & 1) != set) {
      ok = wait_all(&mx_full[(nb - 1) & 1], static_cast<uint32_t>(((nb - 1) >> 1) & 1));
      if (ok) adopt(sMx[((nb - 1) & 1) * 128 + r]);
    }
    if (ok) {
      sL[set * 128 + r] = __fadd_rn(l2.x, l2.y);
      __syncwarp();
      if (lane == 0) mbar_arrive(l_full);
      ok = wait_all(l_full, 0);
    }
    if (ok) ok = wait_all(&pv_done[(nb - 1) & 1], static_cast<uint32_t>(((nb - 1) >> 1) & 1));
    if (ok) {
      tc_fence_after();
      const float inv_l = __fdiv_rn(1.0f, __fadd_rn(sL[r], sL[128 + r]));
      __nv_bfloat16* orow = p.out + int64_t(i) * p.ld_out + h * kAttD + 64 * set;
#pragma unroll 1
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + kAttColO + 64 * set + 32 * hh, o);
        tmem_ld_wait();
        if (i < S) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w[e] = pack_bf16x2(__fmul_rn(__uint_as_float(o[8 * g + 2 * e]), inv_l),
                                 __fmul_rn(__uint_as_float(o[8 * g + 2 * e + 1]), inv_l));
            *reinterpret_cast<uint4*>(orow + 32 * hh + 8 * g) = make_uint4(w[0], w[1], w[2], w[3]);
          }
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
