/*
 * h3q - INT8 ConvRot (W8A8, Hadamard-256) linear layer for NVIDIA B200 (sm_100a).
 *
 * C ABI of libh3q.so. The method, as the pages describe it:
 *  - ConvRot rotation: a group-wise Hadamard rotation along K in 256-wide groups,
 *    written as a conv whose kernel and stride are the group width
 *    (cloud-worker "MiniMax H3 - research findings", "Weight families").
 *  - Weights stored pre-rotated as per-row int8, one scale per output channel
 *    (h3-rs README, model-file table: "int8 per-row + ConvRot (Hadamard-256)").
 *  - Activations rotated inside the quantizer and quantized per row (per token);
 *    an int8 GEMM writes bf16 directly; SwiGLU is fused into the epilogue of the
 *    FFN's gate/up projection (h3-rs README, "Speed", list "What makes it fast").
 *  - The FFN-output projection is INT8 ConvRot too (Minimax_h3_hybrid model
 *    card, "Checkpoints"), so the SwiGLU output is rotated and quantized again.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates, frees or retains them. Tensors are row-major and dense
 *    (leading dimension = width). Every pointer must be 16-byte aligned.
 *  - bf16 tensors are passed as void* (IEEE bfloat16, 2 bytes per element).
 *  - Calls are asynchronous on `stream` (0 = legacy default stream); results are
 *    ready when the stream reaches that point.
 *  - Arguments are checked on the host before anything is launched; a failed
 *    check returns H3Q_ERR_INVALID_ARG (or H3Q_ERR_UNSUPPORTED for a valid
 *    shape outside the implemented range) and launches nothing.
 *  - A launch failure returns H3Q_ERR_CUDA. A device-side bounded wait that ran
 *    out (it never should) is reported later by h3q_get_device_status.
 *  - H = natural-order Sylvester Hadamard matrix, H[i][j] = (-1)^popcount(i&j),
 *    applied as H/16 (orthonormal). Each rotated element is an fp32 sum whose
 *    order is fixed (radix-2 butterflies over index bits 0,1,...,7), so the
 *    int8 codes are reproducible bit for bit.
 *  - Quantizer: s = max|y| / 127 per row (fp32 division), q = clamp(rne(y / s),
 *    -127, 127); an all-zero row gives s = 0 and q = 0.
 */
#ifndef H3Q_H_
#define H3Q_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  H3Q_OK = 0,
  H3Q_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment or workspace: nothing launched */
  H3Q_ERR_UNSUPPORTED = 2,  /* valid request outside the implemented range: nothing launched */
  H3Q_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
  H3Q_ERR_TIMEOUT = 4       /* a bounded device wait expired (reported by h3q_get_device_status) */
} h3q_status;

enum { H3Q_EPI_NONE = 0, H3Q_EPI_SWIGLU = 1 };

/* Largest K (or F) the rotate+quantize kernel holds on chip for one row. */
#define H3Q_MAX_K 16384

/*
 * Rotate + per-token quantize (h3-rs README, "What makes it fast": the quantizer
 * itself applies the ConvRot Hadamard rotation, at warp level, and each row of
 * activations gets its own scale).
 *   x_bf16 [M, K] bf16 in; xq [M, K] int8 out (rotated codes); sx [M] fp32 out.
 *   K % 256 == 0, 256 <= K <= H3Q_MAX_K; M >= 1 (M == 0 is a no-op).
 */
h3q_status h3q_rotate_quant(const void* x_bf16, int64_t M, int64_t K, int8_t* xq, float* sx,
                            cudaStream_t stream);

/*
 * Offline weight preparation (h3-rs README, model-file table: int8 per-row +
 * ConvRot): rotate each fp32 row along K by the same block-diagonal H/16, then
 * per-row int8 with one fp32 scale per output channel.
 *   w [N, K] fp32 in; wq [N, K] int8 out; sw [N] fp32 out. Same K rules as above.
 */
h3q_status h3q_prepare_weight(const float* w, int64_t N, int64_t K, int8_t* wq, float* sw,
                              cudaStream_t stream);

/*
 * W8A8 linear with fused epilogue (h3-rs README, "What makes it fast": the int8
 * GEMM produces bf16 itself, and for fc1 the SwiGLU runs inside its epilogue).
 *   acc[m][n] = sum_k xq[m][k] * wq[n][k] (exact int32);
 *   v = ((float)acc * sx[m]) * sw[n] (+ bias[n]), fp32, no fused multiply-add.
 *   epilogue H3Q_EPI_NONE:   y [M, N] bf16 = bf16_rne(v).
 *   epilogue H3Q_EPI_SWIGLU: N = 2F, rows [0, F) of wq are the gate, [F, 2F) the
 *     up projection; y [M, F] bf16 = bf16_rne(silu(v_gate) * v_up), silu(g) =
 *     g / (1 + e^-g) with e^-g from Cody-Waite reduction and a degree-7 Taylor
 *     polynomial in fp32.
 *   xq [M, K] int8, sx [M] fp32 (from h3q_rotate_quant); wq [N, K] int8, sw [N]
 *   fp32 (from h3q_prepare_weight); bias_bf16 [N] bf16 or NULL.
 *   K % 256 == 0; N % 8 == 0 (SwiGLU: F % 128 == 0); M >= 1.
 */
h3q_status h3q_linear_w8a8(const int8_t* xq, const float* sx, int64_t M, int64_t K,
                           const int8_t* wq, const float* sw, int64_t N,
                           const void* bias_bf16, int epilogue, void* y_bf16, cudaStream_t stream);

/*
 * FFN block, INT8 ConvRot end to end (h3-rs README "What makes it fast";
 * Minimax_h3_hybrid model card, "Checkpoints": the FFN-output projection stays
 * INT8 ConvRot and the SwiGLU path stays fused):
 *   y [M, K] = down( rotquant( swiglu( gate_up( rotquant(x) ) ) ) ).
 *   x_bf16 [M, K]; w_gu [2F, K] int8 with s_gu [2F] (gate rows, then up rows);
 *   b_gu [2F] bf16 or NULL; w_down [K, F] int8 with s_down [K]; b_down [K] bf16
 *   or NULL; y_bf16 [M, K] out.
 *   workspace: caller-owned device scratch of at least
 *   h3q_ffn_workspace_size(M, K, F) bytes, 256-byte aligned (holds xq, sx,
 *   h, hq, sh). K % 256 == 0, F % 256 == 0, K, F <= H3Q_MAX_K.
 */
size_t h3q_ffn_workspace_size(int64_t M, int64_t K, int64_t F);
h3q_status h3q_ffn(const void* x_bf16, int64_t M, int64_t K,
                   const int8_t* w_gu, const float* s_gu, const void* b_gu, int64_t F,
                   const int8_t* w_down, const float* s_down, const void* b_down,
                   void* y_bf16, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * The FFN block of h3q_ffn, for callers that cannot allocate device memory.
 * No passage of the pages corresponds to this call: it exists for the library's
 * users. Some callers have no device allocator of their own (a host program
 * that reaches this library only through plain pointers, or a plug-in whose
 * device memory is owned entirely by the framework hosting it), and some must
 * not allocate while serving, because cudaMalloc and cudaFree can synchronize
 * the device and stall work on other streams. This call takes no workspace:
 * its intermediates (xq, sx, h, hq, sh) live in one scratch array of
 * H3Q_STATIC_SCRATCH_BYTES bytes that the library declares in device global
 * memory. Every GPU that loads the library holds that array until the process
 * exits. It allocates nothing and calls no allocating routine.
 *   Arguments, layouts and results are those of h3q_ffn, minus the workspace.
 *   Limit: h3q_ffn_workspace_size(M, K, F) <= H3Q_STATIC_SCRATCH_BYTES, else
 *   H3Q_ERR_UNSUPPORTED and nothing is launched; for K = 5376, F = 14336 that
 *   is M <= 1386 rows (the rows are independent, so a caller may split a
 *   larger batch into chunks).
 *   The first call on each device looks up the array's device address (with
 *   that device current); make that first call before any stream capture.
 *   After cudaDeviceReset the device has a new context and the next call
 *   looks the address up again: make that call outside stream capture too.
 *   All calls share the one array and it keeps the last call's contents:
 *   calls that may overlap on the GPU (different streams without ordering
 *   between them, or different host threads) race on it and must be
 *   serialized by the caller.
 */
#define H3Q_STATIC_SCRATCH_BYTES (64u << 20)
h3q_status h3q_ffn_static_scratch(const void* x_bf16, int64_t M, int64_t K,
                                  const int8_t* w_gu, const float* s_gu, const void* b_gu, int64_t F,
                                  const int8_t* w_down, const float* s_down, const void* b_down,
                                  void* y_bf16, cudaStream_t stream);

/*
 * LoRA merge into stored int8 weights (h3-rs README, "Speed", "What makes it
 * fast": a LoRA is folded into the int8 weights once, when the model loads, by
 * dequantizing, adding and requantizing, so inference steps pay nothing for
 * it). The codes are in the
 * rotated basis, so the delta is rotated the same way:
 *   A_rot = A blockdiag(H/16) (the rotation of h3q_prepare_weight, fp32);
 *   d[n][k] = fma chain over j = 0..r-1 ascending, from 0, of B[n][j] A_rot[j][k];
 *   w[n][k] = (float)wq[n][k] * sw[n] + alpha * d[n][k]   (fp32, two rounded
 *             products and one rounded add);
 *   then each row is requantized: sw[n] = max_k |w[n][k]| / 127,
 *   wq[n][k] = clamp(rne(w[n][k] / sw[n]), -127, 127) (0 where sw[n] == 0).
 *   wq [N, K] int8 and sw [N] fp32 are read and overwritten in place.
 *   lora_a [r, K] fp32 (the LoRA "down" factor, in the model's basis) and
 *   lora_b [N, r] fp32 (the "up" factor) are read only; alpha is the LoRA
 *   scale (strength times alpha / rank, as the caller defines it).
 *   workspace: caller-owned device scratch of at least
 *   h3q_lora_workspace_size(r, K) bytes, 16-byte aligned (holds A_rot).
 *   K % 256 == 0, K <= H3Q_MAX_K; 1 <= r <= H3Q_LORA_MAX_RANK; N >= 0
 *   (N == 0 is a no-op); all pointers 16-byte aligned. Other calls must not
 *   read or write wq / sw while the merge runs on its stream.
 */
#define H3Q_LORA_MAX_RANK 512
size_t h3q_lora_workspace_size(int64_t r, int64_t K);
h3q_status h3q_lora_merge(int8_t* wq, float* sw, int64_t N, int64_t K, const float* lora_a,
                          const float* lora_b, int64_t r, float alpha, void* workspace,
                          size_t workspace_bytes, cudaStream_t stream);

/*
 * NVFP4 projections. The hybrid checkpoints run the QKV and FFN-input
 * projections in NVFP4 and keep the output projections INT8 ConvRot
 * (Minimax_h3_hybrid model card, "Checkpoints" and "Native NVFP4 projection
 * benchmarks"; h3-rs README, model-file table: "NVFP4 (swizzled fp8 block
 * scales)"). Format (the public NVFP4 definition; no rotation):
 *   s_enc = RN(2688 / max|x|) over the whole tensor (1 for an all-zero tensor);
 *   per 16 consecutive elements of a row, S = e4m3(RN(RN(max|block| / 6) * s_enc))
 *   (round to nearest even, saturating at 448); codes q = e2m1(RN(x * RN(s_enc /
 *   S))) (round to nearest even, saturating at 6; 0 where S = 0).
 * Layouts: codes [rows, K/2] bytes, element 2i in the low nibble of byte i.
 * Block scales: h3q_nvfp4_sf_bytes(rows, K) bytes in 512-byte atoms of 128 rows
 * x 4 scales; scale j of row r at byte ((r/128)(K/64) + j/4) * 512 + 16 (r%32)
 * + 4 ((r%128)/32) + (j%4); rows padded to a multiple of 128 with zero scales.
 * Tensor scale: a device float[2], [0] = max|x| (as written by the quantizer),
 * [1] = s_enc.
 */
enum { H3Q_DTYPE_BF16 = 0, H3Q_DTYPE_F32 = 1 };
size_t h3q_nvfp4_sf_bytes(int64_t rows, int64_t K);

/*
 * x [rows, K] (bf16 activations or fp32 weights, per x_dtype) -> codes, block
 * scales and the tensor scale, as above. Two launches (tensor max, then the
 * blocks) and a 4-byte memset of scale[0]. K % 256 == 0, K <= H3Q_MAX_K; all
 * pointers 16-byte aligned.
 */
h3q_status h3q_nvfp4_quantize(const void* x, int x_dtype, int64_t rows, int64_t K, uint8_t* codes,
                              uint8_t* sf, float* scale, cudaStream_t stream);

/*
 * NVFP4 linear: acc[m][n] = sum_k e2m1(x)[m][k] S_x e2m1(w)[n][k] S_w on the
 * tensor cores (fp32 accumulation); v = RN(RN(acc * alpha) + bias[n]),
 * alpha = RN(1 / RN(s_enc_x * s_enc_w)); epilogue as h3q_linear_w8a8 (bf16, or
 * SwiGLU with rows [0, F) of w the gate and [F, 2F) the up projection).
 *   xc/xsf/x_scale from h3q_nvfp4_quantize of x [M, K]; wc/wsf/w_scale of w [N, K].
 *   N % 256 == 0 (SwiGLU: N = 2F, F % 128 == 0); K % 256 == 0; M >= 0.
 * The fp32 accumulation order is the hardware's: results agree with the exact
 * sum to within fp32 rounding of the K/16 block terms.
 */
h3q_status h3q_linear_nvfp4(const uint8_t* xc, const uint8_t* xsf, const float* x_scale, int64_t M, int64_t K,
                            const uint8_t* wc, const uint8_t* wsf, const float* w_scale, int64_t N,
                            const void* bias_bf16, int epilogue, void* y_bf16, cudaStream_t stream);

/* Test hook: the same NVFP4 GEMM with the raw fp32 accumulators [M, N] as output. */
h3q_status h3q_gemm_nvfp4_f32(const uint8_t* xc, const uint8_t* xsf, int64_t M, int64_t K, const uint8_t* wc,
                              const uint8_t* wsf, int64_t N, float* acc, cudaStream_t stream);

/*
 * int8 attention for the DiT blocks (h3-rs README, "What makes it fast": an
 * int8 Q.K^T / 16-bit P.V flash kernel). Head dim 128; head h of q, k, v and out
 * is columns h*128 .. h*128+127 of a row-major [S, ld] bf16 matrix (q, k and v
 * may be column slices of one QKV projection output).
 *   Q rows (one token of one head) are quantized like weight rows: s = max|x| /
 *   127 (fp32), codes clamp(rne(x / s)); K is quantized the same way per block
 *   of 128 consecutive keys of a head (one scale over the block's keys and
 *   dimensions; the last block takes the keys that remain);
 *   s_ij = (sum_d Qq_id Kq_jd) qs_i ks_b(j) / sqrt(128); O_i = softmax_j(s_i) V;
 *   P is rounded to bf16 and P.V accumulated in fp32 (the hardware's order);
 *   out = bf16(O).
 * workspace: h3q_attention_workspace_size(S, H) bytes, 256-byte aligned (codes,
 * scales and V transposed per head). S % 8 == 0, ld % 8 == 0, ld >= 128 H,
 * ld_out likewise; pointers 16-byte aligned.
 */
size_t h3q_attention_workspace_size(int64_t S, int64_t H);
h3q_status h3q_attention_int8(const void* q, const void* k, const void* v, int64_t S, int64_t H, int64_t ld,
                              void* out, int64_t ld_out, void* workspace, size_t workspace_bytes,
                              cudaStream_t stream);

/*
 * The attention's input pass on its own (test hook and building block): qq, kq
 * int8 [H, S, 128], qs fp32 [H, S], ks fp32 [H, ceil(S / 128)] (one per block of
 * 128 keys), vt bf16 [H*128, S] (V^T per head).
 */
h3q_status h3q_attention_prep(const void* q, const void* k, const void* v, int64_t S, int64_t H, int64_t ld,
                              int8_t* qq, float* qs, int8_t* kq, float* ks, void* vt, cudaStream_t stream);

/*
 * Test hook: the same GEMM kernel with the raw int32 accumulators as output.
 *   xq [M, K], wq [N, K] int8; acc [M, N] int32. K % 128 == 0, N % 8 == 0.
 */
h3q_status h3q_gemm_s32(const int8_t* xq, const int8_t* wq, int64_t M, int64_t N, int64_t K,
                        int32_t* acc, cudaStream_t stream);

/*
 * Synchronizes `stream`, then reports and clears the device status word:
 * H3Q_ERR_TIMEOUT if any bounded wait in a kernel of this library ran out since
 * the last call, H3Q_ERR_CUDA if the synchronization failed, else H3Q_OK.
 */
h3q_status h3q_get_device_status(cudaStream_t stream);

/*
 * Upper bound, in nanoseconds, on every spin-wait inside the GEMM kernel (an
 * mbarrier the kernel waits on). Past it the kernel records H3Q_ERR_TIMEOUT,
 * drains its own copies in flight (again bounded), frees its tensor memory and
 * returns. Default 2 s. Values below 1000 ns are raised to 1000 ns.
 */
void h3q_set_wait_limit_ns(uint64_t ns);

/*
 * Test hook for the bounded-wait path: launches one block whose threads wait,
 * through both of the library's bounded-wait forms (the one single issuing
 * threads use and the one the consumers of a shared-memory ring use), on an
 * mbarrier nothing ever arrives on, with the given limit; afterwards
 * h3q_get_device_status returns H3Q_ERR_TIMEOUT. No fault, no hang.
 */
h3q_status h3q_test_stalled_wait(uint64_t limit_ns, cudaStream_t stream);

/* Human-readable name of a status code (static string). */
const char* h3q_status_string(h3q_status s);

/* Library version string (static). */
const char* h3q_version(void);

#ifdef __cplusplus
}
#endif

#endif /* H3Q_H_ */
