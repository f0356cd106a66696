// libh3q.so: the C ABI declared in include/h3q.h. Host-side argument checks,
// TMA descriptor setup and launches of the kernels in rotquant.cuh and
// gemm_sm100.cuh. Everything is stream-ordered; nothing here allocates device
// memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cmath>
#include <atomic>
#include <mutex>
#include <set>
#include <utility>

#include "h3q.h"
#include "gemm_sm100.cuh"
#include "lora.cuh"
#include "nvfp4.cuh"
#include "attention.cuh"
#include "rotquant.cuh"

namespace {

using h3q::GemmParams;

std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};

// GEMM tile order and L2 policies (0 evict-first, 1 evict-last, 2 evict-normal).
#ifndef H3Q_GEMM_GROUP_ROWS
#define H3Q_GEMM_GROUP_ROWS 16
#endif
#ifndef H3Q_GEMM_POLICY_A
#define H3Q_GEMM_POLICY_A 1
#endif
#ifndef H3Q_GEMM_POLICY_B
#define H3Q_GEMM_POLICY_B 1
#endif
#ifndef H3Q_GEMM_RASTER
#define H3Q_GEMM_RASTER 0
#endif
constexpr int kGemmGroupRows = H3Q_GEMM_GROUP_ROWS;
constexpr int kGemmRaster = H3Q_GEMM_RASTER;
constexpr int kGemmPolicyA = H3Q_GEMM_POLICY_A;
constexpr int kGemmPolicyB = H3Q_GEMM_POLICY_B;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Kernel attributes belong to the context of the device that is current when
// they are set, so a process that drives several GPUs sets them once per
// (kernel, device). The record of what was set is read and written under one
// mutex; a failed set is not recorded and is retried on the next call.
std::mutex g_attr_mu;
std::set<std::pair<const void*, int>> g_attr_done;

cudaError_t ensure_smem_attr(const void* kernel, int smem_bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_attr_mu);
  if (g_attr_done.count({kernel, dev})) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e == cudaSuccess) g_attr_done.insert({kernel, dev});
  return e;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// [rows, cols] int8 row-major, boxes of 128 columns x 128 rows, 128-byte swizzle;
// reads past the edges return zeros.
bool make_tmap_i8(CUtensorMap* map, const void* base, int64_t rows, int64_t cols) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols)};
  const cuuint32_t box[2] = {128, 128};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

template <int EPI>
h3q_status launch_gemm(const int8_t* a, const int8_t* b, int64_t M, int64_t K, int64_t b_rows, int64_t N_out,
                       const float* sx, const float* sw, const void* bias, void* out, cudaStream_t stream) {
  CUtensorMap ta, tb;
  if (!make_tmap_i8(&ta, a, M, K) || !make_tmap_i8(&tb, b, b_rows, K)) return H3Q_ERR_CUDA;
  if (ensure_smem_attr(reinterpret_cast<const void*>(h3q::gemm_i8_kernel<EPI>),
                       static_cast<int>(h3q::kGemmSmem)) != cudaSuccess)
    return H3Q_ERR_CUDA;
  GemmParams p{};
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N_out);
  p.K = static_cast<int>(K);
  p.num_m = static_cast<int>((M + 2 * h3q::kBM - 1) / (2 * h3q::kBM));  // 256-row tiles of a CTA pair
  p.num_n = (EPI == h3q::kEpiSwiGLU) ? static_cast<int>(N_out / 128)
                                     : static_cast<int>((N_out + h3q::kBN - 1) / h3q::kBN);
  p.num_tiles = p.num_m * p.num_n;
  p.b_row_up = (EPI == h3q::kEpiSwiGLU) ? static_cast<int>(N_out) : 0;
  // Tile order: groups of kGemmGroupRows pair-row blocks (the group's A tiles are
  // reused by every N block from L2, each B tile is read once per group); both
  // operands are loaded with an evict-last L2 policy.
  p.raster = kGemmRaster;
  p.group_m = kGemmGroupRows < p.num_m ? kGemmGroupRows : p.num_m;
  p.pol_a = kGemmPolicyA;
  p.pol_b = kGemmPolicyB;
  p.sx = sx;
  p.sw = sw;
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.out = out;
  p.wait_limit_ns = g_wait_limit_ns.load();
  const int sms = sm_count();
  if (sms <= 0) return H3Q_ERR_CUDA;
  const int pairs = p.num_tiles < sms / 2 ? p.num_tiles : sms / 2;
  const int grid = 2 * pairs;  // clusters of two CTAs
  h3q::gemm_i8_kernel<EPI><<<grid, h3q::kGemmThreads, h3q::kGemmSmem, stream>>>(ta, tb, p);
  return cudaGetLastError() == cudaSuccess ? H3Q_OK : H3Q_ERR_CUDA;
}

// Scale-factor atom array viewed as [bytes / 128, 128] uint8: boxes of 16 rows
// (2048 bytes = 4 atoms), no swizzle; reads past the end return zeros.
bool make_tmap_sf(CUtensorMap* map, const void* base, int64_t bytes) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(bytes / 128)};
  const cuuint64_t strides[1] = {128};
  const cuuint32_t box[2] = {128, 16};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPI>
h3q_status launch_gemm_fp4(const uint8_t* a, const uint8_t* a_sf, const float* a_scale, int64_t M, int64_t K,
                           const uint8_t* b, const uint8_t* b_sf, const float* b_scale, int64_t b_rows,
                           int64_t N_out, const void* bias, void* out, cudaStream_t stream) {
  CUtensorMap ta, tb, tsa, tsb;
  if (!make_tmap_i8(&ta, a, M, K / 2) || !make_tmap_i8(&tb, b, b_rows, K / 2) ||
      !make_tmap_sf(&tsa, a_sf, h3q::nvfp4_sf_bytes(M, K)) || !make_tmap_sf(&tsb, b_sf, h3q::nvfp4_sf_bytes(b_rows, K)))
    return H3Q_ERR_CUDA;
  if (ensure_smem_attr(reinterpret_cast<const void*>(h3q::gemm_fp4_kernel<EPI>),
                       static_cast<int>(h3q::kF4Smem)) != cudaSuccess)
    return H3Q_ERR_CUDA;
  h3q::Fp4Params p{};
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N_out);
  p.K = static_cast<int>(K);
  p.num_m = static_cast<int>((M + 2 * h3q::kBM - 1) / (2 * h3q::kBM));
  p.num_n = (EPI == h3q::kEpiSwiGLU) ? static_cast<int>(N_out / 128) : static_cast<int>(N_out / h3q::kBN);
  p.num_tiles = p.num_m * p.num_n;
  p.group_m = kGemmGroupRows < p.num_m ? kGemmGroupRows : p.num_m;
  p.b_row_up = (EPI == h3q::kEpiSwiGLU) ? static_cast<int>(N_out) : 0;
  p.x_scale = a_scale;
  p.w_scale = b_scale;
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.out = out;
  p.wait_limit_ns = g_wait_limit_ns.load();
  const int sms = sm_count();
  if (sms <= 0) return H3Q_ERR_CUDA;
  const int pairs = p.num_tiles < sms / 2 ? p.num_tiles : sms / 2;
  h3q::gemm_fp4_kernel<EPI><<<2 * pairs, h3q::kF4Threads, h3q::kF4Smem, stream>>>(ta, tb, tsa, tsb, p);
  return cudaGetLastError() == cudaSuccess ? H3Q_OK : H3Q_ERR_CUDA;
}

// [rows, cols] bf16 row-major, boxes of 64 columns (128 bytes) x 128 rows,
// 128-byte swizzle; reads past the edges return zeros.
bool make_tmap_bf16(CUtensorMap* map, const void* base, int64_t rows, int64_t cols) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols * 2)};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Rows of K elements (bf16 or fp32) seen as [rows][K * size / 128][128 bytes]
// for the rotate+quantize stages: boxes of `units` 128-byte units x `box_rows`
// rows, 128-byte swizzle; rows past the end read as zeros.
bool make_tmap_rows(CUtensorMap* map, const void* base, int64_t rows, int64_t K, int elem_bytes, int units,
                    int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(128 / elem_bytes),
                              static_cast<cuuint64_t>(K * elem_bytes / 128), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(K * elem_bytes)};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / elem_bytes), static_cast<cuuint32_t>(units),
                             static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
             const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Which rotate+quantize kernel runs: the tensor-memory variant where it measured
// faster (bf16 rows of up to 42 groups with 8192 rows or more: K = 5376 at 8192 to
// 32768 rows 4-6% faster, K = 10752 at 16384 rows 10% faster), the register
// variant otherwise (K = 14336: 5% faster; 4096 rows at K = 5376: 7% faster; fp32
// weight rows).
bool rotquant_use_tm(int64_t rows, int64_t K) { return K / 256 <= 42 && rows >= 8192; }

template <typename T>
h3q_status run_rotquant(const T* x, int64_t rows, int64_t K, int8_t* q, float* s, cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return H3Q_ERR_CUDA;
  int occ = 0, sms = 0;
  if constexpr (sizeof(T) == 2) {
    if (rotquant_use_tm(rows, K)) {
      size_t smem = 0;
      const h3q::RqShape sh = h3q::rotquant_tm_plan<T>(static_cast<int>(K), dev, &occ, &sms, &smem);
      if (sh.gps == 0 || occ < 1 || sms < 1) return H3Q_ERR_CUDA;
      const h3q::RqArgs a = h3q::rotquant_args<T>(sh, rows, K, q, s, g_wait_limit_ns.load());
      CUtensorMap map;
      if (!make_tmap_rows(&map, x, rows, K, static_cast<int>(sizeof(T)), a.units_per_copy, sh.rows))
        return H3Q_ERR_CUDA;
      return h3q::launch_rotquant_tm<T>(map, sh, occ, sms, smem, a, stream) == cudaSuccess ? H3Q_OK : H3Q_ERR_CUDA;
    }
  }
  const h3q::RqShape sh = h3q::rotquant_plan<T>(static_cast<int>(K), dev, &occ, &sms);
  if (sh.gps == 0 || occ < 1 || sms < 1) return H3Q_ERR_CUDA;
  const h3q::RqArgs a = h3q::rotquant_args<T>(sh, rows, K, q, s, g_wait_limit_ns.load());
  CUtensorMap map;
  if (!make_tmap_rows(&map, x, rows, K, static_cast<int>(sizeof(T)), a.units_per_copy, sh.rows))
    return H3Q_ERR_CUDA;
  return h3q::launch_rotquant<T>(map, sh, occ, sms, a, stream) == cudaSuccess ? H3Q_OK : H3Q_ERR_CUDA;
}

bool valid_k(int64_t K) { return K >= 256 && K % 256 == 0; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct FfnLayout {
  size_t xq, sx, h, hq, sh, total;
};

FfnLayout ffn_layout(int64_t M, int64_t K, int64_t F) {
  FfnLayout l;
  size_t off = 0;
  l.xq = off; off = align256(off + size_t(M) * size_t(K));
  l.sx = off; off = align256(off + size_t(M) * 4);
  l.h = off;  off = align256(off + size_t(M) * size_t(F) * 2);
  l.hq = off; off = align256(off + size_t(M) * size_t(F));
  l.sh = off; off = align256(off + size_t(M) * 4);
  l.total = off;
  return l;
}

// Scratch for h3q_ffn_static_scratch: a fixed device array, so that call needs
// no allocation. In host code this name only stands for the array; its device
// address comes from cudaGetSymbolAddress, looked up with the device current.
static __device__ __align__(256) unsigned char g_static_scratch[H3Q_STATIC_SCRATCH_BYTES];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// The current context's ID, unique among all contexts the process creates, so a
// context re-created after cudaDeviceReset never matches an older one. False if
// no context is current or the driver lacks the call.
bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// The array's device address on `device` (the current device), cached per device
// together with the ID of the context it was looked up in; a new context on that
// device (after a device reset) looks it up again. Without context IDs from the
// driver, every call looks it up.
void* static_scratch_address(int device) {
  static std::mutex mu;
  static void* addr[64] = {};
  static unsigned long long ctx_id[64] = {};
  if (device < 0 || device >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  unsigned long long id = 0;
  if (addr[device] != nullptr && current_context_id(&id) && id == ctx_id[device]) return addr[device];
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) return nullptr;
  if (current_context_id(&id)) {  // read after the lookup, which made the device's context current
    addr[device] = p;
    ctx_id[device] = id;
  }
  return p;
}

}  // namespace

extern "C" {

const char* h3q_version(void) { return "h3q 0.1 (sm_100a, tcgen05 int8)"; }

const char* h3q_status_string(h3q_status s) {
  switch (s) {
    case H3Q_OK: return "ok";
    case H3Q_ERR_INVALID_ARG: return "invalid argument";
    case H3Q_ERR_UNSUPPORTED: return "unsupported shape";
    case H3Q_ERR_CUDA: return "CUDA error";
    case H3Q_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

void h3q_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns < 1000 ? 1000 : ns); }

h3q_status h3q_rotate_quant(const void* x_bf16, int64_t M, int64_t K, int8_t* xq, float* sx,
                            cudaStream_t stream) {
  if (M < 0 || !valid_k(K)) return H3Q_ERR_INVALID_ARG;
  if (M == 0) return H3Q_OK;
  if (!x_bf16 || !xq || !sx || !aligned16(x_bf16) || !aligned16(xq) || !aligned16(sx)) return H3Q_ERR_INVALID_ARG;
  if (K > H3Q_MAX_K || M > INT32_MAX) return H3Q_ERR_UNSUPPORTED;
  return run_rotquant(static_cast<const __nv_bfloat16*>(x_bf16), M, K, xq, sx, stream);
}

h3q_status h3q_prepare_weight(const float* w, int64_t N, int64_t K, int8_t* wq, float* sw, cudaStream_t stream) {
  if (N < 0 || !valid_k(K)) return H3Q_ERR_INVALID_ARG;
  if (N == 0) return H3Q_OK;
  if (!w || !wq || !sw || !aligned16(w) || !aligned16(wq) || !aligned16(sw)) return H3Q_ERR_INVALID_ARG;
  if (K > H3Q_MAX_K || N > INT32_MAX) return H3Q_ERR_UNSUPPORTED;
  return run_rotquant(w, N, K, wq, sw, stream);
}

h3q_status h3q_linear_w8a8(const int8_t* xq, const float* sx, int64_t M, int64_t K, const int8_t* wq,
                           const float* sw, int64_t N, const void* bias_bf16, int epilogue, void* y_bf16,
                           cudaStream_t stream) {
  if (M < 0 || !valid_k(K) || N <= 0 || N % 8 != 0) return H3Q_ERR_INVALID_ARG;
  if (epilogue != H3Q_EPI_NONE && epilogue != H3Q_EPI_SWIGLU) return H3Q_ERR_INVALID_ARG;
  if (epilogue == H3Q_EPI_SWIGLU && (N % 256 != 0)) return H3Q_ERR_INVALID_ARG;  // F = N/2 multiple of 128
  if (M == 0) return H3Q_OK;
  if (!xq || !sx || !wq || !sw || !y_bf16) return H3Q_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(sx) || !aligned16(wq) || !aligned16(sw) || !aligned16(y_bf16) ||
      (bias_bf16 && !aligned16(bias_bf16)))
    return H3Q_ERR_INVALID_ARG;
  if (M > INT32_MAX - 256 || N > INT32_MAX - 512 || K > INT32_MAX) return H3Q_ERR_UNSUPPORTED;
  if (epilogue == H3Q_EPI_SWIGLU)
    return launch_gemm<h3q::kEpiSwiGLU>(xq, wq, M, K, N, N / 2, sx, sw, bias_bf16, y_bf16, stream);
  return launch_gemm<h3q::kEpiBF16>(xq, wq, M, K, N, N, sx, sw, bias_bf16, y_bf16, stream);
}

size_t h3q_lora_workspace_size(int64_t r, int64_t K) {
  if (r <= 0 || K <= 0) return 0;
  return size_t(r) * size_t(K) * sizeof(float);
}

h3q_status h3q_lora_merge(int8_t* wq, float* sw, int64_t N, int64_t K, const float* lora_a, const float* lora_b,
                          int64_t r, float alpha, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (N < 0 || !valid_k(K) || r < 1) return H3Q_ERR_INVALID_ARG;
  if (r > H3Q_LORA_MAX_RANK || K > H3Q_MAX_K || N > INT32_MAX) return H3Q_ERR_UNSUPPORTED;
  if (N == 0) return H3Q_OK;
  if (!wq || !sw || !lora_a || !lora_b || !workspace) return H3Q_ERR_INVALID_ARG;
  if (!aligned16(wq) || !aligned16(sw) || !aligned16(lora_a) || !aligned16(lora_b) || !aligned16(workspace))
    return H3Q_ERR_INVALID_ARG;
  if (workspace_bytes < h3q_lora_workspace_size(r, K)) return H3Q_ERR_INVALID_ARG;
  const cudaError_t e = h3q::launch_lora_merge(wq, sw, N, K, lora_a, lora_b, static_cast<int>(r), alpha,
                                               static_cast<float*>(workspace), stream);
  return e == cudaSuccess ? H3Q_OK : H3Q_ERR_CUDA;
}

size_t h3q_nvfp4_sf_bytes(int64_t rows, int64_t K) {
  if (rows < 0 || K <= 0 || K % 64 != 0) return 0;
  return static_cast<size_t>(h3q::nvfp4_sf_bytes(rows, K));
}

h3q_status h3q_nvfp4_quantize(const void* x, int x_dtype, int64_t rows, int64_t K, uint8_t* codes, uint8_t* sf,
                              float* scale, cudaStream_t stream) {
  if (rows < 0 || !valid_k(K) || (x_dtype != H3Q_DTYPE_BF16 && x_dtype != H3Q_DTYPE_F32)) return H3Q_ERR_INVALID_ARG;
  if (K > H3Q_MAX_K || rows > INT32_MAX) return H3Q_ERR_UNSUPPORTED;
  if (rows == 0) return H3Q_OK;
  if (!x || !codes || !sf || !scale || !aligned16(x) || !aligned16(codes) || !aligned16(sf) || !aligned16(scale))
    return H3Q_ERR_INVALID_ARG;
  const int sms = sm_count();
  if (sms <= 0) return H3Q_ERR_CUDA;
  if (cudaMemsetAsync(scale, 0, sizeof(uint32_t), stream) != cudaSuccess) return H3Q_ERR_CUDA;
  const int64_t n16 = rows * K / 16;
  const int64_t rows_pad = (rows + 127) / 128 * 128;
  const int64_t total = rows_pad * (K / 16);
  const unsigned g1 = static_cast<unsigned>(std::min<int64_t>((n16 + 255) / 256, int64_t(sms) * 8));
  const unsigned g2 = static_cast<unsigned>(std::min<int64_t>((total + 255) / 256, int64_t(sms) * 16));
  uint32_t* amax = reinterpret_cast<uint32_t*>(scale);
  if (x_dtype == H3Q_DTYPE_BF16) {
    const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
    h3q::nvfp4_amax_kernel<__nv_bfloat16><<<g1, 256, 0, stream>>>(xb, n16, amax);
    h3q::nvfp4_quantize_kernel<__nv_bfloat16><<<g2, 256, 0, stream>>>(xb, rows, rows_pad, static_cast<int>(K), scale,
                                                                     codes, sf);
  } else {
    const float* xf = static_cast<const float*>(x);
    h3q::nvfp4_amax_kernel<float><<<g1, 256, 0, stream>>>(xf, n16, amax);
    h3q::nvfp4_quantize_kernel<float><<<g2, 256, 0, stream>>>(xf, rows, rows_pad, static_cast<int>(K), scale, codes,
                                                             sf);
  }
  return cudaGetLastError() == cudaSuccess ? H3Q_OK : H3Q_ERR_CUDA;
}

static h3q_status check_fp4_args(const uint8_t* xc, const uint8_t* xsf, const float* x_scale, int64_t M, int64_t K,
                                 const uint8_t* wc, const uint8_t* wsf, const float* w_scale, int64_t N) {
  if (M < 0 || !valid_k(K) || N <= 0 || N % 256 != 0) return H3Q_ERR_INVALID_ARG;
  if (K > H3Q_MAX_K || M > INT32_MAX - 256 || N > INT32_MAX - 512) return H3Q_ERR_UNSUPPORTED;
  if (M == 0) return H3Q_OK;
  if (!xc || !xsf || !x_scale || !wc || !wsf || !w_scale) return H3Q_ERR_INVALID_ARG;
  if (!aligned16(xc) || !aligned16(xsf) || !aligned16(wc) || !aligned16(wsf) ||
      (reinterpret_cast<uintptr_t>(x_scale) & 7u) || (reinterpret_cast<uintptr_t>(w_scale) & 7u))
    return H3Q_ERR_INVALID_ARG;
  return H3Q_OK;
}

h3q_status h3q_linear_nvfp4(const uint8_t* xc, const uint8_t* xsf, const float* x_scale, int64_t M, int64_t K,
                            const uint8_t* wc, const uint8_t* wsf, const float* w_scale, int64_t N,
                            const void* bias_bf16, int epilogue, void* y_bf16, cudaStream_t stream) {
  if (epilogue != H3Q_EPI_NONE && epilogue != H3Q_EPI_SWIGLU) return H3Q_ERR_INVALID_ARG;
  const h3q_status st = check_fp4_args(xc, xsf, x_scale, M, K, wc, wsf, w_scale, N);
  if (st != H3Q_OK || M == 0) return st;
  if (!y_bf16 || !aligned16(y_bf16) || (bias_bf16 && !aligned16(bias_bf16))) return H3Q_ERR_INVALID_ARG;
  if (epilogue == H3Q_EPI_SWIGLU)
    return launch_gemm_fp4<h3q::kEpiSwiGLU>(xc, xsf, x_scale, M, K, wc, wsf, w_scale, N, N / 2, bias_bf16, y_bf16,
                                            stream);
  return launch_gemm_fp4<h3q::kEpiBF16>(xc, xsf, x_scale, M, K, wc, wsf, w_scale, N, N, bias_bf16, y_bf16, stream);
}

h3q_status h3q_gemm_nvfp4_f32(const uint8_t* xc, const uint8_t* xsf, int64_t M, int64_t K, const uint8_t* wc,
                              const uint8_t* wsf, int64_t N, float* acc, cudaStream_t stream) {
  static const float kUnused[2] = {0.0f, 0.0f};  // the raw-accumulator epilogue reads no tensor scale
  const h3q_status st = check_fp4_args(xc, xsf, kUnused, M, K, wc, wsf, kUnused, N);
  if (st != H3Q_OK || M == 0) return st;
  if (!acc || !aligned16(acc)) return H3Q_ERR_INVALID_ARG;
  return launch_gemm_fp4<h3q::kEpiS32>(xc, xsf, nullptr, M, K, wc, wsf, nullptr, N, N, nullptr, acc, stream);
}

struct AttLayout {
  size_t qq, kq, qs, ks, vt, total;
};

AttLayout att_layout(int64_t S, int64_t H) {
  AttLayout l{};
  const size_t codes = size_t(H) * S * 128, scales = size_t(H) * S * 4, vt = size_t(H) * 128 * S * 2;
  const size_t key_scales = size_t(H) * ((S + 127) / 128) * 4;  // one per block of 128 keys
  l.qq = 0;
  l.kq = align256(l.qq + codes);
  l.qs = align256(l.kq + codes);
  l.ks = align256(l.qs + scales);
  l.vt = align256(l.ks + key_scales);
  l.total = align256(l.vt + vt);
  return l;
}

static h3q_status check_att_args(const void* q, const void* k, const void* v, int64_t S, int64_t H, int64_t ld) {
  if (S < 0 || H < 1 || S % 8 != 0 || ld < H * 128 || ld % 8 != 0) return H3Q_ERR_INVALID_ARG;
  if (H * S > INT32_MAX / 2 || S > INT32_MAX - 256) return H3Q_ERR_UNSUPPORTED;
  if (S == 0) return H3Q_OK;
  if (!q || !k || !v || !aligned16(q) || !aligned16(k) || !aligned16(v)) return H3Q_ERR_INVALID_ARG;
  return H3Q_OK;
}

size_t h3q_attention_workspace_size(int64_t S, int64_t H) {
  if (S < 0 || H < 1) return 0;
  return att_layout(S, H).total;
}

h3q_status h3q_attention_prep(const void* q, const void* k, const void* v, int64_t S, int64_t H, int64_t ld,
                              int8_t* qq, float* qs, int8_t* kq, float* ks, void* vt, cudaStream_t stream) {
  const h3q_status st = check_att_args(q, k, v, S, H, ld);
  if (st != H3Q_OK || S == 0) return st;
  if (!qq || !qs || !kq || !ks || !vt || !aligned16(qq) || !aligned16(qs) || !aligned16(kq) || !aligned16(ks) ||
      !aligned16(vt))
    return H3Q_ERR_INVALID_ARG;
  const dim3 grid(static_cast<unsigned>((S + 127) / 128), static_cast<unsigned>(H));
  h3q::attn_prep_kernel<<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(q),
                                                  static_cast<const __nv_bfloat16*>(k),
                                                  static_cast<const __nv_bfloat16*>(v), static_cast<int>(S), ld, qq,
                                                  qs, kq, ks, static_cast<__nv_bfloat16*>(vt));
  return cudaGetLastError() == cudaSuccess ? H3Q_OK : H3Q_ERR_CUDA;
}

h3q_status h3q_attention_int8(const void* q, const void* k, const void* v, int64_t S, int64_t H, int64_t ld,
                              void* out, int64_t ld_out, void* workspace, size_t workspace_bytes,
                              cudaStream_t stream) {
  h3q_status st = check_att_args(q, k, v, S, H, ld);
  if (st != H3Q_OK || S == 0) return st;
  if (!out || !aligned16(out) || ld_out < H * 128 || ld_out % 8 != 0 || !workspace ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return H3Q_ERR_INVALID_ARG;
  const AttLayout lay = att_layout(S, H);
  if (workspace_bytes < lay.total) return H3Q_ERR_INVALID_ARG;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int8_t* qq = reinterpret_cast<int8_t*>(ws + lay.qq);
  int8_t* kq = reinterpret_cast<int8_t*>(ws + lay.kq);
  float* qs = reinterpret_cast<float*>(ws + lay.qs);
  float* ks = reinterpret_cast<float*>(ws + lay.ks);
  void* vt = ws + lay.vt;
  st = h3q_attention_prep(q, k, v, S, H, ld, qq, qs, kq, ks, vt, stream);
  if (st != H3Q_OK) return st;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_i8(&tq, qq, H * S, 128) || !make_tmap_i8(&tk, kq, H * S, 128) ||
      !make_tmap_bf16(&tv, vt, H * 128, S))
    return H3Q_ERR_CUDA;
  if (ensure_smem_attr(reinterpret_cast<const void*>(h3q::attn_kernel), static_cast<int>(h3q::kAttSmem)) !=
      cudaSuccess)
    return H3Q_ERR_CUDA;
  // the kernel's register split assumes this many registers per thread at launch
  // (a property of the compiled kernel, the same on every device)
  static std::once_flag regs_once;
  static bool regs_ok = false;
  std::call_once(regs_once, [] {
    cudaFuncAttributes fa{};
    regs_ok = cudaFuncGetAttributes(&fa, h3q::attn_kernel) == cudaSuccess &&
              fa.numRegs >= static_cast<int>(h3q::kAttRegsLaunch);
  });
  if (!regs_ok) return H3Q_ERR_UNSUPPORTED;
  h3q::AttParams p{};
  p.S = static_cast<int>(S);
  p.H = static_cast<int>(H);
  p.qs = qs;
  p.ks = ks;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.ld_out = ld_out;
  p.c = static_cast<float>(1.4426950408889634 / std::sqrt(128.0));
  p.wait_limit_ns = g_wait_limit_ns.load();
  const dim3 grid(static_cast<unsigned>((S + 127) / 128), static_cast<unsigned>(H));
  h3q::attn_kernel<<<grid, h3q::kAttThreads, h3q::kAttSmem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? H3Q_OK : H3Q_ERR_CUDA;
}

h3q_status h3q_gemm_s32(const int8_t* xq, const int8_t* wq, int64_t M, int64_t N, int64_t K, int32_t* acc,
                        cudaStream_t stream) {
  if (M < 0 || N <= 0 || N % 8 != 0 || K < 128 || K % 128 != 0) return H3Q_ERR_INVALID_ARG;
  if (M == 0) return H3Q_OK;
  if (!xq || !wq || !acc || !aligned16(xq) || !aligned16(wq) || !aligned16(acc)) return H3Q_ERR_INVALID_ARG;
  if (M > INT32_MAX - 256 || N > INT32_MAX - 512 || K > INT32_MAX) return H3Q_ERR_UNSUPPORTED;
  return launch_gemm<h3q::kEpiS32>(xq, wq, M, K, N, N, nullptr, nullptr, nullptr, acc, stream);
}

size_t h3q_ffn_workspace_size(int64_t M, int64_t K, int64_t F) {
  if (M < 0 || K <= 0 || F <= 0) return 0;
  return ffn_layout(M, K, F).total;
}

h3q_status h3q_ffn(const void* x_bf16, int64_t M, int64_t K, const int8_t* w_gu, const float* s_gu,
                   const void* b_gu, int64_t F, const int8_t* w_down, const float* s_down, const void* b_down,
                   void* y_bf16, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (M < 0 || !valid_k(K) || !valid_k(F)) return H3Q_ERR_INVALID_ARG;
  if (M == 0) return H3Q_OK;
  if (!x_bf16 || !w_gu || !s_gu || !w_down || !s_down || !y_bf16 || !workspace) return H3Q_ERR_INVALID_ARG;
  if (!aligned16(x_bf16) || !aligned16(w_gu) || !aligned16(s_gu) || !aligned16(w_down) || !aligned16(s_down) ||
      !aligned16(y_bf16) || (b_gu && !aligned16(b_gu)) || (b_down && !aligned16(b_down)) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return H3Q_ERR_INVALID_ARG;
  if (K > H3Q_MAX_K || F > H3Q_MAX_K || M > INT32_MAX - 256) return H3Q_ERR_UNSUPPORTED;
  const FfnLayout l = ffn_layout(M, K, F);
  if (workspace_bytes < l.total) return H3Q_ERR_INVALID_ARG;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int8_t* xq = reinterpret_cast<int8_t*>(ws + l.xq);
  float* sx = reinterpret_cast<float*>(ws + l.sx);
  void* h = ws + l.h;
  int8_t* hq = reinterpret_cast<int8_t*>(ws + l.hq);
  float* sh = reinterpret_cast<float*>(ws + l.sh);
  h3q_status st = h3q_rotate_quant(x_bf16, M, K, xq, sx, stream);
  if (st != H3Q_OK) return st;
  st = h3q_linear_w8a8(xq, sx, M, K, w_gu, s_gu, 2 * F, b_gu, H3Q_EPI_SWIGLU, h, stream);
  if (st != H3Q_OK) return st;
  st = h3q_rotate_quant(h, M, F, hq, sh, stream);
  if (st != H3Q_OK) return st;
  return h3q_linear_w8a8(hq, sh, M, F, w_down, s_down, K, b_down, H3Q_EPI_NONE, y_bf16, stream);
}

h3q_status h3q_ffn_static_scratch(const void* x_bf16, int64_t M, int64_t K, const int8_t* w_gu, const float* s_gu,
                                  const void* b_gu, int64_t F, const int8_t* w_down, const float* s_down,
                                  const void* b_down, void* y_bf16, cudaStream_t stream) {
  if (M < 0 || !valid_k(K) || !valid_k(F)) return H3Q_ERR_INVALID_ARG;
  if (M == 0) return H3Q_OK;
  if (ffn_layout(M, K, F).total > size_t(H3Q_STATIC_SCRATCH_BYTES)) return H3Q_ERR_UNSUPPORTED;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return H3Q_ERR_CUDA;
  void* scratch = static_scratch_address(device);
  if (scratch == nullptr) return H3Q_ERR_CUDA;
  return h3q_ffn(x_bf16, M, K, w_gu, s_gu, b_gu, F, w_down, s_down, b_down, y_bf16, scratch,
                 size_t(H3Q_STATIC_SCRATCH_BYTES), stream);
}

h3q_status h3q_get_device_status(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return H3Q_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, h3q::g_status, sizeof(v)) != cudaSuccess) return H3Q_ERR_CUDA;
  if (v != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(h3q::g_status, &zero, sizeof(zero)) != cudaSuccess) return H3Q_ERR_CUDA;
    return H3Q_ERR_TIMEOUT;
  }
  return H3Q_OK;
}

h3q_status h3q_test_stalled_wait(uint64_t limit_ns, cudaStream_t stream) {
  if (limit_ns > 10000000000ull) return H3Q_ERR_INVALID_ARG;  // at most 10 s
  h3q::stalled_wait_kernel<<<1, 64, 0, stream>>>(limit_ns < 1000 ? 1000 : limit_ns);
  return cudaGetLastError() == cudaSuccess ? H3Q_OK : H3Q_ERR_CUDA;
}

}  // extern "C"
