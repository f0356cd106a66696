// Seeded synthetic tensors on the device: the generator defined in
// synth/__init__.py (splitmix64 streams, twelve 16-bit draws summed Irwin-Hall
// style). Used to fill large inputs in place; no step of the quantized layer is
// computed here. Built as its own library, separate from the layer's kernels.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t word(uint64_t key, uint64_t c) {
  return mix64(key + (c + 1) * 0x9E3779B97F4A7C15ull);
}

__host__ uint64_t host_word(uint64_t key, uint64_t c) {
  uint64_t z = key + (c + 1) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__global__ void fill_kernel(uint64_t key, int64_t row0, int64_t nrows, int64_t K, float scale,
                            const float* __restrict__ factors, int out_bf16, void* __restrict__ out) {
  const int64_t total = nrows * K;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / K, k = e - r * K;
    const uint64_t i = (uint64_t)((row0 + r) * K + k);
    int s = 0;
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const uint64_t w = word(key, 3 * i + (uint64_t)j);
      s += (int)(w & 0xFFFF) + (int)((w >> 16) & 0xFFFF) + (int)((w >> 32) & 0xFFFF) + (int)(w >> 48);
    }
    float v = __fmul_rn((float)(2 * s - 12 * 65535), 1.0f / 131072.0f);
    v = __fmul_rn(v, scale);
    if (factors) v = __fmul_rn(v, factors[k]);
    if (out_bf16) {
      uint32_t u = __float_as_uint(v);
      u += 0x7FFFu + ((u >> 16) & 1u);
      static_cast<uint16_t*>(out)[e] = (uint16_t)(u >> 16);
    } else {
      static_cast<float*>(out)[e] = v;
    }
  }
}

}  // namespace

extern "C" {

// Fill rows row0 .. row0+nrows-1 of a [*, K] tensor on the device. factors is a
// nullable device array [K]. Returns a cudaError_t value (0 = success).
int synth_fill_device(uint64_t seed, uint64_t tensor_id, int64_t row0, int64_t nrows, int64_t K, float scale,
                      const float* factors, int out_bf16, void* out, cudaStream_t stream) {
  if (nrows <= 0 || K <= 0) return 0;
  const uint64_t key = host_word(seed, tensor_id);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t total = nrows * K;
  int64_t blocks = (total + 255) / 256;
  if (blocks > (int64_t)sms * 32) blocks = (int64_t)sms * 32;
  fill_kernel<<<(unsigned)blocks, 256, 0, stream>>>(key, row0, nrows, K, scale, factors, out_bf16, out);
  return (int)cudaGetLastError();
}

}
