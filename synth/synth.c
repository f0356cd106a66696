/* Seeded synthetic tensors on the host: the generator defined in synth/__init__.py
 * (splitmix64 streams, twelve 16-bit draws summed Irwin-Hall style), written in C
 * for speed. No step of the quantized layer is computed here.
 *
 * out[r][k] = fp32( fp32(z(i) * scale) * factor[k] ), i = row(r) * K + k,
 * stored as fp32 or as bf16 bits (round to nearest even).
 */
#include <stdint.h>
#include <string.h>

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

static inline uint64_t word(uint64_t key, uint64_t c) { return mix64(key + (c + 1) * 0x9E3779B97F4A7C15ull); }

static inline float normal_at(uint64_t key, uint64_t i) {
  int64_t s = 0;
  for (int j = 0; j < 3; ++j) {
    const uint64_t w = word(key, 3 * i + (uint64_t)j);
    s += (int64_t)(w & 0xFFFF) + (int64_t)((w >> 16) & 0xFFFF) + (int64_t)((w >> 32) & 0xFFFF) +
         (int64_t)((w >> 48) & 0xFFFF);
  }
  return (float)(2 * s - 12 * 65535) * (1.0f / 131072.0f);
}

static inline uint16_t bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

uint64_t synth_stream_key(uint64_t seed, uint64_t tensor_id) { return word(seed, tensor_id); }

/* rows: nullable list of row indices (else rows row0 .. row0+nrows-1).
 * factors: nullable per-column multipliers [K]. out_bf16 != 0: out is uint16 bits. */
void synth_fill(uint64_t seed, uint64_t tensor_id, const int64_t* rows, int64_t row0, int64_t nrows, int64_t K,
                float scale, const float* factors, int out_bf16, void* out) {
  const uint64_t key = word(seed, tensor_id);
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < nrows; ++r) {
    const int64_t row = rows ? rows[r] : row0 + r;
    for (int64_t k = 0; k < K; ++k) {
      float v = normal_at(key, (uint64_t)(row * K + k)) * scale;
      if (factors) v = v * factors[k];
      if (out_bf16)
        ((uint16_t*)out)[r * K + k] = bf16_rne(v);
      else
        ((float*)out)[r * K + k] = v;
    }
  }
}
