/*
 * Seeded, counter-based input generator shared by the CPU oracle's tests and
 * the GPU path's tests and benchmark.  It builds synthetic inputs only
 * (weights, KV-cache contents, token ids, context lengths) and holds none of
 * the decode step's arithmetic.
 *
 * Every value is a pure function of (seed, tensor_id, index), so any slice of
 * any tensor can be regenerated on its own, in any order, on any machine:
 *
 *   key  = SplitMix64(seed XOR SplitMix64(tensor_id))
 *   u    = SplitMix64(key + index)                  (64 fresh bits per element)
 *
 * SplitMix64 is the finaliser published by Steele, Lea and Flood ("Fast
 * splittable pseudorandom number generators", OOPSLA 2014) with the constants
 * of Vigna's public-domain reference version.
 *
 * Normal-shaped values use the Irwin-Hall sum of four 16-bit uniforms taken
 * from the 64 bits of u:  S = a0+a1+a2+a3 + 2 - 131072 is an exact integer
 * whose law is that of 65536*(U1+U2+U3+U4-2) with Ui uniform on (0,1), so
 * S*sqrt(3)/65536 has mean 0 and variance 1 (bounded at +-3.46).  The value
 * is the single IEEE fp32 product (float)S * (float)(sqrt(3)*sigma/65536),
 * rounded to bfloat16 with round-to-nearest-even.  Only integer operations and
 * one correctly rounded multiply are involved, so every platform gets the same
 * bits.
 *
 * Uniform integers in [lo, hi] use the high 64 bits of the 128-bit product
 * u * (hi - lo + 1) (Lemire's multiply-shift map).
 */
#include <stdint.h>
#include <math.h>

static inline uint64_t fx_mix(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

uint64_t fx_splitmix64(uint64_t z) { return fx_mix(z); }

uint64_t fx_key(uint64_t seed, uint64_t tensor_id) { return fx_mix(seed ^ fx_mix(tensor_id)); }

/* fp32 -> bf16 bits, round to nearest even (inputs here are finite). */
static inline uint16_t fx_f32_to_bf16(float f) {
  union { float f; uint32_t u; } v;
  v.f = f;
  uint32_t u = v.u;
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

static inline float fx_normal_f32(uint64_t key, uint64_t index, float scale) {
  uint64_t u = fx_mix(key + index);
  int32_t s = (int32_t)(u & 0xFFFF) + (int32_t)((u >> 16) & 0xFFFF) + (int32_t)((u >> 32) & 0xFFFF) +
              (int32_t)((u >> 48) & 0xFFFF) + 2 - 131072;
  return (float)s * scale;
}

/* out[i] = bf16(sigma * N01(seed, tensor_id, offset + i)), i < n. */
void fx_normal_bf16(uint64_t seed, uint64_t tensor_id, uint64_t offset, uint64_t n, double sigma,
                    uint16_t* out) {
  const uint64_t key = fx_key(seed, tensor_id);
  const float scale = (float)(sqrt(3.0) * sigma / 65536.0);
  int64_t nn = (int64_t)n;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < nn; ++i) out[i] = fx_f32_to_bf16(fx_normal_f32(key, offset + (uint64_t)i, scale));
}

/* out[i] = lo + floor(u * (hi - lo + 1) / 2^64), i < n. */
void fx_uniform_int(uint64_t seed, uint64_t tensor_id, uint64_t offset, uint64_t n, int64_t lo, int64_t hi,
                    int32_t* out) {
  const uint64_t key = fx_key(seed, tensor_id);
  const unsigned __int128 span = (unsigned __int128)(uint64_t)(hi - lo + 1);
  for (uint64_t i = 0; i < n; ++i) {
    uint64_t u = fx_mix(key + offset + i);
    out[i] = (int32_t)(lo + (int64_t)(uint64_t)(((unsigned __int128)u * span) >> 64));
  }
}

/* Fill n bf16 words with one bit pattern (used for norm gains of 1.0). */
void fx_fill_u16(uint16_t value, uint64_t n, uint16_t* out) {
  int64_t nn = (int64_t)n;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < nn; ++i) out[i] = value;
}
