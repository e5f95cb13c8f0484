/*
 * Seeded synthetic inputs for the W4A16 group-quantized linear layer.
 *
 * This file holds no quantization or matmul arithmetic: it only draws the
 * fp16 weight matrix W [N][K] and the fp16 activations x [M][K] that both the
 * CPU oracle and the CUDA path consume.
 *
 * Generator (counter-based, so any element can be drawn independently and the
 * work splits across threads without changing the result):
 *   - splitmix64 finaliser (S. Vigna's public-domain mixer):
 *       z = v + 0x9E3779B97F4A7C15
 *       z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9
 *       z = (z ^ (z >> 27)) * 0x94D049BB133111EB
 *       z =  z ^ (z >> 31)
 *   - 64-bit word i of stream `key` is mix(key + i * 0x9E3779B97F4A7C15),
 *     i.e. the i-th output of a splitmix64 generator seeded with `key`.
 *   - uniform u in (0, 1]: ((word >> 11) + 1) * 2^-53.
 *   - Box-Muller on the pair (u1, u2) = (word 2j, word 2j+1):
 *       r = sqrt(-2 ln u1); normal[2j] = r cos(2 pi u2); normal[2j+1] = r sin(2 pi u2)
 *   - the fp16 value is the nearest binary16 (ties to even) of std * normal,
 *     multiplied first by `outlier_mult` for the selected input channels.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t v) {
  uint64_t z = v + GOLDEN;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t word_at(uint64_t key, uint64_t i) { return mix64(key + i * GOLDEN); }

static inline double unit_open0(uint64_t w) { return (double)((w >> 11) + 1) * 0x1.0p-53; }

/* Stream key for (seed, config id, tensor id). */
uint64_t synth_key(uint64_t seed, uint64_t config_id, uint64_t tensor_id) {
  return mix64(mix64(mix64(seed) ^ (config_id * 0xD1B54A32D192ED03ULL)) ^
               (tensor_id * 0x8CB92BA72F3D8DD7ULL));
}

/* Raw 64-bit words (exposed so the tests can pin the mixer). */
void synth_words(uint64_t key, int64_t start, int64_t count, uint64_t* out) {
  for (int64_t i = 0; i < count; ++i) out[i] = word_at(key, (uint64_t)(start + i));
}

/* Standard normal of element e of stream `key`. */
static inline double normal_at(uint64_t key, uint64_t e) {
  uint64_t j = e >> 1;
  double u1 = unit_open0(word_at(key, 2 * j));
  double u2 = unit_open0(word_at(key, 2 * j + 1));
  double r = sqrt(-2.0 * log(u1));
  double a = 6.283185307179586476925286766559 * u2;
  return (e & 1) ? r * sin(a) : r * cos(a);
}

static inline uint16_t to_half_bits(double d) {
  _Float16 h = (_Float16)d;
  uint16_t b;
  memcpy(&b, &h, 2);
  return b;
}

/* out[i] = fp16(std * normal(start + i)), i in [0, count). */
void synth_normal_f16(uint64_t key, int64_t start, int64_t count, double std, uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < count; ++i) out[i] = to_half_bits(std * normal_at(key, (uint64_t)(start + i)));
}

/* Rows [row0, row0 + rows) of a [*][K] matrix whose element (n, k) is
 * fp16(std * normal(n * K + k) * (chan_mult[k])). chan_mult may be NULL. */
void synth_matrix_f16(uint64_t key, int64_t row0, int64_t rows, int64_t K, double std,
                      const double* chan_mult, uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    uint64_t base = (uint64_t)((row0 + r) * K);
    uint16_t* o = out + r * K;
    for (int64_t k = 0; k < K; ++k) {
      double v = std * normal_at(key, base + (uint64_t)k);
      if (chan_mult) v *= chan_mult[k];
      o[k] = to_half_bits(v);
    }
  }
}

/* `count` distinct channel indices out of [0, K): the first `count` entries of
 * a Fisher-Yates shuffle of 0..K-1 driven by stream `key`. */
int synth_pick_channels(uint64_t key, int64_t K, int64_t count, int64_t* perm_scratch, int64_t* out) {
  if (count < 0 || count > K) return -1;
  for (int64_t i = 0; i < K; ++i) perm_scratch[i] = i;
  for (int64_t i = 0; i < count; ++i) {
    uint64_t span = (uint64_t)(K - i);
    /* unbiased draw in [0, span) by rejection */
    uint64_t limit = UINT64_MAX - (UINT64_MAX % span);
    uint64_t w, c = 0;
    do {
      w = word_at(key, (uint64_t)i * 64 + c);
      ++c;
    } while (w >= limit);
    int64_t j = i + (int64_t)(w % span);
    int64_t t = perm_scratch[i];
    perm_scratch[i] = perm_scratch[j];
    perm_scratch[j] = t;
    out[i] = perm_scratch[i];
  }
  return 0;
}
