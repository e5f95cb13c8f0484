/*
 * CPU oracle for the W4A16 group-quantized linear layer  y = x . dequant(Wq)^T.
 *
 * TEST INFRASTRUCTURE ONLY. This file is compiled into liborc.so and is used by
 * the tests, by the smoke check and by the CPU-baseline leg of the benchmark.
 * The product (the CUDA library) never links, loads or calls it, and it shares
 * no code, header, table or constant generator with the CUDA path.
 *
 * What it computes, and the passage each step follows:
 *   - TinyChat README, "Usage" step 3: weights are quantized to 4 bits
 *     ("--w_bit 4") in groups of 128 input channels ("--q_group_size 128"), and
 *     "Speed Benchmarks": the INT4 model runs as W4A16 (4-bit weights, fp16
 *     activations).  Each weight is w = (q - z) * s with an fp16 scale s and a
 *     4-bit zero point z per (output channel, group).
 *   - The pages print no quantization formula.  This oracle takes the plainest
 *     reading, asymmetric min-max over the group's raw values:
 *         lo = min v, hi = max v, R = max(hi - lo, 1e-5)
 *         s  = fp16_rne(R / 15)            (fp64 divide, then one fp16 rounding)
 *         z  = clamp(rint(-lo / s), 0, 15)
 *         q  = clamp(rint(v / s) + z, 0, 15)
 *     with rint = round half to even, every division in fp64 against the
 *     stored fp16 scale.
 *   - dequant: W^[n,k] = fp16_rne((q - z) * s)  (the product is exact in fp64).
 *   - matmul: y[m,n] = sum_k x[m,k] * W^[n,k] in fp64, in increasing k, and the
 *     error scale B[m,n] = sum_k |x[m,k] * W^[n,k]|.
 *   - a second, independent matmul route that factors the zero point out of
 *     each group:  y[m,n] = sum_g s * (sum_{k in g} x*q  -  z * sum_{k in g} x).
 *   - the packed layout (our own; the pages only name a ".pt" checkpoint):
 *       qweight  uint32, 1 KiB blocks of 16 rows x 128 input channels.
 *                Block (nb, kb) holds rows n = 16nb + r (r = 0..15) and
 *                k = 128kb .. 128kb+127; word w of row r holds the eight
 *                inputs k = 128kb + k0(w) + i, i = 0..7, with the nibble of
 *                even i at bits 4*(i/2) and of odd i at bits 16 + 4*(i/2).
 *                (So (word >> 4j) & 0x000F000F holds the adjacent pair
 *                k0+2j, k0+2j+1 as two 16-bit lanes.)  For G = 128 (and any
 *                multiple of 128) k0(w) = 8w. For G = 64 or 32, with
 *                w = 4t + j (t, j = 0..3) and J = G/32:
 *                  k0(w) = G*(j / J) + 8*(t*J + j % J),
 *                so the four words 4t .. 4t+3 that a GPU lane reads at once
 *                hold inputs of every group of the k-block, and the four
 *                words with the same j hold whole groups (group j / J).
 *                Blocks are grouped by 8 row blocks (128 rows): group
 *                gi = nb / 8 has R = min(8, N/16 - 8gi) row blocks and is
 *                stored k-block-major, so block (nb, kb) is block number
 *                8*gi*(K/128) + kb*R + nb%8 and the R blocks of one k-block of
 *                one group are contiguous.
 *       scales   fp16  [K/G][N]
 *       zeros    uint8 [K/G][N/2]: low nibble = even n, high nibble = odd n.
 *
 * A W4A8-FP8 variant (E4M3 activations and weights, fp32 accumulation) is at
 * the end of the file, with its own statement of what it computes.
 *
 * fp16 conversions below are written from the IEEE 754 binary16 definition
 * (1 sign bit, 5 exponent bits with bias 15, 10 fraction bits; exponent field
 * 0 encodes subnormals f * 2^-24).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_SHAPE 2
#define ORC_ERR_NONFINITE 8

/* ------------------------------------------------------------------------- */
/* binary16 <-> binary64                                                      */
/* ------------------------------------------------------------------------- */

double orc_half_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1F;
  int f = h & 0x3FF;
  double v;
  if (e == 0)
    v = ldexp((double)f, -24);                /* subnormal (or zero): f * 2^-24 */
  else if (e == 31)
    v = f ? NAN : INFINITY;
  else
    v = ldexp((double)(1024 + f), e - 25);    /* (1 + f/1024) * 2^(e-15) */
  return sign ? -v : v;
}

/* Nearest binary16, ties to even, with gradual underflow and overflow to inf. */
uint16_t orc_double_to_half(double d) {
  uint16_t sign = signbit(d) ? 0x8000 : 0;
  if (isnan(d)) return 0x7E00;
  double a = fabs(d);
  if (isinf(a) || a >= 65536.0) return sign | 0x7C00;
  if (a == 0.0) return sign;
  int E;
  frexp(a, &E);          /* a = m * 2^E, m in [0.5, 1): floor(log2 a) = E - 1 */
  int e = E - 1;
  if (e < -14) e = -14;  /* below the normal range the spacing stays 2^-24 */
  double quantum = ldexp(1.0, e - 10);   /* spacing of binary16 values near a */
  double t = a / quantum;                /* exact: scaling by a power of two */
  double r = rint(t);                    /* nearest integer, ties to even */
  int biased = e + 15;
  uint32_t bits;
  if (biased == 1 && r < 1024.0) {
    bits = (uint32_t)r;                  /* subnormal: value r * 2^-24 */
  } else {
    if (r >= 2048.0) { r = 1024.0; biased += 1; }  /* carry into the next binade */
    if (biased >= 31) return sign | 0x7C00;
    bits = ((uint32_t)biased << 10) | (uint32_t)(r - 1024.0);
  }
  return sign | (uint16_t)bits;
}

/* ------------------------------------------------------------------------- */
/* quantization                                                              */
/* ------------------------------------------------------------------------- */

static int bad_shape(int64_t N, int64_t K, int G) {
  return N <= 0 || K <= 0 || G <= 0 || K % G != 0 || K % 128 != 0 || N % 16 != 0;
}

/* Quantize one group of G values v[0..G-1] (exact fp16 values held as doubles). */
static int quantize_group(const double* v, int G, uint8_t* q_out, uint8_t* z_out, uint16_t* s_out) {
  double lo = v[0], hi = v[0];
  for (int j = 0; j < G; ++j) {
    if (!isfinite(v[j])) return ORC_ERR_NONFINITE;
    if (v[j] < lo) lo = v[j];
    if (v[j] > hi) hi = v[j];
  }
  double R = hi - lo;            /* exact: both are binary16 values */
  if (R < 1e-5) R = 1e-5;
  uint16_t s16 = orc_double_to_half(R / 15.0);
  double s = orc_half_to_double(s16);
  double z = rint(-lo / s);
  if (z < 0.0) z = 0.0;
  if (z > 15.0) z = 15.0;
  for (int j = 0; j < G; ++j) {
    double q = rint(v[j] / s) + z;
    if (q < 0.0) q = 0.0;
    if (q > 15.0) q = 15.0;
    q_out[j] = (uint8_t)q;
  }
  *z_out = (uint8_t)z;
  *s_out = s16;
  return ORC_OK;
}

/* W fp16 [N][K] -> q uint8 [N][K], z uint8 [N][K/G], s fp16 [N][K/G].
 * Returns ORC_ERR_NONFINITE if any weight is inf/NaN (the other groups are
 * still quantized; the offending group's outputs are left untouched). */
int orc_quantize(const uint16_t* W, int64_t N, int64_t K, int G, uint8_t* q, uint8_t* z, uint16_t* s) {
  if (bad_shape(N, K, G)) return ORC_ERR_SHAPE;
  int64_t ng = K / G;
  int rc = ORC_OK;
  double* v = (double*)malloc(sizeof(double) * (size_t)G);
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t g = 0; g < ng; ++g) {
      for (int j = 0; j < G; ++j) v[j] = orc_half_to_double(W[n * K + g * G + j]);
      int r = quantize_group(v, G, q + n * K + g * G, z + n * ng + g, s + n * ng + g);
      if (r != ORC_OK) rc = r;
    }
  }
  free(v);
  return rc;
}

/* W^ fp16 [N][K] = fp16_rne((q - z) * s). */
int orc_dequant(const uint8_t* q, const uint8_t* z, const uint16_t* s, int64_t N, int64_t K, int G,
                uint16_t* What) {
  if (bad_shape(N, K, G)) return ORC_ERR_SHAPE;
  int64_t ng = K / G;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      int64_t g = k / G;
      double sd = orc_half_to_double(s[n * ng + g]);
      double w = ((double)q[n * K + k] - (double)z[n * ng + g]) * sd;
      What[n * K + k] = orc_double_to_half(w);
    }
  return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* packed layout                                                             */
/* ------------------------------------------------------------------------- */

/* Bit position of element i (0..7) inside its 32-bit word. */
static int nibble_shift(int i) { return (i % 2 == 0) ? 4 * (i / 2) : 16 + 4 * (i / 2); }

/* Word (0..15) of its row that holds input k (0..127) of a k-block, the
 * inverse of k0(w) above; -1 for a group size the layout does not define. */
static int word_in_row(int k, int G) {
  if (G % 128 == 0) return k / 8;
  if (G != 32 && G != 64) return -1;
  int J = G / 32;
  int group = k / G, p = (k % G) / 8;  /* 8-input piece p of group `group` */
  int t = p / J, j = group * J + p % J;
  return 4 * t + j;
}

/* Index of the word holding (n, k): block number (group-major, k-block,
 * row block within the group), then row r and word w inside the block. */
static int64_t word_index(int64_t n, int64_t k, int64_t K, int64_t N, int G) {
  int64_t nb = n / 16, r = n % 16, kb = k / 128, w = word_in_row((int)(k % 128), G);
  int64_t gi = nb / 8, NB = N / 16;
  int64_t rows_in_group = (NB - 8 * gi < 8) ? NB - 8 * gi : 8;
  int64_t block = 8 * gi * (K / 128) + kb * rows_in_group + nb % 8;
  return (block * 16 + r) * 16 + w;
}

int orc_pack(const uint8_t* q, const uint8_t* z, const uint16_t* s, int64_t N, int64_t K, int G,
             uint32_t* qweight, uint16_t* scales, uint8_t* zeros) {
  if (bad_shape(N, K, G) || word_in_row(0, G) < 0) return ORC_ERR_SHAPE;
  int64_t ng = K / G;
  memset(qweight, 0, sizeof(uint32_t) * (size_t)(N * K / 8));
  memset(zeros, 0, (size_t)(ng * N / 2));
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k)
      qweight[word_index(n, k, K, N, G)] |= (uint32_t)(q[n * K + k] & 0xF) << nibble_shift((int)(k % 8));
  for (int64_t g = 0; g < ng; ++g)
    for (int64_t n = 0; n < N; ++n) {
      scales[g * N + n] = s[n * ng + g];
      zeros[g * (N / 2) + n / 2] |= (uint8_t)((z[n * ng + g] & 0xF) << (4 * (n % 2)));
    }
  return ORC_OK;
}

int orc_unpack(const uint32_t* qweight, const uint16_t* scales, const uint8_t* zeros, int64_t N, int64_t K,
               int G, uint8_t* q, uint8_t* z, uint16_t* s) {
  if (bad_shape(N, K, G) || word_in_row(0, G) < 0) return ORC_ERR_SHAPE;
  int64_t ng = K / G;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k)
      q[n * K + k] = (uint8_t)((qweight[word_index(n, k, K, N, G)] >> nibble_shift((int)(k % 8))) & 0xF);
  for (int64_t g = 0; g < ng; ++g)
    for (int64_t n = 0; n < N; ++n) {
      s[n * ng + g] = scales[g * N + n];
      z[n * ng + g] = (uint8_t)((zeros[g * (N / 2) + n / 2] >> (4 * (n % 2))) & 0xF);
    }
  return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* matmul                                                                    */
/* ------------------------------------------------------------------------- */

/* y[m][n] = sum_k x[m][k] * W^[n][k] (fp64, increasing k); bound = sum |.|. */
int orc_matmul(const uint16_t* x, int64_t M, const uint16_t* What, int64_t N, int64_t K, double* y,
               double* bound) {
  if (M < 0 || N <= 0 || K <= 0) return ORC_ERR_SHAPE;
  double* wd = (double*)malloc(sizeof(double) * (size_t)K);
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k) wd[k] = orc_half_to_double(What[n * K + k]);
    for (int64_t m = 0; m < M; ++m) {
      double acc = 0.0, b = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        double p = orc_half_to_double(x[m * K + k]) * wd[k];
        acc += p;
        b += fabs(p);
      }
      y[m * N + n] = acc;
      if (bound) bound[m * N + n] = b;
    }
  }
  free(wd);
  return ORC_OK;
}

/* Second route: zero point factored out of each group. */
int orc_matmul_factored(const uint16_t* x, int64_t M, const uint8_t* q, const uint8_t* z, const uint16_t* s,
                        int64_t N, int64_t K, int G, double* y) {
  if (M < 0 || bad_shape(N, K, G)) return ORC_ERR_SHAPE;
  int64_t ng = K / G;
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int64_t g = 0; g < ng; ++g) {
        double sxq = 0.0, sx = 0.0;
        for (int j = 0; j < G; ++j) {
          double xv = orc_half_to_double(x[m * K + g * G + j]);
          sxq += xv * (double)q[n * K + g * G + j];
          sx += xv;
        }
        acc += orc_half_to_double(s[n * ng + g]) * (sxq - (double)z[n * ng + g] * sx);
      }
      y[m * N + n] = acc;
    }
  return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* the whole linear layer from the packed buffers                            */
/* ------------------------------------------------------------------------- */

/* Dequantized row n of the packed weight: W^[n][0..K). */
static void packed_row(const uint32_t* qweight, const uint16_t* scales, const uint8_t* zeros, int64_t N,
                       int64_t K, int G, int64_t n, double* row) {
  for (int64_t k = 0; k < K; ++k) {
    int64_t g = k / G;
    uint32_t q = (qweight[word_index(n, k, K, N, G)] >> nibble_shift((int)(k % 8))) & 0xF;
    uint32_t z = (zeros[g * (N / 2) + n / 2] >> (4 * (n % 2))) & 0xF;
    double s = orc_half_to_double(scales[g * N + n]);
    row[k] = orc_half_to_double(orc_double_to_half(((double)q - (double)z) * s));
  }
}

/* y, bound [M][n1-n0]: output channels n0..n1-1 of x . W^T, straight from the
 * packed buffers (unpack, dequant, fp64 dot products). */
int orc_linear_rows(const uint16_t* x, int64_t M, const uint32_t* qweight, const uint16_t* scales,
                    const uint8_t* zeros, int64_t N, int64_t K, int G, int64_t n0, int64_t n1, double* y,
                    double* bound) {
  if (M < 0 || bad_shape(N, K, G) || word_in_row(0, G) < 0 || n0 < 0 || n1 > N || n0 > n1) return ORC_ERR_SHAPE;
  int64_t W = n1 - n0;
  double* row = (double*)malloc(sizeof(double) * (size_t)K);
  for (int64_t n = n0; n < n1; ++n) {
    packed_row(qweight, scales, zeros, N, K, G, n, row);
    for (int64_t m = 0; m < M; ++m) {
      double acc = 0.0, b = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        double p = orc_half_to_double(x[m * K + k]) * row[k];
        acc += p;
        b += fabs(p);
      }
      y[m * W + (n - n0)] = acc;
      if (bound) bound[m * W + (n - n0)] = b;
    }
  }
  free(row);
  return ORC_OK;
}

int orc_linear(const uint16_t* x, int64_t M, const uint32_t* qweight, const uint16_t* scales,
               const uint8_t* zeros, int64_t N, int64_t K, int G, double* y, double* bound) {
  return orc_linear_rows(x, M, qweight, scales, zeros, N, K, G, 0, N, y, bound);
}

/* Individual outputs (ms[i], ns[i]) of x . W^T from the packed buffers. */
int orc_linear_entries(const uint16_t* x, int64_t M, const uint32_t* qweight, const uint16_t* scales,
                       const uint8_t* zeros, int64_t N, int64_t K, int G, const int64_t* ms,
                       const int64_t* ns, int64_t count, double* y, double* bound) {
  if (M < 0 || bad_shape(N, K, G) || word_in_row(0, G) < 0) return ORC_ERR_SHAPE;
  double* row = (double*)malloc(sizeof(double) * (size_t)K);
  int64_t cached = -1;
  for (int64_t i = 0; i < count; ++i) {
    int64_t m = ms[i], n = ns[i];
    if (m < 0 || m >= M || n < 0 || n >= N) { free(row); return ORC_ERR_SHAPE; }
    if (n != cached) { packed_row(qweight, scales, zeros, N, K, G, n, row); cached = n; }
    double acc = 0.0, b = 0.0;
    for (int64_t k = 0; k < K; ++k) {
      double p = orc_half_to_double(x[m * K + k]) * row[k];
      acc += p;
      b += fabs(p);
    }
    y[i] = acc;
    if (bound) bound[i] = b;
  }
  free(row);
  return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* W4A8-FP8 variant                                                           */
/* ------------------------------------------------------------------------- */
/*
 * The TensorRT-LLM news item on INT4 AWQ on one H200 says its AWQ kernels
 * compute in FP8 on Hopper's tensor cores. The pages give no recipe; this is
 * the plainest reading, with the 4-bit weights and their fp16 group scales
 * unchanged:
 *   - activations: per token m, sx[m] = fp32(amax_k |x[m,k]|) / 448 and
 *     x8[m,k] = e4m3(x[m,k] / sx[m]), both divisions IEEE binary32 (448 is the
 *     largest finite E4M3 value); a row of zeros gives sx = 0 and x8 = 0.
 *   - weights: per output channel n, S_n = max over its groups of s, and e[n]
 *     the largest integer with 15 * S_n * 2^e <= 448 (every |q - z| <= 15, so
 *     the scaled weights stay within the E4M3 range). With the scale moved by
 *     that power of two, s' = fp16_rne(s * 2^e[n]) (exact unless it falls
 *     below the fp16 normal range), W8[n,k] = e4m3(fp16_rne((q - z) * s')).
 *     Wherever W^ = fp16_rne((q - z) s) is an fp16 normal number this is
 *     e4m3(W^ * 2^e[n]): scaling by a power of two commutes with rounding.
 *   - y[m,n] = sum_k (x8[m,k] sx[m]) (W8[n,k] 2^-e[n]), here in fp64.
 * e4m3(v) rounds v to the nearest E4M3 value, ties to even, and saturates:
 * |v| >= 448 (or infinite) gives +-448; NaN gives 0x7F.
 *
 * E4M3 (OCP 8-bit floating point, the "FN" variant): 1 sign bit, 4 exponent
 * bits with bias 7, 3 fraction bits, no infinities; exponent field 0 encodes
 * subnormals f * 2^-9; exponent 15 with fraction 7 is NaN (0x7F, 0xFF), so
 * the largest finite value is 1.75 * 2^8 = 448.
 */

double orc_e4m3_to_double(uint8_t b) {
  int sign = (b >> 7) & 1;
  int e = (b >> 3) & 0xF;
  int f = b & 7;
  double v;
  if (e == 15 && f == 7)
    v = NAN;
  else if (e == 0)
    v = ldexp((double)f, -9);               /* subnormal: f * 2^-9 */
  else
    v = ldexp((double)(8 + f), e - 10);     /* (1 + f/8) * 2^(e-7) */
  return sign ? -v : v;
}

uint8_t orc_double_to_e4m3(double d) {
  if (isnan(d)) return 0x7F;
  uint8_t sign = signbit(d) ? 0x80 : 0x00;
  double a = fabs(d);
  if (a >= 448.0) return sign | 0x7E;       /* saturate (infinities too) */
  if (a < ldexp(1.0, -6)) {
    /* subnormal spacing 2^-9: n = rint(a / 2^-9) in 0..8; n = 8 is the
       smallest normal value (code 0x08) */
    double n = rint(ldexp(a, 9));
    return sign | (uint8_t)n;
  }
  int ex;
  frexp(a, &ex);                            /* a = m 2^ex, m in [0.5, 1) */
  int e = ex - 1;                           /* 2^e <= a < 2^(e+1), e in -6 .. 8 */
  double n = rint(ldexp(a, 3 - e));         /* a / 2^(e-3), in 8 .. 16 */
  if (n == 16.0) { n = 8.0; ++e; }
  uint8_t code = (uint8_t)(((e + 7) << 3) | ((int)n - 8));
  if (code > 0x7E) code = 0x7E;
  return sign | code;
}

/* x8 [M][K] E4M3 codes and sx [M] (fp32) from x fp16 [M][K]. */
int orc_fp8_quantize_x(const uint16_t* x, int64_t M, int64_t K, uint8_t* x8, float* sx) {
  if (M < 0 || K <= 0) return ORC_ERR_SHAPE;
  for (int64_t m = 0; m < M; ++m) {
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      float a = (float)fabs(orc_half_to_double(x[m * K + k]));   /* exact: fp16 values are fp32 values */
      if (a > amax || isnan(a)) amax = a;
    }
    volatile float s = amax / 448.0f;   /* one IEEE binary32 division */
    sx[m] = s;
    for (int64_t k = 0; k < K; ++k) {
      if (s == 0.0f) { x8[m * K + k] = 0; continue; }
      volatile float v = (float)orc_half_to_double(x[m * K + k]) / s;   /* one IEEE binary32 division */
      x8[m * K + k] = orc_double_to_e4m3((double)v);
    }
  }
  return ORC_OK;
}

/* e [N] from scales fp16 [K/G][N] (packed layout). */
int orc_fp8_row_exponents(const uint16_t* scales, int64_t N, int64_t K, int G, int8_t* e) {
  if (bad_shape(N, K, G)) return ORC_ERR_SHAPE;
  for (int64_t n = 0; n < N; ++n) {
    double S = 0.0;
    for (int64_t g = 0; g < K / G; ++g) {
      double s = orc_half_to_double(scales[g * N + n]);
      if (s > S) S = s;
    }
    int ee = 0;
    if (S > 0.0) {
      int ex;
      frexp(448.0 / (15.0 * S), &ex);
      ee = ex - 1;                                         /* close to the answer */
      while (15.0 * ldexp(S, ee + 1) <= 448.0) ++ee;        /* exact: S 2^e is exact in fp64 */
      while (15.0 * ldexp(S, ee) > 448.0) --ee;
    }
    e[n] = (int8_t)ee;
  }
  return ORC_OK;
}

/* E4M3 code of weight (n, k), from the packed buffers. */
static uint8_t fp8_weight(const uint32_t* qweight, const uint16_t* scales, const uint8_t* zeros, const int8_t* e,
                          int64_t N, int64_t K, int G, int64_t n, int64_t k) {
  int64_t g = k / G;
  uint32_t q = (qweight[word_index(n, k, K, N, G)] >> nibble_shift((int)(k % 8))) & 0xF;
  uint32_t z = (zeros[g * (N / 2) + n / 2] >> (4 * (n % 2))) & 0xF;
  double s2 = orc_half_to_double(orc_double_to_half(ldexp(orc_half_to_double(scales[g * N + n]), e[n])));
  return orc_double_to_e4m3(orc_half_to_double(orc_double_to_half(((double)q - (double)z) * s2)));
}

/* W8 [N][K] E4M3 codes of the packed weight scaled by 2^e[n]. */
int orc_fp8_weights(const uint32_t* qweight, const uint16_t* scales, const uint8_t* zeros, const int8_t* e,
                    int64_t N, int64_t K, int G, uint8_t* w8) {
  if (bad_shape(N, K, G) || word_in_row(0, G) < 0) return ORC_ERR_SHAPE;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) w8[n * K + k] = fp8_weight(qweight, scales, zeros, e, N, K, G, n, k);
  return ORC_OK;
}

/* Row n of the W4A8-FP8 weight as the values it stands for: W8[n,k] 2^-e[n]. */
static void fp8_row(const uint32_t* qweight, const uint16_t* scales, const uint8_t* zeros, const int8_t* e,
                    int64_t N, int64_t K, int G, int64_t n, double* row) {
  for (int64_t k = 0; k < K; ++k)
    row[k] = ldexp(orc_e4m3_to_double(fp8_weight(qweight, scales, zeros, e, N, K, G, n, k)), -e[n]);
}

/* y, bound [M][n1-n0]: output channels n0..n1-1 of the W4A8-FP8 layer, from
 * x8, sx and the packed buffers, in fp64 in increasing k. */
int orc_fp8_linear_rows(const uint8_t* x8, const float* sx, int64_t M, const uint32_t* qweight,
                        const uint16_t* scales, const uint8_t* zeros, const int8_t* e, int64_t N, int64_t K, int G,
                        int64_t n0, int64_t n1, double* y, double* bound) {
  if (M < 0 || bad_shape(N, K, G) || word_in_row(0, G) < 0 || n0 < 0 || n1 > N || n0 > n1) return ORC_ERR_SHAPE;
  int64_t W = n1 - n0;
  double* row = (double*)malloc(sizeof(double) * (size_t)K);
  for (int64_t n = n0; n < n1; ++n) {
    fp8_row(qweight, scales, zeros, e, N, K, G, n, row);
    for (int64_t m = 0; m < M; ++m) {
      double acc = 0.0, b = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        double p = orc_e4m3_to_double(x8[m * K + k]) * (double)sx[m] * row[k];
        acc += p;
        b += fabs(p);
      }
      y[m * W + (n - n0)] = acc;
      if (bound) bound[m * W + (n - n0)] = b;
    }
  }
  free(row);
  return ORC_OK;
}

/* Individual outputs (ms[i], ns[i]) of the W4A8-FP8 layer. */
int orc_fp8_linear_entries(const uint8_t* x8, const float* sx, int64_t M, const uint32_t* qweight,
                           const uint16_t* scales, const uint8_t* zeros, const int8_t* e, int64_t N, int64_t K,
                           int G, const int64_t* ms, const int64_t* ns, int64_t count, double* y, double* bound) {
  if (M < 0 || bad_shape(N, K, G) || word_in_row(0, G) < 0) return ORC_ERR_SHAPE;
  double* row = (double*)malloc(sizeof(double) * (size_t)K);
  int64_t cached = -1;
  for (int64_t i = 0; i < count; ++i) {
    int64_t m = ms[i], n = ns[i];
    if (m < 0 || m >= M || n < 0 || n >= N) { free(row); return ORC_ERR_SHAPE; }
    if (n != cached) { fp8_row(qweight, scales, zeros, e, N, K, G, n, row); cached = n; }
    double acc = 0.0, b = 0.0;
    for (int64_t k = 0; k < K; ++k) {
      double p = orc_e4m3_to_double(x8[m * K + k]) * (double)sx[m] * row[k];
      acc += p;
      b += fabs(p);
    }
    y[i] = acc;
    if (bound) bound[i] = b;
  }
  free(row);
  return ORC_OK;
}
