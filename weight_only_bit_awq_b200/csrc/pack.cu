// Quantize + pack (awq_pack) and dequantize (awq_dequant).
//
// TinyChat README, Usage step 3 ("--w_bit 4 --q_group_size 128 ...
// --q_backend real"): fp16 weights become 4-bit codes with one fp16 scale and
// one 4-bit zero point per (output channel, group of 128 input channels);
// Falcon-7B uses groups of 64 (same step), so G = 64 and 32 are taken too.
// The arithmetic is asymmetric min-max (the pages print no formula; this is
// its plainest reading), done in fp64 against the stored fp16 scale so that
// the result is reproducible bit for bit:
//   R = max(hi - lo, 1e-5), s = fp16_rne(R / 15), z = clamp(rint(-lo / s), 0, 15),
//   q = clamp(rint(v / s) + z, 0, 15).
// This file is compiled with --fmad=false; its fp64 operations are single
// IEEE operations (division, rint, subtraction), none of which can contract.
#include "awq_internal.cuh"

namespace awq {
namespace {

// binary64 -> binary16, one rounding to nearest (ties to even): PTX cvt.rn.f16.f64.
__device__ __forceinline__ __half f64_to_f16_rn(double v) {
  unsigned short r;
  asm("cvt.rn.f16.f64 %0, %1;" : "=h"(r) : "d"(v));
  return __ushort_as_half(r);
}

__device__ __forceinline__ int nibble_shift(int i) { return (i & 1) ? 16 + 4 * (i >> 1) : 4 * (i >> 1); }

// One CTA = one packed block (16 output channels x 128 input channels);
// warp r quantizes row 16*nb + r, lane l owns k = 4l .. 4l+3 of the block, and
// the G/4 lanes of one group (G = 128, 64 or 32) reduce its min and max.
__global__ void __launch_bounds__(512) pack_kernel(const __half* __restrict__ w, int64_t K, int64_t N, int G,
                                                   uint32_t* __restrict__ qweight, __half* __restrict__ scales,
                                                   uint8_t* __restrict__ zeros, uint32_t* status) {
  __shared__ uint8_t zbuf[kRowsPerBlock][kKPerBlock / 32];
  const int64_t nb = blockIdx.x;
  const int kb = blockIdx.y;
  const int r = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t KB = K / kKPerBlock;
  const int64_t n = nb * kRowsPerBlock + r;
  const int gpk = kKPerBlock / G;        // groups per block
  const int lanes = G / 4;               // lanes per group
  const int gk = lane / lanes;           // this lane's group in the block

  uint2 raw = make_uint2(0, 0);
  if (AWQ_CHECK(in_range(n * K + (int64_t)kb * kKPerBlock + 4 * lane, 4, K * N), status))
    raw = *reinterpret_cast<const uint2*>(w + n * K + (int64_t)kb * kKPerBlock + 4 * lane);
  const __half2 h01 = *reinterpret_cast<const __half2*>(&raw.x);
  const __half2 h23 = *reinterpret_cast<const __half2*>(&raw.y);
  float f[4] = {__low2float(h01), __high2float(h01), __low2float(h23), __high2float(h23)};

  bool finite = true;
  float lo = f[0], hi = f[0];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    finite &= isfinite(f[j]);
    lo = fminf(lo, f[j]);
    hi = fmaxf(hi, f[j]);
  }
  for (int off = lanes / 2; off > 0; off >>= 1) {  // fp16 values are exact in fp32
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
  }
  const uint32_t finite_lanes = __ballot_sync(0xffffffffu, finite);
  const uint32_t group_lanes = (lanes == 32 ? 0xffffffffu : ((1u << lanes) - 1u)) << (gk * lanes);
  const bool group_finite = (finite_lanes & group_lanes) == group_lanes;

  uint32_t part = 0;
  uint8_t zq = 0;
  __half s16 = __ushort_as_half(0);
  if (group_finite) {
    double R = (double)hi - (double)lo;  // exact: difference of two fp16 values
    if (R < 1e-5) R = 1e-5;
    s16 = f64_to_f16_rn(R / 15.0);
    const double sd = (double)__half2float(s16);
    double z = rint(-(double)lo / sd);
    z = fmin(fmax(z, 0.0), 15.0);
    zq = (uint8_t)z;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      double q = rint((double)f[j] / sd) + z;
      q = fmin(fmax(q, 0.0), 15.0);
      const int i = 4 * (lane & 1) + j;  // position of this k inside its 8-k word
      part |= (uint32_t)q << nibble_shift(i);
    }
  } else if (lane % lanes == 0) {
    record_status(status, AWQ_ERR_NONFINITE);
  }
  // lanes 2m, 2m+1 hold inputs 8m .. 8m+7, the word word_of_k(8m) of the row
  const uint32_t word = part | __shfl_xor_sync(0xffffffffu, part, 1);
  if ((lane & 1) == 0) {
    const int64_t wi = (block_index(nb, kb, KB, N / kRowsPerBlock) * kRowsPerBlock + r) * kWordsPerRow +
                       word_of_k(4 * lane, G);
    if (AWQ_CHECK(in_range(wi, 1, K * N / 8), status)) qweight[wi] = word;
  }
  if (lane % lanes == 0) {
    if (AWQ_CHECK(in_range(((int64_t)kb * gpk + gk) * N + n, 1, K / G * N), status))
      scales[((int64_t)kb * gpk + gk) * N + n] = s16;
    zbuf[r][gk] = zq;
  }
  __syncthreads();
  if (threadIdx.x < gpk * (kRowsPerBlock / 2)) {
    const int g = threadIdx.x / (kRowsPerBlock / 2), j = threadIdx.x % (kRowsPerBlock / 2);
    const int64_t zi = ((int64_t)kb * gpk + g) * (N / 2) + nb * (kRowsPerBlock / 2) + j;
    if (AWQ_CHECK(in_range(zi, 1, K / G * (N / 2)), status))
      zeros[zi] = (uint8_t)(zbuf[2 * j][g] | (zbuf[2 * j + 1][g] << 4));
  }
}

// One CTA = one packed block; thread t expands word t (row t/16, the 8 inputs
// from word_k0) into eight fp16 weights W^ = fp16_rne((q - z) * s). (q - z) * s
// is exact in fp32 (at most 4 + 11 significant bits), so one rounding to fp16
// remains.
__global__ void __launch_bounds__(256) dequant_kernel(const uint32_t* __restrict__ qweight,
                                                      const __half* __restrict__ scales,
                                                      const uint8_t* __restrict__ zeros, int64_t K, int64_t N, int G,
                                                      __half* __restrict__ w_out) {
  const int64_t nb = blockIdx.x;
  const int kb = blockIdx.y;
  const int t = threadIdx.x;
  const int r = t / kWordsPerRow, wi = t % kWordsPerRow;
  const int64_t KB = K / kKPerBlock;
  const int64_t n = nb * kRowsPerBlock + r;
  const int k0 = word_k0(wi, G);
  const int64_t grow = (int64_t)kb * (kKPerBlock / G) + k0 / G;  // row of the scale / zero tables
  const int64_t widx = block_index(nb, kb, KB, N / kRowsPerBlock) * kWordsPerBlock + t;
  if (!AWQ_CHECK(in_range(widx, 1, K * N / 8) && in_range(grow * N + n, 1, K / G * N) &&
                     in_range(n * K + (int64_t)kb * kKPerBlock + k0, 8, K * N),
                 nullptr))
    return;
  const uint32_t word = qweight[widx];
  const float s = __half2float(scales[grow * N + n]);
  const int z = (zeros[grow * (N / 2) + (n >> 1)] >> (4 * (n & 1))) & 0xF;
  __align__(16) __half out[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int q = (word >> nibble_shift(i)) & 0xF;
    out[i] = __float2half_rn((float)(q - z) * s);
  }
  *reinterpret_cast<uint4*>(w_out + n * K + (int64_t)kb * kKPerBlock + k0) = *reinterpret_cast<uint4*>(out);
}

}  // namespace

cudaError_t launch_pack(const __half* w, int64_t K, int64_t N, int group, uint32_t* qweight, __half* scales,
                        uint8_t* zeros, uint32_t* status, cudaStream_t stream) {
  dim3 grid((unsigned)(N / kRowsPerBlock), (unsigned)(K / kKPerBlock));
  pack_kernel<<<grid, 512, 0, stream>>>(w, K, N, group, qweight, scales, zeros, status);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const uint32_t* qweight, const __half* scales, const uint8_t* zeros, int64_t K,
                           int64_t N, int group, __half* w_out, cudaStream_t stream) {
  dim3 grid((unsigned)(N / kRowsPerBlock), (unsigned)(K / kKPerBlock));
  dequant_kernel<<<grid, 256, 0, stream>>>(qweight, scales, zeros, K, N, group, w_out);
  return cudaGetLastError();
}

}  // namespace awq
