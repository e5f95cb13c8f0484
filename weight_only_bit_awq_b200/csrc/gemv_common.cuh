// Device helpers of the decode GEMV (gemv.cu): the shared-memory sizes of one
// k-block, the nibble-to-fp16 and integer MMA building blocks, and the
// per-k-block MMA sequences of the fp16 paths.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "awq_internal.cuh"

namespace awq {
namespace {
constexpr int kMaxStages = 16;
constexpr int kKbQBytes = kGroupBlocks * 1024;                    // codes of one k-block of a group
constexpr int kKbScaleBytes = kGroupBlocks * kRowsPerBlock * 2;   // 256: one row of scales (one group)
constexpr int kKbZeroBytes = kGroupBlocks * kRowsPerBlock / 2;    // 64: one row of zero points
constexpr int kKbXsBytes = 8 * 2 * 4;                             // 8 tokens x (C, X) fp32, per group
constexpr int kXRowBytes = kKPerBlock * 2;                        // 256 bytes of x per token and k-block

// Integer path (M <= 2, groups of 128): per k-block, the x-prep warp writes
// the B fragments of the integer MMAs -- for each lane column t (0..3), 4 M
// digit columns of 32 bytes, plus one 32-byte pad per t so that its stores are
// bank-conflict free -- and one float4 of coefficients per t.
__host__ __device__ constexpr int int_bfrag_tstride(int M) { return (4 * M + 1) * 32; }
__host__ __device__ constexpr int int_xs_bytes(int M) { return 4 * int_bfrag_tstride(M) + 64; }

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));  // (a & b) | c
  return d;
}
__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// d += A B (m16n8k16, fp16 inputs, fp32 accumulate).
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// d = A B (the accumulator input is zero; no separate clearing of d).
__device__ __forceinline__ void mma_16816_first(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
}

// d += A B (m16n8k32, A unsigned bytes, B signed bytes, exact s32 accumulate);
// the _first form starts from zero.
__device__ __forceinline__ void imma_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void imma_16832_first(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                 uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}

// Group size GS (128, 64 or 32) in the k-block of 128: the packed layout puts
// the inputs of group j / J (J = GS / 32) into word 4t + j of every lane t, so
// the MMAs of step j (one word per lane) see a single group. kGroupsPerKb
// groups per k-block, each with its own scale and zero point.
template <int GS>
struct Grp {
  static constexpr int J = GS / 32;              // MMA steps j per group
  static constexpr int kPerKb = kKPerBlock / GS;  // groups per k-block
  // byte offset, in a token's 128 x values of the k-block, of the 8 inputs in word 4t + j
  __host__ __device__ static constexpr int x_off(int t, int j) { return 2 * word_k0(4 * t + j, GS); }
};

// Accumulators per token tile (M > 8): for GS = 128 the 8 MMAs of a k-block
// are spread over two chains so that consecutive MMAs do not wait on each
// other; for smaller groups there is one accumulator per group.
template <int NT, int GS>
struct Chains {
  static constexpr int value = GS == 128 ? 2 : Grp<GS>::kPerKb;
};

// acc[c][nt] = (q - z) * x over one k-block, rows g and g+8 (M > 8); za, zb
// are the zero points of the rows per group of the k-block.
template <int NT, int GS>
__device__ __forceinline__ void block_mma(float (&acc)[Chains<NT, GS>::value][NT][4], const uint4& wa4,
                                          const uint4& wb4, const uint32_t (&za)[Grp<GS>::kPerKb],
                                          const uint32_t (&zb)[Grp<GS>::kPerKb], const uint4 (&xf)[NT][4]) {
  constexpr int C = Chains<NT, GS>::value, J = Grp<GS>::J;
  const uint32_t kMaskLo = 0x000F000Fu, kMaskHi = 0x00F000F0u, kMagic = 0x64006400u;
  const __half2 sixteenth = u32_as_h2(0x2C002C00u);  // 1/16
  const uint32_t wa[4] = {wa4.x, wa4.y, wa4.z, wa4.w};
  const uint32_t wb[4] = {wb4.x, wb4.y, wb4.z, wb4.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    // Constants built from bit patterns (integer ops only, no conversions):
    // fp16 1024 + z is 0x6400 + z, and -(64 + z) is 0xD400 + 16 z (z <= 15).
    const int gk = j / J;
    const __half2 zlo_a = u32_as_h2((0x6400u + za[gk]) * 0x00010001u);
    const __half2 zlo_b = u32_as_h2((0x6400u + zb[gk]) * 0x00010001u);
    const __half2 zhi_a = u32_as_h2((0xD400u + (za[gk] << 4)) * 0x00010001u);
    const __half2 zhi_b = u32_as_h2((0xD400u + (zb[gk] << 4)) * 0x00010001u);
    uint32_t a = wa[j], b = wb[j];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const uint32_t a0 = h2_as_u32(__hsub2(u32_as_h2(lop3_and_or(a, kMaskLo, kMagic)), zlo_a));
      const uint32_t a1 = h2_as_u32(__hsub2(u32_as_h2(lop3_and_or(b, kMaskLo, kMagic)), zlo_b));
      const uint32_t a2 = h2_as_u32(__hfma2(u32_as_h2(lop3_and_or(a, kMaskHi, kMagic)), sixteenth, zhi_a));
      const uint32_t a3 = h2_as_u32(__hfma2(u32_as_h2(lop3_and_or(b, kMaskHi, kMagic)), sixteenth, zhi_b));
      const int step = 2 * j + half;
      const int idx = GS == 128 ? step % C : gk;
      const bool first = GS == 128 ? step < C : (j % J == 0 && half == 0);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint32_t b0 = half ? xf[nt][j].z : xf[nt][j].x;
        const uint32_t b1 = half ? xf[nt][j].w : xf[nt][j].y;
        if (first)
          mma_16816_first(acc[idx][nt], a0, a1, a2, a3, b0, b1);
        else
          mma_16816(acc[idx][nt], a0, a1, a2, a3, b0, b1);
      }
      a >>= 8;
      b >>= 8;
    }
  }
}

// fp16 bits -> fp32 value of a non-negative fp16 (scales), exact for normal and
// subnormal inputs: the 15 value bits shifted into place read as fp32 are the
// value times 2^-112.
__device__ __forceinline__ float pos_half_bits_to_float(uint32_t h) {
  return __uint_as_float(h << 13) * 5.192296858534828e+33f;  // 2^112; the sign bit of h is 0
}

// M <= 8 (one token tile): the codes go into the MMA unchanged. One lop3
// turns the nibbles at bits 0-3 of each half of a word ("lo" k) into the fp16
// values 1024 + q (0x000F000F mask over 0x6400 = 1024, whose ulp is 1), and
// the nibbles at bits 4-7 ("hi" k) into 64 + q (0x00F000F0 mask over 0x5400 =
// 64, whose ulp is 1/16, so mantissa 16 q adds q). Both kinds accumulate in
// the same fp32 registers, and the offsets come off afterwards with per-group
// sums of x:
//   sum_k x (q - z) = acc - (1024 X_lo + 64 X_hi) - z (X_lo + X_hi)
// with X_lo, X_hi the sums of x over the lo and hi k of the group. This needs
// 5 integer ops per 8 weights and no fp16 arithmetic. LoHi<GS>::kAcc
// accumulators: for GS = 128 two chains (alternate MMA steps), else one per
// group.
template <int GS>
struct LoHi {
  static constexpr int kAcc = GS == 128 ? 2 : Grp<GS>::kPerKb;
};
template <int GS>
__device__ __forceinline__ void block_mma_lohi(float (&acc)[LoHi<GS>::kAcc][4], const uint4& wa4, const uint4& wb4,
                                               const uint4 (&xf)[4]) {
  constexpr int J = Grp<GS>::J;
  const uint32_t kMaskLo = 0x000F000Fu, kMaskHi = 0x00F000F0u, kMagicLo = 0x64006400u, kMagicHi = 0x54005400u;
  const uint32_t wa[4] = {wa4.x, wa4.y, wa4.z, wa4.w};
  const uint32_t wb[4] = {wb4.x, wb4.y, wb4.z, wb4.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t a = wa[j], b = wb[j], a8 = wa[j] >> 8, b8 = wb[j] >> 8;
    // slots (2t, 2t+1) <- k0 + 0, 1 (lo) / 2, 3 (hi); slots (2t+8, 2t+9) <- k0 + 4, 5 / 6, 7
    const uint32_t l0 = lop3_and_or(a, kMaskLo, kMagicLo), l1 = lop3_and_or(b, kMaskLo, kMagicLo);
    const uint32_t l2 = lop3_and_or(a8, kMaskLo, kMagicLo), l3 = lop3_and_or(b8, kMaskLo, kMagicLo);
    const uint32_t h0 = lop3_and_or(a, kMaskHi, kMagicHi), h1 = lop3_and_or(b, kMaskHi, kMagicHi);
    const uint32_t h2 = lop3_and_or(a8, kMaskHi, kMagicHi), h3 = lop3_and_or(b8, kMaskHi, kMagicHi);
    const int idx = GS == 128 ? (j & 1) : j / J;
    if (GS == 128 ? j < 2 : j % J == 0)
      mma_16816_first(acc[idx], l0, l1, l2, l3, xf[j].x, xf[j].z);
    else
      mma_16816(acc[idx], l0, l1, l2, l3, xf[j].x, xf[j].z);
    mma_16816(acc[idx], h0, h1, h2, h3, xf[j].y, xf[j].w);
  }
}

}  // namespace
}  // namespace awq
