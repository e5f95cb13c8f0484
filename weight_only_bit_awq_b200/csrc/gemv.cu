// Decode-stage W4A16 GEMV (awq_w4a16_gemv), 1 <= M <= 32.
//
// TinyChat README, "Speed Benchmarks": the generation stage runs one token
// (or a few) per step through 4-bit-weight linear layers, so each layer is a
// GEMV whose cost is streaming its packed weights from HBM once.
//
// Work split ("stream-K" over units). A unit is one k-block (128 input
// channels, one quantization group) of one group of 8 row blocks (128 output
// channels): R <= 8 KiB of codes that the packed layout stores contiguously,
// plus their 16R scales and 8R zero bytes. Units are numbered group-major,
// k-block-minor, i.e. in memory order, and every CTA (two per SM, one for
// M > 16) streams an equal contiguous range of them, so the load is balanced
// to one unit.
//
// Inside a CTA:
//   warp 0 (producer) keeps an 8-deep shared-memory ring full: per unit one
//     1-D bulk copy of the codes, cp.async copies of the scales and zeros,
//     and one 256-byte bulk copy per token of x[m][128 kb .. 128 kb + 127];
//     completion is tracked by the stage's mbarrier (transaction bytes plus
//     the cp.async arrivals). The codes of the first eight units are requested
//     before the kernel waits for the previous grid in the stream
//     (programmatic dependent launch): they do not depend on it; x does.
//   warps 1-8 (consumers): warp w owns row block w of every unit, so it
//     accumulates its 16 output channels over the whole k-range in registers
//     with no cross-warp reduction. Per unit a lane reads two 16-byte words of
//     codes (rows g and g+8, k = 32t .. 32t+31), turns them into exact fp16
//     (q - z) with one lop3 per pair plus hsub2 / hfma2 (the exponent trick:
//     (word & 0x000F000F) | 0x64006400 is half2(1024 + q_a, 1024 + q_b)), and
//     feeds mma.sync m16n8k16 (A = 16 rows x 16 k from registers, B = 16 k x 8
//     tokens from shared memory). The MMA sums over k, so any permutation of k
//     applied to A and B alike is allowed: a lane pairs the k it loaded
//     (32t + 8j + 0..3 for MMA 2j, + 4..7 for MMA 2j+1) with the fragment
//     slots it owns. The fp32 result of a unit is sum_k x (q - z) over one
//     group; y += s * that, in fp32, so no weight is rounded.
//
// Output. A warp that saw all k-blocks of its row block writes fp16 y. A row
// block split between CTAs (only the first and the last group of a CTA's
// range) gets each CTA's fp32 partial sums in a workspace slot, written with
// plain stores, so streaming never waits on another CTA; a small fixup
// kernel launched right behind the GEMV (programmatic dependent launch) adds
// the slots in CTA order (deterministic) and writes y.
#include "awq_internal.cuh"
#include "sm100_ptx.cuh"

namespace awq {
namespace {

constexpr int kConsumers = kGroupBlocks;  // one consumer warp per row block of a unit
constexpr int kWarpXsum = 1 + kConsumers;  // per-unit sums of x (M <= 8)
constexpr int kThreads = (2 + kConsumers) * 32;
constexpr int kStages = 8;
constexpr int kUnitQBytes = kGroupBlocks * 1024;
constexpr int kUnitScaleBytes = kGroupBlocks * kRowsPerBlock * 2;  // 256
constexpr int kUnitZeroBytes = kGroupBlocks * kRowsPerBlock / 2;   // 64
constexpr int kXRowBytes = kKPerBlock * 2;                          // 256

template <int NT>
struct Layout {
  static constexpr int kQOff = 0;
  static constexpr int kSOff = kQOff + kUnitQBytes;
  static constexpr int kZOff = kSOff + kUnitScaleBytes;
  static constexpr int kXSOff = kZOff + kUnitZeroBytes;  // per token: C = 1024 X_lo + 64 X_hi, X = X_lo + X_hi
  static constexpr int kXOff = kXSOff + 8 * 2 * 4;
  static constexpr int kStageBytes = kXOff + 8 * NT * kXRowBytes;
  static constexpr int kBarOff = kStages * kStageBytes;
  static constexpr int kMiscOff = kBarOff + 3 * kStages * 8;  // full, empty, x_landed
  static constexpr int kBytes = kMiscOff + 16;
  static_assert(kStageBytes % 16 == 0, "stages must stay 16-byte aligned");
};

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));  // (a & b) | c
  return d;
}
__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Independent accumulator chains per token tile: the 8 MMAs of a unit are
// spread over kChains accumulators so that consecutive MMAs do not wait on
// each other's results.
template <int NT>
struct Chains {
  static constexpr int value = NT == 1 ? 4 : 2;
};

// acc[c][nt] += (q - z) * x over one unit's 128 k (split over the chains c),
// rows g and g+8.
template <int NT>
__device__ __forceinline__ void block_mma(float (&acc)[Chains<NT>::value][NT][4], const uint4& wa4, const uint4& wb4,
                                          uint32_t za, uint32_t zb, const uint4 (&xf)[NT][4]) {
  constexpr int C = Chains<NT>::value;
  const uint32_t kMaskLo = 0x000F000Fu, kMaskHi = 0x00F000F0u, kMagic = 0x64006400u;
  // Constants built from bit patterns (integer ops only, no conversions):
  // fp16 1024 + z is 0x6400 + z, and -(64 + z) is 0xD400 + 16 z (z <= 15).
  const __half2 zlo_a = u32_as_h2((0x6400u + za) * 0x00010001u);
  const __half2 zlo_b = u32_as_h2((0x6400u + zb) * 0x00010001u);
  const __half2 zhi_a = u32_as_h2((0xD400u + (za << 4)) * 0x00010001u);
  const __half2 zhi_b = u32_as_h2((0xD400u + (zb << 4)) * 0x00010001u);
  const __half2 sixteenth = u32_as_h2(0x2C002C00u);  // 1/16
  const uint32_t wa[4] = {wa4.x, wa4.y, wa4.z, wa4.w};
  const uint32_t wb[4] = {wb4.x, wb4.y, wb4.z, wb4.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t a = wa[j], b = wb[j];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const uint32_t a0 = h2_as_u32(__hsub2(u32_as_h2(lop3_and_or(a, kMaskLo, kMagic)), zlo_a));
      const uint32_t a1 = h2_as_u32(__hsub2(u32_as_h2(lop3_and_or(b, kMaskLo, kMagic)), zlo_b));
      const uint32_t a2 = h2_as_u32(__hfma2(u32_as_h2(lop3_and_or(a, kMaskHi, kMagic)), sixteenth, zhi_a));
      const uint32_t a3 = h2_as_u32(__hfma2(u32_as_h2(lop3_and_or(b, kMaskHi, kMagic)), sixteenth, zhi_b));
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint32_t b0 = half ? xf[nt][j].z : xf[nt][j].x;
        const uint32_t b1 = half ? xf[nt][j].w : xf[nt][j].y;
        mma_16816(acc[(2 * j + half) % C][nt], a0, a1, a2, a3, b0, b1);
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
  return __uint_as_float((h & 0x7FFFu) << 13) * 5.192296858534828e+33f;  // 2^112
}

// M <= 8 (one token tile): the codes go into the MMA unchanged, as the fp16
// values 1024 + q (pairs taken with the 0x000F000F mask, "lo" k) and
// 1024 + 16 q (0x00F000F0 mask, "hi" k), in separate MMAs so that the two
// offsets can be removed afterwards with per-unit sums of x:
//   sum_k x (q - z) = acc_lo + acc_hi / 16 - (1024 X_lo + 64 X_hi) - z (X_lo + X_hi)
// with X_lo, X_hi the sums of x over the lo and hi k of the unit. This needs
// 5 integer ops per 8 weights and no fp16 arithmetic. acc[0..1] are lo chains,
// acc[2..3] hi chains.
__device__ __forceinline__ void block_mma_lohi(float (&acc)[4][4], const uint4& wa4, const uint4& wb4,
                                               const uint4 (&xf)[4]) {
  const uint32_t kMaskLo = 0x000F000Fu, kMaskHi = 0x00F000F0u, kMagic = 0x64006400u;
  const uint32_t wa[4] = {wa4.x, wa4.y, wa4.z, wa4.w};
  const uint32_t wb[4] = {wb4.x, wb4.y, wb4.z, wb4.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t a = wa[j], b = wb[j], a8 = wa[j] >> 8, b8 = wb[j] >> 8;
    // slots (2t, 2t+1) <- k = 8j + 0, 1 (lo) / 2, 3 (hi); slots (2t+8, 2t+9) <- 4, 5 / 6, 7
    mma_16816(acc[j & 1], lop3_and_or(a, kMaskLo, kMagic), lop3_and_or(b, kMaskLo, kMagic),
              lop3_and_or(a8, kMaskLo, kMagic), lop3_and_or(b8, kMaskLo, kMagic), xf[j].x, xf[j].z);
    mma_16816(acc[2 + (j & 1)], lop3_and_or(a, kMaskHi, kMagic), lop3_and_or(b, kMaskHi, kMagic),
              lop3_and_or(a8, kMaskHi, kMagic), lop3_and_or(b8, kMaskHi, kMagic), xf[j].y, xf[j].w);
  }
}

struct Range {
  int64_t KB, NB, U, P;
  __device__ __forceinline__ int64_t first_unit(int64_t c) const { return c * U / P; }
  __device__ __forceinline__ int64_t cta_of(int64_t u) const { return ((u + 1) * P - 1) / U; }
};

template <int NT>
__global__ void __launch_bounds__(kThreads, NT == 4 ? 1 : 2)
    gemv_kernel(const __half* __restrict__ x, const uint32_t* __restrict__ qweight, const __half* __restrict__ scales,
                const uint8_t* __restrict__ zeros, __half* __restrict__ y, int M, int K, int N,
                float* __restrict__ partial, uint32_t* status) {
  using L = Layout<NT>;
  extern __shared__ __align__(16) uint8_t smem[];
  const uint32_t sbase = ptx::smem_u32(smem);
  auto full = [&](int s) -> uint32_t { return sbase + L::kBarOff + 8 * s; };
  auto empty = [&](int s) -> uint32_t { return sbase + L::kBarOff + 8 * (kStages + s); };
  auto xland = [&](int s) -> uint32_t { return sbase + L::kBarOff + 8 * (2 * kStages + s); };
  constexpr bool kLoHi = NT == 1;
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + L::kMiscOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Range rg;
  rg.KB = K / kKPerBlock;
  rg.NB = N / kRowsPerBlock;
  rg.U = (rg.NB + kGroupBlocks - 1) / kGroupBlocks * rg.KB;
  rg.P = gridDim.x;
  const int64_t c = blockIdx.x;
  const int64_t u0 = rg.first_unit(c), u1 = rg.first_unit(c + 1);
  const int n_units = (int)(u1 - u0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      // 32 cp.async arrivals + 1 arrival carrying the byte count (+ 1 from the x-sum warp)
      ptx::mbar_init(full(s), kLoHi ? 34 : 33);
      ptx::mbar_init(empty(s), kConsumers);
      ptx::mbar_init(xland(s), 1);
    }
    *abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  __syncthreads();
  ptx::griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    // Two cursors walk the CTA's units in order: one for the codes (group,
    // k-block), one for the activations (k-block only).
    int64_t cgi = u0 / rg.KB, ckb = u0 % rg.KB, xkb = u0 % rg.KB;
    auto issue_codes = [&](int i) {  // codes, scales, zeros of unit u0 + i; arms the stage
      const int s = i % kStages;
      const int R = (int)group_rows(cgi, rg.NB);
      const uint32_t st = sbase + s * L::kStageBytes;
      if (lane == 0) ptx::mbar_arrive_expect_tx(full(s), (uint32_t)(R * 1024 + (kLoHi ? 0 : M * kXRowBytes)));
      __syncwarp();
      if (lane == 0)
        ptx::bulk_g2s(st + L::kQOff, qweight + unit_first_block(cgi, ckb, rg.KB, rg.NB) * kWordsPerBlock,
                      (uint32_t)(R * 1024), full(s));
      if (lane < 2 * R)
        ptx::cp_async_16(st + L::kSOff + 16 * lane, scales + ckb * N + kGroupBlocks * kRowsPerBlock * cgi + 8 * lane);
      else if (lane >= 16 && lane < 16 + R)
        ptx::cp_async_8(st + L::kZOff + 8 * (lane - 16), zeros + ckb * (N / 2) + 64 * cgi + 8 * (lane - 16));
      ptx::cp_async_arrive_noinc(full(s));
      if (++ckb == rg.KB) {
        ckb = 0;
        ++cgi;
      }
    };
    auto issue_x = [&](int i) {  // activations of unit u0 + i
      const int s = i % kStages;
      // with the lo/hi split x lands on its own barrier: the x-sum warp reads it first
      const uint32_t xb = kLoHi ? xland(s) : full(s);
      if (kLoHi) {
        if (lane == 0) ptx::mbar_arrive_expect_tx(xb, (uint32_t)(M * kXRowBytes));
        __syncwarp();
      }
      if (lane < M)
        ptx::bulk_g2s(sbase + s * L::kStageBytes + L::kXOff + kXRowBytes * lane,
                      x + (int64_t)lane * K + xkb * kKPerBlock, kXRowBytes, xb);
      if (++xkb == rg.KB) xkb = 0;
    };
    const int pro = n_units < kStages ? n_units : kStages;
    for (int i = 0; i < pro; ++i) issue_codes(i);  // independent of the previous grid
    ptx::griddep_wait();
    for (int i = 0; i < pro; ++i) issue_x(i);
    int i = pro;
    for (; i < n_units; ++i) {
      const int s = i % kStages;
      bool ok = true;
      if (lane == 0) ok = ptx::wait_bar(empty(s), ((i / kStages) & 1) ^ 1, abort_flag, status);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      issue_codes(i);
      issue_x(i);
    }
    if (i < n_units && lane == 0)  // aborting: let the copies already issued land
      for (int j = (i > kStages ? i - kStages : 0); j < i; ++j) ptx::drain_bar(full(j % kStages), (j / kStages) & 1);
    __syncwarp();
    return;
  }

  if (warp == kWarpXsum) {
    // ------------------------------ x sums (M <= 8) ------------------------------
    // Lane (m, t4) = (lane / 4, lane % 4) adds token m's x over k = 32 t4 .. 32 t4 + 31
    // into lo (k % 8 in {0, 1, 4, 5}) and hi (k % 8 in {2, 3, 6, 7}) fp32 sums.
    if (kLoHi) {
      const int m = lane >> 2, t4 = lane & 3;
      for (int i = 0; i < n_units; ++i) {
        const int s = i % kStages;
        if (!ptx::wait_bar(xland(s), (i / kStages) & 1, abort_flag, status)) break;
        const uint8_t* st = smem + s * L::kStageBytes;
        float lo = 0.f, hi = 0.f;
        if (m < M) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 v = *reinterpret_cast<const uint4*>(st + L::kXOff + m * kXRowBytes + 64 * t4 + 16 * j);
            const float2 p0 = __half22float2(u32_as_h2(v.x)), p1 = __half22float2(u32_as_h2(v.y));
            const float2 p2 = __half22float2(u32_as_h2(v.z)), p3 = __half22float2(u32_as_h2(v.w));
            lo += (p0.x + p0.y) + (p2.x + p2.y);
            hi += (p1.x + p1.y) + (p3.x + p3.y);
          }
        }
        lo += __shfl_xor_sync(0xffffffffu, lo, 1);
        hi += __shfl_xor_sync(0xffffffffu, hi, 1);
        lo += __shfl_xor_sync(0xffffffffu, lo, 2);
        hi += __shfl_xor_sync(0xffffffffu, hi, 2);
        if (t4 == 0 && m < M) {
          float* xs = reinterpret_cast<float*>(smem + s * L::kStageBytes + L::kXSOff);
          xs[2 * m] = 1024.f * lo + 64.f * hi;
          xs[2 * m + 1] = lo + hi;
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(full(s));
      }
    }
    return;
  }

  // ------------------------------ consumers ------------------------------
  const int cw = warp - 1;  // row block within each unit
  const int g = lane >> 2, t = lane & 3;
  float yacc[NT][4];
  int64_t cur_gi = -1;

  // ---- output of one row block ----
  auto covered = [&](int64_t g_) { return u0 <= g_ * rg.KB && (g_ + 1) * rg.KB <= u1; };
  auto write_y = [&](int64_t g_, const float (&v)[NT][4]) {
    if (cw >= group_rows(g_, rg.NB)) return;
    const int64_t ra = (g_ * kGroupBlocks + cw) * kRowsPerBlock + g;  // rows ra (c = 0, 1), ra + 8 (c = 2, 3)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const int m = 8 * nt + 2 * t + (cc & 1);
        if (m < M) y[(int64_t)m * N + ra + 8 * (cc >> 1)] = __float2half_rn(v[nt][cc]);
      }
  };
  // Partial slot of CTA `cta` for group g_: [cta][first/last group of cta][row block][16 rows][M].
  auto slot = [&](int64_t cta, int64_t g_) -> float* {
    const int which = (g_ == rg.first_unit(cta) / rg.KB) ? 0 : 1;
    return partial + ((cta * 2 + which) * kGroupBlocks + cw) * kRowsPerBlock * M;
  };
  auto store_partial = [&](int64_t g_, const float (&v)[NT][4]) {
    float* mine = slot(c, g_);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const int m = 8 * nt + 2 * t + (cc & 1);
        if (m < M) mine[(g + 8 * (cc >> 1)) * M + m] = v[nt][cc];
      }
  };
  // Output of a finished group: fp16 y if this CTA saw all of its k-blocks,
  // else this CTA's fp32 partial sums, which the fixup kernel adds up.
  auto finish_group = [&](int64_t g_, const float (&v)[NT][4]) {
    if (cw >= group_rows(g_, rg.NB)) return;
    if (covered(g_))
      write_y(g_, v);
    else
      store_partial(g_, v);
  };

  bool ok = true;
  int64_t gi = u0 / rg.KB, kb = u0 % rg.KB;  // unit u0 + i is (gi, kb)
  for (int i = 0; i < n_units; ++i, ++kb) {
    const int s = i % kStages;
    if (kb == rg.KB) {
      kb = 0;
      ++gi;
    }
    if (gi != cur_gi) {
      if (cur_gi >= 0) finish_group(cur_gi, yacc);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) yacc[nt][cc] = 0.f;
      cur_gi = gi;
    }
    if (!ptx::wait_bar(full(s), (i / kStages) & 1, abort_flag, status)) {
      ok = false;
      break;
    }
    if (cw < group_rows(gi, rg.NB)) {
      const uint8_t* st = smem + s * L::kStageBytes;
      const uint8_t* blk = st + L::kQOff + cw * 1024;
      const uint4 wa = *reinterpret_cast<const uint4*>(blk + g * 64 + 16 * t);
      const uint4 wb = *reinterpret_cast<const uint4*>(blk + (g + 8) * 64 + 16 * t);
      const uint16_t* sc = reinterpret_cast<const uint16_t*>(st + L::kSOff) + cw * kRowsPerBlock;
      const float sa = pos_half_bits_to_float(sc[g]), sb = pos_half_bits_to_float(sc[g + 8]);
      const uint8_t* zr = st + L::kZOff + cw * (kRowsPerBlock / 2);
      const uint32_t za = (zr[g >> 1] >> (4 * (g & 1))) & 0xF;
      const uint32_t zb = (zr[(g + 8) >> 1] >> (4 * (g & 1))) & 0xF;
      uint4 xf[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int m = 8 * nt + g;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          xf[nt][j] = m < M ? *reinterpret_cast<const uint4*>(st + L::kXOff + m * kXRowBytes + 64 * t + 16 * j)
                            : make_uint4(0, 0, 0, 0);
      }
      if constexpr (kLoHi) {
        float acc[4][4];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) acc[ch][cc] = 0.f;
        block_mma_lohi(acc, wa, wb, xf[0]);
        // C and X of tokens 2t and 2t + 1
        const float4 cx = *reinterpret_cast<const float4*>(st + L::kXSOff + 16 * t);
        const float zfa = __uint_as_float(0x4B000000u | za) - 8388608.f;  // exact (float)z
        const float zfb = __uint_as_float(0x4B000000u | zb) - 8388608.f;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const float lo = acc[0][cc] + acc[1][cc], hi = acc[2][cc] + acc[3][cc];
          const float Cm = (cc & 1) ? cx.z : cx.x, Xm = (cc & 1) ? cx.w : cx.y;
          float v = fmaf(hi, 0.0625f, lo) - Cm;
          v = fmaf(-(cc < 2 ? zfa : zfb), Xm, v);
          yacc[0][cc] = fmaf(cc < 2 ? sa : sb, v, yacc[0][cc]);
        }
      } else {
        constexpr int C = Chains<NT>::value;
        float acc[C][NT][4];
#pragma unroll
        for (int ch = 0; ch < C; ++ch)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) acc[ch][nt][cc] = 0.f;
        block_mma<NT>(acc, wa, wb, za, zb, xf);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            float v = acc[0][nt][cc];
#pragma unroll
            for (int ch = 1; ch < C; ++ch) v += acc[ch][nt][cc];
            yacc[nt][cc] += (cc < 2 ? sa : sb) * v;
          }
      }
    }
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(empty(s));
  }
  if (ok && cur_gi >= 0) finish_group(cur_gi, yacc);
}

// Rows split between CTAs: one CTA per group (128 threads, thread = row),
// launched right after the GEMV in the same stream. It waits for the GEMV's
// writes (programmatic dependent launch), adds the contributors' partial
// slots in CTA order and writes fp16 y. Groups that one CTA covered exit.
__global__ void __launch_bounds__(128) gemv_fixup_kernel(const float* __restrict__ partial, __half* __restrict__ y,
                                                          int M, int K, int N, int P) {
  ptx::griddep_launch_dependents();
  Range rg;
  rg.KB = K / kKPerBlock;
  rg.NB = N / kRowsPerBlock;
  rg.U = (rg.NB + kGroupBlocks - 1) / kGroupBlocks * rg.KB;
  rg.P = P;
  const int64_t gi = blockIdx.x;
  const int64_t c_first = rg.cta_of(gi * rg.KB), c_last = rg.cta_of((gi + 1) * rg.KB - 1);
  if (c_first == c_last) return;
  const int rb = threadIdx.x >> 4, row = threadIdx.x & 15;
  if (rb >= group_rows(gi, rg.NB)) return;
  ptx::griddep_wait();
  for (int m = 0; m < M; ++m) {
    float v = 0.f;
    for (int64_t q0 = c_first; q0 <= c_last; q0 += 8) {
      float part[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int64_t q = q0 + k;
        part[k] = 0.f;
        if (q <= c_last) {
          const int which = (gi == rg.first_unit(q) / rg.KB) ? 0 : 1;
          part[k] = __ldcg(partial + (((q * 2 + which) * kGroupBlocks + rb) * kRowsPerBlock + row) * M + m);
        }
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) v += part[k];
    }
    y[(int64_t)m * N + gi * kGroupBlocks * kRowsPerBlock + threadIdx.x] = __float2half_rn(v);
  }
}

template <int NT>
cudaError_t launch_t(const __half* x, const uint32_t* qweight, const __half* scales, const uint8_t* zeros, __half* y,
                     int M, int K, int N, void* workspace, const GemvPlan& p, cudaStream_t stream) {
  using L = Layout<NT>;
  static uint64_t attr_set = 0;  // one bit per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return cudaErrorInvalidDevice;
  if (!(attr_set >> dev & 1)) {
    cudaError_t e = cudaFuncSetAttribute(gemv_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
    if (e != cudaSuccess) return e;
    attr_set |= uint64_t(1) << dev;
  }
  char* ws = static_cast<char*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  float* partial = reinterpret_cast<float*>(ws + p.partial_off);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.ctas);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L::kBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, gemv_kernel<NT>, x, qweight, scales, zeros, y, M, K, N, partial, status);
  if (e != cudaSuccess || !p.has_split) return e;
  cudaLaunchConfig_t fcfg = cfg;
  fcfg.gridDim = dim3((unsigned)p.groups);
  fcfg.blockDim = dim3(kGroupBlocks * kRowsPerBlock);
  fcfg.dynamicSmemBytes = 0;
  return cudaLaunchKernelEx(&fcfg, gemv_fixup_kernel, (const float*)partial, y, M, K, N, p.ctas);
}

}  // namespace

GemvPlan plan_gemv(int64_t M, int64_t K, int64_t N, int sm_count) {
  GemvPlan p{};
  p.nt = M <= 8 ? 1 : (M <= 16 ? 2 : 4);
  const int64_t NB = N / kRowsPerBlock, KB = K / kKPerBlock;
  const int64_t U = (NB + kGroupBlocks - 1) / kGroupBlocks * KB;
  const int64_t per_sm = p.nt == 4 ? 1 : 2;  // resident CTAs per SM (shared memory and registers)
  p.ctas = (int)(U < per_sm * sm_count ? U : per_sm * sm_count);
  p.groups = (int)((NB + kGroupBlocks - 1) / kGroupBlocks);
  p.has_split = false;  // does some CTA boundary fall inside a group?
  for (int64_t cc = 1; cc < p.ctas && !p.has_split; ++cc) p.has_split = (cc * U / p.ctas) % KB != 0;
  p.partial_off = kWsHeaderBytes;
  p.zero_bytes = kWsHeaderBytes;  // the status word starts at zero
  p.ws_bytes = p.partial_off + (size_t)p.ctas * 2 * kGroupBlocks * kRowsPerBlock * (size_t)M * 4;
  return p;
}

cudaError_t launch_gemv(const __half* x, const uint32_t* qweight, const __half* scales, const uint8_t* zeros,
                        __half* y, int64_t M, int64_t K, int64_t N, void* workspace, const GemvPlan& p,
                        cudaStream_t stream) {
  const int m = (int)M, k = (int)K, n = (int)N;
  switch (p.nt) {
    case 1: return launch_t<1>(x, qweight, scales, zeros, y, m, k, n, workspace, p, stream);
    case 2: return launch_t<2>(x, qweight, scales, zeros, y, m, k, n, workspace, p, stream);
    case 4: return launch_t<4>(x, qweight, scales, zeros, y, m, k, n, workspace, p, stream);
    default: return cudaErrorInvalidConfiguration;
  }
}

}  // namespace awq
