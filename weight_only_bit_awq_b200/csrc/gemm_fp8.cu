// W4A8-FP8 variant of the prefill GEMM: awq_fp8_row_exponents,
// awq_fp8_quantize_x, awq_dequant_fp8 and awq_w4a8_gemm.
//
// The TensorRT-LLM news item on INT4 AWQ on one H200 says its AWQ kernels
// compute in FP8 on the tensor cores. The pages give no recipe; the reading
// implemented here keeps the 4-bit weights and their fp16 group scales as
// awq_pack stores them and moves both operands of the MMA to E4M3:
//   - per token m: sx[m] = fp32(amax_k |x[m,k]|) / 448 and
//     x8[m,k] = e4m3(x[m,k] / sx[m]) (IEEE fp32 divisions, round to nearest
//     even, saturating at 448, the largest finite E4M3 value);
//   - per output channel n: e[n], the largest integer with
//     15 * max_g s[n,g] * 2^e <= 448, computed once per weight;
//   - W8[n,k] = e4m3(fp16((q - z) * fp16(s * 2^e[n]))), formed in shared
//     memory just ahead of the MMA (tcgen05.mma kind::f8f6f4, fp32
//     accumulation in tensor memory over all of K);
//   - y[m,n] = fp16(acc * sx[m] * 2^-e[n]).
// With the per-row power of two every nonzero |W8| lies in [448/30, 448]: all
// E4M3 normal numbers, so each weight keeps 4 significant bits.
//
// The GEMM has the structure of the fp16 one (gemm_tc.cu): persistent, one
// CTA per SM over 128-channel x BN-token tiles with two tensor-memory
// accumulators; warp 0 loads x8 by TMA (one 128-byte-wide box per 128-input
// k-block, 128-byte swizzle), warp 1 issues 4 MMAs of K = 32 per k-block,
// warp 2 copies the packed codes and the tile's scale and zero rows, warps
// 3-10 dequantize (two threads per weight row, half of its codes each: two
// warps per SM sub-partition hide the conversion latency) and warps 11-14 run
// the epilogue of one tile while the next is accumulated. Every
// mbarrier wait is bounded; on expiry AWQ_ERR_TIMEOUT goes to the status word
// and the CTA drains and exits.
#include <atomic>
#include <cuda_fp8.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "awq_internal.cuh"
#include "sm100_ptx.cuh"

namespace awq {
namespace {

// ---------------------------------------------------------------------------
// row exponents
// ---------------------------------------------------------------------------

// e for a largest scale given by its fp16 bit pattern (positive): with the
// scale S = Mi * 2^k exactly (Mi an integer below 2048), the largest j with
// 15 Mi 2^j <= 448, minus k.
__device__ __forceinline__ int row_exponent(uint32_t sbits) {
  const uint32_t E = (sbits >> 10) & 31, F = sbits & 1023;
  const int Mi = E ? (int)(1024 + F) : (int)F;
  const int k = E ? (int)E - 25 : -24;
  if (Mi == 0) return 0;
  const int t = 15 * Mi;  // 15 .. 30705
  int j = 0;
  if (t <= 448) {
    while ((t << (j + 1)) <= 448) ++j;
  } else {
    while (t > (448 << -j)) --j;
  }
  return j - k;
}

__global__ void __launch_bounds__(256) fp8_row_exp_kernel(const __half* __restrict__ scales, int64_t N, int64_t KG,
                                                          int8_t* __restrict__ e_out) {
  const int64_t n = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  uint32_t smax = 0;  // positive fp16 scales order like their bit patterns
  for (int64_t g = 0; g < KG; ++g) smax = max(smax, (uint32_t)__half_as_ushort(scales[g * N + n]));
  e_out[n] = (int8_t)row_exponent(smax);
}

// ---------------------------------------------------------------------------
// per-token activation quantization: one CTA per token
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t max_mag8(uint4 v) {
  const uint32_t w[4] = {v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu, v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu};
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) m = max(m, max(w[i] & 0xFFFFu, w[i] >> 16));
  return m;
}

// e4m3 codes of two fp32 values (round to nearest even, saturating), a in the
// low byte.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

__global__ void __launch_bounds__(256) fp8_quant_x_kernel(const __half* __restrict__ x, int64_t K,
                                                          uint8_t* __restrict__ x8, float* __restrict__ sx) {
  __shared__ uint32_t wmax[8];
  const int64_t m = blockIdx.x;
  const __half* xr = x + m * K;
  // pass 1: largest |x| (as fp16 magnitude bits: NaN above inf above every finite value)
  uint32_t mb = 0;
  for (int64_t i = (int64_t)threadIdx.x * 8; i < K; i += 256 * 8)
    mb = max(mb, max_mag8(*reinterpret_cast<const uint4*>(xr + i)));
  mb = __reduce_max_sync(0xffffffffu, mb);
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = mb;
  __syncthreads();
  mb = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) mb = max(mb, wmax[w]);
  const float s = __fdiv_rn(__half2float(__ushort_as_half((unsigned short)mb)), 448.0f);
  if (threadIdx.x == 0) sx[m] = s;
  // pass 2: x / s (IEEE fp32 division) -> E4M3
  uint8_t* outr = x8 + m * K;
  for (int64_t i = (int64_t)threadIdx.x * 8; i < K; i += 256 * 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(xr + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t c[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[j]));
      c[j] = s == 0.0f ? 0u : e4m3x2(__fdiv_rn(f.x, s), __fdiv_rn(f.y, s));
    }
    *reinterpret_cast<uint2*>(outr + i) = make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
  }
}

// ---------------------------------------------------------------------------
// W8 from the packed codes (shared by the GEMM and the dequant test surface)
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));  // (a & b) | c
  return d;
}
__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }
__device__ __forceinline__ uint32_t e4m3x2_h(uint32_t h2) {
  __half2_raw r;
  r.x = (unsigned short)(h2 & 0xFFFFu);
  r.y = (unsigned short)(h2 >> 16);
  return (uint32_t)__nv_cvt_halfraw2_to_fp8x2(r, __NV_SATFINITE, __NV_E4M3);  // r.x in the low byte
}

// Eight codes of one word (inputs k0 .. k0+7) -> eight E4M3 bytes of
// fp16((q - z) * s'), in k order. (word & 0x000F000F) | 0x64006400 is
// half2(1024 + q_even, 1024 + q_odd); with the 0x00F000F0 mask, 1024 + 16 q.
// Subtracting 1024 + z (or scaling by 1/16 and subtracting 64 + z) gives the
// exact q - z, so the only roundings are the fp16 product and the E4M3
// conversion.
__device__ __forceinline__ uint2 w8_word(uint32_t w, __half2 zlo, __half2 zhi, __half2 s2) {
  const __half2 sixteenth = __half2half2(__ushort_as_half(0x2C00));  // 1/16
  const uint32_t a = h2u(__hmul2(__hsub2(u2h(lop3_and_or(w, 0x000F000Fu, 0x64006400u)), zlo), s2));
  const uint32_t b = h2u(__hmul2(__hfma2(u2h(lop3_and_or(w, 0x00F000F0u, 0x64006400u)), sixteenth, zhi), s2));
  w >>= 8;
  const uint32_t c = h2u(__hmul2(__hsub2(u2h(lop3_and_or(w, 0x000F000Fu, 0x64006400u)), zlo), s2));
  const uint32_t d = h2u(__hmul2(__hfma2(u2h(lop3_and_or(w, 0x00F000F0u, 0x64006400u)), sixteenth, zhi), s2));
  return make_uint2(e4m3x2_h(a) | (e4m3x2_h(b) << 16), e4m3x2_h(c) | (e4m3x2_h(d) << 16));
}

// fp16 bit patterns of the group constants: s' = fp16(s * 2^e) (exact unless
// below the fp16 normal range), 1024 + z = 0x6400 + z, -(64 + z) = 0xD400 + 16 z.
struct GroupConsts {
  __half2 s2, zlo, zhi;
};
__device__ __forceinline__ GroupConsts group_consts(uint32_t sbits, uint32_t z, float pow2e) {
  GroupConsts c;
  const __half sp = __float2half_rn(__half2float(__ushort_as_half((unsigned short)sbits)) * pow2e);
  c.s2 = __half2half2(sp);
  c.zlo = u2h((0x6400u + z) * 0x00010001u);
  c.zhi = u2h((0xD400u + (z << 4)) * 0x00010001u);
  return c;
}
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }  // |e| < 127

// W8 [N][K] (test surface): one thread per packed word.
__global__ void __launch_bounds__(256) dequant_fp8_kernel(const uint32_t* __restrict__ qweight,
                                                          const __half* __restrict__ scales,
                                                          const uint8_t* __restrict__ zeros,
                                                          const int8_t* __restrict__ row_exp, int64_t K, int64_t N,
                                                          int G, uint8_t* __restrict__ w8_out) {
  const int64_t nb = blockIdx.x;
  const int kb = blockIdx.y;
  const int t = threadIdx.x;
  const int r = t / kWordsPerRow, wi = t % kWordsPerRow;
  const int64_t KB = K / kKPerBlock;
  const int64_t n = nb * kRowsPerBlock + r;
  const int k0 = word_k0(wi, G);
  const int64_t grow = (int64_t)kb * (kKPerBlock / G) + k0 / G;  // row of the scale / zero tables
  const uint32_t word = qweight[block_index(nb, kb, KB, N / kRowsPerBlock) * kWordsPerBlock + t];
  const uint32_t z = (zeros[grow * (N / 2) + (n >> 1)] >> (4 * (n & 1))) & 0xF;
  const GroupConsts gc = group_consts(__half_as_ushort(scales[grow * N + n]), z, pow2f(row_exp[n]));
  *reinterpret_cast<uint2*>(w8_out + n * K + (int64_t)kb * kKPerBlock + k0) = w8_word(word, gc.zlo, gc.zhi, gc.s2);
}

// ---------------------------------------------------------------------------
// the GEMM
// ---------------------------------------------------------------------------

constexpr int kBM = 128;
constexpr int kXStages = 4;
constexpr int kWStages = 3;
constexpr int kQStages = 3;
constexpr int kQBytes = 8 * 1024;
constexpr int kQScaleOff = kQBytes, kQZeroOff = kQScaleOff + 4 * 256;
constexpr int kQStride = kQZeroOff + 4 * 64;
constexpr int kWBytes = kBM * kKPerBlock;  // 16 KiB: 128 rows x 128 E4M3 weights
constexpr int kWarpX = 0, kWarpMma = 1, kWarpQ = 2, kFirstDeqWarp = 3, kNumDeqWarps = 8;
constexpr int kFirstEpiWarp = kFirstDeqWarp + kNumDeqWarps, kNumEpiWarps = 4;
constexpr int kDeqThreads = kNumDeqWarps * 32, kEpiThreads = kNumEpiWarps * 32;
constexpr int kThreads = (kFirstEpiWarp + kNumEpiWarps) * 32;

constexpr int kBarXFull = 0, kBarXEmpty = kBarXFull + kXStages, kBarWFull = kBarXEmpty + kXStages,
              kBarWEmpty = kBarWFull + kWStages, kBarQFull = kBarWEmpty + kWStages,
              kBarQEmpty = kBarQFull + kQStages, kBarAccFull = kBarQEmpty + kQStages, kBarAccEmpty = kBarAccFull + 2,
              kBarDrain = kBarAccEmpty + 2, kNumBars = kBarDrain + 1;

template <int BN>
struct Layout {
  static constexpr int kXBytes = BN * kKPerBlock;  // BN tokens x 128 E4M3 inputs
  static constexpr int kXOff = 0;
  static constexpr int kWOff = kXOff + kXStages * kXBytes;
  static constexpr int kQOff = kWOff + kWStages * kWBytes;
  static constexpr int kBarOff = kQOff + kQStages * kQStride;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1 KiB
};
static_assert(Layout<256>::kAlloc <= 232448, "shared memory budget");

using ptx::drain_bar;
using ptx::wait_bar;

// Persistent: CTA c computes tiles c, c + P, ... (P = gridDim.x; tile t is
// token tile t % MT of channel tile t / MT); the rings run on across tiles and
// the two accumulators let the epilogue warps drain one tile while the MMA
// warp fills the next.
template <int BN, int GS>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_fp8_kernel(const __grid_constant__ CUtensorMap tmap_x, const float* __restrict__ sx,
                    const uint32_t* __restrict__ qweight, const __half* __restrict__ scales,
                    const uint8_t* __restrict__ zeros, const int8_t* __restrict__ row_exp, __half* __restrict__ y,
                    int M, int K, int N, int GM, uint32_t* status) {
  using L = Layout<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + L::kBarOff + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + L::kMiscOff + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = K / kKPerBlock;
  const int MT = (M + BN - 1) / BN, NT = (N + kBM - 1) / kBM, T = MT * NT;
  const int P = gridDim.x;
  const int ntiles = blockIdx.x < T ? (T - 1 - (int)blockIdx.x) / P + 1 : 0;  // tiles of this CTA
  // Tile order: blocks of GM token tiles; within a block, token tile fastest,
  // then channel tile. The x of one block stays in L2 while the block's
  // channel tiles stream past it.
  auto tile_mn = [&](int it, int& mt, int& nt) {
    const int t = (int)blockIdx.x + it * P;
    const int blk = t / (GM * NT), w = t - blk * GM * NT;
    const int gb = min(GM, MT - blk * GM);  // token tiles in this block
    mt = blk * GM + w % gb;
    nt = w / gb;
  };
  auto tile_m0 = [&](int it) {
    int mt, nt;
    tile_mn(it, mt, nt);
    return mt * BN;
  };
  auto tile_nt = [&](int it) {
    int mt, nt;
    tile_mn(it, mt, nt);
    return nt;
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kXStages; ++i) {
      ptx::mbar_init(bar(kBarXFull + i), 1);
      ptx::mbar_init(bar(kBarXEmpty + i), 1);
    }
    for (int i = 0; i < kWStages; ++i) {
      ptx::mbar_init(bar(kBarWFull + i), kDeqThreads);
      ptx::mbar_init(bar(kBarWEmpty + i), 1);
    }
    for (int i = 0; i < kQStages; ++i) {
      ptx::mbar_init(bar(kBarQFull + i), 33);  // the codes' byte count + 32 cp.async arrivals
      ptx::mbar_init(bar(kBarQEmpty + i), kDeqThreads);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar(kBarAccFull + i), 1);
      ptx::mbar_init(bar(kBarAccEmpty + i), kEpiThreads);
    }
    ptx::mbar_init(bar(kBarDrain), 1);
    *abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  if (warp == kWarpX && lane == 0) ptx::prefetch_tensormap(&tmap_x);
  if (warp == kWarpMma) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), 2 * BN);
    ptx::tmem_relinquish();
    ptx::tc_fence_before();
  }
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == kWarpX) {
    // ---------------- x8 producer: one 128-byte-wide box per k-block ----------------
    if (lane == 0) {
      int i = 0;
      bool ok = true;
      for (int it = 0; it < ntiles && ok; ++it) {
        const int m0 = tile_m0(it);
        for (int kb = 0; kb < KB; ++kb, ++i) {
          const int s = i % kXStages;
          if (!(ok = wait_bar(bar(kBarXEmpty + s), ((i / kXStages) & 1) ^ 1, abort_flag, status))) break;
          ptx::mbar_arrive_expect_tx(bar(kBarXFull + s), L::kXBytes);
          ptx::tma_load_2d(sbase + L::kXOff + s * L::kXBytes, &tmap_x, kb * kKPerBlock, m0, bar(kBarXFull + s));
        }
      }
      if (!ok)  // aborting: let the copies already issued land
        for (int j = (i > kXStages ? i - kXStages : 0); j < i; ++j)
          drain_bar(bar(kBarXFull + j % kXStages), (j / kXStages) & 1);
    }
    __syncwarp();
  } else if (warp == kWarpQ) {
    // ---------------- packed-weight producer (as in the fp16 GEMM) ----------------
    constexpr int kGPK = kKPerBlock / GS;
    const int64_t NB = N / kRowsPerBlock;
    int i = 0;
    bool ok = true;
    for (int it = 0; it < ntiles && ok; ++it) {
      const int64_t gi = tile_nt(it);
      const int n0 = (int)gi * kBM;
      const uint32_t qbytes = (uint32_t)(group_rows(gi, NB) * 1024);
      for (int kb = 0; kb < KB; ++kb, ++i) {
        const int s = i % kQStages;
        if (lane == 0) ok = wait_bar(bar(kBarQEmpty + s), ((i / kQStages) & 1) ^ 1, abort_flag, status);
        if (!(ok = __shfl_sync(0xffffffffu, ok, 0))) break;
        const uint32_t st = sbase + L::kQOff + s * kQStride;
        if (lane == 0) ptx::mbar_arrive_expect_tx(bar(kBarQFull + s), qbytes);
        __syncwarp();
        if (lane == 0)
          ptx::bulk_g2s(st, qweight + unit_first_block(gi, kb, KB, NB) * kWordsPerBlock, qbytes, bar(kBarQFull + s));
        for (int p = lane; p < kGPK * 16; p += 32) {  // kGPK rows of 128 scales: 16 B = 8 output channels
          const int g = p >> 4, l = p & 15;
          if (n0 + 8 * l < N)
            ptx::cp_async_16(st + kQScaleOff + 256 * g + 16 * l, scales + ((int64_t)kb * kGPK + g) * N + n0 + 8 * l);
        }
        for (int p = lane; p < kGPK * 8; p += 32) {  // kGPK rows of 64 zero bytes: 8 B = 16 output channels
          const int g = p >> 3, l = p & 7;
          if (n0 + 16 * l < N)
            ptx::cp_async_8(st + kQZeroOff + 64 * g + 8 * l,
                            zeros + ((int64_t)kb * kGPK + g) * (N / 2) + n0 / 2 + 8 * l);
        }
        ptx::cp_async_arrive_noinc(bar(kBarQFull + s));
      }
    }
    if (!ok && lane == 0)
      for (int j = (i > kQStages ? i - kQStages : 0); j < i; ++j)
        drain_bar(bar(kBarQFull + j % kQStages), (j / kQStages) & 1);
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ---------------- MMA issuer: 4 x (128 x BN x 32) per k-block ----------------
    if (lane == 0) {
      const uint32_t idesc = ptx::idesc_e4m3_f32(kBM, BN);
      bool ok = true;
      int i = 0;  // k-blocks so far (W and x stage uses)
      for (int it = 0; it < ntiles && ok; ++it) {
        const int acc = it & 1;
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        if (!(ok = wait_bar(bar(kBarAccEmpty + acc), ((it >> 1) & 1) ^ 1, abort_flag, status))) break;
        ptx::tc_fence_after();
        for (int kb = 0; kb < KB; ++kb, ++i) {
          const int ws = i % kWStages, xs = i % kXStages;
          if (!(ok = wait_bar(bar(kBarWFull + ws), (i / kWStages) & 1, abort_flag, status))) break;
          if (!(ok = wait_bar(bar(kBarXFull + xs), (i / kXStages) & 1, abort_flag, status))) break;
          ptx::tc_fence_after();
          const uint32_t a_base = sbase + L::kWOff + ws * kWBytes;
          const uint32_t b_base = sbase + L::kXOff + xs * L::kXBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::mma_f8f6f4_ss(d_tmem, ptx::desc_kmajor_sw128(a_base + 32 * kk),
                               ptx::desc_kmajor_sw128(b_base + 32 * kk), idesc, (kb | kk) != 0);
          ptx::mma_commit(bar(kBarXEmpty + xs));
          ptx::mma_commit(bar(kBarWEmpty + ws));
        }
        if (ok) ptx::mma_commit(bar(kBarAccFull + acc));
      }
      if (!ok) {  // aborting: wait for the MMAs already issued
        ptx::mma_commit(bar(kBarDrain));
        drain_bar(bar(kBarDrain), 0);
      }
    }
    __syncwarp();
  } else if (warp < kFirstEpiWarp) {
    // ---------------- dequantize to E4M3 ----------------
    // Thread d = (row, half): row = d / 2 takes codes words 8 half .. 8 half + 7
    // of its row (two 16-byte chunks, read in a rotated order so that the
    // warp's shared loads are bank-conflict free).
    const int d = threadIdx.x - kFirstDeqWarp * 32;  // 0..255
    const int row = d >> 1, hf = d & 1;
    const int rot = (row >> 1) & 1;
    constexpr int kGPK = kKPerBlock / GS;
    bool ok = true;
    int i = 0;  // k-blocks so far (Q and W stage uses)
    for (int it = 0; it < ntiles && ok; ++it) {
      const int nn = tile_nt(it) * kBM + row;
      const float pow2e = pow2f(nn < N ? row_exp[nn] : 0);
      for (int kb = 0; kb < KB; ++kb, ++i) {
        const int qs = i % kQStages;
        if (!(ok = wait_bar(bar(kBarQFull + qs), (i / kQStages) & 1, abort_flag, status))) break;
        const uint8_t* qst = smem + L::kQOff + qs * kQStride;
        const uint8_t* qrow = qst + (row >> 4) * 1024 + (row & 15) * 64 + 32 * hf;
        uint4 c[2];
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) c[jj] = *reinterpret_cast<const uint4*>(qrow + 16 * ((jj + rot) & 1));
        // scale and zero point of this row, per group (rows past N read stale
        // values: their outputs are never stored)
        uint32_t sb[kGPK], z[kGPK];
#pragma unroll
        for (int g = 0; g < kGPK; ++g) {
          sb[g] = reinterpret_cast<const uint16_t*>(qst + kQScaleOff + 256 * g)[row];
          z[g] = (qst[kQZeroOff + 64 * g + (row >> 1)] >> (4 * (row & 1))) & 0xF;
        }
        ptx::mbar_arrive(bar(kBarQEmpty + qs));

        const int ws = i % kWStages;
        if (!(ok = wait_bar(bar(kBarWEmpty + ws), ((i / kWStages) & 1) ^ 1, abort_flag, status))) break;
        GroupConsts gc[kGPK];
#pragma unroll
        for (int g = 0; g < kGPK; ++g) gc[g] = group_consts(sb[g], z[g], pow2e);
        uint8_t* wt = smem + L::kWOff + ws * kWBytes + row * 128;
        // Word ww of code chunk cj = 2 hf + cl (cl = 0, 1; held by c[cl ^ rot])
        // holds inputs k0 .. k0 + 7 with k0 = GS (ww / J) + 8 (cj J + ww % J),
        // i.e. half k0 & 8 of 16-input chunk k0 / 16 of the row. The thread's
        // eight words fill four whole chunks, which go out as four 16-byte
        // stores; at a fixed store the 32 lanes (16 rows x 2 halves) hit the
        // eight swizzled chunk positions four times each (no bank conflict).
        // (Eight-byte stores left half of each chunk's banks idle per store:
        // 4x the ideal wavefronts at groups of 128.)
        constexpr int J = GS / 32;
        uint4 out[4];
#pragma unroll
        for (int cl = 0; cl < 2; ++cl) {
          const uint4 cw = rot ? c[cl ^ 1] : c[cl];
          const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
          for (int ww = 0; ww < 4; ++ww) {
            const int g = ww / J;
            const uint2 v = w8_word(words[ww], gc[g].zlo, gc[g].zhi, gc[g].s2);
            // slot (chunk among the thread's four) and half of this word
            const int slot = GS == 128 ? 2 * cl + (ww >> 1) : (GS == 64 ? 2 * (ww >> 1) + cl : ww);
            const int hi = GS == 32 ? cl : (ww & 1);
            if (hi) {
              out[slot].z = v.x;
              out[slot].w = v.y;
            } else {
              out[slot].x = v.x;
              out[slot].y = v.y;
            }
          }
        }
#pragma unroll
        for (int slot = 0; slot < 4; ++slot) {
          const int chunk = GS == 128 ? 4 * hf + slot : (GS == 64 ? 4 * (slot >> 1) + 2 * hf + (slot & 1) : 2 * slot + hf);
          *reinterpret_cast<uint4*>(wt + ((chunk ^ (row & 7)) << 4)) = out[slot];
        }
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(bar(kBarWFull + ws));
      }
    }
  } else {
    // ---------------- epilogue: y = fp16(acc * sx[m] * 2^-e[n]) ----------------
    const int quad = warp & 3;  // this warp may read TMEM lanes 32*quad .. +31
    const int r = 32 * quad + lane;
    for (int it = 0; it < ntiles; ++it) {
      const int acc = it & 1;
      if (!wait_bar(bar(kBarAccFull + acc), (it >> 1) & 1, abort_flag, status)) break;
      ptx::tc_fence_after();
      const int m0 = tile_m0(it), n = tile_nt(it) * kBM + r;
      const float pow2ne = pow2f(-(n < N ? row_exp[n] : 0));
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        if (m0 + c0 >= M) break;
        uint32_t v[32];
        ptx::tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(32 * quad) << 16) + (uint32_t)(acc * BN + c0), v);
        ptx::tmem_wait_ld();
        if (n < N) {
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const int m = m0 + c0 + j;
            if (m < M) {
              const float s0 = __ldg(sx + m) * pow2ne;
              const float s1 = m + 1 < M ? __ldg(sx + m + 1) * pow2ne : 0.f;
              const __half2 h = __floats2half2_rn(__uint_as_float(v[j]) * s0, __uint_as_float(v[j + 1]) * s1);
              y[(int64_t)m * N + n] = __low2half(h);
              if (m + 1 < M) y[(int64_t)(m + 1) * N + n] = __high2half(h);
            }
          }
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar(kBarAccEmpty + acc));  // this thread's loads of the accumulator are done
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, 2 * BN);
  }
}

// Token tiles per block of the tile order: as many as keep the block's x
// (tiles x BN tokens x K inputs) within ~48 MB of the 126 MB L2, at least one.
int token_tiles_per_block(int64_t M, int64_t K, int BN, int xbytes) {
  const int64_t mt = (M + BN - 1) / BN;
  int64_t g = (int64_t(48) << 20) / ((int64_t)BN * K * xbytes);
  if (g < 1) g = 1;
  return (int)(g < mt ? g : mt);
}

template <int BN, int GS>
cudaError_t launch_bn(const uint8_t* x8, const float* sx, const uint32_t* qweight, const __half* scales,
                      const uint8_t* zeros, const int8_t* row_exp, __half* y, int64_t M, int64_t K, int64_t N,
                      uint32_t* status, cudaStream_t stream) {
  using L = Layout<BN>;
  auto encode = tensor_map_encoder();
  if (!encode) return cudaErrorNotSupported;
  CUtensorMap tx;
  {
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)K};
    cuuint32_t box[2] = {(cuuint32_t)kKPerBlock, (cuuint32_t)BN};
    cuuint32_t estr[2] = {1, 1};
    if (encode(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(x8), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  static std::atomic<uint64_t> attr_set{0};  // one bit per device that has the attribute
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return cudaErrorInvalidDevice;
  if (!(attr_set.load(std::memory_order_acquire) >> dev & 1)) {
    cudaError_t e =
        cudaFuncSetAttribute(gemm_fp8_kernel<BN, GS>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(uint64_t(1) << dev, std::memory_order_acq_rel);
  }
  const int64_t tiles = ((M + BN - 1) / BN) * ((N + kBM - 1) / kBM);
  const int ctas = (int)(tiles < device_info().sm_count ? tiles : device_info().sm_count);  // one per SM
  gemm_fp8_kernel<BN, GS><<<ctas, kThreads, L::kAlloc, stream>>>(tx, sx, qweight, scales, zeros, row_exp, y, (int)M,
                                                                  (int)K, (int)N,
                                                                  token_tiles_per_block(M, K, BN, 1), status);
  return cudaGetLastError();
}

template <int GS>
cudaError_t launch_gs(const uint8_t* x8, const float* sx, const uint32_t* qweight, const __half* scales,
                      const uint8_t* zeros, const int8_t* row_exp, __half* y, int64_t M, int64_t K, int64_t N,
                      uint32_t* status, cudaStream_t stream) {
  // 256-token tiles unless they cannot give every SM a tile and 128-token
  // tiles would give it more (e.g. K=14336, N=4096, M=512: 64 against 128 tiles)
  const int64_t nt = (N + kBM - 1) / kBM;
  if (M > 128 && ((M + 255) / 256 * nt >= device_info().sm_count || (M + 127) / 128 * nt <= (M + 255) / 256 * nt))
    return launch_bn<256, GS>(x8, sx, qweight, scales, zeros, row_exp, y, M, K, N, status, stream);
  return launch_bn<128, GS>(x8, sx, qweight, scales, zeros, row_exp, y, M, K, N, status, stream);
}

}  // namespace

cudaError_t launch_fp8_row_exponents(const __half* scales, int64_t K, int64_t N, int group, int8_t* e_out,
                                     cudaStream_t stream) {
  fp8_row_exp_kernel<<<(unsigned)((N + 255) / 256), 256, 0, stream>>>(scales, N, K / group, e_out);
  return cudaGetLastError();
}

cudaError_t launch_fp8_quantize_x(const __half* x, int64_t M, int64_t K, uint8_t* x8, float* sx,
                                  cudaStream_t stream) {
  fp8_quant_x_kernel<<<(unsigned)M, 256, 0, stream>>>(x, K, x8, sx);
  return cudaGetLastError();
}

cudaError_t launch_dequant_fp8(const uint32_t* qweight, const __half* scales, const uint8_t* zeros,
                               const int8_t* row_exp, int64_t K, int64_t N, int group, uint8_t* w8_out,
                               cudaStream_t stream) {
  dim3 grid((unsigned)(N / kRowsPerBlock), (unsigned)(K / kKPerBlock));
  dequant_fp8_kernel<<<grid, 256, 0, stream>>>(qweight, scales, zeros, row_exp, K, N, group, w8_out);
  return cudaGetLastError();
}

cudaError_t launch_gemm_fp8(const uint8_t* x8, const float* sx, const uint32_t* qweight, const __half* scales,
                            const uint8_t* zeros, const int8_t* row_exp, __half* y, int64_t M, int64_t K, int64_t N,
                            int group, uint32_t* status, cudaStream_t stream) {
  switch (group) {
    case 128: return launch_gs<128>(x8, sx, qweight, scales, zeros, row_exp, y, M, K, N, status, stream);
    case 64: return launch_gs<64>(x8, sx, qweight, scales, zeros, row_exp, y, M, K, N, status, stream);
    case 32: return launch_gs<32>(x8, sx, qweight, scales, zeros, row_exp, y, M, K, N, status, stream);
    default: return cudaErrorInvalidConfiguration;
  }
}

}  // namespace awq
