// Context-stage (prefill) W4A16 GEMM on the sm_100a tensor cores
// (awq_w4a16_gemm).
//
// TinyChat README, "New Optimization of Context Stage": the prompt's tokens
// go through the same 4-bit linear layers as one batch, so for M in the
// hundreds to thousands the layer is a dense contraction and belongs on the
// tensor cores. The weights are dequantized just ahead of the MMA.
//
// Tile: 128 output channels (the MMA M dimension, "swap AB": the weight is
// operand A) x BN tokens (operand B, BN = 128 or 256) x the whole K.
// Persistent: one CTA per SM walks tiles c, c + P, ...; accumulation in tensor
// memory in two accumulators (fp32, 2 x BN columns x 128 lanes), so one tile's
// epilogue overlaps the next tile's main loop, and the rings below run on
// across tile boundaries (no pipeline refill per tile).
//
// Warp roles (480 threads):
//   warp 0  lane 0 issues TMA loads of x: 64-k x BN boxes with the 128-byte
//           swizzle, exactly the K-major operand layout tcgen05 reads.
//   warp 1  allocates tensor memory; lane 0 issues tcgen05.mma (4 per 64-k
//           stage, K = 16 each) into the tile's accumulator and commits to the
//           stage barriers and, at the end of a tile, to its accumulator's.
//   warp 2  issues bulk copies of the packed weight: the tile's 8 row blocks
//           of one 128-k block are one contiguous 8 KiB run.
//   warps 3-10 dequantize: threads 2r and 2r + 1 own weight row r of the
//           tile, each reads half of its 64 B of codes for the k-block from
//           shared memory, forms fp16_rne((q - z) * s) (the exact value the
//           dequant kernel and the CPU oracle produce) and stores it,
//           swizzled, into the A-operand buffer (two warps per SM
//           sub-partition hide the dependent fp16 chains).
//   warps 11-14 drain a finished accumulator (tcgen05.ld; warp w reads TMEM
//           lanes 32 (w % 4) ..) into fp16 y and release it.
// Rings: x 4 x (BN x 64 k), dequantized weight 2 x (128 x 128 k), packed
// weight 3 x 8 KiB, each with full/empty mbarriers. Every wait is bounded
// (2 s of %globaltimer); on expiry the CTA records AWQ_ERR_TIMEOUT in the
// status word, the other roles stop at their next wait, in-flight copies and
// MMAs are drained, tensor memory is freed and the CTA exits.
#include <cudaTypedefs.h>

#include <mutex>

#include "awq_internal.cuh"
#include "sm100_ptx.cuh"

namespace awq {
namespace {

constexpr int kBM = 128;
constexpr int kXStages = 4;
constexpr int kWStages = 2;
constexpr int kQStages = 3;
constexpr int kQBytes = 8 * 1024;
// Behind a stage's codes: the tile's scale rows (up to 4 groups x 128 fp16)
// and zero-point rows (up to 4 x 64 bytes) of that k-block.
constexpr int kQScaleOff = kQBytes, kQZeroOff = kQScaleOff + 4 * 256;
constexpr int kQStride = kQZeroOff + 4 * 64;
constexpr int kWHalfBytes = kBM * 64 * 2;  // 16 KiB: 128 rows x 64 k
constexpr int kWBytes = 2 * kWHalfBytes;
constexpr int kWarpX = 0, kWarpMma = 1, kWarpQ = 2, kFirstDeqWarp = 3, kNumDeqWarps = 8;
constexpr int kFirstEpiWarp = kFirstDeqWarp + kNumDeqWarps, kNumEpiWarps = 4;
constexpr int kDeqThreads = kNumDeqWarps * 32, kEpiThreads = kNumEpiWarps * 32;
constexpr int kThreads = (kFirstEpiWarp + kNumEpiWarps) * 32;

// barrier indices
constexpr int kBarXFull = 0, kBarXEmpty = kBarXFull + kXStages, kBarWFull = kBarXEmpty + kXStages,
              kBarWEmpty = kBarWFull + kWStages, kBarQFull = kBarWEmpty + kWStages,
              kBarQEmpty = kBarQFull + kQStages, kBarAccFull = kBarQEmpty + kQStages, kBarAccEmpty = kBarAccFull + 2,
              kBarDrain = kBarAccEmpty + 2, kNumBars = kBarDrain + 1;

template <int BN>
struct Layout {
  static constexpr int kXBytes = BN * 64 * 2;
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

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// Eight codes of one word (inputs k0 .. k0+7) -> eight fp16 W^ = fp16_rne((q - z) s).
// (word & 0x000F000F) | 0x64006400 = half2(1024 + q_even, 1024 + q_odd); the
// 0x00F000F0 mask gives 1024 + 16 q. Subtracting 1024 + z (or scaling by 1/16
// and subtracting 64 + z) is exact, and so the only rounding is that of the
// final product by s (one IEEE fp16 multiply).
__device__ __forceinline__ uint4 dequant_word(uint32_t w, __half2 zlo, __half2 zhi, __half2 s2) {
  const __half2 sixteenth = __half2half2(__ushort_as_half(0x2C00));  // 1/16
  uint4 o;
  o.x = h2u(__hmul2(__hsub2(u2h(lop3_and_or(w, 0x000F000Fu, 0x64006400u)), zlo), s2));
  o.y = h2u(__hmul2(__hfma2(u2h(lop3_and_or(w, 0x00F000F0u, 0x64006400u)), sixteenth, zhi), s2));
  w >>= 8;
  o.z = h2u(__hmul2(__hsub2(u2h(lop3_and_or(w, 0x000F000Fu, 0x64006400u)), zlo), s2));
  o.w = h2u(__hmul2(__hfma2(u2h(lop3_and_or(w, 0x00F000F0u, 0x64006400u)), sixteenth, zhi), s2));
  return o;
}

// GS: group size (128, 64 or 32), kGPK = 128 / GS groups per k-block.
// Persistent: CTA c computes tiles c, c + P, c + 2P, ... (P = gridDim.x; tile
// t is token tile t % MT of channel tile t / MT, so the CTAs running at the
// same time share a few weight tiles). Every role walks the same tile
// sequence; the rings run on across tile boundaries, and the two accumulators
// let the epilogue warps drain tile j while the MMA warp fills tile j + 1.
template <int BN, int GS>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const uint32_t* __restrict__ qweight,
                const __half* __restrict__ scales, const uint8_t* __restrict__ zeros, __half* __restrict__ y, int M,
                int K, int N, int GM, uint32_t* status) {
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
      // the codes' byte count + 32 cp.async arrivals (scales, zeros)
      ptx::mbar_init(bar(kBarQFull + i), 33);
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
  if (warp == kWarpX && lane == 0) {
    ptx::prefetch_tensormap(&tmap_x);
  }
  if (warp == kWarpMma) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), 2 * BN);
    ptx::tmem_relinquish();
    ptx::tc_fence_before();
  }
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == kWarpX) {
    // ---------------- x producer: 2 boxes of 64 k per k-block ----------------
    if (lane == 0) {
      int i = 0;  // stage uses so far
      bool ok = true;
      for (int it = 0; it < ntiles && ok; ++it) {
        const int m0 = tile_m0(it);
        for (int h = 0; h < 2 * KB; ++h, ++i) {
          const int s = i % kXStages;
          if (!(ok = wait_bar(bar(kBarXEmpty + s), ((i / kXStages) & 1) ^ 1, abort_flag, status))) break;
          ptx::mbar_arrive_expect_tx(bar(kBarXFull + s), L::kXBytes);
          ptx::tma_load_2d(sbase + L::kXOff + s * L::kXBytes, &tmap_x, h * 64, m0, bar(kBarXFull + s));
        }
      }
      if (!ok)  // aborting: let the copies already issued land
        for (int j = (i > kXStages ? i - kXStages : 0); j < i; ++j)
          drain_bar(bar(kBarXFull + j % kXStages), (j / kXStages) & 1);
    }
    __syncwarp();
  } else if (warp == kWarpQ) {
    // ---------------- packed-weight producer ----------------
    // The R <= 8 row blocks of a tile's group are one contiguous run of
    // R KiB per k-block in the packed layout: one 1-D bulk copy each. The
    // tile's scale and zero-point rows of the k-block follow by cp.async.
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
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = ptx::idesc_f16_f32(kBM, BN);
      bool ok = true;
      int wi = 0, xi = 0;  // W and x stage uses so far
      for (int it = 0; it < ntiles && ok; ++it) {
        const int acc = it & 1;
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);  // column offset of this accumulator
        if (!(ok = wait_bar(bar(kBarAccEmpty + acc), ((it >> 1) & 1) ^ 1, abort_flag, status))) break;
        ptx::tc_fence_after();
        for (int kb = 0; kb < KB && ok; ++kb, ++wi) {
          const int ws = wi % kWStages;
          if (!(ok = wait_bar(bar(kBarWFull + ws), (wi / kWStages) & 1, abort_flag, status))) break;
          ptx::tc_fence_after();
          for (int h = 0; h < 2; ++h, ++xi) {
            const int s = xi % kXStages;
            if (!(ok = wait_bar(bar(kBarXFull + s), (xi / kXStages) & 1, abort_flag, status))) break;
            ptx::tc_fence_after();
            const uint32_t a_base = sbase + L::kWOff + ws * kWBytes + h * kWHalfBytes;
            const uint32_t b_base = sbase + L::kXOff + s * L::kXBytes;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              ptx::mma_f16_ss(d_tmem, ptx::desc_kmajor_sw128(a_base + 32 * kk),
                              ptx::desc_kmajor_sw128(b_base + 32 * kk), idesc, (kb | h | kk) != 0);
            ptx::mma_commit(bar(kBarXEmpty + s));
          }
          if (ok) ptx::mma_commit(bar(kBarWEmpty + ws));
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
    // ---------------- dequantize ----------------
    // Thread d = (row, half): row = d / 2 takes words 8 half .. 8 half + 7 of
    // its row, two 16-byte chunks read and stored in a rotated order (the
    // rotation also depends on the half) so that every 8-lane phase of the
    // shared loads and of the swizzled stores touches distinct banks.
    const int d = threadIdx.x - kFirstDeqWarp * 32;  // 0..255
    const int row = d >> 1, hf = d & 1;
    const int rot = ((row >> 1) ^ hf) & 1;
    constexpr int kGPK = kKPerBlock / GS;
    bool ok = true;
    int i = 0;  // k-blocks so far (Q and W stage uses)
    for (int it = 0; it < ntiles && ok; ++it) {
      for (int kb = 0; kb < KB; ++kb, ++i) {
        const int qs = i % kQStages;
        if (!(ok = wait_bar(bar(kBarQFull + qs), (i / kQStages) & 1, abort_flag, status))) break;
        const uint8_t* qst = smem + L::kQOff + qs * kQStride;
        const uint8_t* qrow = qst + (row >> 4) * 1024 + (row & 15) * 64 + 32 * hf;
        uint4 c[2];
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) c[jj] = *reinterpret_cast<const uint4*>(qrow + 16 * ((jj + rot) & 1));
        // fp16 bits of the scale and the zero point of this row, per group (rows
        // past N read stale values: their outputs are never stored)
        uint32_t s[kGPK], z[kGPK];
#pragma unroll
        for (int g = 0; g < kGPK; ++g) {
          s[g] = reinterpret_cast<const uint16_t*>(qst + kQScaleOff + 256 * g)[row];
          z[g] = (qst[kQZeroOff + 64 * g + (row >> 1)] >> (4 * (row & 1))) & 0xF;
        }
        ptx::mbar_arrive(bar(kBarQEmpty + qs));

        const int ws = i % kWStages;
        if (!(ok = wait_bar(bar(kBarWEmpty + ws), ((i / kWStages) & 1) ^ 1, abort_flag, status))) break;
        __half2 s2[kGPK], zlo[kGPK], zhi[kGPK];
#pragma unroll
        for (int g = 0; g < kGPK; ++g) {
          // fp16 bit patterns: s itself, 1024 + z = 0x6400 + z, -(64 + z) = 0xD400 + 16 z
          s2[g] = u2h(s[g] * 0x00010001u);
          zlo[g] = u2h((0x6400u + z[g]) * 0x00010001u);
          zhi[g] = u2h((0xD400u + (z[g] << 4)) * 0x00010001u);
        }
        uint8_t* wt = smem + L::kWOff + ws * kWBytes + row * 128;
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int cj = 2 * hf + ((jj + rot) & 1);  // c[jj] holds words 4 cj .. 4 cj + 3 of the row
          const uint32_t words[4] = {c[jj].x, c[jj].y, c[jj].z, c[jj].w};
#pragma unroll
          for (int ww = 0; ww < 4; ++ww) {
            // word 4 cj + ww holds inputs k0 .. k0 + 7 of group ww / (GS / 32)
            // (word_k0 written out for this word: ww is a constant here)
            constexpr int J = GS / 32;
            const int k0 = GS * (ww / J) + 8 * (cj * J + ww % J), g = ww / J;
            const int chunk = (k0 & 63) >> 3;  // 16-byte chunk (8 k) within the 64-k half
            uint8_t* dst = wt + (k0 >> 6) * kWHalfBytes;
            *reinterpret_cast<uint4*>(dst + ((chunk ^ (row & 7)) << 4)) =
                dequant_word(words[ww], zlo[g], zhi[g], s2[g]);
          }
        }
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(bar(kBarWFull + ws));
      }
    }
  } else {
    // ---------------- epilogue: accumulator -> fp16 y ----------------
    const int quad = warp & 3;  // this warp may read TMEM lanes 32*quad .. +31
    const int r = 32 * quad + lane;
    for (int it = 0; it < ntiles; ++it) {
      const int acc = it & 1;
      if (!wait_bar(bar(kBarAccFull + acc), (it >> 1) & 1, abort_flag, status)) break;
      ptx::tc_fence_after();
      const int m0 = tile_m0(it), nn = tile_nt(it) * kBM + r;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        if (m0 + c0 >= M) break;
        uint32_t v[32];
        ptx::tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(32 * quad) << 16) + (uint32_t)(acc * BN + c0), v);
        ptx::tmem_wait_ld();
        if (nn < N) {
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const int m = m0 + c0 + j;
            // two conversions in one instruction, each rounded to nearest even
            const __half2 h = __floats2half2_rn(__uint_as_float(v[j]), __uint_as_float(v[j + 1]));
            if (m < M) y[(int64_t)m * N + nn] = __low2half(h);
            if (m + 1 < M) y[(int64_t)(m + 1) * N + nn] = __high2half(h);
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

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

template <int BN, int GS>
cudaError_t launch_bn(const __half* x, const uint32_t* qweight, const __half* scales, const uint8_t* zeros,
                      __half* y, int64_t M, int64_t K, int64_t N, uint32_t* status, cudaStream_t stream) {
  using L = Layout<BN>;
  auto encode = get_encode();
  if (!encode) return cudaErrorNotSupported;
  CUtensorMap tx;
  {
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)BN};
    cuuint32_t estr[2] = {1, 1};
    if (encode(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half*>(x), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  static uint64_t attr_set = 0;  // one bit per device that has the attribute
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return cudaErrorInvalidDevice;
  if (!(attr_set >> dev & 1)) {
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel<BN, GS>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return e;
    attr_set |= uint64_t(1) << dev;
  }
  const int64_t tiles = ((M + BN - 1) / BN) * ((N + kBM - 1) / kBM);
  const int ctas = (int)(tiles < device_info().sm_count ? tiles : device_info().sm_count);  // one per SM
  gemm_kernel<BN, GS><<<ctas, kThreads, L::kAlloc, stream>>>(tx, qweight, scales, zeros, y, (int)M, (int)K, (int)N,
                                                             token_tiles_per_block(M, K, BN, 2), status);
  return cudaGetLastError();
}

template <int GS>
cudaError_t launch_gs(const __half* x, const uint32_t* qweight, const __half* scales, const uint8_t* zeros,
                      __half* y, int64_t M, int64_t K, int64_t N, uint32_t* status, cudaStream_t stream) {
  // 256-token tiles unless they cannot give every SM a tile and 128-token
  // tiles would give it more (e.g. K=14336, N=4096, M=512: 64 against 128 tiles)
  const int64_t nt = (N + kBM - 1) / kBM;
  if (M > 128 && ((M + 255) / 256 * nt >= device_info().sm_count || (M + 127) / 128 * nt <= (M + 255) / 256 * nt))
    return launch_bn<256, GS>(x, qweight, scales, zeros, y, M, K, N, status, stream);
  return launch_bn<128, GS>(x, qweight, scales, zeros, y, M, K, N, status, stream);
}

}  // namespace

cudaError_t launch_gemm(const __half* x, const uint32_t* qweight, const __half* scales, const uint8_t* zeros,
                        __half* y, int64_t M, int64_t K, int64_t N, int group, uint32_t* status,
                        cudaStream_t stream) {
  switch (group) {
    case 128: return launch_gs<128>(x, qweight, scales, zeros, y, M, K, N, status, stream);
    case 64: return launch_gs<64>(x, qweight, scales, zeros, y, M, K, N, status, stream);
    case 32: return launch_gs<32>(x, qweight, scales, zeros, y, M, K, N, status, stream);
    default: return cudaErrorInvalidConfiguration;
  }
}

}  // namespace awq
