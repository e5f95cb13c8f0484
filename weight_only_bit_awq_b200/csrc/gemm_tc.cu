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
//   warps 3-10 dequantize in two groups of four that take alternate
//           k-blocks (two k-blocks in flight): in a group, thread r owns
//           weight row r of the tile, reads its 64 B of codes for the k-block
//           from shared memory, forms fp16_rne((q - z) * s) (the exact value
//           the dequant kernel and the CPU oracle produce) and stores it,
//           swizzled, into the A-operand buffer.
//   warps 11-14 drain a finished accumulator (tcgen05.ld; warp w reads TMEM
//           lanes 32 (w % 4) ..) into fp16 y and release it.
// gemm_pair_kernel (below) runs the same roles on clusters of two CTAs that
// share one MMA stream (tcgen05 cta_group::2) for the data-parallel schedule
// at 256-token tiles.
// Rings: x 3 x (BN x 64 k) for BN = 256, 6 x for BN = 128; dequantized weight
// 3 x (128 x 128 k); packed weight 3 x 8 KiB; each with full/empty mbarriers.
// (Measured on B200: 3 + 3 stages beat 4 + 2 by ~1 %; two x stages lose 9 %;
// 6-8 packed-weight stages or an L2 prefetch of the codes a few k-blocks
// ahead gain nothing.) Every wait is bounded
// (2 s of %globaltimer); on expiry the CTA records AWQ_ERR_TIMEOUT in the
// status word, the other roles stop at their next wait, in-flight copies and
// MMAs are drained, tensor memory is freed and the CTA exits.
#include <atomic>
#include <cudaTypedefs.h>

#include <mutex>

#include "awq_internal.cuh"
#include "sm100_ptx.cuh"

namespace awq {
namespace {

constexpr int kBM = 128;
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

template <int BN>
struct Layout {
  // ring depths: x stages of 64 k (BN x 64 fp16), dequantized-weight stages
  // of one 128-k block, code stages (an even number: the two dequant groups
  // take alternate k-blocks, and each stage must belong to one group)
  static constexpr int kXStages = BN == 256 ? 3 : 5;
  static constexpr int kWStages = 3;
  static constexpr int kQStages = BN == 256 ? 2 : 4;
  static_assert(kQStages % 2 == 0, "each code stage belongs to one dequant group");
  // barrier indices
  static constexpr int kBarXFull = 0, kBarXEmpty = kBarXFull + kXStages, kBarWFull = kBarXEmpty + kXStages,
                       kBarWEmpty = kBarWFull + kWStages, kBarQFull = kBarWEmpty + kWStages,
                       kBarQEmpty = kBarQFull + kQStages, kBarAccFull = kBarQEmpty + kQStages,
                       kBarAccEmpty = kBarAccFull + 2, kBarDrain = kBarAccEmpty + 2, kNumBars = kBarDrain + 1;
  static constexpr int kXBytes = BN * 64 * 2;
  static constexpr int kXOff = 0;
  static constexpr int kWOff = kXOff + kXStages * kXBytes;
  static constexpr int kQOff = kWOff + kWStages * kWBytes;
  static constexpr int kBarOff = kQOff + kQStages * kQStride;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1 KiB
};
static_assert(Layout<256>::kAlloc <= 232448 && Layout<128>::kAlloc <= 232448, "shared memory budget");

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

// Tile order: blocks of GM token tiles; within a block, token tile fastest,
// then channel tile. The x of one block stays in L2 while the block's channel
// tiles stream past it.
__device__ __forceinline__ void tile_coords(int t, int MT, int NT, int GM, int& mt, int& nt) {
  const int blk = t / (GM * NT), w = t - blk * GM * NT;
  const int gb = min(GM, MT - blk * GM);  // token tiles in this block
  mt = blk * GM + w % gb;
  nt = w / gb;
}

// ---- pieces shared by gemm_kernel and gemm_pair_kernel ----

// Fill code stage `st` (one lane-0 thread of the producer warp issues the
// bulk copy; the warp's lanes copy the scale and zero rows): the R <= 8 row
// blocks of channel tile gi for k-block kb are one contiguous run of R KiB in
// the packed layout (qbytes = R KiB, 0 for a channel tile past N). The tile's
// scale and zero-point rows of the k-block follow by cp.async; the stage's
// barrier `full` counts the bytes plus one arrival per lane.
template <int GS>
__device__ __forceinline__ void fill_code_stage(uint32_t st, uint32_t full, const uint32_t* __restrict__ qweight,
                                                const __half* __restrict__ scales, const uint8_t* __restrict__ zeros,
                                                int64_t gi, int kb, int KB, int64_t NB, int n0, int K, int N,
                                                uint32_t qbytes, int lane, uint32_t* status) {
  constexpr int kGPK = kKPerBlock / GS;
  const int64_t qw0 = qbytes > 0 ? unit_first_block(gi, kb, KB, NB) * kWordsPerBlock : 0;
  const bool qok = qbytes > 0 && AWQ_CHECK(in_range(qw0, qbytes / 4, (int64_t)K * N / 8), status);
  if (lane == 0) ptx::mbar_arrive_expect_tx(full, qok ? qbytes : 0u);
  __syncwarp();
  if (lane == 0 && qok) ptx::bulk_g2s(st, qweight + qw0, qbytes, full);
  for (int p = lane; p < kGPK * 16; p += 32) {  // kGPK rows of 128 scales: 16 B = 8 output channels
    const int g = p >> 4, l = p & 15;
    if (n0 + 8 * l < N &&
        AWQ_CHECK(in_range(((int64_t)kb * kGPK + g) * N + n0 + 8 * l, 8, (int64_t)(K / GS) * N), status))
      ptx::cp_async_16(st + kQScaleOff + 256 * g + 16 * l, scales + ((int64_t)kb * kGPK + g) * N + n0 + 8 * l);
  }
  for (int p = lane; p < kGPK * 8; p += 32) {  // kGPK rows of 64 zero bytes: 8 B = 16 output channels
    const int g = p >> 3, l = p & 7;
    if (n0 + 16 * l < N &&
        AWQ_CHECK(in_range(((int64_t)kb * kGPK + g) * (N / 2) + n0 / 2 + 8 * l, 8, (int64_t)(K / GS) * (N / 2)),
                  status))
      ptx::cp_async_8(st + kQZeroOff + 64 * g + 8 * l, zeros + ((int64_t)kb * kGPK + g) * (N / 2) + n0 / 2 + 8 * l);
  }
  ptx::cp_async_arrive_noinc(full);
}

// One weight row's codes, scales and zero points of a k-block, read from a
// code stage by the row's dequant thread. It reads the row's 64 B of codes as
// four 16-byte chunks in an order rotated by rot = (row / 2) % 4, so that
// every 8-lane phase of the shared loads (and of the swizzled stores below)
// touches distinct banks. Rows past N read stale values: their outputs are
// never stored.
template <int GS>
struct RowCodes {
  uint4 c[4];                                         // c[jj] holds words 4 ((jj + rot) & 3) ..
  uint32_t s[kKPerBlock / GS], z[kKPerBlock / GS];  // fp16 bits of the scale, zero point, per group
};
template <int GS>
__device__ __forceinline__ void load_row_codes(const uint8_t* qst, int row, int rot, RowCodes<GS>& rc) {
  const uint8_t* qrow = qst + (row >> 4) * 1024 + (row & 15) * 64;
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) rc.c[jj] = *reinterpret_cast<const uint4*>(qrow + 16 * ((jj + rot) & 3));
#pragma unroll
  for (int g = 0; g < kKPerBlock / GS; ++g) {
    rc.s[g] = reinterpret_cast<const uint16_t*>(qst + kQScaleOff + 256 * g)[row];
    rc.z[g] = (qst[kQZeroOff + 64 * g + (row >> 1)] >> (4 * (row & 1))) & 0xF;
  }
}
// fp16_rne((q - z) s) of the row's 128 inputs into its 128-byte line `wt` of
// each 64-k half of an A buffer (K-major, 128-byte swizzle).
template <int GS>
__device__ __forceinline__ void store_row_dequant(uint8_t* wt, int row, int rot, const RowCodes<GS>& rc) {
  constexpr int kGPK = kKPerBlock / GS, J = GS / 32;
  __half2 s2[kGPK], zlo[kGPK], zhi[kGPK];
#pragma unroll
  for (int g = 0; g < kGPK; ++g) {
    // fp16 bit patterns: s itself, 1024 + z = 0x6400 + z, -(64 + z) = 0xD400 + 16 z
    s2[g] = u2h(rc.s[g] * 0x00010001u);
    zlo[g] = u2h((0x6400u + rc.z[g]) * 0x00010001u);
    zhi[g] = u2h((0xD400u + (rc.z[g] << 4)) * 0x00010001u);
  }
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) {
    const int cj = (jj + rot) & 3;  // rc.c[jj] holds words 4 cj .. 4 cj + 3 of the row
    const uint32_t words[4] = {rc.c[jj].x, rc.c[jj].y, rc.c[jj].z, rc.c[jj].w};
#pragma unroll
    for (int ww = 0; ww < 4; ++ww) {
      // word 4 cj + ww holds inputs k0 .. k0 + 7 of group ww / J (word_k0
      // written out for this word: ww is a constant here)
      const int k0 = GS * (ww / J) + 8 * (cj * J + ww % J), g = ww / J;
      const int chunk = (k0 & 63) >> 3;  // 16-byte chunk (8 k) within the 64-k half
      uint8_t* dst = wt + (k0 >> 6) * kWHalfBytes;
      *reinterpret_cast<uint4*>(dst + ((chunk ^ (row & 7)) << 4)) = dequant_word(words[ww], zlo[g], zhi[g], s2[g]);
    }
  }
}

// GS: group size (128, 64 or 32), kGPK = 128 / GS groups per k-block.
// Persistent: CTA c computes the whole tiles c, c + P, c + 2P, ... below Tdp
// (P = gridDim.x; tile t maps to (token tile, channel tile) by tile_coords, so
// the CTAs running at the same time share a few weight tiles), then its share
// of the k-blocks of tiles Tdp .. T - 1 (stream-K; none when Tdp = T). Every
// role walks the same segment sequence; the rings run on across segment
// boundaries, and the two accumulators let the epilogue warps drain segment j
// while the MMA warp fills segment j + 1. `partial` (the workspace slots of
// split tiles) is only used when Tdp < T.
template <int BN, int GS>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const uint32_t* __restrict__ qweight,
                const __half* __restrict__ scales, const uint8_t* __restrict__ zeros, __half* __restrict__ y, int M,
                int K, int N, int GM, int Tdp, float* __restrict__ partial, int64_t part_floats, uint32_t* status) {
  using L = Layout<BN>;
  constexpr int kXStages = L::kXStages, kWStages = L::kWStages, kQStages = L::kQStages;
  constexpr int kBarXFull = L::kBarXFull, kBarXEmpty = L::kBarXEmpty, kBarWFull = L::kBarWFull,
                kBarWEmpty = L::kBarWEmpty, kBarQFull = L::kBarQFull, kBarQEmpty = L::kBarQEmpty,
                kBarAccFull = L::kBarAccFull, kBarAccEmpty = L::kBarAccEmpty, kBarDrain = L::kBarDrain;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + L::kBarOff + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + L::kMiscOff + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = K / kKPerBlock;
  const int MT = (M + BN - 1) / BN, NT = (N + kBM - 1) / kBM, T = MT * NT;
  const int P = gridDim.x, c = blockIdx.x;
  // Segments of this CTA: (tile t, k-blocks kb0 .. kb1 - 1). The first ndp are
  // the whole tiles c, c + P, ... below Tdp; the rest cover this CTA's equal
  // share [ub, ue) of the k-blocks of the last T - Tdp tiles ("stream-K"),
  // which the fixup kernel adds up where a tile is split between CTAs.
  const int ndp = c < Tdp ? (Tdp - 1 - c) / P + 1 : 0;
  const int Usk = (T - Tdp) * KB;
  const int ub = (int)((int64_t)c * Usk / P), ue = (int)((int64_t)(c + 1) * Usk / P);
  const int nseg = ndp + (ub < ue ? (ue - 1) / KB - ub / KB + 1 : 0);
  auto seg = [&](int j, int& t, int& kb0, int& kb1) {
    if (j < ndp) {
      t = c + j * P, kb0 = 0, kb1 = KB;
    } else {
      const int s = ub / KB + (j - ndp);
      t = Tdp + s;
      kb0 = j == ndp ? ub - s * KB : 0;
      kb1 = min(KB, ue - s * KB);
    }
  };
  auto tile_mn = [&](int t, int& mt, int& nt) { tile_coords(t, MT, NT, GM, mt, nt); };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kXStages; ++i) {
      ptx::mbar_init(bar(kBarXFull + i), 1);
      ptx::mbar_init(bar(kBarXEmpty + i), 1);
    }
    for (int i = 0; i < kWStages; ++i) {
      ptx::mbar_init(bar(kBarWFull + i), kDeqThreads / 2);  // one group of dequant warps fills a stage
      ptx::mbar_init(bar(kBarWEmpty + i), 1);
    }
    for (int i = 0; i < kQStages; ++i) {
      // the codes' byte count + 32 cp.async arrivals (scales, zeros)
      ptx::mbar_init(bar(kBarQFull + i), 33);
      ptx::mbar_init(bar(kBarQEmpty + i), kDeqThreads / 2);
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
  ptx::griddep_launch_dependents();  // lets the fixup kernel's CTAs become resident and wait

  if (warp == kWarpX) {
    // ---------------- x producer: 2 boxes of 64 k per k-block ----------------
    if (lane == 0) {
      int i = 0;  // stage uses so far
      bool ok = true;
      for (int j = 0; j < nseg && ok; ++j) {
        int t, kb0, kb1, mt, nt;
        seg(j, t, kb0, kb1);
        tile_mn(t, mt, nt);
        const int m0 = mt * BN;
        for (int h = 2 * kb0; h < 2 * kb1; ++h, ++i) {
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
    const int64_t NB = N / kRowsPerBlock;
    int i = 0;
    bool ok = true;
    for (int j = 0; j < nseg && ok; ++j) {
      int t, kb0, kb1, mt, nt;
      seg(j, t, kb0, kb1);
      tile_mn(t, mt, nt);
      const uint32_t qbytes = (uint32_t)(group_rows(nt, NB) * 1024);
      for (int kb = kb0; kb < kb1; ++kb, ++i) {
        const int s = i % kQStages;
        if (lane == 0) ok = wait_bar(bar(kBarQEmpty + s), ((i / kQStages) & 1) ^ 1, abort_flag, status);
        if (!(ok = __shfl_sync(0xffffffffu, ok, 0))) break;
        fill_code_stage<GS>(sbase + L::kQOff + s * kQStride, bar(kBarQFull + s), qweight, scales, zeros, nt, kb, KB, NB,
                            nt * kBM, K, N, qbytes, lane, status);
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
      for (int j = 0; j < nseg && ok; ++j) {
        int t, kb0, kb1;
        seg(j, t, kb0, kb1);
        const int acc = j & 1;
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);  // column offset of this accumulator
        if (!(ok = wait_bar(bar(kBarAccEmpty + acc), ((j >> 1) & 1) ^ 1, abort_flag, status))) break;
        ptx::tc_fence_after();
        for (int kb = kb0; kb < kb1 && ok; ++kb, ++wi) {
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
                              ptx::desc_kmajor_sw128(b_base + 32 * kk), idesc, ((kb - kb0) | h | kk) != 0);
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
    // Two groups of four warps take alternate k-blocks, so two k-blocks are
    // in flight and one group's barrier waits, loads and proxy fence overlap
    // the other's arithmetic; in a group, thread = weight row.
    const int d = threadIdx.x - kFirstDeqWarp * 32;  // 0..255
    const int grp = d >> 7, row = d & (kBM - 1);
    const int rot = (row >> 1) & 3;
    bool ok = true;
    int i = 0;  // k-blocks so far (Q and W stage uses)
    for (int j = 0; j < nseg && ok; ++j) {
      int t, kb0, kb1;
      seg(j, t, kb0, kb1);
      for (int kb = kb0; kb < kb1; ++kb, ++i) {
        if ((i & 1) != grp) continue;  // the other group's k-block
        // kQStages is even, so stage qs = i % kQStages always belongs to this
        // group and its uses reach this group in order, one phase apart (an
        // odd ring shared by alternating groups let a group wait two phases
        // ahead of a stage whose previous use had not landed, and a parity
        // wait cannot tell those phases apart)
        const int qs = i % kQStages;
        if (!(ok = wait_bar(bar(kBarQFull + qs), (i / kQStages) & 1, abort_flag, status))) break;
        RowCodes<GS> rc;
        load_row_codes<GS>(smem + L::kQOff + qs * kQStride, row, rot, rc);
        ptx::mbar_arrive(bar(kBarQEmpty + qs));
        const int ws = i % kWStages;
        if (!(ok = wait_bar(bar(kBarWEmpty + ws), ((i / kWStages) & 1) ^ 1, abort_flag, status))) break;
        store_row_dequant<GS>(smem + L::kWOff + ws * kWBytes + row * 128, row, rot, rc);
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(bar(kBarWFull + ws));
      }
    }
  } else {
    // ---------------- epilogue: accumulator -> fp16 y ----------------
    const int quad = warp & 3;  // this warp may read TMEM lanes 32*quad .. +31
    const int r = 32 * quad + lane;
    for (int j = 0; j < nseg; ++j) {
      int t, kb0, kb1, mt, nt;
      seg(j, t, kb0, kb1);
      tile_mn(t, mt, nt);
      const int acc = j & 1;
      if (!wait_bar(bar(kBarAccFull + acc), (j >> 1) & 1, abort_flag, status)) break;
      ptx::tc_fence_after();
      const int m0 = mt * BN, nn = nt * kBM + r;
      const bool whole = kb0 == 0 && kb1 == KB;
      // a part of a split tile goes to this CTA's slot: 0 for its first
      // stream-K segment, 1 for its last; layout [column m][row r], fp32
      float* slot = whole ? nullptr : partial + ((int64_t)(2 * c + (j == ndp ? 0 : 1)) * BN) * kBM + r;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        if (m0 + c0 >= M) break;
        uint32_t v[16];
        ptx::tmem_ld_32x32b_x16(tmem_base + ((uint32_t)(32 * quad) << 16) + (uint32_t)(acc * BN + c0), v);
        ptx::tmem_wait_ld();
        if (!whole) {
          if (AWQ_CHECK(in_range(slot - partial + c0 * kBM, 15 * kBM + 1, part_floats), status)) {
#pragma unroll
            for (int q = 0; q < 16; ++q) __stcg(slot + (c0 + q) * kBM, __uint_as_float(v[q]));
          }
        } else if (nn < N) {
#pragma unroll
          for (int q = 0; q < 16; q += 2) {
            const int m = m0 + c0 + q;
            // two conversions in one instruction, each rounded to nearest even
            const __half2 h = __floats2half2_rn(__uint_as_float(v[q]), __uint_as_float(v[q + 1]));
            if (m < M && AWQ_CHECK(in_range((int64_t)m * N + nn, 1, (int64_t)M * N), status))
              y[(int64_t)m * N + nn] = __low2half(h);
            if (m + 1 < M && AWQ_CHECK(in_range((int64_t)(m + 1) * N + nn, 1, (int64_t)M * N), status))
              y[(int64_t)(m + 1) * N + nn] = __high2half(h);
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

// ---------------------------------------------------------------------------
// CTA pairs (tcgen05 cta_group::2): tiles of 256 output channels x 256 tokens
// ---------------------------------------------------------------------------
// A cluster of two CTAs computes one 256-channel x 256-token tile with a
// single stream of tcgen05.mma issued by CTA 0 of the pair (the leader). CTA
// r dequantizes channel tile 2 np + r (its 128 rows of A) and loads tokens
// m0 + 128 r .. m0 + 128 r + 127 of x (its half of B); each MMA reads both
// CTAs' shared memory and accumulates each CTA's 128 rows x 256 tokens in that
// CTA's tensor memory. At the flops per SM of the one-CTA kernel, each SM holds
// and feeds the tensor core only half of the x tile, so the x ring is twice as
// deep in the same shared memory.
// Barriers: the leader's x-full barrier expects both halves' bytes, and both
// CTAs' TMA loads complete on it; the leader's W-full and accumulator-empty
// barriers count the dequant and epilogue threads of both CTAs, which arrive
// across the cluster; the MMA's commits arrive on the x-empty, W-empty and
// accumulator-full barriers of both CTAs (multicast commit). Code stages stay
// per CTA. Used for the data-parallel schedule at 256-token tiles (no
// stream-K), the large prefill shapes.
struct PairLayout {
  static constexpr int kHalfBN = 128;  // tokens of x per CTA
  static constexpr int kXStages = 6, kWStages = 3, kQStages = 2;
  static_assert(kQStages % 2 == 0, "each code stage belongs to one dequant group");
  static constexpr int kBarXFull = 0, kBarXEmpty = kBarXFull + kXStages, kBarWFull = kBarXEmpty + kXStages,
                       kBarWEmpty = kBarWFull + kWStages, kBarQFull = kBarWEmpty + kWStages,
                       kBarQEmpty = kBarQFull + kQStages, kBarAccFull = kBarQEmpty + kQStages,
                       kBarAccEmpty = kBarAccFull + 2, kBarDrain = kBarAccEmpty + 2, kNumBars = kBarDrain + 1;
  static constexpr int kXBytes = kHalfBN * 64 * 2;
  static constexpr int kXOff = 0;
  static constexpr int kWOff = kXOff + kXStages * kXBytes;
  static constexpr int kQOff = kWOff + kWStages * kWBytes;
  static constexpr int kBarOff = kQOff + kQStages * kQStride;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1 KiB
};
static_assert(PairLayout::kAlloc <= 232448, "shared memory budget");

// Pair tiles t = cl, cl + P2, ... of cluster cl (P2 clusters): tile_coords over
// token tiles x channel-tile pairs; this CTA's channel tile is 2 np + rank.
template <int GS>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_x, const uint32_t* __restrict__ qweight,
                     const __half* __restrict__ scales, const uint8_t* __restrict__ zeros, __half* __restrict__ y,
                     int M, int K, int N, int GM, uint32_t* status) {
  using L = PairLayout;
  constexpr int BN = 256;
  constexpr int kXStages = L::kXStages, kWStages = L::kWStages, kQStages = L::kQStages;
  constexpr int kBarXFull = L::kBarXFull, kBarXEmpty = L::kBarXEmpty, kBarWFull = L::kBarWFull,
                kBarWEmpty = L::kBarWEmpty, kBarQFull = L::kBarQFull, kBarQEmpty = L::kBarQEmpty,
                kBarAccFull = L::kBarAccFull, kBarAccEmpty = L::kBarAccEmpty, kBarDrain = L::kBarDrain;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + L::kBarOff + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + L::kMiscOff + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const bool leader = rank == 0;
  const int KB = K / kKPerBlock;
  const int MT = (M + BN - 1) / BN, NT = (N + kBM - 1) / kBM, NP = (NT + 1) / 2, T2 = MT * NP;
  const int P2 = (int)gridDim.x / 2, cl = (int)blockIdx.x / 2;
  const int ntiles = cl < T2 ? (T2 - 1 - cl) / P2 + 1 : 0;
  auto tile = [&](int j, int& mt, int& nt) {
    int np;
    tile_coords(cl + j * P2, MT, NP, GM, mt, np);
    nt = 2 * np + (int)rank;  // >= NT: no channels (the last pair when NT is odd)
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kXStages; ++i) {
      ptx::mbar_init(bar(kBarXFull + i), 1);   // the leader's expect_tx (both halves' bytes)
      ptx::mbar_init(bar(kBarXEmpty + i), 1);  // one commit
    }
    for (int i = 0; i < kWStages; ++i) {
      ptx::mbar_init(bar(kBarWFull + i), kDeqThreads);  // one dequant group in each CTA of the pair
      ptx::mbar_init(bar(kBarWEmpty + i), 1);
    }
    for (int i = 0; i < kQStages; ++i) {
      ptx::mbar_init(bar(kBarQFull + i), 33);
      ptx::mbar_init(bar(kBarQEmpty + i), kDeqThreads / 2);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar(kBarAccFull + i), 1);
      ptx::mbar_init(bar(kBarAccEmpty + i), 2 * kEpiThreads);  // the epilogue threads of both CTAs
    }
    ptx::mbar_init(bar(kBarDrain), 1);
    *abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  if (warp == kWarpX && lane == 0) ptx::prefetch_tensormap(&tmap_x);
  if (warp == kWarpMma) {
    ptx::tmem_alloc_pair(ptx::smem_u32(tmem_slot), 2 * BN);
    ptx::tmem_relinquish_pair();
    ptx::tc_fence_before();
  }
  __syncthreads();
  ptx::cluster_sync();  // both CTAs' barriers exist before any arrive crosses the pair
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  auto lead = [&](int i) -> uint32_t { return ptx::mapa(bar(i), 0); };  // the leader's barrier i

  if (warp == kWarpX) {
    // ---------------- x producer: this CTA's 128 tokens, 2 boxes of 64 k per k-block ----------------
    if (lane == 0) {
      int i = 0;
      bool ok = true;
      for (int j = 0; j < ntiles && ok; ++j) {
        int mt, nt;
        tile(j, mt, nt);
        const int m0 = mt * BN + L::kHalfBN * (int)rank;
        for (int h = 0; h < 2 * KB; ++h, ++i) {
          const int s = i % kXStages;
          if (!(ok = wait_bar(bar(kBarXEmpty + s), ((i / kXStages) & 1) ^ 1, abort_flag, status))) break;
          if (leader) ptx::mbar_arrive_expect_tx(bar(kBarXFull + s), 2 * L::kXBytes);
          ptx::tma_load_2d_pair(sbase + L::kXOff + s * L::kXBytes, &tmap_x, h * 64, m0, lead(kBarXFull + s));
        }
      }
      if (!ok) {
        if (leader) {  // aborting: let the copies the leader's barriers count land
          for (int j = (i > kXStages ? i - kXStages : 0); j < i; ++j)
            drain_bar(bar(kBarXFull + j % kXStages), (j / kXStages) & 1);
        } else {  // the peer's copies count on the leader's barriers: give them time to land
          const uint64_t t0 = ptx::globaltimer_ns();
          while (ptx::globaltimer_ns() - t0 < ptx::kDrainLimitNs) {
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == kWarpQ) {
    // ---------------- packed-weight producer (this CTA's channel tile) ----------------
    const int64_t NB = N / kRowsPerBlock;
    int i = 0;
    bool ok = true;
    for (int j = 0; j < ntiles && ok; ++j) {
      int mt, nt;
      tile(j, mt, nt);
      const uint32_t qbytes = nt < NT ? (uint32_t)(group_rows(nt, NB) * 1024) : 0u;
      for (int kb = 0; kb < KB; ++kb, ++i) {
        const int s = i % kQStages;
        if (lane == 0) ok = wait_bar(bar(kBarQEmpty + s), ((i / kQStages) & 1) ^ 1, abort_flag, status);
        if (!(ok = __shfl_sync(0xffffffffu, ok, 0))) break;
        fill_code_stage<GS>(sbase + L::kQOff + s * kQStride, bar(kBarQFull + s), qweight, scales, zeros, nt, kb, KB, NB,
                            nt * kBM, K, N, qbytes, lane, status);
      }
    }
    if (!ok && lane == 0)
      for (int j = (i > kQStages ? i - kQStages : 0); j < i; ++j)
        drain_bar(bar(kBarQFull + j % kQStages), (j / kQStages) & 1);
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ---------------- MMA issuer (the leader only) ----------------
    if (leader && lane == 0) {
      const uint32_t idesc = ptx::idesc_f16_f32(2 * kBM, BN);  // M = 256 over the pair
      bool ok = true;
      int wi = 0, xi = 0;
      for (int j = 0; j < ntiles && ok; ++j) {
        const int acc = j & 1;
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        if (!(ok = wait_bar(bar(kBarAccEmpty + acc), ((j >> 1) & 1) ^ 1, abort_flag, status))) break;
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
              ptx::mma_f16_ss_pair(d_tmem, ptx::desc_kmajor_sw128(a_base + 32 * kk),
                                   ptx::desc_kmajor_sw128(b_base + 32 * kk), idesc, (kb | h | kk) != 0);
            ptx::mma_commit_pair(bar(kBarXEmpty + s));
          }
          if (ok) ptx::mma_commit_pair(bar(kBarWEmpty + ws));
        }
        if (ok) ptx::mma_commit_pair(bar(kBarAccFull + acc));
      }
      if (!ok) {  // aborting: wait for the MMAs already issued
        ptx::mma_commit_pair(bar(kBarDrain));
        drain_bar(bar(kBarDrain), 0);
      }
    }
    __syncwarp();
  } else if (warp < kFirstEpiWarp) {
    // ---------------- dequantize (as in gemm_kernel; W-full is the leader's) ----------------
    const int d = threadIdx.x - kFirstDeqWarp * 32;
    const int grp = d >> 7, row = d & (kBM - 1);
    const int rot = (row >> 1) & 3;
    bool ok = true;
    int i = 0;
    for (int j = 0; j < ntiles && ok; ++j) {
      for (int kb = 0; kb < KB; ++kb, ++i) {
        if ((i & 1) != grp) continue;
        const int qs = i % kQStages;
        if (!(ok = wait_bar(bar(kBarQFull + qs), (i / kQStages) & 1, abort_flag, status))) break;
        RowCodes<GS> rc;
        load_row_codes<GS>(smem + L::kQOff + qs * kQStride, row, rot, rc);
        ptx::mbar_arrive(bar(kBarQEmpty + qs));
        const int ws = i % kWStages;
        if (!(ok = wait_bar(bar(kBarWEmpty + ws), ((i / kWStages) & 1) ^ 1, abort_flag, status))) break;
        store_row_dequant<GS>(smem + L::kWOff + ws * kWBytes + row * 128, row, rot, rc);
        ptx::fence_proxy_async_smem();
        if (leader)
          ptx::mbar_arrive(bar(kBarWFull + ws));
        else
          ptx::mbar_arrive_cluster(lead(kBarWFull + ws));
      }
    }
  } else {
    // ---------------- epilogue: this CTA's 128 channels x 256 tokens ----------------
    const int quad = warp & 3;
    const int r = 32 * quad + lane;
    for (int j = 0; j < ntiles; ++j) {
      int mt, nt;
      tile(j, mt, nt);
      const int acc = j & 1;
      if (!wait_bar(bar(kBarAccFull + acc), (j >> 1) & 1, abort_flag, status)) break;
      ptx::tc_fence_after();
      const int m0 = mt * BN, nn = nt * kBM + r;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        if (m0 + c0 >= M) break;
        uint32_t v[16];
        ptx::tmem_ld_32x32b_x16(tmem_base + ((uint32_t)(32 * quad) << 16) + (uint32_t)(acc * BN + c0), v);
        ptx::tmem_wait_ld();
        if (nt < NT && nn < N) {
#pragma unroll
          for (int q = 0; q < 16; q += 2) {
            const int m = m0 + c0 + q;
            const __half2 h = __floats2half2_rn(__uint_as_float(v[q]), __uint_as_float(v[q + 1]));
            if (m < M && AWQ_CHECK(in_range((int64_t)m * N + nn, 1, (int64_t)M * N), status))
              y[(int64_t)m * N + nn] = __low2half(h);
            if (m + 1 < M && AWQ_CHECK(in_range((int64_t)(m + 1) * N + nn, 1, (int64_t)M * N), status))
              y[(int64_t)(m + 1) * N + nn] = __high2half(h);
          }
        }
      }
      ptx::tc_fence_before();
      if (leader)
        ptx::mbar_arrive(bar(kBarAccEmpty + acc));
      else
        ptx::mbar_arrive_cluster(lead(kBarAccEmpty + acc));
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // the pair's MMAs, copies and tensor-memory reads are done in both CTAs
  if (warp == kWarpMma) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem_base, 2 * BN);
  }
}

// Stream-K tiles split between CTAs: CTA (s, b) adds the parts of stream-K
// tile s, token columns 32 b .. 32 b + 31, thread = channel row of the tile.
// The contributors are the CTAs whose k-block ranges meet the tile's, in CTA
// order (so y does not depend on timing); a contributor's part is in its
// slot 0 if its range starts inside the tile (the tile is its first
// stream-K segment) and in slot 1 otherwise (the tile is its last). Tiles
// that one CTA covered whole were written by the GEMM itself.
// Launched right behind the GEMM (programmatic dependent launch): its CTAs
// wait for the GEMM's writes in griddepcontrol.wait.
template <int BN>
__global__ void __launch_bounds__(kBM) gemm_fixup_kernel(const float* __restrict__ partial, __half* __restrict__ y,
                                                         int M, int N, int KB, int GM, int Tdp, int P,
                                                         int64_t part_floats, uint32_t* status) {
  ptx::griddep_launch_dependents();
  const int MT = (M + BN - 1) / BN, NT = (N + kBM - 1) / kBM;
  const int64_t Usk = (int64_t)(MT * NT - Tdp) * KB;
  const int s = blockIdx.x;
  auto cta_of = [&](int64_t u) { return (int)(((u + 1) * P - 1) / Usk); };  // CTA whose range holds unit u
  const int c_first = cta_of((int64_t)s * KB), c_last = cta_of((int64_t)(s + 1) * KB - 1);
  if (c_first == c_last) return;
  int mt, nt;
  tile_coords(Tdp + s, MT, NT, GM, mt, nt);
  const int mb = mt * BN + 32 * (int)blockIdx.y;  // first token of this CTA
  const int r = threadIdx.x, n = nt * kBM + r;
  if (mb >= M || n >= N) return;
  const int mcount = min(32, M - mb);
  ptx::griddep_wait();
  float v[32];
#pragma unroll
  for (int q = 0; q < 32; ++q) v[q] = 0.f;
  for (int cc = c_first; cc <= c_last; ++cc) {
    const int which = (int64_t)cc * Usk / P >= (int64_t)s * KB ? 0 : 1;
    const float* p = partial + ((int64_t)(2 * cc + which) * BN + 32 * blockIdx.y) * kBM + r;
    if (!AWQ_CHECK(in_range(p - partial, (int64_t)(mcount - 1) * kBM + 1, part_floats), status)) return;
#pragma unroll
    for (int q = 0; q < 32; ++q)
      if (q < mcount) v[q] += __ldcg(p + q * kBM);
  }
  if (!AWQ_CHECK(in_range((int64_t)mb * N + n, (int64_t)(mcount - 1) * N + 1, (int64_t)M * N), status)) return;
#pragma unroll
  for (int q = 0; q < 32; ++q)
    if (q < mcount) y[(int64_t)(mb + q) * N + n] = __float2half_rn(v[q]);
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
cudaError_t launch_bn(const __half* x, const uint32_t* qweight, const __half* scales, const uint8_t* zeros,
                      __half* y, int64_t M, int64_t K, int64_t N, const GemmPlan& p, void* workspace,
                      cudaStream_t stream) {
  using L = Layout<BN>;
  auto encode = tensor_map_encoder();
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
  static std::atomic<uint64_t> attr_set{0};  // one bit per device that has the attribute
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return cudaErrorInvalidDevice;
  if (!(attr_set.load(std::memory_order_acquire) >> dev & 1)) {
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel<BN, GS>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(uint64_t(1) << dev, std::memory_order_acq_rel);
  }
  char* ws = static_cast<char*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  float* partial = p.stream_k ? reinterpret_cast<float*>(ws + p.partial_off) : nullptr;
  const int64_t part_floats = p.stream_k ? (int64_t)(p.ws_bytes - p.partial_off) / 4 : 0;
  gemm_kernel<BN, GS><<<p.ctas, kThreads, L::kAlloc, stream>>>(tx, qweight, scales, zeros, y, (int)M, (int)K, (int)N,
                                                               p.gm, p.dp_tiles, partial, part_floats, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || !p.stream_k) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.tiles - p.dp_tiles), (unsigned)(BN / 32));
  cfg.blockDim = dim3(kBM);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_fixup_kernel<BN>, (const float*)partial, y, (int)M, (int)N, (int)(K / kKPerBlock),
                            p.gm, p.dp_tiles, p.ctas, part_floats, status);
}

// Pair clusters that can be resident at once on device `dev` (0 if none): the
// grid of gemm_pair_kernel, cached per device.
template <int GS>
int pair_clusters(int dev) {
  static std::atomic<int> cache[64];
  int n = cache[dev].load(std::memory_order_acquire);
  if (n != 0) return n > 0 ? n : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = PairLayout::kAlloc;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, gemm_pair_kernel<GS>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    clusters = 0;
  }
  cache[dev].store(clusters > 0 ? clusters : -1, std::memory_order_release);
  return clusters;
}

template <int GS>
cudaError_t launch_pair(const __half* x, const uint32_t* qweight, const __half* scales, const uint8_t* zeros,
                        __half* y, int64_t M, int64_t K, int64_t N, const GemmPlan& p, void* workspace,
                        cudaStream_t stream) {
  using L = PairLayout;
  auto encode = tensor_map_encoder();
  if (!encode) return cudaErrorNotSupported;
  CUtensorMap tx;
  {
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)L::kHalfBN};
    cuuint32_t estr[2] = {1, 1};
    if (encode(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half*>(x), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  static std::atomic<uint64_t> attr_set{0};  // one bit per device that has the attribute
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return cudaErrorInvalidDevice;
  if (!(attr_set.load(std::memory_order_acquire) >> dev & 1)) {
    cudaError_t e = cudaFuncSetAttribute(gemm_pair_kernel<GS>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(uint64_t(1) << dev, std::memory_order_acq_rel);
  }
  const int64_t NT = (N + kBM - 1) / kBM, T2 = (M + 255) / 256 * ((NT + 1) / 2);
  int clusters = pair_clusters<GS>(dev);
  if (clusters <= 0) return launch_bn<256, GS>(x, qweight, scales, zeros, y, M, K, N, p, workspace, stream);
  if (clusters > T2) clusters = (int)T2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * clusters));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L::kAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  uint32_t* status = reinterpret_cast<uint32_t*>(workspace);
  return cudaLaunchKernelEx(&cfg, gemm_pair_kernel<GS>, tx, qweight, scales, zeros, y, (int)M, (int)K, (int)N,
                            token_tiles_per_block(M, K, 256, 2), status);
}

template <int GS>
cudaError_t launch_gs(const __half* x, const uint32_t* qweight, const __half* scales, const uint8_t* zeros,
                      __half* y, int64_t M, int64_t K, int64_t N, const GemmPlan& p, void* workspace,
                      cudaStream_t stream) {
  if (p.pair) return launch_pair<GS>(x, qweight, scales, zeros, y, M, K, N, p, workspace, stream);
  if (p.bn == 256) return launch_bn<256, GS>(x, qweight, scales, zeros, y, M, K, N, p, workspace, stream);
  return launch_bn<128, GS>(x, qweight, scales, zeros, y, M, K, N, p, workspace, stream);
}

}  // namespace

// Schedule of the W4A16 GEMM.
// Token tile: 256 unless 256-token tiles cannot give every SM a tile and
// 128-token tiles would give it more (e.g. K=14336, N=4096, M=512: 64 against
// 128 tiles).
// Data-parallel: min(tiles, SMs) CTAs walk whole tiles. When that leaves the
// last wave of tiles very short (under 80 % of the SM-tile slots busy), the
// schedule turns "stream-K": all but the last full wave and the partial one
// stay data-parallel, and the k-blocks of the remaining tiles are split
// evenly over one CTA per SM, so every SM gets the same number of k-blocks;
// tiles split between CTAs are finished by the fixup kernel from fp32 parts in
// the workspace (two slots of 128 x BN per CTA). Measured on B200, stream-K
// gains 8 % where 3.03 waves of tiles would take 4 (K=4096, N=28672, M=512)
// but loses up to 4 % at 1.73 or 12.1 waves: the parts and the fixup cost
// about what the idle SMs did. It needs at least 8 k-blocks per CTA and is
// not used for M <= AWQ_GEMV_MAX_M, so decode-sized workspaces stay what the
// GEMV needs.
GemmPlan plan_gemm(int64_t M, int64_t K, int64_t N, int sm_count) {
  GemmPlan p{};
  const int64_t nt = (N + kBM - 1) / kBM;
  p.bn = (M > 128 && ((M + 255) / 256 * nt >= sm_count || (M + 127) / 128 * nt <= (M + 255) / 256 * nt)) ? 256 : 128;
  const int64_t mt = (M + p.bn - 1) / p.bn, KB = K / kKPerBlock;
  p.tiles = (int)(mt * nt);
  p.gm = token_tiles_per_block(M, K, p.bn, 2);
  p.ctas = p.tiles < sm_count ? p.tiles : sm_count;
  p.dp_tiles = p.tiles;
  p.ws_bytes = kWsHeaderBytes;
  const int64_t waves = (p.tiles + sm_count - 1) / sm_count;
  const int64_t tsk = p.tiles < sm_count ? p.tiles : sm_count + p.tiles % sm_count;
  if (M > AWQ_GEMV_MAX_M && p.tiles % sm_count != 0 && 100 * (int64_t)p.tiles < 80 * waves * sm_count &&
      tsk * KB >= 8 * (int64_t)sm_count) {
    p.stream_k = true;
    p.ctas = sm_count;
    p.dp_tiles = (int)(p.tiles - tsk);
    p.partial_off = kWsHeaderBytes;
    p.ws_bytes = p.partial_off + (size_t)p.ctas * 2 * p.bn * kBM * sizeof(float);
  }
  // CTA pairs for the data-parallel schedule at 256-token tiles with at least
  // two channel tiles
  p.pair = p.bn == 256 && !p.stream_k && nt >= 2;
  return p;
}

cudaError_t launch_gemm(const __half* x, const uint32_t* qweight, const __half* scales, const uint8_t* zeros,
                        __half* y, int64_t M, int64_t K, int64_t N, int group, const GemmPlan& plan, void* workspace,
                        cudaStream_t stream) {
  switch (group) {
    case 128: return launch_gs<128>(x, qweight, scales, zeros, y, M, K, N, plan, workspace, stream);
    case 64: return launch_gs<64>(x, qweight, scales, zeros, y, M, K, N, plan, workspace, stream);
    case 32: return launch_gs<32>(x, qweight, scales, zeros, y, M, K, N, plan, workspace, stream);
    default: return cudaErrorInvalidConfiguration;
  }
}

}  // namespace awq
