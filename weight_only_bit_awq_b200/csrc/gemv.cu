// Decode-stage W4A16 GEMV (awq_w4a16_gemv), 1 <= M <= 32.
//
// TinyChat README, "Speed Benchmarks": the generation stage runs one token
// (or a few) per step through 4-bit-weight linear layers, so each layer is a
// GEMV whose cost is streaming its packed weights from HBM once.
//
// Work split ("stream-K" over units). A unit is KU consecutive k-blocks (128
// input channels each, one quantization group) of one group of 8 row blocks
// (128 output channels): up to KU x 8 KiB of codes that the packed layout
// stores contiguously, plus their scales and zeros (one 256-byte and one
// 64-byte row slice per k-block). The last unit of a group is shorter when KU
// does not divide K/128. Units are numbered group-major, i.e. in memory order,
// and every CTA (two per SM, one for M > 16) streams an equal contiguous
// range of them, so the load is balanced to one unit. KU (1, 2 or 4) is
// chosen per layer: bigger units spend less of the producer's issue time on
// the small per-unit copies, smaller units balance small layers better.
//
// Inside a CTA:
//   warp 0 (producer) keeps a ring of shared-memory stages full: per unit one
//     1-D bulk copy of the codes, cp.async copies of the scales and zeros,
//     and one bulk copy per token of x[m][128 kb0 .. 128 (kb0 + KU)); the
//     stage's mbarrier tracks completion (transaction bytes plus the cp.async
//     arrivals). The ring depth follows from the shared memory left for the
//     stage size. The codes of the first stage are requested before the
//     kernel waits for the previous grid in the stream (programmatic
//     dependent launch): they do not depend on it; x does.
//   warps 1-8 (consumers): warp w owns row block w of every unit, so it
//     accumulates its 16 output channels over the whole k-range in registers
//     with no cross-warp reduction. Per k-block a lane reads two 16-byte words
//     of codes (rows g and g+8, k = 32t .. 32t+31) and feeds mma.sync
//     m16n8k16 (A = 16 rows x 16 k from registers, B = 16 k x 8 tokens from
//     shared memory). The MMA sums over k, so any permutation of k applied to
//     A and B alike is allowed: a lane pairs the k it loaded with the fragment
//     slots it owns. The fp32 result of a k-block is sum_k x (q - z) over one
//     group; y += s * that, in fp32, so no weight is rounded. For M <= 2 with
//     groups of 128 the consumers use integer MMAs instead (mma.sync
//     m16n8k32, u8 codes x s8 digits of x; see the integer path below).
//   warp 9 (M <= 8 only) reads each stage's x first: per-k-block sums of x for
//     the lo/hi path (see block_mma_lohi), or, on the integer path, the
//     block fixed-point digits and coefficients of x.
//
// Output. A warp that saw all k-blocks of its row block writes fp16 y. A row
// block split between CTAs (only the first and the last group of a CTA's
// range) gets each CTA's fp32 partial sums in a workspace slot, written with
// plain stores, so streaming never waits on another CTA; a small fixup
// kernel launched right behind the GEMV (programmatic dependent launch) adds
// the slots in CTA order (deterministic) and writes y.
#include <atomic>
#include <type_traits>

#include "awq_internal.cuh"
#include "sm100_ptx.cuh"
#include "gemv_common.cuh"

namespace awq {
namespace {

constexpr int kConsumers = kGroupBlocks;  // one consumer warp per row block of a unit
constexpr int kWarpXsum = 1 + kConsumers;  // per-k-block sums of x (M <= 8)
constexpr int kThreads = (2 + kConsumers) * 32;
// Shared memory one CTA may use (two CTAs per SM share 228 KiB, minus the
// 1 KiB per CTA the hardware reserves).
constexpr int kSmemPerCta2 = 112 * 1024;
constexpr int kSmemPerCta1 = 226 * 1024;


// Byte offsets inside one ring stage for a unit of up to KU k-blocks, M
// tokens and groups of GS inputs (the same numbers on the host and in every
// thread). Scales, zeros and x sums hold one row per group of the unit; on
// the integer path the x-sum slot of a k-block holds its B fragments. Token
// m's KU k-blocks of x start at x + m * xrow: the 16 pad bytes per token put
// the eight tokens a warp's B-fragment load reads at one k on eight different
// 16-byte bank groups (without them all eight share one: an 8-way conflict).
struct Stage {
  int q, s, z, xs, x, xrow, bytes;
  __host__ __device__ Stage(int KU, int M, int GS, bool integer = false) {
    const int rows = KU * (kKPerBlock / GS);
    q = 0;
    s = q + KU * kKbQBytes;
    z = s + rows * kKbScaleBytes;
    xs = z + rows * kKbZeroBytes;
    x = xs + rows * (integer ? int_xs_bytes(M) : kKbXsBytes);
    xrow = KU * kXRowBytes + 16;
    bytes = x + M * xrow;  // every term is a multiple of 16
  }
};

// M <= 2, groups of 128 ("integer path"): exact integer MMAs on the codes.
// Per k-block and token, the x-prep warp writes x as a block fixed-point
// integer, X = rint(x * 2^(44 - eb)) with eb the largest fp16 exponent field
// of the k-block (at least 1), so |X| < 2^30 and X is exact unless |x| is
// below 2^-19 of the k-block's largest value. X is split into four signed
// base-256 digits, X = sum_d 256^d D_d (the bytes of (X + 0x80808080) ^
// 0x80808080), and digit d of token m becomes column 4 m + d of the B operand
// of mma.sync m16n8k32 (u8 x s8 -> s32): the columns an M = 1 GEMV leaves
// idle. The codes enter operand A as bytes without conversion: word &
// 0x0F0F0F0F gives q of inputs {0, 4, 1, 5} of the word ("lo"), word &
// 0xF0F0F0F0 gives 16 q of {2, 6, 3, 7} ("hi"); lo and hi go to separate
// accumulators, and the B bytes are laid out in the same k order. Per column
// the k-block's exact integer sum is then 16 acc_lo + acc_hi = 16 sum_k q D_d,
// so
//   sum_k x (q - z) = sum_d 2^(eb - 48 + 8 d) (16 acc_lo + acc_hi) - z sum_k x,
// with sum_k x in fp32 from the x-prep warp. 4 integer MMAs and 16 lop3 per
// 2048 weights; the digit columns are added across lanes once, at the end.
// A non-finite x sets the k-block's coefficients to NaN, so y is NaN.
//
// Unit numbering: UPG = ceil(KB / KU) units per group; unit u is group
// u / UPG, k-blocks KU (u % UPG) .. min(KB, KU (u % UPG + 1)) - 1. CTA c of P
// streams units [c U / P, (c + 1) U / P).
struct Range {
  int64_t KB, NB, UPG, U, P;
  __host__ __device__ Range(int64_t K, int64_t N, int KU, int64_t P_) {
    KB = K / kKPerBlock;
    NB = N / kRowsPerBlock;
    UPG = (KB + KU - 1) / KU;
    U = (NB + kGroupBlocks - 1) / kGroupBlocks * UPG;
    P = P_;
  }
  __host__ __device__ __forceinline__ int64_t first_unit(int64_t c) const { return c * U / P; }
  __host__ __device__ __forceinline__ int64_t cta_of(int64_t u) const { return ((u + 1) * P - 1) / U; }
};

// kM1: M == 1 (NT == 1), where only the epilogue slots of token 0 are
// computed. GS: group size (128, 64 or 32). kInt: the integer path (NT == 1,
// M <= 2, GS == 128).
template <int NT, int KU, bool kM1, int GS, bool kInt>
__global__ void __launch_bounds__(kThreads, NT == 4 ? 1 : 2)
    gemv_kernel(const __half* __restrict__ x, const uint32_t* __restrict__ qweight, const __half* __restrict__ scales,
                const uint8_t* __restrict__ zeros, __half* __restrict__ y, int M, int K, int N, int NS,
                float* __restrict__ partial, int64_t part_floats, uint32_t* status) {
  extern __shared__ __align__(16) uint8_t smem[];
  static_assert(!kInt || (NT == 1 && GS == 128 && !kM1), "integer path: one token tile, groups of 128");
  constexpr bool kLoHi = NT == 1 && !kInt;
  constexpr bool kXWarp = kLoHi || kInt;  // a ninth warp reads x first and prepares it
  constexpr int kGPK = Grp<GS>::kPerKb;  // groups per k-block
  const Stage L(KU, M, GS, kInt);
  const uint32_t sbase = ptx::smem_u32(smem);
  const uint32_t bar0 = sbase + NS * L.bytes;
  auto full = [&](int s) -> uint32_t { return bar0 + 8 * s; };
  auto empty = [&](int s) -> uint32_t { return bar0 + 8 * (kMaxStages + s); };
  auto xland = [&](int s) -> uint32_t { return bar0 + 8 * (2 * kMaxStages + s); };
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + NS * L.bytes + 3 * kMaxStages * 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Range rg(K, N, KU, gridDim.x);
  const int64_t c = blockIdx.x;
  const int64_t u0 = rg.first_unit(c), u1 = rg.first_unit(c + 1);
  const int n_units = (int)(u1 - u0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      // 32 cp.async arrivals + 1 arrival carrying the byte count (+ 1 from the x-sum warp)
      ptx::mbar_init(full(s), kXWarp ? 34 : 33);
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
    // unit within the group), one for the activations (unit within the group).
    int64_t cgi = u0 / rg.UPG;
    int cj = (int)(u0 % rg.UPG), xj = cj;
    // L2 policies: the codes, scales and zeros are read once, so their lines
    // go first; x is read by every CTA that shares its k-range, so it stays.
    // The previous layer's partial sums, y and the next layer's x then stay
    // in L2 while the weights stream past them.
    const uint64_t pol_stream = ptx::l2_policy_evict_first();
    const uint64_t pol_x = ptx::l2_policy_evict_last();
    auto issue_codes = [&](int s) {  // codes, scales, zeros of the next unit into stage s; arms it
      const int R = (int)group_rows(cgi, rg.NB);
      const int64_t kb0 = (int64_t)cj * KU;
      const int ku = rg.KB - kb0 < KU ? (int)(rg.KB - kb0) : KU;
      const uint32_t st = sbase + s * L.bytes;
      const int64_t qw0 = unit_first_block(cgi, kb0, rg.KB, rg.NB) * kWordsPerBlock;
      const bool qok = AWQ_CHECK(in_range(qw0, (int64_t)ku * R * 256, (int64_t)K * N / 8) &&
                                     in_range(s * L.bytes + L.q, ku * R * 1024, dynamic_smem_bytes()),
                                 status);
      if (lane == 0)
        ptx::mbar_arrive_expect_tx(full(s),
                                   (uint32_t)((qok ? ku * R * 1024 : 0) + (kXWarp ? 0 : M * ku * kXRowBytes)));
      __syncwarp();
      if (lane == 0 && qok)
        ptx::bulk_g2s_hint(st + L.q, qweight + qw0, (uint32_t)(ku * R * 1024), full(s), pol_stream);
      const __half* srow = scales + kb0 * kGPK * N + kGroupBlocks * kRowsPerBlock * cgi;
      for (int p = lane; p < ku * kGPK * 16; p += 32) {  // ku * kGPK rows of 32 R bytes
        const int j = p >> 4, l = p & 15;
        if (l < 2 * R &&
            AWQ_CHECK(in_range(kb0 * kGPK * N + kGroupBlocks * kRowsPerBlock * cgi + (int64_t)j * N + 8 * l, 8,
                               (int64_t)(K / GS) * N) &&
                          in_range(s * L.bytes + L.s + j * kKbScaleBytes + 16 * l, 16, dynamic_smem_bytes()),
                      status))
          ptx::cp_async_16_hint(st + L.s + j * kKbScaleBytes + 16 * l, srow + (int64_t)j * N + 8 * l,
                                pol_stream);
      }
      const uint8_t* zrow = zeros + kb0 * kGPK * (N / 2) + 64 * cgi;
      for (int p = lane; p < ku * kGPK * 8; p += 32) {  // ku * kGPK rows of 8 R bytes
        const int j = p >> 3, l = p & 7;
        if (l < R &&
            AWQ_CHECK(in_range(kb0 * kGPK * (N / 2) + 64 * cgi + (int64_t)j * (N / 2) + 8 * l, 8,
                               (int64_t)(K / GS) * (N / 2)) &&
                          in_range(s * L.bytes + L.z + j * kKbZeroBytes + 8 * l, 8, dynamic_smem_bytes()),
                      status))
          ptx::cp_async_8_hint(st + L.z + j * kKbZeroBytes + 8 * l, zrow + (int64_t)j * (N / 2) + 8 * l,
                               pol_stream);
      }
      ptx::cp_async_arrive_noinc(full(s));
      if (++cj == rg.UPG) {
        cj = 0;
        ++cgi;
      }
    };
    auto issue_x = [&](int s) {  // activations of the next unit into stage s
      const int64_t kb0 = (int64_t)xj * KU;
      const int ku = rg.KB - kb0 < KU ? (int)(rg.KB - kb0) : KU;
      // with an x-prep warp x lands on its own barrier: that warp reads it first
      const uint32_t xb = kXWarp ? xland(s) : full(s);
      if (kXWarp) {
        if (lane == 0) ptx::mbar_arrive_expect_tx(xb, (uint32_t)(M * ku * kXRowBytes));
        __syncwarp();
      }
      if (lane < M) {
        // a copy that fails its check is replaced by an arrival with its byte count
        if (AWQ_CHECK(in_range((int64_t)lane * K + kb0 * kKPerBlock, (int64_t)ku * kKPerBlock, (int64_t)M * K) &&
                          in_range(s * L.bytes + L.x + L.xrow * lane, ku * kXRowBytes, dynamic_smem_bytes()),
                      status))
          ptx::bulk_g2s_hint(sbase + s * L.bytes + L.x + L.xrow * lane, x + (int64_t)lane * K + kb0 * kKPerBlock,
                             (uint32_t)(ku * kXRowBytes), xb, pol_x);
#ifdef AWQ_DEBUG
        else
          asm volatile("mbarrier.complete_tx.shared::cta.b64 [%0], %1;" ::"r"(xb), "r"((uint32_t)(ku * kXRowBytes))
                       : "memory");
#endif
      }
      if (++xj == rg.UPG) xj = 0;
    };
    // Only the first stage's codes go out before the previous grid has
    // finished (they do not depend on it). Every CTA asking for its whole ring
    // at once puts tens of MB in the memory queues, and the loads that the
    // previous layer's fixup and this layer's x wait for then queue behind
    // them: measured on B200, one stage ahead is 6-9% faster per decode layer
    // set than a full ring, and two stages sit in between.
    const int pro = n_units < NS ? n_units : NS;
    if (pro > 0) issue_codes(0);
    ptx::griddep_wait();
    if (pro > 0) issue_x(0);
    for (int i = 1; i < pro; ++i) {
      issue_codes(i);
      issue_x(i);
    }
    // unit i goes to stage s = i % NS as its use ph = (i / NS) & 1 and waits
    // for the consumers' release of the stage's previous use (parity ph ^ 1)
    int i = pro, s = pro % NS, ph = pro / NS;
    for (; i < n_units; ++i) {
      bool ok = true;
      if (lane == 0) ok = ptx::wait_bar(empty(s), ph ^ 1, abort_flag, status);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      issue_codes(s);
      issue_x(s);
      if (++s == NS) {
        s = 0;
        ph ^= 1;
      }
    }
    if (i < n_units && lane == 0)  // aborting: let the copies already issued land
      for (int j = (i > NS ? i - NS : 0); j < i; ++j) ptx::drain_bar(full(j % NS), (j / NS) & 1);
    __syncwarp();
    return;
  }

  if (warp == kWarpXsum) {
    // ------------------------------ x sums (M <= 8) ------------------------------
    // Per k-block j of the unit, lane (m, t4) = (lane / 4, lane % 4) adds token
    // m's x over k = 32 t4 .. 32 t4 + 31 into lo (k % 8 in {0, 1, 4, 5}) and hi
    // (k % 8 in {2, 3, 6, 7}) fp32 sums, then the lanes of one group (all four,
    // two or one) add theirs.
    if (kLoHi) {
      const int m = lane >> 2, t4 = lane & 3;
      int jj = (int)(u0 % rg.UPG), s = 0, ph = 0;
      for (int i = 0; i < n_units; ++i) {
        if (!ptx::wait_bar(xland(s), ph, abort_flag, status)) break;
        const uint8_t* st = smem + s * L.bytes;
        // All KU k-blocks of the stage at once (their latency chains overlap);
        // slots past a short last unit get values that are never read.
        float lo[KU], hi[KU];
#pragma unroll
        for (int j = 0; j < KU; ++j) {
          lo[j] = hi[j] = 0.f;
          if (m < M) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 v = *reinterpret_cast<const uint4*>(st + L.x + m * L.xrow + j * kXRowBytes + 64 * t4 +
                                                              16 * q);
              const float2 p0 = __half22float2(u32_as_h2(v.x)), p1 = __half22float2(u32_as_h2(v.y));
              const float2 p2 = __half22float2(u32_as_h2(v.z)), p3 = __half22float2(u32_as_h2(v.w));
              lo[j] += (p0.x + p0.y) + (p2.x + p2.y);
              hi[j] += (p1.x + p1.y) + (p3.x + p3.y);
            }
          }
        }
#pragma unroll
        for (int off = 1; off < GS / 32; off <<= 1)
#pragma unroll
          for (int j = 0; j < KU; ++j) {
            lo[j] += __shfl_xor_sync(0xffffffffu, lo[j], off);
            hi[j] += __shfl_xor_sync(0xffffffffu, hi[j], off);
          }
        if (t4 % (GS / 32) == 0 && m < M) {
          const int gk = t4 / (GS / 32);
#pragma unroll
          for (int j = 0; j < KU; ++j) {
            float* xs = reinterpret_cast<float*>(smem + s * L.bytes + L.xs + (j * kGPK + gk) * kKbXsBytes);
            xs[2 * m] = 1024.f * lo[j] + 64.f * hi[j];
            xs[2 * m + 1] = lo[j] + hi[j];
          }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(full(s));
        if (++jj == rg.UPG) jj = 0;
        if (++s == NS) {
          s = 0;
          ph ^= 1;
        }
      }
    }
    if constexpr (kInt) {
      // Integer path: lane (ch, hh) = (lane / 2, lane % 2) takes the 8-input
      // chunk ch of the k-block (inputs 8 ch .. 8 ch + 7, i.e. lane column
      // t = ch / 4, word 4 t + ch % 4 of every row) and, of it, the four
      // inputs {0, 4, 1, 5} (hh = 0, the lo bytes of the codes) or {2, 6, 3, 7}
      // (hh = 1, the hi bytes), in that order.
      const int ch = lane >> 1, hh = lane & 1, tq = ch >> 2, cq = ch & 3;
      const int tw = int_bfrag_tstride(M) / 4;       // words per lane column t
      int jj = (int)(u0 % rg.UPG), s = 0, ph = 0;
      for (int i = 0; i < n_units; ++i) {
        if (!ptx::wait_bar(xland(s), ph, abort_flag, status)) break;
        const uint8_t* st = smem + s * L.bytes;
        // All KU k-blocks of the stage at once (their latency chains overlap);
        // slots past a short last unit get values that are never read.
        for (int m = 0; m < M; ++m) {
          uint32_t pa[KU], pb[KU], amax[KU];
#pragma unroll
          for (int j = 0; j < KU; ++j) {
            const uint4 xv = *reinterpret_cast<const uint4*>(st + L.x + m * L.xrow + j * kXRowBytes + 16 * ch);
            pa[j] = hh ? xv.y : xv.x;  // inputs (0|2, 1|3)
            pb[j] = hh ? xv.w : xv.z;  // inputs (4|6, 5|7)
            // largest fp16 magnitude of the k-block (bit patterns order like the values)
            const uint32_t ma = pa[j] & 0x7FFF7FFFu, mb = pb[j] & 0x7FFF7FFFu;
            amax[j] = __reduce_max_sync(0xffffffffu, max(max(ma & 0xFFFFu, ma >> 16), max(mb & 0xFFFFu, mb >> 16)));
          }
          float cs[KU];
#pragma unroll
          for (int j = 0; j < KU; ++j) {
            const int eb = max((int)(amax[j] >> 10), 1);
            const float sc = __int_as_float((171 - eb) << 23);  // 2^(44 - eb), exact scaling
            const float2 fa = __half22float2(u32_as_h2(pa[j])), fb = __half22float2(u32_as_h2(pb[j]));
            // X in the k order {0, 4, 1, 5} / {2, 6, 3, 7}; digits as the bytes of v
            const uint32_t v0 = ((uint32_t)__float2int_rn(fa.x * sc) + 0x80808080u) ^ 0x80808080u;
            const uint32_t v1 = ((uint32_t)__float2int_rn(fb.x * sc) + 0x80808080u) ^ 0x80808080u;
            const uint32_t v2 = ((uint32_t)__float2int_rn(fa.y * sc) + 0x80808080u) ^ 0x80808080u;
            const uint32_t v3 = ((uint32_t)__float2int_rn(fb.y * sc) + 0x80808080u) ^ 0x80808080u;
            // 4 x 4 byte transpose: D_d = digit d of the four inputs
            const uint32_t t01l = __byte_perm(v0, v1, 0x5140), t01h = __byte_perm(v0, v1, 0x7362);
            const uint32_t t23l = __byte_perm(v2, v3, 0x5140), t23h = __byte_perm(v2, v3, 0x7362);
            uint32_t* b = reinterpret_cast<uint32_t*>(smem + s * L.bytes + L.xs + j * int_xs_bytes(M)) + tq * tw +
                          hh * 4 + cq + 4 * m * 8;  // column 4 m + d at + 8 d words
            b[0] = __byte_perm(t01l, t23l, 0x5410);
            b[8] = __byte_perm(t01l, t23l, 0x7632);
            b[16] = __byte_perm(t01h, t23h, 0x5410);
            b[24] = __byte_perm(t01h, t23h, 0x7632);
            cs[j] = (fa.x + fa.y) + (fb.x + fb.y);
          }
#pragma unroll
          for (int off = 16; off >= 1; off >>= 1)
#pragma unroll
            for (int j = 0; j < KU; ++j) cs[j] += __shfl_xor_sync(0xffffffffu, cs[j], off);
          // lane column t' = 2 m + e holds digit columns 4 m + 2 e, 4 m + 2 e + 1:
          // {2^(eb - 48 + 8 d0), sum x if d0 == 0, 2^(eb - 48 + 8 d0 + 8), 0}
          if (lane >> 1 == m) {
            const int d0 = 2 * (lane & 1);
#pragma unroll
            for (int j = 0; j < KU; ++j) {
              const int eb = max((int)(amax[j] >> 10), 1);
              float f0 = __int_as_float((eb + 79 + 8 * d0) << 23), f1 = __int_as_float((eb + 87 + 8 * d0) << 23);
              if (amax[j] >= 0x7C00u) f0 = f1 = __int_as_float(0x7FC00000);  // inf or NaN in x: y is NaN
              float4* coef = reinterpret_cast<float4*>(smem + s * L.bytes + L.xs + j * int_xs_bytes(M) +
                                                       4 * int_bfrag_tstride(M));
              coef[lane] = make_float4(f0, d0 == 0 ? cs[j] : 0.f, f1, 0.f);
            }
          }
        }
        if (M == 1 && (lane == 2 || lane == 3)) {
#pragma unroll
          for (int j = 0; j < KU; ++j)
            reinterpret_cast<float4*>(smem + s * L.bytes + L.xs + j * int_xs_bytes(M) + 4 * int_bfrag_tstride(M))[lane] =
                make_float4(0.f, 0.f, 0.f, 0.f);
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(full(s));
        if (++jj == rg.UPG) jj = 0;
        if (++s == NS) {
          s = 0;
          ph ^= 1;
        }
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
  auto covered = [&](int64_t g_) { return u0 <= g_ * rg.UPG && (g_ + 1) * rg.UPG <= u1; };
  auto write_y = [&](int64_t g_, const float (&v)[NT][4]) {
    const int64_t ra = (g_ * kGroupBlocks + cw) * kRowsPerBlock + g;  // rows ra (c = 0, 1), ra + 8 (c = 2, 3)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const int m = 8 * nt + 2 * t + (cc & 1);
        if (m < M && AWQ_CHECK(in_range((int64_t)m * N + ra + 8 * (cc >> 1), 1, (int64_t)M * N), status))
          y[(int64_t)m * N + ra + 8 * (cc >> 1)] = __float2half_rn(v[nt][cc]);
      }
  };
  // Partial slot of CTA `cta` for group g_: [cta][first/last group of cta][row block][16 rows][M].
  const int64_t first_gi = u0 / rg.UPG;  // this CTA's first group
  auto slot = [&](int64_t cta, int64_t g_) -> float* {
    const int which = (g_ == first_gi) ? 0 : 1;
    return partial + ((cta * 2 + which) * kGroupBlocks + cw) * kRowsPerBlock * M;
  };
  auto store_partial = [&](int64_t g_, const float (&v)[NT][4]) {
    float* mine = slot(c, g_);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        const int m = 8 * nt + 2 * t + (cc & 1);
        if (m < M && AWQ_CHECK(in_range(mine - partial + (g + 8 * (cc >> 1)) * M + m, 1, part_floats), status))
          mine[(g + 8 * (cc >> 1)) * M + m] = v[nt][cc];
      }
  };
  // Output of a finished group: fp16 y if this CTA saw all of its k-blocks,
  // else this CTA's fp32 partial sums, which the fixup kernel adds up.
  auto finish_group = [&](int64_t g_, const float (&v)[NT][4]) {
    if (cw >= group_rows(g_, rg.NB)) return;
    if constexpr (kInt) {
      // add the digit columns: lane t holds columns 2t, 2t+1 (token t / 2),
      // so after the pair sum lanes t = 0 and t = 2 hold tokens 0 and 1
      float r0 = v[0][0] + v[0][1], r1 = v[0][2] + v[0][3];
      r0 += __shfl_xor_sync(0xffffffffu, r0, 1);
      r1 += __shfl_xor_sync(0xffffffffu, r1, 1);
      const int m = t >> 1;
      if ((t & 1) || m >= M) return;
      const int64_t ra = (g_ * kGroupBlocks + cw) * kRowsPerBlock + g;
      if (covered(g_)) {
        if (AWQ_CHECK(in_range((int64_t)m * N + ra, 9, (int64_t)M * N), status)) {
          y[(int64_t)m * N + ra] = __float2half_rn(r0);
          y[(int64_t)m * N + ra + 8] = __float2half_rn(r1);
        }
      } else {
        float* mine = slot(c, g_);
        if (AWQ_CHECK(in_range(mine - partial + g * M + m, 8 * M + 1, part_floats), status)) {
          mine[g * M + m] = r0;
          mine[(g + 8) * M + m] = r1;
        }
      }
      return;
    }
    if (covered(g_))
      write_y(g_, v);
    else
      store_partial(g_, v);
  };

  // ---- integer path: one k-block (index j of the unit in stage st) ----
  auto kblock_int = [&](const uint8_t* st, int j, int R) {
    const uint8_t* blk = st + L.q + (j * R + cw) * 1024;
    const uint4 wa = *reinterpret_cast<const uint4*>(blk + g * 64 + 16 * t);
    const uint4 wb = *reinterpret_cast<const uint4*>(blk + (g + 8) * 64 + 16 * t);
    const uint8_t* xs = st + L.xs + j * int_xs_bytes(M);
    // B fragments of lane (g, t): digit column g, lane column t; zero past the tokens
    uint4 xb0 = make_uint4(0, 0, 0, 0), xb1 = make_uint4(0, 0, 0, 0);
    if (g < 4 * M) {
      const uint8_t* bf = xs + t * int_bfrag_tstride(M) + g * 32;
      xb0 = *reinterpret_cast<const uint4*>(bf);
      xb1 = *reinterpret_cast<const uint4*>(bf + 16);
    }
    const float4 cf = *reinterpret_cast<const float4*>(xs + 4 * int_bfrag_tstride(M) + 16 * t);
    const uint16_t* sc = reinterpret_cast<const uint16_t*>(st + L.s + j * kKbScaleBytes) + cw * kRowsPerBlock;
    const uint8_t* zr = st + L.z + j * kKbZeroBytes + cw * (kRowsPerBlock / 2);
    const float sr[2] = {pos_half_bits_to_float(sc[g]), pos_half_bits_to_float(sc[g + 8])};
    const uint32_t za = (zr[g >> 1] >> (4 * (g & 1))) & 0xF, zb = (zr[(g + 8) >> 1] >> (4 * (g & 1))) & 0xF;
    const float zf[2] = {__uint_as_float(0x4B000000u | za) - 8388608.f,  // exact (float)z
                         __uint_as_float(0x4B000000u | zb) - 8388608.f};
    constexpr uint32_t kLo = 0x0F0F0F0Fu, kHi = 0xF0F0F0F0u;
    int acc_lo[4], acc_hi[4];
    imma_16832_first(acc_lo, wa.x & kLo, wb.x & kLo, wa.y & kLo, wb.y & kLo, xb0.x, xb0.y);
    imma_16832_first(acc_hi, wa.x & kHi, wb.x & kHi, wa.y & kHi, wb.y & kHi, xb1.x, xb1.y);
    imma_16832(acc_lo, wa.z & kLo, wb.z & kLo, wa.w & kLo, wb.w & kLo, xb0.z, xb0.w);
    imma_16832(acc_hi, wa.z & kHi, wb.z & kHi, wa.w & kHi, wb.w & kHi, xb1.z, xb1.w);
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const float f = (cc & 1) ? cf.z : cf.x, cx = (cc & 1) ? cf.w : cf.y;
      const float v = __int2float_rn(acc_lo[cc] * 16 + acc_hi[cc]);  // exact: |.| < 2^22
      yacc[0][cc] = fmaf(sr[cc >> 1], fmaf(f, v, -zf[cc >> 1] * cx), yacc[0][cc]);
    }
  };

  // ---- one k-block (index j of the unit in stage st) of this warp's row block ----
  // kb_issue loads the k-block, issues its MMAs into `acc` and keeps in `ks`
  // what the epilogue needs besides the MMA results; kb_finish adds the
  // k-block to yacc. (Finishing a k-block only after the next one's MMAs were
  // issued measured no faster on B200.)
  constexpr int kC = Chains<NT, GS>::value;
  using Acc = std::conditional_t<kLoHi, float[LoHi<GS>::kAcc][4], float[kC][NT][4]>;
  struct KState {
    float s[kGPK][2];     // scales of rows g, g + 8 per group of the k-block
    float corr[kGPK][4];  // lo/hi path: C + z X of slot cc (rows g / g+8, tokens 2t / 2t+1)
  };
  auto kb_issue = [&](const uint8_t* st, int j, int R, Acc& acc, KState& ks) {
    const uint8_t* blk = st + L.q + (j * R + cw) * 1024;
    const uint4 wa = *reinterpret_cast<const uint4*>(blk + g * 64 + 16 * t);
    const uint4 wb = *reinterpret_cast<const uint4*>(blk + (g + 8) * 64 + 16 * t);
    uint32_t za[kGPK], zb[kGPK];
#pragma unroll
    for (int gk = 0; gk < kGPK; ++gk) {
      const uint16_t* sc =
          reinterpret_cast<const uint16_t*>(st + L.s + (j * kGPK + gk) * kKbScaleBytes) + cw * kRowsPerBlock;
      ks.s[gk][0] = pos_half_bits_to_float(sc[g]);
      ks.s[gk][1] = pos_half_bits_to_float(sc[g + 8]);
      const uint8_t* zr = st + L.z + (j * kGPK + gk) * kKbZeroBytes + cw * (kRowsPerBlock / 2);
      za[gk] = (zr[g >> 1] >> (4 * (g & 1))) & 0xF;
      zb[gk] = (zr[(g + 8) >> 1] >> (4 * (g & 1))) & 0xF;
    }
    // B fragment q of lane t: the token's 8 inputs in word 4t + q
    uint4 xf[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int m = 8 * nt + g;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        xf[nt][q] = m < M ? *reinterpret_cast<const uint4*>(st + L.x + m * L.xrow + j * kXRowBytes + Grp<GS>::x_off(t, q))
                          : make_uint4(0, 0, 0, 0);
    }
    if constexpr (kLoHi) {
      block_mma_lohi<GS>(acc, wa, wb, xf[0]);
#pragma unroll
      for (int gk = 0; gk < kGPK; ++gk) {
        // C and X of tokens 2t and 2t + 1 over group gk
        const float4 cx = *reinterpret_cast<const float4*>(st + L.xs + (j * kGPK + gk) * kKbXsBytes + 16 * t);
        const float zf[2] = {__uint_as_float(0x4B000000u | za[gk]) - 8388608.f,  // exact (float)z
                             __uint_as_float(0x4B000000u | zb[gk]) - 8388608.f};
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          if (kM1 && (cc & 1)) continue;  // slots of token 1
          const float Cm = (cc & 1) ? cx.z : cx.x, Xm = (cc & 1) ? cx.w : cx.y;
          ks.corr[gk][cc] = fmaf(zf[cc >> 1], Xm, Cm);
        }
      }
    } else {
      block_mma<NT, GS>(acc, wa, wb, za, zb, xf);
    }
  };
  auto kb_finish = [&](const Acc& acc, const KState& ks) {
    if constexpr (kLoHi) {
      // y += s (acc - (C + z X)), per group
#pragma unroll
      for (int gk = 0; gk < kGPK; ++gk)
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          if (kM1 && (cc & 1)) continue;
          const float a = GS == 128 ? acc[0][cc] + acc[1][cc] : acc[gk][cc];
          yacc[0][cc] = fmaf(ks.s[gk][cc >> 1], a - ks.corr[gk][cc], yacc[0][cc]);
        }
    } else {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          if (GS == 128) {
            float v = acc[0][nt][cc];
#pragma unroll
            for (int ch = 1; ch < kC; ++ch) v += acc[ch][nt][cc];
            yacc[nt][cc] = fmaf(ks.s[0][cc >> 1], v, yacc[nt][cc]);
          } else {
#pragma unroll
            for (int gk = 0; gk < kGPK; ++gk) yacc[nt][cc] = fmaf(ks.s[gk][cc >> 1], acc[gk][nt][cc], yacc[nt][cc]);
          }
        }
    }
  };

  auto kblock = [&](const uint8_t* st, int j, int R) {
    if constexpr (kInt) {
      kblock_int(st, j, R);
    } else {
      Acc acc;
      KState ks;
      kb_issue(st, j, R, acc, ks);
      kb_finish(acc, ks);
    }
  };

  bool ok = true;
  int64_t gi = u0 / rg.UPG;
  int jj = (int)(u0 % rg.UPG), s = 0, ph = 0, R = 0;
  for (int i = 0; i < n_units; ++i, ++jj) {
    if (jj == rg.UPG) {
      jj = 0;
      ++gi;
    }
    if (gi != cur_gi) {
      if (cur_gi >= 0) finish_group(cur_gi, yacc);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) yacc[nt][cc] = 0.f;
      cur_gi = gi;
      R = (int)group_rows(gi, rg.NB);
    }
    if (!ptx::wait_bar(full(s), ph, abort_flag, status)) {
      ok = false;
      break;
    }
    if (cw < R) {
      const uint8_t* st = smem + s * L.bytes;
      const int64_t kb0 = (int64_t)jj * KU;
      const int ku = rg.KB - kb0 < KU ? (int)(rg.KB - kb0) : KU;
      if (!AWQ_CHECK(in_range(s * L.bytes + L.q, (ku * R) * 1024, dynamic_smem_bytes()) &&
                         in_range(s * L.bytes + L.x, M * L.xrow, dynamic_smem_bytes()),
                     status)) {
        // (debug build) a stage that fails its check is skipped
      } else if (ku == KU) {
        // no guard: for one token tile pairs of k-blocks can interleave (more
        // token tiles would run out of registers)
        constexpr int kUnroll = NT == 1 ? 2 : 1;
#pragma unroll kUnroll
        for (int j = 0; j < KU; ++j) kblock(st, j, R);
      } else {
#pragma unroll 1
        for (int j = 0; j < ku; ++j) kblock(st, j, R);
      }
    }
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(empty(s));
    if (++s == NS) {
      s = 0;
      ph ^= 1;
    }
  }
  if (ok && cur_gi >= 0) finish_group(cur_gi, yacc);
}

// Rows split between CTAs: one CTA per (group, token) (128 threads, thread =
// row), launched right after the GEMV in the same stream. It waits for the
// GEMV's writes (programmatic dependent launch), adds the contributors'
// partial slots in CTA order and writes fp16 y. Groups that one CTA covered
// exit. Every contributor but the first starts its range inside the group, so
// the group is its first one (slot 0); the first contributor holds the group
// in slot 0 only if its range starts exactly at the group's first unit.
// (At most 32 registers a thread: 128 x 32 is what two resident GEMV CTAs
// leave free on an SM, so fixup CTAs can be resident and waiting before the
// GEMV's CTAs exit.)
__global__ void __launch_bounds__(128, 16) gemv_fixup_kernel(const float* __restrict__ partial, __half* __restrict__ y,
                                                          int M, int K, int N, int KU, int P, int64_t part_floats,
                                                          uint32_t* status) {
  ptx::griddep_launch_dependents();
  const Range rg(K, N, KU, P);
  const int64_t gi = blockIdx.x;
  const int64_t c_first = rg.cta_of(gi * rg.UPG), c_last = rg.cta_of((gi + 1) * rg.UPG - 1);
  if (c_first == c_last) return;
  const int rb = threadIdx.x >> 4, row = threadIdx.x & 15;
  if (rb >= group_rows(gi, rg.NB)) return;
  const int m = blockIdx.y;
  const int64_t slot_floats = (int64_t)kGroupBlocks * kRowsPerBlock * M;  // one slot
  const int64_t cta_floats = 2 * slot_floats;                             // one CTA's two slots
  const float* p = partial + c_first * cta_floats + ((int64_t)rb * kRowsPerBlock + row) * M + m;
  const int which_first = rg.first_unit(c_first) == gi * rg.UPG ? 0 : 1;
  const int n = (int)(c_last - c_first);  // contributors after the first
  ptx::griddep_wait();
  if (!AWQ_CHECK(in_range(p - partial + which_first * slot_floats, 1, part_floats) &&
                     in_range(p - partial + (int64_t)n * cta_floats, 1, part_floats) &&
                     in_range((int64_t)m * N + gi * kGroupBlocks * kRowsPerBlock + threadIdx.x, 1, (int64_t)M * N),
                 status))
    return;
  float v = __ldcg(p + which_first * slot_floats);
  for (int q0 = 1; q0 <= n; q0 += 4) {
    float part[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) part[k] = q0 + k <= n ? __ldcg(p + (int64_t)(q0 + k) * cta_floats) : 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) v += part[k];
  }
  y[(int64_t)m * N + gi * kGroupBlocks * kRowsPerBlock + threadIdx.x] = __float2half_rn(v);
}

template <int NT, int KU, bool kM1, int GS, bool kInt>
cudaError_t launch_t(const __half* x, const uint32_t* qweight, const __half* scales, const uint8_t* zeros, __half* y,
                     int M, int K, int N, void* workspace, const GemvPlan& p, cudaStream_t stream) {
  static std::atomic<uint64_t> attr_set{0};  // one bit per device that has the attribute
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return cudaErrorInvalidDevice;
  if (!(attr_set.load(std::memory_order_acquire) >> dev & 1)) {
    cudaError_t e = cudaFuncSetAttribute(gemv_kernel<NT, KU, kM1, GS, kInt>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         NT == 4 ? kSmemPerCta1 : kSmemPerCta2);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(uint64_t(1) << dev, std::memory_order_acq_rel);
  }
  char* ws = static_cast<char*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  float* partial = reinterpret_cast<float*>(ws + p.partial_off);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.ctas);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = p.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int64_t part_floats = (int64_t)(p.ws_bytes - p.partial_off) / 4;
  cudaError_t e = cudaLaunchKernelEx(&cfg, gemv_kernel<NT, KU, kM1, GS, kInt>, x, qweight, scales, zeros, y, M, K, N,
                                     p.stages, partial, part_floats, status);
  if (e != cudaSuccess || !p.has_split) return e;
  cudaLaunchConfig_t fcfg = cfg;
  fcfg.gridDim = dim3((unsigned)p.groups, (unsigned)M);
  fcfg.blockDim = dim3(kGroupBlocks * kRowsPerBlock);
  fcfg.dynamicSmemBytes = 0;
  return cudaLaunchKernelEx(&fcfg, gemv_fixup_kernel, (const float*)partial, y, M, K, N, p.ku, p.ctas, part_floats,
                            status);
}

template <int NT, bool kM1, int GS, bool kInt = false>
cudaError_t launch_nt(const __half* x, const uint32_t* qweight, const __half* scales, const uint8_t* zeros,
                      __half* y, int M, int K, int N, void* workspace, const GemvPlan& p, cudaStream_t stream) {
  switch (p.ku) {
    case 1: return launch_t<NT, 1, kM1, GS, kInt>(x, qweight, scales, zeros, y, M, K, N, workspace, p, stream);
    case 2: return launch_t<NT, 2, kM1, GS, kInt>(x, qweight, scales, zeros, y, M, K, N, workspace, p, stream);
    case 4: return launch_t<NT, 4, kM1, GS, kInt>(x, qweight, scales, zeros, y, M, K, N, workspace, p, stream);
    default: return cudaErrorInvalidConfiguration;
  }
}

template <int GS>
cudaError_t launch_g(const __half* x, const uint32_t* qweight, const __half* scales, const uint8_t* zeros,
                     __half* y, int m, int k, int n, void* workspace, const GemvPlan& p, cudaStream_t stream) {
  if constexpr (GS == 128) {
    if (p.int_path) return launch_nt<1, false, GS, true>(x, qweight, scales, zeros, y, m, k, n, workspace, p, stream);
  }
  switch (p.nt) {
    case 1:
      return m == 1 ? launch_nt<1, true, GS>(x, qweight, scales, zeros, y, m, k, n, workspace, p, stream)
                    : launch_nt<1, false, GS>(x, qweight, scales, zeros, y, m, k, n, workspace, p, stream);
    case 2: return launch_nt<2, false, GS>(x, qweight, scales, zeros, y, m, k, n, workspace, p, stream);
    case 4: return launch_nt<4, false, GS>(x, qweight, scales, zeros, y, m, k, n, workspace, p, stream);
    default: return cudaErrorInvalidConfiguration;
  }
}

}  // namespace

// Unit size: the largest KU in {4, 2, 1} (at most K/128) that leaves room for
// kMinStages ring stages and still gives every SM a unit. Measured on B200
// (LLaMA-2-7B and -70B decode layers, M = 1 and 8), bigger units won even
// where they leave some CTAs idle: one 32 KiB copy per CTA streams faster
// than four 8 KiB ones.
constexpr int kMinStages = 3;

GemvPlan plan_gemv(int64_t M, int64_t K, int64_t N, int group, int sm_count) {
  GemvPlan p{};
  p.group = group;
  p.nt = M <= 8 ? 1 : (M <= 16 ? 2 : 4);
  p.int_path = M <= 2 && group == 128;
  const int64_t NB = N / kRowsPerBlock, KB = K / kKPerBlock;
  p.groups = (int)((NB + kGroupBlocks - 1) / kGroupBlocks);
  const int64_t per_sm = p.nt == 4 ? 1 : 2;  // resident CTAs per SM (shared memory and registers)
  const int budget = (p.nt == 4 ? kSmemPerCta1 : kSmemPerCta2) - 3 * kMaxStages * 8 - 16;
  const int64_t Mi = M < 1 ? 1 : M;
  for (int ku : {4, 2, 1}) {
    const int64_t U = p.groups * ((KB + ku - 1) / ku);
    const int stage = Stage(ku, (int)Mi, group, p.int_path).bytes;
    int stages = budget / stage;
    if (stages > kMaxStages) stages = kMaxStages;
    const bool last = ku == 1;
    if (!last && (ku > KB || stages < kMinStages || U < sm_count)) continue;
    p.ku = ku;
    p.stages = stages;
    p.smem_bytes = (size_t)stages * stage + 3 * kMaxStages * 8 + 16;
    p.ctas = (int)(U < per_sm * sm_count ? U : per_sm * sm_count);
    const Range rg(K, N, ku, p.ctas);
    p.has_split = false;  // does some CTA boundary fall inside a group?
    for (int64_t cc = 1; cc < p.ctas && !p.has_split; ++cc) p.has_split = rg.first_unit(cc) % rg.UPG != 0;
    break;
  }
  p.partial_off = kWsHeaderBytes;
  p.zero_bytes = kWsHeaderBytes;  // the status word starts at zero
  p.ws_bytes = p.partial_off + (size_t)p.ctas * 2 * kGroupBlocks * kRowsPerBlock * (size_t)M * 4;
  return p;
}

cudaError_t launch_gemv(const __half* x, const uint32_t* qweight, const __half* scales, const uint8_t* zeros,
                        __half* y, int64_t M, int64_t K, int64_t N, void* workspace, const GemvPlan& p,
                        cudaStream_t stream) {
  const int m = (int)M, k = (int)K, n = (int)N;
  switch (p.group) {
    case 128: return launch_g<128>(x, qweight, scales, zeros, y, m, k, n, workspace, p, stream);
    case 64: return launch_g<64>(x, qweight, scales, zeros, y, m, k, n, workspace, p, stream);
    case 32: return launch_g<32>(x, qweight, scales, zeros, y, m, k, n, workspace, p, stream);
    default: return cudaErrorInvalidConfiguration;
  }
}

}  // namespace awq
