// Decode-stage W4A16 GEMV (awq_w4a16_gemv), 1 <= M <= 32.
//
// TinyChat README, "Speed Benchmarks": the generation stage runs one token
// (or a few) per step through 4-bit-weight linear layers, so each layer is a
// GEMV that must stream its packed weights from HBM exactly once.
//
// Work split. The packed weight is a grid of 1 KiB blocks (16 output channels
// x 128 input channels). A CTA of 4 warps owns RB consecutive row blocks and
// one of `splits` contiguous ranges of k-blocks; its warps take k-blocks
// round-robin, so at any moment the CTA streams RB x 4 adjacent KiB.
//
// Per k-block a warp holds, in registers:
//   - the activations: lane (g, t) loads x[m = 8*nt + g][128*kb + 32t .. +31]
//     (four 16-byte loads per 8-token tile),
//   - for each row block, two 16-byte weight loads: row g and row g + 8,
//     words 4t .. 4t+3 (k = 32t .. 32t+31 of the block).
// The 4-bit codes are turned into fp16 (q - z) in registers with the
// exponent trick: (word & 0x000F000F) | 0x64006400 is the half2
// (1024 + q_a, 1024 + q_b) exactly, and the 0x00F000F0 mask gives
// (1024 + 16 q); subtracting 1024 + z (or scaling by 1/16 and subtracting
// 64 + z) leaves the exact small integer q - z. Those are the A fragments of
// mma.sync m16n8k16 (A = 16 weight rows x 16 k, B = 16 k x 8 tokens); since the
// MMA sums over k, any permutation of k applied to both A and B is allowed,
// and this kernel pairs the k that one lane loads (32t + 8j + 0..3 for MMA
// 2j, + 4..7 for MMA 2j+1) with the fragment slots that lane owns.
// Each k-block is one quantization group, so the fp32 MMA result of a block
// is sum_k x (q - z); multiplying it by the group's fp32 scale and adding it
// to the running sum gives y in fp32 without ever rounding a weight.
//
// Split-K: with splits > 1 each CTA writes its fp32 partial tile to a
// workspace slot; the last CTA of a row-block group to arrive (atomic
// counter) adds the slots in slot order, writes fp16 y and resets the
// counter, so the result is deterministic and the workspace stays reusable.
#include "awq_internal.cuh"

namespace awq {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));  // (a & b) | c
  return d;
}

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ld_v4(const void* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

struct BlockOperands {
  uint4 wa, wb;     // row g and row g + 8, words 4t .. 4t+3
  float sa, sb;     // scales of those rows
  uint32_t za, zb;  // zero points
};

__device__ __forceinline__ void load_block(BlockOperands& o, const uint32_t* __restrict__ qweight,
                                           const __half* __restrict__ scales, const uint8_t* __restrict__ zeros,
                                           int64_t nb, int kb, int KB, int N, int g, int t) {
  const uint32_t* blk = qweight + ((int64_t)nb * KB + kb) * kWordsPerBlock;
  o.wa = ld_stream_v4(blk + g * kWordsPerRow + 4 * t);
  o.wb = ld_stream_v4(blk + (g + 8) * kWordsPerRow + 4 * t);
  const int64_t na = nb * kRowsPerBlock + g;
  const __half* srow = scales + (int64_t)kb * N;
  o.sa = __half2float(srow[na]);
  o.sb = __half2float(srow[na + 8]);
  const uint8_t* zrow = zeros + (int64_t)kb * (N / 2);
  const int sh = 4 * (int)(na & 1);
  o.za = (zrow[na >> 1] >> sh) & 0xF;
  o.zb = (zrow[(na + 8) >> 1] >> sh) & 0xF;
}

template <int NT>
__device__ __forceinline__ void load_x(uint4 (&xf)[NT][4], const __half* __restrict__ x, int M, int K, int kb,
                                       int g, int t) {
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int m = 8 * nt + g;
    if (m < M) {
      const __half* p = x + (int64_t)m * K + (int64_t)kb * kKPerBlock + 32 * t;
#pragma unroll
      for (int j = 0; j < 4; ++j) xf[nt][j] = ld_v4(p + 8 * j);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) xf[nt][j] = make_uint4(0, 0, 0, 0);
    }
  }
}

// acc[nt] += sum over the block's 128 k of (q - z) * x, for rows g, g+8.
template <int NT>
__device__ __forceinline__ void block_mma(float (&acc)[NT][4], const BlockOperands& o, const uint4 (&xf)[NT][4]) {
  const uint32_t kMaskLo = 0x000F000Fu, kMaskHi = 0x00F000F0u, kMagic = 0x64006400u;
  const __half2 zlo_a = __half2half2(__ushort_as_half((unsigned short)(0x6400u + o.za)));  // 1024 + z
  const __half2 zlo_b = __half2half2(__ushort_as_half((unsigned short)(0x6400u + o.zb)));
  const __half2 zhi_a = __half2half2(__float2half_rn(-64.0f - (float)o.za));              // -(64 + z)
  const __half2 zhi_b = __half2half2(__float2half_rn(-64.0f - (float)o.zb));
  const __half2 sixteenth = __half2half2(__float2half_rn(0.0625f));
  const uint32_t wa[4] = {o.wa.x, o.wa.y, o.wa.z, o.wa.w};
  const uint32_t wb[4] = {o.wb.x, o.wb.y, o.wb.z, o.wb.w};
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
        mma_16816(acc[nt], a0, a1, a2, a3, b0, b1);
      }
      a >>= 8;
      b >>= 8;
    }
  }
}

template <int NT, int RB>
__global__ void __launch_bounds__(kThreads) gemv_kernel(const __half* __restrict__ x,
                                                        const uint32_t* __restrict__ qweight,
                                                        const __half* __restrict__ scales,
                                                        const uint8_t* __restrict__ zeros, __half* __restrict__ y,
                                                        int M, int K, int N, int splits, float* __restrict__ partial,
                                                        uint32_t* __restrict__ counters) {
  __shared__ float red[kWarps][RB][kRowsPerBlock][8 * NT];
  __shared__ int s_last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int KB = K / kKPerBlock, NB = N / kRowsPerBlock;
  const int nb0 = blockIdx.x * RB;
  const int sp = blockIdx.y;
  const int kb_begin = (int)((int64_t)KB * sp / splits);
  const int kb_end = (int)((int64_t)KB * (sp + 1) / splits);

  float yacc[RB][NT][4];
#pragma unroll
  for (int r = 0; r < RB; ++r)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int c = 0; c < 4; ++c) yacc[r][nt][c] = 0.f;

  int kb = kb_begin + warp;
  BlockOperands cur[RB], nxt[RB];
  uint4 xcur[NT][4], xnxt[NT][4];
  if (kb < kb_end) {
    load_x<NT>(xcur, x, M, K, kb, g, t);
#pragma unroll
    for (int r = 0; r < RB; ++r)
      if (nb0 + r < NB) load_block(cur[r], qweight, scales, zeros, nb0 + r, kb, KB, N, g, t);
  }
  for (; kb < kb_end; kb += kWarps) {
    const int kn = kb + kWarps;
    if (kn < kb_end) {  // prefetch the next k-block of this warp
      load_x<NT>(xnxt, x, M, K, kn, g, t);
#pragma unroll
      for (int r = 0; r < RB; ++r)
        if (nb0 + r < NB) load_block(nxt[r], qweight, scales, zeros, nb0 + r, kn, KB, N, g, t);
    }
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      if (nb0 + r < NB) {
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[nt][c] = 0.f;
        block_mma<NT>(acc, cur[r], xcur);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          yacc[r][nt][0] += cur[r].sa * acc[nt][0];
          yacc[r][nt][1] += cur[r].sa * acc[nt][1];
          yacc[r][nt][2] += cur[r].sb * acc[nt][2];
          yacc[r][nt][3] += cur[r].sb * acc[nt][3];
        }
      }
    }
    if (kn < kb_end) {
#pragma unroll
      for (int r = 0; r < RB; ++r) cur[r] = nxt[r];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j) xcur[nt][j] = xnxt[nt][j];
    }
  }

  // Cross-warp reduction. Accumulator c of tile nt covers weight row
  // g + 8*(c >> 1) and token 8*nt + 2t + (c & 1).
#pragma unroll
  for (int r = 0; r < RB; ++r)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int c = 0; c < 4; ++c) red[warp][r][g + 8 * (c >> 1)][8 * nt + 2 * t + (c & 1)] = yacc[r][nt][c];
  __syncthreads();

  const int outs = RB * kRowsPerBlock * M;  // (r, row, m) with m < M
  for (int o = threadIdx.x; o < outs; o += kThreads) {
    const int m = o % M;
    const int row = (o / M) % kRowsPerBlock;
    const int r = o / (M * kRowsPerBlock);
    const int nb = nb0 + r;
    if (nb >= NB) continue;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) v += red[w][r][row][m];
    const int64_t n = (int64_t)nb * kRowsPerBlock + row;
    if (splits == 1)
      y[(int64_t)m * N + n] = __float2half_rn(v);
    else
      partial[((int64_t)sp * M + m) * N + n] = v;
  }
  if (splits == 1) return;

  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t prev = atomicAdd(&counters[blockIdx.x], 1u);
    s_last = (prev == (uint32_t)(splits - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int o = threadIdx.x; o < outs; o += kThreads) {
    const int m = o % M;
    const int row = (o / M) % kRowsPerBlock;
    const int r = o / (M * kRowsPerBlock);
    const int nb = nb0 + r;
    if (nb >= NB) continue;
    const int64_t n = (int64_t)nb * kRowsPerBlock + row;
    float v = 0.f;
    for (int s = 0; s < splits; ++s) v += __ldcg(partial + ((int64_t)s * M + m) * N + n);
    y[(int64_t)m * N + n] = __float2half_rn(v);
  }
  if (threadIdx.x == 0) counters[blockIdx.x] = 0u;
}

template <int NT, int RB>
cudaError_t launch_t(const __half* x, const uint32_t* qweight, const __half* scales, const uint8_t* zeros,
                     __half* y, int M, int K, int N, void* workspace, const GemvPlan& p, cudaStream_t stream) {
  char* ws = static_cast<char*>(workspace);
  uint32_t* counters = reinterpret_cast<uint32_t*>(ws + kWsHeaderBytes);
  float* partial = reinterpret_cast<float*>(ws + kWsHeaderBytes + round_up((size_t)p.ctas_n * 4, 256));
  dim3 grid((unsigned)p.ctas_n, (unsigned)p.splits);
  gemv_kernel<NT, RB><<<grid, kThreads, 0, stream>>>(x, qweight, scales, zeros, y, M, K, N, p.splits, partial,
                                                      counters);
  return cudaGetLastError();
}

}  // namespace

GemvPlan plan_gemv(int64_t M, int64_t K, int64_t N, int sm_count) {
  GemvPlan p{};
  p.nt = M <= 8 ? 1 : (M <= 16 ? 2 : 4);
  const int64_t NB = N / kRowsPerBlock, KB = K / kKPerBlock;
  int rb = 4 / p.nt;
  while (rb > 1 && (NB + rb - 1) / rb < 2 * (int64_t)sm_count) rb /= 2;
  p.rb = rb;
  p.ctas_n = (int)((NB + rb - 1) / rb);
  const int64_t target = 4 * (int64_t)sm_count;
  int64_t s = (target + p.ctas_n - 1) / p.ctas_n;
  int64_t smax = KB / 8 > 1 ? KB / 8 : 1;
  if (s > smax) s = smax;
  if (s < 1) s = 1;
  p.splits = (int)s;
  p.ws_bytes = kWsHeaderBytes + round_up((size_t)p.ctas_n * 4, 256) +
               (p.splits > 1 ? (size_t)p.splits * (size_t)M * (size_t)N * 4 : 0);
  return p;
}

cudaError_t launch_gemv(const __half* x, const uint32_t* qweight, const __half* scales, const uint8_t* zeros,
                        __half* y, int64_t M, int64_t K, int64_t N, void* workspace, const GemvPlan& p,
                        cudaStream_t stream) {
  const int m = (int)M, k = (int)K, n = (int)N;
  switch (p.nt * 10 + p.rb) {
    case 11: return launch_t<1, 1>(x, qweight, scales, zeros, y, m, k, n, workspace, p, stream);
    case 12: return launch_t<1, 2>(x, qweight, scales, zeros, y, m, k, n, workspace, p, stream);
    case 14: return launch_t<1, 4>(x, qweight, scales, zeros, y, m, k, n, workspace, p, stream);
    case 21: return launch_t<2, 1>(x, qweight, scales, zeros, y, m, k, n, workspace, p, stream);
    case 22: return launch_t<2, 2>(x, qweight, scales, zeros, y, m, k, n, workspace, p, stream);
    case 41: return launch_t<4, 1>(x, qweight, scales, zeros, y, m, k, n, workspace, p, stream);
    default: return cudaErrorInvalidConfiguration;
  }
}

}  // namespace awq
