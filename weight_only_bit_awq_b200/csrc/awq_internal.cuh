// Internal declarations shared by the CUDA sources of libawq_b200.so.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include "awq.h"

namespace awq {

// Fixed tiling of the packed weight: a block is 16 output channels x 128
// input channels = 16 rows x 16 words (1 KiB).
constexpr int kRowsPerBlock = 16;
constexpr int kKPerBlock = 128;
constexpr int kWordsPerRow = kKPerBlock / 8;   // 16
constexpr int kWordsPerBlock = kRowsPerBlock * kWordsPerRow;  // 256

// Packed blocks are grouped by 8 row blocks (128 output channels); a group
// holds R = min(8, NB - 8*gi) row blocks and is stored k-block-major, so the
// R blocks of one (group, k-block) unit are one contiguous run of R KiB.
constexpr int kGroupBlocks = 8;

__host__ __device__ __forceinline__ int64_t group_rows(int64_t gi, int64_t NB) {
  const int64_t r = NB - kGroupBlocks * gi;
  return r < kGroupBlocks ? r : kGroupBlocks;
}
// First block of unit (gi, kb).
__host__ __device__ __forceinline__ int64_t unit_first_block(int64_t gi, int64_t kb, int64_t KB, int64_t NB) {
  return kGroupBlocks * gi * KB + kb * group_rows(gi, NB);
}
// Block number of row block nb, k-block kb.
__host__ __device__ __forceinline__ int64_t block_index(int64_t nb, int64_t kb, int64_t KB, int64_t NB) {
  return unit_first_block(nb / kGroupBlocks, kb, KB, NB) + nb % kGroupBlocks;
}

// Workspace layout (bytes):
//   [0, 256)                   header: uint32 status word at offset 0
//   [partial_off, ws_bytes)    decode GEMV (M <= 32): fp32 partial sums of row
//                              blocks split between CTAs, [ctas][2][8][16][M];
//                              stream-K GEMM (M > 32): fp32 parts of tiles split
//                              between CTAs, [ctas][2][bn][128]
constexpr size_t kWsHeaderBytes = 256;

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Record the first device-side error in the status word (later ones are dropped).
__device__ __forceinline__ void record_status(uint32_t* status, uint32_t code) {
  if (status) atomicCAS(status, 0u, code);
}

// Bounds checks of the debug build (compiled with -DAWQ_DEBUG; build.py
// --debug writes libawq_b200_debug.so). A guarded global or shared access
// first checks that its whole range lies inside its buffer; a failed check
// records AWQ_ERR_BOUNDS in the status word and the access is skipped, so the
// kernel neither faults nor traps. In the normal build the checks are `true`
// and compile to nothing.
__host__ __device__ __forceinline__ constexpr bool in_range(int64_t off, int64_t len, int64_t size) {
  return off >= 0 && len >= 0 && off + len <= size;
}
#ifdef AWQ_DEBUG
__device__ __forceinline__ bool debug_check(bool ok, uint32_t* status) {
  if (!ok) record_status(status, AWQ_ERR_BOUNDS);
  return ok;
}
// Bytes of dynamic shared memory this CTA was launched with.
__device__ __forceinline__ uint32_t dynamic_smem_bytes() {
  uint32_t r;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(r));
  return r;
}
#define AWQ_CHECK(cond, status) ::awq::debug_check((cond), (status))
#else
#define AWQ_CHECK(cond, status) true
#endif

// Per-device facts gathered once.
struct DeviceInfo {
  int device = -1;
  int sm_count = 148;
  int cc_major = 0, cc_minor = 0;
  size_t smem_optin = 0;
};
const DeviceInfo& device_info();   // current device

// The driver's cuTensorMapEncodeTiled (looked up once; nullptr if missing).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// GEMV launch plan (shared by awq_workspace_bytes and the launcher).
struct GemvPlan {
  int group;            // quantization group size (128, 64 or 32)
  int nt;               // token tiles of 8 (1, 2 or 4)
  bool int_path;        // M <= 2, groups of 128: integer MMAs on the codes and x digits
  int ku;               // k-blocks per streamed unit
  int stages;           // depth of the shared-memory ring
  size_t smem_bytes;    // dynamic shared memory per CTA
  int ctas;             // persistent CTAs
  int groups;           // groups of 8 row blocks
  bool has_split;       // some group is split between CTAs (the fixup kernel runs)
  size_t partial_off;   // workspace offset of the split-row partial sums (bytes)
  size_t zero_bytes;    // bytes at the start of the workspace that must be zero at launch
  size_t ws_bytes;      // total workspace bytes
};
GemvPlan plan_gemv(int64_t M, int64_t K, int64_t N, int group, int sm_count);

// W4A16 GEMM schedule (shared by awq_workspace_bytes and the launcher).
struct GemmPlan {
  int bn;               // token tile (128 or 256)
  int tiles;            // tiles of 128 channels x bn tokens
  int gm;               // token tiles per block of the tile order
  int ctas;             // persistent CTAs (at most one per SM)
  int dp_tiles;         // the first dp_tiles tiles are computed whole, data-parallel
  bool stream_k;        // the other tiles' k-blocks are split over the CTAs; the fixup kernel runs
  bool pair;            // data-parallel at 256-token tiles on CTA pairs (gemm_pair_kernel)
  size_t partial_off;   // workspace offset of the split tiles' fp32 parts (bytes)
  size_t ws_bytes;      // total workspace bytes
};
GemmPlan plan_gemm(int64_t M, int64_t K, int64_t N, int sm_count);

// Launchers (argument checks are done by the ABI layer).
cudaError_t launch_pack(const __half* w, int64_t K, int64_t N, int group, uint32_t* qweight, __half* scales,
                        uint8_t* zeros, uint32_t* status, cudaStream_t stream);
cudaError_t launch_dequant(const uint32_t* qweight, const __half* scales, const uint8_t* zeros, int64_t K,
                           int64_t N, int group, __half* w_out, cudaStream_t stream);
cudaError_t launch_gemv(const __half* x, const uint32_t* qweight, const __half* scales, const uint8_t* zeros,
                        __half* y, int64_t M, int64_t K, int64_t N, void* workspace, const GemvPlan& plan,
                        cudaStream_t stream);
cudaError_t launch_gemm(const __half* x, const uint32_t* qweight, const __half* scales, const uint8_t* zeros,
                        __half* y, int64_t M, int64_t K, int64_t N, int group, const GemmPlan& plan,
                        void* workspace, cudaStream_t stream);

// W4A8-FP8 variant (gemm_fp8.cu).
cudaError_t launch_fp8_row_exponents(const __half* scales, int64_t K, int64_t N, int group, int8_t* e_out,
                                     cudaStream_t stream);
cudaError_t launch_fp8_quantize_x(const __half* x, int64_t M, int64_t K, uint8_t* x8, float* sx,
                                  cudaStream_t stream);
cudaError_t launch_dequant_fp8(const uint32_t* qweight, const __half* scales, const uint8_t* zeros,
                               const int8_t* row_exp, int64_t K, int64_t N, int group, uint8_t* w8_out,
                               cudaStream_t stream);
cudaError_t launch_gemm_fp8(const uint8_t* x8, const float* sx, const uint32_t* qweight, const __half* scales,
                            const uint8_t* zeros, const int8_t* row_exp, __half* y, int64_t M, int64_t K, int64_t N,
                            int group, uint32_t* status, cudaStream_t stream);

// Packed word order inside a row's 128-input block, for group size G (128, 64
// or 32): word w = 4t + j holds the eight inputs from k0(w) = G (j / J) +
// 8 (t J + j % J), J = G / 32 (for G = 128 simply 8w). The four words with the
// same j hold whole groups, group j / J of the block.
__host__ __device__ __forceinline__ constexpr int word_k0(int w, int G) {
  return G * ((w & 3) / (G / 32)) + 8 * ((w >> 2) * (G / 32) + (w & 3) % (G / 32));
}
__host__ __device__ __forceinline__ constexpr int word_of_k(int k, int G) {
  return 4 * (((k % G) / 8) / (G / 32)) + (k / G) * (G / 32) + ((k % G) / 8) % (G / 32);
}

}  // namespace awq
