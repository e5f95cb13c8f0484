// Internal declarations shared by the CUDA sources of libawq_b200.so.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "awq.h"

namespace awq {

// Fixed tiling of the packed weight: a block is 16 output channels x 128
// input channels = 16 rows x 16 words (1 KiB).
constexpr int kRowsPerBlock = 16;
constexpr int kKPerBlock = 128;
constexpr int kWordsPerRow = kKPerBlock / 8;   // 16
constexpr int kWordsPerBlock = kRowsPerBlock * kWordsPerRow;  // 256

// Workspace layout (bytes):
//   [0, 256)                   header: uint32 status word at offset 0
//   [256, 256 + counters)      split-K arrival counters (uint32, rounded to 256 B)
//   [.., + S*M*N*4)            split-K fp32 partial sums, slot-major [S][M][N]
constexpr size_t kWsHeaderBytes = 256;

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Record the first device-side error in the status word (later ones are dropped).
__device__ __forceinline__ void record_status(uint32_t* status, uint32_t code) {
  if (status) atomicCAS(status, 0u, code);
}

// Per-device facts gathered once.
struct DeviceInfo {
  int device = -1;
  int sm_count = 148;
  int cc_major = 0, cc_minor = 0;
  size_t smem_optin = 0;
};
const DeviceInfo& device_info();   // current device

// GEMV launch plan (shared by awq_workspace_bytes and the launcher).
struct GemvPlan {
  int nt;      // token tiles of 8 (1, 2 or 4)
  int rb;      // row blocks (16 output channels each) per CTA
  int splits;  // split-K factor
  int ctas_n;  // CTAs along N = ceil(N/16 / rb)
  size_t ws_bytes;
};
GemvPlan plan_gemv(int64_t M, int64_t K, int64_t N, int sm_count);

// Launchers (argument checks are done by the ABI layer).
cudaError_t launch_pack(const __half* w, int64_t K, int64_t N, uint32_t* qweight, __half* scales, uint8_t* zeros,
                        uint32_t* status, cudaStream_t stream);
cudaError_t launch_dequant(const uint32_t* qweight, const __half* scales, const uint8_t* zeros, int64_t K,
                           int64_t N, __half* w_out, cudaStream_t stream);
cudaError_t launch_gemv(const __half* x, const uint32_t* qweight, const __half* scales, const uint8_t* zeros,
                        __half* y, int64_t M, int64_t K, int64_t N, void* workspace, const GemvPlan& plan,
                        cudaStream_t stream);
cudaError_t launch_gemm(const __half* x, const uint32_t* qweight, const __half* scales, const uint8_t* zeros,
                        __half* y, int64_t M, int64_t K, int64_t N, uint32_t* status, cudaStream_t stream);

}  // namespace awq
