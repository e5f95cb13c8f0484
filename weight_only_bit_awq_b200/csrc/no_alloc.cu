// awq_w4a16_gemv_no_alloc: the decode GEMV for callers that cannot allocate
// device memory.
//
// Some callers cannot call cudaMalloc or any other allocator: code that runs
// inside a custom memory pool it must not grow, plug-ins loaded into a host
// process that owns all device allocations, or real-time paths where an
// allocation may block on the driver. awq_w4a16_gemv needs a caller-provided
// workspace for its status word and the partial sums of rows split between
// CTAs; this entry
// point instead uses a fixed scratch array that lives in the library itself
// (a file-scope __device__ array, one instance per GPU that loads the
// library, held until the process exits), so the caller passes only its
// inputs and outputs.
//
// Host code cannot use the array's name as a device address (on the host the
// symbol is only a stand-in). The first call on each device, with that device
// current, looks the address up with cudaGetSymbolAddress and caches it; make
// that first call before any stream capture. Calls share the array: two
// calls that can overlap on the GPU (different streams, or different host
// threads on one stream without ordering) race on it. Each call clears the
// status word before its kernels run.
#include <mutex>

#include "awq_internal.cuh"

namespace awq {
namespace {

constexpr size_t kScratchBytes = AWQ_GEMV_NO_ALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];
std::once_flag g_scratch_once[kMaxDevices];

// Device address of this device's scratch array (looked up once per device).
cudaError_t scratch_for_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(g_scratch_once[dev], [dev] {
    void* p = nullptr;
    g_scratch_err[dev] = cudaGetSymbolAddress(&p, g_scratch);
    g_scratch_ptr[dev] = p;
  });
  if (g_scratch_err[dev] != cudaSuccess) return g_scratch_err[dev];
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace awq

extern "C" awq_status awq_w4a16_gemv_no_alloc(const void* x, const void* qweight, const void* scales,
                                              const void* zeros, void* y, int64_t M, int64_t K, int64_t N,
                                              int group, void* stream) {
  using namespace awq;
  if (M < 0 || K <= 0 || N <= 0) return AWQ_ERR_SHAPE;
  if (group != 128 && group != 64 && group != 32) return AWQ_ERR_UNSUPPORTED;
  if (K % kKPerBlock != 0 || N % kRowsPerBlock != 0) return AWQ_ERR_SHAPE;
  if (M > AWQ_GEMV_MAX_M) return AWQ_ERR_UNSUPPORTED;
  if ((M > 0 && (!x || !y)) || !qweight || !scales || !zeros) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros))
    return AWQ_ERR_ALIGNMENT;
  const size_t need = awq_workspace_bytes(M, K, N, group);
  if (need == 0) return AWQ_ERR_UNSUPPORTED;        // K or N above the library's limits
  if (need > kScratchBytes) return AWQ_ERR_WORKSPACE;  // these sizes need more scratch than the array holds
  if (M == 0) return AWQ_OK;
  const DeviceInfo& d = device_info();
  if (d.device < 0 || d.cc_major != 10) return AWQ_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) return AWQ_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const GemvPlan p = plan_gemv(M, K, N, group, d.sm_count);
  // The status word must start at zero; the partial sums are always written
  // before they are read.
  if (cudaMemsetAsync(scratch, 0, p.zero_bytes, s) != cudaSuccess) return AWQ_ERR_CUDA;
  cudaError_t e = launch_gemv(static_cast<const __half*>(x), static_cast<const uint32_t*>(qweight),
                              static_cast<const __half*>(scales), static_cast<const uint8_t*>(zeros),
                              static_cast<__half*>(y), M, K, N, scratch, p, s);
  return e == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}
