// awq_w4a16_gemv_no_alloc: the decode GEMV for callers that cannot allocate
// device memory.
//
// Some callers cannot call cudaMalloc or any other allocator: code that runs
// inside a custom memory pool it must not grow, plug-ins loaded into a host
// process that owns all device allocations, or real-time paths where an
// allocation may block on the driver. awq_w4a16_gemv needs a caller-provided
// workspace for its status word and, when its plan splits output rows
// between CTAs, their partial sums; this entry point instead uses a fixed
// scratch array that lives in the library itself (a file-scope __device__
// array, one instance per GPU that loads the library, held until the process
// exits), so the caller passes only its inputs and outputs.
//
// Host code cannot use the array's name as a device address (on the host the
// symbol is only a stand-in). The first call on each device, with that device
// current, looks the address up with cudaGetSymbolAddress and caches it; make
// that first call before any stream capture. A lookup that fails is not
// cached: the error is cleared and the next call tries again. Calls share the
// array: two calls that can overlap on the GPU (different streams, or
// different host threads on one stream without ordering) race on it. Each
// call clears the status word before its kernels run;
// awq_get_status_no_alloc reads it back.
#include <mutex>

#include "awq_internal.cuh"

namespace awq {
namespace {

constexpr size_t kScratchBytes = AWQ_GEMV_NO_ALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mutex;

// Device address of this device's scratch array (looked up once per device;
// a failed lookup is retried by the next call).
cudaError_t scratch_for_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || !p) {
      cudaGetLastError();  // do not leave the lookup's error pending
      return e != cudaSuccess ? e : cudaErrorInvalidSymbol;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool overlap(const void* a, size_t an, const void* b, size_t bn) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return an && bn && a0 < b0 + bn && b0 < a0 + an;
}

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
  // y may not overlap an input (the same rule as awq_w4a16_gemv)
  const size_t ybytes = (size_t)M * N * 2, ng = (size_t)(K / group);
  if (overlap(y, ybytes, x, (size_t)M * K * 2) || overlap(y, ybytes, qweight, (size_t)K * N / 2) ||
      overlap(y, ybytes, scales, ng * N * 2) || overlap(y, ybytes, zeros, ng * N / 2))
    return AWQ_ERR_INVALID_ARG;
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

extern "C" awq_status awq_get_status_no_alloc(void* stream) {
  using namespace awq;
  void* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) return AWQ_ERR_CUDA;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return AWQ_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, scratch, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return AWQ_ERR_CUDA;
  if (word != 0 && cudaMemset(scratch, 0, sizeof(word)) != cudaSuccess) return AWQ_ERR_CUDA;
  return static_cast<awq_status>(word);
}
