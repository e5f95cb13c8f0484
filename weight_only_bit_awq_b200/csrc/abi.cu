// C ABI entry points of libawq_b200.so (declared in include/awq.h): argument
// checks, workspace layout, dispatch between the GEMV and GEMM paths.
#include <mutex>

#include "awq_internal.cuh"
#include "sm100_ptx.cuh"

namespace awq {

namespace {
// One thread waits, through the kernels' bounded-wait helper, on an mbarrier
// phase that nothing will ever complete; the wait gives up after `limit_ns`
// and records AWQ_ERR_TIMEOUT in the status word.
__global__ void bounded_wait_probe_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t barrier;
  __shared__ uint32_t abort_flag;
  const uint32_t bar = ptx::smem_u32(&barrier);
  ptx::mbar_init(bar, 1);
  abort_flag = 0;
  ptx::fence_mbarrier_init();
  ptx::wait_bar(bar, 0, &abort_flag, status, limit_ns);
}
}  // namespace

namespace {
constexpr int kMaxDevices = 64;
DeviceInfo g_info[kMaxDevices];
std::once_flag g_once[kMaxDevices];

constexpr int64_t kMaxK = int64_t(1) << 22;
constexpr int64_t kMaxN = int64_t(1) << 22;
constexpr int64_t kMaxM = int64_t(1) << 24;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool overlap(const void* a, size_t an, const void* b, size_t bn) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return an && bn && a0 < b0 + bn && b0 < a0 + an;
}

awq_status check_kn(int64_t K, int64_t N, int group) {
  if (K <= 0 || N <= 0) return AWQ_ERR_SHAPE;
  if (group != 128 && group != 64 && group != 32) return AWQ_ERR_UNSUPPORTED;
  if (K % kKPerBlock != 0 || K % group != 0 || N % kRowsPerBlock != 0) return AWQ_ERR_SHAPE;
  if (K > kMaxK || N > kMaxN) return AWQ_ERR_UNSUPPORTED;
  return AWQ_OK;
}

awq_status check_device() {
  const DeviceInfo& d = device_info();
  if (d.device < 0 || d.cc_major != 10) return AWQ_ERR_UNSUPPORTED;
  return AWQ_OK;
}

struct LinearArgs {
  const void *x, *qweight, *scales, *zeros;
  void* y;
  int64_t M, K, N;
  int group;
  void* workspace;
  size_t ws_bytes;
};

awq_status check_linear(const LinearArgs& a) {
  if (a.M < 0) return AWQ_ERR_SHAPE;
  awq_status st = check_kn(a.K, a.N, a.group);
  if (st != AWQ_OK) return st;
  if (a.M > kMaxM) return AWQ_ERR_UNSUPPORTED;
  // x and y may be null for an empty batch (nothing is read or written).
  if ((a.M > 0 && (!a.x || !a.y)) || !a.qweight || !a.scales || !a.zeros || !a.workspace)
    return AWQ_ERR_INVALID_ARG;
  if (!aligned16(a.x) || !aligned16(a.qweight) || !aligned16(a.scales) || !aligned16(a.zeros) ||
      !aligned16(a.y) || !aligned16(a.workspace))
    return AWQ_ERR_ALIGNMENT;
  const size_t ybytes = (size_t)a.M * a.N * 2;
  const size_t ng = (size_t)(a.K / a.group);
  if (overlap(a.y, ybytes, a.x, (size_t)a.M * a.K * 2) || overlap(a.y, ybytes, a.qweight, (size_t)a.K * a.N / 2) ||
      overlap(a.y, ybytes, a.scales, ng * a.N * 2) || overlap(a.y, ybytes, a.zeros, ng * a.N / 2) ||
      overlap(a.y, ybytes, a.workspace, a.ws_bytes))
    return AWQ_ERR_INVALID_ARG;
  if (a.ws_bytes < awq_workspace_bytes(a.M, a.K, a.N, a.group)) return AWQ_ERR_WORKSPACE;
  return AWQ_OK;
}

inline uint32_t* status_word(void* ws) { return static_cast<uint32_t*>(ws); }

}  // namespace

const DeviceInfo& device_info() {
  static DeviceInfo none;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return none;
  }
  std::call_once(g_once[dev], [dev] {
    DeviceInfo& d = g_info[dev];
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess) d.sm_count = v;
    cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) == cudaSuccess) d.smem_optin = v;
    d.device = dev;
  });
  return g_info[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

}  // namespace awq

using namespace awq;

namespace {

int sm_count_or_default() {
  int dev = -1, n = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
      n > 0)
    return n;
  cudaGetLastError();
  return 148;
}

awq_status gemv_impl(const LinearArgs& a, cudaStream_t stream) {
  const GemvPlan p = plan_gemv(a.M, a.K, a.N, a.group, device_info().sm_count);
  cudaError_t e = launch_gemv(static_cast<const __half*>(a.x), static_cast<const uint32_t*>(a.qweight),
                              static_cast<const __half*>(a.scales), static_cast<const uint8_t*>(a.zeros),
                              static_cast<__half*>(a.y), a.M, a.K, a.N, a.workspace, p, stream);
  return e == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

awq_status gemm_impl(const LinearArgs& a, cudaStream_t stream) {
  const GemmPlan p = plan_gemm(a.M, a.K, a.N, device_info().sm_count);
  cudaError_t e = launch_gemm(static_cast<const __half*>(a.x), static_cast<const uint32_t*>(a.qweight),
                              static_cast<const __half*>(a.scales), static_cast<const uint8_t*>(a.zeros),
                              static_cast<__half*>(a.y), a.M, a.K, a.N, a.group, p, a.workspace, stream);
  return e == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

// Dispatch of awq_linear between the decode GEMV and the tensor-core GEMM,
// from measurements on B200 (CUDA graphs, rotating weights, LLaMA-3-8B and
// LLaMA-2-70B decode layers at M = 4 .. 64): the GEMV is faster on every layer
// up to M = 16; at M = 24 and 32 the GEMM is faster on layers with at least
// as many 128-channel tiles as SMs (gate_up: 54.6 against 76.4 us at M = 32
// on LLaMA-3-8B, 195.6 against 256.3 us on 70B) and slower on the narrower
// ones, which leave most SMs without a tile.
constexpr int kGemvAlwaysM = 16;

bool linear_uses_gemv(int64_t M, int64_t N, int sm_count) {
  return M <= kGemvAlwaysM || (M <= AWQ_GEMV_MAX_M && (N + 127) / 128 < sm_count);
}

}  // namespace

extern "C" {

awq_status awq_packed_size(int64_t K, int64_t N, int group, awq_packed_sizes* out) {
  if (!out) return AWQ_ERR_INVALID_ARG;
  awq_status st = check_kn(K, N, group);
  if (st != AWQ_OK) return st;
  out->qweight_bytes = (size_t)K * (size_t)N / 2;
  out->scales_bytes = (size_t)(K / group) * (size_t)N * 2;
  out->zeros_bytes = (size_t)(K / group) * (size_t)N / 2;
  return AWQ_OK;
}

size_t awq_workspace_bytes(int64_t M, int64_t K, int64_t N, int group) {
  if (M < 0 || check_kn(K, N, group) != AWQ_OK || M > kMaxM) return 0;
  size_t need = kWsHeaderBytes;
  if (M >= 1 && M <= AWQ_GEMV_MAX_M) {
    const GemvPlan p = plan_gemv(M, K, N, group, sm_count_or_default());
    if (p.ws_bytes > need) need = p.ws_bytes;
  } else if (M > AWQ_GEMV_MAX_M) {
    const GemmPlan p = plan_gemm(M, K, N, sm_count_or_default());
    if (p.ws_bytes > need) need = p.ws_bytes;
  }
  return need;
}

awq_status awq_workspace_init(void* workspace, size_t ws_bytes, void* stream) {
  if (!workspace || ws_bytes < kWsHeaderBytes) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return AWQ_ERR_ALIGNMENT;
  return cudaMemsetAsync(workspace, 0, ws_bytes, static_cast<cudaStream_t>(stream)) == cudaSuccess ? AWQ_OK
                                                                                                   : AWQ_ERR_CUDA;
}

awq_status awq_pack(const void* w, int64_t K, int64_t N, int group, void* qweight, void* scales, void* zeros,
                    void* workspace, size_t ws_bytes, void* stream) {
  awq_status st = check_kn(K, N, group);
  if (st != AWQ_OK) return st;
  if (!w || !qweight || !scales || !zeros || !workspace) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros) || !aligned16(workspace))
    return AWQ_ERR_ALIGNMENT;
  const size_t wb = (size_t)K * N * 2, ng = (size_t)(K / group);
  if (overlap(w, wb, qweight, (size_t)K * N / 2) || overlap(w, wb, scales, ng * N * 2) ||
      overlap(w, wb, zeros, ng * N / 2) || overlap(qweight, (size_t)K * N / 2, scales, ng * N * 2) ||
      overlap(qweight, (size_t)K * N / 2, zeros, ng * N / 2) || overlap(scales, ng * N * 2, zeros, ng * N / 2))
    return AWQ_ERR_INVALID_ARG;
  if (ws_bytes < kWsHeaderBytes) return AWQ_ERR_WORKSPACE;
  if ((st = check_device()) != AWQ_OK) return st;
  cudaError_t e = launch_pack(static_cast<const __half*>(w), K, N, group, static_cast<uint32_t*>(qweight),
                              static_cast<__half*>(scales), static_cast<uint8_t*>(zeros), status_word(workspace),
                              static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

awq_status awq_dequant(const void* qweight, const void* scales, const void* zeros, int64_t K, int64_t N, int group,
                       void* w_out, void* stream) {
  awq_status st = check_kn(K, N, group);
  if (st != AWQ_OK) return st;
  if (!w_out || !qweight || !scales || !zeros) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(w_out) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros)) return AWQ_ERR_ALIGNMENT;
  const size_t wb = (size_t)K * N * 2, ng = (size_t)(K / group);
  if (overlap(w_out, wb, qweight, (size_t)K * N / 2) || overlap(w_out, wb, scales, ng * N * 2) ||
      overlap(w_out, wb, zeros, ng * N / 2))
    return AWQ_ERR_INVALID_ARG;
  if ((st = check_device()) != AWQ_OK) return st;
  cudaError_t e = launch_dequant(static_cast<const uint32_t*>(qweight), static_cast<const __half*>(scales),
                                 static_cast<const uint8_t*>(zeros), K, N, group, static_cast<__half*>(w_out),
                                 static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

awq_status awq_w4a16_gemv(const void* x, const void* qweight, const void* scales, const void* zeros, void* y,
                          int64_t M, int64_t K, int64_t N, int group, void* workspace, size_t ws_bytes,
                          void* stream) {
  LinearArgs a{x, qweight, scales, zeros, y, M, K, N, group, workspace, ws_bytes};
  awq_status st = check_linear(a);
  if (st != AWQ_OK) return st;
  if (M > AWQ_GEMV_MAX_M) return AWQ_ERR_UNSUPPORTED;
  if (M == 0) return AWQ_OK;
  if ((st = check_device()) != AWQ_OK) return st;
  return gemv_impl(a, static_cast<cudaStream_t>(stream));
}

awq_status awq_w4a16_gemm(const void* x, const void* qweight, const void* scales, const void* zeros, void* y,
                          int64_t M, int64_t K, int64_t N, int group, void* workspace, size_t ws_bytes,
                          void* stream) {
  LinearArgs a{x, qweight, scales, zeros, y, M, K, N, group, workspace, ws_bytes};
  awq_status st = check_linear(a);
  if (st != AWQ_OK) return st;
  if (M == 0) return AWQ_OK;
  if ((st = check_device()) != AWQ_OK) return st;
  return gemm_impl(a, static_cast<cudaStream_t>(stream));
}

awq_status awq_linear(const void* x, const void* qweight, const void* scales, const void* zeros, void* y, int64_t M,
                      int64_t K, int64_t N, int group, void* workspace, size_t ws_bytes, void* stream) {
  LinearArgs a{x, qweight, scales, zeros, y, M, K, N, group, workspace, ws_bytes};
  awq_status st = check_linear(a);
  if (st != AWQ_OK) return st;
  if (M == 0) return AWQ_OK;
  if ((st = check_device()) != AWQ_OK) return st;
  if (linear_uses_gemv(M, N, device_info().sm_count)) return gemv_impl(a, static_cast<cudaStream_t>(stream));
  return gemm_impl(a, static_cast<cudaStream_t>(stream));
}

int awq_linear_gemv_limit(void) { return kGemvAlwaysM; }

awq_status awq_fp8_row_exponents(const void* scales, int64_t K, int64_t N, int group, void* e_out, void* stream) {
  awq_status st = check_kn(K, N, group);
  if (st != AWQ_OK) return st;
  if (!scales || !e_out) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(scales)) return AWQ_ERR_ALIGNMENT;
  if (overlap(e_out, (size_t)N, scales, (size_t)(K / group) * N * 2)) return AWQ_ERR_INVALID_ARG;
  if ((st = check_device()) != AWQ_OK) return st;
  cudaError_t e = launch_fp8_row_exponents(static_cast<const __half*>(scales), K, N, group,
                                           static_cast<int8_t*>(e_out), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

awq_status awq_fp8_quantize_x(const void* x, int64_t M, int64_t K, void* x8, void* sx, void* stream) {
  if (M < 0 || K <= 0) return AWQ_ERR_SHAPE;
  if (K % kKPerBlock != 0) return AWQ_ERR_SHAPE;
  if (K > kMaxK || M > kMaxM) return AWQ_ERR_UNSUPPORTED;
  if (M == 0) return AWQ_OK;
  if (!x || !x8 || !sx) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x8) || !aligned16(sx)) return AWQ_ERR_ALIGNMENT;
  const size_t xb = (size_t)M * K * 2, x8b = (size_t)M * K, sxb = (size_t)M * 4;
  if (overlap(x, xb, x8, x8b) || overlap(x, xb, sx, sxb) || overlap(x8, x8b, sx, sxb)) return AWQ_ERR_INVALID_ARG;
  awq_status st = check_device();
  if (st != AWQ_OK) return st;
  cudaError_t e = launch_fp8_quantize_x(static_cast<const __half*>(x), M, K, static_cast<uint8_t*>(x8),
                                        static_cast<float*>(sx), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

awq_status awq_dequant_fp8(const void* qweight, const void* scales, const void* zeros, const void* row_exp,
                           int64_t K, int64_t N, int group, void* w8_out, void* stream) {
  awq_status st = check_kn(K, N, group);
  if (st != AWQ_OK) return st;
  if (!w8_out || !qweight || !scales || !zeros || !row_exp) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(w8_out) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros)) return AWQ_ERR_ALIGNMENT;
  const size_t wb = (size_t)K * N, ng = (size_t)(K / group);
  if (overlap(w8_out, wb, qweight, (size_t)K * N / 2) || overlap(w8_out, wb, scales, ng * N * 2) ||
      overlap(w8_out, wb, zeros, ng * N / 2) || overlap(w8_out, wb, row_exp, (size_t)N))
    return AWQ_ERR_INVALID_ARG;
  if ((st = check_device()) != AWQ_OK) return st;
  cudaError_t e = launch_dequant_fp8(static_cast<const uint32_t*>(qweight), static_cast<const __half*>(scales),
                                     static_cast<const uint8_t*>(zeros), static_cast<const int8_t*>(row_exp), K, N,
                                     group, static_cast<uint8_t*>(w8_out), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

awq_status awq_w4a8_gemm(const void* x8, const void* sx, const void* qweight, const void* scales, const void* zeros,
                         const void* row_exp, void* y, int64_t M, int64_t K, int64_t N, int group, void* workspace,
                         size_t ws_bytes, void* stream) {
  if (M < 0) return AWQ_ERR_SHAPE;
  awq_status st = check_kn(K, N, group);
  if (st != AWQ_OK) return st;
  if (M > kMaxM) return AWQ_ERR_UNSUPPORTED;
  if ((M > 0 && (!x8 || !sx || !y)) || !qweight || !scales || !zeros || !row_exp || !workspace)
    return AWQ_ERR_INVALID_ARG;
  if (!aligned16(x8) || !aligned16(sx) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros) ||
      !aligned16(y) || !aligned16(workspace))
    return AWQ_ERR_ALIGNMENT;
  const size_t ybytes = (size_t)M * N * 2, ng = (size_t)(K / group);
  if (overlap(y, ybytes, x8, (size_t)M * K) || overlap(y, ybytes, sx, (size_t)M * 4) ||
      overlap(y, ybytes, qweight, (size_t)K * N / 2) || overlap(y, ybytes, scales, ng * N * 2) ||
      overlap(y, ybytes, zeros, ng * N / 2) || overlap(y, ybytes, row_exp, (size_t)N) ||
      overlap(y, ybytes, workspace, ws_bytes))
    return AWQ_ERR_INVALID_ARG;
  if (ws_bytes < kWsHeaderBytes) return AWQ_ERR_WORKSPACE;
  if (M == 0) return AWQ_OK;
  if ((st = check_device()) != AWQ_OK) return st;
  cudaError_t e = launch_gemm_fp8(static_cast<const uint8_t*>(x8), static_cast<const float*>(sx),
                                  static_cast<const uint32_t*>(qweight), static_cast<const __half*>(scales),
                                  static_cast<const uint8_t*>(zeros), static_cast<const int8_t*>(row_exp),
                                  static_cast<__half*>(y), M, K, N, group, status_word(workspace),
                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

int awq_linear_path(int64_t M, int64_t K, int64_t N, int group) {
  if (M <= 0 || M > kMaxM || check_kn(K, N, group) != AWQ_OK) return 0;
  const int sms = sm_count_or_default();
  if (linear_uses_gemv(M, N, sms)) return 1;
  return plan_gemm(M, K, N, sms).pair ? 3 : 2;
}

int awq_linear_launches(int64_t M, int64_t K, int64_t N, int group) {
  if (M <= 0 || M > kMaxM || check_kn(K, N, group) != AWQ_OK) return 0;
  const int sms = sm_count_or_default();
  if (!linear_uses_gemv(M, N, sms)) return plan_gemm(M, K, N, sms).stream_k ? 2 : 1;
  return plan_gemv(M, K, N, group, sms).has_split ? 2 : 1;
}

awq_status awq_check_bounded_wait(void* workspace, size_t ws_bytes, uint32_t limit_us, void* stream) {
  if (!workspace || limit_us == 0 || limit_us > 1000000) return AWQ_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return AWQ_ERR_ALIGNMENT;
  if (ws_bytes < kWsHeaderBytes) return AWQ_ERR_WORKSPACE;
  awq_status st = check_device();
  if (st != AWQ_OK) return st;
  bounded_wait_probe_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(status_word(workspace),
                                                                             (uint64_t)limit_us * 1000);
  return cudaGetLastError() == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}

awq_status awq_get_status(void* workspace, void* stream) {
  if (!workspace) return AWQ_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return AWQ_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return AWQ_ERR_CUDA;
  if (word != 0 && cudaMemset(workspace, 0, sizeof(word)) != cudaSuccess) return AWQ_ERR_CUDA;
  return static_cast<awq_status>(word);
}

const char* awq_status_string(awq_status status) {
  switch (status) {
    case AWQ_OK: return "AWQ_OK";
    case AWQ_ERR_INVALID_ARG: return "AWQ_ERR_INVALID_ARG: null pointer, overlapping buffers or bad workspace";
    case AWQ_ERR_SHAPE: return "AWQ_ERR_SHAPE: need M >= 0, K > 0, N > 0, K % 128 == 0, N % 16 == 0";
    case AWQ_ERR_ALIGNMENT: return "AWQ_ERR_ALIGNMENT: every pointer must be 16-byte aligned";
    case AWQ_ERR_WORKSPACE: return "AWQ_ERR_WORKSPACE: workspace smaller than awq_workspace_bytes()";
    case AWQ_ERR_UNSUPPORTED: return "AWQ_ERR_UNSUPPORTED: group not 32, 64 or 128, size above a limit, or no sm_100 device";
    case AWQ_ERR_CUDA: return "AWQ_ERR_CUDA: a CUDA call or kernel launch failed";
    case AWQ_ERR_TIMEOUT: return "AWQ_ERR_TIMEOUT: a bounded wait on the device expired";
    case AWQ_ERR_NONFINITE: return "AWQ_ERR_NONFINITE: awq_pack met an inf or NaN weight";
    case AWQ_ERR_BOUNDS: return "AWQ_ERR_BOUNDS: a device-side index check of the debug build failed";
  }
  return "unknown awq_status";
}

}  // extern "C"
