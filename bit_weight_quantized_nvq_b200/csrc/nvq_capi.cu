// C ABI of the library: host-side argument validation, device checks and
// dispatch to the kernel launchers.  Nothing here allocates device memory.
#include <atomic>
#include <cstdint>

#include <cuda_runtime.h>

#include "nvq.h"
#include "nvq_internal.h"

namespace {

constexpr int kVersion = 10000;  // 1.0.0
constexpr int kMaxDevices = 64;

thread_local cudaError_t t_last_cuda_error = cudaSuccess;

// 0 = not yet checked, 1 = sm_100, 2 = other architecture.
std::atomic<int> g_device_ok[kMaxDevices];
std::atomic<int> g_device_sms[kMaxDevices];

bool aligned16(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

nvq_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return NVQ_OK;
  t_last_cuda_error = e;
  return NVQ_ERR_CUDA;
}

// The current device must be compute capability 10.0 (B200, sm_100a).
nvq_status check_device() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_status(e);
  }
  if (dev < 0 || dev >= kMaxDevices) return NVQ_ERR_UNSUPPORTED_DEVICE;
  int state = g_device_ok[dev].load(std::memory_order_relaxed);
  if (state == 0) {
    int major = 0, minor = 0, sms = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess)
      e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e == cudaSuccess)
      e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return cuda_status(e);
    }
    state = (major == 10 && minor == 0) ? 1 : 2;
    g_device_sms[dev].store(sms, std::memory_order_relaxed);
    g_device_ok[dev].store(state, std::memory_order_relaxed);
  }
  return state == 1 ? NVQ_OK : NVQ_ERR_UNSUPPORTED_DEVICE;
}

// Shapes and pointers shared by the weight x activation entry points:
// K a positive multiple of 64, M within [m_min, m_max] (or 0), every pointer
// non-NULL and 16-byte aligned unless the product is empty (M == 0 or
// N == 0).  `need_scales` is false for the integer-sum export, which reads
// neither the weight scales nor the activation scales.
nvq_status check_dot_args(const void* codes, const void* scales, int64_t N,
                          int64_t K, const void* q, const void* d, int64_t M,
                          const void* y, int64_t m_min, int64_t m_max,
                          bool need_scales) {
  if (N < 0 || K < 0 || M < 0) return NVQ_ERR_INVALID_ARG;
  if (K == 0 || K % 64 != 0) return NVQ_ERR_BAD_SHAPE;
  if (K > (int64_t{1} << 30) || N > (int64_t{1} << 30)) return NVQ_ERR_BAD_SHAPE;
  if (M != 0 && (M < m_min || M > m_max)) return NVQ_ERR_BAD_SHAPE;
  if (N == 0 || M == 0) return NVQ_OK;
  if (!codes || !q || !y) return NVQ_ERR_INVALID_ARG;
  if (need_scales && (!scales || !d)) return NVQ_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(q) || !aligned16(y)) return NVQ_ERR_MISALIGNED;
  if (need_scales && (!aligned16(scales) || !aligned16(d))) return NVQ_ERR_MISALIGNED;
  return NVQ_OK;
}

}  // namespace

namespace nvq {
void set_last_cuda_error(cudaError_t e) { t_last_cuda_error = e; }

// SMs of the current device: cached on first use (the workspace sizes that
// depend on it are queried before any launch), 148 without a device.
int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 148;
  }
  if (dev < 0 || dev >= kMaxDevices) return 148;
  int sms = g_device_sms[dev].load(std::memory_order_relaxed);
  if (sms > 0) return sms;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      sms <= 0) {
    cudaGetLastError();
    return 148;
  }
  g_device_sms[dev].store(sms, std::memory_order_relaxed);
  return sms;
}
}  // namespace nvq

extern "C" {

int nvq_version(void) { return kVersion; }

const char* nvq_status_string(nvq_status status) {
  switch (status) {
    case NVQ_OK: return "ok";
    case NVQ_ERR_INVALID_ARG: return "invalid argument (NULL pointer, negative size or bad value)";
    case NVQ_ERR_BAD_SHAPE: return "unsupported shape (K must be a multiple of 64; M within the entry point's range)";
    case NVQ_ERR_MISALIGNED: return "device pointer not 16-byte aligned";
    case NVQ_ERR_CUDA: return "CUDA runtime error (see nvq_last_cuda_error)";
    case NVQ_ERR_UNSUPPORTED_DEVICE: return "current device is not an sm_100 (B200) GPU";
    case NVQ_ERR_WORKSPACE: return "workspace missing or smaller than nvq_gemm_workspace_size";
    default: return "unknown status";
  }
}

const char* nvq_last_cuda_error(void) { return cudaGetErrorName(t_last_cuda_error); }

nvq_status nvq_quantize_act_q8_0(const float* x, int64_t M, int64_t K,
                                 int8_t* q, uint16_t* d, void* stream) {
  if (M < 0 || K < 0) return NVQ_ERR_INVALID_ARG;
  if (K % 32 != 0) return NVQ_ERR_BAD_SHAPE;
  if (M == 0 || K == 0) return NVQ_OK;
  if (M * K > (int64_t{1} << 40)) return NVQ_ERR_BAD_SHAPE;
  if (!x || !q || !d) return NVQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(q) || !aligned16(d)) return NVQ_ERR_MISALIGNED;
  nvq_status st = check_device();
  if (st != NVQ_OK) return st;
  return cuda_status(nvq::launch_quantize_q8_0(x, M, K, q, d,
                                               static_cast<cudaStream_t>(stream)));
}

nvq_status nvq_gemv(const uint8_t* codes, const uint8_t* scales, float g,
                    int64_t N, int64_t K, const int8_t* q, const uint16_t* d,
                    int64_t M, float* y, void* stream) {
  nvq_status st = check_dot_args(codes, scales, N, K, q, d, M, y, 1, 16, true);
  if (st != NVQ_OK) return st;
  if (!(g == g)) return NVQ_ERR_INVALID_ARG;  // NaN scale
  if (N == 0 || M == 0) return NVQ_OK;
  st = check_device();
  if (st != NVQ_OK) return st;
  return cuda_status(nvq::launch_gemv(codes, scales, g, N, K, q, d, M, y,
                                      static_cast<cudaStream_t>(stream)));
}

nvq_status nvq_gemv_requant(const uint8_t* codes, const uint8_t* scales, float g, int64_t N,
                            int64_t K, const int8_t* q, const uint16_t* d, float* y,
                            int8_t* q_out, uint16_t* d_out, int32_t* counters, void* stream) {
  nvq_status st = check_dot_args(codes, scales, N, K, q, d, 1, y, 1, 1, true);
  if (st != NVQ_OK) return st;
  if (!(g == g)) return NVQ_ERR_INVALID_ARG;
  if (N % 32 != 0) return NVQ_ERR_BAD_SHAPE;
  if (N == 0) return NVQ_OK;
  if (!q_out || !d_out || !counters) return NVQ_ERR_INVALID_ARG;
  if (!aligned16(q_out) || !aligned16(d_out) || !aligned16(counters)) return NVQ_ERR_MISALIGNED;
  st = check_device();
  if (st != NVQ_OK) return st;
  nvq::GemvTarget t = {codes, scales, g, N, y, q_out, d_out, counters};
  return cuda_status(nvq::launch_gemv_group(&t, 1, K, q, d, static_cast<cudaStream_t>(stream)));
}

nvq_status nvq_gemv_grouped(const nvq_linear* linears, int64_t count, const int8_t* q,
                            const uint16_t* d, int64_t M, float* const* ys, void* stream) {
  if (count < 0 || M < 0) return NVQ_ERR_INVALID_ARG;
  if (count == 0 || M == 0) return NVQ_OK;
  if (!linears || !ys) return NVQ_ERR_INVALID_ARG;
  const int64_t K = linears[0].K;
  int64_t rows = 0;
  for (int64_t i = 0; i < count; ++i) {
    const nvq_linear& L = linears[i];
    if (L.K != K) return NVQ_ERR_BAD_SHAPE;
    nvq_status st = check_dot_args(L.codes, L.scales, L.N, L.K, q, d, M, ys[i], 1, 16, true);
    if (st != NVQ_OK) return st;
    if (!(L.g == L.g)) return NVQ_ERR_INVALID_ARG;
    rows += L.N;
  }
  if (rows > (int64_t{1} << 30)) return NVQ_ERR_BAD_SHAPE;
  nvq_status st = check_device();
  if (st != NVQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M == 1) {
    constexpr int kBatch = 16;
    nvq::GemvTarget t[kBatch];
    for (int64_t i0 = 0; i0 < count; i0 += kBatch) {
      int n = 0;
      for (int64_t i = i0; i < count && n < kBatch; ++i) {
        if (linears[i].N == 0) continue;
        t[n++] = {linears[i].codes, linears[i].scales, linears[i].g, linears[i].N, ys[i],
                  nullptr, nullptr, nullptr};
      }
      st = cuda_status(nvq::launch_gemv_group(t, n, K, q, d, s));
      if (st != NVQ_OK) return st;
    }
    return NVQ_OK;
  }
  for (int64_t i = 0; i < count; ++i) {
    const nvq_linear& L = linears[i];
    if (L.N == 0) continue;
    st = cuda_status(nvq::launch_gemv(L.codes, L.scales, L.g, L.N, K, q, d, M, ys[i], s));
    if (st != NVQ_OK) return st;
  }
  return NVQ_OK;
}

nvq_status nvq_moe_gemv(const uint8_t* codes, const uint8_t* scales, const float* g, int64_t E,
                        int64_t N, int64_t K, const int32_t* ids, int64_t T, int64_t top_k,
                        const int8_t* q, const uint16_t* d, float* y, void* stream) {
  if (E < 0 || N < 0 || K < 0 || T < 0 || top_k < 0) return NVQ_ERR_INVALID_ARG;
  if (K == 0 || K % 64 != 0) return NVQ_ERR_BAD_SHAPE;
  if (T == 0 || top_k == 0 || N == 0) return NVQ_OK;
  if (E == 0) return NVQ_ERR_INVALID_ARG;
  if (!nvq::moe_supported(K, top_k)) return NVQ_ERR_BAD_SHAPE;
  if (T > 65535 || N > (int64_t{1} << 24) || E * N > (int64_t{1} << 32)) return NVQ_ERR_BAD_SHAPE;
  if (!codes || !scales || !g || !ids || !q || !d || !y) return NVQ_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(scales) || !aligned16(q) || !aligned16(d) ||
      !aligned16(y) || !aligned16(ids) || !aligned16(g))
    return NVQ_ERR_MISALIGNED;
  nvq_status st = check_device();
  if (st != NVQ_OK) return st;
  return cuda_status(nvq::launch_moe_gemv(codes, scales, g, E, N, K, ids, T, top_k, q, d, y,
                                          static_cast<cudaStream_t>(stream)));
}

size_t nvq_gemm_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || K <= 0 || N < 0) return 0;
  return nvq::gemm_workspace_size(M, N, K);
}

nvq_status nvq_gemm(const uint8_t* codes, const uint8_t* scales, float g,
                    int64_t N, int64_t K, const int8_t* q, const uint16_t* d,
                    int64_t M, float* y, void* workspace,
                    size_t workspace_bytes, void* stream) {
  nvq_status st = check_dot_args(codes, scales, N, K, q, d, M, y, 1,
                                 int64_t{1} << 24, true);
  if (st != NVQ_OK) return st;
  if (!(g == g)) return NVQ_ERR_INVALID_ARG;
  if (N == 0 || M == 0) return NVQ_OK;
  if (!workspace || workspace_bytes < nvq::gemm_workspace_size(M, N, K))
    return NVQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return NVQ_ERR_MISALIGNED;
  st = check_device();
  if (st != NVQ_OK) return st;
  return cuda_status(nvq::launch_gemm(codes, scales, g, N, K, q, d, M, y, workspace,
                                      static_cast<cudaStream_t>(stream)));
}

nvq_status nvq_gemm_noalloc(const uint8_t* codes, const uint8_t* scales, float g,
                            int64_t N, int64_t K, const int8_t* q, const uint16_t* d,
                            int64_t M, float* y, void* stream) {
  nvq_status st = check_dot_args(codes, scales, N, K, q, d, M, y, 1,
                                 int64_t{1} << 24, true);
  if (st != NVQ_OK) return st;
  if (!(g == g)) return NVQ_ERR_INVALID_ARG;
  if (N == 0 || M == 0) return NVQ_OK;
  if (nvq::gemm_workspace_size(M, N, K) > nvq::gemm_noalloc_limit()) return NVQ_ERR_WORKSPACE;
  st = check_device();
  if (st != NVQ_OK) return st;
  void* scratch = nullptr;
  cudaError_t e = nvq::gemm_noalloc_scratch(&scratch);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_status(e);
  }
  return cuda_status(nvq::launch_gemm(codes, scales, g, N, K, q, d, M, y, scratch,
                                      static_cast<cudaStream_t>(stream)));
}

size_t nvq_gemm_w4a16_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || M > 16 || K <= 0 || K % 256 != 0 || N < 0) return 0;
  return nvq::gemm_small_workspace_size(M, K);
}

nvq_status nvq_gemm_w4a16(const uint8_t* codes, const uint8_t* scales, float g, int64_t N,
                          int64_t K, const uint16_t* x, int64_t M, float* y, void* workspace,
                          size_t workspace_bytes, void* stream) {
  // x plays the part of q for the pointer checks; there is no d
  nvq_status st = check_dot_args(codes, scales, N, K, x, x, M, y, 1, 16, true);
  if (st != NVQ_OK) return st;
  if (!(g == g)) return NVQ_ERR_INVALID_ARG;
  if (K % 256 != 0) return NVQ_ERR_BAD_SHAPE;
  if (N == 0 || M == 0) return NVQ_OK;
  if (!workspace || workspace_bytes < nvq::gemm_small_workspace_size(M, K))
    return NVQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return NVQ_ERR_MISALIGNED;
  st = check_device();
  if (st != NVQ_OK) return st;
  return cuda_status(nvq::launch_gemm_small_f16(codes, scales, g, N, K, x, M, y, workspace,
                                                static_cast<cudaStream_t>(stream)));
}

nvq_status nvq_quantize_act_nvfp4(const float* x, int64_t M, int64_t K, uint8_t* codes,
                                  uint8_t* scales, float* g, void* stream) {
  if (M < 0 || K < 0) return NVQ_ERR_INVALID_ARG;
  if (K % 16 != 0) return NVQ_ERR_BAD_SHAPE;
  if (M == 0 || K == 0) return NVQ_OK;
  if (M > INT32_MAX || K > (int64_t{1} << 30)) return NVQ_ERR_BAD_SHAPE;
  if (!x || !codes || !scales || !g) return NVQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(g))
    return NVQ_ERR_MISALIGNED;
  nvq_status st = check_device();
  if (st != NVQ_OK) return st;
  return cuda_status(nvq::launch_quantize_nvfp4(x, M, K, codes, scales, g,
                                                static_cast<cudaStream_t>(stream)));
}

nvq_status nvq_gemm_nvf4(const uint8_t* w_codes, const uint8_t* w_scales, float g_w, int64_t N,
                         int64_t K, const uint8_t* a_codes, const uint8_t* a_scales,
                         const float* a_g, int64_t M, float* y, void* stream) {
  if (N < 0 || K < 0 || M < 0) return NVQ_ERR_INVALID_ARG;
  if (K == 0 || K % 256 != 0) return NVQ_ERR_BAD_SHAPE;
  if (K > (int64_t{1} << 30) || N > int64_t{65535} * 128 || M > INT32_MAX)
    return NVQ_ERR_BAD_SHAPE;
  if (!(g_w == g_w)) return NVQ_ERR_INVALID_ARG;
  if (N == 0 || M == 0) return NVQ_OK;
  if (!w_codes || !w_scales || !a_codes || !a_scales || !a_g || !y) return NVQ_ERR_INVALID_ARG;
  if (!aligned16(w_codes) || !aligned16(w_scales) || !aligned16(a_codes) ||
      !aligned16(a_scales) || !aligned16(a_g) || !aligned16(y))
    return NVQ_ERR_MISALIGNED;
  nvq_status st = check_device();
  if (st != NVQ_OK) return st;
  return cuda_status(nvq::launch_gemm_nvf4(w_codes, w_scales, g_w, N, K, a_codes, a_scales, a_g,
                                           M, y, static_cast<cudaStream_t>(stream)));
}

nvq_status nvq_debug_subblock_sums(const uint8_t* codes, const uint8_t* scales, float g,
                                   int64_t N, int64_t K, const int8_t* q, const uint16_t* d,
                                   int64_t M, float* y, int32_t* isum, void* stream) {
  nvq_status st = check_dot_args(codes, scales, N, K, q, d, M, y, 1, 16, true);
  if (st != NVQ_OK) return st;
  if (!(g == g)) return NVQ_ERR_INVALID_ARG;
  if (N == 0 || M == 0) return NVQ_OK;
  if (!isum) return NVQ_ERR_INVALID_ARG;
  if (!aligned16(isum)) return NVQ_ERR_MISALIGNED;
  st = check_device();
  if (st != NVQ_OK) return st;
  return cuda_status(nvq::launch_gemv_isum(codes, scales, g, N, K, q, d, M, y, isum,
                                           static_cast<cudaStream_t>(stream)));
}

nvq_status nvq_error_flags(unsigned int* flags, int clear) {
  if (!flags) return NVQ_ERR_INVALID_ARG;
  nvq_status st = check_device();
  if (st != NVQ_OK) return st;
  unsigned int gemv = 0, gemm = 0, gemm_small = 0, nvf4 = 0;
  cudaError_t e = nvq::gemv_error_flags(clear != 0, &gemv);
  if (e == cudaSuccess) e = nvq::gemm_error_flags(clear != 0, &gemm);
  if (e == cudaSuccess) e = nvq::gemm_small_error_flags(clear != 0, &gemm_small);
  if (e == cudaSuccess) e = nvq::nvf4_error_flags(clear != 0, &nvf4);
  gemm |= gemm_small | nvf4;
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_status(e);
  }
  *flags = ((gemv & 1u) ? NVQ_FLAG_GEMV_TIMEOUT : 0u) | (gemm ? NVQ_FLAG_GEMM_TIMEOUT : 0u) |
           ((gemv & 2u) ? NVQ_FLAG_BAD_INDEX : 0u);
  return NVQ_OK;
}

nvq_status nvq_debug_stalled_wait(uint64_t limit_ns, int* result, void* stream) {
  if (!result) return NVQ_ERR_INVALID_ARG;
  if (limit_ns < 1000 || limit_ns > 1000000000ull) return NVQ_ERR_INVALID_ARG;
  if (!aligned16(result)) return NVQ_ERR_MISALIGNED;
  nvq_status st = check_device();
  if (st != NVQ_OK) return st;
  return cuda_status(nvq::launch_stalled_wait(limit_ns, result,
                                              static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
