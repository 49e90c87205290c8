// Internal declarations shared by the library's translation units.
// Launchers assume validated arguments (the C ABI layer checks them).
#pragma once

#include <atomic>
#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

namespace nvq {

// Q8_0 activation quantiser over M*K/32 blocks.
cudaError_t launch_quantize_q8_0(const float* x, int64_t M, int64_t K,
                                 int8_t* q, uint16_t* d, cudaStream_t stream);

// Decode GEMV for M = 1..16.
cudaError_t launch_gemv(const uint8_t* codes, const uint8_t* scales, float g,
                        int64_t N, int64_t K, const int8_t* q,
                        const uint16_t* d, int64_t M, float* y,
                        cudaStream_t stream);
// The same dispatch and kernels, instantiated to also store the integer
// subblock sums they form (isum int32 [M, N, K/16]).
cudaError_t launch_gemv_isum(const uint8_t* codes, const uint8_t* scales, float g,
                             int64_t N, int64_t K, const int8_t* q,
                             const uint16_t* d, int64_t M, float* y, int32_t* isum,
                             cudaStream_t stream);

// One token's GEMV through several matrices with the same K that read the
// same Q8_0 activations, as few launches as the register schedule allows;
// a target with rq_q set also receives the Q8_0 quantisation of its output
// (rq_q [N] codes, rq_d [N/32] fp16 scales, N % 32 == 0), bit-identical to
// launch_quantize_q8_0 of y.  rq_cnt: N/32 ints that are 0 before the launch
// and are left 0.
struct GemvTarget {
  const uint8_t* codes;
  const uint8_t* scales;
  float g;
  int64_t N;
  float* y;
  int8_t* rq_q;
  uint16_t* rq_d;
  int* rq_cnt;
};
cudaError_t launch_gemv_group(const GemvTarget* targets, int n, int64_t K, const int8_t* q,
                              const uint16_t* d, cudaStream_t stream);

// Mixture-of-experts decode GEMV: token t times the experts ids[t, j] of a
// stacked expert tensor, y [T, top_k, N]; supported for the K of the
// register schedule and top_k <= 8.  A routing id outside 0..E-1 raises
// error bit 1 and its slot is left unwritten.
bool moe_supported(int64_t K, int64_t top_k);
cudaError_t launch_moe_gemv(const uint8_t* codes, const uint8_t* scales, const float* g, int64_t E,
                            int64_t N, int64_t K, const int32_t* ids, int64_t T, int64_t top_k,
                            const int8_t* q, const uint16_t* d, float* y, cudaStream_t stream);

// The linears of a decoder stack at one token in one persistent (cooperative)
// launch per 64 layers; see nvq_decoder_stack for the dataflow.  Supported
// for K0 (hidden) 4096 or 5120 and the down K of stack_m1_supported.
struct StackLinear {
  const uint8_t* codes;
  const uint8_t* scales;
  float g;
};
struct StackM1 {
  const StackLinear* lin;        // host [n_layers * 7]: q, k, v, o, up, gate, down
  int64_t n_layers;
  int64_t N[7];
  int64_t K0, Kd;
  float* outs[7];
  const int8_t* x_q;             // Q8_0(x), written before the launch
  const uint16_t* x_d;
  int8_t* b_q[3][2];             // Q8_0 of y_v, y_o, y_up, two buffers each
  uint16_t* b_d[3][2];
  int* cnt[3];                   // block counters of v, o, up: zero, left zero
  unsigned int* bar;             // 3 * 64 unit counters (zeroed by the launcher)
};
bool stack_m1_supported(int64_t K0, int64_t Kd, const int64_t* N);
cudaError_t launch_stack_m1(const StackM1& s, cudaStream_t stream);

// Test-only: a pipeline wait that can never complete, bounded by limit_ns;
// result[0] = 1 if the wait completed (never), result[1] = microseconds waited.
cudaError_t launch_stalled_wait(uint64_t limit_ns, int* result, cudaStream_t stream);

// Error flags raised by the kernels when a bounded pipeline wait times out,
// read synchronously on the current device (optionally clearing them).
cudaError_t gemv_error_flags(bool clear, unsigned int* flags);
cudaError_t gemm_error_flags(bool clear, unsigned int* flags);

// Prefill GEMM (tcgen05) and the size of its activation workspace.
size_t gemm_workspace_size(int64_t M, int64_t N, int64_t K);
cudaError_t launch_gemm(const uint8_t* codes, const uint8_t* scales, float g,
                        int64_t N, int64_t K, const int8_t* q,
                        const uint16_t* d, int64_t M, float* y,
                        void* workspace, cudaStream_t stream);
// Q8_0 activations -> the exact fp16 pairs [hi rows 0..M_pad-1 | lo rows
// M_pad..2*M_pad-1] x K in `act` (rows >= M zero) and M_pad token scales.
cudaError_t expand_activations(const int8_t* q, const uint16_t* d, int64_t M, int64_t M_pad,
                               int64_t K, void* act, float* tok_scale, cudaStream_t stream);
// The small-token tensor-core schedule (M = 1..16, K % 256 == 0), which
// launch_gemm and gemm_workspace_size select by themselves.
bool gemm_small_supported(int64_t M, int64_t K);
size_t gemm_small_workspace_size(int64_t M, int64_t K);
cudaError_t launch_gemm_small(const uint8_t* codes, const uint8_t* scales, float g, int64_t N,
                              int64_t K, const int8_t* q, const uint16_t* d, int64_t M, float* y,
                              void* workspace, cudaStream_t stream);
cudaError_t gemm_small_error_flags(bool clear, unsigned int* flags);
// The same schedule on fp16 activations x [M, K] (W4A16), workspace of
// gemm_small_workspace_size(M, K) bytes.
cudaError_t launch_gemm_small_f16(const uint8_t* codes, const uint8_t* scales, float g,
                                  int64_t N, int64_t K, const uint16_t* x, int64_t M, float* y,
                                  void* workspace, cudaStream_t stream);
// NVFP4 activations: per token row g[m] = amax/2688 and the weight recipe
// (codes [M, K/2], scales [M, K/16]), K % 16 == 0.
cudaError_t launch_quantize_nvfp4(const float* x, int64_t M, int64_t K, uint8_t* codes,
                                  uint8_t* scales, float* g, cudaStream_t stream);
// NVFP4 weights x NVFP4 activations on the block-scaled FP4 tensor-core path,
// y [M, N] fp32, K % 256 == 0.
cudaError_t launch_gemm_nvf4(const uint8_t* w_codes, const uint8_t* w_scales, float g_w,
                             int64_t N, int64_t K, const uint8_t* a_codes,
                             const uint8_t* a_scales, const float* g_a, int64_t M, float* y,
                             cudaStream_t stream);
cudaError_t nvf4_error_flags(bool clear, unsigned int* flags);
// The two halves of launch_gemm for the large-token schedule: expand Q8_0 activations into the
// workspace, then run the tensor-core GEMM on an expanded workspace (which
// several weight matrices with the same K may share).
cudaError_t gemm_expand(const int8_t* q, const uint16_t* d, int64_t M, int64_t K,
                        void* workspace, cudaStream_t stream);
cudaError_t gemm_main(const uint8_t* codes, const uint8_t* scales, float g, int64_t N,
                      int64_t K, int64_t M, float* y, const void* workspace,
                      cudaStream_t stream);

// The allocation-free GEMM: bytes of its library-owned scratch, and the
// scratch's device address on the current device (looked up once per
// device and context, on first use).
size_t gemm_noalloc_limit();
cudaError_t gemm_noalloc_scratch(void** out);

// Record the CUDA error reported by nvq_last_cuda_error() on this thread.
void set_last_cuda_error(cudaError_t e);

// Number of streaming multiprocessors of the current device (cached).
int device_sm_count();

// Sets a kernel's dynamic shared-memory limit once per device.  Safe when
// several host threads make their first calls at the same time (the
// attribute call is idempotent; the flag only skips repeats).
struct SmemAttrOnce {
  static constexpr int kMaxDevices = 64;
  std::atomic<bool> done[kMaxDevices] = {};

  template <typename Kernel>
  cudaError_t ensure(Kernel kernel, int bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const bool cacheable = dev >= 0 && dev < kMaxDevices;
    if (cacheable && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && cacheable) done[dev].store(true, std::memory_order_release);
    return e;
  }
};

}  // namespace nvq
