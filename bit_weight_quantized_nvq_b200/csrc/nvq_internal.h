// Internal declarations shared by the library's translation units.
// Launchers assume validated arguments (the C ABI layer checks them).
#pragma once

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

// Q8_0 quantisation of one fp32 token fused into the decode GEMV (M = 1);
// supported for K = 1024 * T, T in {4, 5, 6, 8, 10, 12, 15, 16, 20, 25}.
bool quant_gemv_supported(int64_t K);
cudaError_t launch_quant_gemv(const uint8_t* codes, const uint8_t* scales, float g,
                              int64_t N, int64_t K, const float* x, float* y,
                              cudaStream_t stream);

// Error flags raised by GEMV kernels (bit 0: a pipeline wait timed out);
// synchronous read, optionally clearing them.
unsigned int gemv_error_flags(bool clear);

// Integer per-16 subblock sums through the GEMV's decode/dot code.
cudaError_t launch_subblock_sums(const uint8_t* codes, int64_t N, int64_t K,
                                 const int8_t* q, int64_t M, int32_t* isum,
                                 cudaStream_t stream);

// Prefill GEMM (tcgen05) and the size of its activation workspace.
size_t gemm_workspace_size(int64_t M, int64_t N, int64_t K);
cudaError_t launch_gemm(const uint8_t* codes, const uint8_t* scales, float g,
                        int64_t N, int64_t K, const int8_t* q,
                        const uint16_t* d, int64_t M, float* y,
                        void* workspace, cudaStream_t stream);
// The two halves of launch_gemm: expand Q8_0 activations into the
// workspace, then run the tensor-core GEMM on an expanded workspace (which
// several weight matrices with the same K may share).
cudaError_t gemm_expand(const int8_t* q, const uint16_t* d, int64_t M, int64_t K,
                        void* workspace, cudaStream_t stream);
cudaError_t gemm_main(const uint8_t* codes, const uint8_t* scales, float g, int64_t N,
                      int64_t K, int64_t M, float* y, const void* workspace,
                      cudaStream_t stream);

// The allocation-free GEMM: bytes of its library-owned scratch, and the
// scratch's device address on the current device (looked up once per
// device, on first use).
size_t gemm_noalloc_limit();
cudaError_t gemm_noalloc_scratch(void** out);

// Error flags raised by the GEMM kernel (bit 0: a pipeline wait timed out).
unsigned int gemm_error_flags(bool clear);

// Record the CUDA error reported by nvq_last_cuda_error() on this thread.
void set_last_cuda_error(cudaError_t e);

// Number of streaming multiprocessors of the current device (cached).
int device_sm_count();

}  // namespace nvq
