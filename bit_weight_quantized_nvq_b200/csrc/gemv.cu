// Decode GEMV: y[M, N] = A[M, K] . W[N, K]^T for M = 1..16, NVFP4 weights
// and Q8_0 activations.
//
// The operation is the row dot of "HANDOFF: flint CPU optimization (Q4_1 +
// NVFP4)", section 3 (ggml_vec_dot_nvfp4_q8_0: one NVFP4 row against one
// Q8_0 row, one scale per 16 weights): per 16-element subblock,
//   y += g * s_w * d_a * 0.5 * sum(c_w * q_a),   c_w = 2*E2M1 in -12..12.
//
// Design (HBM-bound; every weight byte is read exactly once):
//  * one warp per weight row; lane l of the warp owns the 32-element chunks
//    l, l+32, l+64, ... of the row.  A chunk is 16 code bytes (one 128-bit
//    load), two UE4M3 scale bytes (one 16-bit load) and exactly one Q8_0
//    activation block (32 int8 codes + one fp16 d), so lanes read disjoint,
//    contiguous, coalesced spans of both weight streams;
//  * loads of U chunks are issued before any is used, so each warp keeps
//    U * 512 bytes of weights in flight;
//  * codes are decoded in registers to signed bytes c = 2*E2M1 with byte
//    permutes (no shared-memory table); dp4a (s8 x s8) forms the exact
//    integer subblock sums, so the +12 bias of the x86 unsigned-by-signed
//    dot is not needed here;
//  * the two subblock sums of a chunk are rescaled by their UE4M3 scales,
//    multiplied by the chunk's d and accumulated in fp32; the activation
//    block is read through L1 (it is shared by every row on the SM);
//  * one shuffle reduction per row, then y = 0.5*g*acc.
#include <cuda_fp16.h>

#include "nvq_device.cuh"
#include "nvq_internal.h"

namespace nvq {
namespace {

constexpr int kWarps = 4;        // rows per CTA
constexpr int kUnroll = 4;       // chunks per lane in flight

template <int MT>
__global__ void __launch_bounds__(kWarps * 32)
gemv_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
            float half_g, int N, int K, const int8_t* __restrict__ q,
            const __half* __restrict__ d, float* __restrict__ y) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (row >= N) return;
  const int nchunk = K >> 5;
  const uint4* wrow = reinterpret_cast<const uint4*>(codes + static_cast<size_t>(row) * (K >> 1));
  const uint16_t* srow = reinterpret_cast<const uint16_t*>(scales + static_cast<size_t>(row) * (K >> 4));

  float acc[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) acc[m] = 0.0f;

  for (int c0 = 0; c0 < nchunk; c0 += 32 * kUnroll) {
    uint4 wv[kUnroll];
    uint32_t sv[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int c = c0 + u * 32 + lane;
      if (c < nchunk) {
        wv[u] = dev::ld_stream_v4(wrow + c);
        sv[u] = __ldg(srow + c);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int c = c0 + u * 32 + lane;
      if (c < nchunk) {
        uint32_t cw[8];
        dev::decode_e2m1x8(wv[u].x, cw[0], cw[1]);
        dev::decode_e2m1x8(wv[u].y, cw[2], cw[3]);
        dev::decode_e2m1x8(wv[u].z, cw[4], cw[5]);
        dev::decode_e2m1x8(wv[u].w, cw[6], cw[7]);
        const float2 s = dev::ue4m3x2_to_float2(sv[u]);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const uint4* qa = reinterpret_cast<const uint4*>(q + static_cast<size_t>(m) * K) + 2 * c;
          const uint4 q0 = __ldg(qa);
          const uint4 q1 = __ldg(qa + 1);
          const float dm = __half2float(__ldg(d + static_cast<size_t>(m) * (K >> 5) + c));
          const int i0 = dev::dp4a(cw[0], q0.x, dev::dp4a(cw[1], q0.y,
                         dev::dp4a(cw[2], q0.z, dev::dp4a(cw[3], q0.w, 0))));
          const int i1 = dev::dp4a(cw[4], q1.x, dev::dp4a(cw[5], q1.y,
                         dev::dp4a(cw[6], q1.z, dev::dp4a(cw[7], q1.w, 0))));
          acc[m] = fmaf(dm, fmaf(s.x, static_cast<float>(i0), s.y * static_cast<float>(i1)), acc[m]);
        }
      }
    }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    const float v = dev::warp_sum(acc[m]);
    if (lane == 0) y[static_cast<size_t>(m) * N + row] = v * half_g;
  }
}

// Integer subblock sums through the same decode and dot code, one warp per
// row: isum[m, n, 2c + h] for chunk c, half h.
__global__ void __launch_bounds__(kWarps * 32)
subblock_sums_kernel(const uint8_t* __restrict__ codes, int N, int K,
                     const int8_t* __restrict__ q, int M, int32_t* __restrict__ isum) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (row >= N) return;
  const int nchunk = K >> 5;
  const uint4* wrow = reinterpret_cast<const uint4*>(codes + static_cast<size_t>(row) * (K >> 1));
  for (int c = lane; c < nchunk; c += 32) {
    const uint4 w = dev::ld_stream_v4(wrow + c);
    uint32_t cw[8];
    dev::decode_e2m1x8(w.x, cw[0], cw[1]);
    dev::decode_e2m1x8(w.y, cw[2], cw[3]);
    dev::decode_e2m1x8(w.z, cw[4], cw[5]);
    dev::decode_e2m1x8(w.w, cw[6], cw[7]);
    for (int m = 0; m < M; ++m) {
      const uint4* qa = reinterpret_cast<const uint4*>(q + static_cast<size_t>(m) * K) + 2 * c;
      const uint4 q0 = __ldg(qa);
      const uint4 q1 = __ldg(qa + 1);
      int2 out;
      out.x = dev::dp4a(cw[0], q0.x, dev::dp4a(cw[1], q0.y,
              dev::dp4a(cw[2], q0.z, dev::dp4a(cw[3], q0.w, 0))));
      out.y = dev::dp4a(cw[4], q1.x, dev::dp4a(cw[5], q1.y,
              dev::dp4a(cw[6], q1.z, dev::dp4a(cw[7], q1.w, 0))));
      int2* dst = reinterpret_cast<int2*>(isum + (static_cast<size_t>(m) * N + row) * (K >> 4)) + c;
      *dst = out;
    }
  }
}

template <int MT>
cudaError_t launch_gemv_m(const uint8_t* codes, const uint8_t* scales, float g,
                          int64_t N, int64_t K, const int8_t* q, const uint16_t* d,
                          float* y, cudaStream_t stream) {
  const unsigned grid = static_cast<unsigned>((N + kWarps - 1) / kWarps);
  gemv_kernel<MT><<<grid, kWarps * 32, 0, stream>>>(
      codes, scales, 0.5f * g, static_cast<int>(N), static_cast<int>(K), q,
      reinterpret_cast<const __half*>(d), y);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemv(const uint8_t* codes, const uint8_t* scales, float g,
                        int64_t N, int64_t K, const int8_t* q, const uint16_t* d,
                        int64_t M, float* y, cudaStream_t stream) {
  switch (M) {
#define NVQ_GEMV_CASE(mm) \
    case mm: return launch_gemv_m<mm>(codes, scales, g, N, K, q, d, y, stream);
    NVQ_GEMV_CASE(1) NVQ_GEMV_CASE(2) NVQ_GEMV_CASE(3) NVQ_GEMV_CASE(4)
    NVQ_GEMV_CASE(5) NVQ_GEMV_CASE(6) NVQ_GEMV_CASE(7) NVQ_GEMV_CASE(8)
    NVQ_GEMV_CASE(9) NVQ_GEMV_CASE(10) NVQ_GEMV_CASE(11) NVQ_GEMV_CASE(12)
    NVQ_GEMV_CASE(13) NVQ_GEMV_CASE(14) NVQ_GEMV_CASE(15) NVQ_GEMV_CASE(16)
#undef NVQ_GEMV_CASE
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_subblock_sums(const uint8_t* codes, int64_t N, int64_t K,
                                 const int8_t* q, int64_t M, int32_t* isum,
                                 cudaStream_t stream) {
  const unsigned grid = static_cast<unsigned>((N + kWarps - 1) / kWarps);
  subblock_sums_kernel<<<grid, kWarps * 32, 0, stream>>>(
      codes, static_cast<int>(N), static_cast<int>(K), q, static_cast<int>(M), isum);
  return cudaGetLastError();
}

}  // namespace nvq
