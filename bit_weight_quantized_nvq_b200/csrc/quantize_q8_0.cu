// Fused Q8_0 activation quantiser: one pass of amax / scale / round.
//
// Q8_0 (the GGML type table of the spke.com 2-bit GGUF tutorial: 32 values,
// 34 bytes) stores 32 int8 codes and one fp16 scale per block.  Per block,
// in fp32 IEEE arithmetic: amax = max|x|, d32 = amax/127, q = rint(x/d32)
// clamped to +-127, d = fp16(d32).  Both divisions are correctly rounded
// (no fast-math), and rint rounds half to even, so the result is bit-exact.
//
// Layout: x is [M, K] row-major with K % 32 == 0, so every 32-block is 128
// contiguous bytes and the flat array can be processed without row
// arithmetic.  Eight lanes share one block (one float4 each); a warp covers
// four consecutive blocks with fully coalesced 512-byte loads and 128-byte
// code stores; the block amax is reduced with three shuffles inside each
// group of eight lanes.  The kernel is HBM-bound: 4 + 1 + 2/32 bytes per
// element.  It is launched with programmatic stream serialisation (see the
// decode GEMV), so at one token its launch overlaps the previous kernel.
#include <cuda_fp16.h>

#include "nvq_device.cuh"
#include "nvq_internal.h"

namespace nvq {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
quantize_q8_0_kernel(const float4* __restrict__ x, int64_t nblocks,
                     uint32_t* __restrict__ q, __half* __restrict__ d) {
  // programmatic dependent launch: let the next kernel launch early, and
  // read x only once the kernel that wrote it has completed
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  const int64_t b = t >> 3;
  if (b >= nblocks) return;  // whole groups of eight leave together
  const unsigned lane = threadIdx.x & 31u;
  const unsigned group_mask = 0xFFu << (lane & 24u);

  const float4 v = x[t];
  float a = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
  a = fmaxf(a, __shfl_xor_sync(group_mask, a, 1, 8));
  a = fmaxf(a, __shfl_xor_sync(group_mask, a, 2, 8));
  a = fmaxf(a, __shfl_xor_sync(group_mask, a, 4, 8));

  const float d32 = __fdiv_rn(a, 127.0f);
  uint32_t packed = 0;
  if (d32 > 0.0f) {
    const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int qi = __float2int_rn(__fdiv_rn(e[i], d32));
      qi = max(-127, min(127, qi));
      packed |= (static_cast<uint32_t>(qi) & 0xFFu) << (8 * i);
    }
  }
  q[t] = packed;
  if ((t & 7) == 0) d[b] = __float2half_rn(d32);
}

}  // namespace

cudaError_t launch_quantize_q8_0(const float* x, int64_t M, int64_t K,
                                 int8_t* q, uint16_t* d, cudaStream_t stream) {
  const int64_t nblocks = M * (K / 32);
  if (nblocks == 0) return cudaSuccess;
  const int64_t threads = nblocks * 8;
  const int64_t grid = (threads + kThreads - 1) / kThreads;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, quantize_q8_0_kernel, reinterpret_cast<const float4*>(x),
                            nblocks, reinterpret_cast<uint32_t*>(q), reinterpret_cast<__half*>(d));
}

}  // namespace nvq
