// NVFP4 x NVFP4: NVFP4 activations and the product on the tensor core's
// native block-scaled FP4 path (tcgen05.mma.kind::mxf4nvf4.block_scale with
// one UE4M3 scale per 16 elements on both operands).
//
// The NVFP4 serving engines that "TKintegers K5: 3.21x prefill and 3.10x
// decode throughput vs TorchAO FP8 on NVIDIA L4" links to, and the NVFP4
// rows of the protolabsai lab-benchmarks card, run both operands in the
// weights' 4-bit format.  Here the activations take the weight recipe with
// one fp32 scale per token: g[m] = amax(|x[m]|)/(6*448); per 16 elements
// s = UE4M3(amax_blk/(6*g)); code = E2M1(x/(g*s)), round to nearest, ties
// to even, saturating, a zero magnitude stored as +0.
//
// The product needs no decode: the packed codes go from HBM to shared
// memory by TMA exactly as stored (two E2M1 per byte, element 2i in the low
// nibble), the tensor core reads them there, and the per-16 scales, copied
// into tensor memory (lane = row, one 32-bit column per 64-wide K step,
// byte j for K block j), are applied inside the MMA.  Every product of two
// E2M1 values and two UE4M3 scales is exact in fp32; the accumulation is
// fp32, promoted to registers every 1024 K; y = g_w * g_a[m] * sum.
//
// gemm_nvf4_kernel: one CTA per (128 weight rows, 128 tokens) tile.
//   warp 0     TMA: per 256-wide K stage the 128 x 128-byte code tiles of
//              weights and tokens (128-byte swizzle) and their 128 x 16-byte
//              scale tiles, into a 6-deep ring (216 KB in flight per SM);
//   warp 1     allocates tensor memory; issues 4 block-scaled MMAs per stage
//              (M = 128 weight rows, N = 128 tokens, K = 64);
//   warps 2-5  (one per tensor-memory lane quarter) copy each stage's scales
//              to tensor memory with tcgen05.st;
//   warps 2-9  drain finished 1024-wide K chunks into fp32 registers (two
//              warps per lane quarter, 64 token columns each) and store y.
// Every wait is bounded (4 s): a timeout raises the GEMM error flag and the
// CTA drains what it issued before freeing tensor memory.
#include <algorithm>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include "nvq_device.cuh"
#include "nvq_internal.h"
#include "tcgen05.cuh"

namespace nvq {
namespace {

// ---------------------------------------------------------------------------
// NVFP4 activation quantiser (one CTA per token row)
// ---------------------------------------------------------------------------
// UE4M3 byte nearest to r >= 0 (ties to the even code), saturating at
// 0x7E = 448.  Bytes 0..7 are m * 2^-9 and byte 8e + m (e >= 1) is
// (8 + m) * 2^(e-10): inside exponent e the code is (e-1)*8 + rint(r*2^(10-e)),
// e = (fp32 biased exponent of r) - 120, at least 1 (the subnormal bytes
// share the spacing of e = 1).  2^(10-e) is built from its exponent bits, so
// the scaling is exact.
__device__ __forceinline__ uint32_t ue4m3_encode(float r) {
  if (!(r > 0.0f)) return 0;
  if (r >= 448.0f) return 0x7E;
  const int e = max(1, static_cast<int>(__float_as_uint(r) >> 23) - 120);
  const int n = __float2int_rn(r * __uint_as_float(static_cast<uint32_t>(137 - e) << 23));
  const int code = (e - 1) * 8 + n;
  return static_cast<uint32_t>(code > 0x7E ? 0x7E : code);
}
// Value of a UE4M3 byte (b <= 0x7E): m * 2^-9 for exponent 0, else the fp32
// with exponent e - 7 and the three mantissa bits on top.
__device__ __forceinline__ float ue4m3_value(uint32_t b) {
  const uint32_t e = (b >> 3) & 0xF, m = b & 0x7;
  return e == 0 ? static_cast<float>(m) * 0x1p-9f : __uint_as_float(((e + 120) << 23) | (m << 20));
}
// E2M1 magnitude code nearest to q >= 0 (ties to the even code), saturating
// at 6; the magnitudes 0, .5, 1, 1.5 | 2, 3 | 4, 6 have spacings 0.5, 1 and
// 2, so the codes are rint(2q), rint(q) + 2 and rint(q/2) + 4 there.
__device__ __forceinline__ uint32_t e2m1_mag(float q) {
  int code;
  if (q >= 6.0f)
    code = 7;
  else if (q < 2.0f)
    code = __float2int_rn(q * 2.0f);
  else if (q < 4.0f)
    code = __float2int_rn(q) + 2;
  else
    code = __float2int_rn(q * 0.5f) + 4;
  return static_cast<uint32_t>(code);
}
// E2M1 code of the correctly rounded fp32 quotient x / gs, by IEEE division
// and round-to-nearest-even on the E2M1 grid (a zero magnitude stored as +0).
__device__ __forceinline__ uint32_t e2m1_code_exact(float x, float gs) {
  uint32_t c = e2m1_mag(__fdiv_rn(fabsf(x), gs));
  if (c != 0 && x < 0.0f) c |= 0x8;
  return c;
}

// Eight fp32 values to eight E2M1 codes with the hardware conversion
// (round to nearest, saturating at 6), value i in bits 4i..4i+3; a zero
// magnitude is stored as +0.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&v)[8]) {
  uint32_t w;
  asm("{\n\t.reg .b8 c0, c1, c2, c3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c3, %8, %7;\n\t"
      "mov.b32 %0, {c0, c1, c2, c3};\n\t}"
      : "=r"(w)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  const uint32_t mag = w & 0x77777777u;
  return mag | (w & ((mag + 0x77777777u) & 0x88888888u));   // sign only where the magnitude is not 0
}

// The codes and scale of one subblock held by one thread (16 values).
// Codes: the quotient x/gs is bracketed by x*inv*(1 - 2^-16) and
// x*inv*(1 + 2^-16) (inv = 1/gs rounded; the correctly rounded quotient lies
// strictly between them, their error being below 2^-22), and both brackets
// are converted; rounding is monotone, so where the two codes agree that is
// the code of the correctly rounded quotient, whatever the tie rule.  Where
// they differ (the quotient is within 2^-16 of a rounding tie of the grid),
// and when 1/gs could overflow (gs < 2^-120), the code is computed from the
// IEEE quotient with ties to the even code.
__device__ __forceinline__ void quantize_subblock(const float4 (&v)[4], float g, float six_g,
                                                  uint2* cdst, uint8_t* sdst) {
  float e[16];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    e[4 * j] = v[j].x;
    e[4 * j + 1] = v[j].y;
    e[4 * j + 2] = v[j].z;
    e[4 * j + 3] = v[j].w;
  }
  float ab = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) ab = fmaxf(ab, fabsf(e[i]));
  const float r = six_g > 0.0f ? __fdiv_rn(ab, six_g) : 0.0f;
  const uint32_t sc = ue4m3_encode(r);
  const float gs = __fmul_rn(g, ue4m3_value(sc));
  uint32_t w[2] = {0u, 0u};
  if (gs > 0.0f) {
    uint32_t diff[2] = {0xFFFFFFFFu, 0xFFFFFFFFu};
    if (gs >= 0x1p-120f) {
      const float inv = __frcp_rn(gs);
      const float ilo = inv * (1.0f - 0x1p-16f), ihi = inv * (1.0f + 0x1p-16f);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float lo[8], hi[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          lo[i] = e[8 * h + i] * ilo;
          hi[i] = e[8 * h + i] * ihi;
        }
        w[h] = cvt_e2m1x8(lo);
        diff[h] = w[h] ^ cvt_e2m1x8(hi);
      }
    }
    if (__builtin_expect((diff[0] | diff[1]) != 0u, 0)) {
      for (int i = 0; i < 16; ++i) {
        const int h = i >> 3, sh = 4 * (i & 7);
        if ((diff[h] >> sh) & 0xFu)
          w[h] = (w[h] & ~(0xFu << sh)) | (e2m1_code_exact(e[i], gs) << sh);
      }
    }
  }
  *cdst = make_uint2(w[0], w[1]);
  *sdst = static_cast<uint8_t>(sc);
}

// One cluster of P CTAs per token row (P = gridDim.y <= 8), one thread per
// 16-element subblock: CTA p takes subblocks [p*T, p*T + T).  Every load is
// issued before any is used and the subblocks stay in registers between the
// amax and the codes, so the row is read from memory once.  The row amax is
// each CTA's block maximum, combined over the cluster through distributed
// shared memory (the second cluster barrier keeps every CTA's shared memory
// alive until all have read it).
__global__ void __launch_bounds__(1024)
quantize_nvfp4_kernel(const float* __restrict__ x, int K, uint8_t* __restrict__ codes,
                      uint8_t* __restrict__ scales, float* __restrict__ g_out) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int row = blockIdx.x;
  const int T = blockDim.x;
  const int P = gridDim.y;
  const int nsub = K / 16;
  const int sb = blockIdx.y * T + threadIdx.x;
  const bool in = sb < nsub;
  const float4* xr = reinterpret_cast<const float4*>(x + static_cast<size_t>(row) * K);
  float4 v[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) v[j] = in ? __ldcs(xr + 4 * sb + j) : make_float4(0.f, 0.f, 0.f, 0.f);
  float a = 0.0f;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    a = fmaxf(a, fmaxf(fmaxf(fabsf(v[j].x), fabsf(v[j].y)), fmaxf(fabsf(v[j].z), fabsf(v[j].w))));
  __shared__ float red[32];
  __shared__ float cta_max;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = red[0];
    for (int w = 1; w < (T + 31) / 32; ++w) m = fmaxf(m, red[w]);
    cta_max = m;
  }
  float amax;
  if (P == 1) {
    __syncthreads();
    amax = cta_max;
  } else {
    ptx::cluster_sync();
    amax = 0.0f;
    const uint32_t local = ptx::smem_addr(&cta_max);
    for (int r = 0; r < P; ++r) {
      float m;
      asm volatile("ld.shared::cluster.f32 %0, [%1];"
                   : "=f"(m) : "r"(ptx::mapa_shared(local, r)) : "memory");
      amax = fmaxf(amax, m);
    }
    ptx::cluster_sync();
  }
  const float g = __fdiv_rn(amax, 2688.0f);
  const float six_g = __fmul_rn(6.0f, g);
  if (blockIdx.y == 0 && threadIdx.x == 0) g_out[row] = g;
  if (in)
    quantize_subblock(v, g, six_g,
                      reinterpret_cast<uint2*>(codes + static_cast<size_t>(row) * (K / 2)) + sb,
                      scales + static_cast<size_t>(row) * (K / 16) + sb);
}

// Rows of more than 8 x 256 subblocks (K > 32768): two passes over the row (amax,
// then the subblocks), the second pass reading it again.
__global__ void __launch_bounds__(1024)
quantize_nvfp4_long_kernel(const float* __restrict__ x, int K, uint8_t* __restrict__ codes,
                           uint8_t* __restrict__ scales, float* __restrict__ g_out) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int row = blockIdx.x;
  const int T = blockDim.x;
  const int n4 = K / 4;
  const float4* xr = reinterpret_cast<const float4*>(x + static_cast<size_t>(row) * K);
  float a = 0.0f;
  for (int i = threadIdx.x; i < n4; i += T) {
    const float4 t = xr[i];
    a = fmaxf(a, fmaxf(fmaxf(fabsf(t.x), fabsf(t.y)), fmaxf(fabsf(t.z), fabsf(t.w))));
  }
  __shared__ float red[32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
  __syncthreads();
  float amax = red[0];
  for (int w = 1; w < T / 32; ++w) amax = fmaxf(amax, red[w]);
  const float g = __fdiv_rn(amax, 2688.0f);
  const float six_g = __fmul_rn(6.0f, g);
  if (threadIdx.x == 0) g_out[row] = g;
  uint2* crow = reinterpret_cast<uint2*>(codes + static_cast<size_t>(row) * (K / 2));
  uint8_t* srow = scales + static_cast<size_t>(row) * (K / 16);
  for (int sb = threadIdx.x; sb < K / 16; sb += T) {   // one subblock per thread and pass
    float4 v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = xr[4 * sb + j];
    quantize_subblock(v, g, six_g, crow + sb, srow + sb);
  }
}

// ---------------------------------------------------------------------------
// NVFP4 x NVFP4 GEMM
// ---------------------------------------------------------------------------
constexpr int kTile = 128;                 // weight rows per CTA (MMA M)
constexpr int kStageK = 256;               // K per stage: 128 code bytes per row
constexpr int kMmaK = 64;                  // K per block-scaled MMA
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitLimitNs = 4000000000ull;

// The tile shape: TN tokens per CTA (the MMA's N).  TN = 128: a 6-deep ring
// of 36 KB stages and two 128-column accumulators promoted every 1024 K.
// TN = 256: twice the products per byte in flight (the kernel is bound by the
// bytes it can keep in flight per SM against the memory latency), a 4-deep
// ring of 54 KB stages and one 256-column accumulator promoted every 4096 K
// (at most 64 accumulations in tensor memory, a relative error below
// 64 * 2^-23 of the sum of |terms|, inside the accuracy bound).
template <int TN>
struct Nvf4Cfg {
  static constexpr int kStages = TN == 128 ? 6 : 4;
  static constexpr int kBufs = TN == 128 ? 2 : 1;          // accumulator buffers
  static constexpr int kChunkStages = TN == 128 ? 4 : 16;  // stages per accumulator chunk
  static constexpr int kEpiWarps = TN / 16;                // 64 token columns per warp
  static constexpr int kThreads = 32 * (2 + kEpiWarps);
  static constexpr uint32_t kCodeA = kTile * kStageK / 2;  // 16 KB
  static constexpr uint32_t kCodeB = TN * kStageK / 2;     // 16 or 32 KB
  static constexpr uint32_t kScaleA = kTile * kStageK / 16;
  static constexpr uint32_t kScaleB = TN * kStageK / 16;
  static constexpr uint32_t kOffB = kCodeA;
  static constexpr uint32_t kOffSa = kCodeA + kCodeB;
  static constexpr uint32_t kOffSb = kOffSa + kScaleA;
  static constexpr uint32_t kSlot = kOffSb + kScaleB;
  static constexpr uint32_t kAccCols = TN;
  static constexpr uint32_t kSfCol0 = kBufs * kAccCols;
  static constexpr uint32_t kSfA = kTile / 32;             // columns per K step: weights
  static constexpr uint32_t kSfB = TN / 32;                //                     tokens
  static constexpr uint32_t kSfColsA = (kStageK / kMmaK) * kSfA;
  static constexpr uint32_t kSfColsPerStage = (kStageK / kMmaK) * (kSfA + kSfB);
  static constexpr int kNumBars = 3 * kStages + 2 * kBufs + 1;
  static constexpr uint32_t kSmemBytes = kStages * kSlot + kNumBars * 8 + 16 + 1024;
  static_assert(kSlot % 1024 == 0, "slots stay 1024-byte aligned for the 128-byte swizzle");
  static_assert(kSfCol0 + kStages * kSfColsPerStage <= kTmemCols, "tensor memory");
  static_assert(kSmemBytes <= 232448, "shared memory");
};

// bit 0: a pipeline wait timed out
__device__ unsigned int g_nvf4_error_flags = 0;

// Instruction descriptor of kind::mxf4nvf4 with block scaling: A and B E2M1
// (format 1), K-major, scale format E4M3 (bit 23 = 0), N >> 3 at bits
// 17-22, M >> 4 at bits 24-28, scale-factor byte ids 0 (bits 4-5, 29-30),
// dense K = 64 (bit 31 = 0).
__host__ __device__ constexpr uint32_t idesc_nvf4(int m, int n) {
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}

__device__ __forceinline__ void mma_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], "
      "[%6], p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// Scale-factor layout in tensor memory, per operand of R rows and per 64-wide
// K step: R/32 columns; lane i, column j holds the four scales (byte b for K
// block b) of row 32*j + i, the same in every lane quarter.  A lane writes the
// columns of one stage (4 K steps) of an R-row operand from the stage's
// R x 16 scale bytes in shared memory.
template <int R>
__device__ __forceinline__ void store_scales(uint32_t smem_scales, uint32_t taddr, int lane) {
  constexpr int J = R / 32;
  // 16 columns (four K steps of J = 4 row groups, or two of J = 8) at a time
  constexpr int kSteps = 16 / J;
#pragma unroll
  for (int h = 0; h < 4 / kSteps; ++h) {
    uint32_t v[16];
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const uint4 w = lds128(smem_scales + 16u * (32 * j + lane));
      const uint32_t wk[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int t = 0; t < kSteps; ++t) v[t * J + j] = wk[h * kSteps + t];
    }
    ptx::tmem_st_16cols(taddr + 16u * h, v);
  }
}

template <int TN>
__global__ void __launch_bounds__(Nvf4Cfg<TN>::kThreads, 1)
gemm_nvf4_kernel(const __grid_constant__ CUtensorMap wcode_map,
                 const __grid_constant__ CUtensorMap wscale_map,
                 const __grid_constant__ CUtensorMap acode_map,
                 const __grid_constant__ CUtensorMap ascale_map, int N, int K, int M,
                 float g_w, const float* __restrict__ g_a, float* __restrict__ y) {
  using C = Nvf4Cfg<TN>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_addr(smem_raw);
  const uint32_t sbase = raw + ((1024u - (raw & 1023u)) & 1023u);
  uint8_t* smem = smem_raw + (sbase - raw);
  const uint32_t bars = sbase + S * C::kSlot;
  auto full = [&](int s) { return bars + 8u * s; };
  auto sf_full = [&](int s) { return bars + 8u * (S + s); };
  auto empty = [&](int s) { return bars + 8u * (2 * S + s); };
  auto acc_full = [&](int b) { return bars + 8u * (3 * S + b); };
  auto acc_empty = [&](int b) { return bars + 8u * (3 * S + C::kBufs + b); };
  const uint32_t mma_done = bars + 8u * (C::kNumBars - 1);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + S * C::kSlot + C::kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  auto slot = [&](int s) { return sbase + s * C::kSlot; };

  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // token tiles vary fastest, so the CTAs of a wave share weight tiles
  const int m0 = blockIdx.x * TN;             // tokens
  const int n0 = blockIdx.y * kTile;          // weight rows
  const int num_k = K / kStageK;
  const int num_chunks = (num_k + C::kChunkStages - 1) / C::kChunkStages;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(full(s), 1);
      ptx::mbar_init(sf_full(s), 4);
      ptx::mbar_init(empty(s), 1);
    }
    for (int b = 0; b < C::kBufs; ++b) {
      ptx::mbar_init(acc_full(b), 1);
      ptx::mbar_init(acc_empty(b), C::kEpiWarps);
    }
    ptx::mbar_init(mma_done, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tensormap(&wcode_map);
    ptx::prefetch_tensormap(&wscale_map);
    ptx::prefetch_tensormap(&acode_map);
    ptx::prefetch_tensormap(&ascale_map);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_addr(tmem_holder), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  auto fail = [&]() {
    *abort_flag = 1;
    atomicOr(&g_nvf4_error_flags, 1u);
  };
  auto warp_wait = [&](uint32_t bar, uint32_t parity) -> bool {
    if (__all_sync(0xffffffffu, ptx::mbar_try_wait(bar, parity))) return true;
    const bool got = ptx::mbar_wait_bounded(bar, parity, abort_flag, kWaitLimitNs);
    return __all_sync(0xffffffffu, got);
  };

  if (warp == 0) {
    // ------------------------------- TMA producer ------------------------------
    // the weights are never written by the kernels before this one: the first
    // slots' weight tiles are requested before waiting for the token tiles
    const int early = min(num_k, S);
    if (lane == 0) {
      for (int k = 0; k < early; ++k) {
        ptx::mbar_arrive_expect_tx(full(k), C::kSlot);
        ptx::tma_load_2d(slot(k), &wcode_map, k * (kStageK / 2), n0, full(k));
        ptx::tma_load_2d(slot(k) + C::kOffSa, &wscale_map, k * (kStageK / 16), n0, full(k));
      }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (lane == 0) {
      for (int k = 0; k < early; ++k) {
        ptx::tma_load_2d(slot(k) + C::kOffB, &acode_map, k * (kStageK / 2), m0, full(k));
        ptx::tma_load_2d(slot(k) + C::kOffSb, &ascale_map, k * (kStageK / 16), m0, full(k));
      }
    }
    __syncwarp();
    int issued = early;
    for (int k = early; k < num_k; ++k) {
      const int s = k % S;
      if (!warp_wait(empty(s), ((k / S) & 1) ^ 1)) {
        fail();
        break;
      }
      if (lane == 0) {
        ptx::mbar_arrive_expect_tx(full(s), C::kSlot);
        ptx::tma_load_2d(slot(s), &wcode_map, k * (kStageK / 2), n0, full(s));
        ptx::tma_load_2d(slot(s) + C::kOffB, &acode_map, k * (kStageK / 2), m0, full(s));
        ptx::tma_load_2d(slot(s) + C::kOffSa, &wscale_map, k * (kStageK / 16), n0, full(s));
        ptx::tma_load_2d(slot(s) + C::kOffSb, &ascale_map, k * (kStageK / 16), m0, full(s));
      }
      __syncwarp();
      ++issued;
    }
    if (*abort_flag) {
      for (int k = max(0, issued - S); k < issued; ++k)
        ptx::mbar_wait_bounded(full(k % S), (k / S) & 1, nullptr, kWaitLimitNs);
    }
  } else if (warp == 1) {
    // -------------------------------- MMA issuer -------------------------------
    constexpr uint32_t idesc = idesc_nvf4(kTile, TN);
    bool ok = true;
    for (int c = 0; c < num_chunks && ok; ++c) {
      const int b = c % C::kBufs;
      // a buffer is reused once the epilogue drained its previous chunk
      if (c >= C::kBufs && !warp_wait(acc_empty(b), ((c / C::kBufs) - 1) & 1)) {
        fail();
        break;
      }
      const uint32_t d_tmem = tmem_base + b * C::kAccCols;
      const int k_end = min(num_k, (c + 1) * C::kChunkStages);
      for (int k = c * C::kChunkStages; k < k_end; ++k) {
        const int s = k % S;
        if (!warp_wait(sf_full(s), (k / S) & 1)) {
          fail();
          ok = false;
          break;
        }
        if (lane == 0) {
          ptx::tc_fence_after();
          const uint64_t adesc0 = ptx::sw128_kmajor_desc(slot(s));
          const uint64_t bdesc0 = ptx::sw128_kmajor_desc(slot(s) + C::kOffB);
          const uint32_t sf = tmem_base + C::kSfCol0 + s * C::kSfColsPerStage;
#pragma unroll
          for (int j = 0; j < kStageK / kMmaK; ++j) {
            // 64 E2M1 = 32 bytes per K step inside the 128-byte swizzled rows
            mma_nvf4(d_tmem, adesc0 + 2u * j, bdesc0 + 2u * j, idesc, sf + C::kSfA * j,
                     sf + C::kSfColsA + C::kSfB * j,
                     (k == c * C::kChunkStages && j == 0) ? 0u : 1u);
          }
          ptx::mma_commit(empty(s));
          if (k == k_end - 1) ptx::mma_commit(acc_full(b));
        }
        __syncwarp();
      }
    }
    if (lane == 0) ptx::mma_commit(mma_done);
    __syncwarp();
    ptx::mbar_wait_bounded(mma_done, 0, nullptr, kWaitLimitNs);
  } else {
    // ------------- scale factors to tensor memory; then the epilogue -----------
    const int q = warp & 3;                   // lane quarter
    const int part = (warp - 2) >> 2;         // token columns [64*part, 64*part + 64)
    const int r = q * 32 + lane;              // weight row of the accumulator lane
    const uint32_t tlane = static_cast<uint32_t>(q * 32) << 16;
    const bool mover = part == 0;
    float run[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) run[i] = 0.0f;
    int drained = 0;
    auto drain = [&]() -> bool {
      const int b = drained % C::kBufs;
      if (!warp_wait(acc_full(b), (drained / C::kBufs) & 1)) return false;
      ptx::tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t v[16];
        ptx::tmem_ld_16cols(tmem_base + tlane + b * C::kAccCols + 64 * part + 16 * cc, v);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) run[16 * cc + i] += __uint_as_float(v[i]);
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(acc_empty(b));
      ++drained;
      return true;
    };
    bool ok = true;
    for (int k = 0; k < num_k && ok; ++k) {
      // before the chunk that reuses a buffer, drain the chunk that used it
      if (k % C::kChunkStages == 0 && k / C::kChunkStages >= C::kBufs) {
        if (!drain()) {
          fail();
          ok = false;
          break;
        }
      }
      if (!mover) continue;
      const int s = k % S;
      if (!warp_wait(full(s), (k / S) & 1)) {
        fail();
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t sf = tmem_base + tlane + C::kSfCol0 + s * C::kSfColsPerStage;
      store_scales<kTile>(slot(s) + C::kOffSa, sf, lane);
      store_scales<TN>(slot(s) + C::kOffSb, sf + C::kSfColsA, lane);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(sf_full(s));
    }
    while (ok && drained < num_chunks) {
      if (!drain()) {
        fail();
        ok = false;
      }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (ok) {
      const int n = n0 + r;
      if (n < N) {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const int m = m0 + 64 * part + i;
          if (m < M) y[static_cast<size_t>(m) * N + n] = run[i] * (g_w * g_a[m]);
        }
      }
    }
  }

  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool encode_bytes_2d(CUtensorMap* map, const void* base, uint64_t row_bytes, uint64_t rows,
                     uint32_t box_bytes, uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = encoder();
  if (encode == nullptr) return false;
  const cuuint64_t dims[2] = {row_bytes, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_bytes, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

cudaLaunchAttribute pdl_attr() {
  cudaLaunchAttribute a = {};
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
  return a;
}

}  // namespace

cudaError_t launch_quantize_nvfp4(const float* x, int64_t M, int64_t K, uint8_t* codes,
                                  uint8_t* scales, float* g, cudaStream_t stream) {
  // one thread per subblock, about 256 per CTA, a row split over a cluster
  // of P <= 8 CTAs; rows of more than 2048 subblocks take the two-pass kernel
  const int64_t nsub = K / 16;
  const int64_t P = std::max<int64_t>(1, (nsub + 255) / 256);
  cudaLaunchConfig_t cfg = {};
  cfg.stream = stream;
  cudaLaunchAttribute attr[2] = {pdl_attr(), {}};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int k = static_cast<int>(K);
  if (P > 8) {
    cfg.gridDim = dim3(static_cast<unsigned>(M));
    cfg.blockDim = dim3(1024);
    return cudaLaunchKernelEx(&cfg, quantize_nvfp4_long_kernel, x, k, codes, scales, g);
  }
  const int64_t T = ((nsub + P - 1) / P + 31) / 32 * 32;
  cfg.gridDim = dim3(static_cast<unsigned>(M), static_cast<unsigned>(P));
  cfg.blockDim = dim3(static_cast<unsigned>(T));
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 1;
  attr[1].val.clusterDim.y = static_cast<unsigned>(P);
  attr[1].val.clusterDim.z = 1;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, quantize_nvfp4_kernel, x, k, codes, scales, g);
}

template <int TN>
cudaError_t launch_nvf4_t(const uint8_t* w_codes, const uint8_t* w_scales, float g_w, int64_t N,
                          int64_t K, const uint8_t* a_codes, const uint8_t* a_scales,
                          const float* g_a, int64_t M, float* y, cudaStream_t stream) {
  using C = Nvf4Cfg<TN>;
  CUtensorMap wc, ws, ac, as;
  if (!encode_bytes_2d(&wc, w_codes, K / 2, N, 128, kTile, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_bytes_2d(&ws, w_scales, K / 16, N, 16, kTile, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_bytes_2d(&ac, a_codes, K / 2, M, 128, TN, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_bytes_2d(&as, a_scales, K / 16, M, 16, TN, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  static SmemAttrOnce attr;
  cudaError_t e = attr.ensure(gemm_nvf4_kernel<TN>, static_cast<int>(C::kSmemBytes));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((M + TN - 1) / TN),
                     static_cast<unsigned>((N + kTile - 1) / kTile));
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute a[1] = {pdl_attr()};
  cfg.attrs = a;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_nvf4_kernel<TN>, wc, ws, ac, as, static_cast<int>(N),
                            static_cast<int>(K), static_cast<int>(M), g_w, g_a, y);
}

cudaError_t launch_gemm_nvf4(const uint8_t* w_codes, const uint8_t* w_scales, float g_w,
                             int64_t N, int64_t K, const uint8_t* a_codes,
                             const uint8_t* a_scales, const float* g_a, int64_t M, float* y,
                             cudaStream_t stream) {
  // the 256-token tile when its grid still fills every SM at least twice
  const int64_t tiles256 = ((M + 255) / 256) * ((N + kTile - 1) / kTile);
  if (tiles256 >= 2 * static_cast<int64_t>(device_sm_count()))
    return launch_nvf4_t<256>(w_codes, w_scales, g_w, N, K, a_codes, a_scales, g_a, M, y, stream);
  return launch_nvf4_t<128>(w_codes, w_scales, g_w, N, K, a_codes, a_scales, g_a, M, y, stream);
}

cudaError_t nvf4_error_flags(bool clear, unsigned int* flags) {
  cudaError_t e = cudaMemcpyFromSymbol(flags, g_nvf4_error_flags, sizeof(unsigned int));
  if (e == cudaSuccess && clear) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_nvf4_error_flags, &zero, sizeof(zero));
  }
  return e;
}

}  // namespace nvq
