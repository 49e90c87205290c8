// Small-token GEMM on the tcgen05 tensor cores: y[M, N] = A[M, K] . W[N, K]^T
// for M = 1..16 tokens (the small-batch decode of several sequences),
// NVFP4 weights and Q8_0 activations.
//
// The arithmetic is that of the prefill GEMM ("TKintegers K5: 3.21x prefill
// and 3.10x decode throughput vs TorchAO FP8 on NVIDIA L4": compact weight
// tiles expanded to FP16 tensor-core operands with FP32 accumulation; the
// per-16 scaled dot of "HANDOFF: flint CPU optimization (Q4_1 + NVFP4)",
// section 3): the weights are expanded to the exact fp16 w' = E2M1*s_w, the
// activations to the exact fp16 pair hi + lo = d*q, every product is exact
// and only the fp32 accumulation rounds.  At a few tokens the product is
// bound by HBM (0.5625 bytes per weight, read once) and by the CUDA-core
// work of expanding the weights, not by the tensor core, so the schedule is
// built around the expansion:
//
//  * one CTA per SM (persistent); the work, (128-row weight tile, 256-wide
//    K stage) units, is split into equal contiguous ranges of units in
//    tile-major order (stream-K), so every SM expands the same number of
//    weights whatever the shape.  A tile covered by one CTA is written to y
//    directly; a tile split between CTAs leaves fp32 partial sums in the
//    workspace, which a second small kernel adds in a fixed order;
//  * warp 0 streams each stage with TMA: the 128 x 128-byte tile of packed
//    codes (128-byte swizzle), the 128 x 16-byte tile of UE4M3 scales and
//    the four 64-wide sub-tiles of the expanded activations (hi rows then lo
//    rows of every token, 128-byte swizzle), into a 4-deep shared ring;
//  * warps 2..17 (four per tensor-memory lane quarter, each taking 64 of a
//    stage's 256 K) expand the codes to fp16 w' and store them with
//    tcgen05.st into a 3-deep ring in tensor memory (row r in lane r);
//  * warps 1 and 18 (on different sub-partitions: one thread issues a small
//    MMA only every ~70 cycles, far below the tensor core's rate) issue
//    tcgen05.mma.kind::f16 (M = 128, N = 2 x padded tokens: hi and lo
//    columns side by side, K = 16) with A from tensor memory and B from
//    shared memory, 8 each per stage (the K steps of one parity) into their
//    own accumulators; these are promoted to fp32 registers every 1024 K
//    (4 stages), alternating between two tensor-memory buffers each (the
//    tensor core's fp32 accumulation truncates, so long chains are split);
//  * the four warps with the first K part also drain the accumulators (the
//    two issuers' added in a fixed order) and write y = g * tok_scale * (hi + lo).
// Every wait is bounded (4 s); a timeout raises an error flag and the CTA
// drains what it issued before freeing tensor memory and leaving.
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

constexpr int kRows = 128;            // weight rows per tile = TMEM lanes = MMA M
constexpr int kStageK = 256;          // K per stage
constexpr int kSubK = 64;             // K per 128-byte fp16 swizzle row (one activation box)
constexpr int kSubs = kStageK / kSubK;
constexpr int kSmemStages = 4;        // shared-memory ring (codes, scales, activations)
constexpr int kAStages = 3;           // tensor-memory ring of expanded weights
constexpr int kChunkStages = 4;       // stages accumulated per TMEM buffer (1024 K)
constexpr int kDecWarps = 16;
constexpr int kIssuers = 2;          // MMA-issuing warps (1 and kIssuer2)
constexpr int kIssuer2 = 2 + kDecWarps;   // warp 18: another sub-partition than warp 1
constexpr int kThreads = 32 * (3 + kDecWarps);
constexpr uint32_t kACols = kStageK / 2;                 // 128 columns per A stage
constexpr uint32_t kAccCol0 = kAStages * kACols;         // 384: accumulators after the A ring
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitLimitNs = 4000000000ull;
constexpr int kMaxCtas = 256;                            // bound of the partial-sum slots

constexpr uint32_t kCodeBytes = kRows * kStageK / 2;     // 16 KB
constexpr uint32_t kScaleBytes = kRows * kStageK / 16;   // 2 KB

// shared memory of one ring slot: codes | activation sub-tiles | scales
__host__ __device__ constexpr uint32_t act_sub_bytes(int n) { return static_cast<uint32_t>(n) * 128; }
__host__ __device__ constexpr uint32_t slot_bytes(int n) {
  return kCodeBytes + kSubs * act_sub_bytes(n) + kScaleBytes;
}
// barriers: full[4] empty[4] a_full[3] a_empty[3] acc_full[2] acc_empty[2] mma_done
constexpr int kNumBars = 2 * kSmemStages + 2 * kAStages + 4 + 1;
__host__ __device__ constexpr uint32_t smem_bytes(int n) {
  return kSmemStages * slot_bytes(n) + kNumBars * 8 + 16 + 1024;
}
static_assert(slot_bytes(16) % 1024 == 0 && slot_bytes(32) % 1024 == 0, "1 KB aligned slots");
static_assert(smem_bytes(32) <= 232448, "over the opt-in shared memory of one CTA");
static_assert(kAccCol0 + kIssuers * 2 * 32 <= kTmemCols, "tensor memory");

// bit 0: a pipeline wait timed out
__device__ unsigned int g_gemm_small_error_flags = 0;

// The CTA whose unit range [u0(c), u0(c+1)) holds unit u, u0(c) = c*W/G.
__host__ __device__ __forceinline__ int64_t unit_begin(int64_t c, int64_t W, int64_t G) {
  return c * W / G;
}

// Slot and phase of a ring of `depth` stages, advanced one stage at a time.
struct Ring {
  int depth;
  int slot = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void advance() {
    if (++slot == depth) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

// Iterates the (tile, stage range) pieces of a CTA's unit range.
struct Pieces {
  int64_t u, u_end, Ks;
  __device__ bool next(int& t, int& j0, int& j1) {
    if (u >= u_end) return false;
    t = static_cast<int>(u / Ks);
    j0 = static_cast<int>(u % Ks);
    const int64_t left = u_end - u;
    j1 = static_cast<int>(j0 + left < Ks ? j0 + left : Ks);
    u += j1 - j0;
    return true;
  }
};

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

template <int NT>   // MMA N = 2 * padded tokens (16 or 32)
__global__ void __launch_bounds__(kThreads, 1)
gemm_small_kernel(const __grid_constant__ CUtensorMap code_map,
                  const __grid_constant__ CUtensorMap scale_map,
                  const __grid_constant__ CUtensorMap act_map, int N, int K, int M,
                  float g, const float* __restrict__ tok_scale, float* __restrict__ y,
                  float* __restrict__ partial) {
  constexpr int MP = NT / 2;                     // padded tokens
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_addr(smem_raw);
  const uint32_t sbase = raw + ((1024u - (raw & 1023u)) & 1023u);
  uint8_t* smem = smem_raw + (sbase - raw);
  const uint32_t bars = sbase + kSmemStages * slot_bytes(NT);
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (kSmemStages + s); };
  auto a_full = [&](int s) { return bars + 8u * (2 * kSmemStages + s); };
  auto a_empty = [&](int s) { return bars + 8u * (2 * kSmemStages + kAStages + s); };
  auto acc_full = [&](int b) { return bars + 8u * (2 * kSmemStages + 2 * kAStages + b); };
  auto acc_empty = [&](int b) { return bars + 8u * (2 * kSmemStages + 2 * kAStages + 2 + b); };
  const uint32_t mma_done = bars + 8u * (kNumBars - 1);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + (bars - sbase) + kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  auto slot_addr = [&](int s) { return sbase + s * slot_bytes(NT); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t Ks = K / kStageK;
  const int64_t T = (N + kRows - 1) / kRows;
  const int64_t W = T * Ks;
  const int64_t G = gridDim.x;
  const int64_t c = blockIdx.x;
  const int64_t u0 = unit_begin(c, W, G), u1 = unit_begin(c + 1, W, G);
  const int t_first = static_cast<int>(u0 / Ks);

  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (threadIdx.x == 0) {
    for (int s = 0; s < kSmemStages; ++s) {
      ptx::mbar_init(full(s), 1);
      ptx::mbar_init(empty(s), kIssuers);
    }
    for (int s = 0; s < kAStages; ++s) {
      ptx::mbar_init(a_full(s), kDecWarps);
      ptx::mbar_init(a_empty(s), kIssuers);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(acc_full(b), kIssuers);
      ptx::mbar_init(acc_empty(b), 4);
    }
    ptx::mbar_init(mma_done, kIssuers);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tensormap(&code_map);
    ptx::prefetch_tensormap(&scale_map);
    ptx::prefetch_tensormap(&act_map);
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
    atomicOr(&g_gemm_small_error_flags, 1u);
  };
  // whole warp waits, outcome warp-uniform
  auto warp_wait = [&](uint32_t bar, uint32_t parity) -> bool {
    if (__all_sync(0xffffffffu, ptx::mbar_try_wait(bar, parity))) return true;
    const bool got = ptx::mbar_wait_bounded(bar, parity, abort_flag, kWaitLimitNs);
    return __all_sync(0xffffffffu, got);
  };

  if (warp == 0) {
    // ------------------------------ TMA producer -------------------------------
    // The weights are never written by the kernels before this one, so the
    // codes and scales of the first ring slots are requested before waiting
    // for the previous kernel (the activation expansion); the activations of
    // those slots follow the wait.
    auto load_weights = [&](uint32_t dst, uint32_t bar, int t, int j) {
      ptx::tma_load_2d(dst, &code_map, j * (kStageK / 2), t * kRows, bar);
      ptx::tma_load_2d(dst + kCodeBytes + kSubs * act_sub_bytes(NT), &scale_map,
                       j * (kStageK / 16), t * kRows, bar);
    };
    auto load_acts = [&](uint32_t dst, uint32_t bar, int j) {
#pragma unroll
      for (int sub = 0; sub < kSubs; ++sub)
        ptx::tma_load_2d(dst + kCodeBytes + sub * act_sub_bytes(NT), &act_map,
                         j * kStageK + sub * kSubK, 0, bar);
    };
    int early_j[kSmemStages];
    int early = 0;
    {
      Pieces pc{u0, u1, Ks};
      int t, j0, j1;
      while (early < kSmemStages && pc.next(t, j0, j1)) {
        for (int j = j0; j < j1 && early < kSmemStages; ++j, ++early) {
          if (lane == 0) {
            ptx::mbar_arrive_expect_tx(full(early), slot_bytes(NT));
            load_weights(slot_addr(early), full(early), t, j);
          }
          early_j[early] = j;
        }
      }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (lane == 0)
      for (int e = 0; e < early; ++e) load_acts(slot_addr(e), full(e), early_j[e]);
    __syncwarp();
    Pieces pc{u0, u1, Ks};
    int t, j0, j1;
    Ring sm{kSmemStages};
    int issued = 0;
    bool ok = true;
    while (ok && pc.next(t, j0, j1)) {
      for (int j = j0; j < j1; ++j, sm.advance()) {
        if (issued < early) {   // requested above
          ++issued;
          continue;
        }
        if (!warp_wait(empty(sm.slot), sm.phase ^ 1u)) {
          fail();
          ok = false;
          break;
        }
        if (lane == 0) {
          const uint32_t dst = slot_addr(sm.slot);
          const uint32_t bar = full(sm.slot);
          ptx::mbar_arrive_expect_tx(bar, slot_bytes(NT));
          load_weights(dst, bar, t, j);
          load_acts(dst, bar, j);
        }
        __syncwarp();
        ++issued;
      }
    }
    if (!ok) {
      // let this CTA's copies in flight land before it can leave
      for (int k = max(0, issued - kSmemStages); k < issued; ++k)
        ptx::mbar_wait_bounded(full(k % kSmemStages), static_cast<uint32_t>((k / kSmemStages) & 1),
                               nullptr, kWaitLimitNs);
    }
  } else if (warp == 1 || warp == kIssuer2) {
    // ------------------------------ MMA issuers ---------------------------------
    // One thread issues a small MMA only every ~70 cycles, far slower than the
    // tensor core runs it, so two warps on different sub-partitions issue:
    // issuer i takes the K steps of parity i of every stage into its own
    // double-buffered accumulator (the drain adds the two).
    const int is = warp == 1 ? 0 : 1;
    constexpr uint32_t idesc = ptx::idesc_f16_f32(kRows, NT);
    Pieces pc{u0, u1, Ks};
    int t, j0, j1;
    Ring sm{kSmemStages}, ar{kAStages};
    int ch = 0;
    bool ok = true;
    while (ok && pc.next(t, j0, j1)) {
      for (int jc = j0; jc < j1 && ok; jc += kChunkStages, ++ch) {
        const int b = ch & 1;
        if (ch >= 2 && !warp_wait(acc_empty(b), static_cast<uint32_t>(((ch >> 1) - 1) & 1))) {
          fail();
          ok = false;
          break;
        }
        const uint32_t d_tmem = tmem_base + kAccCol0 + (is * 2 + b) * NT;
        const int je = min(j1, jc + kChunkStages);
        for (int j = jc; j < je; ++j, sm.advance(), ar.advance()) {
          if (!warp_wait(full(sm.slot), sm.phase) || !warp_wait(a_full(ar.slot), ar.phase)) {
            fail();
            ok = false;
            break;
          }
          if (lane == 0) {
            ptx::tc_fence_after();
            const uint32_t a_cols = tmem_base + ar.slot * kACols;
            const uint64_t bdesc0 = ptx::sw128_kmajor_desc(slot_addr(sm.slot) + kCodeBytes);
#pragma unroll
            for (int sub = 0; sub < kSubs; ++sub) {
#pragma unroll
              for (int k = is; k < kSubK / 16; k += kIssuers) {
                const uint32_t a = a_cols + sub * (kSubK / 2) + 8u * k;
                const uint64_t bd = bdesc0 + ((sub * act_sub_bytes(NT)) >> 4) + 2u * k;
                ptx::mma_f16_ts(d_tmem, a, bd, idesc, (j == jc && sub == 0 && k == is) ? 0u : 1u);
              }
            }
            ptx::mma_commit(empty(sm.slot));
            ptx::mma_commit(a_empty(ar.slot));
            if (j == je - 1) ptx::mma_commit(acc_full(b));
          }
          __syncwarp();
        }
      }
    }
    // no MMA may still be running when tensor memory is released
    if (lane == 0) ptx::mma_commit(mma_done);
    __syncwarp();
    ptx::mbar_wait_bounded(mma_done, 0, nullptr, kWaitLimitNs);
  } else {
    // ------------------ weight expansion, then the epilogue --------------------
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int p = (warp - 2) >> 2;          // K part of the stage: 64 elements
    const int r = q * 32 + lane;            // tile row = TMEM lane
    const uint32_t tlane = static_cast<uint32_t>(q * 32) << 16;
    const bool drainer = p == 0;
    // y, the partial sums and tok_scale are touched only after the previous
    // kernels are complete
    if (drainer) asm volatile("griddepcontrol.wait;" ::: "memory");
    const uint32_t row_off = r * 128u;
    const uint32_t sw = static_cast<uint32_t>(r & 7);
    const uint32_t c0_off = row_off + ((2u * p) ^ sw) * 16u;
    const uint32_t c1_off = row_off + ((2u * p + 1u) ^ sw) * 16u;
    const uint32_t s_off = kCodeBytes + kSubs * act_sub_bytes(NT) + r * 16u + 4u * p;
    float run[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) run[n] = 0.0f;

    // drain cursor: walks the same pieces and chunks as the MMA issuer
    Pieces dpc{u0, u1, Ks};
    int dt = 0, dj0 = 0, dj1 = 0;
    bool dvalid = dpc.next(dt, dj0, dj1);
    int djc = dj0;
    int drained = 0;
    auto drain_one = [&]() -> bool {
      const int b = drained & 1;
      if (!warp_wait(acc_full(b), static_cast<uint32_t>((drained >> 1) & 1))) return false;
      ptx::tc_fence_after();
      // the two issuers' accumulators of buffer b, added in a fixed order
#pragma unroll
      for (int i = 0; i < kIssuers; ++i) {
#pragma unroll
        for (int h = 0; h < NT / 16; ++h) {
          uint32_t v[16];
          ptx::tmem_ld_16cols(tmem_base + tlane + kAccCol0 + (i * 2 + b) * NT + 16 * h, v);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int n = 0; n < 16; ++n) run[16 * h + n] += __uint_as_float(v[n]);
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(acc_empty(b));
      ++drained;
      djc += kChunkStages;
      if (djc >= dj1) {
        // the piece is complete: write it
        const int row = dt * kRows + r;
        if (dj0 == 0 && dj1 == Ks) {
          if (row < N) {
#pragma unroll
            for (int m = 0; m < MP; ++m)
              if (m < M) y[static_cast<size_t>(m) * N + row] = (run[m] + run[MP + m]) * (g * tok_scale[m]);
          }
        } else {
          const int slot = dt == t_first ? 0 : 1;
          float* dst = partial + (static_cast<size_t>(c) * 2 + slot) * MP * kRows;
#pragma unroll
          for (int m = 0; m < MP; ++m) dst[m * kRows + r] = run[m] + run[MP + m];
        }
#pragma unroll
        for (int n = 0; n < NT; ++n) run[n] = 0.0f;
        dvalid = dpc.next(dt, dj0, dj1);
        djc = dj0;
      }
      return true;
    };

    Pieces pc{u0, u1, Ks};
    int t, j0, j1;
    Ring sm{kSmemStages}, ar{kAStages};
    int ch = 0;
    int prev_slot = -1;                      // A stage stored but not yet announced
    bool ok = true;
    // The store of a stage is waited for (and the stage announced to the MMA
    // issuer) only after the next stage is decoded, so the tensor-memory
    // store latency overlaps the decode instead of stalling the warp.
    auto announce_prev = [&]() {
      if (prev_slot >= 0) {
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(a_full(prev_slot));
        prev_slot = -1;
      }
    };
    while (ok && pc.next(t, j0, j1)) {
      int in_chunk = 0;
      for (int j = j0; j < j1; ++j, sm.advance(), ar.advance()) {
        if (in_chunk == 0) {
          // before the chunk that reuses a buffer, drain the chunk that used it
          if (drainer && ch >= 2) {
            announce_prev();
            if (!drain_one()) {
              fail();
              ok = false;
              break;
            }
          }
          ++ch;
        }
        in_chunk = in_chunk + 1 == kChunkStages ? 0 : in_chunk + 1;
        if (!warp_wait(full(sm.slot), sm.phase)) {
          fail();
          ok = false;
          break;
        }
        const uint32_t slot = slot_addr(sm.slot);
        const uint4 c0 = lds128(slot + c0_off);
        const uint4 c1 = lds128(slot + c1_off);
        const uint32_t sc = lds32(slot + s_off);
        const __half2 sp01 = dev::ue4m3x2_to_half2(sc & 0xFFFFu);
        const __half2 sp23 = dev::ue4m3x2_to_half2(sc >> 16);
        const __half2 s0 = __low2half2(sp01), s1 = __high2half2(sp01);
        const __half2 s2 = __low2half2(sp23), s3 = __high2half2(sp23);
        const uint4 e0 = dev::expand8(c0.x, s0), e1 = dev::expand8(c0.y, s0);
        const uint4 e2 = dev::expand8(c0.z, s1), e3 = dev::expand8(c0.w, s1);
        const uint4 e4 = dev::expand8(c1.x, s2), e5 = dev::expand8(c1.y, s2);
        const uint4 e6 = dev::expand8(c1.z, s3), e7 = dev::expand8(c1.w, s3);
        const uint32_t v[32] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w,
                                e2.x, e2.y, e2.z, e2.w, e3.x, e3.y, e3.z, e3.w,
                                e4.x, e4.y, e4.z, e4.w, e5.x, e5.y, e5.z, e5.w,
                                e6.x, e6.y, e6.z, e6.w, e7.x, e7.y, e7.z, e7.w};
        announce_prev();
        if (!warp_wait(a_empty(ar.slot), ar.phase ^ 1u)) {
          fail();
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        ptx::tmem_st_32cols(tmem_base + tlane + ar.slot * kACols + p * 32u, v);
        prev_slot = ar.slot;
      }
    }
    if (ok) announce_prev();
    // the chunks not drained yet
    while (ok && drainer && dvalid) {
      if (!drain_one()) {
        fail();
        ok = false;
      }
    }
  }

  // nobody leaves (or frees tensor memory) while MMAs may still run
  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, kTmemCols);
  }
}

// Adds the partial sums of the tiles that several CTAs shared, in CTA order,
// and writes y.  One block of 128 threads (rows) per tile.
template <int MP>
__global__ void __launch_bounds__(kRows)
gemm_small_reduce_kernel(const float* __restrict__ partial, int N, int K, int M, int G,
                         float g, const float* __restrict__ tok_scale, float* __restrict__ y) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t Ks = K / kStageK;
  const int64_t T = (N + kRows - 1) / kRows;
  const int64_t W = T * Ks;
  const int64_t t = blockIdx.x;
  auto cta_of = [&](int64_t u) {
    int64_t cc = u * G / W;
    while (cc + 1 < G && unit_begin(cc + 1, W, G) <= u) ++cc;
    while (cc > 0 && unit_begin(cc, W, G) > u) --cc;
    return cc;
  };
  const int64_t ca = cta_of(t * Ks), cb = cta_of((t + 1) * Ks - 1);
  if (ca == cb) return;                      // one CTA wrote this tile itself
  const int r = threadIdx.x;
  const int row = static_cast<int>(t * kRows + r);
  if (row >= N) return;
  float acc[MP];
#pragma unroll
  for (int m = 0; m < MP; ++m) acc[m] = 0.0f;
  for (int64_t cc = ca; cc <= cb; ++cc) {
    const int slot = (unit_begin(cc, W, G) / Ks == t) ? 0 : 1;
    const float* src = partial + (static_cast<size_t>(cc) * 2 + slot) * MP * kRows;
#pragma unroll
    for (int m = 0; m < MP; ++m) acc[m] += src[m * kRows + r];
  }
#pragma unroll
  for (int m = 0; m < MP; ++m)
    if (m < M) y[static_cast<size_t>(m) * N + row] = acc[m] * (g * tok_scale[m]);
}

// fp16 activations (W4A16) into the operand layout of the small-token
// schedule: hi rows = x (exact), lo rows = 0, rows >= M zero, token scales 1.
__global__ void __launch_bounds__(256)
expand_f16_kernel(const uint4* __restrict__ x, int M, int K, int MP, uint4* __restrict__ act,
                  float* __restrict__ tok_scale) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int row = blockIdx.x;
  const int K8 = K / 8;
  uint4* hi = act + static_cast<size_t>(row) * K8;
  uint4* lo = act + static_cast<size_t>(MP + row) * K8;
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  for (int i = threadIdx.x; i < K8; i += blockDim.x) {
    hi[i] = row < M ? x[static_cast<size_t>(row) * K8 + i] : z;
    lo[i] = z;
  }
  if (threadIdx.x == 0) tok_scale[row] = 1.0f;
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

bool encode_2d(CUtensorMap* map, CUtensorMapDataType type, const void* base, uint64_t inner,
               uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
               CUtensorMapSwizzle swizzle) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = encoder();
  if (encode == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return encode(map, type, 2, const_cast<void*>(base), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int64_t small_padded_tokens(int64_t M) { return M <= 8 ? 8 : 16; }

struct SmallLayout {
  int64_t mp;
  size_t act, tok, partial, total;
};

SmallLayout small_layout(int64_t M, int64_t K) {
  SmallLayout L;
  L.mp = small_padded_tokens(M);
  L.act = 0;
  L.tok = static_cast<size_t>(4 * L.mp * K);
  L.partial = (L.tok + 4 * L.mp + 255) / 256 * 256;
  L.total = L.partial + static_cast<size_t>(kMaxCtas) * 2 * L.mp * kRows * 4;
  return L;
}

template <int NT>
cudaError_t launch_small(const uint8_t* codes, const uint8_t* scales, float g, int64_t N,
                         int64_t K, int64_t M, float* y, const SmallLayout& L, uint8_t* ws,
                         cudaStream_t stream) {
  CUtensorMap code_map, scale_map, act_map;
  if (!encode_2d(&code_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, K / 2, N, K / 2, 128, kRows,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&scale_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, scales, K / 16, N, K / 16, 16, kRows,
                 CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_2d(&act_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ws + L.act, K, NT, K * 2, kSubK, NT,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  static SmemAttrOnce attr;
  cudaError_t e = attr.ensure(gemm_small_kernel<NT>, static_cast<int>(smem_bytes(NT)));
  if (e != cudaSuccess) return e;
  const int64_t T = (N + kRows - 1) / kRows;
  const int64_t W = T * (K / kStageK);
  const int64_t G = std::min<int64_t>({static_cast<int64_t>(device_sm_count()), W,
                                        static_cast<int64_t>(kMaxCtas)});
  const float* tok = reinterpret_cast<const float*>(ws + L.tok);
  float* partial = reinterpret_cast<float*>(ws + L.partial);
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(G));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem_bytes(NT);
    cfg.stream = stream;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, gemm_small_kernel<NT>, code_map, scale_map, act_map,
                           static_cast<int>(N), static_cast<int>(K), static_cast<int>(M), g, tok,
                           y, partial);
    if (e != cudaSuccess) return e;
  }
  // a tile is split between CTAs when a CTA's range starts inside it
  const int64_t Ks = K / kStageK;
  bool split = false;
  for (int64_t cc = 1; cc < G && !split; ++cc) split = unit_begin(cc, W, G) % Ks != 0;
  if (!split) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(T));
  cfg.blockDim = dim3(kRows);
  cfg.stream = stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_small_reduce_kernel<NT / 2>,
                            static_cast<const float*>(partial), static_cast<int>(N),
                            static_cast<int>(K), static_cast<int>(M), static_cast<int>(G), g,
                            tok, y);
}

}  // namespace

bool gemm_small_supported(int64_t M, int64_t K) {
  return M >= 1 && M <= 16 && K % kStageK == 0;
}

size_t gemm_small_workspace_size(int64_t M, int64_t K) { return small_layout(M, K).total; }

cudaError_t launch_gemm_small(const uint8_t* codes, const uint8_t* scales, float g, int64_t N,
                              int64_t K, const int8_t* q, const uint16_t* d, int64_t M, float* y,
                              void* workspace, cudaStream_t stream) {
  const SmallLayout L = small_layout(M, K);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaError_t e = expand_activations(q, d, M, L.mp, K, ws + L.act,
                                     reinterpret_cast<float*>(ws + L.tok), stream);
  if (e != cudaSuccess) return e;
  if (L.mp == 8) return launch_small<16>(codes, scales, g, N, K, M, y, L, ws, stream);
  return launch_small<32>(codes, scales, g, N, K, M, y, L, ws, stream);
}

cudaError_t launch_gemm_small_f16(const uint8_t* codes, const uint8_t* scales, float g,
                                  int64_t N, int64_t K, const uint16_t* x, int64_t M, float* y,
                                  void* workspace, cudaStream_t stream) {
  const SmallLayout L = small_layout(M, K);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(L.mp));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, expand_f16_kernel, reinterpret_cast<const uint4*>(x),
                                     static_cast<int>(M), static_cast<int>(K),
                                     static_cast<int>(L.mp), reinterpret_cast<uint4*>(ws + L.act),
                                     reinterpret_cast<float*>(ws + L.tok));
  if (e != cudaSuccess) return e;
  if (L.mp == 8) return launch_small<16>(codes, scales, g, N, K, M, y, L, ws, stream);
  return launch_small<32>(codes, scales, g, N, K, M, y, L, ws, stream);
}

cudaError_t gemm_small_error_flags(bool clear, unsigned int* flags) {
  cudaError_t e = cudaMemcpyFromSymbol(flags, g_gemm_small_error_flags, sizeof(unsigned int));
  if (e == cudaSuccess && clear) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_gemm_small_error_flags, &zero, sizeof(zero));
  }
  return e;
}

}  // namespace nvq
