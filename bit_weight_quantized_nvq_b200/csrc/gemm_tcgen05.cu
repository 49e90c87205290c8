// Prefill GEMM on the 5th-generation tensor cores (tcgen05, TMEM, TMA):
//   y[M, N] = A[M, K] . W[N, K]^T,  NVFP4 weights, Q8_0 activations.
//
// The tiled prefill kernels of "HANDOFF: flint CPU optimization (Q4_1 +
// NVFP4)", section 3, unpack NVFP4 weight tiles and Q8_0 activation tiles
// and accumulate per-16 scaled integer sums; the K5 runtime of "TKintegers
// K5: 3.21x prefill and 3.10x decode throughput vs TorchAO FP8 on NVIDIA L4"
// expands compact weight tiles to FP16 tensor-core operands with FP32
// accumulation.  This kernel keeps the exact arithmetic of the first with
// the operand expansion of the second:
//
//  * weights: w' = E2M1(code) * s_w is exact in fp16 (at most 6 significant
//    bits, range 2^-10 .. 2688), so the per-16 rescale is folded into the
//    operand, expanded into tensor memory from the packed codes;
//  * activations: a = d*q has at most 18 significant bits, so it is split
//    into the exact fp16 pair hi = fp16(a), lo = fp16(a - hi) (hi + lo == a;
//    lo is a multiple of the ulp of d and below half an ulp of hi);
//  * every product w'*hi and w'*lo is exact in fp32; the tensor core sums
//    them in fp32, and y = g * 0.5 * sum(c*s*d*q) = g * (acc_hi + acc_lo).
//  * the tensor core's fp32 accumulation does not round to nearest (its
//    error grows with the number of chained MMAs and is biased toward
//    zero: about 1e-5 of sum|terms| after 1600 of them at K = 25600), so
//    partial sums are promoted: each chunk of up to 5120 K accumulates in TMEM
//    and the epilogue threads add it (hi + lo) to the tile's running sum in
//    fp32 (round to nearest).
//
// Kernels:
//  1. expand_act_kernel: Q8_0 (q, d) -> fp16 [hi rows | lo rows] in the
//     caller's workspace, once per call (tokens padded to 128 with zeros).
//     A token whose largest |d*q| would overflow fp16 (|x| > 65504) is
//     scaled by 2^-e first and the epilogue multiplies by 2^e.
//  2. gemm_kernel: persistent CTA pairs (clusters of 2, one per two SMs).
//     A tile is 128 tokens x 256 weight rows; each CTA owns 128 of the rows
//     and the even CTA issues tcgen05.mma.cta_group::2 (M = 256, N = 256,
//     K = 16) for both.  Whole tiles go round-robin over the pairs; the K
//     stages of the last partial wave's tiles are split evenly over all
//     pairs (PairWork).  Roles:
//       warp 0    TMA: this CTA's hi and lo rows of 64 of the tokens, for
//                 the two 64-wide K sub-tiles of a 128-wide stage (four
//                 64 x 64 fp16 boxes, 128-byte swizzle), into a 4-stage ring;
//       warp 1    allocates the pair's 512 TMEM columns; in the even CTA it
//                 waits for each stage and issues 8 pair MMAs (M = 256,
//                 N = 256, K = 16): each CTA's B rows are its 64 tokens' hi
//                 rows followed by their lo rows, one 128-row operand, so a
//                 single MMA forms the hi and the lo products of all 128
//                 tokens in 256 accumulator columns.  A is read from tensor
//                 memory and B from both CTAs' shared memory;
//       warps 2-9 two threads per weight row, one per sub-tile: cp.async the
//                 packed codes and scales, decode them to fp16 w' and
//                 tcgen05.st them into the 4-stage A ring in tensor memory
//                 (row m in lane m); drain each finished K chunk (hi + lo
//                 of each token) into y (a whole tile's last chunk, scaled)
//                 or the fp32 part slot of the workspace;
//       warp 10   forwards "this CTA's rows of the stage landed" to the even
//                 CTA's stage barrier.
//     Every role runs with its whole warp converged on the waits (a wait in
//     a diverged lane stalls the issuing loop by ~150-200 cycles a stage)
//     and one lane issuing.  Every wait is bounded (4 s); a timeout raises
//     an error flag and the CTA drains what it issued, and the pair frees
//     TMEM together after a cluster barrier.  No CTA waits for another
//     pair.
//  3. gemm_fixup_kernel: y of the tiles whose stages were split, the parts
//     added in K order (results do not depend on timing).
#include <algorithm>
#include <atomic>
#include <climits>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include "nvq_device.cuh"
#include "nvq_internal.h"
#include "tcgen05.cuh"

namespace nvq {
namespace {

constexpr int kBN = 128;            // weight rows per CTA = TMEM lanes
constexpr int kBT = 128;            // tokens per tile; the pair MMA's N = 256 holds their hi and lo
constexpr int kBTc = kBT / 2;       // tokens whose hi and lo rows one CTA of the pair loads
constexpr int kBK = 128;            // K per stage: two 64-wide sub-tiles
constexpr int kSubK = 64;           // K per 128-byte fp16 swizzle row (TMA box, MMA tile)
constexpr int kSubs = kBK / kSubK;
constexpr int kStages = 4;          // pipeline depth: activation ring (shared memory) and
                                    // expanded-weight ring (tensor memory) advance together
constexpr int kCStages = 6;         // packed-weight staging (shared memory)
constexpr int kTPR = 2;             // expansion threads per weight row: one per sub-tile
constexpr int kExpThreads = kTPR * kBN;   // weight expansion + epilogue
constexpr int kExpWarps = kExpThreads / 32;
constexpr int kFwdWarp = 2 + kExpWarps;   // forwarder: after the expansion warps
constexpr int kThreads = 32 * (kFwdWarp + 1);
constexpr int kEPT = kBK / kTPR;    // K elements one thread expands per stage (64)
constexpr int kCPT = kEPT / 2;      // their code bytes = TMEM columns (32)
static_assert(kTPR == kSubs && kEPT == kSubK, "thread part p expands sub-tile p");
// K stages accumulated in TMEM before promotion: at most kChunk (5120 K),
// a tile's part split into chunks of equal length.  A promotion stops the
// issuer until the tensor core has finished every queued MMA and the
// epilogue has read the accumulator (~1.6 us), so chunks are as long as the
// accumulation error allows.
constexpr int kChunk = 40;
__host__ __device__ __forceinline__ int chunk_len(int left) {
  const int n = (left + kChunk - 1) / kChunk;
  return (left + n - 1) / n;
}
// The accumulator: 256 fp32 columns, [hi | lo of tokens 0-63 | hi | lo of
// tokens 64-127] (each CTA's 128 B rows in turn).  There is room for one:
// the issuer waits while the epilogue drains it, once per chunk.
constexpr uint32_t kAccCols = 2 * kBT;
constexpr uint32_t kACols = kBK / 2;                // one A stage: 128 fp16 = 64 columns
constexpr uint32_t kAColBase = kAccCols;            // A ring after the accumulator
constexpr uint32_t kTmemCols = kAColBase + kStages * kACols;   // 512
static_assert(kTmemCols == 512, "the tile uses all of tensor memory");
constexpr uint64_t kWaitLimitNs = 4000000000ull;

constexpr uint32_t kBSubBytes = kBTc * kSubK * 2;       // 8 KB: this CTA's hi (or lo) rows of a sub-tile
constexpr uint32_t kBStageBytes = kSubs * 2 * kBSubBytes;   // 32 KB: [sub0 hi | sub0 lo | sub1 hi | sub1 lo]
constexpr uint32_t kCodeStageBytes = kBN * kBK / 2;     // 8 KB of codes
constexpr uint32_t kScaleStageBytes = kExpThreads * 4;  // 4 scale bytes per thread
constexpr uint32_t kOffB = 0;
constexpr uint32_t kOffCodes = kOffB + kStages * kBStageBytes;
constexpr uint32_t kOffScales = kOffCodes + kCStages * kCodeStageBytes;
constexpr uint32_t kOffBars = kOffScales + kCStages * kScaleStageBytes;
// full_b, stage_full, stage_empty, acc_full, acc_empty, mma_done
constexpr uint32_t kNumBars = 3 * kStages + 3;
constexpr uint32_t kOffMisc = kOffBars + kNumBars * 8;
constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;   // + slack to align to 1024
static_assert(kOffCodes % 1024 == 0, "swizzled tiles need 1 KB alignment");
static_assert(kSmemBytes <= 232448, "over the opt-in shared memory of one CTA");

// bit 0: a pipeline wait of the GEMM timed out
__device__ unsigned int g_gemm_error_flags = 0;

using dev::bits_h2;
using dev::expand8;
using dev::h2_bits;
using dev::ue4m3x2_to_half2;

// ---------------------------------------------------------------------------
// 1. activation expansion
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
expand_act_kernel(const int8_t* __restrict__ q, const __half* __restrict__ d, int M, int K,
                  int M_pad, __half* __restrict__ act, float* __restrict__ tok_scale) {
  // programmatic dependent launch: the next kernel may start its prologue
  // (and its weight copies); q and d are read once the previous kernel is done
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int row = blockIdx.x;
  uint4* hi = reinterpret_cast<uint4*>(act + static_cast<size_t>(row) * K);
  uint4* lo = reinterpret_cast<uint4*>(act + static_cast<size_t>(M_pad + row) * K);
  const int K8 = K / 8;
  if (row >= M) {
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    for (int i = threadIdx.x; i < K8; i += blockDim.x) {
      hi[i] = z;
      lo[i] = z;
    }
    if (threadIdx.x == 0) tok_scale[row] = 1.0f;
    return;
  }
  const __half* drow = d + static_cast<size_t>(row) * (K / 32);
  float dmax = 0.0f;
  for (int b = threadIdx.x; b < K / 32; b += blockDim.x)
    dmax = fmaxf(dmax, fabsf(__half2float(drow[b])));
  __shared__ float red[8];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dmax = fmaxf(dmax, __shfl_xor_sync(0xffffffffu, dmax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = dmax;
  __syncthreads();
  dmax = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) dmax = fmaxf(dmax, red[i]);
  // smallest e >= 0 with |d*q| * 2^-e <= 65504 for every element of the row
  int e = 0;
  while (ldexpf(dmax * 127.0f, -e) > 65504.0f) ++e;
  const float inv = ldexpf(1.0f, -e);
  if (threadIdx.x == 0) tok_scale[row] = ldexpf(1.0f, e);

  const uint2* qrow = reinterpret_cast<const uint2*>(q + static_cast<size_t>(row) * K);
  for (int i = threadIdx.x; i < K8; i += blockDim.x) {
    const uint2 qv = qrow[i];
    const float dv = __half2float(drow[i >> 2]) * inv;
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t word = j < 2 ? qv.x : qv.y;
      const int sh = (j & 1) * 16;
      const float a0 = static_cast<float>(static_cast<int8_t>((word >> sh) & 0xFF)) * dv;
      const float a1 = static_cast<float>(static_cast<int8_t>((word >> (sh + 8)) & 0xFF)) * dv;
      const __half h0 = __float2half_rn(a0), h1 = __float2half_rn(a1);
      const __half l0 = __float2half_rn(a0 - __half2float(h0));
      const __half l1 = __float2half_rn(a1 - __half2float(h1));
      hw[j] = h2_bits(__halves2half2(h0, h1));
      lw[j] = h2_bits(__halves2half2(l0, l1));
    }
    hi[i] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    lo[i] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
}

// ---------------------------------------------------------------------------
// 2. the tcgen05 GEMM
// ---------------------------------------------------------------------------
// The work of one CTA pair.  The T tiles (128 tokens x 256 weight rows) are
// numbered as the launcher orders them; with P pairs, the first W * P tiles
// (W = T / P) go round-robin, whole: pair j takes tiles j, j + P, ..., so a
// wave of pairs shares operand tiles as in a plain tiled grid.  The K stages
// of the R = T - W * P remaining tiles are split evenly over all pairs
// (stream-K): pair j takes the stages [R * num_kb * j / P, R * num_kb *
// (j + 1) / P) of those tiles in order, so no pair idles in a last partial
// wave.  A tile whose stages are split leaves each part's fp32 sums in a
// slot of the workspace (a pair's first and last stream-K parts: slots 0
// and 1), and gemm_fixup_kernel adds the parts in K order.  The pair's
// stages are numbered g = 0 .. G-1 in the order it processes them.
struct PairWork {
  int num_kb, P, j, W, T_dp;
  int sk_b;       // first stream-K stage of this pair (over the R last tiles)
  int G;          // stages of this pair
  int tile_sk0;   // tile of the pair's first stream-K stage (-1: none)

  __device__ __forceinline__ void init(int T, int nkb, int pairs, int pair) {
    num_kb = nkb;
    P = pairs;
    j = pair;
    W = T / P;
    T_dp = W * P;
    // the launcher keeps T * num_kb within int32
    const int64_t U_r = static_cast<int64_t>(T - T_dp) * num_kb;
    sk_b = static_cast<int>(U_r * j / P);
    const int sk_e = static_cast<int>(U_r * (j + 1) / P);
    G = W * num_kb + (sk_e - sk_b);
    tile_sk0 = sk_e > sk_b ? T_dp + static_cast<int>(sk_b / num_kb) : -1;
  }
  // tile (in the launcher's order) and K stage of stage g
  __device__ __forceinline__ void stage(int g, int& tile, int& kb) const {
    const int dp = W * num_kb;
    if (g < dp) {
      tile = j + (g / num_kb) * P;
      kb = g % num_kb;
    } else {
      const int u = sk_b + (g - dp);
      tile = T_dp + u / num_kb;
      kb = u - (u / num_kb) * num_kb;
    }
  }
  // stages from g (K stage kb) to the end of its tile's part
  __device__ __forceinline__ int part_left(int g, int kb) const {
    return min(num_kb - kb, G - g);
  }
};

// The pair's stages one after another, without a division but where the
// walk enters the stream-K stages.
struct StageCursor {
  int g, tile, kb;
  __device__ __forceinline__ void begin(const PairWork& w) {
    g = 0;
    w.stage(0, tile, kb);
  }
  __device__ __forceinline__ void next(const PairWork& w) {
    ++g;
    ++kb;
    const int dp = w.W * w.num_kb;
    if (g == dp) {
      if (g < w.G) w.stage(g, tile, kb);
    } else if (kb == w.num_kb) {
      kb = 0;
      tile += g < dp ? w.P : 1;
    }
  }
};

// Tile index -> (token tile, weight pair).  With token tiles fastest
// (tok_fast) consecutive tiles share the weight rows, else the tokens.
__host__ __device__ __forceinline__ void tile_coords(int tile, int mt, int np, int tok_fast,
                                                     int& tt, int& wp) {
  tt = tok_fast ? tile % mt : tile / np;
  wp = tok_fast ? tile / mt : tile % np;
}

// fp32 sums of one CTA's part of a tile: [p][j / 4][rt] float4, where thread
// (rt, p) of the epilogue holds tokens 64 p + j of weight row rt
constexpr int kPartFloats = kBN * kBT;   // 64 KB
__device__ __forceinline__ float4* part_slot(float* parts, int cta, int slot) {
  return reinterpret_cast<float4*>(parts + (static_cast<size_t>(cta) * 2 + slot) * kPartFloats);
}

__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap act_map, const uint8_t* __restrict__ codes,
            const uint8_t* __restrict__ scales, int N, int K, int M, int M_pad, float g,
            const float* __restrict__ tok_scale, float* __restrict__ y, int T, int np,
            int tok_fast, float* __restrict__ parts) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_addr(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw + pad;
  // full_b(s):      this CTA's activation rows of stage s landed (TMA tx)
  // stage_full(s):  (leader) stage s complete in both CTAs: A written by all
  //                 expansion warps of the pair, both CTAs' B rows forwarded
  // stage_empty(s): the pair MMAs of stage s finished (committed to both CTAs)
  // acc_full:       the MMAs of a chunk finished;  acc_empty: both CTAs'
  //                 epilogues read the accumulator
  auto full_b = [&](int s) { return sbase + kOffBars + 8u * s; };
  auto stage_full = [&](int s) { return sbase + kOffBars + 8u * (kStages + s); };
  auto stage_empty = [&](int s) { return sbase + kOffBars + 8u * (2 * kStages + s); };
  constexpr uint32_t kOffAcc = 8u * (3 * kStages);
  const uint32_t acc_full = sbase + kOffBars + kOffAcc;
  const uint32_t acc_empty = acc_full + 8u;
  const uint32_t mma_done = acc_full + 16u;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // The two CTAs of a cluster are a pair: CTA 0 (the leader) issues the
  // pair MMAs for both.  Each CTA owns 128 weight rows of a tile and loads
  // the hi and lo rows of half of its 128 tokens.
  const uint32_t rank = ptx::cluster_ctarank();
  const bool leader = rank == 0;
  const int mt = M_pad / kBT;
  const int num_kb = (K + kBK - 1) / kBK;   // the last stage may hold one sub-tile
  // the pair's schedule lives in shared memory: its fields are read where
  // the walks change tiles, and kept out of the registers of the loops
  __shared__ PairWork work_s;
  const PairWork& work = work_s;

  if (threadIdx.x == 0) {
    work_s.init(T, num_kb, static_cast<int>(gridDim.x >> 1), static_cast<int>(blockIdx.x >> 1));
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(full_b(s), 1);
      ptx::mbar_init(stage_full(s), 2 * kExpWarps + 2);
      ptx::mbar_init(stage_empty(s), 1);
    }
    ptx::mbar_init(acc_full, 1);
    ptx::mbar_init(acc_empty, 2 * kExpWarps);
    ptx::mbar_init(mma_done, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tensormap(&act_map);
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(ptx::smem_addr(tmem_holder), kTmemCols);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  ptx::cluster_sync();   // both CTAs' barriers exist before any remote arrival
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int G = work.G;

  auto fail = [&]() {
    *abort_flag = 1;
    atomicOr(&g_gemm_error_flags, 1u);
  };
  // Every role runs its loop with the whole warp converged: all lanes wait
  // (a wait in a diverged lane costs the tensor pipe ~150-200 cycles per
  // stage), one lane issues, and the outcome is made warp-uniform.
  auto warp_wait = [&](uint32_t bar, uint32_t parity) -> bool {
    if (__all_sync(0xffffffffu, ptx::mbar_try_wait(bar, parity))) return true;
    const bool got = ptx::mbar_wait_bounded(bar, parity, abort_flag, kWaitLimitNs);
    return __all_sync(0xffffffffu, got);
  };

  if (warp == 0) {
    // ------------------------------- TMA producer ------------------------------
    int issued = 0;
    StageCursor cur;
    cur.begin(work);
    int tok_tile = -1, tok0 = 0;   // this CTA's first token row of the current tile
    for (int gs = 0; gs < G; ++gs, cur.next(work)) {
      const int s = gs % kStages;
      const uint32_t ph = (gs / kStages) & 1;
      if (!warp_wait(stage_empty(s), ph ^ 1)) {
        fail();
        break;
      }
      if (cur.tile != tok_tile) {
        int tt, wp;
        tile_coords(cur.tile, mt, np, tok_fast, tt, wp);
        tok_tile = cur.tile;
        tok0 = tt * kBT + kBTc * static_cast<int>(rank);
      }
      if (lane == 0) {
        const int kb = cur.kb;
        const uint32_t dst = sbase + kOffB + s * kBStageBytes;
        const int nsub = min(kSubs, (K - kb * kBK) / kSubK);
        ptx::mbar_arrive_expect_tx(full_b(s), nsub * 2 * kBSubBytes);
        for (int sub = 0; sub < nsub; ++sub) {
          const uint32_t d0 = dst + sub * 2 * kBSubBytes;
          const int kx = kb * kBK + sub * kSubK;
          ptx::tma_load_2d(d0, &act_map, kx, tok0, full_b(s));
          ptx::tma_load_2d(d0 + kBSubBytes, &act_map, kx, M_pad + tok0, full_b(s));
        }
      }
      __syncwarp();
      ++issued;
    }
    if (*abort_flag) {
      // the MMAs may have stopped: wait for this CTA's copies in flight
      // before the CTA can leave
      for (int gs = std::max(0, issued - kStages); gs < issued; ++gs)
        ptx::mbar_wait_bounded(full_b(gs % kStages), (gs / kStages) & 1, nullptr, kWaitLimitNs);
    }
  } else if (warp == kFwdWarp) {
    // ------------ forwarder: this CTA's activation rows have landed ---------
    const uint32_t leader_stage_full0 = ptx::mapa_shared(stage_full(0), 0);
    for (int gs = 0; gs < G; ++gs) {
      const int s = gs % kStages;
      if (!warp_wait(full_b(s), (gs / kStages) & 1)) {
        fail();
        break;
      }
      if (lane == 0) ptx::mbar_arrive_cluster(leader_stage_full0 + 8u * s);
      __syncwarp();
    }
  } else if (warp == 1) {
    // -------------------------- pair MMA issuer (leader) ------------------------
    if (leader) {
      constexpr uint32_t idesc = ptx::idesc_f16_f32(2 * kBN, 2 * kBT);
      // completion of the pair MMAs is signalled to the same barrier in both CTAs
      auto commit_both = [&](uint32_t bar) {
        ptx::mma_commit_pair(ptx::mapa_shared(bar, 0));
        ptx::mma_commit_pair(ptx::mapa_shared(bar, 1));
      };
      // The issuing thread is on the tensor core's critical path (it issues
      // about as fast as the MMAs run), so the loop keeps its ring position,
      // barrier and operand addresses in registers and advances them by
      // constants: a few instructions per stage besides the MMAs.
      const uint32_t a_cols0 = tmem_base + kAColBase;
      const uint64_t bdesc0 = ptx::sw128_kmajor_desc(sbase + kOffB);
      const uint32_t d_tmem = tmem_base;
      const uint32_t full0 = stage_full(0);
      const uint32_t empty0_r0 = ptx::mapa_shared(stage_empty(0), 0);
      const uint32_t empty0_r1 = ptx::mapa_shared(stage_empty(0), 1);
      const uint32_t accf_r0 = ptx::mapa_shared(acc_full, 0);
      const uint32_t accf_r1 = ptx::mapa_shared(acc_full, 1);
      const int kb_one = K % kBK != 0 ? num_kb - 1 : -1;   // the stage with one sub-tile
      int s = 0;            // ring slot of the next stage
      uint32_t ph = 0;      // its phase parity
      bool ok_mma = true;
      // chunks: at most kChunk stages of one tile's part; the accumulator
      // starts from zero at each
      int gc = 0;
      for (int gs = 0; gs < G && ok_mma; ++gc) {
        int tile, kb;
        work.stage(gs, tile, kb);
        const int n = chunk_len(work.part_left(gs, kb));
        gs += n;
        // the accumulator is reused once the epilogue drained the last chunk
        if (gc >= 1 && !warp_wait(acc_empty, (gc - 1) & 1)) {
          fail();
          break;
        }
        for (int i = 0; i < n; ++i, ++kb) {
          if (!warp_wait(full0 + 8u * s, ph)) {
            fail();
            ok_mma = false;
            break;
          }
          if (lane == 0) {
            ptx::tc_fence_after();
            const uint32_t a_cols = a_cols0 + s * kACols;
            const uint64_t bdesc = bdesc0 + s * (kBStageBytes >> 4);
#pragma unroll
            for (int sub = 0; sub < kSubs; ++sub) {
              if (sub == 1 && kb == kb_one) break;
#pragma unroll
              for (int k = 0; k < kSubK / 16; ++k) {
                // B: this CTA's [hi | lo] rows of the sub-tile, one 128-row
                // operand; descriptor start addresses are in 16-byte units
                // (32 bytes = next 16 K)
                const uint32_t a = a_cols + sub * (kSubK / 2) + 8u * k;
                const uint64_t bk = bdesc + ((sub * 2 * kBSubBytes) >> 4) + 2u * k;
                ptx::mma_f16_ts_pair(d_tmem, a, bk, idesc,
                                     (i == 0 && sub == 0 && k == 0) ? 0u : 1u);
              }
            }
            ptx::mma_commit_pair(empty0_r0 + 8u * s);
            ptx::mma_commit_pair(empty0_r1 + 8u * s);
            if (i == n - 1) {
              ptx::mma_commit_pair(accf_r0);
              ptx::mma_commit_pair(accf_r1);
            }
          }
          __syncwarp();
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      // no MMA may still be reading or writing tensor memory when it is released
      if (lane == 0) commit_both(mma_done);
      __syncwarp();
      ptx::mbar_wait_bounded(mma_done, 0, nullptr, kWaitLimitNs);
    }
  } else {
    // ------------------- weight expansion, then the epilogue ------------------
    // A warp may only touch the TMEM lanes of its quarter (warp % 4), so the
    // threads of TMEM lane rt = 32 * (warp % 4) + lane expand weight row
    // rt of the CTA's 128 rows of each tile: warp group p = (warp - 2) / 4
    // takes sub-tile p of each 128-wide K stage (kEPT = 64 elements, TMEM
    // columns kCPT * p ..).  In the epilogue the same threads split the 128
    // token columns.
    const int quarter = warp & 3;
    const int p = (warp - 2) >> 2;
    const int rt = quarter * 32 + lane;
    const uint32_t stg_c = sbase + kOffCodes + 64u * rt + kCPT * p;
    const int t = threadIdx.x - 64;    // 0 .. kExpThreads - 1
    const uint32_t stg_s = sbase + kOffScales + 4u * t;
    // weight row of this thread in tile `tile` (N: none)
    auto tile_row = [&](int tile) {
      int tt, wp;
      tile_coords(tile, mt, np, tok_fast, tt, wp);
      return (wp * 2 + static_cast<int>(rank)) * kBN + rt;
    };
    // Prefetch of the packed codes and scales, kCStages - 1 stages ahead of
    // the expansion: source pointers advance by one stage's bytes, and are
    // set again (with the divisions of the pair's schedule) only where the
    // walk starts another tile's part.
    const uint8_t* pf_c = codes;
    const uint8_t* pf_s = scales;
    int pf_kb = 0, pf_left = 0;
    bool pf_row_ok = false;
    auto issue = [&](int gs) {
      if (gs < G) {
        if (pf_left == 0) {
          int tile;
          work.stage(gs, tile, pf_kb);
          pf_left = work.part_left(gs, pf_kb);
          const int row = tile_row(tile);
          pf_row_ok = row < N;
          const size_t r = pf_row_ok ? static_cast<size_t>(row) : 0;
          pf_c = codes + r * (K / 2) + kCPT * p + (kBK / 2) * static_cast<size_t>(pf_kb);
          pf_s = scales + r * (K / 16) + 4 * p + (kBK / 16) * static_cast<size_t>(pf_kb);
        }
        const uint32_t slot = gs % kCStages;
        // this thread's sub-tile exists (K is a multiple of 64): else zero
        // fill from an in-bounds address
        const bool in = pf_row_ok && pf_kb * kBK + p * kSubK < K;
        const uint8_t* c_src = in ? pf_c : codes;
        const uint8_t* s_src = in ? pf_s : scales;
        ptx::cp_async_16(stg_c + slot * kCodeStageBytes, c_src, in ? 16u : 0u);
        ptx::cp_async_16(stg_c + slot * kCodeStageBytes + 16, c_src + (in ? 16 : 0), in ? 16u : 0u);
        ptx::cp_async_4(stg_s + slot * kScaleStageBytes, s_src, in ? 4u : 0u);
        pf_c += kBK / 2;
        pf_s += kBK / 16;
        ++pf_kb;
        --pf_left;
      }
      ptx::cp_async_commit();
    };
    for (int i = 0; i < kCStages - 1; ++i) issue(i);
    // One arrival per warp (lane 0, after __syncwarp); arrivals go to the
    // leader's barriers.
    const uint32_t leader_stage_full0 = ptx::mapa_shared(stage_full(0), 0);
    const uint32_t leader_acc_empty = ptx::mapa_shared(acc_empty, 0);
    bool ok = true;
    const uint32_t tlane = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t a_dst = tmem_base + tlane + kAColBase + kCPT * p;
    constexpr int kCols = kBT / kTPR;
    // The chunk to drain next: first stage dg, dn stages, the chunk count,
    // and about the tile's part it belongs to: whether the chunk is its
    // first, whether the part is the whole tile, and its slot if not (0: the
    // pair's first stream-K part, else 1).
    int dg = 0, dn = 0, dc = 0, slot_idx = 0;
    bool chunk_first = true, whole = true;
    auto next_chunk = [&]() {
      if (dg >= G) return;
      int tile, kb;
      work.stage(dg, tile, kb);
      const int left = work.part_left(dg, kb);
      dn = chunk_len(left);
      chunk_first = kb == 0 || dg == 0 || dg == work.W * num_kb;
      if (chunk_first) {
        whole = kb == 0 && left == num_kb;
        slot_idx = tile == work.tile_sk0 ? 0 : 1;
      }
    };
    next_chunk();
    // Drain the next chunk: this thread's 64 token sums (hi + lo: columns
    // 2 * kCols * p + j and + kCols), then hand the accumulator back.  The
    // sums go to the part's destination: y (a whole tile, scaled when the
    // part is complete) or the part's slot.  A part of several chunks keeps
    // its running sum there: each later chunk adds itself to it, in order.
    auto drain = [&]() -> bool {
      // everything but the accumulator is worked out before its wait: this
      // chunk's destination, and the next chunk
      int tile, kb;
      work.stage(dg, tile, kb);
      const bool last = dn == work.part_left(dg, kb);
      const bool first = chunk_first, to_y = whole;
      int tt, wp;
      tile_coords(tile, mt, np, tok_fast, tt, wp);
      const int nrow = tile_row(tile);
      const int m0t = tt * kBT + kCols * p;   // this thread's first token
      // the part's slot; a whole tile of several chunks keeps its running
      // sum in slot 1 (free until the pair's last stream-K part, which comes
      // after its whole tiles) and writes y only at its last chunk
      float4* slot = part_slot(parts, blockIdx.x, to_y ? 1 : slot_idx) + p * (kCols / 4) * kBN + rt;
      const int this_dc = dc;
      dg += dn;
      ++dc;
      next_chunk();
      // the running sum of the part (every load issued before any use, and
      // before the wait, so that they overlap it)
      float acc[kCols];
#pragma unroll
      for (int j = 0; j < kCols; ++j) acc[j] = 0.0f;
      if (!first) {
#pragma unroll
        for (int j = 0; j < kCols; j += 4) {
          const float4 o = __ldcg(slot + (j / 4) * kBN);
          acc[j] = o.x, acc[j + 1] = o.y, acc[j + 2] = o.z, acc[j + 3] = o.w;
        }
      }
      if (!warp_wait(acc_full, this_dc & 1)) return false;
      ptx::tc_fence_after();
      const uint32_t base = tmem_base + tlane + 2 * kCols * p;
#pragma unroll
      for (int h = 0; h < kCols / 16; ++h) {
        uint32_t hi[16], lo[16];
        ptx::tmem_ld_16cols(base + 16u * h, hi);
        ptx::tmem_ld_16cols(base + kCols + 16u * h, lo);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j)
          acc[h * 16 + j] += __uint_as_float(hi[j]) + __uint_as_float(lo[j]);
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_cluster(leader_acc_empty);
      if (to_y && last) {
        if (nrow < N) {
#pragma unroll
          for (int j = 0; j < kCols; ++j) {
            const int m = m0t + j;
            if (m < M) y[static_cast<size_t>(m) * N + nrow] = acc[j] * (g * tok_scale[m]);
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < kCols; j += 4)
          slot[(j / 4) * kBN] = make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
      }
      return true;
    };
    // A chunk is drained at the top of the iteration kStages stages after its
    // last one: that stage waits for the chunk's last MMAs anyway, and the
    // issuer waits for the accumulator before the next chunk, whose first
    // stages are ready by then.  After the last stage the loop only drains
    // (one copy of the drain in the code: the warps' loops share the
    // instruction cache with the issuing thread).
    int next_drain = G > 0 ? dn - 1 + kStages : INT_MAX;
    for (int gs = 0;; ++gs) {
      while (gs >= next_drain) {
        if (!drain()) {
          fail();
          ok = false;
          break;
        }
        next_drain = dg < G ? dg + dn - 1 + kStages : INT_MAX;
      }
      if (!ok || next_drain == INT_MAX) break;
      if (gs >= G) continue;
      ptx::cp_async_wait<kCStages - 2>();
      const int s = gs % kStages;
      if (!warp_wait(stage_empty(s), ((gs / kStages) & 1) ^ 1)) {
        fail();
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const int cs = gs % kCStages;
      const uint8_t* stg = smem + kOffCodes + cs * kCodeStageBytes + 64 * rt + kCPT * p;
      const uint32_t sc = *reinterpret_cast<const uint32_t*>(
          smem + kOffScales + cs * kScaleStageBytes + 4 * t);
      // The previous stage's tensor-memory store is waited for (and the
      // stage announced) only after this stage's decode, so the store's
      // latency overlaps the decode instead of stalling the warp; the last
      // stage is announced right after its store.
      auto announce = [&](int st) {
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(leader_stage_full0 + 8u * (st % kStages));
      };
      {
        // sub-tile p: subblocks 0..3 of it, 8 codes per 32-bit word
        const uint4 c0 = *reinterpret_cast<const uint4*>(stg);
        const uint4 c1 = *reinterpret_cast<const uint4*>(stg + 16);
        const __half2 sp01 = ue4m3x2_to_half2(sc & 0xFFFFu);
        const __half2 sp23 = ue4m3x2_to_half2(sc >> 16);
        const __half2 s0 = __low2half2(sp01), s1 = __high2half2(sp01);
        const __half2 s2 = __low2half2(sp23), s3 = __high2half2(sp23);
        const uint4 e0 = expand8(c0.x, s0), e1 = expand8(c0.y, s0);
        const uint4 e2 = expand8(c0.z, s1), e3 = expand8(c0.w, s1);
        const uint4 e4 = expand8(c1.x, s2), e5 = expand8(c1.y, s2);
        const uint4 e6 = expand8(c1.z, s3), e7 = expand8(c1.w, s3);
        const uint32_t v[32] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w,
                                e2.x, e2.y, e2.z, e2.w, e3.x, e3.y, e3.z, e3.w,
                                e4.x, e4.y, e4.z, e4.w, e5.x, e5.y, e5.z, e5.w,
                                e6.x, e6.y, e6.z, e6.w, e7.x, e7.y, e7.z, e7.w};
        if (gs > 0) announce(gs - 1);
        ptx::tmem_st_32cols(a_dst + s * kACols, v);
      }
      if (gs == G - 1) announce(gs);
      issue(gs + kCStages - 1);
    }
    ptx::cp_async_wait<0>();
  }

  // Neither CTA leaves (or frees tensor memory) while the pair's MMAs or the
  // peer's remote arrivals may still touch it.
  __syncwarp();
  ptx::tc_fence_before();
  ptx::cluster_sync();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// The tiles whose K stages were split over several pairs: y = g * tok_scale *
// (sum of the parts in K order).  Grid (R, 2): the R stream-K tiles and the
// two CTAs' 128-row halves; 256 threads, thread (rt, p) as in the epilogue.
// A tile done by one pair was stored by the GEMM.
__global__ void __launch_bounds__(kExpThreads)
gemm_fixup_kernel(const float* __restrict__ parts, int T, int P, int num_kb, int mt, int np,
                  int tok_fast, int N, int M, float g, const float* __restrict__ tok_scale,
                  float* __restrict__ y) {
  asm volatile("griddepcontrol.wait;" ::: "memory");   // the GEMM's parts are written
  const int T_dp = T / P * P;
  const int64_t U_r = static_cast<int64_t>(T - T_dp) * num_kb;
  const int tr = blockIdx.x;
  const int r = blockIdx.y;
  const int64_t ts = static_cast<int64_t>(tr) * num_kb, te = ts + num_kb;
  auto start = [&](int i) { return U_r * i / P; };
  // the pair whose stream-K stages include ts
  int i0 = static_cast<int>(ts * P / U_r);
  while (i0 + 1 < P && start(i0 + 1) <= ts) ++i0;
  while (i0 > 0 && start(i0) > ts) --i0;
  int parts_n = 0;
  for (int i = i0; i < P && start(i) < te; ++i)
    if (max(start(i), ts) < min(start(i + 1), te)) ++parts_n;
  if (parts_n < 2) return;
  const int t = threadIdx.x;
  const int p = t / kBN, rt = t % kBN;
  constexpr int kCols = kBT / kTPR;
  float acc[kCols];
  bool first = true;
  for (int i = i0; i < P && start(i) < te; ++i) {
    if (max(start(i), ts) >= min(start(i + 1), te)) continue;
    const float4* slot = part_slot(const_cast<float*>(parts), 2 * i + r, start(i) >= ts ? 0 : 1);
#pragma unroll
    for (int j = 0; j < kCols; j += 4) {
      const float4 v = __ldcg(slot + (p * (kCols / 4) + j / 4) * kBN + rt);
      if (first) {
        acc[j] = v.x, acc[j + 1] = v.y, acc[j + 2] = v.z, acc[j + 3] = v.w;
      } else {
        acc[j] += v.x, acc[j + 1] += v.y, acc[j + 2] += v.z, acc[j + 3] += v.w;
      }
    }
    first = false;
  }
  int tt, wp;
  tile_coords(T_dp + tr, mt, np, tok_fast, tt, wp);
  const int nrow = (wp * 2 + r) * kBN + rt;
  if (nrow >= N) return;
#pragma unroll
  for (int j = 0; j < kCols; ++j) {
    const int m = tt * kBT + kCols * p + j;
    if (m < M) y[static_cast<size_t>(m) * N + nrow] = acc[j] * (g * tok_scale[m]);
  }
}

// Scratch of nvq_gemm_noalloc: the expanded activations [2 * M_pad, K] fp16
// and the M_pad token scales of one call, in device memory that the library
// itself owns (a file-scope array exists on every GPU that loads the library,
// from module load until the process exits), so that the call needs no
// allocation and no workspace from its caller.
constexpr size_t kNoAllocScratchBytes = size_t{64} << 20;   // 64 MiB
static __device__ __align__(256) unsigned char g_gemm_noalloc_scratch[kNoAllocScratchBytes];

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

int64_t padded_tokens(int64_t M) { return (M + kBT - 1) / kBT * kBT; }

// Workspace of the prefill GEMM: the expanded activations [2 * M_pad, K]
// fp16, the M_pad token scales, then two part slots (64 KB each) for every
// CTA a launch may have (one per SM).
size_t parts_offset(int64_t M, int64_t K) {
  const int64_t mp = padded_tokens(M);
  return static_cast<size_t>((4 * mp * K + 4 * mp + 255) / 256 * 256);
}
size_t parts_bytes() {
  return static_cast<size_t>(device_sm_count()) * 2 * kPartFloats * sizeof(float);
}

// CTA pairs of the GEMM that fit on the device at once (cached per device)
int gemm_pairs() {
  constexpr int kMaxDevices = 64;
  static std::atomic<int> cache[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return device_sm_count() / 2;
  if (dev >= 0 && dev < kMaxDevices) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int pairs = device_sm_count() / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cudaLaunchAttribute cluster[1];
  cluster[0].id = cudaLaunchAttributeClusterDimension;
  cluster[0].val.clusterDim.x = 2;
  cluster[0].val.clusterDim.y = 1;
  cluster[0].val.clusterDim.z = 1;
  cfg.attrs = cluster;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_kernel, &cfg) == cudaSuccess && n > 0)
    pairs = std::min(pairs, n);
  else
    cudaGetLastError();   // leave no sticky error behind; keep the SM-count bound
  pairs = std::max(pairs, 1);
  if (dev >= 0 && dev < kMaxDevices) cache[dev].store(pairs, std::memory_order_relaxed);
  return pairs;
}

// token counts that nvq_gemm hands to the decode GEMV
constexpr int64_t kGemvTokensMax = 4;

// The scratch array's device address in the current context.  Host code may
// not use the array's name as an address (it names a host-side shadow), so
// the address is looked up with cudaGetSymbolAddress, with the device
// current, and cached per device together with the context it was looked up
// in; a different current context (for example after cudaDeviceReset) makes
// the next call look it up again.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

}  // namespace

size_t gemm_workspace_size(int64_t M, int64_t, int64_t K) {
  if (gemm_small_supported(M, K)) return gemm_small_workspace_size(M, K);
  return parts_offset(M, K) + parts_bytes();
}

size_t gemm_noalloc_limit() { return kNoAllocScratchBytes; }

cudaError_t gemm_noalloc_scratch(void** out) {
  constexpr int kMaxDevices = 64;
  struct Entry {
    CUcontext ctx;
    void* ptr;
  };
  static Entry cache[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  CUcontext ctx = nullptr;
  if (CtxGetCurrentFn get = ctx_get_current()) get(&ctx);
  std::lock_guard<std::mutex> lock(mu);
  Entry& c = cache[dev];
  if (c.ptr == nullptr || c.ctx != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_gemm_noalloc_scratch);
    if (e != cudaSuccess) return e;
    c.ptr = p;
    c.ctx = ctx;
  }
  *out = c.ptr;
  return cudaSuccess;
}

cudaError_t gemm_error_flags(bool clear, unsigned int* flags) {
  cudaError_t e = cudaMemcpyFromSymbol(flags, g_gemm_error_flags, sizeof(unsigned int));
  if (e == cudaSuccess && clear) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_gemm_error_flags, &zero, sizeof(zero));
  }
  return e;
}

cudaError_t expand_activations(const int8_t* q, const uint16_t* d, int64_t M, int64_t M_pad,
                               int64_t K, void* act, float* tok_scale, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(M_pad));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, expand_act_kernel, q, reinterpret_cast<const __half*>(d),
                            static_cast<int>(M), static_cast<int>(K), static_cast<int>(M_pad),
                            static_cast<__half*>(act), tok_scale);
}

cudaError_t gemm_expand(const int8_t* q, const uint16_t* d, int64_t M, int64_t K,
                        void* workspace, cudaStream_t stream) {
  const int64_t M_pad = padded_tokens(M);
  float* tok_scale = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + 4 * M_pad * K);
  return expand_activations(q, d, M, M_pad, K, workspace, tok_scale, stream);
}

cudaError_t gemm_main(const uint8_t* codes, const uint8_t* scales, float g, int64_t N,
                      int64_t K, int64_t M, float* y, const void* workspace,
                      cudaStream_t stream) {
  const int64_t M_pad = padded_tokens(M);
  void* act = const_cast<void*>(workspace);
  const float* tok_scale =
      reinterpret_cast<const float*>(static_cast<const uint8_t*>(workspace) + 4 * M_pad * K);
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (encode == nullptr) return cudaErrorNotSupported;
  CUtensorMap map;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(2 * M_pad)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kSubK), static_cast<cuuint32_t>(kBTc)};
  const cuuint32_t estr[2] = {1, 1};
  if (encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, act, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
      CUDA_SUCCESS)
    return cudaErrorInvalidValue;

  static SmemAttrOnce attr;
  cudaError_t e = attr.ensure(gemm_kernel, static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  // tiles: 128 tokens x a pair of 128-row weight tiles (an odd last tile
  // gets an all-padding partner)
  const int64_t mt = M_pad / kBT;
  const int64_t np = ((N + kBN - 1) / kBN + 1) / 2;
  const int64_t T = mt * np;
  const int64_t num_kb = (K + kBK - 1) / kBK;
  if (T > INT32_MAX / 2 || T * num_kb > INT32_MAX) return cudaErrorInvalidValue;
  const int P = static_cast<int>(std::min<int64_t>(gemm_pairs(), T * num_kb));
  float* parts = reinterpret_cast<float*>(static_cast<uint8_t*>(act) + parts_offset(M, K));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * P));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute cluster[1];
  cluster[0].id = cudaLaunchAttributeClusterDimension;
  cluster[0].val.clusterDim.x = 2;
  cluster[0].val.clusterDim.y = 1;
  cluster[0].val.clusterDim.z = 1;
  cfg.attrs = cluster;
  cfg.numAttrs = 1;
  // token tiles fastest when the packed weights are the larger operand
  // (0.5625 B per weight against 4 B per token and K of expanded activations)
  const int tok_fast = 9 * N >= 64 * M_pad ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, gemm_kernel, map, codes, scales, static_cast<int>(N),
                         static_cast<int>(K), static_cast<int>(M), static_cast<int>(M_pad), g,
                         tok_scale, y, static_cast<int>(T), static_cast<int>(np), tok_fast,
                         parts);
  if (e != cudaSuccess) return e;
  // the stream-K tiles: add their parts
  const int64_t R = T - T / P * P;
  if (R > 0) {
    cudaLaunchConfig_t fcfg = {};
    fcfg.gridDim = dim3(static_cast<unsigned>(R), 2);
    fcfg.blockDim = dim3(kExpThreads);
    fcfg.stream = stream;
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    fcfg.attrs = pdl;
    fcfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&fcfg, gemm_fixup_kernel, static_cast<const float*>(parts),
                           static_cast<int>(T), P, static_cast<int>(num_kb),
                           static_cast<int>(mt), static_cast<int>(np), tok_fast,
                           static_cast<int>(N), static_cast<int>(M), g, tok_scale, y);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

cudaError_t launch_gemm(const uint8_t* codes, const uint8_t* scales, float g, int64_t N,
                        int64_t K, const int8_t* q, const uint16_t* d, int64_t M, float* y,
                        void* workspace, cudaStream_t stream) {
  // up to four tokens the CUDA-core decode GEMV streams the weights faster
  // (its integer dot costs little per token); beyond, the tensor-core
  // small-token schedule, whose per-weight cost does not grow with M
  if (M <= kGemvTokensMax) return launch_gemv(codes, scales, g, N, K, q, d, M, y, stream);
  if (gemm_small_supported(M, K))
    return launch_gemm_small(codes, scales, g, N, K, q, d, M, y, workspace, stream);
  cudaError_t e = gemm_expand(q, d, M, K, workspace, stream);
  if (e != cudaSuccess) return e;
  return gemm_main(codes, scales, g, N, K, M, y, workspace, stream);
}

}  // namespace nvq
