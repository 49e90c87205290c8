// Decode GEMV: y[M, N] = A[M, K] . W[N, K]^T for M = 1..16, NVFP4 weights
// and Q8_0 activations.
//
// The operation is the row dot of "HANDOFF: flint CPU optimization (Q4_1 +
// NVFP4)", section 3 (ggml_vec_dot_nvfp4_q8_0: one NVFP4 row against one
// Q8_0 row, one scale per 16 weights): per 16-element subblock,
//   y += g * s_w * d_a * 0.5 * sum(c_w * q_a),   c_w = 2*E2M1 in -12..12.
//
// Arithmetic shared by every schedule (HBM-bound; every weight byte is read
// exactly once):
//  * lane l of a warp owns whole 32-element chunks of a row: 16 code bytes
//    (one 128-bit load), two UE4M3 scale bytes and exactly one Q8_0
//    activation block (32 int8 codes + one fp16 d);
//  * codes are decoded in registers with byte permutes (no shared-memory
//    table) and the two exact integer subblock sums of a chunk are formed
//    with dp4a; they are rescaled by their UE4M3 scales, multiplied by the
//    chunk's d and accumulated in fp32;
//  * one shuffle reduction per row (and, for rows split over several warps,
//    a fixed-order sum of the warps' partials), then y = 0.5*g*acc.
// Every kernel has an ISUM instantiation that also stores the integer
// subblock sums it formed, isum[m, n, 2c + h] for chunk c, half h, so that
// nvq_debug_subblock_sums can export the sums of the very code that
// produces y (the y it writes is the same bit pattern).
//
// Schedules:
//  * gemv_m1_reg_kernel (M = 1, K = 1024 * T for the common T; the decode
//    path): one CTA per SM owning a balanced row range; a producer thread
//    streams stages of R whole contiguous rows (two 1-D TMA bulk copies,
//    <= 46 KB, 4 stages in flight); 16 consumer warps.  Every lane always
//    handles the same chunk positions of every row, so its activation codes,
//    d and the bias corrections sit in registers for the whole kernel.  The
//    weights are decoded to the +12-biased integer LUT of the "Bias trick"
//    paragraph with sign-replicating byte permutes, and the bias is removed
//    by starting each subblock's dp4a chain at corr = -12 * bsum16.  One
//    launch may cover up to three matrices that read the same activations
//    (their rows concatenated, so the row ranges stay balanced), and a matrix
//    may also emit the Q8_0 quantisation of its output: the CTA that stores
//    the last of a 32-row block's outputs (per-block arrival counters)
//    quantises that block, with the activation quantiser's IEEE operations.
//  * gemv_m1_kernel (M = 1, other K % 256 == 0): the same ring with groups
//    of 16 rows (whole K, or K segments of at most 5120 elements) and the
//    activations staged once per CTA in shared memory; biased LUT with an
//    OR-merge of the two table halves.
//  * gemv_tma_kernel (M = 2..16, or M = 1 when the shared memory of the M = 1
//    schedule does not fit; K % 256 == 0): persistent CTAs, two per SM, each
//    owning a balanced row range; groups of 8 rows through a 4-stage ring;
//    the signed LUT, decoded once and used for all M tokens.
//  * gemv_kernel (any K % 64 == 0): one warp per row, loads straight to
//    registers.
#include <algorithm>

#include <cuda_fp16.h>

#include "nvq_device.cuh"
#include "nvq_internal.h"
#include "tcgen05.cuh"

namespace nvq {
namespace {

constexpr int kWarps = 4;        // rows per CTA of gemv_kernel
constexpr int kUnroll = 4;       // chunks per lane in flight in gemv_kernel

// TMA-staged schedule
constexpr int kTmaConsumers = 8;                  // consumer warps = rows per group
constexpr int kTmaStages = 4;
constexpr int kTmaThreads = (kTmaConsumers + 1) * 32;
constexpr int kTmaMaxSeg = 5120;                  // K elements per stage and row
constexpr uint64_t kWaitLimitNs = 4000000000ull;  // 4 s per pipeline wait

// bit 0 (NVQ_FLAG_GEMV_TIMEOUT): a pipeline wait of a GEMV kernel timed out
__device__ unsigned int g_gemv_error_flags = 0;

__device__ __forceinline__ void raise_timeout() { atomicOr(&g_gemv_error_flags, 1u); }

// Store the two subblock sums of chunk c of row n for token m.
__device__ __forceinline__ void store_isum(int32_t* isum, int64_t m, int N, int n, int K, int c,
                                           int i0, int i1) {
  int2* dst = reinterpret_cast<int2*>(isum + (m * N + n) * static_cast<int64_t>(K >> 4));
  dst[c] = make_int2(i0, i1);
}

// The two signed-LUT subblock sums of one chunk against token m's block c.
__device__ __forceinline__ int2 chunk_isums(const uint32_t (&cw)[8], const int8_t* q, int c) {
  const uint4* qa = reinterpret_cast<const uint4*>(q) + 2 * c;
  const uint4 q0 = __ldg(qa);
  const uint4 q1 = __ldg(qa + 1);
  int2 r;
  r.x = dev::dp4a(cw[0], q0.x, dev::dp4a(cw[1], q0.y,
        dev::dp4a(cw[2], q0.z, dev::dp4a(cw[3], q0.w, 0))));
  r.y = dev::dp4a(cw[4], q1.x, dev::dp4a(cw[5], q1.y,
        dev::dp4a(cw[6], q1.z, dev::dp4a(cw[7], q1.w, 0))));
  return r;
}

__device__ __forceinline__ void decode_chunk_signed(const uint4 w, uint32_t (&cw)[8]) {
  dev::decode_e2m1x8(w.x, cw[0], cw[1]);
  dev::decode_e2m1x8(w.y, cw[2], cw[3]);
  dev::decode_e2m1x8(w.z, cw[4], cw[5]);
  dev::decode_e2m1x8(w.w, cw[6], cw[7]);
}

// Shared memory of the TMA schedule: kTmaStages stages of
// [8 rows x seg/2 code bytes][8 rows x seg/16 scale bytes], then the
// full/empty barriers and the abort flag.
__host__ __device__ constexpr uint32_t tma_stage_bytes(int seg) {
  return static_cast<uint32_t>(kTmaConsumers) * (seg / 2 + seg / 16);
}
__host__ __device__ constexpr uint32_t tma_smem_bytes(int seg) {
  return kTmaStages * tma_stage_bytes(seg) + 2 * kTmaStages * 8 + 16;
}

// ---------------------------------------------------------------------------
// M = 1 schedule, activations staged in shared memory
// ---------------------------------------------------------------------------
constexpr int kM1Consumers = 16;                       // rows per group
constexpr int kM1Threads = (kM1Consumers + 1) * 32;    // + producer warp
constexpr int kM1Stages = 4;
constexpr uint32_t kSmemPerCtaMax = 227 * 1024;

// per 32-element activation chunk: its fp32 scale and the bias corrections
// -12 * (sum of its 16 codes) of its two subblocks
struct __align__(16) ActMeta {
  float d;
  int corr0;
  int corr1;
  int pad;
};

__host__ __device__ constexpr uint32_t m1_stage_bytes(int seg) {
  return static_cast<uint32_t>(kM1Consumers) * (seg / 2 + seg / 16);
}
// stages | qa [K/32 x 16 B] | qb [K/32 x 16 B] | meta [K/32 x 16 B] | barriers
__host__ __device__ constexpr uint32_t m1_smem_bytes(int K, int seg) {
  return kM1Stages * m1_stage_bytes(seg) + static_cast<uint32_t>(K / 32) * 48 +
         2 * kM1Stages * 8 + 16;
}

template <int NPL, bool ISUM>   // NPL: chunks per lane per stage (seg / 1024); 0 = any seg
__global__ void __launch_bounds__(kM1Threads, 1)
gemv_m1_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
               float half_g, int N, int K, int seg, const int8_t* __restrict__ q,
               const __half* __restrict__ d, float* __restrict__ y,
               int32_t* __restrict__ isum) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t stage_bytes = m1_stage_bytes(seg);
  const uint32_t codes_bytes = kM1Consumers * (seg / 2);
  const int nchunk = K / 32;
  uint4* qa = reinterpret_cast<uint4*>(smem + kM1Stages * stage_bytes);
  uint4* qb = qa + nchunk;
  ActMeta* meta = reinterpret_cast<ActMeta*>(qb + nchunk);
  uint64_t* full = reinterpret_cast<uint64_t*>(meta + nchunk);
  uint64_t* empty = full + kM1Stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kM1Stages);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int r_begin = static_cast<int>(static_cast<int64_t>(blockIdx.x) * N / G);
  const int r_end = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * N / G);
  const int ngroups = (r_end - r_begin + kM1Consumers - 1) / kM1Consumers;
  const int nseg = K / seg;
  const int total = ngroups * nseg;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kM1Stages; ++i) {
      ptx::mbar_init(ptx::smem_addr(full + i), 1);
      ptx::mbar_init(ptx::smem_addr(empty + i), kM1Consumers);
    }
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  // stage the activation vector once per CTA
  for (int c = threadIdx.x; c < nchunk; c += blockDim.x) {
    const uint4* src = reinterpret_cast<const uint4*>(q) + 2 * c;
    const uint4 a = src[0], b = src[1];
    qa[c] = a;
    qb[c] = b;
    const int s0 = dev::dp4a(a.x, 0x01010101u, dev::dp4a(a.y, 0x01010101u,
                   dev::dp4a(a.z, 0x01010101u, dev::dp4a(a.w, 0x01010101u, 0))));
    const int s1 = dev::dp4a(b.x, 0x01010101u, dev::dp4a(b.y, 0x01010101u,
                   dev::dp4a(b.z, 0x01010101u, dev::dp4a(b.w, 0x01010101u, 0))));
    ActMeta mt;
    mt.d = __half2float(d[c]);
    mt.corr0 = -12 * s0;
    mt.corr1 = -12 * s1;
    mt.pad = 0;
    meta[c] = mt;
  }
  __syncthreads();

  if (warp == kM1Consumers) {
    // ---------------- producer: one thread issues the bulk copies ----------
    if (lane != 0) return;
    int issued = 0;
    for (int it = 0; it < total; ++it) {
      const int s = it % kM1Stages;
      const uint32_t ph = (it / kM1Stages) & 1;
      if (!ptx::mbar_wait_bounded(ptx::smem_addr(empty + s), ph ^ 1, abort_flag, kWaitLimitNs)) {
        *abort_flag = 1;
        raise_timeout();
        break;
      }
      const int grp = it / nseg, sg = it % nseg;
      const int row0 = r_begin + grp * kM1Consumers;
      const int nrows = min(kM1Consumers, r_end - row0);
      const uint32_t bar = ptx::smem_addr(full + s);
      uint8_t* st = smem + s * stage_bytes;
      ptx::mbar_arrive_expect_tx(bar, nrows * (seg / 2 + seg / 16));
      if (nseg == 1) {
        ptx::bulk_load(ptx::smem_addr(st), codes + static_cast<size_t>(row0) * (K / 2),
                       nrows * (K / 2), bar);
        ptx::bulk_load(ptx::smem_addr(st + codes_bytes),
                       scales + static_cast<size_t>(row0) * (K / 16), nrows * (K / 16), bar);
      } else {
        for (int r = 0; r < nrows; ++r) {
          ptx::bulk_load(ptx::smem_addr(st + r * (seg / 2)),
                         codes + static_cast<size_t>(row0 + r) * (K / 2) + sg * (seg / 2),
                         seg / 2, bar);
          ptx::bulk_load(ptx::smem_addr(st + codes_bytes + r * (seg / 16)),
                         scales + static_cast<size_t>(row0 + r) * (K / 16) + sg * (seg / 16),
                         seg / 16, bar);
        }
      }
      ++issued;
    }
    if (*abort_flag) {
      for (int it = max(0, issued - kM1Stages); it < issued; ++it)
        ptx::mbar_wait_bounded(ptx::smem_addr(full + it % kM1Stages), (it / kM1Stages) & 1,
                               nullptr, kWaitLimitNs);
    }
    return;
  }

  // ---------------- consumers: warp w owns row w of each group --------------
  float acc = 0.0f;
  const int nch = seg / 32;
  for (int it = 0; it < total; ++it) {
    const int s = it % kM1Stages;
    const uint32_t ph = (it / kM1Stages) & 1;
    if (!ptx::mbar_wait_bounded(ptx::smem_addr(full + s), ph, abort_flag, kWaitLimitNs)) {
      *abort_flag = 1;
      raise_timeout();
      break;
    }
    const int grp = it / nseg, sg = it % nseg;
    const int row0 = r_begin + grp * kM1Consumers;
    const int nrows = min(kM1Consumers, r_end - row0);
    if (warp < nrows) {
      const uint8_t* st = smem + s * stage_bytes;
      const uint4* cw = reinterpret_cast<const uint4*>(st + warp * (seg / 2));
      const uint16_t* sw = reinterpret_cast<const uint16_t*>(st + codes_bytes + warp * (seg / 16));
      const int cbase = sg * nch;
      auto chunk = [&](const uint4 w, uint32_t s2, const uint4 a, const uint4 b, const ActMeta mt,
                       int cidx) {
        uint32_t c[8];
        dev::decode_e2m1x8_biased(w.x, c[0], c[1]);
        dev::decode_e2m1x8_biased(w.y, c[2], c[3]);
        dev::decode_e2m1x8_biased(w.z, c[4], c[5]);
        dev::decode_e2m1x8_biased(w.w, c[6], c[7]);
        const int i0 = dev::dp4a_us(c[0], a.x, dev::dp4a_us(c[1], a.y,
                       dev::dp4a_us(c[2], a.z, dev::dp4a_us(c[3], a.w, mt.corr0))));
        const int i1 = dev::dp4a_us(c[4], b.x, dev::dp4a_us(c[5], b.y,
                       dev::dp4a_us(c[6], b.z, dev::dp4a_us(c[7], b.w, mt.corr1))));
        if constexpr (ISUM) store_isum(isum, 0, N, row0 + warp, K, cidx, i0, i1);
        const float2 sf = dev::ue4m3x2_to_float2(s2);
        acc = fmaf(mt.d, fmaf(sf.x, static_cast<float>(i0), sf.y * static_cast<float>(i1)), acc);
      };
      if constexpr (NPL > 0) {
        uint4 w[NPL], a[NPL], b[NPL];
        ActMeta mt[NPL];
        uint32_t s2[NPL];
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
          const int j = lane + 32 * i;
          w[i] = cw[j];
          s2[i] = sw[j];
          a[i] = qa[cbase + j];
          b[i] = qb[cbase + j];
          mt[i] = meta[cbase + j];
        }
#pragma unroll
        for (int i = 0; i < NPL; ++i) chunk(w[i], s2[i], a[i], b[i], mt[i], cbase + lane + 32 * i);
      } else {
#pragma unroll 2
        for (int j = lane; j < nch; j += 32)
          chunk(cw[j], sw[j], qa[cbase + j], qb[cbase + j], meta[cbase + j], cbase + j);
      }
    }
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(empty + s));
    if (sg == nseg - 1) {
      if (warp < nrows) {
        const float v = dev::warp_sum(acc);
        if (lane == 0) y[row0 + warp] = v * half_g;
      }
      acc = 0.0f;
    }
  }
}

// ---------------------------------------------------------------------------
// M = 1 schedule with the activations in registers (K = 1024 * NPL * WPR)
// ---------------------------------------------------------------------------
// Every lane of a consumer warp handles the same NPL chunk positions of
// every row it ever processes, so the activation data of those chunks (32
// codes, d and the two bias corrections) is loaded once into registers and
// held there for the whole kernel.
// A row is split across WPR warps (warp part p owns the p-th contiguous K
// segment of 1024 * NPL elements); a stage is R = 16/WPR (or fewer, to fit
// 46 KB) whole, contiguous rows, fetched with two bulk copies.  With
// WPR > 1 each warp leaves its row partial in shared memory (one slot per
// stage) and the producer thread adds the WPR partials in a fixed order when
// it recycles the stage, so results are deterministic.
// The kernel is launched with programmatic stream serialisation: it lets
// the next kernel of the stream launch early and waits for the previous
// one (griddepcontrol) before it reads the activations or writes anything,
// so launch latency, prologue and the first weight copies (the weights are
// never written by the kernels before it) overlap the previous kernel's tail
// without changing results.
constexpr uint32_t kRegStageMax = 46080;
constexpr int kMaxGroup = 8;       // matrices per register-schedule launch

__host__ __device__ constexpr int reg_rows(int K, int wpr) {
  int r = kM1Consumers / wpr;
  while (r > 1 && static_cast<uint32_t>(r) * (K / 2 + K / 16) > kRegStageMax) --r;
  return r;
}
// stages | row partials [stage][warp] | barriers
__host__ __device__ constexpr uint32_t reg_smem_bytes(int K, int wpr) {
  return kM1Stages * static_cast<uint32_t>(reg_rows(K, wpr)) * (K / 2 + K / 16) +
         kM1Stages * kM1Consumers * 4 + 2 * kM1Stages * 8 + 16;
}

__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// The matrices of one register-schedule launch: up to kMaxGroup weight
// matrices with the same K that read the same activations (q, k, v of a
// layer; up and gate), their rows concatenated; each may also emit the Q8_0
// quantisation of its output (the requantisation that feeds the next
// product), which the CTA completing a 32-row block carries out.
struct RegMat {
  const uint8_t* codes;
  const uint8_t* scales;
  float* y;
  int8_t* rq_q;      // Q8_0 codes of y [N] (nullptr: no requantisation)
  __half* rq_d;      // Q8_0 scales of y [N / 32]
  int* rq_cnt;       // per 32-row block: rows written so far (0 between launches)
  float half_g;
  int N;
  int row_off;       // first row of this matrix among the concatenated rows
};
struct RegGroup {
  RegMat m[kMaxGroup];
  int count;
  int rows;          // concatenated rows
};

// dynamic shared memory the register schedule may request: the opt-in
// maximum less room for its static shared memory (the group of matrices)
constexpr uint32_t kRegDynSmemMax = kSmemPerCtaMax - 2048;
static_assert(sizeof(RegGroup) <= 2048, "static shared memory of the register schedule");

// A mixture-of-experts launch: grid row t handles token t, whose group is
// the experts ids[t, 0..top_k) of a stacked expert tensor, built on the
// device once the routing ids are visible (ids == nullptr: not a MoE launch).
struct MoeArgs {
  const int32_t* ids;     // [T, top_k]
  const uint8_t* codes;   // [E, N, K/2]
  const uint8_t* scales;  // [E, N, K/16]
  const float* g;         // [E]
  float* y;               // [T, top_k, N]
  int E;
  int N;
  int top_k;
};

// bit 1 of the GEMV error flags: a routing id outside 0..E-1 (its slot is skipped)
__device__ __forceinline__ void raise_bad_index() { atomicOr(&g_gemv_error_flags, 2u); }

// Q8_0 of the 32 outputs of block b, one lane per output: the same IEEE
// operations as the activation quantiser (amax, d32 = amax/127, q =
// rint(y/d32) clamped to +-127, d = fp16(d32)), so the codes are those the
// quantiser would produce from y.
__device__ __forceinline__ void requant_block_warp(const RegMat& m, int b, int lane) {
  const float v = __ldcg(m.y + 32 * b + lane);
  float a = fabsf(v);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  const float d32 = __fdiv_rn(a, 127.0f);
  int qi = 0;
  if (d32 > 0.0f) qi = max(-127, min(127, __float2int_rn(__fdiv_rn(v, d32))));
  m.rq_q[32 * b + lane] = static_cast<int8_t>(qi);
  if (lane == 0) m.rq_d[b] = __float2half_rn(d32);
}
// The same by one thread.
__device__ __forceinline__ void requant_block_thread(const RegMat& m, int b) {
  float a = 0.0f;
  for (int i = 0; i < 32; ++i) a = fmaxf(a, fabsf(__ldcg(m.y + 32 * b + i)));
  const float d32 = __fdiv_rn(a, 127.0f);
  for (int i = 0; i < 32; ++i) {
    int qi = 0;
    if (d32 > 0.0f) qi = max(-127, min(127, __float2int_rn(__fdiv_rn(__ldcg(m.y + 32 * b + i), d32))));
    m.rq_q[32 * b + i] = static_cast<int8_t>(qi);
  }
  m.rq_d[b] = __float2half_rn(d32);
}
// Row `row` of m (concatenated row `grow`) has been stored by this thread.
// Returns 0, or the way its 32-row block became complete: 1 = every row of
// the block belongs to this CTA and this was the last of them; 2 = the block
// is shared with a neighbouring CTA and this CTA's rows arrived last.  Rows
// are first counted per CTA in shared memory (a CTA-scope fence before the
// count makes the store visible to the warp that completes the block); only
// a CTA's share of a block that straddles two CTAs goes through the global
// counter (device-scope fence, one atomic per CTA and block).
__device__ __forceinline__ int arrive_row(const RegMat& m, int row, int grow, int r_begin,
                                          int r_end, int* scnt) {
  const int bstart = grow & ~31;
  const int mine = min(r_end, bstart + 32) - max(r_begin, bstart);
  __threadfence_block();
  if (atomicAdd(scnt + ((grow >> 5) - (r_begin >> 5)), 1) + 1 != mine) return 0;
  if (mine == 32) return 1;
  __threadfence();
  return atomicAdd(m.rq_cnt + (row >> 5), mine) + mine == 32 ? 2 : 0;
}

// Shared-memory block counters a CTA needs: its row range covers at most
// ceil(rows / G) rows, i.e. this many 32-row blocks.
__host__ __device__ __forceinline__ int reg_block_slots(int rows, int G) {
  return (rows + G - 1) / G / 32 + 2;
}

// A CTA's walk over its concatenated rows, stage by stage: the matrix of the
// next row and that matrix's concatenated rows [off, end), held in
// registers.  The group (launch parameters, or shared memory) is read again
// only when the walk enters another matrix, not at every stage: a lookup
// per stage sits on the consumers' path from one stage to the next.
struct RowWalk {
  int gr;        // next concatenated row
  int mi;        // its matrix
  int off, end;
};
__device__ __forceinline__ RowWalk walk_begin(const RegGroup& grp, int r_begin) {
  RowWalk w;
  w.gr = r_begin;
  w.mi = 0;
  while (w.mi + 1 < grp.count && r_begin >= grp.m[w.mi + 1].row_off) ++w.mi;
  w.off = grp.m[w.mi].row_off;
  w.end = w.off + grp.m[w.mi].N;
  return w;
}
// The next stage (called while w.gr < r_end): at most R rows, all of one
// matrix.  Returns true when the walk entered another matrix.
__device__ __forceinline__ bool walk_next(const RegGroup& grp, RowWalk& w, int r_end, int R,
                                          int& row0, int& nrows) {
  bool entered = false;
  while (w.gr >= w.end) {
    ++w.mi;
    w.off = grp.m[w.mi].row_off;
    w.end = w.off + grp.m[w.mi].N;
    entered = true;
  }
  row0 = w.gr - w.off;
  nrows = min(R, min(r_end, w.end) - w.gr);
  w.gr += nrows;
  return entered;
}

template <int NPL, int WPR, bool ISUM, bool MOE>
__global__ void __launch_bounds__(kM1Threads, 1)
gemv_m1_reg_kernel(const __grid_constant__ RegGroup grp_param, const __grid_constant__ MoeArgs moe,
                   int K, const int8_t* __restrict__ q_all, const __half* __restrict__ d_all,
                   int32_t* __restrict__ isum) {
  extern __shared__ __align__(128) uint8_t smem[];
  // the matrices: from the launch parameters, or (mixture of experts) built
  // in shared memory from the routing ids
  __shared__ RegGroup moe_grp;
  const RegGroup& grp = MOE ? moe_grp : grp_param;
  // token of this grid row (several only for mixture-of-experts launches)
  const int8_t* __restrict__ q = q_all + static_cast<size_t>(blockIdx.y) * K;
  const __half* __restrict__ d = d_all + static_cast<size_t>(blockIdx.y) * (K / 32);
  const int R = reg_rows(K, WPR);
  const int active = R * WPR;                      // consumer warps in use
  const uint32_t row_code = K / 2, row_scale = K / 16;
  const uint32_t stage_bytes = static_cast<uint32_t>(R) * (row_code + row_scale);
  const uint32_t codes_bytes = static_cast<uint32_t>(R) * row_code;
  float* part = reinterpret_cast<float*>(smem + kM1Stages * stage_bytes);  // [stage][warp]
  uint64_t* full = reinterpret_cast<uint64_t*>(part + kM1Stages * kM1Consumers);
  uint64_t* empty = full + kM1Stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kM1Stages);
  int* scnt = reinterpret_cast<int*>(empty + kM1Stages + 2);   // block counters of this CTA

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;

  grid_dependents_launch();
  if constexpr (MOE) {
    // the routing ids come from the previous kernel
    grid_dependency_wait();
    if (threadIdx.x == 0) {
      const int t = blockIdx.y;
      int rows = 0, cnt = 0;
      for (int j = 0; j < moe.top_k; ++j) {
        const int e = moe.ids[t * moe.top_k + j];
        if (e < 0 || e >= moe.E) {
          raise_bad_index();
          continue;
        }
        RegMat m = {};
        m.codes = moe.codes + static_cast<size_t>(e) * moe.N * (K / 2);
        m.scales = moe.scales + static_cast<size_t>(e) * moe.N * (K / 16);
        m.y = moe.y + (static_cast<size_t>(t) * moe.top_k + j) * moe.N;
        m.half_g = 0.5f * moe.g[e];
        m.N = moe.N;
        m.row_off = rows;
        rows += moe.N;
        moe_grp.m[cnt++] = m;
      }
      moe_grp.count = cnt;
      moe_grp.rows = rows;
    }
  } else {
    for (int i = threadIdx.x; i < reg_block_slots(grp_param.rows, G); i += blockDim.x) scnt[i] = 0;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < kM1Stages; ++i) {
      ptx::mbar_init(ptx::smem_addr(full + i), 1);
      ptx::mbar_init(ptx::smem_addr(empty + i), active);
    }
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  const int r_begin = static_cast<int>(static_cast<int64_t>(blockIdx.x) * grp.rows / G);
  const int r_end = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * grp.rows / G);

  if (warp == kM1Consumers) {
    // ------------- producer: bulk copies, and the sum of row partials --------
    // The weights are not written by the kernels before this one, so the
    // first ring stages are requested before waiting for them; everything
    // the producer writes (row sums, requantisation) comes after the wait.
    if (lane != 0) return;
    bool waited = false;
    int smi[kM1Stages] = {}, srow[kM1Stages] = {}, snr[kM1Stages] = {};   // stages in flight
    auto finalize = [&](int it) {   // rows of stage `it`, once its slot is empty
      if (WPR == 1) return;
      const int s = it % kM1Stages;
      const RegMat& m = grp.m[smi[s]];
      for (int r = 0; r < snr[s]; ++r) {
        float v = 0.0f;
#pragma unroll
        for (int p = 0; p < WPR; ++p) v += part[s * kM1Consumers + r * WPR + p];
        const int row = srow[s] + r;
        m.y[row] = v * m.half_g;
        if (m.rq_q != nullptr) {
          const int how = arrive_row(m, row, m.row_off + row, r_begin, r_end, scnt);
          if (how != 0) {
            if (how == 1) __threadfence_block(); else __threadfence();
            requant_block_thread(m, row >> 5);
            if (how == 2) atomicExch(m.rq_cnt + (row >> 5), 0);
          }
        }
      }
    };
    int issued = 0;
    bool ok = true;
    RowWalk wk = walk_begin(grp, r_begin);
    const uint8_t* m_codes = grp.m[wk.mi].codes;
    const uint8_t* m_scales = grp.m[wk.mi].scales;
    for (int it = 0; wk.gr < r_end; ++it) {
      const int s = it % kM1Stages;
      const uint32_t ph = (it / kM1Stages) & 1;
      if (it == kM1Stages) {
        grid_dependency_wait();
        waited = true;
      }
      if (!ptx::mbar_wait_bounded(ptx::smem_addr(empty + s), ph ^ 1, abort_flag, kWaitLimitNs)) {
        *abort_flag = 1;
        raise_timeout();
        ok = false;
        break;
      }
      if (it >= kM1Stages) finalize(it - kM1Stages);
      int row0, nrows;
      if (walk_next(grp, wk, r_end, R, row0, nrows)) {
        m_codes = grp.m[wk.mi].codes;
        m_scales = grp.m[wk.mi].scales;
      }
      smi[s] = wk.mi;
      srow[s] = row0;
      snr[s] = nrows;
      const uint32_t bar = ptx::smem_addr(full + s);
      uint8_t* st = smem + s * stage_bytes;
      ptx::mbar_arrive_expect_tx(bar, nrows * (row_code + row_scale));
      ptx::bulk_load(ptx::smem_addr(st), m_codes + static_cast<size_t>(row0) * row_code,
                     nrows * row_code, bar);
      ptx::bulk_load(ptx::smem_addr(st + codes_bytes),
                     m_scales + static_cast<size_t>(row0) * row_scale, nrows * row_scale, bar);
      ++issued;
    }
    if (!waited) grid_dependency_wait();
    if (ok) {
      // the last stages: wait until consumed, then add their partials
      for (int it = max(0, issued - kM1Stages); it < issued; ++it) {
        if (!ptx::mbar_wait_bounded(ptx::smem_addr(empty + it % kM1Stages),
                                    (it / kM1Stages) & 1, abort_flag, kWaitLimitNs)) {
          *abort_flag = 1;
          raise_timeout();
          break;
        }
        finalize(it);
      }
    } else {
      for (int it = max(0, issued - kM1Stages); it < issued; ++it)
        ptx::mbar_wait_bounded(ptx::smem_addr(full + it % kM1Stages), (it / kM1Stages) & 1,
                               nullptr, kWaitLimitNs);
    }
    return;
  }

  // ------------- consumers: warp w = (row w / WPR, part w % WPR) -------------
  if (warp >= active) return;
  grid_dependency_wait();   // the activations (and y's readers) of the previous kernel
  const int rl = warp / WPR;
  const int p = warp % WPR;
  uint4 qa[NPL], qb[NPL];
  float dd[NPL];
  int c0[NPL], c1[NPL];
  // each lane loads its own activation chunks straight into registers
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int c = p * (NPL * 32) + lane + 32 * i;
    const uint4* src = reinterpret_cast<const uint4*>(q) + 2 * c;
    qa[i] = __ldg(src);
    qb[i] = __ldg(src + 1);
    dd[i] = __half2float(__ldg(d + c));
    const int s0 = dev::dp4a(qa[i].x, 0x01010101u, dev::dp4a(qa[i].y, 0x01010101u,
                   dev::dp4a(qa[i].z, 0x01010101u, dev::dp4a(qa[i].w, 0x01010101u, 0))));
    const int s1 = dev::dp4a(qb[i].x, 0x01010101u, dev::dp4a(qb[i].y, 0x01010101u,
                   dev::dp4a(qb[i].z, 0x01010101u, dev::dp4a(qb[i].w, 0x01010101u, 0))));
    c0[i] = -12 * s0;
    c1[i] = -12 * s1;
  }
  // the epilogue's fields of the current matrix, in registers
  RowWalk wk = walk_begin(grp, r_begin);
  float* m_y = grp.m[wk.mi].y;
  float m_half_g = grp.m[wk.mi].half_g;
  bool m_rq = grp.m[wk.mi].rq_q != nullptr;
  for (int it = 0; wk.gr < r_end; ++it) {
    const int s = it % kM1Stages;
    const uint32_t ph = (it / kM1Stages) & 1;
    int row0, nrows;
    if (walk_next(grp, wk, r_end, R, row0, nrows)) {
      m_y = grp.m[wk.mi].y;
      m_half_g = grp.m[wk.mi].half_g;
      m_rq = grp.m[wk.mi].rq_q != nullptr;
    }
    if (!ptx::mbar_wait_bounded(ptx::smem_addr(full + s), ph, abort_flag, kWaitLimitNs)) {
      *abort_flag = 1;
      raise_timeout();
      break;
    }
    float acc = 0.0f;
    if (rl < nrows) {
      const uint8_t* st = smem + s * stage_bytes;
      const uint4* cw = reinterpret_cast<const uint4*>(st + rl * row_code) + p * (NPL * 32);
      const uint16_t* sw =
          reinterpret_cast<const uint16_t*>(st + codes_bytes + rl * row_scale) + p * (NPL * 32);
      uint4 w[NPL];
      uint32_t s2[NPL];
#pragma unroll
      for (int i = 0; i < NPL; ++i) {
        w[i] = cw[lane + 32 * i];
        s2[i] = sw[lane + 32 * i];
      }
#pragma unroll
      for (int i = 0; i < NPL; ++i) {
        const int i0 = dev::dot16_biased(w[i].x, w[i].y, qa[i], c0[i]);
        const int i1 = dev::dot16_biased(w[i].z, w[i].w, qb[i], c1[i]);
        if constexpr (ISUM)
          store_isum(isum, 0, grp.m[wk.mi].N, row0 + rl, K, p * (NPL * 32) + lane + 32 * i, i0,
                     i1);
        const float2 sf = dev::ue4m3x2_to_float2(s2[i]);
        acc = fmaf(dd[i], fmaf(sf.x, static_cast<float>(i0), sf.y * static_cast<float>(i1)), acc);
      }
      acc = dev::warp_sum(acc);
      if (WPR == 1) {
        const int row = row0 + rl;
        int how = 0;
        if (lane == 0) m_y[row] = acc * m_half_g;
        if (m_rq) {
          const RegMat& m = grp.m[wk.mi];
          if (lane == 0) how = arrive_row(m, row, m.row_off + row, r_begin, r_end, scnt);
          how = __shfl_sync(0xffffffffu, how, 0);
          if (how != 0) {
            if (how == 1) __threadfence_block(); else __threadfence();
            requant_block_warp(m, row >> 5, lane);
            if (how == 2 && lane == 0) atomicExch(m.rq_cnt + (row >> 5), 0);
          }
        }
      } else if (lane == 0) {
        part[s * kM1Consumers + warp] = acc;
      }
    }
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(empty + s));
  }
}

// ---------------------------------------------------------------------------
// The linears of a decoder stack at one token in one persistent launch
// ---------------------------------------------------------------------------
// Matrices of a layer: q, k, v (input Q8_0(x)), o (input Q8_0(y_v)), up,
// gate (input Q8_0(y_o)), down (input Q8_0(y_up)); v, o and up also emit the
// Q8_0 of their output.  Every CTA takes an even slice of the rows of every
// matrix, always in the same order of units (matrix, layer):
//   v0 q0 k0 o0 | v1 q1 k1 up0 gate0 down0 o1 | v2 q2 k2 up1 gate1 down1 o2 | ...
// so each unit that needs another unit's output finds it finished long
// before: v before q and k (o waits for v), the next layer's v, q, k between
// o and up (up and gate wait for o), up before gate (down waits for up).  A
// finished unit raises a grid counter (its warps count in shared memory and
// the last one adds 1 per CTA); a waiting warp reads the counter with
// acquire semantics, so usually it is already complete.  The weights do not
// depend on any activation, so the producer streams stage after stage across
// units and layers.  The requantised activations alternate between two
// buffers by layer parity, so no unit overwrites an input that a slower CTA
// may still read.  The launch is cooperative (all CTAs resident); every wait
// is bounded (4 s) and a timeout raises the GEMV error flag and stops the CTA.
constexpr int kStackMaxLayers = 64;
constexpr int kStackLin = 7;
constexpr int kStackScnt = 16;     // block counters per requantised matrix and CTA
constexpr int kStackArr = 8;       // ring of per-CTA arrival counters
enum : int { kSq = 0, kSk, kSv, kSo, kSup, kSgate, kSdown };

struct StackArgs {
  const uint8_t* codes[kStackMaxLayers * kStackLin];
  const uint8_t* scales[kStackMaxLayers * kStackLin];
  float half_g[kStackMaxLayers * kStackLin];
  float* outs[kStackLin];
  const int8_t* x_q;              // Q8_0(x)
  const __half* x_d;
  int8_t* b_q[3][2];              // Q8_0 of y_v, y_o, y_up, by layer parity
  __half* b_d[3][2];
  int* rq_cnt[3];                 // global block counters of v, o, up
  unsigned int* bar;              // [layer][3] CTAs done with v, o, up
  int n_layers;
  int N[kStackLin];
  int K0;                         // K of q, k, v, o, up, gate
  int Kd;                         // K of down (= N of up)
};

// Unit u of the schedule -> (layer, matrix).  7 units per layer: the first
// four are v0 q0 k0 o0, then per layer l a block v(l+1) q(l+1) k(l+1) up(l)
// gate(l) down(l) o(l+1), the last layer's block only up, gate, down.
__device__ __forceinline__ void stack_unit(int u, int L, int& l, int& m) {
  if (u < 4) {
    l = 0;
    m = u == 3 ? kSo : (u == 0 ? kSv : u - 1);
    return;
  }
  u -= 4;
  l = u / 7;
  int r = u % 7;
  if (l >= L - 1) {
    l = L - 1;
    r = u - 7 * (L - 1) + 3;
  }
  if (r < 3) {
    m = r == 0 ? kSv : r - 1;
    ++l;
  } else if (r < 6) {
    m = kSup + (r - 3);
  } else {
    m = kSo;
    ++l;
  }
}
// requantised-matrix index (v, o, up) or -1; its counter instance k = 3l + index
__device__ __forceinline__ int stack_rq(int m) {
  return m == kSv ? 0 : m == kSo ? 1 : m == kSup ? 2 : -1;
}
// the unit a matrix waits for: o waits for v, up for o, down for up
__device__ __forceinline__ int stack_dep(int m) {
  return m == kSo ? 0 : m == kSup ? 1 : m == kSdown ? 2 : -1;
}

__device__ __forceinline__ unsigned int ld_acquire_u32(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// Waits until *ctr >= target (bounded; false on timeout or abort).
__device__ __forceinline__ bool wait_counter(const unsigned int* ctr, unsigned int target,
                                             volatile int* abort_flag) {
  const uint64_t t0 = ptx::globaltimer_ns();
  while (ld_acquire_u32(ctr) < target) {
    if (*abort_flag) return false;
    if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) return false;
    __nanosleep(256);
  }
  return true;
}

struct StackCta {                 // what a consumer warp needs of its CTA
  uint8_t* smem;
  float* part;
  uint64_t* full;
  uint64_t* empty;
  int* arrived;                   // [kStackArr] warps done, per counter instance
  int* scnt;                      // [3][kStackScnt] rows per 32-row block
  volatile int* abort_flag;
  int warp, lane, G;
};

// A warp waits until every CTA has finished a unit (lane 0 polls).
__device__ __forceinline__ bool stack_wait(const unsigned int* ctr, const StackCta& c) {
  int ok = 1;
  if (c.lane == 0) ok = wait_counter(ctr, static_cast<unsigned int>(c.G), c.abort_flag) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// A run of units with the same input for one consumer warp: the activations
// once into registers, then for each unit its wait (if any), its stages and
// its arrival (if it is v, o or up).  Returns false on a timeout or abort.
template <int NPL, int WPR>
__device__ __forceinline__ bool stack_consume(const StackArgs& a, const StackCta& c, int u0,
                                              int u1, const int8_t* q, const __half* d, int K,
                                              int& it) {
  const int warp = c.warp, lane = c.lane;
  const int R = reg_rows(K, WPR);
  const int active = R * WPR;
  const uint32_t row_code = K / 2, row_scale = K / 16;
  const uint32_t codes_bytes = static_cast<uint32_t>(R) * row_code;
  const int rl = warp / WPR;
  const int pt = warp % WPR;
  // the first unit's wait comes before its input is read
  {
    int l, m;
    stack_unit(u0, a.n_layers, l, m);
    const int dep = stack_dep(m);
    if (dep >= 0 && !stack_wait(a.bar + 3 * l + dep, c)) return false;
  }
  uint4 qa[NPL], qb[NPL];
  float dd[NPL];
  int c0[NPL], c1[NPL];
  // written during this launch by other CTAs: read through L2
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int ch = pt * (NPL * 32) + lane + 32 * i;
    const uint4* src = reinterpret_cast<const uint4*>(q) + 2 * ch;
    qa[i] = __ldcg(src);
    qb[i] = __ldcg(src + 1);
    dd[i] = __half2float(__ushort_as_half(__ldcg(reinterpret_cast<const unsigned short*>(d) + ch)));
    const int s0 = dev::dp4a(qa[i].x, 0x01010101u, dev::dp4a(qa[i].y, 0x01010101u,
                   dev::dp4a(qa[i].z, 0x01010101u, dev::dp4a(qa[i].w, 0x01010101u, 0))));
    const int s1 = dev::dp4a(qb[i].x, 0x01010101u, dev::dp4a(qb[i].y, 0x01010101u,
                   dev::dp4a(qb[i].z, 0x01010101u, dev::dp4a(qb[i].w, 0x01010101u, 0))));
    c0[i] = -12 * s0;
    c1[i] = -12 * s1;
  }
  for (int u = u0; u < u1; ++u) {
    int l, m;
    stack_unit(u, a.n_layers, l, m);
    const int dep = stack_dep(m);
    if (u > u0 && dep >= 0 && !stack_wait(a.bar + 3 * l + dep, c)) return false;
    const int N = a.N[m];
    const int r_begin = static_cast<int>(static_cast<int64_t>(blockIdx.x) * N / c.G);
    const int r_end = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * N / c.G);
    const int li = l * kStackLin + m;
    const int rq = stack_rq(m);
    float* y = a.outs[m];
    const float half_g = a.half_g[li];   // once per unit (see the producer)
    for (int row0 = r_begin; row0 < r_end; row0 += R, ++it) {
      const int nrows = min(R, r_end - row0);
      const int s = it % kM1Stages;
      const uint32_t ph = (it / kM1Stages) & 1;
      if (!ptx::mbar_wait_bounded(ptx::smem_addr(c.full + s), ph, c.abort_flag, kWaitLimitNs))
        return false;
      if (warp < active && rl < nrows) {
        const uint8_t* st = c.smem + s * kRegStageMax;
        const uint4* cw = reinterpret_cast<const uint4*>(st + rl * row_code) + pt * (NPL * 32);
        const uint16_t* sw =
            reinterpret_cast<const uint16_t*>(st + codes_bytes + rl * row_scale) + pt * (NPL * 32);
        uint4 w[NPL];
        uint32_t s2[NPL];
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
          w[i] = cw[lane + 32 * i];
          s2[i] = sw[lane + 32 * i];
        }
        float acc = 0.0f;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
          const int i0 = dev::dot16_biased(w[i].x, w[i].y, qa[i], c0[i]);
          const int i1 = dev::dot16_biased(w[i].z, w[i].w, qb[i], c1[i]);
          const float2 sf = dev::ue4m3x2_to_float2(s2[i]);
          acc = fmaf(dd[i], fmaf(sf.x, static_cast<float>(i0), sf.y * static_cast<float>(i1)), acc);
        }
        acc = dev::warp_sum(acc);
        if (WPR == 1) {
          const int row = row0 + rl;
          int how = 0;
          if (lane == 0) {
            y[row] = acc * half_g;
            if (rq >= 0) {
              // rows of this CTA per 32-row block counted in shared memory
              // (reset by the row that completes the CTA's share), the share
              // of a block that straddles two CTAs through the global counter
              const int bstart = row & ~31;
              const int mine = min(r_end, bstart + 32) - max(r_begin, bstart);
              int* sc = c.scnt + rq * kStackScnt + ((row >> 5) - (r_begin >> 5));
              __threadfence_block();
              if (atomicAdd(sc, 1) + 1 == mine) {
                atomicExch(sc, 0);
                if (mine == 32) {
                  how = 1;
                } else {
                  __threadfence();
                  if (atomicAdd(a.rq_cnt[rq] + (row >> 5), mine) + mine == 32) how = 2;
                }
              }
            }
          }
          if (rq >= 0) {
            how = __shfl_sync(0xffffffffu, how, 0);
            if (how != 0) {
              if (how == 1) __threadfence_block(); else __threadfence();
              RegMat rm = {};
              rm.y = y;
              rm.rq_q = a.b_q[rq][l & 1];
              rm.rq_d = a.b_d[rq][l & 1];
              requant_block_warp(rm, row >> 5, lane);
              if (how == 2 && lane == 0) atomicExch(a.rq_cnt[rq] + (row >> 5), 0);
            }
          }
        } else if (lane == 0) {
          c.part[s * kM1Consumers + warp] = acc;
        }
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(c.empty + s));
    }
    if (rq >= 0) {
      // this warp's rows and requantisations of the unit are written: count
      // it; the CTA's last warp raises the grid counter once
      const int k = 3 * l + rq;
      __threadfence();
      __syncwarp();
      if (lane == 0 && atomicAdd(c.arrived + k % kStackArr, 1) == kM1Consumers - 1) {
        c.arrived[k % kStackArr] = 0;
        __threadfence();
        atomicAdd(a.bar + k, 1u);
      }
      __syncwarp();
    }
  }
  return true;
}

template <int NPL0, int NPL3, int WPR3>
__global__ void __launch_bounds__(kM1Threads, 1)
stack_m1_kernel(const __grid_constant__ StackArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  float* part = reinterpret_cast<float*>(smem + kM1Stages * kRegStageMax);   // [stage][warp]
  uint64_t* full = reinterpret_cast<uint64_t*>(part + kM1Stages * kM1Consumers);
  uint64_t* empty = full + kM1Stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kM1Stages);
  int* arrived = reinterpret_cast<int*>(empty + kM1Stages + 1);   // [kStackArr]
  int* scnt = arrived + kStackArr;                                 // [3][kStackScnt]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int L = a.n_layers;
  const int units = kStackLin * L;

  grid_dependents_launch();
  for (int i = threadIdx.x; i < kStackArr + 3 * kStackScnt; i += blockDim.x) arrived[i] = 0;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kM1Stages; ++i) {
      ptx::mbar_init(ptx::smem_addr(full + i), 1);
      ptx::mbar_init(ptx::smem_addr(empty + i), kM1Consumers);
    }
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();

  if (warp == kM1Consumers) {
    // ---------------- producer: the weight stages of every unit --------------
    if (lane != 0) return;
    bool waited = false;
    int sli[kM1Stages] = {}, srow[kM1Stages] = {}, snr[kM1Stages] = {};
    bool sfin[kM1Stages] = {};
    auto finalize = [&](int it) {   // rows of a down stage: sum of the WPR3 partials
      const int s = it % kM1Stages;
      if (!sfin[s]) return;
      float* y = a.outs[kSdown];
      const float hg = a.half_g[sli[s]];
      for (int r = 0; r < snr[s]; ++r) {
        float v = 0.0f;
#pragma unroll
        for (int pp = 0; pp < WPR3; ++pp) v += part[s * kM1Consumers + r * WPR3 + pp];
        y[srow[s] + r] = v * hg;
      }
    };
    int it = 0;
    bool ok = true;
    for (int u = 0; u < units && ok; ++u) {
      int l, m;
      stack_unit(u, L, l, m);
      const int K = m == kSdown ? a.Kd : a.K0;
      const int R = m == kSdown ? reg_rows(K, WPR3) : reg_rows(K, 1);
      const uint32_t row_code = K / 2, row_scale = K / 16;
      const uint32_t codes_bytes = static_cast<uint32_t>(R) * row_code;
      const int N = a.N[m];
      const int r_begin = static_cast<int>(static_cast<int64_t>(blockIdx.x) * N / G);
      const int r_end = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * N / G);
      const int li = l * kStackLin + m;
      // the unit's matrix, read once from the launch parameters (a lookup
      // with a dynamic index is a generic load that a store may not pass)
      const uint8_t* const codes = a.codes[li];
      const uint8_t* const scales = a.scales[li];
      for (int row0 = r_begin; row0 < r_end; row0 += R) {
        const int nrows = min(R, r_end - row0);
        const int s = it % kM1Stages;
        const uint32_t ph = (it / kM1Stages) & 1;
        if (it == kM1Stages) {
          grid_dependency_wait();
          waited = true;
        }
        if (!ptx::mbar_wait_bounded(ptx::smem_addr(empty + s), ph ^ 1, abort_flag, kWaitLimitNs)) {
          *abort_flag = 1;
          raise_timeout();
          ok = false;
          break;
        }
        if (it >= kM1Stages) finalize(it - kM1Stages);
        sli[s] = li;
        srow[s] = row0;
        snr[s] = nrows;
        sfin[s] = m == kSdown && WPR3 > 1;
        const uint32_t bar = ptx::smem_addr(full + s);
        uint8_t* st = smem + s * kRegStageMax;
        ptx::mbar_arrive_expect_tx(bar, nrows * (row_code + row_scale));
        ptx::bulk_load(ptx::smem_addr(st), codes + static_cast<size_t>(row0) * row_code,
                       nrows * row_code, bar);
        ptx::bulk_load(ptx::smem_addr(st + codes_bytes),
                       scales + static_cast<size_t>(row0) * row_scale, nrows * row_scale, bar);
        ++it;
      }
    }
    if (!waited) grid_dependency_wait();
    if (ok) {
      for (int i = max(0, it - kM1Stages); i < it; ++i) {
        if (!ptx::mbar_wait_bounded(ptx::smem_addr(empty + i % kM1Stages), (i / kM1Stages) & 1,
                                    abort_flag, kWaitLimitNs)) {
          *abort_flag = 1;
          raise_timeout();
          break;
        }
        finalize(i);
      }
    } else {
      for (int i = max(0, it - kM1Stages); i < it; ++i)
        ptx::mbar_wait_bounded(ptx::smem_addr(full + i % kM1Stages), (i / kM1Stages) & 1, nullptr,
                               kWaitLimitNs);
    }
    return;
  }

  // ---------------- consumers: runs of units with the same input ----------------
  grid_dependency_wait();   // Q8_0(x) from the quantiser before this kernel
  const StackCta c = {smem, part, full, empty, arrived, scnt, abort_flag, warp, lane, G};
  int it = 0;
  int u = 0;
  while (u < units) {
    int l, m;
    stack_unit(u, L, l, m);
    // the run: v q k (Q8_0(x)), o, up gate, down
    const int len = (m == kSv || m == kSup) ? (m == kSv ? 3 : 2) : 1;
    bool ok;
    if (m == kSdown) {
      ok = stack_consume<NPL3, WPR3>(a, c, u, u + len, a.b_q[2][l & 1], a.b_d[2][l & 1], a.Kd, it);
    } else {
      const int8_t* q = m == kSv ? a.x_q : m == kSo ? a.b_q[0][l & 1] : a.b_q[1][l & 1];
      const __half* d = m == kSv ? a.x_d : m == kSo ? a.b_d[0][l & 1] : a.b_d[1][l & 1];
      ok = stack_consume<NPL0, 1>(a, c, u, u + len, q, d, a.K0, it);
    }
    if (!ok) {
      *abort_flag = 1;
      raise_timeout();
      return;
    }
    u += len;
  }
}

// ---------------------------------------------------------------------------
// M = 2..16 (and fallback M = 1) schedule: persistent CTAs, TMA ring
// ---------------------------------------------------------------------------
template <int MT, bool ISUM>
__global__ void __launch_bounds__(kTmaThreads, 2)
gemv_tma_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                float half_g, int N, int K, int seg, const int8_t* __restrict__ q,
                const __half* __restrict__ d, float* __restrict__ y,
                int32_t* __restrict__ isum) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t stage_bytes = tma_stage_bytes(seg);
  const uint32_t codes_bytes = kTmaConsumers * (seg / 2);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kTmaStages * stage_bytes);
  uint64_t* empty = full + kTmaStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kTmaStages);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int r_begin = static_cast<int>(static_cast<int64_t>(blockIdx.x) * N / G);
  const int r_end = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * N / G);
  const int ngroups = (r_end - r_begin + kTmaConsumers - 1) / kTmaConsumers;
  const int nseg = K / seg;
  const int total = ngroups * nseg;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kTmaStages; ++i) {
      ptx::mbar_init(ptx::smem_addr(full + i), 1);
      ptx::mbar_init(ptx::smem_addr(empty + i), kTmaConsumers);
    }
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();

  if (warp == kTmaConsumers) {
    // ---------------- producer: one thread issues the bulk copies ----------
    if (lane != 0) return;
    int issued = 0;
    for (int it = 0; it < total; ++it) {
      const int s = it % kTmaStages;
      const uint32_t ph = (it / kTmaStages) & 1;
      if (!ptx::mbar_wait_bounded(ptx::smem_addr(empty + s), ph ^ 1, abort_flag, kWaitLimitNs)) {
        *abort_flag = 1;
        raise_timeout();
        break;
      }
      const int grp = it / nseg, sg = it % nseg;
      const int row0 = r_begin + grp * kTmaConsumers;
      const int nrows = min(kTmaConsumers, r_end - row0);
      const uint32_t bar = ptx::smem_addr(full + s);
      uint8_t* st = smem + s * stage_bytes;
      ptx::mbar_arrive_expect_tx(bar, nrows * (seg / 2 + seg / 16));
      if (nseg == 1) {
        ptx::bulk_load(ptx::smem_addr(st), codes + static_cast<size_t>(row0) * (K / 2),
                       nrows * (K / 2), bar);
        ptx::bulk_load(ptx::smem_addr(st + codes_bytes),
                       scales + static_cast<size_t>(row0) * (K / 16), nrows * (K / 16), bar);
      } else {
        for (int r = 0; r < nrows; ++r) {
          ptx::bulk_load(ptx::smem_addr(st + r * (seg / 2)),
                         codes + static_cast<size_t>(row0 + r) * (K / 2) + sg * (seg / 2),
                         seg / 2, bar);
          ptx::bulk_load(ptx::smem_addr(st + codes_bytes + r * (seg / 16)),
                         scales + static_cast<size_t>(row0 + r) * (K / 16) + sg * (seg / 16),
                         seg / 16, bar);
        }
      }
      ++issued;
    }
    if (*abort_flag) {
      // let the copies already in flight land before the CTA exits
      for (int it = max(0, issued - kTmaStages); it < issued; ++it)
        ptx::mbar_wait_bounded(ptx::smem_addr(full + it % kTmaStages),
                               (it / kTmaStages) & 1, nullptr, kWaitLimitNs);
    }
    return;
  }

  // ---------------- consumers: warp w owns row w of each group ------------
  float acc[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
  const int nch = seg / 32;
  for (int it = 0; it < total; ++it) {
    const int s = it % kTmaStages;
    const uint32_t ph = (it / kTmaStages) & 1;
    if (!ptx::mbar_wait_bounded(ptx::smem_addr(full + s), ph, abort_flag, kWaitLimitNs)) {
      *abort_flag = 1;
      raise_timeout();
      break;
    }
    const int grp = it / nseg, sg = it % nseg;
    const int row0 = r_begin + grp * kTmaConsumers;
    const int nrows = min(kTmaConsumers, r_end - row0);
    if (warp < nrows) {
      const uint8_t* st = smem + s * stage_bytes;
      const uint4* sc = reinterpret_cast<const uint4*>(st + warp * (seg / 2));
      const uint16_t* ss = reinterpret_cast<const uint16_t*>(st + codes_bytes + warp * (seg / 16));
      const int cbase = sg * nch;
#pragma unroll 4
      for (int j = lane; j < nch; j += 32) {
        uint32_t cw[8];
        decode_chunk_signed(sc[j], cw);
        const float2 sf = dev::ue4m3x2_to_float2(ss[j]);
        const int c = cbase + j;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const int2 is = chunk_isums(cw, q + static_cast<size_t>(m) * K, c);
          if constexpr (ISUM) store_isum(isum, m, N, row0 + warp, K, c, is.x, is.y);
          const float dm = __half2float(__ldg(d + static_cast<size_t>(m) * (K >> 5) + c));
          acc[m] += dm * fmaf(sf.x, static_cast<float>(is.x), sf.y * static_cast<float>(is.y));
        }
      }
    }
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(empty + s));
    if (sg == nseg - 1) {
      if (warp < nrows) {
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const float v = dev::warp_sum(acc[m]);
          if (lane == 0) y[static_cast<size_t>(m) * N + row0 + warp] = v * half_g;
        }
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
    }
  }
}

// ---------------------------------------------------------------------------
// any K % 64 == 0: one warp per row, loads straight to registers
// ---------------------------------------------------------------------------
template <int MT, bool ISUM>
__global__ void __launch_bounds__(kWarps * 32)
gemv_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
            float half_g, int N, int K, const int8_t* __restrict__ q,
            const __half* __restrict__ d, float* __restrict__ y, int32_t* __restrict__ isum) {
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
        decode_chunk_signed(wv[u], cw);
        const float2 s = dev::ue4m3x2_to_float2(sv[u]);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const int2 is = chunk_isums(cw, q + static_cast<size_t>(m) * K, c);
          if constexpr (ISUM) store_isum(isum, m, N, row, K, c, is.x, is.y);
          const float dm = __half2float(__ldg(d + static_cast<size_t>(m) * (K >> 5) + c));
          acc[m] = fmaf(dm, fmaf(s.x, static_cast<float>(is.x), s.y * static_cast<float>(is.y)), acc[m]);
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

// ---------------------------------------------------------------------------
// test-only: a pipeline wait that never completes
// ---------------------------------------------------------------------------
// One consumer waits, through the same bounded wait as the GEMV pipelines,
// for a stage whose producer never issues its copy (the barrier's phase can
// never complete).  The wait gives up after limit_ns, raises the GEMV
// timeout flag exactly as a stalled GEMV would, and the kernel returns.
__global__ void __launch_bounds__(32)
stalled_wait_kernel(uint64_t limit_ns, int* __restrict__ result) {
  __shared__ __align__(8) uint64_t full;
  if (threadIdx.x != 0) return;
  ptx::mbar_init(ptx::smem_addr(&full), 1);
  ptx::fence_mbar_init();
  const uint64_t t0 = ptx::globaltimer_ns();
  const bool got = ptx::mbar_wait_bounded(ptx::smem_addr(&full), 0, nullptr, limit_ns);
  if (!got) raise_timeout();
  result[0] = got ? 1 : 0;
  const uint64_t us = (ptx::globaltimer_ns() - t0) / 1000;
  result[1] = us > 0x7fffffffull ? 0x7fffffff : static_cast<int>(us);
}

// K elements per TMA stage and row: the largest multiple of 256 that divides
// K and is at most kTmaMaxSeg; 0 when K is not a multiple of 256 (scale rows
// would not be 16-byte aligned for the bulk copies).
int tma_segment(int64_t K) {
  if (K % 256 != 0) return 0;
  for (int64_t seg = (kTmaMaxSeg / 256) * 256; seg >= 256; seg -= 256)
    if (K % seg == 0) return static_cast<int>(seg);
  return 0;
}

template <int NPL, bool ISUM>
cudaError_t launch_m1(const uint8_t* codes, const uint8_t* scales, float g, int64_t N,
                      int64_t K, int seg, const int8_t* q, const uint16_t* d, float* y,
                      int32_t* isum, cudaStream_t stream) {
  static SmemAttrOnce attr;
  cudaError_t e = attr.ensure(gemv_m1_kernel<NPL, ISUM>, static_cast<int>(kSmemPerCtaMax));
  if (e != cudaSuccess) return e;
  const int64_t ctas = std::min<int64_t>(device_sm_count(), N);
  gemv_m1_kernel<NPL, ISUM><<<static_cast<unsigned>(ctas), kM1Threads,
                              m1_smem_bytes(static_cast<int>(K), seg), stream>>>(
      codes, scales, 0.5f * g, static_cast<int>(N), static_cast<int>(K), seg, q,
      reinterpret_cast<const __half*>(d), y, isum);
  return cudaGetLastError();
}

template <int NPL, int WPR, bool ISUM>
cudaError_t launch_m1_reg(const RegGroup& grp, int64_t K, const int8_t* q, const uint16_t* d,
                          int32_t* isum, cudaStream_t stream) {
  auto kernel = gemv_m1_reg_kernel<NPL, WPR, ISUM, false>;
  static SmemAttrOnce attr;
  cudaError_t e = attr.ensure(kernel, static_cast<int>(kRegDynSmemMax));
  if (e != cudaSuccess) return e;
  const int64_t ctas = std::min<int64_t>(device_sm_count(), grp.rows);
  const uint32_t smem = reg_smem_bytes(static_cast<int>(K), WPR) +
                        4u * reg_block_slots(grp.rows, static_cast<int>(ctas));
  if (smem > kRegDynSmemMax) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas));
  cfg.blockDim = dim3(kM1Threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  const MoeArgs no_moe = {};
  return cudaLaunchKernelEx(&cfg, kernel, grp, no_moe, static_cast<int>(K), q,
                            reinterpret_cast<const __half*>(d), isum);
}

template <int NPL, int WPR>
cudaError_t launch_moe_reg(const MoeArgs& moe, int64_t T, int64_t K, const int8_t* q,
                           const uint16_t* d, cudaStream_t stream) {
  auto kernel = gemv_m1_reg_kernel<NPL, WPR, false, true>;
  static SmemAttrOnce attr;
  cudaError_t e = attr.ensure(kernel, static_cast<int>(kRegDynSmemMax));
  if (e != cudaSuccess) return e;
  // the SMs split evenly over the tokens; each token's rows over its CTAs
  const int64_t per_token = std::max<int64_t>(1, device_sm_count() / T);
  const int64_t rows = static_cast<int64_t>(moe.top_k) * moe.N;
  const int64_t ctas = std::min<int64_t>(per_token, rows);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas), static_cast<unsigned>(T));
  cfg.blockDim = dim3(kM1Threads);
  cfg.dynamicSmemBytes = reg_smem_bytes(static_cast<int>(K), WPR);
  cfg.stream = stream;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  const RegGroup none = {};
  return cudaLaunchKernelEx(&cfg, kernel, none, moe, static_cast<int>(K), q,
                            reinterpret_cast<const __half*>(d), static_cast<int32_t*>(nullptr));
}

// The register schedule covers K = 1024 * NPL * WPR for the (NPL, WPR) pairs
// instantiated here; returns cudaErrorNotSupported for other K.
bool reg_supported(int64_t K) {
  if (K % 1024 != 0) return false;
  switch (K / 1024) {
    case 2: case 3: case 4: case 5: case 6: case 8: case 10: case 12: case 15: case 16:
    case 20: case 25:
      return true;
    default:
      return false;
  }
}

template <bool ISUM>
cudaError_t launch_m1_reg_group(const RegGroup& grp, int64_t K, const int8_t* q,
                                const uint16_t* d, int32_t* isum, cudaStream_t stream) {
  if (!reg_supported(K)) return cudaErrorNotSupported;
#define NVQ_REG(npl, wpr) return launch_m1_reg<npl, wpr, ISUM>(grp, K, q, d, isum, stream)
  switch (K / 1024) {
    case 2: NVQ_REG(2, 1);
    case 3: NVQ_REG(3, 1);
    case 4: NVQ_REG(4, 1);
    case 5: NVQ_REG(5, 1);
    case 6: NVQ_REG(6, 1);
    case 8: NVQ_REG(4, 2);
    case 10: NVQ_REG(5, 2);
    case 12: NVQ_REG(6, 2);
    case 15: NVQ_REG(5, 3);
    case 16: NVQ_REG(4, 4);
    case 20: NVQ_REG(5, 4);
    case 25: NVQ_REG(5, 5);
    default: return cudaErrorNotSupported;
  }
#undef NVQ_REG
}

RegMat reg_mat(const uint8_t* codes, const uint8_t* scales, float g, int64_t N, float* y) {
  RegMat m = {};
  m.codes = codes;
  m.scales = scales;
  m.y = y;
  m.half_g = 0.5f * g;
  m.N = static_cast<int>(N);
  return m;
}

template <bool ISUM>
cudaError_t launch_m1_reg_dispatch(const uint8_t* codes, const uint8_t* scales, float g,
                                   int64_t N, int64_t K, const int8_t* q, const uint16_t* d,
                                   float* y, int32_t* isum, cudaStream_t stream) {
  RegGroup grp = {};
  grp.m[0] = reg_mat(codes, scales, g, N, y);
  grp.count = 1;
  grp.rows = static_cast<int>(N);
  return launch_m1_reg_group<ISUM>(grp, K, q, d, isum, stream);
}

template <int MT, bool ISUM>
cudaError_t launch_gemv_m(const uint8_t* codes, const uint8_t* scales, float g,
                          int64_t N, int64_t K, const int8_t* q, const uint16_t* d,
                          float* y, int32_t* isum, cudaStream_t stream) {
  const int seg = tma_segment(K);
  if (MT == 1) {
    const cudaError_t e =
        launch_m1_reg_dispatch<ISUM>(codes, scales, g, N, K, q, d, y, isum, stream);
    if (e != cudaErrorNotSupported) return e;
  }
  if (MT == 1 && seg > 0 && m1_smem_bytes(static_cast<int>(K), seg) <= kSmemPerCtaMax) {
    if (seg == 5120) return launch_m1<5, ISUM>(codes, scales, g, N, K, seg, q, d, y, isum, stream);
    if (seg == 4096) return launch_m1<4, ISUM>(codes, scales, g, N, K, seg, q, d, y, isum, stream);
    return launch_m1<0, ISUM>(codes, scales, g, N, K, seg, q, d, y, isum, stream);
  }
  if (seg > 0) {
    const uint32_t smem = tma_smem_bytes(seg);
    static SmemAttrOnce attr;
    cudaError_t e = attr.ensure(gemv_tma_kernel<MT, ISUM>,
                                static_cast<int>(tma_smem_bytes(kTmaMaxSeg)));
    if (e != cudaSuccess) return e;
    const int64_t ctas = std::min<int64_t>(2 * static_cast<int64_t>(device_sm_count()), N);
    gemv_tma_kernel<MT, ISUM><<<static_cast<unsigned>(ctas), kTmaThreads, smem, stream>>>(
        codes, scales, 0.5f * g, static_cast<int>(N), static_cast<int>(K), seg, q,
        reinterpret_cast<const __half*>(d), y, isum);
    return cudaGetLastError();
  }
  const unsigned grid = static_cast<unsigned>((N + kWarps - 1) / kWarps);
  gemv_kernel<MT, ISUM><<<grid, kWarps * 32, 0, stream>>>(
      codes, scales, 0.5f * g, static_cast<int>(N), static_cast<int>(K), q,
      reinterpret_cast<const __half*>(d), y, isum);
  return cudaGetLastError();
}

template <bool ISUM>
cudaError_t launch_gemv_any(const uint8_t* codes, const uint8_t* scales, float g, int64_t N,
                            int64_t K, const int8_t* q, const uint16_t* d, int64_t M, float* y,
                            int32_t* isum, cudaStream_t stream) {
  switch (M) {
#define NVQ_GEMV_CASE(mm) \
    case mm: return launch_gemv_m<mm, ISUM>(codes, scales, g, N, K, q, d, y, isum, stream);
    NVQ_GEMV_CASE(1) NVQ_GEMV_CASE(2) NVQ_GEMV_CASE(3) NVQ_GEMV_CASE(4)
    NVQ_GEMV_CASE(5) NVQ_GEMV_CASE(6) NVQ_GEMV_CASE(7) NVQ_GEMV_CASE(8)
    NVQ_GEMV_CASE(9) NVQ_GEMV_CASE(10) NVQ_GEMV_CASE(11) NVQ_GEMV_CASE(12)
    NVQ_GEMV_CASE(13) NVQ_GEMV_CASE(14) NVQ_GEMV_CASE(15) NVQ_GEMV_CASE(16)
#undef NVQ_GEMV_CASE
    default: return cudaErrorInvalidValue;
  }
}

// ---- the persistent stack launch ----
constexpr uint32_t kStackSmem = kM1Stages * kRegStageMax + kM1Stages * kM1Consumers * 4 +
                                2 * kM1Stages * 8 + 8 + (kStackArr + 3 * kStackScnt) * 4;
static_assert(kStackSmem <= kSmemPerCtaMax, "shared memory of the stack kernel");

template <int NPL0, int NPL3, int WPR3>
cudaError_t launch_stack_t(const StackM1& s, cudaStream_t stream) {
  auto kernel = stack_m1_kernel<NPL0, NPL3, WPR3>;
  static SmemAttrOnce attr;
  cudaError_t e = attr.ensure(kernel, static_cast<int>(kStackSmem));
  if (e != cudaSuccess) return e;
  const int G = device_sm_count();
  StackArgs a = {};
  for (int i = 0; i < kStackLin; ++i) {
    a.outs[i] = s.outs[i];
    a.N[i] = static_cast<int>(s.N[i]);
  }
  a.x_q = s.x_q;
  a.x_d = reinterpret_cast<const __half*>(s.x_d);
  for (int i = 0; i < 3; ++i) {
    for (int par = 0; par < 2; ++par) {
      a.b_q[i][par] = s.b_q[i][par];
      a.b_d[i][par] = reinterpret_cast<__half*>(s.b_d[i][par]);
    }
    a.rq_cnt[i] = s.cnt[i];
  }
  a.bar = s.bar;
  a.K0 = static_cast<int>(s.K0);
  a.Kd = static_cast<int>(s.Kd);
  for (int64_t l0 = 0; l0 < s.n_layers; l0 += kStackMaxLayers) {
    const int nl = static_cast<int>(std::min<int64_t>(kStackMaxLayers, s.n_layers - l0));
    a.n_layers = nl;
    for (int l = 0; l < nl; ++l)
      for (int i = 0; i < kStackLin; ++i) {
        const StackLinear& w = s.lin[(l0 + l) * kStackLin + i];
        a.codes[l * kStackLin + i] = w.codes;
        a.scales[l * kStackLin + i] = w.scales;
        a.half_g[l * kStackLin + i] = 0.5f * w.g;
      }
    // the unit counters start at zero in every launch
    e = cudaMemsetAsync(s.bar, 0, 3 * kStackMaxLayers * sizeof(unsigned int), stream);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(G));
    cfg.blockDim = dim3(kM1Threads);
    cfg.dynamicSmemBytes = kStackSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attrs[1];
    attrs[0].id = cudaLaunchAttributeCooperative;
    attrs[0].val.cooperative = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kernel, a);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

bool stack_m1_supported(int64_t K0, int64_t Kd, const int64_t* N) {
  if (K0 != 4096 && K0 != 5120) return false;
  switch (Kd) {
    case 8192: case 10240: case 12288: case 16384: case 20480: case 25600: break;
    default: return false;
  }
  // requantised matrices (v, o, up) in whole 32-row blocks; a CTA's slice of
  // one spans at most kStackScnt - 2 blocks
  const int64_t G = device_sm_count();
  for (int i : {2, 3, 4}) {
    if (N[i] % 32 != 0) return false;
    if ((N[i] + G - 1) / G / 32 + 2 > kStackScnt) return false;
  }
  for (int i = 0; i < 7; ++i)
    if (N[i] >= (int64_t{1} << 30)) return false;
  return true;
}

cudaError_t launch_stack_m1(const StackM1& s, cudaStream_t stream) {
#define NVQ_STACK(n0, n3, w3) return launch_stack_t<n0, n3, w3>(s, stream)
  const bool k4 = s.K0 == 4096;
  switch (s.Kd) {
    case 8192: if (k4) NVQ_STACK(4, 4, 2); NVQ_STACK(5, 4, 2);
    case 10240: if (k4) NVQ_STACK(4, 5, 2); NVQ_STACK(5, 5, 2);
    case 12288: if (k4) NVQ_STACK(4, 6, 2); NVQ_STACK(5, 6, 2);
    case 16384: if (k4) NVQ_STACK(4, 4, 4); NVQ_STACK(5, 4, 4);
    case 20480: if (k4) NVQ_STACK(4, 5, 4); NVQ_STACK(5, 5, 4);
    case 25600: if (k4) NVQ_STACK(4, 5, 5); NVQ_STACK(5, 5, 5);
    default: return cudaErrorNotSupported;
  }
#undef NVQ_STACK
}

cudaError_t launch_gemv(const uint8_t* codes, const uint8_t* scales, float g,
                        int64_t N, int64_t K, const int8_t* q, const uint16_t* d,
                        int64_t M, float* y, cudaStream_t stream) {
  return launch_gemv_any<false>(codes, scales, g, N, K, q, d, M, y, nullptr, stream);
}

cudaError_t launch_gemv_isum(const uint8_t* codes, const uint8_t* scales, float g,
                             int64_t N, int64_t K, const int8_t* q, const uint16_t* d,
                             int64_t M, float* y, int32_t* isum, cudaStream_t stream) {
  return launch_gemv_any<true>(codes, scales, g, N, K, q, d, M, y, isum, stream);
}

cudaError_t launch_gemv_group(const GemvTarget* t, int n, int64_t K, const int8_t* q,
                              const uint16_t* d, cudaStream_t stream) {
  int done = 0;
  while (done < n) {
    // one launch for up to kMaxGroup matrices of the register schedule
    if (reg_supported(K)) {
      RegGroup grp = {};
      int rows = 0;
      // a requantised matrix must start on a 32-row block of the
      // concatenated rows (its blocks are counted there)
      int cnt = 0;
      while (cnt < kMaxGroup && done + cnt < n &&
             (t[done + cnt].rq_q == nullptr || rows % 32 == 0)) {
        rows += static_cast<int>(t[done + cnt].N);
        ++cnt;
      }
      rows = 0;
      for (int i = 0; i < cnt; ++i) {
        const GemvTarget& x = t[done + i];
        RegMat m = reg_mat(x.codes, x.scales, x.g, x.N, x.y);
        m.rq_q = x.rq_q;
        m.rq_d = reinterpret_cast<__half*>(x.rq_d);
        m.rq_cnt = x.rq_cnt;
        m.row_off = rows;
        rows += static_cast<int>(x.N);
        grp.m[i] = m;
      }
      grp.count = cnt;
      grp.rows = rows;
      const cudaError_t e = launch_m1_reg_group<false>(grp, K, q, d, nullptr, stream);
      if (e != cudaSuccess) return e;
      done += cnt;
      continue;
    }
    // other K: the product, then the quantiser on its output
    const GemvTarget& x = t[done];
    cudaError_t e = launch_gemv(x.codes, x.scales, x.g, x.N, K, q, d, 1, x.y, stream);
    if (e == cudaSuccess && x.rq_q != nullptr)
      e = launch_quantize_q8_0(x.y, 1, x.N, x.rq_q, x.rq_d, stream);
    if (e != cudaSuccess) return e;
    ++done;
  }
  return cudaSuccess;
}

cudaError_t launch_moe_gemv(const uint8_t* codes, const uint8_t* scales, const float* g, int64_t E,
                            int64_t N, int64_t K, const int32_t* ids, int64_t T, int64_t top_k,
                            const int8_t* q, const uint16_t* d, float* y, cudaStream_t stream) {
  if (!reg_supported(K) || top_k < 1 || top_k > kMaxGroup) return cudaErrorNotSupported;
  MoeArgs moe = {};
  moe.ids = ids;
  moe.codes = codes;
  moe.scales = scales;
  moe.g = g;
  moe.y = y;
  moe.E = static_cast<int>(E);
  moe.N = static_cast<int>(N);
  moe.top_k = static_cast<int>(top_k);
#define NVQ_MOE(npl, wpr) return launch_moe_reg<npl, wpr>(moe, T, K, q, d, stream)
  switch (K / 1024) {
    case 2: NVQ_MOE(2, 1);
    case 3: NVQ_MOE(3, 1);
    case 4: NVQ_MOE(4, 1);
    case 5: NVQ_MOE(5, 1);
    case 6: NVQ_MOE(6, 1);
    case 8: NVQ_MOE(4, 2);
    case 10: NVQ_MOE(5, 2);
    case 12: NVQ_MOE(6, 2);
    case 15: NVQ_MOE(5, 3);
    case 16: NVQ_MOE(4, 4);
    case 20: NVQ_MOE(5, 4);
    case 25: NVQ_MOE(5, 5);
    default: return cudaErrorNotSupported;
  }
#undef NVQ_MOE
}

bool moe_supported(int64_t K, int64_t top_k) {
  return reg_supported(K) && top_k >= 1 && top_k <= kMaxGroup;
}

cudaError_t launch_stalled_wait(uint64_t limit_ns, int* result, cudaStream_t stream) {
  stalled_wait_kernel<<<1, 32, 0, stream>>>(limit_ns, result);
  return cudaGetLastError();
}

cudaError_t gemv_error_flags(bool clear, unsigned int* flags) {
  cudaError_t e = cudaMemcpyFromSymbol(flags, g_gemv_error_flags, sizeof(unsigned int));
  if (e == cudaSuccess && clear) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_gemv_error_flags, &zero, sizeof(zero));
  }
  return e;
}

}  // namespace nvq
