// Device helpers for the NVFP4 x Q8_0 kernels (sm_100a).
#pragma once

#include <cstdint>

#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace nvq {
namespace dev {

// Integer LUT c = 2*E2M1(code), as packed signed bytes.  E2M1 (OCP MX):
// codes 0..7 are 0, .5, 1, 1.5, 2, 3, 4, 6 and bit 3 is the sign, so c runs
// over 0, 1, 2, 3, 4, 6, 8, 12 and their negatives ("HANDOFF: flint CPU
// optimization (Q4_1 + NVFP4)", section 3, "Bias trick": the integer codes
// lie in -12..12).  Byte j of the pair (lo, hi) is the value of index j.
constexpr uint32_t kLutPosLo = 0x03020100u;  // codes 0..3   ->  0,  1,  2,  3
constexpr uint32_t kLutPosHi = 0x0C080604u;  // codes 4..7   ->  4,  6,  8, 12
constexpr uint32_t kLutNegLo = 0xFDFEFF00u;  // codes 8..11  ->  0, -1, -2, -3
constexpr uint32_t kLutNegHi = 0xF4F8FAFCu;  // codes 12..15 -> -4, -6, -8,-12

// Look up the eight 4-bit codes of one 32-bit word (nibble i = element i)
// in a 16-entry byte table given as four packed words (entries 0-3, 4-7,
// 8-11, 12-15).  `lo` receives the bytes of elements 0..3, `hi` those of
// elements 4..7.  Each byte is looked up twice with a byte permute (in the
// table half of codes 0-7 and of codes 8-15, indexed by the code's low three
// bits) and bit 3 of the code picks between the two.
template <uint32_t T0, uint32_t T1, uint32_t T2, uint32_t T3>
__device__ __forceinline__ void lut16_x8(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t idx = w & 0x77777777u;
  // selector of the final permute: byte i from p (i) or from n (4 + i)
  const uint32_t pick = ((w >> 1) & 0x44444444u) | 0x32103210u;
  const uint32_t idx_hi = idx >> 16;
  const uint32_t pick_hi = pick >> 16;
  const uint32_t p0 = __byte_perm(T0, T1, idx);
  const uint32_t n0 = __byte_perm(T2, T3, idx);
  const uint32_t p1 = __byte_perm(T0, T1, idx_hi);
  const uint32_t n1 = __byte_perm(T2, T3, idx_hi);
  lo = __byte_perm(p0, n0, pick);
  hi = __byte_perm(p1, n1, pick_hi);
}

// Decode eight E2M1 codes to signed bytes c = 2*E2M1.
__device__ __forceinline__ void decode_e2m1x8(uint32_t w, uint32_t& lo, uint32_t& hi) {
  lut16_x8<kLutPosLo, kLutPosHi, kLutNegLo, kLutNegHi>(w, lo, hi);
}

// The same integer LUT biased by +12 (0..24, unsigned bytes), the storage
// form of the "Bias trick" paragraph of "HANDOFF: flint CPU optimization
// (Q4_1 + NVFP4)", section 3: c + 12 for codes 0..7 and for codes 8..15.
constexpr uint32_t kBiasPosLo = 0x0F0E0D0Cu;  // codes 0..3   -> 12, 13, 14, 15
constexpr uint32_t kBiasPosHi = 0x18141210u;  // codes 4..7   -> 16, 18, 20, 24
constexpr uint32_t kBiasNegLo = 0x090A0B0Cu;  // codes 8..11  -> 12, 11, 10,  9
constexpr uint32_t kBiasNegHi = 0x00040608u;  // codes 12..15 ->  8,  6,  4,  0

// Byte permute with the sign-replicating selector mode: a selector nibble
// with bit 3 set yields the sign (bit 7) of the selected byte, replicated.
__device__ __forceinline__ uint32_t prmt_sr(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// Decode eight E2M1 codes to the biased bytes c + 12.  Every table byte is
// below 0x80, so a lookup whose selector has bit 3 set gives 0: the lookup
// in the positive half with the raw codes fills the bytes of codes 0..7 and
// zeroes the others, the lookup in the negative half with bit 3 flipped
// does the converse, and an OR merges them (9 operations per 8 codes).
__device__ __forceinline__ void decode_e2m1x8_biased(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t wn = w ^ 0x88888888u;
  lo = prmt_sr(kBiasPosLo, kBiasPosHi, w) | prmt_sr(kBiasNegLo, kBiasNegHi, wn);
  hi = prmt_sr(kBiasPosLo, kBiasPosHi, w >> 16) | prmt_sr(kBiasNegLo, kBiasNegHi, wn >> 16);
}

// dp4a with unsigned bytes in a and signed bytes in b.
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int r;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

// Integer sum of one 16-element subblock, sum((c + 12) * q) + corr, from its
// two code words and four activation words.  The two lookups of each group
// of four codes (positive and negative table half, each zero where the
// other applies) go to dp4a separately instead of being OR-merged: this
// moves work from the integer ALU pipe, which limits the decode GEMV, to the
// dp4a pipe (measured +6 % on the decode sweep, +8 % on the largest shape).
__device__ __forceinline__ int dot16_biased(uint32_t w0, uint32_t w1, const uint4 q, int corr) {
  const uint32_t n0 = w0 ^ 0x88888888u, n1 = w1 ^ 0x88888888u;
  int a = corr;
  a = dp4a_us(prmt_sr(kBiasPosLo, kBiasPosHi, w0), q.x, a);
  a = dp4a_us(prmt_sr(kBiasNegLo, kBiasNegHi, n0), q.x, a);
  a = dp4a_us(prmt_sr(kBiasPosLo, kBiasPosHi, w0 >> 16), q.y, a);
  a = dp4a_us(prmt_sr(kBiasNegLo, kBiasNegHi, n0 >> 16), q.y, a);
  a = dp4a_us(prmt_sr(kBiasPosLo, kBiasPosHi, w1), q.z, a);
  a = dp4a_us(prmt_sr(kBiasNegLo, kBiasNegHi, n1), q.z, a);
  a = dp4a_us(prmt_sr(kBiasPosLo, kBiasPosHi, w1 >> 16), q.w, a);
  a = dp4a_us(prmt_sr(kBiasNegLo, kBiasNegHi, n1 >> 16), q.w, a);
  return a;
}

// Two UE4M3 scale bytes (low byte = first subblock) to fp32, exactly.  UE4M3
// is E4M3 with the sign bit 0, so the hardware E4M3 -> f16 conversion
// applies; every UE4M3 value (2^-9 .. 448) is exact in fp16.
__device__ __forceinline__ float2 ue4m3x2_to_float2(uint32_t two_bytes) {
  uint32_t h2;
  const uint16_t in = static_cast<uint16_t>(two_bytes);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  __half2 h = *reinterpret_cast<__half2*>(&h2);
  return __half22float2(h);
}

__device__ __forceinline__ int dp4a(uint32_t a, uint32_t b, int c) {
  return __dp4a(static_cast<int>(a), static_cast<int>(b), c);
}

// 128-bit streaming load: read-only path, no L1 allocation (each weight
// byte is used once), 256-byte L2 prefetch.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile(
      "ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}

// ---- fp16 operand expansion (tensor-core paths) ------------------------------
__device__ __forceinline__ uint32_t h2_bits(__half2 h) {
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ __half2 bits_h2(uint32_t u) {
  return *reinterpret_cast<__half2*>(&u);
}

// Eight codes (one word, element i in nibble i) -> eight fp16
// w' = E2M1 * s as four half2 words (element 2i in the low half of word i).
// The hardware E2M1 -> f16x2 conversion takes one byte (two codes, the low
// nibble to the low half) and is exact: every E2M1 value is an fp16 value
// (code 8 gives -0, as a signed zero should).  E2M1 * s has at most 6
// significant bits and lies in 2^-10 .. 2688, so the fp16 product is exact.
__device__ __forceinline__ uint4 expand8(uint32_t w, __half2 s2) {
  uint32_t e0, e1, e2, e3;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(e0), "=r"(e1), "=r"(e2), "=r"(e3)
      : "r"(w));
  uint4 r;
  r.x = h2_bits(__hmul2(bits_h2(e0), s2));
  r.y = h2_bits(__hmul2(bits_h2(e1), s2));
  r.z = h2_bits(__hmul2(bits_h2(e2), s2));
  r.w = h2_bits(__hmul2(bits_h2(e3), s2));
  return r;
}

// Two UE4M3 scale bytes (low byte = first subblock) to an exact half2.
__device__ __forceinline__ __half2 ue4m3x2_to_half2(uint32_t two_bytes) {
  uint32_t h2;
  const uint16_t in = static_cast<uint16_t>(two_bytes);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  return bits_h2(h2);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace dev
}  // namespace nvq
