// Host-side NVFP4 packer (nvq_pack_nvfp4): fp32 weights -> E2M1 codes, UE4M3
// per-16 scales and the per-tensor fp32 scale g.
//
// Recipe (fp32, one IEEE rounding per operation, evaluated left to right):
//   g  = amax(|w|) / (6*448)                       (6*448 = 2688 exactly)
//   s  = UE4M3(amax_blk / (6*g))                   per 16-element subblock
//   c  = E2M1(w / (g*s))                           per element
// UE4M3 and E2M1 round to nearest with ties to the even code and saturate at
// their largest finite value (448 and 6); a zero E2M1 magnitude is stored
// as +0, and a subblock whose 6*g or g*s is 0 stores codes 0.
//
// Both formats space their values uniformly inside each binade and number
// them in increasing order, so rounding reduces to rint() of the value
// divided by the local spacing (an exact power-of-two scaling); rint rounds
// half to even, and the parity of that integer is the parity of the code.
// This file must be compiled without floating-point contraction
// (-ffp-contract=off) so that no multiply and add fuse.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

#include "nvq.h"

namespace {

// UE4M3 byte nearest to r >= 0 (finite).  Bytes 0..7 are m * 2^-9 and byte
// 8e + m (e >= 1) is 2^(e-7) * (1 + m/8) = (8 + m) * 2^(e-10), so within
// exponent e the code is (e-1)*8 + rint(r * 2^(10-e)); bytes 0..15 share the
// spacing 2^-9.  Saturates at 0x7E (448).
uint8_t ue4m3_encode(float r) {
  if (!(r > 0.0f)) return 0;
  if (r >= 448.0f) return 0x7E;
  int ex = 0;
  std::frexp(r, &ex);                 // r = f * 2^ex, f in [0.5, 1)
  int e = ex + 6;                     // UE4M3 exponent field of r's binade
  if (e < 1) e = 1;                   // subnormal range shares e = 1 spacing
  const float scaled = std::ldexp(r, 10 - e);   // exact
  const int n = static_cast<int>(std::nearbyint(scaled));
  int code = (e - 1) * 8 + n;
  if (code > 0x7E) code = 0x7E;
  return static_cast<uint8_t>(code);
}

float ue4m3_value(uint8_t b) {
  const int e = (b >> 3) & 0xF;
  const int m = b & 0x7;
  if (e == 0) return std::ldexp(static_cast<float>(m), -9);
  return std::ldexp(static_cast<float>(8 + m), e - 10);
}

// E2M1 code nearest to x: magnitudes 0, .5, 1, 1.5 | 2, 3 | 4, 6 have
// spacings 0.5, 1 and 2 in [0, 2), [2, 4) and [4, 6]; the codes are
// rint(2|x|), rint(|x|) + 2 and rint(|x|/2) + 4 there.
uint8_t e2m1_encode(float x) {
  const float a = std::fabs(x);
  int code;
  if (a >= 6.0f) {
    code = 7;
  } else if (a < 2.0f) {
    code = static_cast<int>(std::nearbyint(a * 2.0f));
  } else if (a < 4.0f) {
    code = static_cast<int>(std::nearbyint(a)) + 2;
  } else {
    code = static_cast<int>(std::nearbyint(a * 0.5f)) + 4;
  }
  if (code != 0 && x < 0.0f) code |= 0x8;
  return static_cast<uint8_t>(code);
}

template <class F>
void parallel_rows(int64_t N, F&& fn) {
  unsigned hw = std::thread::hardware_concurrency();
  int64_t nthreads = std::max<int64_t>(1, std::min<int64_t>(hw ? hw : 1, 64));
  nthreads = std::min<int64_t>(nthreads, std::max<int64_t>(1, N / 64));
  if (nthreads <= 1) {
    fn(int64_t{0}, N, 0);
    return;
  }
  std::vector<std::thread> pool;
  const int64_t per = (N + nthreads - 1) / nthreads;
  for (int64_t t = 0; t < nthreads; ++t) {
    const int64_t r0 = t * per, r1 = std::min(N, r0 + per);
    if (r0 >= r1) break;
    pool.emplace_back([&fn, r0, r1, t] { fn(r0, r1, t); });
  }
  for (auto& th : pool) th.join();
}

}  // namespace

extern "C" nvq_status nvq_pack_nvfp4(const float* w, int64_t N, int64_t K,
                                     uint8_t* codes, uint8_t* scales, float* g_out) {
  if (N < 0 || K < 0) return NVQ_ERR_INVALID_ARG;
  if (K % 16 != 0) return NVQ_ERR_BAD_SHAPE;
  if (!g_out) return NVQ_ERR_INVALID_ARG;
  if (N == 0 || K == 0) {
    *g_out = 0.0f;
    return NVQ_OK;
  }
  if (!w || !codes || !scales) return NVQ_ERR_INVALID_ARG;

  // tensor amax (and a finiteness check), one partial per thread
  std::vector<float> part(64, 0.0f);
  std::vector<int> bad(64, 0);
  parallel_rows(N, [&](int64_t r0, int64_t r1, int64_t t) {
    float a = 0.0f;
    int b = 0;
    for (int64_t i = r0 * K; i < r1 * K; ++i) {
      const float v = w[i];
      if (!std::isfinite(v)) b = 1;
      a = std::max(a, std::fabs(v));
    }
    part[t] = a;
    bad[t] = b;
  });
  float amax = 0.0f;
  for (int t = 0; t < 64; ++t) {
    if (bad[t]) return NVQ_ERR_INVALID_ARG;
    amax = std::max(amax, part[t]);
  }
  const float g = amax / 2688.0f;
  const float six_g = 6.0f * g;

  parallel_rows(N, [&](int64_t r0, int64_t r1, int64_t) {
    for (int64_t n = r0; n < r1; ++n) {
      const float* wr = w + n * K;
      uint8_t* cr = codes + n * (K / 2);
      uint8_t* sr = scales + n * (K / 16);
      for (int64_t b = 0; b < K / 16; ++b) {
        const float* blk = wr + b * 16;
        float amax_blk = 0.0f;
        for (int j = 0; j < 16; ++j) amax_blk = std::max(amax_blk, std::fabs(blk[j]));
        const float r = six_g > 0.0f ? amax_blk / six_g : 0.0f;
        const uint8_t s_code = ue4m3_encode(r);
        const float gs = g * ue4m3_value(s_code);
        sr[b] = s_code;
        for (int j = 0; j < 16; j += 2) {
          const uint8_t c0 = gs > 0.0f ? e2m1_encode(blk[j] / gs) : 0;
          const uint8_t c1 = gs > 0.0f ? e2m1_encode(blk[j + 1] / gs) : 0;
          cr[b * 8 + j / 2] = static_cast<uint8_t>(c0 | (c1 << 4));
        }
      }
    }
  });
  *g_out = g;
  return NVQ_OK;
}
