// nvq_decoder_stack: the linear layers of a dense decoder stack enqueued
// from native code (7 products and 4 Q8_0 quantisations per layer), so a
// 64-layer token pass issues its launches without crossing back into
// Python.  The dataflow of a layer is documented in include/nvq.h.
//
// One token (M = 1), for the common shapes (hidden 4096 or 5120, v and o
// as wide as the hidden size): Q8_0(x) once (every layer reads the same x),
// then one persistent launch per 64 layers that runs all their products,
// layer after layer pipelined, with the requantisations of y_v, y_o and
// y_up fused into the products (launch_stack_m1).  Other one-token shapes take five launches per
// layer: the quantiser of x; one GEMV over q, k and v together (they read
// the same activations) that also emits Q8_0(y_v); the o GEMV that emits
// Q8_0(y_o); one GEMV over up and gate that emits Q8_0(y_up); the down GEMV.
// Other token counts run the quantiser and the products separately (GEMV for
// M <= 16, the tensor-core GEMM above, whose fp16 expansion of the
// activations is shared by the products that read it).
#include <algorithm>
#include <cstdint>
#include <vector>

#include <cuda_runtime.h>

#include "nvq.h"
#include "nvq_internal.h"

namespace {

constexpr int kQ = 0, kK = 1, kV = 2, kO = 3, kUp = 4, kGate = 5, kDown = 6;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round256(size_t v) { return (v + 255) / 256 * 256; }

int64_t max_k(const nvq_linear* L) {
  int64_t k = 0;
  for (int i = 0; i < NVQ_STACK_LINEARS; ++i) k = std::max(k, L[i].K);
  return k;
}

// Shapes of layer 0 chain, and every matrix is well formed.
bool layer_shapes_ok(const nvq_linear* L) {
  for (int i = 0; i < NVQ_STACK_LINEARS; ++i) {
    if (L[i].N < 1 || L[i].K < 64 || L[i].K % 64 != 0) return false;
    if (L[i].K > (int64_t{1} << 30) || L[i].N > (int64_t{1} << 30)) return false;
  }
  return L[kK].K == L[kQ].K && L[kV].K == L[kQ].K && L[kO].K == L[kV].N &&
         L[kUp].K == L[kO].N && L[kGate].K == L[kO].N && L[kDown].K == L[kUp].N;
}

// Workspace: Q8_0 activation buffers (codes, scales; two, or seven for one
// token: x and two each for y_v, y_o, y_up), the requantisation block
// counters of v, o and up and the unit counters of the persistent launch
// (one token), and the GEMM's expansion.
constexpr int kBuffers = 7;
constexpr size_t kBarBytes = 3 * 64 * sizeof(unsigned int);

struct Layout {
  size_t q_off[kBuffers], d_off[kBuffers], cnt_off, cnt_bytes, bar_off, gemm_off, total;
};

Layout workspace_layout(const nvq_linear* L, int64_t M) {
  const int64_t km = max_k(L);
  const size_t qb = round256(static_cast<size_t>(M * km));
  const size_t db = round256(static_cast<size_t>(M * (km / 32) * 2));
  const int nb = M == 1 ? kBuffers : 2;
  Layout w = {};
  for (int i = 0; i < nb; ++i) {
    w.q_off[i] = i * (qb + db);
    w.d_off[i] = i * (qb + db) + qb;
  }
  w.cnt_off = nb * (qb + db);
  w.cnt_bytes = M == 1 ? round256(static_cast<size_t>((L[kV].N + L[kO].N + L[kUp].N) / 32) * 4) : 0;
  w.bar_off = w.cnt_off + w.cnt_bytes;
  w.gemm_off = w.bar_off + (M == 1 ? round256(kBarBytes) : 0);
  w.total = w.gemm_off + (M > 16 ? nvq::gemm_workspace_size(M, 0, km) : 0);
  return w;
}

}  // namespace

extern "C" size_t nvq_decoder_stack_workspace_size(const nvq_linear* linears, int64_t M) {
  if (!linears || M < 1 || !layer_shapes_ok(linears)) return 0;
  return workspace_layout(linears, M).total;
}

extern "C" nvq_status nvq_decoder_stack(const nvq_linear* linears, int64_t n_layers,
                                        const float* x, int64_t M, float* const* outs,
                                        void* workspace, size_t workspace_bytes,
                                        void* stream) {
  if (n_layers < 0 || M < 0) return NVQ_ERR_INVALID_ARG;
  if (n_layers == 0 || M == 0) return NVQ_OK;
  if (!linears || !x || !outs) return NVQ_ERR_INVALID_ARG;
  if (M > (int64_t{1} << 24)) return NVQ_ERR_BAD_SHAPE;
  const nvq_linear* L0 = linears;
  if (!layer_shapes_ok(L0)) return NVQ_ERR_BAD_SHAPE;
  for (int64_t l = 0; l < n_layers; ++l) {
    const nvq_linear* L = linears + NVQ_STACK_LINEARS * l;
    for (int i = 0; i < NVQ_STACK_LINEARS; ++i) {
      if (L[i].N != L0[i].N || L[i].K != L0[i].K) return NVQ_ERR_BAD_SHAPE;
      if (!L[i].codes || !L[i].scales || !(L[i].g == L[i].g)) return NVQ_ERR_INVALID_ARG;
      if (!aligned16(L[i].codes) || !aligned16(L[i].scales)) return NVQ_ERR_MISALIGNED;
    }
  }
  for (int i = 0; i < NVQ_STACK_LINEARS; ++i) {
    if (!outs[i]) return NVQ_ERR_INVALID_ARG;
    if (!aligned16(outs[i])) return NVQ_ERR_MISALIGNED;
  }
  if (!aligned16(x)) return NVQ_ERR_MISALIGNED;
  const Layout lay = workspace_layout(L0, M);
  if (!workspace || workspace_bytes < lay.total) return NVQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return NVQ_ERR_MISALIGNED;
  {
    int dev = 0, major = 0, minor = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) {
      cudaGetLastError();
      nvq::set_last_cuda_error(e);
      return NVQ_ERR_CUDA;
    }
    if (major != 10 || minor != 0) return NVQ_ERR_UNSUPPORTED_DEVICE;
  }

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int8_t* qa[kBuffers];
  uint16_t* da[kBuffers];
  for (int i = 0; i < kBuffers; ++i) {
    qa[i] = reinterpret_cast<int8_t*>(ws + lay.q_off[i]);
    da[i] = reinterpret_cast<uint16_t*>(ws + lay.d_off[i]);
  }
  void* gws = ws + lay.gemm_off;
  cudaError_t err = cudaSuccess;

  int64_t Ns[NVQ_STACK_LINEARS];
  for (int i = 0; i < NVQ_STACK_LINEARS; ++i) Ns[i] = L0[i].N;
  const bool persistent = M == 1 && L0[kV].N == L0[kQ].K && L0[kO].N == L0[kQ].K &&
                          nvq::stack_m1_supported(L0[kQ].K, L0[kDown].K, Ns);
  if (persistent) {
    int* cnt = reinterpret_cast<int*>(ws + lay.cnt_off);
    err = cudaMemsetAsync(cnt, 0, lay.cnt_bytes, st);
    if (err == cudaSuccess) err = nvq::launch_quantize_q8_0(x, 1, L0[kQ].K, qa[0], da[0], st);
    if (err == cudaSuccess) {
      std::vector<nvq::StackLinear> lin(static_cast<size_t>(n_layers) * NVQ_STACK_LINEARS);
      for (size_t i = 0; i < lin.size(); ++i)
        lin[i] = {linears[i].codes, linears[i].scales, linears[i].g};
      nvq::StackM1 sm = {};
      sm.lin = lin.data();
      sm.n_layers = n_layers;
      for (int i = 0; i < NVQ_STACK_LINEARS; ++i) {
        sm.N[i] = Ns[i];
        sm.outs[i] = outs[i];
      }
      sm.K0 = L0[kQ].K;
      sm.Kd = L0[kDown].K;
      sm.x_q = qa[0];
      sm.x_d = da[0];
      for (int i = 0; i < 3; ++i)
        for (int par = 0; par < 2; ++par) {
          sm.b_q[i][par] = qa[1 + 2 * i + par];
          sm.b_d[i][par] = da[1 + 2 * i + par];
        }
      sm.cnt[0] = cnt;
      sm.cnt[1] = cnt + L0[kV].N / 32;
      sm.cnt[2] = sm.cnt[1] + L0[kO].N / 32;
      sm.bar = reinterpret_cast<unsigned int*>(ws + lay.bar_off);
      err = nvq::launch_stack_m1(sm, st);
    }
  } else if (M == 1) {
    // block counters start at zero; every launch leaves them at zero
    int* cnt = reinterpret_cast<int*>(ws + lay.cnt_off);
    int* cnt_v = cnt;
    int* cnt_o = cnt_v + L0[kV].N / 32;
    int* cnt_up = cnt_o + L0[kO].N / 32;
    err = cudaMemsetAsync(cnt, 0, lay.cnt_bytes, st);
    auto target = [&](const nvq_linear& W, float* y, int b, int* c) {
      nvq::GemvTarget t = {W.codes, W.scales, W.g, W.N, y, nullptr, nullptr, nullptr};
      if (b >= 0) {
        t.rq_q = qa[b];
        t.rq_d = da[b];
        t.rq_cnt = c;
      }
      return t;
    };
    for (int64_t l = 0; l < n_layers && err == cudaSuccess; ++l) {
      const nvq_linear* L = linears + NVQ_STACK_LINEARS * l;
      err = nvq::launch_quantize_q8_0(x, 1, L[kQ].K, qa[0], da[0], st);
      if (err != cudaSuccess) break;
      const nvq::GemvTarget qkv[3] = {target(L[kQ], outs[kQ], -1, nullptr),
                                      target(L[kK], outs[kK], -1, nullptr),
                                      target(L[kV], outs[kV], 1, cnt_v)};
      err = nvq::launch_gemv_group(qkv, 3, L[kQ].K, qa[0], da[0], st);
      if (err != cudaSuccess) break;
      const nvq::GemvTarget o = target(L[kO], outs[kO], 0, cnt_o);
      err = nvq::launch_gemv_group(&o, 1, L[kO].K, qa[1], da[1], st);
      if (err != cudaSuccess) break;
      const nvq::GemvTarget ug[2] = {target(L[kUp], outs[kUp], 1, cnt_up),
                                     target(L[kGate], outs[kGate], -1, nullptr)};
      err = nvq::launch_gemv_group(ug, 2, L[kUp].K, qa[0], da[0], st);
      if (err != cudaSuccess) break;
      const nvq::GemvTarget dn = target(L[kDown], outs[kDown], -1, nullptr);
      err = nvq::launch_gemv_group(&dn, 1, L[kDown].K, qa[1], da[1], st);
    }
  } else {
    const bool decode = M <= 16;
    auto quantize = [&](const float* in, int64_t K) {
      if (err != cudaSuccess) return;
      err = nvq::launch_quantize_q8_0(in, M, K, qa[0], da[0], st);
      if (err == cudaSuccess && !decode) err = nvq::gemm_expand(qa[0], da[0], M, K, gws, st);
    };
    auto dot = [&](const nvq_linear& W, float* y) {
      if (err != cudaSuccess) return;
      if (decode)
        err = nvq::launch_gemv(W.codes, W.scales, W.g, W.N, W.K, qa[0], da[0], M, y, st);
      else
        err = nvq::gemm_main(W.codes, W.scales, W.g, W.N, W.K, M, y, gws, st);
    };
    for (int64_t l = 0; l < n_layers && err == cudaSuccess; ++l) {
      const nvq_linear* L = linears + NVQ_STACK_LINEARS * l;
      quantize(x, L[kQ].K);
      dot(L[kQ], outs[kQ]);
      dot(L[kK], outs[kK]);
      dot(L[kV], outs[kV]);
      quantize(outs[kV], L[kO].K);
      dot(L[kO], outs[kO]);
      quantize(outs[kO], L[kUp].K);
      dot(L[kUp], outs[kUp]);
      dot(L[kGate], outs[kGate]);
      quantize(outs[kUp], L[kDown].K);
      dot(L[kDown], outs[kDown]);
    }
  }
  if (err != cudaSuccess) {
    nvq::set_last_cuda_error(err);
    return NVQ_ERR_CUDA;
  }
  return NVQ_OK;
}
