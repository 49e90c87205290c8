// nvq_decoder_stack: the linear layers of a dense decoder stack enqueued
// from native code (7 products and 4 Q8_0 quantisations per layer), so a
// 64-layer token pass issues its 700-odd launches without crossing back
// into Python.  The dataflow of a layer is documented in include/nvq.h.
#include <algorithm>
#include <cstdint>

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

struct Layout {
  size_t q_off, d_off, gemm_off, total;
};

Layout workspace_layout(const nvq_linear* L, int64_t M) {
  const int64_t km = max_k(L);
  Layout w;
  w.q_off = 0;
  w.d_off = round256(static_cast<size_t>(M * km));
  w.gemm_off = w.d_off + round256(static_cast<size_t>(M * (km / 32) * 2));
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
  int8_t* qa = reinterpret_cast<int8_t*>(ws + lay.q_off);
  uint16_t* da = reinterpret_cast<uint16_t*>(ws + lay.d_off);
  void* gws = ws + lay.gemm_off;
  const bool decode = M <= 16;

  cudaError_t err = cudaSuccess;
  auto quantize = [&](const float* in, int64_t K) {
    if (err != cudaSuccess) return;
    err = nvq::launch_quantize_q8_0(in, M, K, qa, da, st);
    if (err == cudaSuccess && !decode) err = nvq::gemm_expand(qa, da, M, K, gws, st);
  };
  auto dot = [&](const nvq_linear& W, float* y) {
    if (err != cudaSuccess) return;
    if (decode)
      err = nvq::launch_gemv(W.codes, W.scales, W.g, W.N, W.K, qa, da, M, y, st);
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
  if (err != cudaSuccess) {
    nvq::set_last_cuda_error(err);
    return NVQ_ERR_CUDA;
  }
  return NVQ_OK;
}
