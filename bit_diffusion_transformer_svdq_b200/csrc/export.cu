// Canonical-layout host copies of prepared weights and of activation
// scales (declared in include/svdq.h): the inverse of the tiled layouts the
// kernels read, for inspection and parity checks.  Host code only: the
// device buffers are copied to host memory with cudaMemcpyAsync on the
// caller's stream, synchronised, then rearranged on the CPU.
#include <cuda_runtime.h>

#include <cstdlib>
#include <cstring>
#include <vector>

#include "internal.h"

namespace svdq {
namespace {

// Byte offset of (row m, 16-group j) in the tiled NVFP4 scale layout of
// include/svdq.h (K/64 atoms of 128 rows x 4 groups per 128-row block).
inline size_t tiled_scale_offset(int64_t m, int64_t j, int K) {
  return static_cast<size_t>(((m / 128) * (K / 64) + j / 4) * 512 + (m % 32) * 16 + ((m / 32) % 4) * 4 + j % 4);
}

svdq_status d2h(void* dst, const void* src, size_t bytes, cudaStream_t s) {
  if (bytes == 0) return SVDQ_OK;
  return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToHost, s) == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

svdq_status sync(cudaStream_t s) { return cudaStreamSynchronize(s) == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA; }

}  // namespace
}  // namespace svdq

using namespace svdq;

extern "C" {

svdq_status svdq_export_weights(const svdq_weights* w, svdq_weights_export* out, void* stream) {
  if (!w || !out) return SVDQ_ERR_INVALID_ARG;
  const int K = w->desc.K, N = w->desc.N, r = w->desc.rank, rp = w->rank_pad;
  const bool nvfp4 = w->desc.precision == SVDQ_NVFP4;
  const bool awq = w->desc.precision == SVDQ_AWQ_W4A16;
  const int64_t np = w->n_pad;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  svdq_status st = SVDQ_OK;

  if (out->qw) {
    if (!awq) {
      st = d2h(out->qw, w->qw, static_cast<size_t>(N) * K / 2, s);
      if (st == SVDQ_OK) st = sync(s);
    } else {
      // GEMV tiles: the 16 bytes of codes 32c .. 32c+31 of row n at
      // ((n / 32) * (K / 32) + c) * 512 + (n % 32) * 16
      std::vector<uint8_t> t(static_cast<size_t>(np) * K / 2);
      st = d2h(t.data(), w->qw, t.size(), s);
      if (st == SVDQ_OK) st = sync(s);
      if (st == SVDQ_OK)
        for (int64_t n = 0; n < N; ++n)
          for (int c = 0; c < K / 32; ++c)
            std::memcpy(out->qw + n * (K / 2) + c * 16, t.data() + ((n / 32) * (K / 32) + c) * 512 + (n % 32) * 16,
                        16);
    }
    if (st != SVDQ_OK) return st;
  }
  if (out->sw) {
    std::vector<uint8_t> t(w->sw_bytes);
    st = d2h(t.data(), w->sw, t.size(), s);
    if (st == SVDQ_OK) st = sync(s);
    if (st != SVDQ_OK) return st;
    if (nvfp4) {
      uint8_t* dst = static_cast<uint8_t*>(out->sw);
      for (int64_t n = 0; n < N; ++n)
        for (int j = 0; j < K / 16; ++j) dst[n * (K / 16) + j] = t[tiled_scale_offset(n, j, K)];
    } else {  // fp16, group-major [K/64][n_pad] -> row-major N x K/64
      const uint16_t* src = reinterpret_cast<const uint16_t*>(t.data());
      uint16_t* dst = static_cast<uint16_t*>(out->sw);
      for (int64_t n = 0; n < N; ++n)
        for (int g = 0; g < K / 64; ++g) dst[n * (K / 64) + g] = src[static_cast<size_t>(g) * np + n];
    }
  }
  if (out->l1s && r > 0) {
    st = d2h(out->l1s, w->l1s, static_cast<size_t>(r) * K * 2, s);  // rows are K apart; padding rows follow
    if (st == SVDQ_OK) st = sync(s);
    if (st != SVDQ_OK) return st;
  }
  if (out->l2 && r > 0) {
    std::vector<float> t(static_cast<size_t>(N) * rp);
    st = d2h(t.data(), w->l2, t.size() * 4, s);
    if (st == SVDQ_OK) st = sync(s);
    if (st != SVDQ_OK) return st;
    for (int64_t n = 0; n < N; ++n) std::memcpy(out->l2 + n * r, t.data() + n * rp, static_cast<size_t>(r) * 4);
  }
  if (out->inv_lambda) {
    st = d2h(out->inv_lambda, w->inv_lambda, static_cast<size_t>(K) * 4, s);
    if (st != SVDQ_OK) return st;
  }
  if (out->bias) {
    st = d2h(out->bias, w->bias, static_cast<size_t>(N) * 4, s);
    if (st != SVDQ_OK) return st;
  }
  if ((st = sync(s)) != SVDQ_OK) return st;
  if (out->g_w) *out->g_w = w->g_w;
  return SVDQ_OK;
}

svdq_status svdq_export_act_scales(const svdq_weights* w, const void* sx, int32_t M, void* out, void* stream) {
  if (!w || w->desc.precision == SVDQ_AWQ_W4A16) return SVDQ_ERR_INVALID_ARG;
  if (M < 0) return SVDQ_ERR_SHAPE;
  if (M == 0) return SVDQ_OK;
  if (!sx || !out) return SVDQ_ERR_INVALID_ARG;
  const int K = w->desc.K;
  const int64_t mp = m_pad_of(M);
  const bool nvfp4 = w->desc.precision == SVDQ_NVFP4;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::vector<uint8_t> t(svdq_act_scale_bytes(w, M));
  svdq_status st = d2h(t.data(), sx, t.size(), s);
  if (st == SVDQ_OK) st = sync(s);
  if (st != SVDQ_OK) return st;
  if (nvfp4) {
    uint8_t* dst = static_cast<uint8_t*>(out);
    for (int64_t m = 0; m < M; ++m)
      for (int j = 0; j < K / 16; ++j) dst[m * (K / 16) + j] = t[tiled_scale_offset(m, j, K)];
  } else {
    const uint16_t* src = reinterpret_cast<const uint16_t*>(t.data());
    uint16_t* dst = static_cast<uint16_t*>(out);
    for (int64_t m = 0; m < M; ++m)
      for (int g = 0; g < K / 64; ++g) dst[m * (K / 64) + g] = src[static_cast<size_t>(g) * mp + m];
  }
  return SVDQ_OK;
}

}  // extern "C"
