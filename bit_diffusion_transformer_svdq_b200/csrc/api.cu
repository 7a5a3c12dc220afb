// The C ABI of libsvdq (declared in include/svdq.h): argument checks,
// weight-storage layout, tensor-map encoding and kernel dispatch.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdlib>
#include <cstring>
#include <mutex>

#include "internal.h"

namespace svdq {

namespace {

constexpr int kMaxDevices = 64;
int g_sms[kMaxDevices] = {0};
int g_cc_ok[kMaxDevices] = {0};  // 0 unknown, 1 ok, -1 unsupported
std::mutex g_mu;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

svdq_status current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess) return SVDQ_ERR_CUDA;
  const svdq_status st = svdq_check_device(*dev);
  return st;
}

svdq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA; }

svdq_status check_desc(const svdq_layer_desc* d) {
  if (!d) return SVDQ_ERR_INVALID_ARG;
  if (d->precision == SVDQ_NVFP4) {
    if (d->group_size != 16) return SVDQ_ERR_INVALID_ARG;
  } else if (d->precision == SVDQ_INT4) {
    if (d->group_size != 64) return SVDQ_ERR_INVALID_ARG;
  } else if (d->precision == SVDQ_AWQ_W4A16) {
    if (d->group_size != 64) return SVDQ_ERR_INVALID_ARG;
    if (d->rank != 0) return SVDQ_ERR_SHAPE;  // no low-rank branch in this family
  } else {
    return SVDQ_ERR_INVALID_ARG;
  }
  if (d->K <= 0 || d->K % 64 != 0) return SVDQ_ERR_SHAPE;
  if (d->N <= 0 || d->N % 16 != 0) return SVDQ_ERR_SHAPE;
  if (d->rank < 0 || d->rank > kRankMax || d->rank % 8 != 0) return SVDQ_ERR_SHAPE;
  if (static_cast<int64_t>(d->K) * d->N > (int64_t(1) << 40)) return SVDQ_ERR_SHAPE;
  return SVDQ_OK;
}

}  // namespace

int num_sms(int device) {
  if (device < 0 || device >= kMaxDevices) return 148;
  if (g_sms[device] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || v <= 0) v = 148;
    g_sms[device] = v;
  }
  return g_sms[device];
}

bool encode_tmap_2d_swizzle(CUtensorMap* tm, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                            uint64_t rows, uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows,
                            CUtensorMapSwizzle swizzle) {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode || rows == 0) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(tm, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap_2d(CUtensorMap* tm, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t rows,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, bool swizzle128) {
  return encode_tmap_2d_swizzle(tm, dtype, base, inner, rows, row_bytes, box_inner, box_rows,
                                swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
}

bool encode_tmap_chunked_bf16(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t K, uint32_t box_rows,
                              uint32_t box_chunks) {
  CUtensorMap probe;
  if (!encode_tmap_2d(&probe, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, K, rows, K * 2, 64, box_rows))
    return false;  // also loads the encoder entry point
  cuuint64_t dims[3] = {64, rows, K / 64};
  cuuint64_t strides[2] = {K * 2, 128};
  cuuint32_t box[3] = {64, box_rows, box_chunks};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

WeightLayout weight_layout(const svdq_layer_desc& d) {
  WeightLayout L{};
  const int rp = rank_pad_of(d.rank);
  const int64_t np = n_pad_of(d.N);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = static_cast<size_t>(round_up(static_cast<int64_t>(off + bytes), 1024));
    return at;
  };
  const bool awq = d.precision == SVDQ_AWQ_W4A16;
  L.qw = take(static_cast<size_t>(awq ? np : d.N) * d.K / 2);  // awq: GEMV tiles over n_pad rows
  L.sw_bytes = d.precision == SVDQ_NVFP4 ? nvfp4_scale_bytes(np, d.K) : int4_scale_bytes(np, d.K);
  L.sw = take(L.sw_bytes);
  L.l1s = take(static_cast<size_t>(rp) * d.K * 2);
  L.l2 = take(static_cast<size_t>(d.N) * rp * 4);
  L.inv_lambda = take(static_cast<size_t>(d.K) * 4);
  L.bias = take(static_cast<size_t>(d.N) * 4);
  L.status = take(16);
  L.amax = take(16);
  if (d.precision == SVDQ_INT4) {
    L.qw8 = take(static_cast<size_t>(np) * d.K);
  }
  L.total = off;
  return L;
}

}  // namespace svdq

using namespace svdq;

extern "C" {

const char* svdq_status_string(svdq_status s) {
  switch (s) {
    case SVDQ_OK: return "ok";
    case SVDQ_ERR_INVALID_ARG: return "invalid argument";
    case SVDQ_ERR_SHAPE: return "unsupported shape";
    case SVDQ_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    case SVDQ_ERR_UNSUPPORTED_DEVICE: return "unsupported device: the 4-bit kernels need compute capability 10.0 (B200)";
    case SVDQ_ERR_CUDA: return "CUDA error";
    case SVDQ_ERR_TIMEOUT: return "a bounded wait inside a kernel timed out";
    case SVDQ_ERR_WORKSPACE: return "storage or workspace too small";
  }
  return "unknown status";
}

svdq_status svdq_check_device(int device) {
  if (device < 0 || device >= kMaxDevices) return SVDQ_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_cc_ok[device] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device) != cudaSuccess) {
      cudaGetLastError();
      return SVDQ_ERR_CUDA;
    }
    g_cc_ok[device] = (major == 10 && minor == 0) ? 1 : -1;
  }
  return g_cc_ok[device] == 1 ? SVDQ_OK : SVDQ_ERR_UNSUPPORTED_DEVICE;
}

size_t svdq_weights_bytes(const svdq_layer_desc* desc) {
  if (check_desc(desc) != SVDQ_OK) return 0;
  return weight_layout(*desc).total;
}

svdq_status svdq_smoothing_lambda(const uint16_t* X, int32_t M, const float* W, int32_t N, int32_t K, float* lambda,
                                  float* scratch, void* stream) {
  if (!X || !W || !lambda || !scratch) return SVDQ_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0) return SVDQ_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(W) || !aligned16(lambda) || !aligned16(scratch)) return SVDQ_ERR_ALIGNMENT;
  int dev;
  svdq_status st = current_device(&dev);
  if (st != SVDQ_OK) return st;
  return from_cuda(launch_smoothing_lambda(X, M, W, N, K, lambda, scratch, static_cast<cudaStream_t>(stream)));
}

size_t svdq_lowrank_workspace_bytes(int32_t N, int32_t K) {
  if (N <= 0 || K <= 0) return 0;
  return lowrank_workspace_bytes(N, K);
}

svdq_status svdq_lowrank_factors(const float* W, int32_t N, int32_t K, const float* lambda, int32_t rank,
                                 int32_t oversample, int32_t power_steps, const float* omega, uint16_t* L1,
                                 uint16_t* L2, void* workspace, size_t ws_bytes, void* stream) {
  if (!W || !lambda || !omega || !L1 || !L2 || !workspace) return SVDQ_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0 || rank < 1 || rank % 8 != 0 || oversample < 0 || power_steps < 0 || power_steps > 16)
    return SVDQ_ERR_SHAPE;
  const int ell = rank + oversample;
  if (ell > 64 || ell > N || ell > K) return SVDQ_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(lambda) || !aligned16(omega) || !aligned16(L1) || !aligned16(L2) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return SVDQ_ERR_ALIGNMENT;
  if (ws_bytes < lowrank_workspace_bytes(N, K)) return SVDQ_ERR_WORKSPACE;
  int dev;
  svdq_status st = current_device(&dev);
  if (st != SVDQ_OK) return st;
  return from_cuda(launch_lowrank(W, N, K, lambda, rank, ell, power_steps, omega, L1, L2, workspace,
                                  static_cast<cudaStream_t>(stream)));
}

svdq_status svdq_prepare_weights(const svdq_layer_desc* desc, const float* W, const float* lambda, const uint16_t* L1,
                                 const uint16_t* L2, const uint16_t* bias, void* storage, size_t storage_bytes,
                                 svdq_weights** out, void* stream) {
  if (!out) return SVDQ_ERR_INVALID_ARG;
  *out = nullptr;
  svdq_status st = check_desc(desc);
  if (st != SVDQ_OK) return st;
  if (!W || !lambda || !storage) return SVDQ_ERR_INVALID_ARG;
  if (desc->rank > 0 && (!L1 || !L2)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(lambda) || (L1 && !aligned16(L1)) || (bias && !aligned16(bias)))
    return SVDQ_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(storage) & 1023u) != 0) return SVDQ_ERR_ALIGNMENT;
  const WeightLayout L = weight_layout(*desc);
  if (storage_bytes < L.total) return SVDQ_ERR_WORKSPACE;
  int dev;
  if ((st = current_device(&dev)) != SVDQ_OK) return st;

  svdq_weights* w = static_cast<svdq_weights*>(std::calloc(1, sizeof(svdq_weights)));
  if (!w) return SVDQ_ERR_INVALID_ARG;
  w->desc = *desc;
  w->rank_pad = rank_pad_of(desc->rank);
  w->n_pad = n_pad_of(desc->N);
  w->device = dev;
  uint8_t* b = static_cast<uint8_t*>(storage);
  w->base = b;
  w->qw = b + L.qw;
  w->sw = b + L.sw;
  w->sw_bytes = L.sw_bytes;
  w->l1s = reinterpret_cast<uint16_t*>(b + L.l1s);
  w->l2 = reinterpret_cast<float*>(b + L.l2);
  w->inv_lambda = reinterpret_cast<float*>(b + L.inv_lambda);
  w->bias = reinterpret_cast<float*>(b + L.bias);
  w->status = reinterpret_cast<int*>(b + L.status);
  w->amax = reinterpret_cast<uint32_t*>(b + L.amax);
  w->qw8 = desc->precision == SVDQ_INT4 ? b + L.qw8 : nullptr;

  bool ok = encode_tmap_2d(&w->tm_qw, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->qw, desc->K / 2, desc->N, desc->K / 2, 128,
                           128);
  if (ok && desc->precision == SVDQ_NVFP4)
    ok = encode_tmap_2d(&w->tm_sw, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->sw, 256, L.sw_bytes / 256, 256, 256, 8, false);
  if (ok && desc->precision == SVDQ_INT4)
    ok = encode_tmap_2d(&w->tm_qw8, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->qw8, desc->K, w->n_pad, desc->K, 128, 128);
  else
    w->tm_qw8 = w->tm_qw;
  if (ok && w->rank_pad > 0) {
    ok = encode_tmap_2d(&w->tm_l2, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, w->l2, w->rank_pad, desc->N,
                        static_cast<uint64_t>(w->rank_pad) * 4, 32, 128);
    if (ok)
      ok = encode_tmap_chunked_bf16(&w->tm_l1s, w->l1s, w->rank_pad, desc->K, w->rank_pad, kQChunks);
  } else {
    w->tm_l2 = w->tm_qw;
    w->tm_l1s = w->tm_qw;
  }
  if (!ok) {
    std::free(w);
    return SVDQ_ERR_CUDA;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_prepare(w, W, lambda, L1, L2, bias, s);
  float g = 1.0f;
  if (e == cudaSuccess && desc->precision == SVDQ_NVFP4)
    e = cudaMemcpyAsync(&g, w->amax + 1, sizeof(float), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    std::free(w);
    return SVDQ_ERR_CUDA;
  }
  w->g_w = g;
  *out = w;
  return SVDQ_OK;
}

void svdq_weights_destroy(svdq_weights* w) { std::free(w); }

svdq_status svdq_weights_get_view(const svdq_weights* w, svdq_weights_view* v) {
  if (!w || !v) return SVDQ_ERR_INVALID_ARG;
  v->K = w->desc.K;
  v->N = w->desc.N;
  v->rank = w->desc.rank;
  v->rank_pad = w->rank_pad;
  v->precision = w->desc.precision;
  v->group_size = w->desc.group_size;
  v->n_pad = static_cast<int32_t>(w->n_pad);
  v->g_w = w->g_w;
  v->qw = w->qw;
  v->sw = w->sw;
  v->sw_bytes = w->sw_bytes;
  v->l1s = w->l1s;
  v->l2 = w->l2;
  v->inv_lambda = w->inv_lambda;
  v->bias = w->bias;
  return SVDQ_OK;
}

svdq_status svdq_act_global_scale(const svdq_weights* w, const uint16_t* X, int32_t M, float* g_x, void* stream) {
  if (!w || !X || !g_x || w->desc.precision == SVDQ_AWQ_W4A16) return SVDQ_ERR_INVALID_ARG;
  if (M <= 0) return SVDQ_ERR_SHAPE;
  if (!aligned16(X) || (reinterpret_cast<uintptr_t>(g_x) & 3u)) return SVDQ_ERR_ALIGNMENT;
  int dev;
  svdq_status st = current_device(&dev);
  if (st != SVDQ_OK) return st;
  return from_cuda(launch_act_global_scale(w, X, M, g_x, static_cast<cudaStream_t>(stream)));
}

svdq_status svdq_act_amax(const svdq_weights* w, const uint16_t* X, int32_t M, float* amax, void* stream) {
  if (!w || !X || !amax || w->desc.precision == SVDQ_AWQ_W4A16) return SVDQ_ERR_INVALID_ARG;
  if (M <= 0) return SVDQ_ERR_SHAPE;
  if (!aligned16(X) || (reinterpret_cast<uintptr_t>(amax) & 3u)) return SVDQ_ERR_ALIGNMENT;
  int dev;
  svdq_status st = current_device(&dev);
  if (st != SVDQ_OK) return st;
  return from_cuda(launch_act_amax(w, X, M, amax, static_cast<cudaStream_t>(stream)));
}

size_t svdq_act_scale_bytes(const svdq_weights* w, int32_t M) {
  if (!w || M < 0) return 0;
  const int64_t mp = m_pad_of(M);
  return w->desc.precision == SVDQ_NVFP4 ? nvfp4_scale_bytes(mp, w->desc.K) : int4_scale_bytes(mp, w->desc.K);
}

namespace {
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Shared by the quantiser entry points.  `x_amax` (dynamic tensor scale)
// replaces g_x for NVFP4; `zero_word` (may be null) is set to 0 by the
// kernel before it ends.
svdq_status quantize_entry(const svdq_weights* w, const uint16_t* X, int32_t M, float g_x, const float* x_amax,
                           uint8_t* qx, void* sx, float* lora_act, float* zero_word, void* stream) {
  if (!w || w->desc.precision == SVDQ_AWQ_W4A16) return SVDQ_ERR_INVALID_ARG;  // 16-bit activations there
  if (M < 0) return SVDQ_ERR_SHAPE;
  if (M == 0) return SVDQ_OK;
  if (!X || !qx || !sx || (w->rank_pad > 0 && !lora_act)) return SVDQ_ERR_INVALID_ARG;
  const bool nvfp4 = w->desc.precision == SVDQ_NVFP4;
  if (nvfp4 && !x_amax && !(g_x > 0.0f && g_x < 3.0e38f)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(qx) || !aligned16(sx) || (lora_act && !aligned16(lora_act)))
    return SVDQ_ERR_ALIGNMENT;
  if ((x_amax && !aligned4(x_amax)) || (zero_word && !aligned4(zero_word))) return SVDQ_ERR_ALIGNMENT;
  int dev;
  svdq_status st = current_device(&dev);
  if (st != SVDQ_OK) return st;
  return from_cuda(launch_quantize(w, X, M, x_amax ? 1.0f : g_x, nvfp4 ? x_amax : nullptr, qx, sx, lora_act,
                                   zero_word, static_cast<cudaStream_t>(stream)));
}

// The epilogue extras' limits (see svdq.h).
svdq_status check_epi(const svdq_weights* w, const svdq_epilogue_next* epi, const svdq_qkv_prologue* pro) {
  if (!epi) return SVDQ_OK;
  if (epi->activation != SVDQ_ACT_NONE && epi->activation != SVDQ_ACT_GELU_TANH) return SVDQ_ERR_INVALID_ARG;
  if (!epi->next_inv_lambda != !epi->next_amax) return SVDQ_ERR_INVALID_ARG;
  const bool asks = epi->activation != SVDQ_ACT_NONE || epi->next_amax;
  if (asks && (pro || w->desc.precision != SVDQ_NVFP4)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned4(epi->next_inv_lambda) || !aligned4(epi->next_amax)) return SVDQ_ERR_ALIGNMENT;
  return SVDQ_OK;
}
}  // namespace

svdq_status svdq_quantize_act_lora_down(const svdq_weights* w, const uint16_t* X, int32_t M, float g_x, uint8_t* qx,
                                        void* sx, float* lora_act, void* stream) {
  return quantize_entry(w, X, M, g_x, nullptr, qx, sx, lora_act, nullptr, stream);
}

svdq_status svdq_quantize_act_lora_down_dyn(const svdq_weights* w, const uint16_t* X, int32_t M, const float* x_amax,
                                            uint8_t* qx, void* sx, float* lora_act, void* stream) {
  if (w && w->desc.precision == SVDQ_NVFP4 && !x_amax) return SVDQ_ERR_INVALID_ARG;
  return quantize_entry(w, X, M, 1.0f, x_amax, qx, sx, lora_act, nullptr, stream);
}

namespace {
// Shared by the GEMM entry points: argument checks, then the launch.
svdq_status gemm_entry(const svdq_weights* w, const uint8_t* qx, const void* sx, float g_x, const float* x_amax,
                       const float* lora_act, int32_t M, const svdq_qkv_prologue* pro, const svdq_epilogue_next* epi,
                       void* Y, int32_t out_dtype, void* stream) {
  if (!w || w->desc.precision == SVDQ_AWQ_W4A16) return SVDQ_ERR_INVALID_ARG;
  if (M < 0) return SVDQ_ERR_SHAPE;
  const svdq_status ce = check_epi(w, epi, pro);
  if (ce != SVDQ_OK) return ce;
  if (M == 0) return SVDQ_OK;
  if (!qx || !sx || !Y || (w->rank_pad > 0 && !lora_act)) return SVDQ_ERR_INVALID_ARG;
  if (out_dtype != SVDQ_OUT_BF16 && out_dtype != SVDQ_OUT_F32) return SVDQ_ERR_INVALID_ARG;
  const bool nvfp4 = w->desc.precision == SVDQ_NVFP4;
  if (nvfp4 && !x_amax && !(g_x > 0.0f && g_x < 3.0e38f)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(qx) || !aligned16(sx) || !aligned16(Y) || (lora_act && !aligned16(lora_act)))
    return SVDQ_ERR_ALIGNMENT;
  if (x_amax && !aligned4(x_amax)) return SVDQ_ERR_ALIGNMENT;
  int dev;
  svdq_status st = current_device(&dev);
  if (st != SVDQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (nvfp4) {
    const bool asks = epi && (epi->activation != SVDQ_ACT_NONE || epi->next_amax);
    return from_cuda(launch_gemm_nvfp4(w, qx, static_cast<const uint8_t*>(sx), x_amax ? 1.0f : g_x, x_amax, lora_act,
                                       M, Y, out_dtype, pro, asks ? epi : nullptr, s));
  }
  return from_cuda(launch_gemm_int4(w, qx, sx, lora_act, M, Y, out_dtype, pro, s));
}

// The QKV prologue's limits (see svdq.h).
svdq_status check_qkv(const svdq_weights* w, const svdq_qkv_prologue* pro) {
  if (!w || !pro) return SVDQ_ERR_INVALID_ARG;
  if (!pro->norm_q || !pro->norm_k || !pro->rope_cos || !pro->rope_sin) return SVDQ_ERR_INVALID_ARG;
  if (!(pro->eps > 0.0f && pro->eps < 3.0e38f)) return SVDQ_ERR_INVALID_ARG;
  if (pro->head_dim != 128 || pro->heads < 2 || (pro->heads & 1)) return SVDQ_ERR_SHAPE;
  if (static_cast<int64_t>(w->desc.N) != 3LL * pro->heads * pro->head_dim) return SVDQ_ERR_SHAPE;
  if (!aligned16(pro->norm_q) || !aligned16(pro->norm_k) || !aligned16(pro->rope_cos) || !aligned16(pro->rope_sin))
    return SVDQ_ERR_ALIGNMENT;
  return SVDQ_OK;
}
}  // namespace

svdq_status svdq_w4a4_gemm_lora_up(const svdq_weights* w, const uint8_t* qx, const void* sx, float g_x,
                                   const float* lora_act, int32_t M, void* Y, int32_t out_dtype, void* stream) {
  return gemm_entry(w, qx, sx, g_x, nullptr, lora_act, M, nullptr, nullptr, Y, out_dtype, stream);
}

svdq_status svdq_w4a4_gemm_lora_up_qkv(const svdq_weights* w, const uint8_t* qx, const void* sx, float g_x,
                                       const float* lora_act, int32_t M, const svdq_qkv_prologue* pro, void* Y,
                                       int32_t out_dtype, void* stream) {
  const svdq_status st = check_qkv(w, pro);
  if (st != SVDQ_OK) return st;
  return gemm_entry(w, qx, sx, g_x, nullptr, lora_act, M, pro, nullptr, Y, out_dtype, stream);
}

svdq_status svdq_w4a4_gemm_lora_up_dyn(const svdq_weights* w, const uint8_t* qx, const void* sx, const float* x_amax,
                                       const float* lora_act, int32_t M, const svdq_qkv_prologue* pro,
                                       const svdq_epilogue_next* epi, void* Y, int32_t out_dtype, void* stream) {
  if (w && w->desc.precision == SVDQ_NVFP4 && !x_amax) return SVDQ_ERR_INVALID_ARG;
  if (pro) {
    const svdq_status st = check_qkv(w, pro);
    if (st != SVDQ_OK) return st;
  }
  return gemm_entry(w, qx, sx, 1.0f, x_amax, lora_act, M, pro, epi, Y, out_dtype, stream);
}

size_t svdq_act_codes_bytes(const svdq_weights* w, int32_t M) {
  if (!w || M < 0 || w->desc.precision == SVDQ_AWQ_W4A16) return 0;
  const size_t packed = static_cast<size_t>(M) * (w->desc.K / 2);
  if (w->desc.precision != SVDQ_INT4) return packed;
  return int4_q8_offset(M, w->desc.K) + static_cast<size_t>(M) * w->desc.K;
}

size_t svdq_workspace_bytes(const svdq_weights* w, int32_t M) {
  if (!w || M < 0) return 0;
  const size_t qx = static_cast<size_t>(round_up(static_cast<int64_t>(svdq_act_codes_bytes(w, M)), 1024));
  const size_t sx = static_cast<size_t>(round_up(static_cast<int64_t>(svdq_act_scale_bytes(w, M)), 1024));
  const size_t la = static_cast<size_t>(round_up(static_cast<int64_t>(M) * w->rank_pad * 4, 1024));
  return qx + sx + la + 1024;  // + the dynamic tensor scale's amax word
}

namespace {
// The layer forward: quantiser then GEMM on one stream.  dyn: the dynamic
// tensor scale from `x_amax`, or, when that is null, from an amax pass
// into the workspace's last 1024 bytes.
svdq_status forward_entry(const svdq_weights* w, const uint16_t* X, int32_t M, float g_x, bool dyn,
                          const float* x_amax, const svdq_qkv_prologue* pro, const svdq_epilogue_next* epi, void* Y,
                          int32_t out_dtype, void* workspace, size_t ws_bytes, void* stream) {
  if (!w || w->desc.precision == SVDQ_AWQ_W4A16) return SVDQ_ERR_INVALID_ARG;
  if (M < 0) return SVDQ_ERR_SHAPE;
  svdq_status st = check_epi(w, epi, pro);
  if (st != SVDQ_OK) return st;
  if (M == 0) return SVDQ_OK;
  if (!workspace) return SVDQ_ERR_INVALID_ARG;
  const size_t need = svdq_workspace_bytes(w, M);
  if (ws_bytes < need) return SVDQ_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 1023u) return SVDQ_ERR_ALIGNMENT;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* qx = ws;
  uint8_t* sx = qx + round_up(static_cast<int64_t>(svdq_act_codes_bytes(w, M)), 1024);
  float* la = reinterpret_cast<float*>(sx + round_up(static_cast<int64_t>(svdq_act_scale_bytes(w, M)), 1024));
  float* amax_slot = reinterpret_cast<float*>(ws + need - 1024);
  const bool nvfp4 = w->desc.precision == SVDQ_NVFP4;
  float* next_amax = epi ? epi->next_amax : nullptr;
  if (dyn && nvfp4 && !x_amax) {
    if (!X) return SVDQ_ERR_INVALID_ARG;
    if ((st = svdq_act_amax(w, X, M, amax_slot, stream)) != SVDQ_OK) return st;
    x_amax = amax_slot;
  }
  if (next_amax && next_amax == x_amax) return SVDQ_ERR_INVALID_ARG;
  // the quantiser zeroes the next layer's amax word (stream order puts the
  // GEMM's max-reduction after it): no separate memset
  st = quantize_entry(w, X, M, g_x, dyn && nvfp4 ? x_amax : nullptr, qx, sx, w->rank_pad ? la : nullptr, next_amax,
                      stream);
  if (st != SVDQ_OK) return st;
  return gemm_entry(w, qx, sx, g_x, dyn && nvfp4 ? x_amax : nullptr, w->rank_pad ? la : nullptr, M, pro, epi, Y,
                    out_dtype, stream);
}
}  // namespace

svdq_status svdq_linear_forward(const svdq_weights* w, const uint16_t* X, int32_t M, float g_x, void* Y,
                                int32_t out_dtype, void* workspace, size_t ws_bytes, void* stream) {
  return forward_entry(w, X, M, g_x, false, nullptr, nullptr, nullptr, Y, out_dtype, workspace, ws_bytes, stream);
}

svdq_status svdq_linear_forward_qkv(const svdq_weights* w, const uint16_t* X, int32_t M, float g_x,
                                    const svdq_qkv_prologue* pro, void* Y, int32_t out_dtype, void* workspace,
                                    size_t ws_bytes, void* stream) {
  const svdq_status st = check_qkv(w, pro);
  if (st != SVDQ_OK) return st;
  return forward_entry(w, X, M, g_x, false, nullptr, pro, nullptr, Y, out_dtype, workspace, ws_bytes, stream);
}

svdq_status svdq_linear_forward_dyn(const svdq_weights* w, const uint16_t* X, int32_t M, const float* x_amax,
                                    const svdq_qkv_prologue* pro, const svdq_epilogue_next* epi, void* Y,
                                    int32_t out_dtype, void* workspace, size_t ws_bytes, void* stream) {
  if (pro) {
    const svdq_status st = check_qkv(w, pro);
    if (st != SVDQ_OK) return st;
  }
  return forward_entry(w, X, M, 1.0f, true, x_amax, pro, epi, Y, out_dtype, workspace, ws_bytes, stream);
}

svdq_status svdq_awq_w4a16_forward(const svdq_weights* w, const uint16_t* X, int32_t M, void* Y, int32_t out_dtype,
                                   void* stream) {
  if (!w || w->desc.precision != SVDQ_AWQ_W4A16) return SVDQ_ERR_INVALID_ARG;
  if (M < 0) return SVDQ_ERR_SHAPE;
  if (M == 0) return SVDQ_OK;
  if (!X || !Y) return SVDQ_ERR_INVALID_ARG;
  if (out_dtype != SVDQ_OUT_BF16 && out_dtype != SVDQ_OUT_F32) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Y)) return SVDQ_ERR_ALIGNMENT;
  int dev;
  svdq_status st = current_device(&dev);
  if (st != SVDQ_OK) return st;
  return from_cuda(launch_awq_gemv(w, X, M, Y, out_dtype, static_cast<cudaStream_t>(stream)));
}

svdq_status svdq_device_status(const svdq_weights* w, void* stream) {
  if (!w) return SVDQ_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaMemcpyAsync(&v, w->status, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (v != 0) {
    if (cudaMemsetAsync(w->status, 0, sizeof(int), s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
      return SVDQ_ERR_CUDA;
    return static_cast<svdq_status>(v);
  }
  return SVDQ_OK;
}

}  // extern "C"
