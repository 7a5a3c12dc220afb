// Weight preparation of the SVDQuant W4A4 layer, on the GPU.
//
// The pages' offline quantiser (Nunchaku 4-bit in Diffusers, "Eigenes
// Modell quantisieren", steps 1-2) turns each dense weight into the 4-bit
// residual plus the 16-bit low-rank branch ("Nunchaku und SVDQuant").  Here:
//   inv_lambda = RN32(1/lambda), W_til = RN32(W * lambda),
//   R[n,k] = RN32(fp64 chain W_til - L1[0,k] L2[n,0] - ... in t order),
//   NVFP4: g_w = RN32(amax|R| / 2688) (1 if 0), per-16 E4M3 scale + E2M1
//   codes; INT4: per-64 fp16 scale + signed codes;
//   L1s = bf16(RN32(L1 * inv_lambda)) (rows padded with zeros to rank_pad),
//   L2 widened to fp32 (columns padded with zeros), bias widened to fp32.
// R is recomputed in the quantisation pass instead of being stored: the
// chain is deterministic, so both passes see the same bits.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace svdq {
namespace {

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

__global__ void inv_lambda_kernel(const float* __restrict__ lam, int K, float* __restrict__ inv) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k < K) inv[k] = __frcp_rn(lam[k]);
}

// Residual of 16 consecutive columns [k0, k0+16) of row n.
__device__ __forceinline__ void residual16(const float* __restrict__ W, const float* __restrict__ lam,
                                           const uint16_t* __restrict__ L1, const uint16_t* __restrict__ L2, int K,
                                           int r, int n, int k0, float (&R)[16]) {
  const float* wr = W + static_cast<size_t>(n) * K + k0;
  double acc[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j] = static_cast<double>(__fmul_rn(__ldg(wr + j), __ldg(lam + k0 + j)));
  for (int t = 0; t < r; ++t) {
    const double b = static_cast<double>(bf16_to_f32(__ldg(L2 + static_cast<size_t>(n) * r + t)));
    const uint16_t* l1 = L1 + static_cast<size_t>(t) * K + k0;
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = __fma_rn(-static_cast<double>(bf16_to_f32(__ldg(l1 + j))), b, acc[j]);
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) R[j] = __double2float_rn(acc[j]);
}

// Pass 1 (NVFP4 only): amax |R| over the matrix into *amax_bits.
__global__ void residual_amax_kernel(const float* __restrict__ W, const float* __restrict__ lam,
                                     const uint16_t* __restrict__ L1, const uint16_t* __restrict__ L2, int N, int K,
                                     int r, uint32_t* amax_bits) {
  const int groups = K / 16;
  const size_t total = static_cast<size_t>(N) * groups;
  float amax = 0.0f;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int n = static_cast<int>(i / groups);
    const int k0 = static_cast<int>(i % groups) * 16;
    float R[16];
    residual16(W, lam, L1, L2, K, r, n, k0, R);
#pragma unroll
    for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(R[j]));
  }
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(amax));
}

__global__ void weight_scale_kernel(const uint32_t* __restrict__ amax_bits, float* __restrict__ g_w) {
  const float amax = __uint_as_float(*amax_bits);
  *g_w = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 2688.0f);
}

// Pass 2: quantise R.  One thread per (row n, 16-column chunk); for INT4 the
// four chunks of a 64-group sit in four consecutive lanes.
template <bool kInt4>
__global__ void quantize_weights_kernel(const float* __restrict__ W, const float* __restrict__ lam,
                                        const uint16_t* __restrict__ L1, const uint16_t* __restrict__ L2, int N,
                                        int K, int r, const float* __restrict__ g_w_ptr, int64_t n_pad,
                                        uint8_t* __restrict__ qw, uint8_t* __restrict__ sw, int gemv_tiles) {
  const int groups = K / 16;
  const size_t total = static_cast<size_t>(N) * groups;
  const size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  const bool valid = i < total;
  const int n = valid ? static_cast<int>(i / groups) : 0;
  const int j = valid ? static_cast<int>(i % groups) : 0;
  const int k0 = j * 16;
  float R[16];
  if (valid) {
    residual16(W, lam, L1, L2, K, r, n, k0, R);
  } else {
#pragma unroll
    for (int e = 0; e < 16; ++e) R[e] = 0.0f;
  }
  uint32_t lo = 0, hi = 0;
  if constexpr (!kInt4) {
    const float g = *g_w_ptr;
    float amax = 0.0f;
#pragma unroll
    for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(R[e]));
    const uint32_t sq = cvt_e4m3(__fdiv_rn(__fdiv_rn(amax, 6.0f), g));
    const float s = e4m3_to_f32(sq);
    if (s != 0.0f) {
      const float rcp = __frcp_rn(__fmul_rn(s, g));
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        lo |= cvt_e2m1x2(__fmul_rn(R[e], rcp), __fmul_rn(R[e + 1], rcp)) << (4 * e);
        hi |= cvt_e2m1x2(__fmul_rn(R[8 + e], rcp), __fmul_rn(R[9 + e], rcp)) << (4 * e);
      }
    }
    if (valid) {
      const size_t off = (static_cast<size_t>(n >> 7) * (K / 64) + (j >> 2)) * 512 + (n & 31) * 16 +
                         ((n >> 5) & 3) * 4 + (j & 3);
      sw[off] = static_cast<uint8_t>(sq);
    }
  } else {
    float amax = 0.0f;
#pragma unroll
    for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(R[e]));
    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
    const __half s_h = __float2half_rn(__fdiv_rn(amax, 7.0f));
    const float s32 = __half2float(s_h);
    if (s32 != 0.0f) {
      const float rcp = __frcp_rn(s32);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        float v = rintf(__fmul_rn(R[e], rcp));
        v = fminf(fmaxf(v, -8.0f), 7.0f);
        const uint32_t nib = static_cast<uint32_t>(static_cast<int>(v)) & 0xFu;
        if (e < 8)
          lo |= nib << (4 * e);
        else
          hi |= nib << (4 * (e - 8));
      }
    }
    if (valid && (j & 3) == 0) reinterpret_cast<__half*>(sw)[static_cast<size_t>(j >> 2) * n_pad + n] = s_h;
  }
  if (valid) {
    // row-major, or (awq_w4a16) the GEMV tiles: 16 bytes per 32 codes of a
    // row, 32 rows of a chunk contiguous
    const size_t off = gemv_tiles ? (static_cast<size_t>(n >> 5) * (K / 32) + (k0 >> 5)) * 512 + (n & 31) * 16 +
                                        ((k0 >> 4) & 1) * 8
                                  : static_cast<size_t>(n) * (K / 2) + k0 / 2;
    *reinterpret_cast<uint2*>(qw + off) = make_uint2(lo, hi);
  }
}

// INT4 working copy: the codes as E4M3 bytes in natural K order (rows
// N..n_pad zero).
__global__ void int4_e4m3_kernel(const uint8_t* __restrict__ qw, int N, int K, int64_t n_pad,
                                 uint8_t* __restrict__ qw8) {
  const size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  const size_t blocks = static_cast<size_t>(n_pad) * (K / 8);
  if (i < blocks) {
    const int64_t n = static_cast<int64_t>(i / (K / 8));
    const int j = static_cast<int>(i % (K / 8));
    uint2 out = make_uint2(0u, 0u);
    if (n < N) {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(qw + static_cast<size_t>(n) * (K / 2) + 4 * j);
      uint32_t b[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint32_t nib = (w >> (4 * e)) & 0xFu;
        const uint32_t tab = nib < 4 ? kI4E4m3Lo0 : nib < 8 ? kI4E4m3Lo1 : nib < 12 ? kI4E4m3Hi0 : kI4E4m3Hi1;
        b[e] = (tab >> (8 * (nib & 3))) & 0xFFu;
      }
      out.x = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
      out.y = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
    }
    *reinterpret_cast<uint2*>(qw8 + static_cast<size_t>(n) * K + 8 * j) = out;
  }
}

__global__ void l1s_kernel(const uint16_t* __restrict__ L1, const float* __restrict__ inv, int K, int r, int r_pad,
                           uint16_t* __restrict__ l1s) {
  const size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  if (i >= static_cast<size_t>(r_pad) * K) return;
  const int t = static_cast<int>(i / K);
  const int k = static_cast<int>(i % K);
  float v = 0.0f;
  if (t < r) v = __fmul_rn(bf16_to_f32(L1[static_cast<size_t>(t) * K + k]), inv[k]);
  l1s[i] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

__global__ void l2_bias_kernel(const uint16_t* __restrict__ L2, const uint16_t* __restrict__ bias_in, int N, int r,
                               int r_pad, float* __restrict__ l2, float* __restrict__ bias) {
  const size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  if (i < static_cast<size_t>(N) * r_pad) {
    const int n = static_cast<int>(i / r_pad);
    const int t = static_cast<int>(i % r_pad);
    l2[i] = t < r ? bf16_to_f32(L2[static_cast<size_t>(n) * r + t]) : 0.0f;
  }
  if (i < static_cast<size_t>(N)) bias[i] = bias_in ? bf16_to_f32(bias_in[i]) : 0.0f;
}

}  // namespace

cudaError_t launch_prepare(const svdq_weights* w, const float* W, const float* lambda, const uint16_t* L1,
                           const uint16_t* L2, const uint16_t* bias, cudaStream_t s) {
  const int K = w->desc.K, N = w->desc.N, r = w->desc.rank, rp = w->rank_pad;
  const bool int4 = w->desc.precision == SVDQ_INT4;
  const bool awq = w->desc.precision == SVDQ_AWQ_W4A16;
  float* g_w_dev = reinterpret_cast<float*>(w->amax + 1);
  cudaError_t e;
  if ((e = cudaMemsetAsync(w->sw, 0, w->sw_bytes, s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(w->amax, 0, 16, s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(w->status, 0, sizeof(int), s)) != cudaSuccess) return e;
  inv_lambda_kernel<<<(K + 255) / 256, 256, 0, s>>>(lambda, K, w->inv_lambda);
  const size_t chunks = static_cast<size_t>(N) * (K / 16);
  const int sms = num_sms(w->device);
  if (awq) {
    // the tile layout covers n_pad rows: the rows past N keep zero codes
    if ((e = cudaMemsetAsync(w->qw, 0, static_cast<size_t>(w->n_pad) * (K / 2), s)) != cudaSuccess) return e;
    quantize_weights_kernel<true><<<static_cast<unsigned>((chunks + 255) / 256), 256, 0, s>>>(
        W, lambda, L1, L2, N, K, r, g_w_dev, w->n_pad, w->qw, static_cast<uint8_t*>(w->sw), 1);
  } else if (!int4) {
    const int blocks = static_cast<int>(std::min<size_t>((chunks + 255) / 256, static_cast<size_t>(sms) * 16));
    residual_amax_kernel<<<std::max(blocks, 1), 256, 0, s>>>(W, lambda, L1, L2, N, K, r, w->amax);
    weight_scale_kernel<<<1, 1, 0, s>>>(w->amax, g_w_dev);
    quantize_weights_kernel<false><<<static_cast<unsigned>((chunks + 255) / 256), 256, 0, s>>>(
        W, lambda, L1, L2, N, K, r, g_w_dev, w->n_pad, w->qw, static_cast<uint8_t*>(w->sw), 0);
  } else {
    quantize_weights_kernel<true><<<static_cast<unsigned>((chunks + 255) / 256), 256, 0, s>>>(
        W, lambda, L1, L2, N, K, r, g_w_dev, w->n_pad, w->qw, static_cast<uint8_t*>(w->sw), 0);
    const size_t work = static_cast<size_t>(w->n_pad) * (K / 8);
    int4_e4m3_kernel<<<static_cast<unsigned>((work + 255) / 256), 256, 0, s>>>(w->qw, N, K, w->n_pad, w->qw8);
  }
  if (rp > 0) {
    const size_t n1 = static_cast<size_t>(rp) * K;
    l1s_kernel<<<static_cast<unsigned>((n1 + 255) / 256), 256, 0, s>>>(L1, w->inv_lambda, K, r, rp, w->l1s);
  }
  const size_t n2 = std::max(static_cast<size_t>(N) * std::max(rp, 1), static_cast<size_t>(N));
  l2_bias_kernel<<<static_cast<unsigned>((n2 + 255) / 256), 256, 0, s>>>(L2, bias, N, r, rp, w->l2, w->bias);
  return cudaGetLastError();
}

}  // namespace svdq
