// The awq_w4a16 layer: INT4 group-64 weights against 16-bit activations
// (Nunchaku 4-bit in Diffusers, the second kernel family: 4-bit weights,
// 16-bit activations, for the memory-bound, precision-sensitive modulation
// projections; quantization_config block "awq_w4a16": int4, group_size 64).
//
//     Y = X_hat (s_h q)^T + b,   X_hat = RN32(X * inv_alpha),  fp32 sums
//
// sm_100a design: the activations are a handful of rows (the batch), so
// the work is a stream over the weight codes with a few multiply-adds per
// code: CUDA cores, no tensor cores.  One CTA of 8 warps per block of 32
// output rows (and up to 8 activation rows); lane = output row, warp w takes
// the 64-groups g = w, w + 8, ...  The codes are stored in GEMV tiles (32
// rows x 16 bytes of one 32-code chunk contiguous), so every warp load is
// 512 contiguous bytes and a CTA streams 16 KB-aligned runs of the codes.
// X_hat is staged in shared memory as fp32 (one RN32 multiply per element
// and CTA); reads of it are warp-wide broadcasts.
//
// Decoding: a 4-bit two's-complement code v becomes an fp32 without a
// conversion instruction.  One XOR per 32-bit word of eight codes turns
// every nibble into v + 8; two masks split the word into the low and the
// high nibbles of its bytes; a byte permute then puts one of them under the
// bytes of 0x4B000000, giving bits 0x4B0000(v + 8) = 2^23 + v + 8, and one
// packed subtraction of 2^23 + 8 leaves v exactly.  Every decoded pair
// feeds a packed FMA with its two activations; a group's four partial sums
// are added before the group scale multiplies them, and the 8 warps'
// partial rows are added in warp order through shared memory.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>

#include "internal.h"

namespace svdq {
namespace {

constexpr int kAwqWarps = 8;
constexpr int kAwqThreads = 32 * kAwqWarps;

template <int MT, bool kF32Out>
__global__ void __launch_bounds__(kAwqThreads)
    awq_gemv_kernel(const uint8_t* __restrict__ qg, const __half* __restrict__ sw, const float* __restrict__ inv_alpha,
                    const float* __restrict__ bias, const uint16_t* __restrict__ X, int M, int N, int K, int64_t n_pad,
                    void* __restrict__ Y) {
  extern __shared__ float awq_smem[];
  float* xs = awq_smem;                 // MT x K: X_hat rows m0 .. m0 + MT - 1 (zeros past M)
  float* part = awq_smem + MT * K;      // kAwqWarps x MT x 32 partial sums
  const int m0 = blockIdx.y * MT;
  const int nb = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = nb * 32 + lane;  // < n_pad: padding rows hold zero codes and scales
  const int groups = K / 64;
  const uint8_t* tile = qg + static_cast<size_t>(nb) * (K / 32) * 512 + lane * 16;
  // the upper three bytes of 2^23 as fp32, in a register for the byte permutes
  const uint32_t kMagic = 0x4B000000u;
  float y[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) y[m] = 0.0f;

  // this warp's groups g = warp + 8 it, it < iters; the codes and scale of
  // the next kD groups are in flight while one is decoded (rotating slots).
  // The first loads are issued before X_hat is staged, so that their
  // latency overlaps it.
  constexpr int kD = 2;
  const int iters = groups > warp ? (groups - warp + kAwqWarps - 1) / kAwqWarps : 0;
  uint4 ca[kD], cb[kD];
  float sc[kD];
  auto load = [&](int d, int it) {
    const int g = warp + kAwqWarps * it;
    ca[d] = __ldg(reinterpret_cast<const uint4*>(tile + static_cast<size_t>(2 * g) * 512));
    cb[d] = __ldg(reinterpret_cast<const uint4*>(tile + static_cast<size_t>(2 * g + 1) * 512));
    sc[d] = __half2float(sw[static_cast<size_t>(g) * n_pad + n]);
  };
#pragma unroll
  for (int d = 0; d < kD; ++d)
    if (d < iters) load(d, d);
  // X_hat rows, eight values per thread and step (16-byte loads)
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    for (int j = threadIdx.x; j < K / 8; j += kAwqThreads) {
      float4 lo = make_float4(0.0f, 0.0f, 0.0f, 0.0f), hi = lo;
      if (m0 + m < M) {
        const uint4 xb = __ldg(reinterpret_cast<const uint4*>(X + static_cast<size_t>(m0 + m) * K) + j);
        const float4 a0 = __ldg(reinterpret_cast<const float4*>(inv_alpha) + 2 * j);
        const float4 a1 = __ldg(reinterpret_cast<const float4*>(inv_alpha) + 2 * j + 1);
        lo = make_float4(__fmul_rn(__uint_as_float(xb.x << 16), a0.x), __fmul_rn(__uint_as_float(xb.x & 0xFFFF0000u), a0.y),
                         __fmul_rn(__uint_as_float(xb.y << 16), a0.z), __fmul_rn(__uint_as_float(xb.y & 0xFFFF0000u), a0.w));
        hi = make_float4(__fmul_rn(__uint_as_float(xb.z << 16), a1.x), __fmul_rn(__uint_as_float(xb.z & 0xFFFF0000u), a1.y),
                         __fmul_rn(__uint_as_float(xb.w << 16), a1.z), __fmul_rn(__uint_as_float(xb.w & 0xFFFF0000u), a1.w));
      }
      reinterpret_cast<float4*>(xs + m * K)[2 * j] = lo;
      reinterpret_cast<float4*>(xs + m * K)[2 * j + 1] = hi;
    }
  }
  __syncthreads();

  for (int it0 = 0; it0 < iters; it0 += kD) {
#pragma unroll
    for (int d = 0; d < kD; ++d) {
      const int it = it0 + d;
      if (it < iters) {
        const uint4 c0 = ca[d], c1 = cb[d];
        const float s = sc[d];
        if (it + kD < iters) load(d, it + kD);
        const int g = warp + kAwqWarps * it;
        const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        const float2 kOff = make_float2(-(8388608.0f + 8.0f), -(8388608.0f + 8.0f));
        float2 a0[MT], a1[MT];  // codes of bytes 0, 2 and of bytes 1, 3 of every word
#pragma unroll
        for (int m = 0; m < MT; ++m) a0[m] = a1[m] = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int wd = 0; wd < 8; ++wd) {  // 8 codes: k = 64 g + 8 wd + (0..7), low nibble = even k
          const uint32_t wq = words[wd] ^ 0x88888888u;    // every nibble v -> v + 8
          const uint32_t lo = wq & 0x0F0F0F0Fu;            // byte j: code 2j
          const uint32_t hi = (wq >> 4) & 0x0F0F0F0Fu;     // byte j: code 2j + 1
          const int k = 64 * g + 8 * wd;
#pragma unroll
          for (int jj = 0; jj < 4; jj += 2) {  // bytes jj, jj + 1: codes k + 2 jj .. k + 2 jj + 3
            const float2 v0 = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(lo, kMagic, 0x7650u + jj)),
                                                     __uint_as_float(__byte_perm(hi, kMagic, 0x7650u + jj))),
                                         kOff);
            const float2 v1 = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(lo, kMagic, 0x7651u + jj)),
                                                     __uint_as_float(__byte_perm(hi, kMagic, 0x7651u + jj))),
                                         kOff);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
              const float4 x = *reinterpret_cast<const float4*>(xs + m * K + k + 2 * jj);  // broadcast
              a0[m] = __ffma2_rn(v0, make_float2(x.x, x.y), a0[m]);
              a1[m] = __ffma2_rn(v1, make_float2(x.z, x.w), a1[m]);
            }
          }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const float gsum = __fadd_rn(__fadd_rn(a0[m].x, a0[m].y), __fadd_rn(a1[m].x, a1[m].y));
          y[m] = __fmaf_rn(s, gsum, y[m]);
        }
      }
    }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) part[(warp * MT + m) * 32 + lane] = y[m];
  __syncthreads();
  if (threadIdx.x < 32 * MT) {
    const int m = threadIdx.x >> 5;
    float t = 0.0f;
#pragma unroll
    for (int w = 0; w < kAwqWarps; ++w) t = __fadd_rn(t, part[(w * MT + m) * 32 + lane]);
    if (m0 + m < M && n < N) {
      t = __fadd_rn(t, __ldg(bias + n));
      const size_t o = static_cast<size_t>(m0 + m) * N + n;
      if constexpr (kF32Out)
        static_cast<float*>(Y)[o] = t;
      else
        static_cast<__nv_bfloat16*>(Y)[o] = __float2bfloat16_rn(t);
    }
  }
}

template <int MT, bool kF32Out>
cudaError_t launch_mt(const svdq_weights* w, const uint16_t* X, int M, void* Y, cudaStream_t s) {
  const int K = w->desc.K, N = w->desc.N;
  const size_t smem = (static_cast<size_t>(MT) * K + kAwqWarps * MT * 32) * sizeof(float);
  auto kern = awq_gemv_kernel<MT, kF32Out>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>((N + 31) / 32), static_cast<unsigned>((M + MT - 1) / MT));
  kern<<<grid, kAwqThreads, smem, s>>>(w->qw, static_cast<const __half*>(w->sw), w->inv_lambda, w->bias, X, M, N, K,
                                        w->n_pad, Y);
  return cudaGetLastError();
}

template <bool kF32Out>
cudaError_t launch_out(const svdq_weights* w, const uint16_t* X, int M, void* Y, cudaStream_t s) {
  // rows of X per CTA: the smallest power of two >= M up to 8, within the
  // shared memory that stages them (8 rows of K = 3072 take 96 KB)
  const size_t per_row = static_cast<size_t>(w->desc.K) * sizeof(float);
  int mt = M >= 8 ? 8 : (M >= 4 ? (M == 4 ? 4 : 8) : (M >= 2 ? (M == 2 ? 2 : 4) : 1));
  while (mt > 1 && mt * per_row > 200 * 1024) mt >>= 1;
  if (per_row > 200 * 1024) return cudaErrorInvalidValue;
  switch (mt) {
    case 8: return launch_mt<8, kF32Out>(w, X, M, Y, s);
    case 4: return launch_mt<4, kF32Out>(w, X, M, Y, s);
    case 2: return launch_mt<2, kF32Out>(w, X, M, Y, s);
    default: return launch_mt<1, kF32Out>(w, X, M, Y, s);
  }
}

}  // namespace

cudaError_t launch_awq_gemv(const svdq_weights* w, const uint16_t* X, int M, void* Y, int out_dtype, cudaStream_t s) {
  return out_dtype == SVDQ_OUT_F32 ? launch_out<true>(w, X, M, Y, s) : launch_out<false>(w, X, M, Y, s);
}

}  // namespace svdq
