// The 4-bit GEMM of the SVDQuant W4A4 layer with the lora-up and the bias
// fused into the epilogue (charmloop.ai Nunchaku news item, second
// paragraph: "the up-projection into the 4-bit compute kernel").
//
// sm_100a design, one persistent CTA per SM, 128 x 256 output tiles:
//   warp 0      TMA producer: qx / qw tiles (128-byte swizzle) and the
//               per-16 E4M3 scale atoms (bulk copies) into a 4-stage ring.
//   warp 1      TMEM owner and MMA issuer: per tile, ceil(rank/32) ring
//               slots carry the lora_act / L2 tiles and are multiplied with
//               tcgen05 kind::tf32 into the accumulator, then every K stage
//               copies its scales to TMEM (tcgen05.cp) and issues
//               tcgen05 kind::mxf4nvf4 block-scaled MMAs (K = 64 each).
//   warps 2-9   epilogue: drain the 128 x 256 fp32 accumulator from TMEM,
//               release it to the MMA warp, then y = acc * g_x g_w + b.
// The lora-up shares the accumulator with the 4-bit product because
// lora_act arrives pre-divided by g_x g_w: one TMEM read per output.
//
// TMEM columns: [0, 256) accumulator, [256, 272) A scales, [272, 304) B
// scales (4 x 32-bit columns per 128 rows per MMA; lane i of every 32-lane
// quarter holds rows i, i+32, i+64, i+96 in its four columns).
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace svdq {
namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 256;  // fp4 elements per ring stage (128 bytes per row)
constexpr int kStages = 4;
constexpr int kABytes = BM * BK / 2;                                   // 16 KB
constexpr int kBBytes = BN * BK / 2;                                   // 32 KB
constexpr int kSfaBytes = BM * BK / 16;                                // 2 KB
constexpr int kSfbBytes = BN * BK / 16;                                // 4 KB
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;  // 54 KB
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColAcc = 0, kColSfa = 256, kColSfb = 272;
constexpr size_t kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;

static_assert(kStageBytes % 1024 == 0, "stages must keep 1024-byte alignment");
static_assert(kSmemBytes <= 232448, "shared memory budget");

// Instruction descriptors (kind::mxf4nvf4 block-scaled and kind::tf32),
// M = 128, N = 256, both operands K-major.
constexpr uint32_t kIdescNvfp4 = (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);
constexpr uint32_t kIdescTf32 =
    (1u << 4) | (2u << 7) | (2u << 10) | (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);

struct GemmParams {
  const uint8_t* sfa;
  const uint8_t* sfb;
  const float* bias;
  void* Y;
  int* status;
  int M, N, K, n_lora;
  float gxgw;
};

template <bool kF32Out>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                      const __grid_constant__ CUtensorMap tm_la, const __grid_constant__ CUtensorMap tm_lb,
                      const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_m = (p.M + BM - 1) / BM;
  const int num_n = (p.N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int k_sub = p.K / 64;               // 64-wide MMA steps along K
  const int num_kb = (k_sub + 3) / 4;       // ring stages per tile for the 4-bit product

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kEpiWarps);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    if (p.n_lora) {
      prefetch_tmap(&tm_la);
      prefetch_tmap(&tm_lb);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  uint32_t issued_mask = 0, issued_par = 0;  // producer bookkeeping for the teardown drain

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        const int mb = tile % num_m, nb = tile / num_m;
        const int m0 = mb * BM, n0 = nb * BN;
        for (int j = 0; j < p.n_lora; ++j) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) goto teardown;
          uint8_t* st = smem + stage * kStageBytes;
          mbar_arrive_expect_tx(&full[stage], kABytes + kBBytes);
          tma_load_2d(st, &tm_la, 32 * j, m0, &full[stage]);
          tma_load_2d(st + kABytes, &tm_lb, 32 * j, n0, &full[stage]);
          issued_mask |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        for (int kb = 0; kb < num_kb; ++kb) {
          const int nsub = min(4, k_sub - 4 * kb);
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) goto teardown;
          uint8_t* st = smem + stage * kStageBytes;
          mbar_arrive_expect_tx(&full[stage], kABytes + kBBytes + 3 * nsub * 512);
          tma_load_2d(st, &tm_a, kb * 128, m0, &full[stage]);
          tma_load_2d(st + kABytes, &tm_b, kb * 128, n0, &full[stage]);
          const size_t sf_off = static_cast<size_t>(4 * kb) * 512;
          bulk_load(st + kABytes + kBBytes, p.sfa + static_cast<size_t>(mb) * k_sub * 512 + sf_off, nsub * 512,
                    &full[stage]);
          bulk_load(st + kABytes + kBBytes + kSfaBytes, p.sfb + static_cast<size_t>(2 * nb) * k_sub * 512 + sf_off,
                    nsub * 512, &full[stage]);
          bulk_load(st + kABytes + kBBytes + kSfaBytes + 2048,
                    p.sfb + static_cast<size_t>(2 * nb + 1) * k_sub * 512 + sf_off, nsub * 512, &full[stage]);
          issued_mask |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      const uint32_t d_acc = tmem + kColAcc;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        if (!mbar_wait(acc_empty, acc_phase ^ 1, abort_flag)) goto teardown;
        tc_fence_after();
        uint32_t accumulate = 0;
        for (int j = 0; j < p.n_lora; ++j) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) goto teardown;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * kStageBytes);
          const uint64_t da = sdesc_sw128(sa), db = sdesc_sw128(sa + kABytes);
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // 4 x K=8 tf32 steps of 32 bytes
            mma_tf32(d_acc, da + 2 * k, db + 2 * k, kIdescTf32, accumulate);
            accumulate = 1;
          }
          tc_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        for (int kb = 0; kb < num_kb; ++kb) {
          const int nsub = min(4, k_sub - 4 * kb);
          if (!mbar_wait(&full[stage], phase, abort_flag)) goto teardown;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * kStageBytes);
          const uint32_t s_sfa = sa + kABytes + kBBytes;
          const uint32_t s_sfb = s_sfa + kSfaBytes;
          for (int k = 0; k < nsub; ++k) {
            tc_cp_32x128b_warpx4(tmem + kColSfa + 4 * k, sdesc_rows16(s_sfa + 512 * k));
            tc_cp_32x128b_warpx4(tmem + kColSfb + 8 * k, sdesc_rows16(s_sfb + 512 * k));
            tc_cp_32x128b_warpx4(tmem + kColSfb + 8 * k + 4, sdesc_rows16(s_sfb + 2048 + 512 * k));
          }
          const uint64_t da = sdesc_sw128(sa), db = sdesc_sw128(sa + kABytes);
          for (int k = 0; k < nsub; ++k) {  // K=64 fp4 steps of 32 bytes
            mma_nvfp4(d_acc, da + 2 * k, db + 2 * k, kIdescNvfp4, tmem + kColSfa + 4 * k, tmem + kColSfb + 8 * k,
                      accumulate);
            accumulate = 1;
          }
          tc_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        tc_commit(acc_full);
        acc_phase ^= 1;
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int m0 = (tile % num_m) * BM, n0 = (tile / num_m) * BN;
      if (!mbar_wait(acc_full, acc_phase, abort_flag)) break;
      acc_phase ^= 1;
      tc_fence_after();
      uint32_t v[4][32];
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + kColAcc + half * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(taddr + 32 * c, v[c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);

      const int row = m0 + quarter * 32 + lane;
      if (row < p.M) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            const int n = n0 + half * 128 + 32 * c + i;
            if (n < p.N) {
              const float4 b0 = __ldg(reinterpret_cast<const float4*>(p.bias + n));
              const float4 b1 = __ldg(reinterpret_cast<const float4*>(p.bias + n + 4));
              const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
              float y[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) y[e] = __fadd_rn(__fmul_rn(__uint_as_float(v[c][i + e]), p.gxgw), bb[e]);
              if constexpr (kF32Out) {
                float* dst = static_cast<float*>(p.Y) + static_cast<size_t>(row) * p.N + n;
                reinterpret_cast<float4*>(dst)[0] = make_float4(y[0], y[1], y[2], y[3]);
                reinterpret_cast<float4*>(dst)[1] = make_float4(y[4], y[5], y[6], y[7]);
              } else {
                uint4 o;
                __nv_bfloat162 h;
                h = __floats2bfloat162_rn(y[0], y[1]); o.x = *reinterpret_cast<uint32_t*>(&h);
                h = __floats2bfloat162_rn(y[2], y[3]); o.y = *reinterpret_cast<uint32_t*>(&h);
                h = __floats2bfloat162_rn(y[4], y[5]); o.z = *reinterpret_cast<uint32_t*>(&h);
                h = __floats2bfloat162_rn(y[6], y[7]); o.w = *reinterpret_cast<uint32_t*>(&h);
                *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.Y) + static_cast<size_t>(row) * p.N + n) = o;
              }
            }
          }
        }
      }
    }
  }

teardown:
  __syncthreads();
  if (warp == 0 && lane == 0) {
    // every TMA / bulk copy this CTA issued must land before shared memory is released
    for (int s = 0; s < kStages; ++s)
      if (issued_mask & (1u << s)) mbar_wait_limited(&full[s], (issued_par >> s) & 1u, 200000000ull);
  }
  if (warp == 1 && lane == 0) {
    tc_commit(drain);  // arrives once every MMA / copy issued so far has finished
    mbar_wait_limited(drain, 0, 200000000ull);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicExch(p.status, static_cast<int>(SVDQ_ERR_TIMEOUT));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_gemm_nvfp4(const svdq_weights* w, const uint8_t* qx, const uint8_t* sx, float g_x,
                              const float* lora_act, int M, void* Y, int out_dtype, cudaStream_t s) {
  const int K = w->desc.K, N = w->desc.N;
  CUtensorMap tm_a, tm_la;
  if (!encode_tmap_2d(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, qx, K / 2, M, K / 2, 128, BM))
    return cudaErrorInvalidValue;
  if (w->rank_pad > 0) {
    if (!encode_tmap_2d(&tm_la, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, lora_act, w->rank_pad, M,
                         static_cast<uint64_t>(w->rank_pad) * 4, 32, BM))
      return cudaErrorInvalidValue;
  } else {
    tm_la = tm_a;  // unused when there is no low-rank branch
  }
  GemmParams p;
  p.sfa = sx;
  p.sfb = static_cast<const uint8_t*>(w->sw);
  p.bias = w->bias;
  p.Y = Y;
  p.status = w->status;
  p.M = M;
  p.N = N;
  p.K = K;
  p.n_lora = w->rank_pad / 32;
  p.gxgw = g_x * w->g_w;  // RN32(g_x * g_w)
  const int tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int grid = std::min(tiles, num_sms(w->device));
  auto kern = out_dtype == SVDQ_OUT_F32 ? gemm_nvfp4_kernel<true> : gemm_nvfp4_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, kSmemBytes, s>>>(tm_a, w->tm_qw, tm_la, w->tm_l2, p);
  return cudaGetLastError();
}

}  // namespace svdq
