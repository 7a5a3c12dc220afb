// The 4-bit GEMM of the SVDQuant W4A4 layer with the lora-up and the bias
// fused into the epilogue (charmloop.ai Nunchaku news item, second
// paragraph: the up-projection runs inside the 4-bit compute kernel).
//
// sm_100a design: CTA pairs (clusters of 2) run tcgen05 cta_group::2 MMAs on
// 256 x 256 output tiles; the pair is persistent over the tile list.
// Each CTA stages its own 128 rows of A (codes of X_hat) and its own 128
// rows of B (codes of R) per 256-wide K step, so a pair reads the B tile
// once for 256 output rows: 38 KB per SM per K step instead of the 54 KB of
// a 128 x 256 single-CTA tile.  All loads are plain 2-D TMA copies into the
// issuing CTA's own shared memory, counted on the first CTA's barrier.
//   warp 0      TMA producer (both CTAs): codes, per-16 E4M3 scale atoms,
//               and, per tile, the lora_act / L2 slots of the low-rank branch.
//   warp 1      TMEM owner (both CTAs); in the first CTA the MMA issuer:
//               tf32 lora-up MMAs into the accumulator, then per K step the
//               scale copies to TMEM (tcgen05.cp) and the block-scaled
//               kind::mxf4nvf4 MMAs (K = 64 each).
//   warps 2-17  epilogue (both CTAs): drain the CTA's 128 x 256 fp32 rows
//               from TMEM (16 warps, 64 columns each, so the drain that
//               holds up the next tile is short), release them to the MMA
//               issuer with one arrival per CTA, then
//               y = acc * RN32(g_x g_w) + b (the tile's bias read once into
//               shared memory), written as bf16 or fp32 into 64-byte-
//               swizzled staging boxes and stored by TMA.
// The lora-up shares the accumulator with the 4-bit product because
// lora_act arrives pre-divided by g_x g_w.
//
// QKV variant (the FLUX to_qkv module of Nunchaku 4-bit in Diffusers,
// "Quantisierung von Modellen mit strukturellen Umschreibungen": one fused
// operator for the QKV projection, the Q/K normalisation and the rotary
// embedding): Y = [Q | K | V] with sections of 256-column multiples, so a
// tile is all Q, all K or all V.  In Q and K tiles the epilogue normalises
// every 128-column head by its RMS (the head spans the 64 columns of two
// warps of the same lane quarter, which add their sums of squares through
// shared memory), scales by the per-dimension weight and turns the pairs
// (2i, 2i+1) by the row's rotary angle, all in fp32 before the one
// rounding to the output type.
//
// Chained variant (a layer whose output feeds the next W4A4 layer, e.g. the
// FLUX feed-forward's up-projection, GELU and down-projection): the
// epilogue optionally applies the tanh-form GELU before the rounding and
// reduces max |RN(y_stored * 1/lambda')| over its outputs (lambda' the next
// layer's smoothing factors) into one device word, the next layer's
// dynamic tensor-scale amax, with one atomic max per warp.
//
// TMEM columns (same in both CTAs): [0, 256) accumulator (this CTA's 128
// rows), then one scale slot of 48 columns per ring stage: 16 columns of A
// scales (this CTA's rows) and 32 of B scales (all 256 columns; each CTA
// holds a copy), 4 x 32-bit columns per 128 rows per MMA; lane i of every
// 32-lane quarter holds rows i, i+32, i+64, i+96.
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace svdq {
namespace {

constexpr int BM = 256;  // rows of a pair tile (128 per CTA)
constexpr int BN = 256;
constexpr int BK = 256;  // fp4 elements per ring stage (128 bytes per row)
constexpr int kStages = 5;
constexpr int kABytes = 128 * BK / 2;                                  // 16 KB
constexpr int kBBytes = 128 * BK / 2;                                  // 16 KB (this CTA's N half)
constexpr int kSfaBytes = 128 * BK / 16;                               // 2 KB
constexpr int kSfbBytes = 256 * BK / 16;                               // 4 KB (all 256 N)
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;  // 38 KB
constexpr int kEpiWarps = 16;                       // 4 TMEM lane quarters x 4 column quarters
constexpr int kColsPerWarp = BN * 4 / kEpiWarps;    // 64
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColAcc = 0, kColSf = 256, kSfSlotCols = 48;
// one 32-row x 64-byte output box per epilogue warp (64-byte swizzle): the
// ring keeps five stages (190 KB of TMA loads in flight, which the L2 needs
// to deliver a K step per MMA time)
constexpr int kStagingPerWarp = 2048;
constexpr int kStagingOff = kStages * kStageBytes;
constexpr int kBiasOff = kStagingOff + kEpiWarps * kStagingPerWarp;  // 2 x 256 floats
constexpr int kBarOff = kBiasOff + 2 * BN * 4;
constexpr int kGxOff = kBarOff + 192;                      // dynamic variants: RN(g_x g_w)
constexpr int kRedOff = kBarOff + 256;                     // QKV: one float per row of a head pair
constexpr size_t kSmemBytes = kRedOff + 4 * 2 * 32 * 4 + 1024 /*align*/;

static_assert(kStageBytes % 1024 == 0, "stages must keep 1024-byte alignment");
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kColSf + kStages * kSfSlotCols <= kTmemCols, "TMEM budget");

// Instruction descriptors (kind::mxf4nvf4 block-scaled and kind::tf32),
// M = 256 (a CTA pair), N = 256, both operands K-major.
constexpr uint32_t kIdescNvfp4 = (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);
constexpr uint32_t kIdescTf32 =
    (1u << 4) | (2u << 7) | (2u << 10) | (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);

// epilogue variants
constexpr int kModePlain = 0, kModeQkv = 1, kModeChain = 2, kModeChainGelu = 3;

// GELU in its tanh form, 0.5 y (1 + tanh(u)) with u = sqrt(2/pi) (y +
// 0.044715 y^3), through the identity 0.5 (1 + tanh(u)) = 1 / (1 + e^(-2u)):
// y / (1 + 2^z), z = y (c0 + c1 y^2), c0 = -2 log2(e) sqrt(2/pi), c1 =
// 0.044715 c0.  No cancellation for negative y (unlike 1 + tanh), so the
// hardware exp2 and reciprocal keep the relative error near 1e-6.  z is
// clamped so that 1 + 2^z stays finite.
// Two values at once with packed fp32 operations (each lane rounded as
// the scalar form would be).
__device__ __forceinline__ float2 gelu_tanh2(float2 y) {
  const float2 t = __ffma2_rn(__fmul2_rn(y, y), make_float2(-0.10294324f, -0.10294324f),
                              make_float2(-2.3022082f, -2.3022082f));
  float2 z = __fmul2_rn(y, t);
  z.x = fminf(z.x, 120.0f);
  z.y = fminf(z.y, 120.0f);
  float2 e, r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e.x) : "f"(z.x));
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e.y) : "f"(z.y));
  const float2 d = __fadd2_rn(e, make_float2(1.0f, 1.0f));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r.x) : "f"(d.x));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r.y) : "f"(d.y));
  return __fmul2_rn(y, r);
}

struct GemmParams {
  const float* bias;
  void* Y;
  int* status;
  int M, N, K, n_lora;
  float gxgw;
  // dynamic tensor scale: when set, gxgw = RN(RN(*x_amax / 2688) * g_w)
  // (g_x = 1 for a zero amax)
  const float* x_amax;
  float g_w;
  // chained variant: the next layer's 1/lambda (N values, or null) and the
  // word its amax is max-reduced into
  const float* next_il;
  float* next_amax;
  int tma_store;  // Y rows are whole multiples of 16 bytes: store through tm_y
  // QKV attention prologue (the kQkv variant only)
  const float* norm_q;
  const float* norm_k;
  const float* rope_cos;  // 64 x M, frequency-major
  const float* rope_sin;
  float eps;
  int qk_cols;  // columns of Q and K (2 * heads * 128); K starts at qk_cols / 2
};

template <bool kF32Out, int kMode, bool kDyn>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                      const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
                      const __grid_constant__ CUtensorMap tm_la, const __grid_constant__ CUtensorMap tm_lb,
                      const __grid_constant__ CUtensorMap tm_y, const GemmParams p) {
  constexpr bool kQkv = kMode == kModeQkv;
  constexpr bool kChain = kMode >= kModeChain;
  // programmatic dependent launch: the CTA may be resident while the
  // previous kernel drains; every global-memory access comes after this wait
  // (the descriptors are kernel parameters: their fetch may start before it)
  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_sfa);
    prefetch_tmap(&tm_sfb);
  }
  grid_dep_wait();
  if (threadIdx.x == 0) grid_dep_launch();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* bias_s = reinterpret_cast<float*>(smem + kBiasOff);
  float* red_s = reinterpret_cast<float*>(smem + kRedOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs; 1: its peer
  const int pair = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;
  const int num_m = (p.M + BM - 1) / BM;
  const int num_n = (p.N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int k_sub = p.K / 64;           // 64-wide MMA steps along K
  const int num_kb = (k_sub + 3) / 4;   // ring stages per tile for the 4-bit product

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2);  // one arrival per CTA, after all its epilogue warps have drained
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA arrive or TMA completion
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  uint32_t issued_mask = 0, issued_par = 0;  // producer bookkeeping for the teardown drain

  if (warp == 0) {
    // ------------------------------------------------ TMA producer (whole warp)
    int stage = 0;
    uint32_t phase = 0;
    for (int tile = pair; tile < num_tiles; tile += num_pairs) {
      const int mb = tile % num_m, nb = tile / num_m;
      const int m_cta = mb * BM + 128 * static_cast<int>(rank);  // this CTA's A rows
      const int n_cta = nb * BN + 128 * static_cast<int>(rank);  // this CTA's B rows
      for (int j = 0; j < p.n_lora; ++j) {
        if (!mbar_wait_warp(&empty[stage], phase ^ 1, abort_flag)) goto teardown;
        if (elect_one()) {
          uint8_t* st = smem + stage * kStageBytes;
          const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * (kABytes + kBBytes));
          tma_load_2d_pair(st, &tm_la, 32 * j, m_cta, fb);
          tma_load_2d_pair(st + kABytes, &tm_lb, 32 * j, n_cta, fb);
        }
        __syncwarp();
        issued_mask |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        if (++stage == kStages) { stage = 0; phase ^= 1; }
      }
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!mbar_wait_warp(&empty[stage], phase ^ 1, abort_flag)) goto teardown;
        if (elect_one()) {
          uint8_t* st = smem + stage * kStageBytes;
          const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * kStageBytes);
          tma_load_2d_pair(st, &tm_a, kb * 128, m_cta, fb);
          tma_load_2d_pair(st + kABytes, &tm_b, kb * 128, n_cta, fb);
          // scale atoms: rows of 256 bytes, 8 rows = the 4 atoms of this K step
          tma_load_2d_pair(st + kABytes + kBBytes, &tm_sfa, 0, ((m_cta >> 7) * k_sub + 4 * kb) * 2, fb);
          tma_load_2d_pair(st + kABytes + kBBytes + kSfaBytes, &tm_sfb, 0, ((nb * 2) * k_sub + 4 * kb) * 2, fb);
          tma_load_2d_pair(st + kABytes + kBBytes + kSfaBytes + 2048, &tm_sfb, 0,
                           ((nb * 2 + 1) * k_sub + 4 * kb) * 2, fb);
        }
        __syncwarp();
        issued_mask |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        if (++stage == kStages) { stage = 0; phase ^= 1; }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------- MMA issuer (whole warp, first CTA only)
    if (rank == 0) {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      const uint32_t d_acc = tmem + kColAcc;
      for (int tile = pair; tile < num_tiles; tile += num_pairs) {
        if (!mbar_wait_warp(acc_empty, acc_phase ^ 1, abort_flag)) goto teardown;
        tc_fence_after();
        uint32_t accumulate = 0;
        for (int j = 0; j < p.n_lora; ++j) {
          if (!mbar_wait_warp(&full[stage], phase, abort_flag)) goto teardown;
          if (elect_one()) {
            const uint32_t sa = smem_u32(smem + stage * kStageBytes);
            const uint64_t da = sdesc_sw128(sa), db = sdesc_sw128(sa + kABytes);
#pragma unroll
            for (int k = 0; k < 4; ++k)  // 4 x K=8 tf32 steps of 32 bytes
              mma_tf32_pair(d_acc, da + 2 * k, db + 2 * k, kIdescTf32, (accumulate | k) ? 1u : 0u);
            tc_commit_pair(&empty[stage], 0x3);
          }
          __syncwarp();
          accumulate = 1;
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        for (int kb = 0; kb < num_kb; ++kb) {
          const int nsub = min(4, k_sub - 4 * kb);
          if (!mbar_wait_warp(&full[stage], phase, abort_flag)) goto teardown;
          if (elect_one()) {
            const uint32_t sa = smem_u32(smem + stage * kStageBytes);
            const uint32_t s_sfa = sa + kABytes + kBBytes;
            const uint32_t s_sfb = s_sfa + kSfaBytes;
            const uint32_t t_sfa = tmem + kColSf + stage * kSfSlotCols;
            const uint32_t t_sfb = t_sfa + 16;
            const uint64_t da = sdesc_sw128(sa), db = sdesc_sw128(sa + kABytes);
            // scale copies and MMAs alternate so that each copy overlaps the
            // MMA issued just before it in the tensor pipe's in-order stream
            for (int k = 0; k < nsub; ++k) {  // K=64 fp4 steps of 32 bytes
              tc_cp_32x128b_warpx4_pair(t_sfa + 4 * k, sdesc_rows16(s_sfa + 512 * k));
              tc_cp_32x128b_warpx4_pair(t_sfb + 8 * k, sdesc_rows16(s_sfb + 512 * k));
              tc_cp_32x128b_warpx4_pair(t_sfb + 8 * k + 4, sdesc_rows16(s_sfb + 2048 + 512 * k));
              mma_nvfp4_pair(d_acc, da + 2 * k, db + 2 * k, kIdescNvfp4, t_sfa + 4 * k, t_sfb + 8 * k,
                             (accumulate | k) ? 1u : 0u);
            }
            tc_commit_pair(&empty[stage], 0x3);
          }
          __syncwarp();
          accumulate = 1;
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        if (elect_one()) tc_commit_pair(acc_full, 0x3);
        __syncwarp();
        acc_phase ^= 1;
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue
    // Warp (quarter, part) owns rows quarter*32 .. +31 (its TMEM lane
    // quarter) and columns part*64 .. +63 of the CTA's 128 x 256 tile.
    const int quarter = warp & 3;
    const int part = (warp - 2) >> 2;
    const int et = (warp - 2) * 32 + lane;  // 0..511 over the epilogue warps
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
    uint8_t* const stg = smem + kStagingOff + (warp - 2) * kStagingPerWarp;  // a 128-byte-swizzled box
    // RN(g_x g_w): as given (a kernel parameter, no register), or from the
    // device amax, published in shared memory by the first barrier and
    // re-read where it is used (the epilogue sits at the register limit)
    float gxgw = p.gxgw;
    const uint32_t gx_s = smem_u32(smem + kGxOff);
    if constexpr (kDyn) {
      const float a = *p.x_amax;
      gxgw = __fmul_rn(a == 0.0f ? 1.0f : __fdiv_rn(a, 2688.0f), p.g_w);
      if (et == 0) *reinterpret_cast<float*>(smem + kGxOff) = gxgw;
    }
    float amax_next = 0.0f;  // chained variant: max |y_stored / lambda'| over this thread's rows < M
    uint32_t acc_phase = 0;
    int tcount = 0;
    for (int tile = pair; tile < num_tiles; tile += num_pairs, ++tcount) {
      const int m0 = (tile % num_m) * BM + 128 * static_cast<int>(rank), n0 = (tile / num_m) * BN;
      float* bias_t;
      if constexpr (!kChain) {
        // the tile's 256 bias values, once, into this tile's half of the double buffer
        bias_t = bias_s + (tcount & 1) * BN;
        if (et < BN) bias_t[et] = n0 + et < p.N ? __ldg(p.bias + n0 + et) : 0.0f;
        named_bar_sync(1, 32 * kEpiWarps);
      } else {
        // single buffers of the tile's bias and next-layer 1/lambda: written
        // once every epilogue warp is past the previous tile (barrier 1),
        // read after barrier 2
        bias_t = bias_s;
        float bz = 0.0f, lz = 0.0f;
        if (et < BN && n0 + et < p.N) {
          bz = __ldg(p.bias + n0 + et);
          if (p.next_il != nullptr) lz = __ldg(p.next_il + n0 + et);
        }
        named_bar_sync(1, 32 * kEpiWarps);
        if (et < BN) {
          bias_s[et] = bz;
          bias_s[BN + et] = lz;
        }
      }
      if (!mbar_wait(acc_full, acc_phase, abort_flag)) break;
      acc_phase ^= 1;
      tc_fence_after();
      uint32_t v[kColsPerWarp];  // this warp's 32 rows x 64 columns, one load
      tmem_ld64(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + kColAcc + part * kColsPerWarp, v);
      tmem_ld_wait();
      tc_fence_before();
      // once every epilogue warp of this CTA holds its columns, one arrival
      // (local or remote) frees the accumulator for the next tile
      named_bar_sync(2, 32 * kEpiWarps);
      if (warp == 2 && lane == 0) {
        // the loads above have completed (wait::ld), so the signal orders no
        // memory access: the first CTA arrives locally, its peer remotely
        // without a cluster-scope release (which cost ~1000 cycles per tile)
        if (rank == 0) mbar_arrive(acc_empty);
        else mbar_arrive_cluster_relaxed(acc_empty_leader);
      }

      const int row = m0 + quarter * 32 + lane;
      const float* bb = bias_t + part * kColsPerWarp;
      if constexpr (kQkv) {
        // y = acc * RN32(g_x g_w) + b in place, then in Q / K tiles the
        // head's RMS normalisation and rotary embedding (n0 is CTA-uniform,
        // so every epilogue warp takes the same barriers)
#pragma unroll
        for (int c = 0; c < kColsPerWarp; ++c)
          v[c] = __float_as_uint(__fadd_rn(__fmul_rn(__uint_as_float(v[c]), gxgw), bb[c]));
        if (n0 < p.qk_cols) {
          const int hcol = (part & 1) * kColsPerWarp;  // first column of this half within its head
          // rotary tables are frequency-major (pair i of token m at i * M + m):
          // the warp's 32 rows of one frequency are one line.  The first
          // group of four pairs is requested before the sum exchange, so
          // that its L2 latency overlaps the barriers.
          const bool in_rows = row < p.M;
          const size_t trow = static_cast<size_t>(hcol / 2) * p.M + (in_rows ? row : 0);
          const float* ct = p.rope_cos + trow;
          const float* st = p.rope_sin + trow;
          float c0[4], s0[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            c0[j] = in_rows ? __ldg(ct + static_cast<size_t>(j) * p.M) : 1.0f;
            s0[j] = in_rows ? __ldg(st + static_cast<size_t>(j) * p.M) : 0.0f;
          }
          float ss = 0.0f;
#pragma unroll
          for (int c = 0; c < kColsPerWarp; ++c) ss = __fmaf_rn(__uint_as_float(v[c]), __uint_as_float(v[c]), ss);
          // the head = parts (2h, 2h+1) of this quarter: the odd half posts
          // its sum, the even half adds it to its own (even half first) and
          // posts the head's total, which both then read.  The slot is next
          // written after the next tile's first barrier, which every reader
          // of this tile has passed.
          float* slot = red_s + (quarter * 2 + (part >> 1)) * 32 + lane;
          if (part & 1) *slot = ss;
          named_bar_sync(3, 32 * kEpiWarps);
          if (!(part & 1)) *slot = __fadd_rn(ss, *slot);
          named_bar_sync(3, 32 * kEpiWarps);
          const float r = rsqrtf(__fmaf_rn(*slot, 1.0f / 128.0f, p.eps));
          const float4* wn = reinterpret_cast<const float4*>((n0 < p.qk_cols / 2 ? p.norm_q : p.norm_k) + hcol);
#pragma unroll
          for (int q4 = 0; q4 < kColsPerWarp / 8; ++q4) {  // four pairs per step
            float cc[4], sc[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              cc[j] = q4 == 0 ? c0[j] : (in_rows ? __ldg(ct + static_cast<size_t>(4 * q4 + j) * p.M) : 1.0f);
              sc[j] = q4 == 0 ? s0[j] : (in_rows ? __ldg(st + static_cast<size_t>(4 * q4 + j) * p.M) : 0.0f);
            }
            const float4 w0 = __ldg(wn + 2 * q4), w1 = __ldg(wn + 2 * q4 + 1);
            // the head's scale folded into the weights: (y r) w = y (r w)
            const float rw[8] = {__fmul_rn(r, w0.x), __fmul_rn(r, w0.y), __fmul_rn(r, w0.z), __fmul_rn(r, w0.w),
                                 __fmul_rn(r, w1.x), __fmul_rn(r, w1.y), __fmul_rn(r, w1.z), __fmul_rn(r, w1.w)};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int c = 8 * q4 + 2 * j;
              const float a = __fmul_rn(__uint_as_float(v[c]), rw[2 * j]);
              const float b = __fmul_rn(__uint_as_float(v[c + 1]), rw[2 * j + 1]);
              v[c] = __float_as_uint(__fmaf_rn(a, cc[j], -__fmul_rn(b, sc[j])));
              v[c + 1] = __float_as_uint(__fmaf_rn(a, sc[j], __fmul_rn(b, cc[j])));
            }
          }
        }
      }
      // the dynamic variants also compute y in place first, so that the
      // scale's register is free in the store loop
      if constexpr (kMode == kModeChainGelu) {
        const float g = ld_shared_f32_fresh(gx_s);
        const float2 g2 = make_float2(g, g);
#pragma unroll
        for (int c = 0; c < kColsPerWarp; c += 2) {
          const float2 b2 = *reinterpret_cast<const float2*>(bb + c);
          const float2 y = __fadd2_rn(__fmul2_rn(make_float2(__uint_as_float(v[c]), __uint_as_float(v[c + 1])), g2), b2);
          const float2 o = gelu_tanh2(y);
          v[c] = __float_as_uint(o.x);
          v[c + 1] = __float_as_uint(o.y);
        }
      }
      // the value stored for column `col` of the warp's 64
      auto yv = [&](int col, float g) -> float {
        if constexpr (kQkv || kMode == kModeChainGelu) return __uint_as_float(v[col]);
        else return __fadd_rn(__fmul_rn(__uint_as_float(v[col]), g), bb[col]);
      };
      // the scale for a group of columns: the parameter, or a fresh shared load
      auto scale = [&]() -> float {
        if constexpr (kDyn && !kQkv && kMode != kModeChainGelu) return ld_shared_f32_fresh(gx_s);
        else return gxgw;
      };
      // chained variant: max |y_stored / lambda'| over the rows < M (columns
      // past N carry 1/lambda' = 0); the 1/lambda' buffer follows the bias
      const bool row_ok = row < p.M;
      auto track = [&](float ys, int col) {
        if constexpr (kChain)
          if (row_ok) amax_next = fmaxf(amax_next, fabsf(__fmul_rn(ys, bb[BN + col])));
      };
      if (p.tma_store) {
        // y rows into a 64-byte-wide swizzled box (32 rows; row r's 16-byte
        // unit u at r * 64 + ((u ^ ((r >> 1) & 3)) << 4)), then a TMA store
        // per box; rows past M / columns past N are clipped
        constexpr int kColsPerBox = kF32Out ? 16 : 32;
        constexpr int kPasses = kColsPerWarp / kColsPerBox;
#pragma unroll
        for (int pass = 0; pass < kPasses; ++pass) {
          if (lane == 0) bulk_wait_read_all();  // the previous store no longer reads the box
          __syncwarp();
#pragma unroll
          for (int j = 0; j < kColsPerBox; j += 4) {
            const int col = pass * kColsPerBox + j;  // within the warp's columns
            const float g = scale();
            const float y0 = yv(col, g), y1 = yv(col + 1, g), y2 = yv(col + 2, g), y3 = yv(col + 3, g);
            const int byte = j * (kF32Out ? 4 : 2);  // within the box's 64-byte row
            uint8_t* line = stg + lane * 64;
            const int unit = (byte >> 4) ^ ((lane >> 1) & 3);
            if constexpr (kF32Out) {
              *reinterpret_cast<float4*>(line + (unit << 4)) = make_float4(y0, y1, y2, y3);
              track(y0, col);
              track(y1, col + 1);
              track(y2, col + 2);
              track(y3, col + 3);
            } else {
              __nv_bfloat162 h0 = __floats2bfloat162_rn(y0, y1), h1 = __floats2bfloat162_rn(y2, y3);
              *reinterpret_cast<uint2*>(line + (unit << 4) + (byte & 15)) =
                  make_uint2(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1));
              track(__low2float(h0), col);
              track(__high2float(h0), col + 1);
              track(__low2float(h1), col + 2);
              track(__high2float(h1), col + 3);
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tm_y, stg, n0 + part * kColsPerWarp + pass * kColsPerBox, m0 + quarter * 32);
            bulk_commit_group();
          }
        }
      } else if (row < p.M) {
        // rows whose byte length is not a multiple of 16: plain stores
#pragma unroll
        for (int col = 0; col < kColsPerWarp; ++col) {
          const int n = n0 + part * kColsPerWarp + col;
          if (n < p.N) {
            const float y = yv(col, scale());
            if constexpr (kF32Out) {
              static_cast<float*>(p.Y)[static_cast<size_t>(row) * p.N + n] = y;
              track(y, col);
            } else {
              const __nv_bfloat16 h = __float2bfloat16_rn(y);
              static_cast<__nv_bfloat16*>(p.Y)[static_cast<size_t>(row) * p.N + n] = h;
              track(__bfloat162float(h), col);
            }
          }
        }
      }
    }
    if constexpr (kChain) {
      // one atomic max per warp: non-negative floats order as their bit patterns
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax_next = fmaxf(amax_next, __shfl_xor_sync(0xffffffffu, amax_next, o));
      if (lane == 0 && p.next_amax != nullptr && amax_next > 0.0f)
        atomicMax(reinterpret_cast<unsigned int*>(p.next_amax), __float_as_uint(amax_next));
    }
    if (lane == 0) bulk_wait_all();  // every store of this warp has landed
  }

teardown:
  __syncthreads();
  if (rank == 0 && warp == 0 && lane == 0) {
    // every TMA copy of the pair completes on the first CTA's barriers:
    // they must all have landed before either CTA releases its memory
    for (int s = 0; s < kStages; ++s)
      if (issued_mask & (1u << s)) mbar_wait_limited(&full[s], (issued_par >> s) & 1u, 200000000ull);
  }
  if (rank == 0 && warp == 1) {
    // the lane that issued the MMAs commits: arrives once all of them have finished
    if (elect_one()) {
      tc_commit_pair(drain, 0x1);
      mbar_wait_limited(drain, 0, 200000000ull);
    }
    __syncwarp();
  }
  if (threadIdx.x == 0 && *abort_flag) atomicExch(p.status, static_cast<int>(SVDQ_ERR_TIMEOUT));
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_gemm_nvfp4(const svdq_weights* w, const uint8_t* qx, const uint8_t* sx, float g_x,
                              const float* x_amax, const float* lora_act, int M, void* Y, int out_dtype,
                              const svdq_qkv_prologue* pro, const svdq_epilogue_next* epi, cudaStream_t s) {
  const int K = w->desc.K, N = w->desc.N;
  const int64_t m_pad = m_pad_of(M);
  CUtensorMap tm_a, tm_sfa, tm_la;
  if (!encode_tmap_2d(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, qx, K / 2, M, K / 2, 128, 128))
    return cudaErrorInvalidValue;
  if (!encode_tmap_2d(&tm_sfa, CU_TENSOR_MAP_DATA_TYPE_UINT8, sx, 256, nvfp4_scale_bytes(m_pad, K) / 256, 256, 256, 8,
                      false))
    return cudaErrorInvalidValue;
  if (w->rank_pad > 0) {
    if (!encode_tmap_2d(&tm_la, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, lora_act, w->rank_pad, M,
                        static_cast<uint64_t>(w->rank_pad) * 4, 32, 128))
      return cudaErrorInvalidValue;
  } else {
    tm_la = tm_a;  // unused when there is no low-rank branch
  }
  GemmParams p;
  p.bias = w->bias;
  p.Y = Y;
  p.status = w->status;
  p.M = M;
  p.N = N;
  p.K = K;
  p.n_lora = w->rank_pad / 32;
  p.gxgw = g_x * w->g_w;  // RN32(g_x * g_w)
  p.norm_q = pro ? pro->norm_q : nullptr;
  p.norm_k = pro ? pro->norm_k : nullptr;
  p.rope_cos = pro ? pro->rope_cos : nullptr;
  p.rope_sin = pro ? pro->rope_sin : nullptr;
  p.eps = pro ? pro->eps : 0.0f;
  p.qk_cols = pro ? 2 * pro->heads * pro->head_dim : 0;
  p.x_amax = x_amax;
  p.g_w = w->g_w;
  p.next_il = epi ? epi->next_inv_lambda : nullptr;
  p.next_amax = epi ? epi->next_amax : nullptr;
  // Y through TMA stores when its rows are whole multiples of 16 bytes
  const bool f32 = out_dtype == SVDQ_OUT_F32;
  const uint64_t row_bytes = static_cast<uint64_t>(N) * (f32 ? 4 : 2);
  CUtensorMap tm_y = tm_a;
  p.tma_store = row_bytes % 16 == 0 &&
                encode_tmap_2d_swizzle(&tm_y, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y,
                                       N, M, row_bytes, f32 ? 16 : 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
  const int tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int pairs = std::min(tiles, num_sms(w->device) / 2);
  const int mode = pro ? kModeQkv
                   : !epi ? kModePlain
                   : epi->activation == SVDQ_ACT_GELU_TANH ? kModeChainGelu
                                                          : kModeChain;
  // the chained variants are reached through the dynamic entry points only
  const bool dyn = x_amax != nullptr;
  decltype(&gemm_nvfp4_kernel<false, kModePlain, false>) kern;
  switch (mode) {
    case kModeQkv:
      kern = dyn ? (f32 ? gemm_nvfp4_kernel<true, kModeQkv, true> : gemm_nvfp4_kernel<false, kModeQkv, true>)
                 : (f32 ? gemm_nvfp4_kernel<true, kModeQkv, false> : gemm_nvfp4_kernel<false, kModeQkv, false>);
      break;
    case kModeChain:
      kern = f32 ? gemm_nvfp4_kernel<true, kModeChain, true> : gemm_nvfp4_kernel<false, kModeChain, true>;
      break;
    case kModeChainGelu:
      kern = f32 ? gemm_nvfp4_kernel<true, kModeChainGelu, true> : gemm_nvfp4_kernel<false, kModeChainGelu, true>;
      break;
    default:
      kern = dyn ? (f32 ? gemm_nvfp4_kernel<true, kModePlain, true> : gemm_nvfp4_kernel<false, kModePlain, true>)
                 : (f32 ? gemm_nvfp4_kernel<true, kModePlain, false> : gemm_nvfp4_kernel<false, kModePlain, false>);
  }
  if (mode >= kModeChain && !dyn) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, tm_a, w->tm_qw, tm_sfa, w->tm_sw, tm_la, w->tm_l2, tm_y, p);
}

}  // namespace svdq
