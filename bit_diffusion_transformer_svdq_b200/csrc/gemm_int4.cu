// INT4 (group 64) variant of the 4-bit GEMM with the low-rank up-projection
// fused in: Y = sum_g s_x[m,g] s_w[n,g] (sum_{k in g} qx qw) + lora_act L2^T + b.
// tcgen05 has no 4-bit integer kind, so the codes go to the tensor core as
// 8-bit operands: E4M3 bytes, which hold every integer in [-8, 7] exactly,
// multiplied by kind::f8f6f4 MMAs into fp32 TMEM accumulators.  Every
// product is an integer of magnitude at most 64 and a group's sum P at most
// 4096, so the accumulator holds each group's integer dot product exactly.
// The scales change with every 64-group, so each group's product leaves TMEM
// and is added into an fp32 accumulator held in registers.  The tensor core
// also forms the group's scale products C[m,n] = s_x[m,g] s_w[n,g]: one
// kind::f16 MMA whose operands are zero but for their first K row (s_x and
// s_w, both fp16), which gives the 22-bit products exactly.  The epilogue
// then takes one FMA per element and group, acc = RN(P C + acc): the same
// single rounding as acc = RN(RN(P s_w) s_x + acc), since P s_w (at most
// 13 x 11 significant bits) is exact in fp32.
//
// sm_100a design, one CTA per 128 x 128 output tile (persistent over the
// tile list):
//   warp 0      TMA producer: per ring stage (128 K = two groups) the
//               activation codes as E4M3 bytes (the copy the quantiser writes
//               beside the packed codes) and the prepared E4M3 weight codes,
//               128 rows x 128 B each, 128-byte swizzled; per tile one stage
//               of lora_act / L2 (fp32).
//   warp 18     scale producer: per group the tile's 128 fp16 s_x and 128
//               fp16 s_w into the first K row of a scale slot (four 128-byte
//               bulk copies), eight slots ahead of the MMAs.
//   warps 1, 19 MMA issuers (warp 1 also owns TMEM), one per buffer: for
//               the groups whose buffer use is even (warp 1) or odd (warp 19)
//               two kind::f8f6f4 MMAs (K = 32) into P and one kind::f16 MMA
//               (K = 16, MN-major operands from the scale slot) into C, the
//               buffer's 256 columns; per tile four kind::tf32 MMAs of the
//               lora-up into the next use's P, as one more "group".
//   warps 2-17  epilogue: warp w owns rows 32 (w % 4) .. + 31 (its TMEM
//               lane quarter) and columns 32 ((w - 2) / 4) .. + 31; per group
//               it loads P and C in two halves of 16 columns, frees the
//               buffer and adds P C into its fp32 accumulator with packed
//               two-wide FMAs.  Finally y = acc + b is stored; the QKV variant
//               first applies the attention prologue (per 128-column head of
//               Q and K: RMS normalisation, weight, rotary embedding), the
//               four column slices of a row adding their sums of squares
//               through shared memory.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace svdq {
namespace {

constexpr int kTileM = 128, kTileN = 128;
constexpr int kI4Stages = 5;
constexpr int kA8Bytes = kTileM * 128;   // activation codes of a stage (E4M3): 128 K per row
constexpr int kB8Bytes = kTileN * 128;   // prepared weight codes (E4M3)
constexpr int kI4StageBytes = kA8Bytes + kB8Bytes;  // 32 KB
constexpr int kI4EpiWarps = 16;  // 4 lane quarters x 4 column slices of 32
constexpr int kScaleWarp = 2 + kI4EpiWarps;
constexpr int kMma2Warp = 3 + kI4EpiWarps;  // the second MMA issuer
constexpr int kI4Threads = 32 * (4 + kI4EpiWarps);
constexpr int kAccBufs = 2;      // group buffers of 256 TMEM columns: P (128) then C (128)
constexpr uint32_t kI4TmemCols = 256 * kAccBufs;
// Scale slots: the two operands of a group's C MMA, each an MN-major
// 128-byte-swizzled tile of two 1 KB atoms (64 fp16 along M or N x K rows
// 0-7); only row 0 of each atom is ever written (the group's scales), rows
// 1-7 stay zero, and K rows 8-15 of every operand are one shared 2 KB block
// of zeros (reached through the descriptor's K-group stride).
constexpr int kScaleSlots = 8;
constexpr int kSlotBytes = 4096;  // s_x operand (2 KB), then s_w operand (2 KB)
constexpr int kScaleOff = kI4Stages * kI4StageBytes;
constexpr int kZeroOff = kScaleOff + kScaleSlots * kSlotBytes;
constexpr int kI4BarOff = kZeroOff + 2048;
constexpr int kI4RedOff = kI4BarOff + 512;  // QKV: one float per row and column slice (16 x 32)
constexpr size_t kI4Smem = kI4RedOff + kI4EpiWarps * 32 * 4 + 1024 /*align*/;
static_assert(kI4StageBytes % 1024 == 0 && kScaleOff % 1024 == 0 && kZeroOff % 1024 == 0, "1 KB atoms");
static_assert(kI4Smem <= 232448, "shared memory budget");

// kind::f8f6f4: fp32 D, E4M3 A and B, K-major, N = 128, M = 128.
constexpr uint32_t kIdescF8 = (1u << 4) | (uint32_t(kTileN >> 3) << 17) | (uint32_t(kTileM >> 4) << 24);
// kind::f16: fp32 D, fp16 A and B, both MN-major, N = 128, M = 128.
constexpr uint32_t kIdescScale =
    (1u << 4) | (1u << 15) | (1u << 16) | (uint32_t(kTileN >> 3) << 17) | (uint32_t(kTileM >> 4) << 24);
// kind::tf32: fp32 D, tf32 A and B, K-major, N = 128, M = 128.
constexpr uint32_t kIdescTf32x = (1u << 4) | (2u << 7) | (2u << 10) | (uint32_t(kTileN >> 3) << 17) | (uint32_t(kTileM >> 4) << 24);

struct I4Params {
  const __half* sx;   // [K/64][m_pad]
  const __half* sw;   // [K/64][n_pad]
  const float* bias;
  void* Y;
  int* status;
  int M, N, K, m_pad, n_lora;
  int64_t n_pad;
  // QKV attention prologue (the kQkv variant only); a 128-column tile is
  // one head of Q, K or V
  const float* norm_q;
  const float* norm_k;
  const float* rope_cos;  // 64 x M, frequency-major
  const float* rope_sin;
  float eps;
  int qk_cols;  // 2 * heads * 128; K starts at qk_cols / 2
};

template <bool kF32Out, bool kQkv>
__global__ void __launch_bounds__(kI4Threads, 1)
    gemm_int4_kernel(const __grid_constant__ CUtensorMap tm_a8, const __grid_constant__ CUtensorMap tm_b8,
                     const __grid_constant__ CUtensorMap tm_la, const __grid_constant__ CUtensorMap tm_lb,
                     const I4Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* red_s = reinterpret_cast<float*>(smem + kI4RedOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kI4BarOff);
  uint64_t* empty = full + kI4Stages;          // MMAs done with the stage
  uint64_t* acc_full = empty + kI4Stages;      // [kAccBufs]
  uint64_t* acc_empty = acc_full + kAccBufs;   // [kAccBufs], one arrival per epilogue warp
  uint64_t* sc_full = acc_empty + kAccBufs;    // [kScaleSlots], bulk copies of a group's scales
  uint64_t* sc_empty = sc_full + kScaleSlots;  // [kScaleSlots], the C MMA that read the slot is done
  uint64_t* drain = sc_empty + kScaleSlots;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_m = (p.M + kTileM - 1) / kTileM;
  const int num_n = (p.N + kTileN - 1) / kTileN;
  const int num_tiles = num_m * num_n;
  const int groups = p.K / 64;
  const int num_kb = (groups + 1) / 2;  // ring stages per tile (the last may hold one group)

  // the scale slots and the shared K rows 8-15 start (and, but for the
  // scale rows the copies write, stay) zero
  for (int o = threadIdx.x * 16; o < kScaleSlots * kSlotBytes + 2048; o += kI4Threads * 16)
    *reinterpret_cast<uint4*>(smem + kScaleOff + o) = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kI4Stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 2);  // both MMA issuers
    }
    for (int b = 0; b < kAccBufs; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kI4EpiWarps);
    }
    for (int b = 0; b < kScaleSlots; ++b) {
      mbar_init(&sc_full[b], 1);
      mbar_init(&sc_empty[b], 1);
    }
    mbar_init(drain, 2);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kI4TmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // programmatic dependent launch: the setup above may overlap the previous
  // kernel; every global-memory access comes after this wait (the
  // descriptors are kernel parameters: their fetch may start before it)
  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_a8);
    prefetch_tmap(&tm_b8);
  }
  grid_dep_wait();
  if (threadIdx.x == 0) grid_dep_launch();
  const uint32_t tmem = *tmem_slot;
  uint32_t issued_mask = 0, issued_par = 0;
  uint32_t sc_mask = 0, sc_par = 0;  // scale slots issued (teardown drain)

  if (warp == 0) {
    // ------------------------------------------------ TMA producer (whole warp)
    int stage = 0;
    uint32_t phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int m0 = (tile % num_m) * kTileM, n0 = (tile / num_m) * kTileN;
      for (int kb = 0; kb < num_kb + p.n_lora; ++kb) {
        if (!mbar_wait_warp(&empty[stage], phase ^ 1, abort_flag)) goto teardown;
        if (elect_one()) {
          uint8_t* st = smem + stage * kI4StageBytes;
          mbar_arrive_expect_tx(&full[stage], kA8Bytes + kB8Bytes);
          if (kb < num_kb) {  // activation and weight codes (E4M3)
            tma_load_2d(st, &tm_a8, kb * 128, m0, &full[stage]);
            tma_load_2d(st + kA8Bytes, &tm_b8, kb * 128, n0, &full[stage]);
          } else {  // lora_act and L2 columns 32 j .. 32 j + 31 (fp32)
            const int j = kb - num_kb;
            tma_load_2d(st, &tm_la, 32 * j, m0, &full[stage]);
            tma_load_2d(st + kA8Bytes, &tm_lb, 32 * j, n0, &full[stage]);
          }
        }
        __syncwarp();
        issued_mask |= 1u << stage;
        issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
        if (++stage == kI4Stages) { stage = 0; phase ^= 1; }
      }
    }
  } else if (warp == kScaleWarp) {
    // ------------------------------------------ scale producer (whole warp)
    // one slot per group: row 0 of the two atoms of each operand (64 fp16 =
    // 128 bytes each)
    uint32_t sc_count = 0;  // scale slots filled so far
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int m0 = (tile % num_m) * kTileM, n0 = (tile / num_m) * kTileN;
      for (int g = 0; g < groups; ++g, ++sc_count) {
        const uint32_t ss = sc_count % kScaleSlots;
        const uint32_t sp = (sc_count / kScaleSlots) & 1;
        if (!mbar_wait_warp(&sc_empty[ss], sp ^ 1, abort_flag)) goto teardown;
        if (elect_one()) {
          uint8_t* dst = smem + kScaleOff + ss * kSlotBytes;
          const __half* sxg = p.sx + static_cast<size_t>(g) * p.m_pad + m0;
          const __half* swg = p.sw + static_cast<size_t>(g) * p.n_pad + n0;
          mbar_arrive_expect_tx(&sc_full[ss], 512);
          bulk_load(dst, sxg, 128, &sc_full[ss]);
          bulk_load(dst + 1024, sxg + 64, 128, &sc_full[ss]);
          bulk_load(dst + 2048, swg, 128, &sc_full[ss]);
          bulk_load(dst + 3072, swg + 64, 128, &sc_full[ss]);
        }
        __syncwarp();
        sc_mask |= 1u << ss;
        sc_par = (sc_par & ~(1u << ss)) | (sp << ss);
      }
    }
  } else if (warp == 1 || warp == kMma2Warp) {
    // -------------------------------------------- MMA issuers (whole warps)
    // Warp 1 issues the buffer uses of even count (TMEM buffer 0), warp 19
    // those of odd count (buffer 1): two independent instruction streams
    // feed the tensor core.  Both walk every ring stage, waiting until it
    // is full and then releasing it (empty counts both warps); a stage's
    // group is multiplied by the warp that owns its use.
    const uint32_t par = warp == 1 ? 0u : 1u;
    const uint32_t d = tmem + par * 256;
    int stage = 0;
    uint32_t phase = 0;
    uint32_t use = 0;     // buffer uses so far, both warps': use u goes to buffer u % 2
    uint32_t sc_use = 0;  // scale slots consumed so far, both warps'
    // Descriptors move with the slot or stage in their address field only
    // (and, for the scale operands, the K-group stride to the shared zero
    // block, which shrinks by as much): one add each.
    const uint32_t sx0 = smem_u32(smem + kScaleOff), zero_blk = smem_u32(smem + kZeroOff);
    const uint64_t dsx0 = sdesc_sw128_mn(sx0, 1024, zero_blk - sx0);
    constexpr uint64_t kSlotStep = (uint64_t(kSlotBytes) >> 4) - ((uint64_t(kSlotBytes) >> 4) << 32);
    constexpr uint64_t kSwStep = (uint64_t(2048) >> 4) - ((uint64_t(2048) >> 4) << 32);
    const uint64_t da0 = sdesc_sw128(smem_u32(smem));
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!mbar_wait_warp(&full[stage], phase, abort_flag)) goto teardown;
        const int ng = min(2, groups - 2 * kb);
        const int gi = static_cast<int>((par ^ use) & 1u);  // the stage's group whose use is this warp's
        if (gi < ng) {
          const uint32_t ss = (sc_use + gi) % kScaleSlots;
          if (!mbar_wait_warp(&sc_full[ss], ((sc_use + gi) / kScaleSlots) & 1, abort_flag) ||
              !mbar_wait_warp(&acc_empty[par], (((use + gi) >> 1) & 1) ^ 1, abort_flag))
            goto teardown;
          tc_fence_after();
          if (elect_one()) {
            const uint64_t da = da0 + static_cast<uint64_t>(stage) * (kI4StageBytes >> 4), db = da + (kA8Bytes >> 4);
            const uint64_t dsx = dsx0 + ss * kSlotStep;
#pragma unroll
            for (int k = 0; k < 2; ++k)  // K = 32 E4M3 (32 bytes) per MMA
              mma_f8(d, da + 4 * gi + 2 * k, db + 4 * gi + 2 * k, kIdescF8, k ? 1u : 0u);
            // C = s_x s_w^T: MN-major operands, atoms 1 KB apart along M / N,
            // K rows 8-15 in the shared zero block
            mma_bf16(d + 128, dsx, dsx + kSwStep, kIdescScale, 0u);
            tc_commit(&acc_full[par]);
            tc_commit(&sc_empty[ss]);
            tc_commit(&empty[stage]);
          }
          __syncwarp();
        } else {
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[stage]);
        }
        use += ng;
        sc_use += ng;
        if (++stage == kI4Stages) { stage = 0; phase ^= 1; }
      }
      if (p.n_lora > 0) {  // the lora-up as one more buffer use (P only), of scale 1
        const bool own = (use & 1u) == par;
        if (own && !mbar_wait_warp(&acc_empty[par], ((use >> 1) & 1) ^ 1, abort_flag)) goto teardown;
        for (int j = 0; j < p.n_lora; ++j) {
          if (!mbar_wait_warp(&full[stage], phase, abort_flag)) goto teardown;
          if (own) {
            tc_fence_after();
            if (elect_one()) {
              const uint64_t da = da0 + static_cast<uint64_t>(stage) * (kI4StageBytes >> 4), db = da + (kA8Bytes >> 4);
#pragma unroll
              for (int k = 0; k < 4; ++k)  // K = 8 tf32 (32 bytes) per MMA
                mma_tf32(d, da + 2 * k, db + 2 * k, kIdescTf32x, (j | k) ? 1u : 0u);
              tc_commit(&empty[stage]);
            }
            __syncwarp();
          } else {
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
          }
          if (++stage == kI4Stages) { stage = 0; phase ^= 1; }
        }
        if (own) {
          if (elect_one()) tc_commit(&acc_full[par]);
          __syncwarp();
        }
        ++use;
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue
    // warp w = 2..17 owns rows 32 (w % 4) .. + 31 (its TMEM lane quarter)
    // and columns 32 ((w - 2) / 4) .. + 31.  Per group it reads its 32
    // products P (fp32: exact integers) and scale products C in two halves,
    // frees the buffer (one arrival per warp) and adds RN(P C + acc) into
    // its fp32 accumulator in registers: the warps never wait for one
    // another.  A warp reaches only the TMEM lanes of its rank in its
    // warpgroup (warp % 4); the four warps 2 + 4c .. 5 + 4c cover the four
    // quarters.
    const int q4 = warp & 3;
    const int cs = (warp - 2) >> 2;         // column slice
    const int r = 32 * q4 + lane;           // row within the tile
    const uint32_t tq = tmem + (static_cast<uint32_t>(32 * q4) << 16) + 32 * cs;
    uint32_t gcount = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
      const int m0 = (tile % num_m) * kTileM, n0 = (tile / num_m) * kTileN;
      const int row = m0 + r;
      const int nc = n0 + 32 * cs;  // first column of this warp
      float acc[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) acc[c] = 0.0f;
      const int uses = groups + (p.n_lora > 0 ? 1 : 0);
      for (int g = 0; g < uses; ++g, ++gcount) {
        const uint32_t buf = gcount % kAccBufs;
        if (!mbar_wait_sleep(&acc_full[buf], (gcount / kAccBufs) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tb = tq + buf * 256;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t P[16], C[16];
          tmem_ld16x2_wait(tb + 16 * h, tb + 128 + 16 * h, P, C);  // C is not read for the lora-up
          if (h == 1) {  // both halves are in registers: free the buffer
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
          }
          if (g < groups) {
#pragma unroll
            for (int c = 0; c < 16; c += 2) {
              const float2 a = __ffma2_rn(make_float2(__uint_as_float(P[c]), __uint_as_float(P[c + 1])),
                                          make_float2(__uint_as_float(C[c]), __uint_as_float(C[c + 1])),
                                          make_float2(acc[16 * h + c], acc[16 * h + c + 1]));
              acc[16 * h + c] = a.x;
              acc[16 * h + c + 1] = a.y;
            }
          } else {  // the lora-up, fp32
#pragma unroll
            for (int c = 0; c < 16; ++c) acc[16 * h + c] = __fadd_rn(acc[16 * h + c], __uint_as_float(P[c]));
          }
        }
      }
      if (!ok) break;
      if constexpr (kQkv) {
        // y = acc + b in place (N is a multiple of 128 here), then in Q / K
        // tiles the head's RMS normalisation and rotary embedding.  A row's
        // head is the whole tile: the four column slices of a lane quarter
        // add their sums of squares through shared memory in slice order.
        // Every epilogue warp works on the same tile, so the barriers are
        // uniform; the slot is next written after this tile's second
        // barrier, which every reader has passed.
#pragma unroll
        for (int c = 0; c < 32; ++c) acc[c] = __fadd_rn(acc[c], __ldg(p.bias + nc + c));
        if (n0 < p.qk_cols) {
          float ss = 0.0f;
#pragma unroll
          for (int c = 0; c < 32; ++c) ss = __fmaf_rn(acc[c], acc[c], ss);
          red_s[(q4 * 4 + cs) * 32 + lane] = ss;
          named_bar_sync(2, 32 * kI4EpiWarps);
          const float tot = __fadd_rn(__fadd_rn(red_s[(q4 * 4 + 0) * 32 + lane], red_s[(q4 * 4 + 1) * 32 + lane]),
                                      __fadd_rn(red_s[(q4 * 4 + 2) * 32 + lane], red_s[(q4 * 4 + 3) * 32 + lane]));
          named_bar_sync(2, 32 * kI4EpiWarps);
          const float rs = rsqrtf(__fmaf_rn(tot, 1.0f / 128.0f, p.eps));
          const float4* wn = reinterpret_cast<const float4*>((n0 < p.qk_cols / 2 ? p.norm_q : p.norm_k) + 32 * cs);
          // frequency-major rotary tables: one line per frequency per warp
          const bool in_rows = row < p.M;
          const size_t trow = static_cast<size_t>(16 * cs) * p.M + (in_rows ? row : 0);
          const float* ct = p.rope_cos + trow;
          const float* st = p.rope_sin + trow;
#pragma unroll
          for (int q = 0; q < 4; ++q) {  // four pairs per step
            float cc[4], sc[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              cc[j] = in_rows ? __ldg(ct + static_cast<size_t>(4 * q + j) * p.M) : 1.0f;
              sc[j] = in_rows ? __ldg(st + static_cast<size_t>(4 * q + j) * p.M) : 0.0f;
            }
            const float4 w0 = __ldg(wn + 2 * q), w1 = __ldg(wn + 2 * q + 1);
            // the head's scale folded into the weights: (y r) w = y (r w)
            const float rw[8] = {__fmul_rn(rs, w0.x), __fmul_rn(rs, w0.y), __fmul_rn(rs, w0.z), __fmul_rn(rs, w0.w),
                                 __fmul_rn(rs, w1.x), __fmul_rn(rs, w1.y), __fmul_rn(rs, w1.z), __fmul_rn(rs, w1.w)};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int c = 8 * q + 2 * j;
              const float a = __fmul_rn(acc[c], rw[2 * j]);
              const float b = __fmul_rn(acc[c + 1], rw[2 * j + 1]);
              acc[c] = __fmaf_rn(a, cc[j], -__fmul_rn(b, sc[j]));
              acc[c + 1] = __fmaf_rn(a, sc[j], __fmul_rn(b, cc[j]));
            }
          }
        }
      }
      if (row < p.M) {
#pragma unroll
        for (int c = 0; c < 32; c += 8) {
          const int n = nc + c;
          if (n >= p.N) break;
          float y[8];
#pragma unroll
          for (int j = 0; j < 8; ++j)
            y[j] = kQkv ? acc[c + j] : __fadd_rn(acc[c + j], n + j < p.N ? __ldg(p.bias + n + j) : 0.0f);
          if (n + 8 <= p.N && (p.N & 7) == 0) {
            if constexpr (kF32Out) {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.Y) + static_cast<size_t>(row) * p.N + n);
              dst[0] = make_float4(y[0], y[1], y[2], y[3]);
              dst[1] = make_float4(y[4], y[5], y[6], y[7]);
            } else {
              uint4 o;
              __nv_bfloat162 h;
              h = __floats2bfloat162_rn(y[0], y[1]); o.x = *reinterpret_cast<uint32_t*>(&h);
              h = __floats2bfloat162_rn(y[2], y[3]); o.y = *reinterpret_cast<uint32_t*>(&h);
              h = __floats2bfloat162_rn(y[4], y[5]); o.z = *reinterpret_cast<uint32_t*>(&h);
              h = __floats2bfloat162_rn(y[6], y[7]); o.w = *reinterpret_cast<uint32_t*>(&h);
              *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.Y) + static_cast<size_t>(row) * p.N + n) = o;
            }
          } else {
            for (int j = 0; j < 8 && n + j < p.N; ++j) {
              if constexpr (kF32Out)
                static_cast<float*>(p.Y)[static_cast<size_t>(row) * p.N + n + j] = y[j];
              else
                static_cast<__nv_bfloat16*>(p.Y)[static_cast<size_t>(row) * p.N + n + j] = __float2bfloat16_rn(y[j]);
            }
          }
        }
      }
    }
  }

teardown:
  __syncthreads();
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kI4Stages; ++s)
      if (issued_mask & (1u << s)) mbar_wait_limited(&full[s], (issued_par >> s) & 1u, 200000000ull);
  }
  if (warp == kScaleWarp && lane == 0) {
    for (int s = 0; s < kScaleSlots; ++s)
      if (sc_mask & (1u << s)) mbar_wait_limited(&sc_full[s], (sc_par >> s) & 1u, 200000000ull);
  }
  if (warp == 1 || warp == kMma2Warp) {
    if (elect_one()) {
      tc_commit(drain);  // the lane that issued the MMAs: arrives once they have finished
      mbar_wait_limited(drain, 0, 200000000ull);
    }
    __syncwarp();
  }
  if (threadIdx.x == 0 && *abort_flag) atomicExch(p.status, static_cast<int>(SVDQ_ERR_TIMEOUT));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kI4TmemCols);
}

}  // namespace

cudaError_t launch_gemm_int4(const svdq_weights* w, const uint8_t* qx, const void* sx, const float* lora_act, int M,
                             void* Y, int out_dtype, const svdq_qkv_prologue* pro, cudaStream_t s) {
  const int K = w->desc.K, N = w->desc.N;
  const int m_pad = static_cast<int>(m_pad_of(M));
  CUtensorMap tm_a8, tm_la;
  // the codes' E4M3 copy after the packed codes: M rows of K bytes, 128-byte
  // swizzled boxes of 128 rows x 128 bytes (128 K)
  if (!encode_tmap_2d_swizzle(&tm_a8, CU_TENSOR_MAP_DATA_TYPE_UINT8, qx + int4_q8_offset(M, K), K, M, K, 128, kTileM,
                              CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (w->rank_pad > 0) {
    if (!encode_tmap_2d(&tm_la, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, lora_act, w->rank_pad, M,
                        static_cast<uint64_t>(w->rank_pad) * 4, 32, kTileM))
      return cudaErrorInvalidValue;
  } else {
    tm_la = tm_a8;  // unused without a low-rank branch
  }
  I4Params p;
  p.sx = static_cast<const __half*>(sx);
  p.sw = static_cast<const __half*>(w->sw);
  p.bias = w->bias;
  p.Y = Y;
  p.status = w->status;
  p.M = M;
  p.N = N;
  p.K = K;
  p.m_pad = m_pad;
  p.n_lora = w->rank_pad / 32;
  p.n_pad = w->n_pad;
  p.norm_q = pro ? pro->norm_q : nullptr;
  p.norm_k = pro ? pro->norm_k : nullptr;
  p.rope_cos = pro ? pro->rope_cos : nullptr;
  p.rope_sin = pro ? pro->rope_sin : nullptr;
  p.eps = pro ? pro->eps : 0.0f;
  p.qk_cols = pro ? 2 * pro->heads * pro->head_dim : 0;
  const int tiles = ((M + kTileM - 1) / kTileM) * ((N + kTileN - 1) / kTileN);
  const int grid = std::min(tiles, num_sms(w->device));
  const bool f32 = out_dtype == SVDQ_OUT_F32;
  auto kern = pro ? (f32 ? gemm_int4_kernel<true, true> : gemm_int4_kernel<false, true>)
                  : (f32 ? gemm_int4_kernel<true, false> : gemm_int4_kernel<false, false>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kI4Smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kI4Threads, 1, 1);
  cfg.dynamicSmemBytes = kI4Smem;
  cfg.stream = s;
  // programmatic dependent launch (the kernel waits before any memory access)
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tm_a8, w->tm_qw8, tm_la, w->tm_l2, p);
}

}  // namespace svdq
