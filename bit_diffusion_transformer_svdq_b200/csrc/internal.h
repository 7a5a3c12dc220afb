// Host-side internals shared by the translation units of libsvdq: the
// prepared-weights handle, layout helpers and the kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "../../include/svdq.h"

namespace svdq {

constexpr int kRankMax = 64;

inline int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }
inline int rank_pad_of(int rank) { return rank == 0 ? 0 : static_cast<int>(round_up(rank, 32)); }
inline int64_t n_pad_of(int64_t n) { return round_up(n, 256); }
inline int64_t m_pad_of(int64_t m) { return round_up(m, 128); }

// Byte size of the scale buffer for `rows` rows (rows padded per precision).
inline size_t nvfp4_scale_bytes(int64_t rows_padded, int K) { return static_cast<size_t>(rows_padded) * (K / 16); }
inline size_t int4_scale_bytes(int64_t rows_padded, int K) { return static_cast<size_t>(rows_padded) * (K / 64) * 2; }

// INT4 activation codes: the packed codes (M x K/2 bytes) are followed, at
// this 1024-aligned offset of the same buffer, by the codes as E4M3 bytes
// (M x K), the A operand of the INT4 GEMM.
inline size_t int4_q8_offset(int64_t M, int K) { return static_cast<size_t>(round_up(M * (K / 2), 1024)); }

// Offsets (bytes) of the sub-buffers inside the caller's weight storage.
struct WeightLayout {
  size_t qw, sw, l1s, l2, inv_lambda, bias, status, amax, total;
  size_t sw_bytes;
  size_t qw8;  // INT4 only (0 otherwise): codes as E4M3 bytes
};

// INT4 working copies for the tensor-core GEMM.  tcgen05 has no 4-bit
// integer kind, so the codes go to the tensor core as 8-bit operands: E4M3
// bytes, which hold every integer in [-8, 7] exactly (kind::f8f6f4).  Each
// product is an integer of magnitude at most 64 and a 64-group's sum at
// most 4096, exact in the fp32 accumulator, so a group's TMEM result is the
// integer dot product itself, already a float.  Codes keep their natural K
// order.  E4M3 of the two's-complement nibble n: kI4E4m3[n].
constexpr uint32_t kI4E4m3Lo0 = 0x44403800u, kI4E4m3Lo1 = 0x4E4C4A48u;  // n = 0..7: 0, 1, 2, ..., 7
constexpr uint32_t kI4E4m3Hi0 = 0xCACCCED0u, kI4E4m3Hi1 = 0xB8C0C4C8u;  // n = 8..15: -8, -7, ..., -1
WeightLayout weight_layout(const svdq_layer_desc& d);

}  // namespace svdq

// The opaque handle of the C ABI.
struct svdq_weights {
  svdq_layer_desc desc;
  int rank_pad;
  int64_t n_pad;
  float g_w;
  uint8_t* base;  // caller's storage
  uint8_t* qw;
  void* sw;
  size_t sw_bytes;
  uint16_t* l1s;
  float* l2;
  float* inv_lambda;
  float* bias;
  int* status;    // written by the kernels when a bounded wait runs out
  uint32_t* amax; // scratch: [0], [1] the preparation's amax and g_w; [2], [3] the activation amax
                  // reduction (max, block count), zero between calls
  uint8_t* qw8;   // INT4: n_pad x K codes as E4M3 bytes (rows past N zero); NVFP4: null
  int device;
  CUtensorMap tm_qw;  // weight codes, 128-byte swizzled boxes of 128 rows
  CUtensorMap tm_l2;  // fp32 L2, 128-byte swizzled boxes of 128 rows
  CUtensorMap tm_sw;  // NVFP4 weight scales viewed as rows of 256 bytes, boxes of 8 rows (4 atoms)
  CUtensorMap tm_l1s; // bf16 L1s as 64-column chunks: boxes of all rank_pad rows x kQChunks chunks
  CUtensorMap tm_qw8; // INT4: E4M3 codes, 128-byte swizzled boxes of 128 rows x 128 K
};

namespace svdq {

// Launchers (return cudaGetLastError() of the launch).
cudaError_t launch_smoothing_lambda(const uint16_t* X, int M, const float* W, int N, int K, float* lambda,
                                    float* scratch, cudaStream_t s);
cudaError_t launch_prepare(const svdq_weights* w, const float* W, const float* lambda, const uint16_t* L1,
                           const uint16_t* L2, const uint16_t* bias, cudaStream_t s);
cudaError_t launch_act_amax(const svdq_weights* w, const uint16_t* X, int M, float* amax, cudaStream_t s);
cudaError_t launch_act_global_scale(const svdq_weights* w, const uint16_t* X, int M, float* g_x, cudaStream_t s);
// `x_amax` (may be null): the dynamic tensor scale's device amax, which
// then replaces g_x (NVFP4)
// `zero_word` (may be null) is set to 0 by the kernel
cudaError_t launch_quantize(const svdq_weights* w, const uint16_t* X, int M, float g_x, const float* x_amax,
                            uint8_t* qx, void* sx, float* lora_act, float* zero_word, cudaStream_t s);
// `pro` (may be null): the QKV attention prologue applied in the epilogue;
// `epi` (may be null, never with `pro`): activation and next-layer amax
cudaError_t launch_gemm_nvfp4(const svdq_weights* w, const uint8_t* qx, const uint8_t* sx, float g_x,
                              const float* x_amax, const float* lora_act, int M, void* Y, int out_dtype,
                              const svdq_qkv_prologue* pro, const svdq_epilogue_next* epi, cudaStream_t s);
size_t lowrank_workspace_bytes(int N, int K);
cudaError_t launch_lowrank(const float* W, int N, int K, const float* lambda, int rank, int ell, int power_steps,
                           const float* omega, uint16_t* L1, uint16_t* L2, void* workspace, cudaStream_t s);
cudaError_t launch_awq_gemv(const svdq_weights* w, const uint16_t* X, int M, void* Y, int out_dtype, cudaStream_t s);
cudaError_t launch_gemm_int4(const svdq_weights* w, const uint8_t* qx, const void* sx, const float* lora_act, int M,
                             void* Y, int out_dtype, const svdq_qkv_prologue* pro, cudaStream_t s);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no
// link-time dependency on libcuda).  2-D, row-major, `inner` elements per
// row of `row_bytes` stride, box {box_inner, box_rows}, 128-byte swizzle.
bool encode_tmap_2d(CUtensorMap* tm, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t rows,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, bool swizzle128 = true);
bool encode_tmap_2d_swizzle(CUtensorMap* tm, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                            uint64_t rows, uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows,
                            CUtensorMapSwizzle swizzle);
// A K-major bf16 matrix (rows x K, row pitch K * 2 bytes) seen as 64-column
// chunks: dims {64, rows, K / 64}.  A {64, box_rows, box_chunks} box lands
// in shared memory as box_chunks consecutive 128-byte-swizzled tiles of
// box_rows x 64, the same bytes that box_chunks separate 2-D boxes would
// write, in one request.
bool encode_tmap_chunked_bf16(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t K, uint32_t box_rows,
                              uint32_t box_chunks);

// 64-column chunks per stage of the activation quantiser (the L1s map's box).
constexpr int kQChunks = 1;

int num_sms(int device);

}  // namespace svdq
