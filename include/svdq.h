/*
 * svdq.h - C ABI of the B200 (sm_100a) SVDQuant W4A4 linear layer.
 *
 * What the layer computes (Nunchaku 4-bit quantisation in Diffusers,
 * section "Nunchaku und SVDQuant"; charmloop.ai Nunchaku news item,
 * second paragraph):
 *
 *     X_hat = X / lambda                 activation outliers moved into W
 *     W_til = W * diag(lambda)
 *     R     = W_til - (L1 L2)^T          residual of a 16-bit low-rank branch
 *     Y     = X_hat L1 L2 + Q(X_hat) Q(R)^T + b
 *
 * Q() is 4-bit group quantisation: NVFP4 (E2M1 values, one E4M3 scale per
 * 16 values, one fp32 tensor scale) or INT4 (one fp16 scale per 64 values);
 * the precision / group_size / rank triple is the svdq_w4a4 block of the
 * page's quantization_config ("Native Ladefunktion").  The lora-down
 * X_hat L1 runs inside the activation-quantisation kernel and the lora-up
 * inside the 4-bit GEMM, as the news item describes.
 *
 * Conventions for every entry point:
 *   - Matrices are row-major.  "bf16" buffers hold raw bfloat16 bit
 *     patterns in uint16_t.  Orientation follows nn.Linear: X is M x K,
 *     W is N x K, Y is M x N.  L1 ("lora_down") is stored rank x K and
 *     L2 ("lora_up") N x rank, so that the branch is X_hat L1^T L2^T.
 *   - Every buffer is caller-owned.  Pointers marked [device] must be CUDA
 *     device memory of the current device, 16-byte aligned; [host] pointers
 *     are host memory.  The library never allocates device memory.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous on that stream unless stated otherwise.
 *   - Errors are returned as svdq_status; nothing aborts or exits.  Shape
 *     and argument checks happen on the host before any launch.
 *   - Only compute capability 10.0 (B200, sm_100a) is supported; other
 *     devices get SVDQ_ERR_UNSUPPORTED_DEVICE (the pages' load-time GPU
 *     capability check, "Hardware-Unterstuetzung").
 *
 * Shape limits: K % 64 == 0 (NVFP4: four 16-wide groups per MMA step;
 * INT4: one 64-wide group), N % 16 == 0, 0 <= rank <= 64 with rank % 8 == 0,
 * (precision, group_size) in {(NVFP4, 16), (INT4, 64)}, M >= 0.
 */
#ifndef SVDQ_H
#define SVDQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SVDQ_API __attribute__((visibility("default")))
#else
#define SVDQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum svdq_status {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,        /* null pointer, bad enum, bad combination */
  SVDQ_ERR_SHAPE = 2,              /* a size outside the limits above */
  SVDQ_ERR_ALIGNMENT = 3,          /* a device pointer not 16-byte aligned */
  SVDQ_ERR_UNSUPPORTED_DEVICE = 4, /* current device is not compute capability 10.0 */
  SVDQ_ERR_CUDA = 5,               /* a CUDA runtime call or launch failed */
  SVDQ_ERR_TIMEOUT = 6,            /* a bounded wait inside a kernel ran out */
  SVDQ_ERR_WORKSPACE = 7           /* storage / workspace smaller than required */
} svdq_status;

typedef enum svdq_precision {
  SVDQ_NVFP4 = 0,     /* E2M1 codes, E4M3 scale per 16, fp32 tensor scale */
  SVDQ_INT4 = 1,      /* signed 4-bit codes, fp16 scale per 64 */
  SVDQ_AWQ_W4A16 = 2  /* the awq_w4a16 family: INT4 group-64 weights, 16-bit
                         activations (see svdq_awq_w4a16_forward) */
} svdq_precision;

typedef enum svdq_out_dtype {
  SVDQ_OUT_BF16 = 0, /* production output: bf16, round to nearest even */
  SVDQ_OUT_F32 = 1   /* parity/debug output: the same epilogue stored in fp32 */
} svdq_out_dtype;

/* One quantised linear layer (the svdq_w4a4 block of quantization_config;
 * with precision SVDQ_AWQ_W4A16 the awq_w4a16 block: group_size 64,
 * rank 0). */
typedef struct svdq_layer_desc {
  int32_t K;          /* input features */
  int32_t N;          /* output features */
  int32_t rank;       /* low-rank branch width r (0 = no branch) */
  int32_t precision;  /* svdq_precision */
  int32_t group_size; /* 16 for NVFP4, 64 for INT4 */
} svdq_layer_desc;

/* Opaque host handle of prepared weights.  The device data it refers to
 * lives in the caller's `storage` buffer (see svdq_prepare_weights); the
 * handle must not outlive that buffer. */
typedef struct svdq_weights svdq_weights;

/* Read-only view of prepared weights, for inspection and parity checks.
 * All pointers are [device] and point into the caller's storage.
 *   qw        N x K/2 bytes, two codes per byte, even k in the low nibble.
 *             NVFP4: E2M1 nibbles (bit 3 = sign); INT4: two's complement.
 *             AWQ_W4A16: two's complement in the GEMV tile layout: rows
 *             padded to n_pad (zero codes), and the 16 bytes holding codes
 *             32c .. 32c+31 of row n at
 *                 ((n / 32) * (K / 32) + c) * 512 + (n % 32) * 16,
 *             so that 32 consecutive rows of one 32-code chunk are 512
 *             contiguous bytes.
 *   sw        NVFP4: E4M3 bytes in the tiled scale layout (below) with
 *             rows = N padded to a multiple of 256.
 *             INT4 and AWQ_W4A16: fp16, group-major: sw[g * n_pad + n], g < K/64.
 *   l1s       rank_pad x K bf16: bf16(RN32(L1[t,k] * inv_lambda[k])),
 *             rows t >= rank are zero.
 *   l2        N x rank_pad fp32 copy of L2 (exact), columns t >= rank zero.
 *   inv_lambda K fp32 = RN32(1 / lambda).
 *   bias      N fp32 (widened from bf16; zeros when no bias was given).
 *
 * Tiled scale layout (NVFP4 sx and sw; the layout the tensor cores read):
 * rows are padded to a multiple of 128 (256 for sw); the byte of row m and
 * 16-wide group j (j < K/16) sits at
 *     ((m / 128) * (K / 64) + j / 4) * 512 + (m % 32) * 16 + ((m / 32) % 4) * 4 + j % 4.
 */
typedef struct svdq_weights_view {
  int32_t K, N, rank, rank_pad, precision, group_size;
  int32_t n_pad;       /* scale rows: N rounded up to a multiple of 256 */
  float g_w;           /* NVFP4 weight tensor scale (1 for INT4) */
  const uint8_t* qw;
  const void* sw;
  size_t sw_bytes;
  const uint16_t* l1s;
  const float* l2;
  const float* inv_lambda;
  const float* bias;
} svdq_weights_view;

/* Human-readable name of a status code (static string). */
SVDQ_API const char* svdq_status_string(svdq_status s);

/* SVDQ_OK when `device` is a compute capability 10.0 GPU. */
SVDQ_API svdq_status svdq_check_device(int device);

/* Per-input-channel smoothing factor (the migration of activation outliers
 * into the weights, "Nunchaku und SVDQuant"):
 *     lambda[k] = RN32(sqrt(max_m |X[m,k]| / max_n |W[n,k]|)) in fp64,
 *     lambda[k] = 1 when either maximum is 0.
 * X [device] M x K bf16, W [device] N x K fp32, lambda [device] K fp32 out,
 * scratch [device] 2*K fp32, overwritten.  M, N >= 1. */
SVDQ_API svdq_status svdq_smoothing_lambda(const uint16_t* X, int32_t M, const float* W, int32_t N, int32_t K,
                                  float* lambda, float* scratch, void* stream);

/* Device bytes of the storage that svdq_prepare_weights fills. */
SVDQ_API size_t svdq_weights_bytes(const svdq_layer_desc* desc);

/* Weight preparation on the GPU (offline; the pages' quantiser step):
 *   inv_lambda = RN32(1/lambda); W_til = RN32(W * lambda);
 *   R[n,k] = RN32(fp64 chain W_til[n,k] - L1[0,k] L2[n,0] - ... - L1[r-1,k] L2[n,r-1]);
 *   NVFP4: g_w = RN32(amax|R| / 2688) (1 if amax is 0), E4M3 scale per 16
 *   and E2M1 codes by the rule of svdq_quantize_act_lora_down; INT4: fp16
 *   scale per 64 and signed codes;  L1s = bf16(RN32(L1 * inv_lambda)).
 * Inputs [device]: W N x K fp32, lambda K fp32, L1 rank x K bf16,
 * L2 N x rank bf16, bias N bf16 or NULL.  L1/L2 may be NULL when rank == 0.
 * storage [device] at least svdq_weights_bytes(desc) bytes, 1024-byte
 * aligned, caller-owned; *out receives a host handle (free it with
 * svdq_weights_destroy).  SYNCHRONOUS: returns after the GPU work is done
 * (g_w is read back to the host). */
SVDQ_API svdq_status svdq_prepare_weights(const svdq_layer_desc* desc, const float* W, const float* lambda,
                                 const uint16_t* L1, const uint16_t* L2, const uint16_t* bias,
                                 void* storage, size_t storage_bytes, svdq_weights** out, void* stream);

/* The low-rank factors L1 (rank x K) and L2 (N x rank) that
 * svdq_prepare_weights takes, computed on the GPU: a truncated SVD of the
 * smoothed weight W_til^T = (RN32(W * lambda))^T (K x N) by randomized block
 * subspace iteration (Halko, Martinsson and Tropp 2011; the pages name the
 * method, "Nunchaku und SVDQuant", but not the factorisation):
 *     Q = orth(W_til^T Omega);  power_steps times: Z = orth(W_til Q),
 *     Q = orth(W_til^T Z);  B = Q^T W_til^T = U_b diag(s) V^T;
 *     L1 = bf16((Q U_b)_r diag(s_r))^T,  L2 = bf16(V_r)
 * with orth() two passes of Cholesky QR (fp64 Gram matrices) and the small
 * SVD from the fp64 eigendecomposition of B B^T.  The signs of matching
 * columns of U and V are arbitrary; L2 L1 is not.
 * Inputs [device]: W N x K fp32, lambda K fp32, omega N x ell fp32 (the
 * start block, e.g. standard normal draws; ell = rank + oversample).
 * Outputs [device]: L1 rank x K bf16, L2 N x rank bf16.  workspace [device]
 * >= svdq_lowrank_workspace_bytes(N, K) bytes, 256-byte aligned.
 * Limits: 1 <= rank, rank % 8 == 0, oversample >= 0, ell <= 64,
 * ell <= min(N, K), 0 <= power_steps <= 16.  Asynchronous on `stream`. */
SVDQ_API size_t svdq_lowrank_workspace_bytes(int32_t N, int32_t K);
SVDQ_API svdq_status svdq_lowrank_factors(const float* W, int32_t N, int32_t K, const float* lambda, int32_t rank,
                                 int32_t oversample, int32_t power_steps, const float* omega, uint16_t* L1,
                                 uint16_t* L2, void* workspace, size_t ws_bytes, void* stream);

/* Frees the host handle (not the caller's device storage).  NULL is a no-op. */
SVDQ_API void svdq_weights_destroy(svdq_weights* w);

SVDQ_API svdq_status svdq_weights_get_view(const svdq_weights* w, svdq_weights_view* view);

/* Host buffers that svdq_export_weights fills, in the canonical row-major
 * layouts of the pages' quantised layer (the svdq_w4a4 block of
 * quantization_config, "Native Ladefunktion": 4-bit codes, group scales,
 * the 16-bit low-rank pair, the smoothing factor and the bias).  Every
 * pointer is [host], caller-owned, and may be NULL to skip that part.
 *   qw          N x K/2 bytes, two codes per byte, even k in the low nibble
 *               (NVFP4: E2M1 nibbles; INT4 and AWQ_W4A16: two's complement)
 *   sw          NVFP4: N x K/16 E4M3 bytes; INT4, AWQ_W4A16: N x K/64 fp16
 *   l1s         rank x K bf16 bit patterns: bf16(RN32(L1 * inv_lambda))
 *   l2          N x rank fp32 (the bf16 values of L2, exact)
 *   inv_lambda  K fp32
 *   bias        N fp32 (bf16 values; zeros when no bias was given)
 *   g_w         one fp32: the NVFP4 weight tensor scale (1 otherwise) */
typedef struct svdq_weights_export {
  uint8_t* qw;
  void* sw;
  uint16_t* l1s;
  float* l2;
  float* inv_lambda;
  float* bias;
  float* g_w;
} svdq_weights_export;

/* Copies prepared weights to the host buffers of `out`, untiling the
 * kernels' layouts (svdq_weights_view) into the canonical ones above.
 * SYNCHRONOUS: the copies run on `stream`, which is synchronised before
 * the call returns.  Allocates host memory only (temporary staging).
 * Errors: SVDQ_ERR_INVALID_ARG for a NULL handle or `out`, SVDQ_ERR_CUDA
 * when a copy or the synchronisation fails. */
SVDQ_API svdq_status svdq_export_weights(const svdq_weights* w, svdq_weights_export* out, void* stream);

/* Canonical host copy of an activation scale buffer written by
 * svdq_quantize_act_lora_down for M rows of weights `w`: NVFP4 -> M x K/16
 * E4M3 bytes, INT4 -> M x K/64 fp16, both row-major (the tiled and the
 * group-major device layouts are described with svdq_weights_view and
 * svdq_act_scale_bytes).  sx [device], out [host].  SYNCHRONOUS on
 * `stream`.  SVDQ_ERR_INVALID_ARG for AWQ_W4A16 weights (no activation
 * quantisation there) or NULL buffers; M == 0 is a no-op. */
SVDQ_API svdq_status svdq_export_act_scales(const svdq_weights* w, const void* sx, int32_t M, void* out,
                                            void* stream);

/* Static activation tensor scale for NVFP4: g_x = RN32(amax |X_hat| / 2688)
 * with X_hat = RN32(X * inv_lambda) (1 when amax is 0), written to
 * g_x [device] (one fp32).  X [device] M x K bf16, M >= 1. */
SVDQ_API svdq_status svdq_act_global_scale(const svdq_weights* w, const uint16_t* X, int32_t M, float* g_x, void* stream);

/* Dynamic activation tensor scale (NVFP4): writes amax |X_hat|, X_hat =
 * RN32(X * inv_lambda), to amax [device] (one fp32, 4-byte aligned; NaN
 * inputs are skipped).  The reduction runs in one kernel through a scratch
 * slot of the weight storage, so calls that compute an amax on one weight
 * set (this one, svdq_act_global_scale, svdq_linear_forward_dyn without
 * x_amax) must not overlap on the GPU.  The
 * _dyn entry points take such a word and use g_x = RN32(amax / 2688)
 * (1 when amax is 0) on the device, with no host round trip: the same
 * value svdq_act_global_scale writes.  X [device] M x K bf16, M >= 1. */
SVDQ_API svdq_status svdq_act_amax(const svdq_weights* w, const uint16_t* X, int32_t M, float* amax, void* stream);

/* Bytes of the activation code buffer qx for M rows (0 for awq_w4a16
 * weights, which quantise no activations):
 *   NVFP4: M * K/2, the packed codes;
 *   INT4:  the packed codes (M * K/2 bytes), then, from byte offset
 *          round_up(M * K/2, 1024), the same codes as E4M3 bytes (M x K,
 *          row-major, code k of row m at m * K + k): every integer in
 *          [-8, 7] is exact in E4M3, and this copy is the INT4 GEMM's
 *          tensor-core operand.
 * svdq_quantize_act_lora_down writes the whole buffer and
 * svdq_w4a4_gemm_lora_up reads it: allocate this many bytes. */
SVDQ_API size_t svdq_act_codes_bytes(const svdq_weights* w, int32_t M);

/* Bytes of the activation scale buffer sx for M rows:
 * NVFP4: ceil(M/128)*128 * K/16 (tiled layout); INT4: 2 * K/64 * ceil(M/128)*128. */
SVDQ_API size_t svdq_act_scale_bytes(const svdq_weights* w, int32_t M);

/* Fused smoothing + 4-bit activation quantisation + lora-down (one pass
 * over X).  For every row m and group:
 *   x_hat = RN32(X[m,k] * inv_lambda[k])
 *   NVFP4 (group 16, tensor scale g_x > 0):
 *     s_q = E4M3_RNE_satfinite(RN32(RN32(amax/6) / g_x)), s = value(s_q);
 *     s == 0 -> codes +0; else code = E2M1_RNE_satfinite(RN32(x_hat *
 *     RN32(1 / RN32(s * g_x)))), the sign of a zero result kept.
 *   INT4 (group 64; g_x ignored): s_h = fp16(RN32(amax/7)); s_h == 0 ->
 *     codes 0; else q = clamp(rint(RN32(x_hat * RN32(1/s_h))), -8, 7).
 *   lora_act[m,t] = sum_k X[m,k] * L1s[t,k] (fp32 accumulation), then
 *     multiplied by RN32(1 / RN32(g_x * g_w)) (NVFP4; 1 for INT4) and
 *     rounded to tf32 (10-bit mantissa): the unit of the GEMM accumulator.
 * X [device] M x K bf16.  Outputs [device]: qx svdq_act_codes_bytes(w, M)
 * bytes (the packed codes; for INT4 also their E4M3 copy); sx
 * svdq_act_scale_bytes(w, M) bytes (padding rows are written with zeros);
 * lora_act M x rank_pad fp32 (may be NULL when rank == 0). */
SVDQ_API svdq_status svdq_quantize_act_lora_down(const svdq_weights* w, const uint16_t* X, int32_t M, float g_x,
                                        uint8_t* qx, void* sx, float* lora_act, void* stream);

/* svdq_quantize_act_lora_down with the dynamic tensor scale: g_x =
 * RN32(*x_amax / 2688) (1 when *x_amax is 0), derived on the device by the
 * kernel with the same correctly rounded operations, so the outputs equal
 * those of the static call given that g_x.  x_amax [device] one fp32
 * (4-byte aligned), from svdq_act_amax or a previous layer's epilogue
 * (svdq_epilogue_next); required for NVFP4, ignored (may be NULL) for
 * INT4.  A derived g_x that is not finite and positive sets the status
 * word to SVDQ_ERR_INVALID_ARG (svdq_device_status); the outputs are then
 * unspecified. */
SVDQ_API svdq_status svdq_quantize_act_lora_down_dyn(const svdq_weights* w, const uint16_t* X, int32_t M,
                                                     const float* x_amax, uint8_t* qx, void* sx, float* lora_act,
                                                     void* stream);

/* 4-bit GEMM with the lora-up and the bias fused into its epilogue:
 *   NVFP4: Y = RN32(g_x * g_w) * (sum_b s_x s_w sum_{k in b} e2m1(qx) e2m1(qw)
 *                                 + lora_act L2^T) + b
 *   INT4:  Y = sum_g s_x s_w sum_{k in g} qx qw + lora_act L2^T + b
 * stored as bf16 (RNE) or fp32 (out_dtype).  Inputs as written by
 * svdq_quantize_act_lora_down: qx is the whole svdq_act_codes_bytes(w, M)
 * buffer (INT4 reads only its E4M3 copy).  Y [device] M x N. */
SVDQ_API svdq_status svdq_w4a4_gemm_lora_up(const svdq_weights* w, const uint8_t* qx, const void* sx, float g_x,
                                   const float* lora_act, int32_t M, void* Y, int32_t out_dtype, void* stream);

/* Attention prologue fused into the epilogue of a QKV projection.  The
 * pages ("Quantisierung von Modellen mit strukturellen Umschreibungen",
 * Nunchaku 4-bit in Diffusers) describe the FLUX to_qkv module: one
 * quantised projection whose fused operator also applies the Q/K
 * normalisation and the rotary embedding.  With Y = [Q | K | V] (each
 * heads * head_dim columns) the epilogue stores
 *     Q' = rope(rmsnorm(Q) * norm_q),  K' = rope(rmsnorm(K) * norm_k),  V
 * where, per row and head, rmsnorm(q)[d] = q[d] / sqrt(mean_d(q^2) + eps)
 * and rope turns the pairs (2i, 2i+1) of every head by the row's angle:
 * (a, b) -> (a cos[m,i] - b sin[m,i], a sin[m,i] + b cos[m,i]).  The values
 * normalised are the layer outputs before rounding (accumulator, lora-up
 * and bias in fp32); the result is rounded once to the output dtype.
 * Limits: head_dim == 128; the layer's N == 3 * heads * 128 with heads
 * even; eps > 0.  All pointers [device], 16-byte aligned:
 *   norm_q, norm_k   head_dim fp32 weights,
 *   rope_cos, rope_sin   head_dim/2 x M fp32, frequency-major: the value
 *                    for pair i of token m at [i * M + m] (32 consecutive
 *                    tokens of one frequency are one 128-byte line, which
 *                    is what the epilogue, one thread per token, reads). */
typedef struct svdq_qkv_prologue {
  int32_t heads;
  int32_t head_dim;
  float eps;
  const float* norm_q;
  const float* norm_k;
  const float* rope_cos;
  const float* rope_sin;
} svdq_qkv_prologue;

/* svdq_w4a4_gemm_lora_up with the QKV attention prologue above applied in
 * its epilogue (NVFP4 and INT4).  Same arguments plus `pro` [host]. */
SVDQ_API svdq_status svdq_w4a4_gemm_lora_up_qkv(const svdq_weights* w, const uint8_t* qx, const void* sx, float g_x,
                                       const float* lora_act, int32_t M, const svdq_qkv_prologue* pro, void* Y,
                                       int32_t out_dtype, void* stream);

/* Activations applied in the GEMM epilogue (svdq_epilogue_next). */
typedef enum svdq_activation {
  SVDQ_ACT_NONE = 0,
  SVDQ_ACT_GELU_TANH = 1 /* 0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3))) */
} svdq_activation;

/* Epilogue extras for a layer whose output is the next W4A4 layer's input
 * (the FLUX feed-forward: up-projection, GELU, down-projection), so that
 * the next layer's dynamic tensor scale needs no pass of its own over Y.
 *   activation       applied to y (fp32: accumulator, lora-up and bias)
 *                    before the one rounding to the output dtype.  The
 *                    GELU is evaluated as y / (1 + e^(-2u)), an identity
 *                    of the tanh form, with the hardware exp2 and
 *                    reciprocal (relative error near 1e-6).
 *   next_inv_lambda  [device] N fp32: 1/lambda of the next layer (whose K
 *                    is this N), 4-byte aligned; or NULL.
 *   next_amax        [device] one fp32, 4-byte aligned; NULL exactly when
 *                    next_inv_lambda is.  The epilogue max-reduces
 *                    |RN32(y_stored * next_inv_lambda[n])| over the stored
 *                    outputs (rows < M, columns < N; NaN skipped) into it,
 *                    so that a word that held 0 ends as the amax that
 *                    svdq_act_amax(next layer, Y) writes.  The GEMM entry
 *                    point leaves zeroing it to the caller; the forward
 *                    entry point zeroes it in its quantiser kernel (no
 *                    extra launch), and it must not be that call's x_amax.
 * NVFP4 weights only (INT4 takes NULL or extras that ask for nothing); not
 * combined with the QKV prologue. */
typedef struct svdq_epilogue_next {
  int32_t activation;
  const float* next_inv_lambda;
  float* next_amax;
} svdq_epilogue_next;

/* svdq_w4a4_gemm_lora_up with the dynamic tensor scale (x_amax as in
 * svdq_quantize_act_lora_down_dyn: required for NVFP4, ignored for INT4),
 * the optional QKV prologue `pro` [host] and the optional epilogue extras
 * `epi` [host] (at most one of the two). */
SVDQ_API svdq_status svdq_w4a4_gemm_lora_up_dyn(const svdq_weights* w, const uint8_t* qx, const void* sx,
                                                const float* x_amax, const float* lora_act, int32_t M,
                                                const svdq_qkv_prologue* pro, const svdq_epilogue_next* epi, void* Y,
                                                int32_t out_dtype, void* stream);

/* Workspace bytes of svdq_linear_forward for M rows (qx, sx, lora_act and
 * one 1024-byte slot for the dynamic tensor scale's amax). */
SVDQ_API size_t svdq_workspace_bytes(const svdq_weights* w, int32_t M);

/* The whole layer: svdq_quantize_act_lora_down then svdq_w4a4_gemm_lora_up
 * on one stream, intermediates in `workspace` [device] (>=
 * svdq_workspace_bytes(w, M), 1024-byte aligned). */
SVDQ_API svdq_status svdq_linear_forward(const svdq_weights* w, const uint16_t* X, int32_t M, float g_x, void* Y,
                                int32_t out_dtype, void* workspace, size_t ws_bytes, void* stream);

/* svdq_linear_forward whose GEMM is svdq_w4a4_gemm_lora_up_qkv. */
SVDQ_API svdq_status svdq_linear_forward_qkv(const svdq_weights* w, const uint16_t* X, int32_t M, float g_x,
                                    const svdq_qkv_prologue* pro, void* Y, int32_t out_dtype, void* workspace,
                                    size_t ws_bytes, void* stream);

/* The whole layer with the dynamic tensor scale: svdq_quantize_act_lora_down_dyn
 * then svdq_w4a4_gemm_lora_up_dyn.  x_amax [device] as there, or NULL
 * (NVFP4): then svdq_act_amax runs first, into the workspace's amax slot.
 * `pro`, `epi` [host] as in svdq_w4a4_gemm_lora_up_dyn; the quantiser
 * zeroes epi->next_amax, so a chain of layers can alternate two words. */
SVDQ_API svdq_status svdq_linear_forward_dyn(const svdq_weights* w, const uint16_t* X, int32_t M,
                                             const float* x_amax, const svdq_qkv_prologue* pro,
                                             const svdq_epilogue_next* epi, void* Y, int32_t out_dtype,
                                             void* workspace, size_t ws_bytes, void* stream);

/* The layer forward without a caller-provided workspace.  No counterpart
 * in the pages: this exists for callers that cannot allocate device memory
 * at all, for example code that runs under a host framework which owns
 * every device allocation through its own pool and forbids extra ones, or
 * a latency-critical serving loop that must never call cudaMalloc (which
 * can synchronise the device).  The intermediates (codes, scales,
 * lora_act) live in one static device array of 16 MiB that every GPU
 * loading this library holds until the process exits.
 * Same computation and arguments as svdq_linear_forward minus the
 * workspace; returns SVDQ_ERR_WORKSPACE when svdq_workspace_bytes(w, M)
 * plus 1024 bytes of alignment exceeds 16 MiB (e.g. M = 4608 at K = 3072
 * fits; M = 9216 does not).  Allocates nothing: no cudaMalloc, cudaFree
 * or allocating library call.  The first call on each device looks up the
 * array's device address (with that device current), so make that first
 * call before any stream capture.  `w` must have been prepared on the
 * current device, whose copy of the array the call uses (another device's
 * weights give SVDQ_ERR_INVALID_ARG, as do awq_w4a16 weights, before any
 * size check).  All calls on a device share the array
 * and leave the last call's intermediates in it; every call rewrites all
 * it reads, so nothing needs clearing, but calls that overlap on the GPU
 * (other streams, other host threads) race on it. */
SVDQ_API svdq_status svdq_linear_forward_noalloc(const svdq_weights* w, const uint16_t* X, int32_t M, float g_x,
                                                 void* Y, int32_t out_dtype, void* stream);

/* The awq_w4a16 layer (Nunchaku 4-bit in Diffusers: the second kernel
 * family, 4-bit weights with 16-bit activations, for the memory-bound and
 * precision-sensitive modulation projections such as FLUX adanorm_zero /
 * adanorm_single; quantization_config "awq_w4a16": int4, group_size 64).
 * Weights come from svdq_prepare_weights with precision SVDQ_AWQ_W4A16,
 * rank 0, `lambda` = the activation-aware per-input-channel scale alpha
 * (K fp32; ones when there is none): W_til = RN32(W * alpha) quantised by
 * the INT4 group-64 rule of svdq_prepare_weights.  This call computes
 *     Y = X_hat (s_h q)^T + b,   X_hat = RN32(X * RN32(1 / alpha)),
 * with fp32 accumulation, stored as bf16 (RNE) or fp32 (out_dtype).
 * X [device] M x K bf16 (M >= 0, typically the batch), Y [device] M x N.
 * Memory-bound GEMV-shaped work on the CUDA cores; no workspace.  Returns
 * SVDQ_ERR_INVALID_ARG for weights of another precision. */
SVDQ_API svdq_status svdq_awq_w4a16_forward(const svdq_weights* w, const uint16_t* X, int32_t M, void* Y,
                                   int32_t out_dtype, void* stream);

/* Synchronises `stream` and returns (then clears) the status word that the
 * kernels of this weight set write: SVDQ_ERR_TIMEOUT when a bounded wait
 * ran out, SVDQ_ERR_INVALID_ARG when a dynamic tensor scale was not finite
 * and positive, else SVDQ_OK (or SVDQ_ERR_CUDA if the sync failed). */
SVDQ_API svdq_status svdq_device_status(const svdq_weights* w, void* stream);

/* Self-test of the failure path every kernel shares (no counterpart in the
 * pages).  Launches a one-thread kernel whose bounded wait on an mbarrier
 * that nothing arrives on runs out at its limit (2 s of globaltimer) and
 * records SVDQ_ERR_TIMEOUT; synchronises `stream` and returns that status.
 * The kernel neither faults nor traps, so the context stays usable: a
 * healthy library returns SVDQ_ERR_TIMEOUT here (SVDQ_OK would mean the
 * wait completed without its arrival, SVDQ_ERR_CUDA a launch or copy
 * failure, SVDQ_ERR_UNSUPPORTED_DEVICE a device that is not sm_100). */
SVDQ_API svdq_status svdq_selftest_bounded_wait(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H */
