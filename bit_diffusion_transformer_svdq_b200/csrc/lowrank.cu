// Truncated SVD of the smoothed weight on the GPU: the low-rank factors L1,
// L2 of the SVDQuant branch (Nunchaku 4-bit in Diffusers, "Nunchaku und
// SVDQuant": the hardest part of each weight matrix goes to a 16-bit
// low-rank branch; the ai2day page names the method Singular Value
// Decomposition Quantization).  The pages do not spell the factorisation
// out; this is randomized block subspace iteration (Halko, Martinsson and
// Tropp, "Finding structure with randomness", 2011), the same steps as the
// oracle's large-matrix path, from a start block Omega given by the caller:
//
//     A = W_til^T (K x N),  W_til = RN32(W * lambda)
//     Q = orth(A Omega);  q times: Z = orth(A^T Q), Q = orth(A Z)
//     B = Q^T A (ell x N);  B = U_b diag(s) V^T
//     L1 = bf16((Q U_b)_r diag(s_r))^T (r x K),  L2 = bf16(V_r) (N x r)
//
// sm_100a design: offline work dominated by skinny products with the
// weight (N x K against K x ell or N x ell, ell <= 64), done by tiled
// CUDA-core kernels that read W once per product and form W_til on the fly;
// the split reductions over N are added in a fixed order.  orth() is
// Cholesky QR applied twice (Gram matrix in fp64 from fixed-order partial
// sums, one-block Cholesky and triangular inverse in fp64).  The small
// ell x ell eigenproblem B B^T = U_b diag(s^2) U_b^T is cyclic Jacobi in one
// block in fp64.  Every ell-wide array is stored 64 wide (zeros past ell).
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"

namespace svdq {
namespace {

constexpr int kL = 64;       // stored width of every ell-wide array
constexpr int kSplit = 8;    // slices of N in the reductions over N
constexpr int kGramRows = 256;

// Out[N x 64] = W_til In[K x 64] (columns >= ell of In are zero)
__global__ void __launch_bounds__(256) wt_mul_kernel(const float* __restrict__ W, const float* __restrict__ lam, int N,
                                                     int K, const float* __restrict__ In, float* __restrict__ Out) {
  __shared__ float ws[64][33];
  __shared__ float is[32][kL];
  const int n0 = blockIdx.x * 64;
  const int t = threadIdx.x;
  const int row = t >> 2, jb = (t & 3) * 16;
  float acc[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
  for (int k0 = 0; k0 < K; k0 += 32) {
    for (int i = t; i < 64 * 32; i += 256) {
      const int r = i >> 5, c = i & 31, n = n0 + r, k = k0 + c;
      ws[r][c] = (n < N && k < K) ? __fmul_rn(W[static_cast<size_t>(n) * K + k], lam[k]) : 0.0f;
    }
    for (int i = t; i < 32 * kL; i += 256) {
      const int r = i >> 6, c = i & 63, k = k0 + r;
      is[r][c] = k < K ? In[static_cast<size_t>(k) * kL + c] : 0.0f;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < 32; ++kk) {
      const float a = ws[row][kk];
#pragma unroll
      for (int j = 0; j < 16; ++j) acc[j] = __fmaf_rn(a, is[kk][jb + j], acc[j]);
    }
    __syncthreads();
  }
  if (n0 + row < N) {
#pragma unroll
    for (int j = 0; j < 16; ++j) Out[static_cast<size_t>(n0 + row) * kL + jb + j] = acc[j];
  }
}

// Part[s][K x 64] = sum over slice s of n of W_til[n, k] In[n, j]
__global__ void __launch_bounds__(256) wtT_mul_kernel(const float* __restrict__ W, const float* __restrict__ lam, int N,
                                                      int K, const float* __restrict__ In, float* __restrict__ Part) {
  __shared__ float ws[32][65];
  __shared__ float is[32][kL];
  const int k0 = blockIdx.x * 64;
  const int s = blockIdx.y;
  const int nb = static_cast<int>(static_cast<int64_t>(N) * s / kSplit);
  const int ne = static_cast<int>(static_cast<int64_t>(N) * (s + 1) / kSplit);
  const int t = threadIdx.x;
  const int kc = t >> 2, jb = (t & 3) * 16;
  float acc[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
  for (int n0 = nb; n0 < ne; n0 += 32) {
    for (int i = t; i < 32 * 64; i += 256) {
      const int r = i >> 6, c = i & 63, n = n0 + r, k = k0 + c;
      ws[r][c] = (n < ne && k < K) ? __fmul_rn(W[static_cast<size_t>(n) * K + k], lam[k]) : 0.0f;
    }
    for (int i = t; i < 32 * kL; i += 256) {
      const int r = i >> 6, c = i & 63, n = n0 + r;
      is[r][c] = n < ne ? In[static_cast<size_t>(n) * kL + c] : 0.0f;
    }
    __syncthreads();
#pragma unroll 4
    for (int nn = 0; nn < 32; ++nn) {
      const float a = ws[nn][kc];
#pragma unroll
      for (int j = 0; j < 16; ++j) acc[j] = __fmaf_rn(a, is[nn][jb + j], acc[j]);
    }
    __syncthreads();
  }
  if (k0 + kc < K) {
#pragma unroll
    for (int j = 0; j < 16; ++j) Part[(static_cast<size_t>(s) * K + k0 + kc) * kL + jb + j] = acc[j];
  }
}

// Out = sum_s Part[s] in slice order
__global__ void reduce_parts_kernel(const float* __restrict__ Part, int K, float* __restrict__ Out) {
  const size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  const size_t total = static_cast<size_t>(K) * kL;
  if (i >= total) return;
  float v = 0.0f;
  for (int s = 0; s < kSplit; ++s) v = __fadd_rn(v, Part[s * total + i]);
  Out[i] = v;
}

// start block: Z[n, j] = Omega[n * ell + j] (j < ell), zero past ell
__global__ void load_omega_kernel(const float* __restrict__ omega, int N, int ell, float* __restrict__ Z) {
  const size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  if (i >= static_cast<size_t>(N) * kL) return;
  const int n = static_cast<int>(i / kL), j = static_cast<int>(i % kL);
  Z[i] = j < ell ? omega[static_cast<size_t>(n) * ell + j] : 0.0f;
}

// Gp[b][64 x 64] = sum over rows of block b of Y[r, i] Y[r, j] (fp64)
__global__ void __launch_bounds__(256) gram_partial_kernel(const float* __restrict__ Y, int R, double* __restrict__ Gp) {
  __shared__ float ys[64][kL + 1];
  const int t = threadIdx.x;
  const int i = t >> 2, jb = (t & 3) * 16;
  double acc[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j] = 0.0;
  const int r0 = blockIdx.x * kGramRows;
  for (int c0 = r0; c0 < min(R, r0 + kGramRows); c0 += 64) {
    for (int e = t; e < 64 * kL; e += 256) {
      const int r = e >> 6, c = e & 63, row = c0 + r;
      ys[r][c] = row < R ? Y[static_cast<size_t>(row) * kL + c] : 0.0f;
    }
    __syncthreads();
    for (int r = 0; r < 64; ++r) {
      const double a = ys[r][i];
#pragma unroll
      for (int j = 0; j < 16; ++j) acc[j] = __fma_rn(a, static_cast<double>(ys[r][jb + j]), acc[j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) Gp[(static_cast<size_t>(blockIdx.x) * kL + i) * kL + jb + j] = acc[j];
}

__global__ void gram_reduce_kernel(const double* __restrict__ Gp, int blocks, double* __restrict__ G) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= kL * kL) return;
  double v = 0.0;
  for (int b = 0; b < blocks; ++b) v += Gp[static_cast<size_t>(b) * kL * kL + e];
  G[e] = v;
}

// dynamic shared memory of the two one-block kernels: two padded squares
constexpr size_t kSquareSmem = 2 * kL * (kL + 1) * sizeof(double) + kL * sizeof(int);

// G = R^T R (upper R, ell x ell, fp64), then Rinv = R^-1, stored 64 x 64
// with zeros past ell.  One block; the column updates are spread over its
// threads.  A pivot that is not positive (a numerically dependent column)
// is replaced by a tiny positive one so that the factorisation stays finite.

__global__ void __launch_bounds__(64) chol_inv_kernel(const double* __restrict__ G, int ell, double* __restrict__ Rinv) {
  extern __shared__ double sq_smem[];
  double (*R)[kL + 1] = reinterpret_cast<double (*)[kL + 1]>(sq_smem);
  double (*Ri)[kL + 1] = reinterpret_cast<double (*)[kL + 1]>(sq_smem + kL * (kL + 1));
  const int t = threadIdx.x;
  for (int i = 0; i < kL; ++i) {
    R[i][t] = (i < ell && t < ell) ? G[i * kL + t] : 0.0;
    Ri[i][t] = 0.0;
  }
  __syncthreads();
  const double floor_d = 1e-300 + 1e-30 * fabs(R[0][0]);
  for (int k = 0; k < ell; ++k) {
    // row k of R: R[k][k] = sqrt(G[k][k] - sum_{i<k} R[i][k]^2), R[k][j] = (G[k][j] - sum R[i][k] R[i][j]) / R[k][k]
    if (t == 0) {
      double d = R[k][k];
      for (int i = 0; i < k; ++i) d -= R[i][k] * R[i][k];
      R[k][k] = sqrt(d > floor_d ? d : floor_d);
    }
    __syncthreads();
    if (t > k && t < ell) {
      double v = R[k][t];
      for (int i = 0; i < k; ++i) v -= R[i][k] * R[i][t];
      R[k][t] = v / R[k][k];
    }
    __syncthreads();
  }
  // upper-triangular inverse by columns: thread t owns column t of Rinv
  if (t < ell) {
    for (int i = t; i >= 0; --i) {
      double v = (i == t) ? 1.0 : 0.0;
      for (int j = i + 1; j <= t; ++j) v -= R[i][j] * Ri[j][t];
      Ri[i][t] = v / R[i][i];
    }
  }
  __syncthreads();
  for (int i = 0; i < kL; ++i) Rinv[i * kL + t] = (i < ell && t < ell && i <= t) ? Ri[i][t] : 0.0;
}

// Y[r, :] <- Y[r, :] Rinv (upper triangular), fp64 arithmetic, one row per thread
__global__ void __launch_bounds__(128) apply_rinv_kernel(float* __restrict__ Y, int R, int ell,
                                                          const double* __restrict__ Rinv) {
  __shared__ double ri[kL * kL];
  for (int e = threadIdx.x; e < kL * kL; e += blockDim.x) ri[e] = Rinv[e];
  __syncthreads();
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= R) return;
  float* y = Y + static_cast<size_t>(r) * kL;
  double in[kL];
#pragma unroll 16
  for (int i = 0; i < kL; ++i) in[i] = i < ell ? static_cast<double>(y[i]) : 0.0;
  for (int j = 0; j < ell; ++j) {
    double v = 0.0;
    for (int i = 0; i <= j; ++i) v = __fma_rn(in[i], ri[i * kL + j], v);
    y[j] = static_cast<float>(v);
  }
}

// Symmetric eigendecomposition of the ell x ell matrix A (fp64) by cyclic
// Jacobi (one warp; the two rows and columns of each rotation are spread
// over the lanes).  Writes the eigenvalues in decreasing order to ev and the
// matching eigenvectors as the columns of V (64 x 64, zeros past ell).
__global__ void __launch_bounds__(32) jacobi_eig_kernel(const double* __restrict__ Ain, int ell, double* __restrict__ V,
                                                         double* __restrict__ ev) {
  extern __shared__ double sq_smem[];
  double (*A)[kL + 1] = reinterpret_cast<double (*)[kL + 1]>(sq_smem);
  double (*U)[kL + 1] = reinterpret_cast<double (*)[kL + 1]>(sq_smem + kL * (kL + 1));
  int* order = reinterpret_cast<int*>(sq_smem + 2 * kL * (kL + 1));
  const int lane = threadIdx.x;
  for (int i = 0; i < kL; ++i)
    for (int j = lane; j < kL; j += 32) {
      A[i][j] = (i < ell && j < ell) ? Ain[i * kL + j] : 0.0;
      U[i][j] = (i == j) ? 1.0 : 0.0;
    }
  __syncwarp();
  for (int sweep = 0; sweep < 40; ++sweep) {
    double off = 0.0, diag = 0.0;
    for (int i = 0; i < ell; ++i)
      for (int j = lane; j < ell; j += 32) {
        if (i != j) off += A[i][j] * A[i][j];
        else diag += A[i][i] * A[i][i];
      }
    for (int o = 16; o > 0; o >>= 1) {
      off += __shfl_xor_sync(0xFFFFFFFFu, off, o);
      diag += __shfl_xor_sync(0xFFFFFFFFu, diag, o);
    }
    if (off <= 1e-30 * diag || off == 0.0) break;
    for (int p = 0; p < ell - 1; ++p)
      for (int q = p + 1; q < ell; ++q) {
        const double apq = A[p][q];
        if (apq == 0.0) continue;  // uniform across the warp
        const double app = A[p][p], aqq = A[q][q];
        const double theta = (aqq - app) / (2.0 * apq);
        const double tt = (theta >= 0 ? 1.0 : -1.0) / (fabs(theta) + sqrt(theta * theta + 1.0));
        const double c = 1.0 / sqrt(tt * tt + 1.0), s = tt * c;
        __syncwarp();
        // A <- J^T A J with J the rotation in the (p, q) plane
        for (int k = lane; k < ell; k += 32) {
          const double akp = A[k][p], akq = A[k][q];
          A[k][p] = c * akp - s * akq;
          A[k][q] = s * akp + c * akq;
        }
        __syncwarp();
        for (int k = lane; k < ell; k += 32) {
          const double apk = A[p][k], aqk = A[q][k];
          A[p][k] = c * apk - s * aqk;
          A[q][k] = s * apk + c * aqk;
          const double ukp = U[k][p], ukq = U[k][q];
          U[k][p] = c * ukp - s * ukq;
          U[k][q] = s * ukp + c * ukq;
        }
        __syncwarp();
      }
  }
  if (lane == 0) {  // order by decreasing eigenvalue (selection sort; ell <= 64)
    for (int i = 0; i < ell; ++i) order[i] = i;
    for (int i = 0; i < ell; ++i) {
      int b = i;
      for (int j = i + 1; j < ell; ++j)
        if (A[order[j]][order[j]] > A[order[b]][order[b]]) b = j;
      const int tmp = order[i];
      order[i] = order[b];
      order[b] = tmp;
    }
  }
  __syncwarp();
  for (int i = 0; i < kL; ++i) {
    for (int j = lane; j < kL; j += 32) V[i * kL + j] = (i < ell && j < ell) ? U[i][order[j]] : 0.0;
  }
  for (int j = lane; j < kL; j += 32) ev[j] = j < ell ? A[order[j]][order[j]] : 0.0;
}

// L1[t, k] = bf16(s_t sum_j Q[k, j] Ub[j, t]),  t < r
__global__ void l1_out_kernel(const float* __restrict__ Q, int K, int r, int ell, const double* __restrict__ Ub,
                              const double* __restrict__ ev, __nv_bfloat16* __restrict__ L1) {
  const size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  if (i >= static_cast<size_t>(r) * K) return;
  const int t = static_cast<int>(i / K), k = static_cast<int>(i % K);
  double v = 0.0;
  for (int j = 0; j < ell; ++j) v = __fma_rn(static_cast<double>(Q[static_cast<size_t>(k) * kL + j]), Ub[j * kL + t], v);
  const double s = sqrt(ev[t] > 0.0 ? ev[t] : 0.0);
  L1[i] = __float2bfloat16_rn(static_cast<float>(v * s));
}

// L2[n, t] = bf16(sum_j Bt[n, j] Ub[j, t] / s_t),  zero when s_t is 0
__global__ void l2_out_kernel(const float* __restrict__ Bt, int N, int r, int ell, const double* __restrict__ Ub,
                              const double* __restrict__ ev, __nv_bfloat16* __restrict__ L2) {
  const size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  if (i >= static_cast<size_t>(N) * r) return;
  const int n = static_cast<int>(i / r), t = static_cast<int>(i % r);
  double v = 0.0;
  for (int j = 0; j < ell; ++j) v = __fma_rn(static_cast<double>(Bt[static_cast<size_t>(n) * kL + j]), Ub[j * kL + t], v);
  const double s = sqrt(ev[t] > 0.0 ? ev[t] : 0.0);
  L2[i] = __float2bfloat16_rn(s > 0.0 ? static_cast<float>(v / s) : 0.0f);
}

struct LowrankWs {
  float *Q, *Z, *part;
  double *gp, *G, *Rinv, *Ub, *ev;
};

size_t ws_layout(int N, int K, LowrankWs* w, void* base) {
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = static_cast<size_t>(round_up(static_cast<int64_t>(off + bytes), 256));
    return at;
  };
  const size_t q = take(static_cast<size_t>(K) * kL * 4);
  const size_t z = take(static_cast<size_t>(N) * kL * 4);
  const size_t part = take(static_cast<size_t>(kSplit) * K * kL * 4);
  const int blocks = (std::max(N, K) + kGramRows - 1) / kGramRows;
  const size_t gp = take(static_cast<size_t>(blocks) * kL * kL * 8);
  const size_t g = take(kL * kL * 8), ri = take(kL * kL * 8), ub = take(kL * kL * 8), ev = take(kL * 8);
  if (w && base) {
    uint8_t* b = static_cast<uint8_t*>(base);
    w->Q = reinterpret_cast<float*>(b + q);
    w->Z = reinterpret_cast<float*>(b + z);
    w->part = reinterpret_cast<float*>(b + part);
    w->gp = reinterpret_cast<double*>(b + gp);
    w->G = reinterpret_cast<double*>(b + g);
    w->Rinv = reinterpret_cast<double*>(b + ri);
    w->Ub = reinterpret_cast<double*>(b + ub);
    w->ev = reinterpret_cast<double*>(b + ev);
  }
  return off;
}

// Y (R x 64) <- an orthonormal basis of its first ell columns: Cholesky QR, twice
cudaError_t orth(float* Y, int R, int ell, const LowrankWs& w, cudaStream_t s) {
  const int blocks = (R + kGramRows - 1) / kGramRows;
  for (int pass = 0; pass < 2; ++pass) {
    gram_partial_kernel<<<blocks, 256, 0, s>>>(Y, R, w.gp);
    gram_reduce_kernel<<<(kL * kL + 255) / 256, 256, 0, s>>>(w.gp, blocks, w.G);
    chol_inv_kernel<<<1, kL, kSquareSmem, s>>>(w.G, ell, w.Rinv);
    apply_rinv_kernel<<<(R + 127) / 128, 128, 0, s>>>(Y, R, ell, w.Rinv);
  }
  return cudaGetLastError();
}

cudaError_t mul_wt(const float* W, const float* lam, int N, int K, const float* In, float* Out, cudaStream_t s) {
  wt_mul_kernel<<<(N + 63) / 64, 256, 0, s>>>(W, lam, N, K, In, Out);
  return cudaGetLastError();
}

cudaError_t mul_wtT(const float* W, const float* lam, int N, int K, const float* In, float* Out, const LowrankWs& w,
                    cudaStream_t s) {
  wtT_mul_kernel<<<dim3((K + 63) / 64, kSplit), 256, 0, s>>>(W, lam, N, K, In, w.part);
  const size_t total = static_cast<size_t>(K) * kL;
  reduce_parts_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, s>>>(w.part, K, Out);
  return cudaGetLastError();
}

}  // namespace

size_t lowrank_workspace_bytes(int N, int K) { return ws_layout(N, K, nullptr, nullptr); }

cudaError_t launch_lowrank(const float* W, int N, int K, const float* lambda, int rank, int ell, int power_steps,
                           const float* omega, uint16_t* L1, uint16_t* L2, void* workspace, cudaStream_t s) {
  LowrankWs w;
  ws_layout(N, K, &w, workspace);
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(chol_inv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(kSquareSmem))) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(jacobi_eig_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(kSquareSmem))) != cudaSuccess)
    return e;
  // Q = orth(A Omega), A Omega = W_til^T Omega
  load_omega_kernel<<<static_cast<unsigned>((static_cast<size_t>(N) * kL + 255) / 256), 256, 0, s>>>(omega, N, ell, w.Z);
  if ((e = mul_wtT(W, lambda, N, K, w.Z, w.Q, w, s)) != cudaSuccess) return e;
  if ((e = orth(w.Q, K, ell, w, s)) != cudaSuccess) return e;
  for (int it = 0; it < power_steps; ++it) {
    if ((e = mul_wt(W, lambda, N, K, w.Q, w.Z, s)) != cudaSuccess) return e;  // A^T Q
    if ((e = orth(w.Z, N, ell, w, s)) != cudaSuccess) return e;
    if ((e = mul_wtT(W, lambda, N, K, w.Z, w.Q, w, s)) != cudaSuccess) return e;  // A Z
    if ((e = orth(w.Q, K, ell, w, s)) != cudaSuccess) return e;
  }
  // B^T = A^T Q = W_til Q (N x ell);  B B^T = Bt^T Bt
  if ((e = mul_wt(W, lambda, N, K, w.Q, w.Z, s)) != cudaSuccess) return e;
  const int blocks = (N + kGramRows - 1) / kGramRows;
  gram_partial_kernel<<<blocks, 256, 0, s>>>(w.Z, N, w.gp);
  gram_reduce_kernel<<<(kL * kL + 255) / 256, 256, 0, s>>>(w.gp, blocks, w.G);
  jacobi_eig_kernel<<<1, 32, kSquareSmem, s>>>(w.G, ell, w.Ub, w.ev);
  l1_out_kernel<<<static_cast<unsigned>((static_cast<size_t>(rank) * K + 255) / 256), 256, 0, s>>>(
      w.Q, K, rank, ell, w.Ub, w.ev, reinterpret_cast<__nv_bfloat16*>(L1));
  l2_out_kernel<<<static_cast<unsigned>((static_cast<size_t>(N) * rank + 255) / 256), 256, 0, s>>>(
      w.Z, N, rank, ell, w.Ub, w.ev, reinterpret_cast<__nv_bfloat16*>(L2));
  return cudaGetLastError();
}

}  // namespace svdq
