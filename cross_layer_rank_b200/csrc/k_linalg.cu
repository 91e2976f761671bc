// Small dense linear algebra of the factorisation path, on CUDA cores:
//   - a strided SIMT GEMM (fp32 or fp64 accumulation, optionally split along
//     K with the slices summed in a fixed order) for the Rayleigh-Ritz and
//     Cholesky-QR products and the f32 fall-backs;
//   - shifted Cholesky QR pieces (Gram of a tall block, Cholesky, triangular
//     inverse) in fp64;
//   - a one-sided block Jacobi eigen-solver (fp64) for symmetric positive
//     semi-definite matrices: the Rayleigh-Ritz step (eigenvalues + vectors),
//     all sweeps in one cooperative launch of CTA clusters;
//   - ordering of eigenvalues, and the NER and energy-rank reductions of
//     KV-CoRE's spectra (2.B), whose eigenvalues come from k_spectrum.cu.
#include <cooperative_groups.h>
#include <stdlib.h>

#include <algorithm>

#include "xkv_common.cuh"
#include "xkv_internal.h"
#include "xkv_linalg.cuh"

namespace xkv {

// --------------------------------------------------------------- SIMT GEMM
// 64 x 64 output tile per CTA, 16-deep K slabs through shared memory; the next
// slab's global loads are issued before the current slab's products, so their
// latency overlaps the arithmetic.  Split K (gridDim.z > 1): slice z covers
// K rows [z kchunk, (z + 1) kchunk) and writes alpha * its sum to
// part[z][M][N]; gemm_reduce_kernel then sums the slices in a fixed order
// (deterministic).  lower: tiles wholly above the diagonal are skipped.
template <typename TA, typename TB, typename TC, typename ACC>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const TA* __restrict__ A, int64_t sam, int64_t sak,
                                                        const TB* __restrict__ B, int64_t sbk, int64_t sbn,
                                                        TC* __restrict__ C, int64_t ldc, int M, int N, int K,
                                                        double alpha, double beta, ACC* __restrict__ part,
                                                        int kchunk, int lower) {
  __shared__ ACC As[16][65];
  __shared__ ACC Bs[16][65];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  if (lower && n0 >= m0 + 64) return;
  const int kb = blockIdx.z * kchunk, ke = min(K, kb + kchunk);
  // element q of this thread's share of a slab: A at (kk, mm), B at (kb2, nn);
  // the order makes consecutive threads touch consecutive memory
  auto a_idx = [&](int q, int& kk, int& mm) {
    const int i = threadIdx.x + q * 256;
    if (sam == 1) { mm = i & 63; kk = i >> 6; } else { kk = i & 15; mm = i >> 4; }
  };
  auto b_idx = [&](int q, int& kk, int& nn) {
    const int i = threadIdx.x + q * 256;
    if (sbn == 1) { nn = i & 63; kk = i >> 6; } else { kk = i & 15; nn = i >> 4; }
  };
  ACC ra[4], rb[4];
  auto load = [&](int k0) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      int kk, mm, k2, nn;
      a_idx(q, kk, mm);
      b_idx(q, k2, nn);
      const int m = m0 + mm, k = k0 + kk, n = n0 + nn, kB = k0 + k2;
      ra[q] = (m < M && k < ke) ? static_cast<ACC>(to_f_any(A[m * sam + k * sak])) : ACC(0);
      rb[q] = (n < N && kB < ke) ? static_cast<ACC>(to_f_any(B[kB * sbk + n * sbn])) : ACC(0);
    }
  };
  ACC acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = ACC(0);
  if (kb < ke) load(kb);
  for (int k0 = kb; k0 < ke; k0 += 16) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      int kk, mm, k2, nn;
      a_idx(q, kk, mm);
      b_idx(q, k2, nn);
      As[kk][mm] = ra[q];
      Bs[k2][nn] = rb[q];
    }
    __syncthreads();
    if (k0 + 16 < ke) load(k0 + 16);
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      ACC a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] += a[i] * b[j];
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty + 16 * i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx + 16 * j;
      if (n >= N) continue;
      if (part) {
        part[(static_cast<int64_t>(blockIdx.z) * M + m) * N + n] = static_cast<ACC>(alpha * static_cast<double>(acc[i][j]));
      } else {
        TC* c = C + static_cast<int64_t>(m) * ldc + n;
        const double prev = beta != 0.0 ? static_cast<double>(to_f_any(*c)) : 0.0;
        store_any(c, alpha * static_cast<double>(acc[i][j]) + beta * prev);
      }
    }
  }
}

template <typename TC, typename ACC>
__global__ void gemm_reduce_kernel(const ACC* __restrict__ part, int splits, TC* __restrict__ C, int64_t ldc, int M,
                                   int N, double beta, int lower) {
  const int64_t total = static_cast<int64_t>(M) * N;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int m = static_cast<int>(e / N), n = static_cast<int>(e % N);
    if (lower && (n >> 6) > (m >> 6)) continue;
    double v = 0.0;
    for (int z = 0; z < splits; ++z) v += static_cast<double>(part[z * total + e]);
    TC* c = C + static_cast<int64_t>(m) * ldc + n;
    if (beta != 0.0) v += beta * static_cast<double>(to_f_any(*c));
    store_any(c, v);
  }
}

template <typename TA, typename TB, typename TC, typename ACC>
void gemm_simt(const TA* A, int64_t sam, int64_t sak, const TB* B, int64_t sbk, int64_t sbn, TC* C, int64_t ldc,
               int M, int N, int K, double alpha, double beta, cudaStream_t st) {
  dim3 grid((N + 63) / 64, (M + 63) / 64);
  gemm_simt_kernel<TA, TB, TC, ACC><<<grid, 256, 0, st>>>(A, sam, sak, B, sbk, sbn, C, ldc, M, N, K, alpha, beta,
                                                          nullptr, K, 0);
}

int gemm_splits(int M, int N, int K) {
  const int tiles = ((M + 63) / 64) * ((N + 63) / 64);
  int s = (2 * 148 + tiles - 1) / tiles;
  s = std::min(s, kGemmMaxSplits);
  s = std::min(s, std::max(1, K / 256));
  return std::max(s, 1);
}

template <typename TA, typename TB, typename TC, typename ACC>
void gemm_simt_split(const TA* A, int64_t sam, int64_t sak, const TB* B, int64_t sbk, int64_t sbn, TC* C,
                     int64_t ldc, int M, int N, int K, double alpha, double beta, ACC* part, bool lower,
                     cudaStream_t st) {
  const int splits = gemm_splits(M, N, K);
  if (splits <= 1 || part == nullptr) {
    dim3 grid((N + 63) / 64, (M + 63) / 64);
    gemm_simt_kernel<TA, TB, TC, ACC><<<grid, 256, 0, st>>>(A, sam, sak, B, sbk, sbn, C, ldc, M, N, K, alpha, beta,
                                                            nullptr, K, lower ? 1 : 0);
    return;
  }
  const int kchunk = ((K + splits - 1) / splits + 15) / 16 * 16;
  dim3 grid((N + 63) / 64, (M + 63) / 64, splits);
  gemm_simt_kernel<TA, TB, TC, ACC><<<grid, 256, 0, st>>>(A, sam, sak, B, sbk, sbn, C, ldc, M, N, K, alpha, 0.0,
                                                          part, kchunk, lower ? 1 : 0);
  gemm_reduce_kernel<TC, ACC><<<256, 256, 0, st>>>(part, splits, C, ldc, M, N, beta, lower ? 1 : 0);
}

#define XKV_GEMM_INST(TA, TB, TC, ACC)                                                                        \
  template void gemm_simt<TA, TB, TC, ACC>(const TA*, int64_t, int64_t, const TB*, int64_t, int64_t, TC*, \
                                           int64_t, int, int, int, double, double, cudaStream_t);
XKV_GEMM_INST(float, float, float, float)
XKV_GEMM_INST(__nv_bfloat16, __nv_bfloat16, float, float)
XKV_GEMM_INST(__nv_bfloat16, float, float, float)
XKV_GEMM_INST(__nv_bfloat16, __nv_bfloat16, __nv_bfloat16, float)
XKV_GEMM_INST(float, double, float, double)
XKV_GEMM_INST(float, float, double, double)
XKV_GEMM_INST(float, double, double, double)
XKV_GEMM_INST(double, double, double, double)
#undef XKV_GEMM_INST
template void gemm_simt_split<float, float, double, double>(const float*, int64_t, int64_t, const float*, int64_t,
                                                            int64_t, double*, int64_t, int, int, int, double,
                                                            double, double*, bool, cudaStream_t);

// ---------------------------------------------------- Cholesky QR pieces
// Lower Cholesky factor of (W + shift I), b x b fp64 row-major, in place (only
// the lower triangle is meaningful afterwards), right-looking and blocked by
// kCholNB: per block column k
//   1. chol_diag_kernel  factors the diagonal block in shared memory (one CTA)
//      and writes its inverse to dblk[k];
//   2. chol_panel_kernel  L_ik = W_ik L_kk^{-T} for the rows below (64 rows a CTA);
//   3. the trailing update W_ij -= L_ik L_jk^T as an fp64 GEMM over the whole
//      trailing square (the upper part of W is scratch).
// shift = shift_rel * trace(W) when a device trace is given; it is added to
// each diagonal element when its block is factored.  A non-positive pivot is
// recorded as a numerical fault and replaced by a unit pivot over a zero
// column, so that results stay finite.
constexpr int kCholNB = 64;

// The diagonal block is eliminated in the unscaled (L D L^T) form, one barrier
// per column: a_il -= a_ij a_lj / d_j for j < l <= i; afterwards
// L_ij = a_ij / sqrt(d_j) and L_jj = sqrt(d_j).  Its inverse X = L^{-1} is then
// formed row by row, X_ic = (delta_ic - sum_{c <= k < i} L_ik X_kc) / L_ii, with
// four threads sharing each column's sum.
__global__ void __launch_bounds__(256) chol_diag_kernel(double* __restrict__ W, int b, int k0, double shift_rel,
                                                        const double* __restrict__ trace, int* status,
                                                        double* __restrict__ dinv) {
  extern __shared__ double chol_sm[];
  double(*a)[kCholNB + 1] = reinterpret_cast<double(*)[kCholNB + 1]>(chol_sm);
  double(*x)[kCholNB + 1] = reinterpret_cast<double(*)[kCholNB + 1]>(chol_sm + kCholNB * (kCholNB + 1));
  __shared__ double dg[kCholNB];
  const int tid = threadIdx.x;
  const int nb = min(kCholNB, b - k0);
  const double shift = trace ? shift_rel * (*trace) : 0.0;
  for (int e = tid; e < nb * nb; e += blockDim.x) {
    const int i = e / nb, j = e % nb;
    double v = j <= i ? W[static_cast<int64_t>(k0 + i) * b + k0 + j] : 0.0;
    if (i == j) v += shift;
    a[i][j] = v;
  }
  __syncthreads();
  // thread (ty, tx) of a 16 x 16 grid owns rows ty + 16 u and columns tx + 16 v
  const int ty = tid >> 4, tx = tid & 15;
  for (int j = 0; j < nb; ++j) {
    const double d = a[j][j];
    const bool bad = !(d > 0.0) || !isfinite(d);
    if (tid == 0) {
      dg[j] = bad ? 0.0 : d;
      if (bad) record_status(status, kDevNumerical);
    }
    if (!bad) {
      const double inv = 1.0 / d;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = ty + 16 * u;
        if (i <= j || i >= nb) continue;
        const double aij = a[i][j] * inv;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int l = tx + 16 * v;
          if (l > j && l <= i) a[i][l] -= aij * a[l][j];
        }
      }
    }
    __syncthreads();
  }
  // 1 / L_jj = 1 / sqrt(d_j), once per column (1 for a replaced pivot, whose
  // column below the diagonal is zeroed)
  __shared__ double rl[kCholNB];
  if (tid < nb) rl[tid] = dg[tid] > 0.0 ? rsqrt(dg[tid]) : 1.0;
  __syncthreads();
  for (int e = tid; e < nb * nb; e += blockDim.x) {
    const int i = e / nb, j = e % nb;
    if (j > i) continue;
    const double d = dg[j];
    if (j == i) a[i][i] = d > 0.0 ? sqrt(d) : 1.0;
    else a[i][j] = d > 0.0 ? a[i][j] * rl[j] : 0.0;
  }
  __syncthreads();
  {
    const int c = tid >> 2, q = tid & 3;  // column c, quarter q of its sums
    for (int i = 0; i < nb; ++i) {
      double sm = 0.0;
      if (c < i)
        for (int k = c + q; k < i; k += 4) sm += a[i][k] * x[k][c];
      sm += __shfl_xor_sync(0xffffffffu, sm, 1);
      sm += __shfl_xor_sync(0xffffffffu, sm, 2);
      if (q == 0 && c < nb) x[i][c] = c > i ? 0.0 : ((c == i ? 1.0 : 0.0) - sm) * rl[i];
      __syncthreads();
    }
  }
  for (int e = tid; e < nb * nb; e += blockDim.x) {
    const int i = e / nb, j = e % nb;
    if (j <= i) W[static_cast<int64_t>(k0 + i) * b + k0 + j] = a[i][j];
    dinv[i * kCholNB + j] = x[i][j];
  }
}

// Rows [k0 + nb + 64 blockIdx.x, +64) of block column k: L_ik = W_ik Linv_kk^T.
__global__ void __launch_bounds__(256) chol_panel_kernel(double* __restrict__ W, int b, int k0,
                                                         const double* __restrict__ dinv) {
  extern __shared__ double chol_sm[];
  double(*w)[kCholNB + 1] = reinterpret_cast<double(*)[kCholNB + 1]>(chol_sm);
  double(*x)[kCholNB + 1] = reinterpret_cast<double(*)[kCholNB + 1]>(chol_sm + 64 * (kCholNB + 1));
  const int tid = threadIdx.x;
  const int nb = min(kCholNB, b - k0);
  const int r0 = k0 + nb + 64 * blockIdx.x;
  const int rows = min(64, b - r0);
  for (int e = tid; e < rows * nb; e += blockDim.x) {
    const int i = e / nb, j = e % nb;
    w[i][j] = W[static_cast<int64_t>(r0 + i) * b + k0 + j];
  }
  for (int e = tid; e < nb * nb; e += blockDim.x) x[e / nb][e % nb] = dinv[(e / nb) * kCholNB + e % nb];
  __syncthreads();
  // thread (ty, tx): rows ty + 16 u, columns tx + 16 v of the panel block
  const int ty = tid >> 4, tx = tid & 15;
  double acc[4][4];
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) acc[u][v] = 0.0;
  for (int k = 0; k < nb; ++k) {
    double wv[4], xv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) wv[u] = w[ty + 16 * u][k];
#pragma unroll
    for (int v = 0; v < 4; ++v) xv[v] = x[tx + 16 * v][k];  // zero above the diagonal (k > column)
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[u][v] += wv[u] * xv[v];
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = ty + 16 * u;
    if (i >= rows) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int j = tx + 16 * v;
      if (j < nb) W[static_cast<int64_t>(r0 + i) * b + k0 + j] = acc[u][v];
    }
  }
}

// dblk: one 64 x 64 block per block column (the inverse of its diagonal block)
void cholesky_blocked(double* W, int b, double shift_rel, const double* trace, int* status, double* dblk,
                      cudaStream_t st) {
  const int smem = 2 * 64 * (kCholNB + 1) * 8;
  cudaFuncSetAttribute(chol_diag_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  cudaFuncSetAttribute(chol_panel_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  for (int k0 = 0; k0 < b; k0 += kCholNB) {
    double* dinv = dblk + static_cast<int64_t>(k0 / kCholNB) * kCholNB * kCholNB;
    chol_diag_kernel<<<1, 256, smem, st>>>(W, b, k0, shift_rel, trace, status, dinv);
    const int nb = std::min(kCholNB, b - k0);
    const int rem = b - k0 - nb;
    if (rem <= 0) break;
    chol_panel_kernel<<<(rem + 63) / 64, 256, smem, st>>>(W, b, k0, dinv);
    double* P = W + static_cast<int64_t>(k0 + nb) * b + k0;  // rem x nb panel, row stride b
    gemm_simt<double, double, double, double>(P, b, 1, P, 1, b, W + static_cast<int64_t>(k0 + nb) * b + k0 + nb,
                                              b, rem, rem, nb, -1.0, 1.0, st);
  }
}

// X = L^{-1} for the lower factor L (row-major b x b, the Cholesky above),
// blocked by 64: X_JJ = dblk[J], and for I > J
//   X_IJ = -dblk[I] (sum_{J <= K < I} L_IK X_KJ).
// One CTA per block column J walks I downwards (each X_IJ needs the X_KJ above
// it, written by the same CTA); the strict upper part of X is set to zero.
__global__ void __launch_bounds__(256) tri_inverse_kernel(const double* __restrict__ L,
                                                          const double* __restrict__ dblk, double* X, int b) {
  extern __shared__ double tsm[];
  double(*P)[kCholNB + 1] = reinterpret_cast<double(*)[kCholNB + 1]>(tsm);
  double(*Q)[kCholNB + 1] = reinterpret_cast<double(*)[kCholNB + 1]>(tsm + kCholNB * (kCholNB + 1));
  const int J = blockIdx.x, nblk = (b + kCholNB - 1) / kCholNB;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int j0 = J * kCholNB, nj = min(kCholNB, b - j0);
  for (int e = tid; e < j0 * nj; e += 256) X[static_cast<int64_t>(e / nj) * b + j0 + e % nj] = 0.0;
  for (int e = tid; e < nj * nj; e += 256) {
    const int i = e / nj, c = e % nj;
    X[static_cast<int64_t>(j0 + i) * b + j0 + c] = dblk[static_cast<int64_t>(J) * kCholNB * kCholNB + i * kCholNB + c];
  }
  __syncthreads();
  for (int I = J + 1; I < nblk; ++I) {
    const int i0 = I * kCholNB, ni = min(kCholNB, b - i0);
    double acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
    for (int K = J; K < I; ++K) {  // K < I <= nblk - 1: a full block
      const int kb0 = K * kCholNB;
      for (int e = tid; e < kCholNB * kCholNB; e += 256) {
        const int r = e >> 6, c = e & 63;
        P[r][c] = r < ni ? L[static_cast<int64_t>(i0 + r) * b + kb0 + c] : 0.0;
        Q[r][c] = c < nj ? __ldcg(X + static_cast<int64_t>(kb0 + r) * b + j0 + c) : 0.0;
      }
      __syncthreads();
#pragma unroll 8
      for (int kk = 0; kk < kCholNB; ++kk) {
        double av[4], bv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) av[i] = P[ty + 16 * i][kk];
#pragma unroll
        for (int j = 0; j < 4; ++j) bv[j] = Q[kk][tx + 16 * j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] += av[i] * bv[j];
      }
      __syncthreads();
    }
    // X_IJ = -dblk[I] S
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) Q[ty + 16 * i][tx + 16 * j] = acc[i][j];
    for (int e = tid; e < kCholNB * kCholNB; e += 256) {
      const int r = e >> 6, c = e & 63;  // a partial last block holds ni x ni entries
      P[r][c] = r < ni && c < ni ? dblk[static_cast<int64_t>(I) * kCholNB * kCholNB + e] : 0.0;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
#pragma unroll 8
    for (int kk = 0; kk < kCholNB; ++kk) {
      double av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = P[ty + 16 * i][kk];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Q[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] += av[i] * bv[j];
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = ty + 16 * i;
      if (r >= ni) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = tx + 16 * j;
        if (c < nj) X[static_cast<int64_t>(i0 + r) * b + j0 + c] = -acc[i][j];
      }
    }
    __syncthreads();
  }
}

__global__ void trace_kernel(const double* __restrict__ W, int b, double* __restrict__ out) {
  __shared__ double red[32];
  double s = 0.0;
  for (int i = threadIdx.x; i < b; i += blockDim.x) s += W[static_cast<int64_t>(i) * b + i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) t += red[i];
    *out = t;
  }
}

size_t cholqr_dblk_bytes(int b) {
  return align_up(static_cast<size_t>((b + kCholNB - 1) / kCholNB) * kCholNB * kCholNB * 8);
}

size_t cholqr_part_bytes(int n, int b) {
  const int s = gemm_splits(b, b, n);
  return s > 1 ? align_up(static_cast<size_t>(s) * b * b * 8) : 0;
}

// One pass of (shifted) Cholesky QR: W = Y^T Y (fp64, lower tiles, split K),
// L = chol(W + shift I), Q = Y L^{-T}.  Y, Q: n x b fp32 row-major (distinct
// buffers).
void cholqr_pass(const float* Y, float* Q, int n, int b, double shift_rel, const CholQRScratch& s, int* status,
                 cudaStream_t st) {
  gemm_simt_split<float, float, double, double>(Y, 1, b, Y, b, 1, s.W, b, b, b, n, 1.0, 0.0, s.part, true, st);
  if (shift_rel > 0.0) trace_kernel<<<1, 256, 0, st>>>(s.W, b, s.scal);
  cholesky_blocked(s.W, b, shift_rel, shift_rel > 0.0 ? s.scal : nullptr, status, s.dblk, st);
  const int smem2 = 2 * kCholNB * (kCholNB + 1) * 8;
  cudaFuncSetAttribute(tri_inverse_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2);
  tri_inverse_kernel<<<(b + kCholNB - 1) / kCholNB, 256, smem2, st>>>(s.W, s.dblk, s.Linv, b);
  // Q(m, j) = sum_k Y(m, k) Linv(j, k)
  gemm_simt<float, double, float, double>(Y, b, 1, s.Linv, 1, b, Q, b, n, b, b, 1.0, 0.0, st);
}

// ------------------------------------------------------ one-sided Jacobi
// count independent problems of size n (column-major n x n each; symmetric
// matrices may be given in either order).  Columns are grouped in blocks of
// 16; every round pairs the blocks by the round-robin schedule and each CTA
// orthogonalises the 32 columns of its pair: Gram G = Wc^T Wc, eigenvectors R
// of G by cyclic Jacobi, Wc <- Wc R, Vc <- Vc R.  A sweep is nblk - 1 rounds;
// a sweep that rotates nothing ends the iteration.  On convergence column i of
// W is lambda_i v_i, so |lambda_i| is its norm and v_i is column i of V.
constexpr int kJB = 16;
constexpr int kJacobiInnerSweeps = 1;

// Sweep limit: 40, or XKV_JACOBI_MAX_SWEEPS (a diagnostic override, e.g. 1 to
// see the non-convergence report), at most kJacobiSweepCap.
constexpr int kJacobiSweepCap = 64;

struct JacobiState {
  int converged;
  int pad;
  int active[kJacobiSweepCap];  // pairs rotated in each sweep
  GroupBarrier bar;             // the problem's CTAs (cooperative launch)
};

__device__ __forceinline__ int rr_player(int pos, int round, int nplayers) {
  if (pos == 0) return 0;
  return ((pos - 1 + round) % (nplayers - 1)) + 1;
}

// One round for the pair of CTA blockIdx.x of problem blockIdx.y; rotations
// are counted in state->active[sweep].  W and V are read through L2 (__ldcg):
// in the persistent kernel other CTAs rewrote them since this SM last read.
//
// With nparts > 1 (a cluster of nparts CTAs per pair, cluster rank = part),
// each CTA forms the Gram over its share of the rows and rotates only those
// rows; the partial Grams are added through distributed shared memory in
// rank order, so every CTA of the cluster holds the same Gram and computes
// the same rotation.
__device__ void jacobi_pair(double* __restrict__ W, double* __restrict__ V, int n, int nblk, int round, int sweep,
                            JacobiState* __restrict__ state, double tol, int nparts) {
  __shared__ double G[32][33];   // this CTA's Gram (its rows' share of it when nparts > 1)
  __shared__ double Gt[32][33];  // the pair's Gram, summed over the cluster (nparts > 1)
  __shared__ __align__(16) double R[32][34];  // even row stride: 16-byte pairs R[e][c..c+1]
  __shared__ double tile[64][33];
  __shared__ double cs[16], sn[16];
  __shared__ int pp[16], qq[16];
  const int prob = blockIdx.y;
  JacobiState* stp = state + prob;
  double* Wp = W + static_cast<int64_t>(prob) * n * n;
  double* Vp = V ? V + static_cast<int64_t>(prob) * n * n : nullptr;
  const int pair = blockIdx.x / nparts, part = blockIdx.x % nparts;
  // rows of this CTA: a multiple of 64 per part
  const int rows_per = ((n + nparts - 1) / nparts + 63) / 64 * 64;
  const int r_lo = min(n, part * rows_per), r_hi = min(n, r_lo + rows_per);
  const int I = rr_player(pair, round, nblk), J = rr_player(nblk - 1 - pair, round, nblk);
  const int tid = threadIdx.x;
  __shared__ int cols[32];
  if (tid < 32) {
    const int blk = tid < 16 ? I : J;
    const int c = blk * kJB + (tid & 15);
    cols[tid] = c < n ? c : -1;
  }
  // every thread reads the pair's column list (which the previous round of a
  // persistent CTA left different) only after it is complete
  __syncthreads();
  // Gram of the 32 columns: thread (kg, ti, tj) owns the 4 x 4 block
  // G[4 ti .. 4 ti + 3][4 tj .. 4 tj + 3] over rows kg, kg + 4, ... of each
  // 64-row pass; the four row groups' blocks are then added in a fixed order
  {
    const int kg = tid >> 6, ti = (tid >> 3) & 7, tj = tid & 7;
    double acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
    for (int r0 = r_lo; r0 < r_hi; r0 += 64) {  // 64 rows a pass: 8 loads in flight per thread
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int i = tid + 256 * q;
        const int c = i >> 6, r = i & 63;
        const int cc = cols[c];
        tile[r][c] = (cc >= 0 && r0 + r < r_hi) ? __ldcg(Wp + static_cast<int64_t>(cc) * n + r0 + r) : 0.0;
      }
      __syncthreads();
#pragma unroll 4
      for (int r = kg; r < 64; r += 4) {
        double av[4], bv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) av[i] = tile[r][4 * ti + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) bv[j] = tile[r][4 * tj + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] += av[i] * bv[j];
      }
      __syncthreads();
    }
    for (int g = 0; g < 4; ++g) {
      if (kg == g)
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) G[4 * ti + i][4 * tj + j] = g == 0 ? acc[i][j] : G[4 * ti + i][4 * tj + j] + acc[i][j];
      __syncthreads();
    }
  }
  double(*Gw)[33] = G;
  if (nparts > 1) {
    namespace cg = cooperative_groups;
    cg::cluster_group cl = cg::this_cluster();
    cl.sync();  // every part's Gram is complete
    for (int i = tid; i < 32 * 32; i += 256) {
      double v = 0.0;
      for (int q = 0; q < nparts; ++q) v += cl.map_shared_rank(&G[0][0], q)[(i >> 5) * 33 + (i & 31)];
      Gt[i >> 5][i & 31] = v;
    }
    // (the parts' G stay untouched until the next round, which starts after
    // the grid barrier that every part reaches only after these reads)
    Gw = Gt;
    __syncthreads();
  }
  // the pair is converged when every fresh column product is tiny relative to
  // the column norms: |w_p . w_q| <= tol ||w_p|| ||w_q||
  __shared__ int s_need;
  if (tid == 0) s_need = 0;
  __syncthreads();
  for (int i = tid; i < 32 * 32; i += 256) {
    const int p = i / 32, q = i % 32;
    if (p < q && fabs(Gw[p][q]) > tol * sqrt(fabs(Gw[p][p] * Gw[q][q])) && Gw[p][q] != 0.0) s_need = 1;
  }
  for (int i = tid; i < 32 * 32; i += 256) R[i / 32][i % 32] = (i / 32 == i % 32) ? 1.0 : 0.0;
  __syncthreads();
  if (!s_need) return;
  // cyclic Jacobi on G (round-robin over 32 indices: 31 steps of 16 pairs);
  // entries already below 1e-14 of the diagonal scale are left alone.  At
  // most kJacobiInnerSweeps sweeps: the pair need not be fully diagonalised,
  // since it meets again in the next outer sweep, and the outer test above
  // decides convergence
  for (int sweep = 0; sweep < kJacobiInnerSweeps; ++sweep) {
    __shared__ int s_any;
    if (tid == 0) s_any = 0;
    __syncthreads();
    for (int step = 0; step < 31; ++step) {
      if (tid < 16) {
        int p = rr_player(tid, step, 32), q = rr_player(31 - tid, step, 32);
        if (p > q) { const int t = p; p = q; q = t; }
        pp[tid] = p;
        qq[tid] = q;
        const double gpq = Gw[p][q], gpp = Gw[p][p], gqq = Gw[q][q];
        if (gpq * gpq > 1e-28 * fabs(gpp * gqq) && gpq != 0.0) {
          // t = tan(theta) of the rotation that zeroes gpq, from the difference
          // d = gqq - gpp without forming tau = d / (2 gpq):
          //   t = sign(d) 2 gpq / (|d| + sqrt(d^2 + 4 gpq^2)),
          // then c = (1 + t^2)^(-1/2), s = t c (one division, one square
          // root, one reciprocal square root, all fp64)
          const double d = gqq - gpp;
          const double t = (d >= 0.0 ? 2.0 : -2.0) * gpq / (fabs(d) + sqrt(fma(d, d, 4.0 * gpq * gpq)));
          const double c = rsqrt(fma(t, t, 1.0));
          cs[tid] = c;
          sn[tid] = t * c;
          s_any = 1;
        } else {
          cs[tid] = 1.0;
          sn[tid] = 0.0;
        }
      }
      __syncthreads();
      // columns of G and R
      for (int i = tid; i < 16 * 32; i += 256) {
        const int k = i / 32, r = i % 32;
        const int p = pp[k], q = qq[k];
        const double c = cs[k], s = sn[k];
        if (s == 0.0) continue;
        const double gp = Gw[r][p], gq = Gw[r][q];
        Gw[r][p] = c * gp - s * gq;
        Gw[r][q] = s * gp + c * gq;
        const double rp = R[r][p], rq = R[r][q];
        R[r][p] = c * rp - s * rq;
        R[r][q] = s * rp + c * rq;
      }
      __syncthreads();
      for (int i = tid; i < 16 * 32; i += 256) {
        const int k = i / 32, cidx = i % 32;
        const int p = pp[k], q = qq[k];
        const double c = cs[k], s = sn[k];
        if (s == 0.0) continue;
        const double gp = Gw[p][cidx], gq = Gw[q][cidx];
        Gw[p][cidx] = c * gp - s * gq;
        Gw[q][cidx] = s * gp + c * gq;
      }
      __syncthreads();
    }
    const int any = s_any;
    __syncthreads();
    if (!any) break;
  }
  if (tid == 0 && part == 0) atomicAdd(&stp->active[sweep], 1);
  // Wc <- Wc R, Vc <- Vc R: each thread rotates two rows, r and r + 256, so
  // every 16-byte pair R[e][c..c+1] read from shared memory serves four
  // products (columns beyond n, cols[c] < 0, hold zeros and are not stored)
  for (int mat = 0; mat < (Vp ? 2 : 1); ++mat) {
    double* M = mat == 0 ? Wp : Vp;
    for (int r0 = r_lo; r0 < r_hi; r0 += 512) {
      const int ra = r0 + tid, rb = ra + 256;
      double xa[32], xb[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const int64_t off = static_cast<int64_t>(cols[c]) * n;
        xa[c] = (cols[c] >= 0 && ra < r_hi) ? __ldcg(M + off + ra) : 0.0;
        xb[c] = (cols[c] >= 0 && rb < r_hi) ? __ldcg(M + off + rb) : 0.0;
      }
#pragma unroll 1
      for (int c = 0; c < 32; c += 2) {
        double ya0 = 0.0, ya1 = 0.0, yb0 = 0.0, yb1 = 0.0;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const double2 rv = *reinterpret_cast<const double2*>(&R[e][c]);
          ya0 = fma(xa[e], rv.x, ya0);
          ya1 = fma(xa[e], rv.y, ya1);
          yb0 = fma(xb[e], rv.x, yb0);
          yb1 = fma(xb[e], rv.y, yb1);
        }
        const int c0 = cols[c], c1 = cols[c + 1];
        if (ra < r_hi) {
          if (c0 >= 0) M[static_cast<int64_t>(c0) * n + ra] = ya0;
          if (c1 >= 0) M[static_cast<int64_t>(c1) * n + ra] = ya1;
        }
        if (rb < r_hi) {
          if (c0 >= 0) M[static_cast<int64_t>(c0) * n + rb] = yb0;
          if (c1 >= 0) M[static_cast<int64_t>(c1) * n + rb] = yb1;
        }
      }
    }
  }
}

// Per-round launches (used when the pairs of all problems cannot be resident
// at once): a problem marked converged returns at once.
__global__ void __launch_bounds__(256) jacobi_round_kernel(double* __restrict__ W, double* __restrict__ V, int n,
                                                           int nblk, int round, int sweep,
                                                           JacobiState* __restrict__ state, double tol) {
  if (state[blockIdx.y].converged) return;
  jacobi_pair(W, V, n, nblk, round, sweep, state, tol, 1);
}

__global__ void jacobi_sweep_end_kernel(JacobiState* state, int count, int sweep) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= count) return;
  if (!state[i].converged && state[i].active[sweep] == 0) state[i].converged = 1;
}

// Every sweep in one cooperative launch: the CTAs of a problem (one per pair)
// meet at the problem's bounded barrier after each round; after the last round
// of a sweep all of them read the sweep's rotation count, and a problem that
// rotated nothing is converged.  A barrier that gives up (recorded as a device
// timeout) ends the problem unconverged.
__global__ void __launch_bounds__(256) jacobi_sweeps_kernel(double* __restrict__ W, double* __restrict__ V, int n,
                                                            int nblk, int max_sweeps, JacobiState* __restrict__ state,
                                                            double tol, int* status, int nparts) {
  JacobiState* stp = state + blockIdx.y;
  const unsigned nctas = gridDim.x;  // nparts CTAs (one cluster) per pair
  // the partial Grams are read from the cluster's other CTAs: a launch whose
  // cluster shape is not the one asked for (e.g. under a tool that drops the
  // attribute) touches no distributed shared memory; the problem stays
  // unconverged and is reported as such
  if (nparts > 1 && cooperative_groups::this_cluster().num_blocks() != static_cast<unsigned>(nparts)) {
    if (threadIdx.x == 0) record_status(status, kDevNumerical);
    return;
  }
  for (int sweep = 0; sweep < max_sweeps; ++sweep) {
    for (int round = 0; round < nblk - 1; ++round) {
      jacobi_pair(W, V, n, nblk, round, sweep, state, tol, nparts);
      if (!group_barrier(&stp->bar, nctas, status)) return;
    }
    if (*reinterpret_cast<volatile int*>(&stp->active[sweep]) == 0) {
      if (blockIdx.x == 0 && threadIdx.x == 0) stp->converged = 1;
      return;
    }
  }
}

__global__ void jacobi_init_kernel(double* V, int n, int count, JacobiState* state) {
  const int64_t total = static_cast<int64_t>(count) * n * n;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    if (V) {
      const int64_t w = i % (static_cast<int64_t>(n) * n);
      V[i] = (w / n == w % n) ? 1.0 : 0.0;
    }
    if (i < count) state[i] = JacobiState{};
  }
}

__global__ void column_norms_kernel(const double* __restrict__ W, double* __restrict__ lam, int n, int count) {
  const int prob = blockIdx.y;
  const int c = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (c >= n) return;
  const double* col = W + static_cast<int64_t>(prob) * n * n + static_cast<int64_t>(c) * n;
  double s = 0.0;
  for (int r = lane; r < n; r += 32) s += col[r] * col[r];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) lam[static_cast<int64_t>(prob) * n + c] = sqrt(s);
}

// A problem still rotating after the last sweep has not converged: its
// eigenvalues (and vectors) are not final, which is recorded as a numerical
// fault rather than returned silently.
__global__ void jacobi_check_kernel(const JacobiState* state, int count, int* status) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < count && !state[i].converged) record_status(status, kDevNumerical);
}

size_t jacobi_workspace(int, int count) { return align_up(static_cast<size_t>(count) * sizeof(JacobiState)); }

static int jacobi_max_sweeps() {
  static int v = 0;
  if (v == 0) {
    const char* e = getenv("XKV_JACOBI_MAX_SWEEPS");
    const int x = e ? atoi(e) : 0;
    v = std::min(x > 0 ? x : 40, kJacobiSweepCap);
  }
  return v;
}

xkv_status jacobi_launch(double* W, double* V, double* lam, int n, int count, void* ws, cudaStream_t st) {
  JacobiState* state = static_cast<JacobiState*>(ws);
  int* status = device_status_ptr();
  if (!status) return XKV_ERR_CUDA;
  int nblk = (n + kJB - 1) / kJB;
  if (nblk & 1) ++nblk;
  if (nblk < 2) nblk = 2;
  jacobi_init_kernel<<<256, 256, 0, st>>>(V, n, count, state);
  int max_sweeps = jacobi_max_sweeps();
  double tol = 1e-11;
  // One cooperative launch when every pair of every problem can be resident:
  // with clusters of 4 (else 2) CTAs per pair when that many clusters fit,
  // else one CTA per pair.
  const int npairs = nblk / 2;
  bool launched = false;
  for (int nparts : {4, 2}) {
    if (count > 65535 || n < 64 * nparts) continue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(npairs * nparts, count);
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = nparts;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeCooperative;
    attr[1].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;  // the occupancy query takes the cluster shape only
    int nclusters = 0;
    if (cudaOccupancyMaxActiveClusters(&nclusters, jacobi_sweeps_kernel, &cfg) != cudaSuccess) {
      (void)cudaGetLastError();
      continue;
    }
    if (static_cast<int64_t>(nclusters) < static_cast<int64_t>(npairs) * count) continue;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, jacobi_sweeps_kernel, W, V, n, nblk, max_sweeps, state, tol, status, nparts) ==
        cudaSuccess) {
      launched = true;
      break;
    }
    (void)cudaGetLastError();
  }
  int per_sm = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, jacobi_sweeps_kernel, 256, 0);
  const int64_t ctas = static_cast<int64_t>(npairs) * count;
  if (launched) {
  } else if (per_sm > 0 && ctas <= static_cast<int64_t>(per_sm) * num_sms() && count <= 65535) {
    int one = 1;
    void* args[] = {&W, &V, &n, &nblk, &max_sweeps, &state, &tol, &status, &one};
    if (cudaLaunchCooperativeKernel(reinterpret_cast<void*>(jacobi_sweeps_kernel), dim3(npairs, count), dim3(256),
                                    args, 0, st) != cudaSuccess)
      return XKV_ERR_CUDA;
  } else {
    for (int s = 0; s < max_sweeps; ++s) {
      for (int r = 0; r < nblk - 1; ++r)
        jacobi_round_kernel<<<dim3(nblk / 2, count), 256, 0, st>>>(W, V, n, nblk, r, s, state, tol);
      jacobi_sweep_end_kernel<<<(count + 127) / 128, 128, 0, st>>>(state, count, s);
    }
  }
  jacobi_check_kernel<<<(count + 127) / 128, 128, 0, st>>>(state, count, status);
  column_norms_kernel<<<dim3((n + 7) / 8, count), 256, 0, st>>>(W, lam, n, count);
  return cudaPeekAtLastError() == cudaSuccess ? XKV_OK : XKV_ERR_CUDA;
}

// --------------------------------------------------------------- ordering
// order[k] = index of the k-th largest value (ties: lower index first).
__global__ void order_desc_kernel(const double* __restrict__ v, int n, int* __restrict__ order) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const double x = v[i];
    int rank = 0;
    for (int j = 0; j < n; ++j) {
      const double y = v[j];
      rank += (y > x) || (y == x && j < i);
    }
    order[rank] = i;
  }
}

void order_desc(const double* v, int n, int* order, cudaStream_t st) {
  order_desc_kernel<<<(n + 255) / 256, 256, 0, st>>>(v, n, order);
}

// ------------------------------------------------------------------- NER
// One CTA per block: from |lambda| of the block (unsorted), numerical rank
// r = #{lambda > tol lambda_max}; sigma = sqrt(lambda); p = sigma / sum sigma;
// erank = exp(-sum p ln p); NER = erank / r.
__global__ void __launch_bounds__(256) ner_kernel(const double* __restrict__ lam, int n, double tol,
                                                  float* __restrict__ ner, float* __restrict__ erank,
                                                  int32_t* __restrict__ rank) {
  __shared__ double red[8];
  __shared__ double s_val;
  const double* l = lam + static_cast<int64_t>(blockIdx.x) * n;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  auto block_reduce = [&](double v, bool is_max) -> double {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double w = __shfl_xor_sync(0xffffffffu, v, o);
      v = is_max ? fmax(v, w) : v + w;
    }
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (tid == 0) {
      double t = red[0];
      for (int i = 1; i < 8; ++i) t = is_max ? fmax(t, red[i]) : t + red[i];
      s_val = t;
    }
    __syncthreads();
    const double r = s_val;
    __syncthreads();
    return r;
  };
  double mx = 0.0;
  for (int i = tid; i < n; i += 256) mx = fmax(mx, l[i]);
  const double lmax = block_reduce(mx, true);
  double cnt = 0.0, ssum = 0.0;
  for (int i = tid; i < n; i += 256)
    if (lmax > 0.0 && l[i] > tol * lmax) { cnt += 1.0; ssum += sqrt(l[i]); }
  const double r = block_reduce(cnt, false);
  const double S = block_reduce(ssum, false);
  double h = 0.0;
  for (int i = tid; i < n; i += 256)
    if (lmax > 0.0 && l[i] > tol * lmax) {
      const double p = sqrt(l[i]) / S;
      if (p > 0.0) h -= p * log(p);
    }
  const double H = block_reduce(h, false);
  if (tid == 0) {
    const double er = r > 0.0 ? exp(H) : 0.0;
    ner[blockIdx.x] = static_cast<float>(r > 0.0 ? er / r : 0.0);
    if (erank) erank[blockIdx.x] = static_cast<float>(er);
    if (rank) rank[blockIdx.x] = static_cast<int32_t>(r);
  }
}

// ---------------------------------------------------------- energy rank
// One CTA per block (xKV explainer, Fig. 2(c)): the block's eigenvalues
// (negative ones count as 0) placed in descending order by their rank (ties:
// lower index first), a block-wide prefix sum, and the smallest k whose k
// largest eigenvalues reach `energy` of the total (0 for a zero block).
__global__ void __launch_bounds__(256) energy_rank_kernel(const double* __restrict__ lam, int n, double energy,
                                                          int32_t* __restrict__ rank_out, float* __restrict__ lam_out) {
  extern __shared__ double srt[];  // [n] descending
  __shared__ double wsum[8];
  __shared__ double s_total;
  __shared__ int s_rank;
  const double* l = lam + static_cast<int64_t>(blockIdx.x) * n;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < n; i += blockDim.x) {
    const double x = fmax(l[i], 0.0);
    int pos = 0;
    for (int j = 0; j < n; ++j) {
      const double y = fmax(l[j], 0.0);
      pos += (y > x) || (y == x && j < i);
    }
    srt[pos] = x;
  }
  if (tid == 0) s_rank = n;
  __syncthreads();
  // thread t sums its contiguous run [t c, (t+1) c) of the sorted values
  const int c = (n + blockDim.x - 1) / blockDim.x, i0 = min(n, tid * c), i1 = min(n, i0 + c);
  double run = 0.0;
  for (int i = i0; i < i1; ++i) run += srt[i];
  double incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  double before = 0.0;
  for (int w = 0; w < warp; ++w) before += wsum[w];
  if (tid == 0) {
    double t = 0.0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += wsum[w];
    s_total = t;
  }
  __syncthreads();
  const double total = s_total, target = energy * total;
  double cum = before + incl - run;  // sum of the values ahead of this run
  for (int i = i0; i < i1; ++i) {
    cum += srt[i];
    if (total > 0.0 && cum >= target) {
      atomicMin(&s_rank, i + 1);
      break;
    }
  }
  __syncthreads();
  if (tid == 0) rank_out[blockIdx.x] = total > 0.0 ? s_rank : 0;
  if (lam_out)
    for (int i = tid; i < n; i += blockDim.x) lam_out[static_cast<int64_t>(blockIdx.x) * n + i] = static_cast<float>(srt[i]);
}

// diagonal blocks of an n x n fp32 Gram -> count x (block x block) fp64
__global__ void extract_blocks_kernel(const float* __restrict__ C, int n, int block, double* __restrict__ out) {
  const int b = blockIdx.y;
  const int64_t total = static_cast<int64_t>(block) * block;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(i / block), c = static_cast<int>(i % block);
    out[static_cast<int64_t>(b) * total + i] =
        static_cast<double>(C[static_cast<int64_t>(b * block + r) * n + b * block + c]);
  }
}

size_t ner_workspace(int n, int block) {
  const int count = n / block;
  return align_up(static_cast<size_t>(count) * block * block * 8) + align_up(static_cast<size_t>(count) * block * 8) +
         spectrum_workspace(block, count);
}

xkv_status ner_launch(const float* gram, int n, int block, double tol, float* ner, float* erank, int32_t* rank,
                      void* ws, cudaStream_t st) {
  const int count = n / block;
  uint8_t* w = static_cast<uint8_t*>(ws);
  double* Wb = reinterpret_cast<double*>(w);
  double* lam = reinterpret_cast<double*>(w + align_up(static_cast<size_t>(count) * block * block * 8));
  void* jws = w + align_up(static_cast<size_t>(count) * block * block * 8) + align_up(static_cast<size_t>(count) * block * 8);
  extract_blocks_kernel<<<dim3(128, count), 256, 0, st>>>(gram, n, block, Wb);
  xkv_status s = spectrum_launch(Wb, lam, block, count, jws, st);
  if (s != XKV_OK) return s;
  ner_kernel<<<count, 256, 0, st>>>(lam, block, tol, ner, erank, rank);
  return cudaPeekAtLastError() == cudaSuccess ? XKV_OK : XKV_ERR_CUDA;
}

xkv_status energy_rank_launch(const float* gram, int n, int block, double energy, int32_t* rank, float* lam_out,
                               void* ws, cudaStream_t st) {
  const int count = n / block;
  uint8_t* w = static_cast<uint8_t*>(ws);
  double* Wb = reinterpret_cast<double*>(w);
  double* lam = reinterpret_cast<double*>(w + align_up(static_cast<size_t>(count) * block * block * 8));
  void* jws = w + align_up(static_cast<size_t>(count) * block * block * 8) + align_up(static_cast<size_t>(count) * block * 8);
  extract_blocks_kernel<<<dim3(128, count), 256, 0, st>>>(gram, n, block, Wb);
  xkv_status s = spectrum_launch(Wb, lam, block, count, jws, st);
  if (s != XKV_OK) return s;
  const size_t smem = static_cast<size_t>(block) * 8;
  cudaFuncSetAttribute(energy_rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  energy_rank_kernel<<<count, 256, smem, st>>>(lam, block, energy, rank, lam_out);
  return cudaPeekAtLastError() == cudaSuccess ? XKV_OK : XKV_ERR_CUDA;
}

}  // namespace xkv
