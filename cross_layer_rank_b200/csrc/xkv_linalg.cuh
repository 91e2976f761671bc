// Declarations shared by the factorisation kernels (k_linalg.cu, k_compress.cu).
#pragma once

#include "xkv_common.cuh"

namespace xkv {

__device__ __forceinline__ float to_f_any(float x) { return x; }
__device__ __forceinline__ double to_f_any(double x) { return x; }
__device__ __forceinline__ float to_f_any(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void store_any(float* p, double v) { *p = static_cast<float>(v); }
__device__ __forceinline__ void store_any(double* p, double v) { *p = v; }
__device__ __forceinline__ void store_any(__nv_bfloat16* p, double v) {
  *p = __float2bfloat16_rn(static_cast<float>(v));
}

// C[m][n] = alpha * sum_k A(m,k) B(k,n) + beta * C[m][n] with A(m,k) = A[m sam + k sak]
// and B(k,n) = B[k sbk + n sbn]; ACC is the accumulation type.
template <typename TA, typename TB, typename TC, typename ACC>
void gemm_simt(const TA* A, int64_t sam, int64_t sak, const TB* B, int64_t sbk, int64_t sbn, TC* C, int64_t ldc,
               int M, int N, int K, double alpha, double beta, cudaStream_t st);

// The same product with K split into gemm_splits(M, N, K) slices summed in a
// fixed order through part (gemm_splits x M x N of ACC), for small outputs
// with a long K; lower: only the tiles on or below the diagonal are formed.
constexpr int kGemmMaxSplits = 8;
int gemm_splits(int M, int N, int K);
template <typename TA, typename TB, typename TC, typename ACC>
void gemm_simt_split(const TA* A, int64_t sam, int64_t sak, const TB* B, int64_t sbk, int64_t sbn, TC* C,
                     int64_t ldc, int M, int N, int K, double alpha, double beta, ACC* part, bool lower,
                     cudaStream_t st);

// Scratch of one Cholesky QR pass on an n x b block (all fp64): W and Linv
// b x b, dblk the inverses of the 64 x 64 diagonal blocks of the factor,
// part the split-K slices of the Gram, scal one scalar.
struct CholQRScratch {
  double* W;
  double* Linv;
  double* dblk;
  double* part;
  double* scal;
};
size_t cholqr_dblk_bytes(int b);
size_t cholqr_part_bytes(int n, int b);
void cholqr_pass(const float* Y, float* Q, int n, int b, double shift_rel, const CholQRScratch& s, int* status,
                 cudaStream_t st);

void order_desc(const double* v, int n, int* order, cudaStream_t st);

}  // namespace xkv
