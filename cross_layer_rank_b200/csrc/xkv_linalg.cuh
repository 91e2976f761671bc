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

void cholqr_pass(const float* Y, float* Q, int n, int b, double shift_rel, double* W, double* Linv, double* scal,
                 int* status, cudaStream_t st);

void order_desc(const double* v, int n, int* order, cudaStream_t st);

}  // namespace xkv
