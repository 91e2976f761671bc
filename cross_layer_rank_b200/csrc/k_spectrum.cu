// Eigenvalues (no vectors) of symmetric matrices, for KV-CoRE's effective rank
// (2.B) and the xKV explainer's energy rank (Fig. 2(c)): per problem
//   1. Householder reduction to tridiagonal form in fp64: one cooperative
//      kernel in which the CTAs of a problem share the trailing rows (row i
//      belongs to CTA i mod cpp for the whole reduction) and meet at two
//      bounded grid-group barriers per column;
//   2. bisection on Sturm counts of the tridiagonal matrix, one thread per
//      eigenvalue, down to 1e-15 of the spectrum's span.
// Householder step for column k (x = A[k+1:, k], m = n - k - 1 entries):
//   alpha = -sign(x_0) ||x||, v = x - alpha e_1, beta = 2 / v^T v,
//   p = beta A22 v, K = beta p^T v / 2, w = p - K v, A22 -= v w^T + w v^T,
// leaving d_k = A[k][k] and e_k = alpha.  Both steps are backward stable: the
// eigenvalues come out with errors of a few fp64 ulps of ||A||.
#include <float.h>

#include <algorithm>

#include "xkv_common.cuh"
#include "xkv_internal.h"

namespace xkv {
namespace {

constexpr int kTriThreads = 256;

__device__ double block_sum(double v, double* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = 0.0;
  for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) t += red[i];
  return t;
}

// count problems of size n, A (row-major, full symmetric) overwritten; d, e
// receive the tridiagonal's diagonal (n) and off-diagonal (n - 1) per problem;
// pbuf holds p (n per problem); cpp CTAs per problem.
__global__ void __launch_bounds__(kTriThreads) tridiag_kernel(double* __restrict__ A, int n, int cpp,
                                                               double* __restrict__ d, double* __restrict__ e,
                                                               double* __restrict__ pbuf, GroupBarrier* bars,
                                                               int* status) {
  extern __shared__ double tri_sm[];
  double* v = tri_sm;       // [n]
  double* w = v + n;        // [n]
  double* red = w + n;      // [32]
  const int prob = blockIdx.x / cpp, c = blockIdx.x % cpp;
  double* Ap = A + static_cast<int64_t>(prob) * n * n;
  double* dp = d + static_cast<int64_t>(prob) * n;
  double* ep = e + static_cast<int64_t>(prob) * n;
  double* pp = pbuf + static_cast<int64_t>(prob) * n;
  GroupBarrier* bar = bars + prob;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  for (int k = 0; k + 2 < n; ++k) {
    const int m = n - k - 1;
    // 1. the reflector of column k (every CTA, from row k = column k)
    const double* xk = Ap + static_cast<int64_t>(k) * n + k + 1;
    double ss = 0.0;
    for (int i = tid; i < m; i += blockDim.x) {
      const double x = __ldcg(xk + i);
      v[i] = x;
      ss += x * x;
    }
    const double norm2 = block_sum(ss, red);
    const double x0 = v[0];
    const double alpha = norm2 > 0.0 ? (x0 >= 0.0 ? -sqrt(norm2) : sqrt(norm2)) : 0.0;
    const double v0 = x0 - alpha;
    // v^T v = ||x||^2 - x0^2 + (x0 - alpha)^2 = 2 (||x||^2 + |x0| ||x||), without cancellation
    const double vtv = 2.0 * (norm2 + fabs(x0) * sqrt(norm2));
    const double beta = vtv > 0.0 ? 2.0 / vtv : 0.0;
    __syncthreads();
    if (tid == 0) v[0] = v0;
    if (c == 0 && tid == 0) {
      dp[k] = __ldcg(Ap + static_cast<int64_t>(k) * n + k);
      ep[k] = beta > 0.0 ? alpha : x0;
    }
    __syncthreads();
    // 2. p = beta A22 v for this CTA's rows (a warp per row)
    for (int r = k + 1 + ((c - (k + 1) % cpp + cpp) % cpp) + warp * cpp; r < n; r += nwarps * cpp) {
      const double* row = Ap + static_cast<int64_t>(r) * n + k + 1;
      double s = 0.0;
      for (int j = lane; j < m; j += 32) s += row[j] * v[j];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) pp[r] = beta * s;
    }
    if (!group_barrier(bar, cpp, status)) return;
    // 3. w = p - (beta p^T v / 2) v (every CTA)
    double pv = 0.0;
    for (int i = tid; i < m; i += blockDim.x) {
      const double p = __ldcg(pp + k + 1 + i);
      w[i] = p;
      pv += p * v[i];
    }
    const double K = 0.5 * beta * block_sum(pv, red);
    __syncthreads();
    for (int i = tid; i < m; i += blockDim.x) w[i] -= K * v[i];
    __syncthreads();
    // 4. A22 -= v w^T + w v^T on this CTA's rows
    for (int r = k + 1 + ((c - (k + 1) % cpp + cpp) % cpp) + warp * cpp; r < n; r += nwarps * cpp) {
      double* row = Ap + static_cast<int64_t>(r) * n + k + 1;
      const double vi = v[r - k - 1], wi = w[r - k - 1];
      for (int j = lane; j < m; j += 32) row[j] -= vi * w[j] + wi * v[j];
    }
    if (!group_barrier(bar, cpp, status)) return;
  }
  if (c == 0 && tid == 0) {
    if (n >= 2) {
      dp[n - 2] = __ldcg(Ap + static_cast<int64_t>(n - 2) * n + n - 2);
      ep[n - 2] = __ldcg(Ap + static_cast<int64_t>(n - 1) * n + n - 2);
    }
    dp[n - 1] = __ldcg(Ap + static_cast<int64_t>(n - 1) * n + n - 1);
  }
}

// Number of eigenvalues of the tridiagonal (d, e) below x (Sturm sequence of
// the LDL^T pivots; pivots smaller than pivmin are replaced by -pivmin).
__device__ int sturm_count(const double* d, const double* e2, int n, double x, double pivmin) {
  int cnt = 0;
  double q = d[0] - x;
  if (fabs(q) < pivmin) q = -pivmin;
  cnt += q < 0.0;
  for (int i = 1; i < n; ++i) {
    q = d[i] - x - e2[i - 1] / q;
    if (fabs(q) < pivmin) q = -pivmin;
    cnt += q < 0.0;
  }
  return cnt;
}

// lam[prob][i] = the i-th smallest eigenvalue of problem prob's tridiagonal,
// by bisection of [lo, hi] (Gershgorin) on the Sturm count.
__global__ void __launch_bounds__(256) bisect_kernel(const double* __restrict__ d, const double* __restrict__ e, int n,
                                                     double* __restrict__ lam) {
  extern __shared__ double bis_sm[];
  double* ds = bis_sm;     // [n]
  double* e2 = ds + n;     // [n]
  __shared__ double s_lo, s_hi, s_piv;
  const int prob = blockIdx.y;
  const double* dp = d + static_cast<int64_t>(prob) * n;
  const double* ep = e + static_cast<int64_t>(prob) * n;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    ds[i] = dp[i];
    e2[i] = i + 1 < n ? ep[i] * ep[i] : 0.0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double lo = DBL_MAX, hi = -DBL_MAX, emax = 0.0;
    for (int i = 0; i < n; ++i) {
      const double r = (i > 0 ? fabs(ep[i - 1]) : 0.0) + (i + 1 < n ? fabs(ep[i]) : 0.0);
      lo = fmin(lo, ds[i] - r);
      hi = fmax(hi, ds[i] + r);
      if (i + 1 < n) emax = fmax(emax, e2[i]);
    }
    const double span = fmax(hi - lo, DBL_MIN);
    s_lo = lo - 1e-14 * span;
    s_hi = hi + 1e-14 * span;
    s_piv = DBL_MIN * fmax(1.0, emax);
  }
  __syncthreads();
  // stop once the bracket is below 1e-15 of the Gershgorin span (plus a few
  // ulps of the value): the eigenvalues are then as accurate as the fp64
  // reduction that produced the tridiagonal
  const double tol = 1e-15 * (s_hi - s_lo);
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    double lo = s_lo, hi = s_hi;
    for (int it = 0; it < 80; ++it) {
      const double mid = 0.5 * (lo + hi);
      if (mid <= lo || mid >= hi || hi - lo <= tol + 4.0 * DBL_EPSILON * fabs(mid)) break;
      if (sturm_count(ds, e2, n, mid, s_piv) > i) hi = mid;
      else lo = mid;
    }
    lam[static_cast<int64_t>(prob) * n + i] = 0.5 * (lo + hi);
  }
}

}  // namespace

size_t spectrum_workspace(int n, int count) {
  return align_up(static_cast<size_t>(count) * n * 8) * 3 + align_up(static_cast<size_t>(count) * sizeof(GroupBarrier));
}

xkv_status spectrum_launch(double* W, double* lam, int n, int count, void* ws, cudaStream_t st) {
  int* status = device_status_ptr();
  if (!status) return XKV_ERR_CUDA;
  uint8_t* w = static_cast<uint8_t*>(ws);
  const size_t vec = align_up(static_cast<size_t>(count) * n * 8);
  double* d = reinterpret_cast<double*>(w);
  double* e = reinterpret_cast<double*>(w + vec);
  double* pbuf = reinterpret_cast<double*>(w + 2 * vec);
  GroupBarrier* bars = reinterpret_cast<GroupBarrier*>(w + 3 * vec);
  if (cudaMemsetAsync(bars, 0, static_cast<size_t>(count) * sizeof(GroupBarrier), st) != cudaSuccess)
    return XKV_ERR_CUDA;
  {
    // CTAs per problem: all problems' CTAs resident at once (cooperative launch)
    const size_t smem = static_cast<size_t>(2 * n + 32) * 8;
    if (smem > 227 * 1024) return XKV_ERR_UNSUPPORTED;
    cudaFuncSetAttribute(tridiag_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, tridiag_kernel, kTriThreads, smem) != cudaSuccess ||
        per_sm < 1)
      return XKV_ERR_CUDA;
    const int resident = per_sm * num_sms();
    if (resident < count) return XKV_ERR_UNSUPPORTED;
    const int cpp = std::max(1, std::min({64, resident / count, (n + 7) / 8}));
    void* args[] = {&W, &n, const_cast<int*>(&cpp), &d, &e, &pbuf, &bars, &status};
    if (cudaLaunchCooperativeKernel(reinterpret_cast<void*>(tridiag_kernel), dim3(count * cpp), dim3(kTriThreads),
                                    args, smem, st) != cudaSuccess)
      return XKV_ERR_CUDA;
  }
  const size_t smem2 = static_cast<size_t>(2 * n) * 8;
  cudaFuncSetAttribute(bisect_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem2));
  bisect_kernel<<<dim3((n + 255) / 256, count), 256, smem2, st>>>(d, e, n, lam);
  return cudaPeekAtLastError() == cudaSuccess ? XKV_OK : XKV_ERR_CUDA;
}

}  // namespace xkv
