// Full reconstruction, dense decode attention and chunk landmarks.
//   - full reconstruction (the comparison path of the xKV explainer's Fig. 6):
//     out = A Bt^T (+ RoPE per head) for every row, on tcgen05 for bf16;
//   - dense decode attention over a full cache (KQ-SVD page, 3.2), split over
//     tokens with an online-softmax merge;
//   - landmarks for the top-k chunk selector (xKV explainer, "选择性重建"): the
//     mean of each middle chunk's post-RoPE keys.
#include <algorithm>

#include "k_gemm_tc.cuh"
#include "xkv_common.cuh"
#include "xkv_internal.h"
#include "xkv_linalg.cuh"

namespace xkv {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kMaxGQ = 8;

// CUDA-core reconstruction (f32 and shapes outside the tensor-core path): one
// thread per output pair (t, head, j): y0 = A[t] . Bt[h hd + j], y1 = A[t] .
// Bt[h hd + j + hd/2], rotated when RoPE applies, rounded once to the output.
template <typename T>
__global__ void __launch_bounds__(256) recon_simt_kernel(const T* __restrict__ A, const T* __restrict__ Bt,
                                                         int64_t rows, int rank, int d, int hd, int apply_rope,
                                                         float theta, T* __restrict__ out) {
  const int half = hd / 2;
  const int64_t total = rows * (d / 2);
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / (d / 2);
    const int pr = static_cast<int>(i % (d / 2));
    const int h = pr / half, j = pr % half;
    const T* a = A + t * rank;
    const T* b0 = Bt + static_cast<int64_t>(h * hd + j) * rank;
    const T* b1 = Bt + static_cast<int64_t>(h * hd + j + half) * rank;
    float y0 = 0.f, y1 = 0.f;
    for (int c = 0; c < rank; ++c) {
      const float av = to_f(a[c]);
      y0 = fmaf(av, to_f(b0[c]), y0);
      y1 = fmaf(av, to_f(b1[c]), y1);
    }
    if (apply_rope) {
      float cs, sn;
      rope_cs(rope_turns(theta, j, hd), static_cast<double>(t), &cs, &sn);
      const float r0 = y0 * cs - y1 * sn, r1 = y1 * cs + y0 * sn;
      y0 = r0;
      y1 = r1;
    }
    T* o = out + t * d + h * hd;
    store_f(o + j, y0);
    store_f(o + j + half, y1);
  }
}

// ------------------------------------------------------------ dense decode
// CTA (split, unit): tokens [t0, t1) of one KV head; 256 rows per pass, one
// thread scores one row; values are accumulated by (column pair, row group).
__device__ __forceinline__ void load2(const __nv_bfloat16* p, float* x) {
  const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
  x[0] = f.x;
  x[1] = f.y;
}
__device__ __forceinline__ void load2(const float* p, float* x) {
  const float2 f = *reinterpret_cast<const float2*>(p);
  x[0] = f.x;
  x[1] = f.y;
}
__device__ __forceinline__ void store2(__nv_bfloat16* p, float a, float b) {
  *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b);
}
__device__ __forceinline__ void store2(float* p, float a, float b) { *reinterpret_cast<float2*>(p) = make_float2(a, b); }

template <typename T>
__global__ void __launch_bounds__(256) dense_partial_kernel(const T* __restrict__ q, const T* __restrict__ K,
                                                            const T* __restrict__ V, int64_t Tn, int Hq, int Hkv,
                                                            int hd, int64_t per_split, float* __restrict__ part) {
  extern __shared__ float sm[];
  const int gq = Hq / Hkv;
  const int u = blockIdx.y, b = u / Hkv, h = u % Hkv, split = blockIdx.x;
  const int d = Hkv * hd;
  float* qs = sm;                    // [gq][hd]
  float* ps = qs + gq * hd;          // [256][gq]
  float* red = ps + 256 * gq;        // [8][gq]
  float* ms = red + 8 * kMaxGQ;      // [gq]
  float* ls = ms + kMaxGQ;           // [gq]
  float* al = ls + kMaxGQ;           // [gq]
  float* oacc = al + kMaxGQ;         // [rgroups][gq][hd]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float qscale = rsqrtf(static_cast<float>(hd)) * kLog2e;
  for (int i = tid; i < gq * hd; i += 256) qs[i] = to_f(q[(static_cast<int64_t>(b) * Hq + h * gq) * hd + i]) * qscale;
  if (tid < gq) { ms[tid] = -INFINITY; ls[tid] = 0.f; }
  const int cpairs = hd / 2, rgroups = 256 / cpairs;
  const int cp = tid % cpairs, rg = tid / cpairs;
  float acc[kMaxGQ][2];
#pragma unroll
  for (int g = 0; g < kMaxGQ; ++g) acc[g][0] = acc[g][1] = 0.f;
  __syncthreads();
  const int64_t t0 = split * per_split, t1 = std::min<int64_t>(Tn, t0 + per_split);
  for (int64_t tb = t0; tb < t1; tb += 256) {
    const int nr = static_cast<int>(std::min<int64_t>(256, t1 - tb));
    float s[kMaxGQ];
#pragma unroll
    for (int g = 0; g < kMaxGQ; ++g) s[g] = -INFINITY;
    if (tid < nr) {
      const T* kr = K + (static_cast<int64_t>(b) * Tn + tb + tid) * d + h * hd;
#pragma unroll
      for (int g = 0; g < kMaxGQ; ++g) s[g] = 0.f;
      if (sizeof(T) == 2 && hd % 8 == 0 && d % 8 == 0) {
        // the row in 16-byte vectors (8 values per load)
        for (int j0 = 0; j0 < hd; j0 += 64) {
          // eight vectors' loads in flight before their use
          uint4 w[8];
#pragma unroll
          for (int v = 0; v < 8; ++v)
            w[v] = j0 + 8 * v < hd ? *reinterpret_cast<const uint4*>(kr + j0 + 8 * v) : make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            if (j0 + 8 * v >= hd) break;
            const uint32_t ww[4] = {w[v].x, w[v].y, w[v].z, w[v].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 kv = bf2_to_f2(ww[e]);
              const int j = j0 + 8 * v + 2 * e;
#pragma unroll
              for (int g = 0; g < kMaxGQ; ++g)
                if (g < gq) s[g] = fmaf(qs[g * hd + j], kv.x, fmaf(qs[g * hd + j + 1], kv.y, s[g]));
            }
          }
        }
      } else {
        for (int j = 0; j < hd; ++j) {
          const float kv = to_f(kr[j]);
#pragma unroll
          for (int g = 0; g < kMaxGQ; ++g)
            if (g < gq) s[g] = fmaf(qs[g * hd + j], kv, s[g]);
        }
      }
    }
#pragma unroll
    for (int g = 0; g < kMaxGQ; ++g) {
      if (g >= gq) break;
      const float w = warp_max(s[g]);
      if (lane == 0) red[warp * kMaxGQ + g] = w;
    }
    __syncthreads();
    if (tid < gq) {
      float mx = ms[tid];
      for (int i = 0; i < 8; ++i) mx = fmaxf(mx, red[i * kMaxGQ + tid]);
      al[tid] = exp2f(ms[tid] - mx);
      ms[tid] = mx;
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < kMaxGQ; ++g) {
      if (g >= gq) break;
      const float p = tid < nr ? exp2f(s[g] - ms[g]) : 0.f;
      ps[tid * gq + g] = p;
      const float w = warp_sum(p);
      if (lane == 0) red[warp * kMaxGQ + g] = w;
    }
    __syncthreads();
    if (tid < gq) {
      float sum = 0.f;
      for (int i = 0; i < 8; ++i) sum += red[i * kMaxGQ + tid];
      ls[tid] = ls[tid] * al[tid] + sum;
    }
#pragma unroll
    for (int g = 0; g < kMaxGQ; ++g) {
      if (g >= gq) break;
      acc[g][0] *= al[g];
      acc[g][1] *= al[g];
    }
    for (int r = rg; r < nr; r += rgroups) {
      const T* vr = V + (static_cast<int64_t>(b) * Tn + tb + r) * d + h * hd + 2 * cp;
      float vv[2];
      load2(vr, vv);
      const float v0 = vv[0], v1 = vv[1];
#pragma unroll
      for (int g = 0; g < kMaxGQ; ++g) {
        if (g >= gq) break;
        const float p = ps[r * gq + g];
        acc[g][0] = fmaf(p, v0, acc[g][0]);
        acc[g][1] = fmaf(p, v1, acc[g][1]);
      }
    }
    __syncthreads();
  }
  for (int g = 0; g < gq; ++g) {
    oacc[(rg * gq + g) * hd + 2 * cp] = acc[g][0];
    oacc[(rg * gq + g) * hd + 2 * cp + 1] = acc[g][1];
  }
  __syncthreads();
  const int slot_floats = 2 * kMaxGQ + gq * hd;
  float* slot = part + (static_cast<int64_t>(u) * gridDim.x + split) * slot_floats;
  for (int i = tid; i < gq * hd; i += 256) {
    float o = 0.f;
    for (int r = 0; r < rgroups; ++r) o += oacc[r * gq * hd + i];
    slot[2 * kMaxGQ + i] = o;
  }
  if (tid < gq) { slot[tid] = ms[tid]; slot[kMaxGQ + tid] = ls[tid]; }
}

__global__ void dense_combine_kernel(const float* __restrict__ part, int splits, int gq, int hd, float* __restrict__ out) {
  const int u = blockIdx.x;
  const int slot_floats = 2 * kMaxGQ + gq * hd;
  const float* base = part + static_cast<int64_t>(u) * splits * slot_floats;
  for (int i = threadIdx.x; i < gq * hd; i += blockDim.x) {
    const int g = i / hd;
    float M = -INFINITY;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, base[s * slot_floats + g]);
    float L = 0.f, O = 0.f;
    for (int s = 0; s < splits; ++s) {
      const float* sl = base + s * slot_floats;
      const float f = sl[g] == -INFINITY ? 0.f : exp2f(sl[g] - M);
      L += sl[kMaxGQ + g] * f;
      O += sl[2 * kMaxGQ + i] * f;
    }
    out[static_cast<int64_t>(u) * gq * hd + i] = O / L;
  }
}

void dense_split(const xkv_dense_params* p, int* splits, int64_t* per) {
  const int units = p->batch * p->n_kv_heads;
  int s = std::max(1, (4 * num_sms() + units - 1) / units);
  int64_t pr = (p->T + s - 1) / s;
  pr = (pr + 255) / 256 * 256;
  s = static_cast<int>((p->T + pr - 1) / pr);
  *splits = std::max(1, s);
  *per = pr;
}

// --------------------------------------------------------------- landmarks

template <typename T>
__global__ void __launch_bounds__(256) landmarks_kernel(const T* __restrict__ K, int64_t ldk, int hd, int chunk,
                                                        int sink, int64_t n_mid, float theta, int chunks_per_block,
                                                        T* __restrict__ out) {
  __shared__ double ft[128];
  const int h = blockIdx.y, half = hd / 2;
  for (int j = threadIdx.x; j < half; j += blockDim.x) ft[j] = rope_turns(theta, j, hd);
  __syncthreads();
  const int lanes = 256 / half;  // chunks handled in parallel
  const int j = threadIdx.x % half, cl = threadIdx.x / half;
  if (cl >= lanes) return;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * chunks_per_block;
  const int64_t c1 = std::min<int64_t>(n_mid, c0 + chunks_per_block);
  const float inv = 1.0f / static_cast<float>(chunk);
  for (int64_t c = c0 + cl; c < c1; c += lanes) {
    float a0 = 0.f, a1 = 0.f;
    for (int e = 0; e < chunk; ++e) {
      const int64_t t = sink + c * chunk + e;
      const T* kr = K + t * ldk + h * hd;
      const float x0 = to_f(kr[j]), x1 = to_f(kr[j + half]);
      float cs, sn;
      rope_cs(ft[j], static_cast<double>(t), &cs, &sn);
      a0 = fmaf(x0, cs, fmaf(-x1, sn, a0));
      a1 = fmaf(x1, cs, fmaf(x0, sn, a1));
    }
    T* o = out + (static_cast<int64_t>(h) * n_mid + c) * hd;
    store_f(o + j, a0 * inv);
    store_f(o + j + half, a1 * inv);
  }
}

// Same landmarks, one warp per chunk: lane l owns the frequency pairs
// (2l, 2l + 1) (+ 64 per further pass) and reads them as 2-element vectors;
// the angle of token t0 + e is the chunk's base angle (one turn reduction per
// chunk and frequency) rotated by the offset e from a shared table (angle
// addition), so a chunk costs one sin/cos pair per frequency instead of one
// per token.
constexpr int kLmRotMax = 40 * 1024;  // rotation table bytes: chunk x half x (cos, sin), under the 48 KiB default

template <typename T>
__global__ void __launch_bounds__(256) landmarks_rot_kernel(const T* __restrict__ K, int64_t ldk, int hd, int chunk,
                                                            int sink, int64_t n_mid, float theta,
                                                            int chunks_per_block, T* __restrict__ out) {
  extern __shared__ float2 rot[];  // [chunk][half] (cos, sin) of e f_j turns
  __shared__ double ft[128];
  const int h = blockIdx.y, half = hd / 2;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int j = threadIdx.x; j < half; j += blockDim.x) ft[j] = rope_turns(theta, j, hd);
  __syncthreads();
  for (int i = threadIdx.x; i < chunk * half; i += blockDim.x) {
    float c, sn;
    rope_cs(ft[i % half], static_cast<double>(i / half), &c, &sn);
    rot[i] = make_float2(c, sn);
  }
  __syncthreads();
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * chunks_per_block;
  const int64_t c1 = min(n_mid, c0 + chunks_per_block);
  const float inv = 1.0f / static_cast<float>(chunk);
  for (int64_t c = c0 + warp; c < c1; c += nwarps) {
    const int64_t t0 = sink + c * chunk;
    T* o = out + (static_cast<int64_t>(h) * n_mid + c) * hd;
    for (int jp = 2 * lane; jp < half; jp += 64) {
      float bc[2], bs[2];
      rope_cs(ft[jp], static_cast<double>(t0), &bc[0], &bs[0]);
      rope_cs(ft[jp + 1], static_cast<double>(t0), &bc[1], &bs[1]);
      float a0[2] = {0.f, 0.f}, a1[2] = {0.f, 0.f};
      for (int e = 0; e < chunk; ++e) {
        const T* kr = K + (t0 + e) * ldk + h * hd;
        float x0[2], x1[2];
        load2(kr + jp, x0);
        load2(kr + jp + half, x1);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const float2 r = rot[e * half + jp + q];
          const float cs = bc[q] * r.x - bs[q] * r.y;
          const float sn = bs[q] * r.x + bc[q] * r.y;
          a0[q] = fmaf(x0[q], cs, fmaf(-x1[q], sn, a0[q]));
          a1[q] = fmaf(x1[q], cs, fmaf(x0[q], sn, a1[q]));
        }
      }
      store2(o + jp, a0[0] * inv, a0[1] * inv);
      store2(o + jp + half, a1[0] * inv, a1[1] * inv);
    }
  }
}

bool recon_tc_ok(int rank, int d, int hd, int apply_rope, xkv_dtype dt) {
  if (dt != XKV_BF16 || rank % 64 != 0 || d % 64 != 0 || force_simt()) return false;
  const int bn = d % 128 == 0 ? 128 : 64;
  if (apply_rope && (bn % hd != 0 || hd % 32 != 0)) return false;
  return true;
}

}  // namespace

xkv_status recon_launch(const void* A, const void* Bt, int64_t T, int rank, int d, int hkv, int hd, int apply_rope,
                        float theta, xkv_dtype dt, void* out, cudaStream_t st) {
  if (T == 0) return XKV_OK;
  (void)hkv;
  if (recon_tc_ok(rank, d, hd, apply_rope, dt)) {
    const int bn = d % 128 == 0 ? 128 : 64;
    TmapSet am;
    CUtensorMap bm;
    {
      const uint64_t dims[2] = {static_cast<uint64_t>(rank), static_cast<uint64_t>(T)};
      const uint64_t str[1] = {static_cast<uint64_t>(rank) * 2};
      const uint32_t box[2] = {64, 128};
      if (!make_tmap(&am.m[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, A, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
        return XKV_ERR_CUDA;
    }
    {
      const uint64_t dims[2] = {static_cast<uint64_t>(rank), static_cast<uint64_t>(d)};
      const uint64_t str[1] = {static_cast<uint64_t>(rank) * 2};
      const uint32_t box[2] = {64, static_cast<uint32_t>(bn)};
      if (!make_tmap(&bm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Bt, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
        return XKV_ERR_CUDA;
    }
    GemmArgs g{};
    g.M = static_cast<int>(T);
    g.N = d;
    g.K = rank;
    g.bn = bn;
    g.out = out;
    g.ldo = d;
    g.hd = apply_rope ? hd : 0;
    g.theta = theta;
    g.status = device_status_ptr();
    const size_t smem = gemm_smem_bytes<kRecon>();
    cudaFuncSetAttribute(gemm_tc_kernel<kRecon>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if ((T + 127) / 128 > 65535) return XKV_ERR_UNSUPPORTED;  // row tiles on grid.y
    dim3 grid(d / bn, static_cast<unsigned>((T + 127) / 128));
    gemm_tc_kernel<kRecon><<<grid, kGemmThreads, smem, st>>>(am, bm, bm, g);
  } else {
    const int64_t pairs = T * (d / 2);
    const int grid = static_cast<int>(std::min<int64_t>((pairs + 255) / 256, 8 * 1024));
    if (dt == XKV_BF16)
      recon_simt_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(A),
                                                             static_cast<const __nv_bfloat16*>(Bt), T, rank, d, hd,
                                                             apply_rope, theta, static_cast<__nv_bfloat16*>(out));
    else
      recon_simt_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(A), static_cast<const float*>(Bt), T,
                                                     rank, d, hd, apply_rope, theta, static_cast<float*>(out));
  }
  return cudaPeekAtLastError() == cudaSuccess ? XKV_OK : XKV_ERR_CUDA;
}

size_t dense_workspace(const xkv_dense_params* p) {
  int splits;
  int64_t per;
  dense_split(p, &splits, &per);
  const int gq = p->n_q_heads / p->n_kv_heads;
  return align_up(static_cast<size_t>(p->batch) * p->n_kv_heads * splits * (2 * kMaxGQ + gq * p->head_dim) * 4);
}

template <typename T>
static xkv_status dense_launch_t(const xkv_dense_params* p, const void* q, const void* K, const void* V, float* out,
                                 void* ws, cudaStream_t st) {
  int splits;
  int64_t per;
  dense_split(p, &splits, &per);
  const int gq = p->n_q_heads / p->n_kv_heads, hd = p->head_dim;
  const int units = p->batch * p->n_kv_heads;
  const size_t smem = (static_cast<size_t>(gq) * hd + 256 * gq + 8 * kMaxGQ + 3 * kMaxGQ +
                       static_cast<size_t>(256 / (hd / 2)) * gq * hd) * 4;
  cudaFuncSetAttribute(dense_partial_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  dense_partial_kernel<T><<<dim3(splits, units), 256, smem, st>>>(static_cast<const T*>(q), static_cast<const T*>(K),
                                                                  static_cast<const T*>(V), p->T, p->n_q_heads,
                                                                  p->n_kv_heads, hd, per, static_cast<float*>(ws));
  dense_combine_kernel<<<units, 256, 0, st>>>(static_cast<const float*>(ws), splits, gq, hd, out);
  return cudaPeekAtLastError() == cudaSuccess ? XKV_OK : XKV_ERR_CUDA;
}

xkv_status dense_launch(const xkv_dense_params* p, const void* q, const void* K, const void* V, float* out, void* ws,
                        cudaStream_t st) {
  if (p->dtype == XKV_BF16) return dense_launch_t<__nv_bfloat16>(p, q, K, V, out, ws, st);
  return dense_launch_t<float>(p, q, K, V, out, ws, st);
}

xkv_status landmarks_launch(const void* K, int64_t T, int64_t ldk, int hkv, int hd, xkv_dtype dt, int chunk, int sink,
                            int recent, float theta, void* out, cudaStream_t st) {
  const int64_t n_mid = (T - sink - recent) / chunk;
  if (n_mid <= 0) return XKV_OK;
  const size_t rot_bytes = static_cast<size_t>(chunk) * (hd / 2) * sizeof(float2);
  if (hd % 4 == 0 && ldk % 2 == 0 && rot_bytes <= static_cast<size_t>(kLmRotMax)) {
    const int cpb = 64;
    dim3 grid(static_cast<unsigned>((n_mid + cpb - 1) / cpb), hkv);
    if (dt == XKV_BF16)
      landmarks_rot_kernel<__nv_bfloat16><<<grid, 256, rot_bytes, st>>>(static_cast<const __nv_bfloat16*>(K), ldk, hd,
                                                                       chunk, sink, n_mid, theta, cpb,
                                                                       static_cast<__nv_bfloat16*>(out));
    else
      landmarks_rot_kernel<float><<<grid, 256, rot_bytes, st>>>(static_cast<const float*>(K), ldk, hd, chunk, sink,
                                                               n_mid, theta, cpb, static_cast<float*>(out));
    return cudaPeekAtLastError() == cudaSuccess ? XKV_OK : XKV_ERR_CUDA;
  }
  const int cpb = 64;
  dim3 grid(static_cast<unsigned>((n_mid + cpb - 1) / cpb), hkv);
  if (dt == XKV_BF16)
    landmarks_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(K), ldk, hd, chunk, sink,
                                                          n_mid, theta, cpb, static_cast<__nv_bfloat16*>(out));
  else
    landmarks_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(K), ldk, hd, chunk, sink, n_mid, theta, cpb,
                                                  static_cast<float*>(out));
  return cudaPeekAtLastError() == cudaSuccess ? XKV_OK : XKV_ERR_CUDA;
}

}  // namespace xkv
