// Multi-step decode (xKV explainer, the editor's note after "仅仅压缩还不够，
// xKV 还做了“选择性重建”": the factorisation covers the long prefill; tokens
// generated afterwards stay raw).  One call appends one token per layer of a
// group to the raw recent window; when the window then holds recent + chunk
// rows, its oldest chunk joins the compressed cache:
//   1. one landmark per layer and KV head: the mean of the chunk's keys, each
//      rotated at its absolute position (the prefill landmark of "选择性重建");
//   2. the chunk's rows of A_K and A_V: x V on the stored group bases (the
//      factorisation's A = X V_r, "xKV 到底做了什么"), on tcgen05 for bf16;
//   3. the window moves down by one chunk.
// The state is a function of the length T alone: with n0 = T - sink - recent
// tokens beyond the prefill windows, the window holds recent + n0 mod chunk
// rows and n_mid = n0 / chunk chunks are compressed.
#include <algorithm>

#include "xkv_common.cuh"
#include "xkv_internal.h"

namespace xkv {
namespace {

struct Ptr8 {
  const void* p[8];
};
struct Turns {
  double ft[128];  // RoPE turns per position of each frequency pair (host fp64)
};
struct MutPtr8 {
  void* p[8];
};

// win[l][b][row] = src[l][b] for keys (z = 0) and values (z = 1)
template <typename T>
__global__ void __launch_bounds__(128) append_rows_kernel(Ptr8 k_new, Ptr8 v_new, MutPtr8 win_K, MutPtr8 win_V, int d,
                                                          int64_t row, int64_t wbs) {
  const int l = blockIdx.x, b = blockIdx.y, z = blockIdx.z;
  const T* src = static_cast<const T*>(z ? v_new.p[l] : k_new.p[l]) + static_cast<int64_t>(b) * d;
  T* dst = static_cast<T*>(z ? win_V.p[l] : win_K.p[l]) + static_cast<int64_t>(b) * wbs + row * d;
  for (int j = threadIdx.x; j < d; j += blockDim.x) dst[j] = src[j];
}

// landmark[l][b][h][c_new] = mean_i RoPE_{t0+i}(win_K[l][b][sink + i][h]); one
// thread per frequency pair (j, j + hd/2), fp32 sums, RNE store.
template <typename T>
__global__ void roll_landmark_kernel(Ptr8 win_K, MutPtr8 lms, int Hkv, int hd, int chunk, int sink, int64_t t0,
                                     int64_t wbs, int64_t cap, int64_t c_new, const __grid_constant__ Turns tu) {
  const int l = blockIdx.x, b = blockIdx.y, h = blockIdx.z;
  const int half = hd / 2, d = Hkv * hd;
  const T* K = static_cast<const T*>(win_K.p[l]) + static_cast<int64_t>(b) * wbs + static_cast<int64_t>(sink) * d +
               h * hd;
  T* out = static_cast<T*>(lms.p[l]) + ((static_cast<int64_t>(b) * Hkv + h) * cap + c_new) * hd;
  for (int j = threadIdx.x; j < half; j += blockDim.x) {
    float a0 = 0.f, a1 = 0.f;
    for (int i = 0; i < chunk; ++i) {
      const float x0 = to_f(K[static_cast<int64_t>(i) * d + j]), x1 = to_f(K[static_cast<int64_t>(i) * d + j + half]);
      float c, s;
      rope_cs(tu.ft[j], static_cast<double>(t0 + i), &c, &s);
      a0 += x0 * c - x1 * s;
      a1 += x1 * c + x0 * s;
    }
    const float inv = 1.0f / static_cast<float>(chunk);
    store_f(out + j, a0 * inv);
    store_f(out + j + half, a1 * inv);
  }
}

// rows sink + chunk .. sink + chunk + recent - 1 move to sink .. sink + recent - 1.
// Each block owns a 64-column slice of one window (layer, sequence, K|V), reads
// all of its rows before writing any, so the overlapping move is race-free.
template <typename T>
__global__ void __launch_bounds__(256) shift_window_kernel(MutPtr8 win_K, MutPtr8 win_V, int G, int d, int sink,
                                                           int chunk, int recent, int64_t wbs) {
  extern __shared__ float shift_sm[];  // [recent][64]
  const int l = blockIdx.x % G, z = (blockIdx.x / G) % 2, cs = blockIdx.x / (2 * G);
  const int b = blockIdx.y;
  const int c0 = cs * 64, nc = min(64, d - c0);
  T* w = static_cast<T*>(z ? win_V.p[l] : win_K.p[l]) + static_cast<int64_t>(b) * wbs;
  for (int i = threadIdx.x; i < recent * 64; i += blockDim.x) {
    const int r = i / 64, c = i % 64;
    if (c < nc) shift_sm[i] = to_f(w[static_cast<int64_t>(sink + chunk + r) * d + c0 + c]);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < recent * 64; i += blockDim.x) {
    const int r = i / 64, c = i % 64;
    if (c < nc) store_f(w + static_cast<int64_t>(sink + r) * d + c0 + c, shift_sm[i]);
  }
}

template <typename T>
xkv_status append_launch_t(const xkv_append_params* p, const void* const* k_new, const void* const* v_new,
                           void* const* win_K, void* const* win_V, const void* Bt_K, const void* Bt_V, void* A_K,
                           void* A_V, void* const* landmarks, int* rolled, void* ws, cudaStream_t st) {
  const int G = p->group, B = p->batch, d = p->n_kv_heads * p->head_dim, C = p->chunk;
  const int64_t n0 = p->T - p->sink - p->recent;
  const int w_cur = p->recent + static_cast<int>(n0 % C);
  const int64_t n_mid = n0 / C;
  const int64_t wbs = p->window_batch_stride;
  Ptr8 kn{}, vn{}, wKc{};
  MutPtr8 wKm{}, wVm{}, lmm{};
  for (int l = 0; l < G; ++l) {
    kn.p[l] = k_new[l];
    vn.p[l] = v_new[l];
    wKm.p[l] = win_K[l];
    wVm.p[l] = win_V[l];
    wKc.p[l] = win_K[l];
    lmm.p[l] = landmarks[l];
  }
  // 1. the new token's rows
  append_rows_kernel<T><<<dim3(G, B, 2), 128, 0, st>>>(kn, vn, wKm, wVm, d, p->sink + w_cur, wbs);
  const bool roll = w_cur + 1 == p->recent + C;
  if (rolled) *rolled = roll ? 1 : 0;
  if (!roll) return cudaPeekAtLastError() == cudaSuccess ? XKV_OK : XKV_ERR_CUDA;
  const int64_t t0 = p->sink + n_mid * C;
  // 2. landmarks of the rolled chunk
  Turns tu{};
  for (int j = 0; j < p->head_dim / 2; ++j) tu.ft[j] = rope_turns(p->rope_theta, j, p->head_dim);
  roll_landmark_kernel<T><<<dim3(G, B, p->n_kv_heads), 64, 0, st>>>(wKc, lmm, p->n_kv_heads, p->head_dim, C,
                                                                     p->sink, t0, wbs, p->landmark_capacity, n_mid,
                                                                     tu);
  // 3. A rows of the chunk on the stored bases, one sequence at a time
  void* pws = ws;
  const size_t es = sizeof(T);
  const xkv_dtype dt = p->dtype;
  for (int b = 0; b < B; ++b) {
    const void* XK[8];
    const void* XV[8];
    for (int l = 0; l < G; ++l) {
      XK[l] = static_cast<const uint8_t*>(win_K[l]) + (static_cast<int64_t>(b) * wbs + static_cast<int64_t>(p->sink) * d) * es;
      XV[l] = static_cast<const uint8_t*>(win_V[l]) + (static_cast<int64_t>(b) * wbs + static_cast<int64_t>(p->sink) * d) * es;
    }
    const void* bk = static_cast<const uint8_t*>(Bt_K) + static_cast<int64_t>(b) * p->bt_k_batch_stride * es;
    const void* bv = static_cast<const uint8_t*>(Bt_V) + static_cast<int64_t>(b) * p->bt_v_batch_stride * es;
    void* ak = static_cast<uint8_t*>(A_K) + (static_cast<int64_t>(b) * p->a_k_batch_stride + t0 * p->rank_k) * es;
    void* av = static_cast<uint8_t*>(A_V) + (static_cast<int64_t>(b) * p->a_v_batch_stride + t0 * p->rank_v) * es;
    xkv_status s = project_launch(XK, G, C, d, d, dt, bk, dt, p->rank_k, ak, p->rank_k, pws, st);
    if (s != XKV_OK) return s;
    s = project_launch(XV, G, C, d, d, dt, bv, dt, p->rank_v, av, p->rank_v, pws, st);
    if (s != XKV_OK) return s;
  }
  // 4. the window moves down by one chunk
  const int slices = (d + 63) / 64;
  shift_window_kernel<T><<<dim3(2 * G * slices, B), 256, static_cast<size_t>(p->recent) * 64 * 4, st>>>(
      wKm, wVm, G, d, p->sink, C, p->recent, wbs);
  return cudaPeekAtLastError() == cudaSuccess ? XKV_OK : XKV_ERR_CUDA;
}

}  // namespace

size_t append_workspace(const xkv_append_params* p) {
  const int n = p->group * p->n_kv_heads * p->head_dim;
  return project_workspace(n, std::max(p->rank_k, p->rank_v));
}

xkv_status append_launch(const xkv_append_params* p, const void* const* k_new, const void* const* v_new,
                         void* const* win_K, void* const* win_V, const void* Bt_K, const void* Bt_V, void* A_K,
                         void* A_V, void* const* landmarks, int* rolled, void* ws, cudaStream_t st) {
  if (p->dtype == XKV_BF16)
    return append_launch_t<__nv_bfloat16>(p, k_new, v_new, win_K, win_V, Bt_K, Bt_V, A_K, A_V, landmarks, rolled,
                                          ws, st);
  return append_launch_t<float>(p, k_new, v_new, win_K, win_V, Bt_K, Bt_V, A_K, A_V, landmarks, rolled, ws, st);
}

}  // namespace xkv
