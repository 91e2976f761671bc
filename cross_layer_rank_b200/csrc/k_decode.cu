// Decode-time Selective Reconstruction (xKV explainer, "仅仅压缩还不够，xKV 还做了
// “选择性重建”"; xKV abstract): landmark scoring, exact top-k chunk selection,
// reconstruction of only the selected rows of K and V from the shared basis A
// and the layer's B_l, RoPE on the rebuilt keys, and online-softmax GQA
// attention (KQ-SVD page, 3.2) over them plus the raw sink/recent window.
// The same kernels serve the xK-SR mode of the explainer (keys compressed,
// values read whole from a [B][T][d] cache): the value operand is then head
// h's columns of V and the combine skips the Bt_V projection.
//
// Kernels (one decode step of one layer = 4 launches, chained with
// programmatic dependent launch):
//   sr_score   : s_c = (sum_g q_g) . landmark_c            (HBM stream of landmarks)
//   sr_topk    : exact top-k per unit in one CTA (bucket histogram, a refining
//                histogram of the boundary bucket, then a rank count or radix
//                passes over its candidates; ties to the lower chunk),
//                ascending output; extra blocks of the same grid compute the
//                raw sink/recent window's partial (m, l, o)
//   sr_attend  : persistent CTAs over (unit, 128-row tile) ranges.  tcgen05
//                path: TMA gathers the selected 8-row chunk slabs of A_K
//                (8 x 64 bf16 = one 1 KiB swizzle atom each) and the head's
//                Bt_K slice, tcgen05.mma rebuilds the 128 x 128 key tile in
//                TMEM, the epilogue applies RoPE and the q . k products, and a
//                second MMA folds p into u_g = sum_t p_gt A_V[t] (the value
//                path is re-associated: o_g = (u_g / l_g) Bt_V^T, exact up to
//                rounding).  A SIMT path covers f32 and other shapes.
//   sr_combine : merges the per-CTA (m, l, u) partials with the window
//                partial and applies Bt_V.
#include <float.h>

#include <algorithm>
#include <utility>

#include "xkv_common.cuh"
#include "xkv_internal.h"

namespace xkv {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kTileChunks = 16;   // chunks of 8 rows per 128-row tile (tcgen05 path)
constexpr int kMaxGQ = 8;
constexpr int kKStages = 3;   // key stages: 16 chunks x kKAtoms 64-column atoms
constexpr int kKAtoms = 2;
constexpr int kBStages = 3;   // Bt_K atoms (128 rows x 64 columns): one stage and the next one's first
constexpr int kVStages = 3;   // value stages: 2 chunks x full rank
constexpr int kAtomBytes = 16384;  // 128 rows x 64 bf16
constexpr int kAttendThreads = 512;  // 16 warps: 8 key epilogue, 4 value epilogue, 2 TMA, 2 MMA

// ----------------------------------------------------------------- helpers
// Programmatic dependent launch: the later kernels of a decode step may start
// while the previous one drains; each waits here before its first read of the
// previous kernel's output (a no-op when launched without the attribute).
__device__ __forceinline__ void wait_prior_grid() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// lets the next kernel of the step be scheduled once every CTA of this grid
// has started (its CTAs then wait in wait_prior_grid for this grid's end)
__device__ __forceinline__ void allow_next_grid() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// 16-byte asynchronous global -> shared copies (L2 only)
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__host__ __device__ inline int tile_begin(int c, int n_tiles, int ctas) {
  return static_cast<int>((static_cast<int64_t>(c) * n_tiles) / ctas);
}

__device__ inline int cta_of_tile(int x, int n_tiles, int ctas) {
  int c = static_cast<int>((static_cast<int64_t>(x) * ctas) / n_tiles);
  while (c + 1 < ctas && tile_begin(c + 1, n_tiles, ctas) <= x) ++c;
  while (c > 0 && tile_begin(c, n_tiles, ctas) > x) --c;
  return c;
}

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f == 0.0f ? 0.0f : f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <typename T>
__device__ __forceinline__ float ldf(const T* p) {
  return to_f(*p);
}

// Block-wide exclusive scan of one uint per thread (blockDim.x == 1024).
__device__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* warp_tot, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = warp_tot[lane];
    uint32_t s = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_tot[lane] = s - w;
    if (lane == 31) *total = s;
  }
  __syncthreads();
  const uint32_t r = warp_tot[warp] + x - v;
  __syncthreads();
  return r;
}

// ------------------------------------------------------------ sr_score
// One block per (unit, slice of chunks).  s_c = qbar . l_c with qbar = sum of
// the GQA group's queries (sum_g q_g . l_c regrouped).
template <typename T>
__global__ void __launch_bounds__(256) sr_score_kernel(const T* __restrict__ q, const T* __restrict__ lm,
                                                       float* __restrict__ scores, int Hq, int Hkv, int hd,
                                                       int64_t n_mid, int64_t lm_cap, int64_t ld,
                                                       int chunks_per_block) {
  allow_next_grid();
  __shared__ float qbar[256];
  const int unit = blockIdx.y;
  const int b = unit / Hkv, h = unit % Hkv, gq = Hq / Hkv;
  for (int j = threadIdx.x; j < hd; j += blockDim.x) {
    float s = 0.f;
    for (int g = 0; g < gq; ++g) s += ldf(q + (static_cast<int64_t>(b) * Hq + h * gq + g) * hd + j);
    qbar[j] = s;
  }
  __syncthreads();
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * chunks_per_block;
  const int64_t c1 = min(c0 + chunks_per_block, n_mid);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const T* base = lm + static_cast<int64_t>(unit) * lm_cap * hd;
  float* out = scores + static_cast<int64_t>(unit) * ld;
  if (sizeof(T) == 2 && hd == 128) {
    // 16 lanes x 16 B cover one 256-B landmark row; a warp scores 2 rows per
    // load and keeps 8 rows (4 loads per lane) in flight.
    const int half = lane >> 4, hl = lane & 15;
    float qv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) qv[i] = qbar[hl * 8 + i];
    constexpr int U = 8;
    for (int64_t cb = c0 + warp * 2 * U; cb < c1; cb += 16 * U) {
      uint4 w[U];
#pragma unroll
      for (int k = 0; k < U; ++k) {
        const int64_t c = cb + 2 * k + half;
        w[k] = c < c1 ? *reinterpret_cast<const uint4*>(base + c * 128 + hl * 8) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int k = 0; k < U; ++k) {
        const uint32_t ww[4] = {w[k].x, w[k].y, w[k].z, w[k].w};
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = bf2_to_f2(ww[i]);
          s = fmaf(qv[2 * i], f.x, s);
          s = fmaf(qv[2 * i + 1], f.y, s);
        }
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        const int64_t c = cb + 2 * k + half;
        if (hl == 0 && c < c1) out[c] = s;
      }
    }
  } else {
    for (int64_t c = c0 + warp; c < c1; c += 8) {
      float s = 0.f;
      for (int j = lane; j < hd; j += 32) s = fmaf(qbar[j], ldf(base + c * hd + j), s);
      s = warp_sum(s);
      if (lane == 0) out[c] = s;
    }
  }
}

// ------------------------------------------------------------- sr_topk
// Exact top-k of one unit's chunk scores (1024 threads, one CTA per unit).
//   1. scores -> order-preserving 32-bit keys (coalesced 16-byte loads of the
//      padded score row) and their range [lo, hi];
//   2. a 1024-bucket histogram of floor((key - lo) * 1024 / (hi - lo + 1))
//      (fp32 arithmetic: a monotone map, so every key of a higher bucket is
//      larger than every key of a lower one);
//   3. a suffix scan finds the boundary bucket B holding the k-th largest key;
//      keys above B are kept, `need` more come from B;
//   4. the keys of B are compacted in ascending index order and the `need`
//      largest of them chosen (ties -> lower index): up to 1024 candidates by
//      counting, per candidate (one warp each), the candidates ranked above it;
//      more by 8-bit radix passes and an ordered scan of the equal keys;
//   5. an ordered compaction writes the selection ascending by chunk.
// Thread t owns the contiguous index segment [t per, (t+1) per), stored
// transposed (element j of every thread's segment is contiguous) so that the
// segment loops are free of shared-memory bank conflicts.
constexpr int kTopkThreads = 1024;
constexpr int kBuckets = 1024;
constexpr uint32_t kRefineMin = 64;  // boundary buckets above this size get a second histogram

__device__ __forceinline__ uint32_t topk_bucket(uint32_t key, uint32_t lo, float scale) {
  const float x = static_cast<float>(key - lo) * scale;
  return min(static_cast<uint32_t>(x), static_cast<uint32_t>(kBuckets - 1));
}

// ------------------------------------------------------------ sr_window
// Raw sink/recent window of one unit, computed by extra blocks of the top-k
// grid (the top-k itself occupies one SM per unit): the uncompressed rows are
// staged in shared memory with one round of loads, RoPE is applied in place at
// their true positions, then the scores, their softmax statistics and the
// unnormalised weighted value sum o_g = sum_t 2^(s_gt - m_g) V_t.
// Window slot layout: [0..7] m_g (log2 domain), [8..15] l_g, [16 + g hd + j] o_g[j].
struct WinArgs {
  const void* q;
  const void* srK;
  const void* srV;
  float* win;
  int64_t T;
  int64_t wbs;  // elements between sequences of the raw window
  int64_t pos_off;  // global position of local token row 0
  int Hq, Hkv, hd, sink, recent;
  double ft[128];  // RoPE frequency of pair j in turns per position
};

inline size_t window_smem(int gq, int hd, int nsr) {
  return 128 * 8 + (static_cast<size_t>(nsr) * (2 * hd + 1) + static_cast<size_t>(gq) * hd + nsr * kMaxGQ) * 4;
}

template <typename T>
__device__ void window_partial(const WinArgs& wa, int unit, uint8_t* smem) {
  const int hd = wa.hd, gq = wa.Hq / wa.Hkv, half = hd / 2, nsr = wa.sink + wa.recent, d = wa.Hkv * hd;
  const int b = unit / wa.Hkv, h = unit % wa.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nt = blockDim.x, nwarps = nt >> 5;
  const int ks = hd + 1;  // padded key row stride
  double* fts = reinterpret_cast<double*>(smem);  // [128]
  float* wK = reinterpret_cast<float*>(fts + 128);  // [nsr][hd + 1]
  float* wV = wK + nsr * ks;                        // [nsr][hd]
  float* qs = wV + nsr * hd;                        // [gq][hd]
  float* ws = qs + gq * hd;                         // [nsr][8] scores, then weights
  const T* q = static_cast<const T*>(wa.q);
  const T* srK = static_cast<const T*>(wa.srK);
  const T* srV = static_cast<const T*>(wa.srV);
  float* slot = wa.win + static_cast<int64_t>(unit) * (16 + gq * hd);
  const float qscale = rsqrtf(static_cast<float>(hd)) * kLog2e;
  // 1. loads
  for (int i = tid; i < gq * hd; i += nt) qs[i] = ldf(q + (static_cast<int64_t>(b) * wa.Hq + h * gq) * hd + i) * qscale;
  for (int j = tid; j < half; j += nt) fts[j] = wa.ft[j];
  if (sizeof(T) == 2 && hd % 8 == 0) {
    const int vpr = hd / 8;
    for (int v = tid; v < 2 * nsr * vpr; v += nt) {
      const int mat = v / (nsr * vpr), r = (v / vpr) % nsr, c8 = v % vpr;
      const T* src = (mat ? srV : srK) + static_cast<int64_t>(b) * wa.wbs + static_cast<int64_t>(r) * d + h * hd + c8 * 8;
      const uint4 w = *reinterpret_cast<const uint4*>(src);
      float* dst = mat ? wV + r * hd + c8 * 8 : wK + r * ks + c8 * 8;
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = bf2_to_f2(ww[e]);
        dst[2 * e] = f.x;
        dst[2 * e + 1] = f.y;
      }
    }
  } else {
    for (int i = tid; i < nsr * hd; i += nt) {
      const int r = i / hd, j = i % hd;
      const int64_t off = static_cast<int64_t>(b) * wa.wbs + static_cast<int64_t>(r) * d + h * hd + j;
      wK[r * ks + j] = ldf(srK + off);
      wV[r * hd + j] = ldf(srV + off);
    }
  }
  __syncthreads();
  // 2. RoPE of the window keys at their positions
  for (int i = tid; i < nsr * half; i += nt) {
    const int r = i / half, jj = i % half;
    const int64_t t = wa.pos_off + (r < wa.sink ? r : wa.T - wa.recent + (r - wa.sink));
    float c, sn;
    rope_cs(fts[jj], static_cast<double>(t), &c, &sn);
    float* kr = wK + r * ks;
    const float x0 = kr[jj], x1 = kr[jj + half];
    kr[jj] = x0 * c - x1 * sn;
    kr[jj + half] = x1 * c + x0 * sn;
  }
  __syncthreads();
  // 3. scores: warp per row
  for (int r = warp; r < nsr; r += nwarps) {
    float acc[kMaxGQ];
#pragma unroll
    for (int g = 0; g < kMaxGQ; ++g) acc[g] = 0.f;
    for (int j = lane; j < hd; j += 32) {
      const float kv = wK[r * ks + j];
#pragma unroll
      for (int g = 0; g < kMaxGQ; ++g)
        if (g < gq) acc[g] = fmaf(qs[g * hd + j], kv, acc[g]);
    }
#pragma unroll
    for (int g = 0; g < kMaxGQ; ++g) {
      if (g >= gq) break;
      const float v = warp_sum(acc[g]);
      if (lane == 0) ws[r * kMaxGQ + g] = v;
    }
  }
  __syncthreads();
  // 4. softmax statistics: warp per query head
  for (int g = warp; g < gq; g += nwarps) {
    float m = -INFINITY;
    for (int r = lane; r < nsr; r += 32) m = fmaxf(m, ws[r * kMaxGQ + g]);
    m = warp_max(m);
    float l = 0.f;
    for (int r = lane; r < nsr; r += 32) {
      const float w = exp2f(ws[r * kMaxGQ + g] - m);
      ws[r * kMaxGQ + g] = w;
      l += w;
    }
    l = warp_sum(l);
    if (lane == 0) { slot[g] = m; slot[8 + g] = l; }
  }
  __syncthreads();
  // 5. o_g[j]: thread per (g, j)
  for (int i = tid; i < gq * hd; i += nt) {
    const int g = i / hd, j = i % hd;
    float acc = 0.f;
    for (int r = 0; r < nsr; ++r) acc = fmaf(ws[r * kMaxGQ + g], wV[r * hd + j], acc);
    slot[16 + i] = acc;
  }
}

template <typename T>
__global__ void __launch_bounds__(kTopkThreads) sr_topk_kernel(const float* __restrict__ scores, int64_t ld,
                                                               int32_t* __restrict__ sel,
                                                               int32_t* __restrict__ sel_out, int64_t n_mid, int k,
                                                               int units, const __grid_constant__ WinArgs wa) {
  extern __shared__ uint32_t ksm[];  // [per][1024] keys (transposed), [n] candidate keys, [n] decisions
  allow_next_grid();
  if (static_cast<int>(blockIdx.x) >= units) {
    window_partial<T>(wa, blockIdx.x - units, reinterpret_cast<uint8_t*>(ksm));
    return;
  }
  __shared__ uint32_t hist[kBuckets];
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t s_lo, s_hi, s_total, s_bucket, s_need, s_all, s_digit, s_kk, s_eq;
  const int unit = blockIdx.x;
  const int n = static_cast<int>(n_mid);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nt = static_cast<int>(blockDim.x), nwarps = nt >> 5;
  const int per = (n + nt - 1) / nt;
  const float inv_per = 1.0f / static_cast<float>(per);
  uint32_t* ckey = ksm + per * nt;
  uint8_t* ckeep = reinterpret_cast<uint8_t*>(ckey + n);
  hist[tid] = 0u;
  if (tid == 0) { s_lo = 0xFFFFFFFFu; s_hi = 0u; }
  wait_prior_grid();  // the chunk scores
  // 1. keys (row start 16-byte aligned: ld is a multiple of 4) and their range
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  {
    const float4* row = reinterpret_cast<const float4*>(scores + static_cast<int64_t>(unit) * ld);
    const int n4 = (n + 3) / 4;
    for (int i4 = tid; i4 < n4; i4 += nt) {
      const float4 v = row[i4];
      const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = 4 * i4 + e;
        if (i < n) {
          const uint32_t key = order_key(vv[e]);
          // i / per by a float product: exact, since (i + 0.5) / per lies at
          // least 0.5 / per from an integer, i + 0.5 is exact (n < 2^23) and
          // the product's relative error is below 2^-23 (per <= 32 here)
          const int t = static_cast<int>((static_cast<float>(i) + 0.5f) * inv_per);
          ksm[(i - t * per) * nt + t] = key;
          kmin = min(kmin, key);
          kmax = max(kmax, key);
        }
      }
    }
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  __syncthreads();
  if (lane == 0) { atomicMin(&s_lo, kmin); atomicMax(&s_hi, kmax); }
  __syncthreads();
  const uint32_t lo = s_lo;
  const float scale = static_cast<float>(kBuckets) / (static_cast<float>(s_hi - lo) + 1.0f);
  const int i0 = tid * per, cnt = max(0, min(per, n - i0));
  // 2. histogram
  for (int j = 0; j < cnt; ++j) atomicAdd(&hist[topk_bucket(ksm[j * nt + tid], lo, scale)], 1u);
  __syncthreads();
  // 3. suffix scan: thread t owns bucket kBuckets - 1 - t; the bucket where
  // the running count reaches kk, and how many keys it must still give
  auto find_boundary = [&](uint32_t kk) {
    const uint32_t hv = hist[kBuckets - 1 - tid];
    const uint32_t excl = block_exclusive_scan(hv, warp_tot, &s_total);  // keys in higher buckets
    if (excl < kk && excl + hv >= kk) {
      s_bucket = kBuckets - 1 - tid;
      s_need = kk - excl;
    }
    __syncthreads();
  };
  find_boundary(static_cast<uint32_t>(k));
  const uint32_t B = s_bucket, need1 = s_need;
  const uint32_t m1 = hist[B];
  // 4. a crowded boundary bucket is refined by a second histogram over its own
  // key range (same monotone map), so few keys remain to be ranked one by one
  const bool two = m1 > kRefineMin;
  uint32_t lo2 = 0u, B2 = 0u, need = need1;
  float scale2 = 0.f;
  if (two) {
    uint32_t bmin = 0xFFFFFFFFu, bmax = 0u;
    for (int j = 0; j < cnt; ++j) {
      const uint32_t key = ksm[j * nt + tid];
      if (topk_bucket(key, lo, scale) == B) { bmin = min(bmin, key); bmax = max(bmax, key); }
    }
    bmin = __reduce_min_sync(0xffffffffu, bmin);
    bmax = __reduce_max_sync(0xffffffffu, bmax);
    __syncthreads();  // every thread has read hist[B]
    hist[tid] = 0u;
    if (tid == 0) { s_lo = 0xFFFFFFFFu; s_hi = 0u; }
    __syncthreads();
    if (lane == 0) { atomicMin(&s_lo, bmin); atomicMax(&s_hi, bmax); }
    __syncthreads();
    lo2 = s_lo;
    scale2 = static_cast<float>(kBuckets) / (static_cast<float>(s_hi - lo2) + 1.0f);
    for (int j = 0; j < cnt; ++j) {
      const uint32_t key = ksm[j * nt + tid];
      if (topk_bucket(key, lo, scale) == B) atomicAdd(&hist[topk_bucket(key, lo2, scale2)], 1u);
    }
    __syncthreads();
    find_boundary(need1);
    B2 = s_bucket;
    need = s_need;
  }
  // key classes: 2 = kept outright, 1 = final candidate, 0 = dropped
  auto klass = [&](uint32_t key) -> int {
    const uint32_t b1 = topk_bucket(key, lo, scale);
    if (b1 != B) return b1 > B ? 2 : 0;
    if (!two) return 1;
    const uint32_t b2 = topk_bucket(key, lo2, scale2);
    return b2 > B2 ? 2 : (b2 == B2 ? 1 : 0);
  };
  // 5. every key's class once, as bit masks over the thread's segment
  // (per <= 32): kmask = kept outright, cmask = final candidates
  uint32_t kmask = 0u, cmask = 0u;
  for (int j = 0; j < cnt; ++j) {
    const int c = klass(ksm[j * nt + tid]);
    kmask |= static_cast<uint32_t>(c == 2) << j;
    cmask |= static_cast<uint32_t>(c == 1) << j;
  }
  // final candidates (their keys, ascending index)
  uint32_t cpos = block_exclusive_scan(__popc(cmask), warp_tot, &s_total);
  const uint32_t m = s_total;
  const uint32_t cbase = cpos;
  for (uint32_t bits = cmask; bits; bits &= bits - 1) ckey[cpos++] = ksm[(__ffs(bits) - 1) * nt + tid];
  __syncthreads();
  if (m == need) {
    if (tid == 0) s_all = 1u;
  } else if (m <= static_cast<uint32_t>(nt)) {
    // rank of candidate c: candidates with a larger key, or an equal key and
    // a lower index; the `need` lowest ranks are kept
    if (tid == 0) s_all = 0u;
    for (uint32_t c = warp; c < m; c += nwarps) {
      const uint32_t key = ckey[c];
      uint32_t r = 0;
      for (uint32_t o = lane; o < m; o += 32) {
        const uint32_t ko = ckey[o];
        r += (ko > key) || (ko == key && o < c);
      }
      r = __reduce_add_sync(0xffffffffu, r);
      if (lane == 0) ckeep[c] = r < need;
    }
  } else {
    // 8-bit radix passes over the candidates: the k-th key's digits top down
    uint32_t prefix = 0u, mask = 0u, kk = need;
    bool all = false;
    for (int shift = 24; shift >= 0 && !all; shift -= 8) {
      if (tid < 256) hist[tid] = 0u;
      __syncthreads();
      for (uint32_t c = tid; c < m; c += nt) {
        const uint32_t key = ckey[c];
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (warp == 0) {
        // lane l holds digits 255 - 8l .. 248 - 8l (descending)
        uint32_t h[8], sum = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) { h[e] = hist[255 - 8 * lane - e]; sum += h[e]; }
        uint32_t incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        uint32_t above = incl - sum;
        if (above < kk && incl >= kk) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (above < kk && above + h[e] >= kk) {
              s_digit = 255 - 8 * lane - e;
              s_kk = kk - above;
              s_eq = h[e];
            }
            above += h[e];
          }
        }
      }
      __syncthreads();
      prefix |= s_digit << shift;
      mask |= 255u << shift;
      kk = s_kk;
      all = s_eq == kk;  // every candidate with this prefix is kept
    }
    // decisions: above the prefix kept; equal to it kept when all are, else
    // the first kk in index order (ordered scan over contiguous candidate runs)
    const uint32_t cpt = (m + nt - 1) / nt, c0 = min(m, tid * cpt), c1 = min(m, c0 + cpt);
    uint32_t eq = 0;
    for (uint32_t c = c0; c < c1; ++c) eq += (ckey[c] & mask) == prefix;
    uint32_t rank = block_exclusive_scan(eq, warp_tot, &s_total);
    for (uint32_t c = c0; c < c1; ++c) {
      const uint32_t km = ckey[c] & mask;
      bool keep;
      if (km > prefix) keep = true;
      else if (km < prefix) keep = false;
      else keep = all || rank++ < kk;
      ckeep[c] = keep;
    }
    if (tid == 0) s_all = 0u;
  }
  __syncthreads();
  const bool all_taken = s_all != 0u;
  // 6. ordered compaction of the selection: a final candidate is kept when
  // its decision says so (candidates are numbered in index order)
  uint32_t take = kmask;
  {
    uint32_t ci = cbase;
    for (uint32_t bits = cmask; bits; bits &= bits - 1, ++ci)
      if (all_taken || ckeep[ci]) take |= 1u << (__ffs(bits) - 1);
  }
  uint32_t pos = block_exclusive_scan(__popc(take), warp_tot, &s_total);
  {
    int32_t* o = sel + static_cast<int64_t>(unit) * k;
    int32_t* o2 = sel_out ? sel_out + static_cast<int64_t>(unit) * k : nullptr;
    for (uint32_t bits = take; bits; bits &= bits - 1, ++pos) {
      const int idx = i0 + __ffs(bits) - 1;
      o[pos] = idx;
      if (o2) o2[pos] = idx;
    }
  }
}

// ------------------------------------------------- sr_attend (tcgen05)
struct AttendArgs {
  const int32_t* sel;
  const void* q;
  float* part;
  int* status;
  int64_t T;
  int64_t sbk, sbv;  // batch strides of Bt_K / Bt_V (elements, 0 = shared)
  int Hq, Hkv, k, sink, recent, rK, rV;
  int v_raw;  // values uncompressed (xK-SR), rV = hd: 1 = the value operand is V [B][T][d], head h at
              // column h hd; 2 = the kept rows gathered from host memory, [units][k][chunk][hd]
  int tiles_per_unit, n_tiles, ctas, max_units;
  int slot_floats;
  float theta;
  // token sharding: local row 0 is global position pos_off; selection entries
  // are global chunk indices, kept only in [c_lo, c_hi), whose rows sit at
  // local row sink + (c - c_lo) chunk (the whole sequence: 0, 0, n_mid)
  int64_t pos_off;
  int c_lo, c_hi;
  float* ml_out;  // (M, L) per (sequence, query head) when the caller merges partials, or null
  double ft[128];  // RoPE turns per position of each frequency pair (host-computed, fp64)
};

__device__ __forceinline__ bool kept_here(const AttendArgs& a, int c) { return c >= a.c_lo && c < a.c_hi; }

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                            int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                            int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Shared-memory plan of the tensor-core attend kernel (offsets from a 1 KiB
// aligned base): K ring (A atoms, Bt atoms), V ring (value slabs, 128-byte
// swizzled so they serve directly as the MN-major operand of the value MMA),
// P double buffer (bf16 softmax weights, K-major swizzled B operand), alpha,
// scaled queries ([j][g] interleaved), RoPE tables (per-chunk base angle and
// per-offset rotation, rows padded to 130 floats so lanes of different chunks
// hit different banks), reductions, barriers.
constexpr int kRopeStride = 130;
constexpr int kPBytes = 4096;  // [2 K-atoms][16 rows][128 B]
constexpr int kKStageBytes = kTileChunks * kKAtoms * 1024;
constexpr int kSmemKa = 0;
constexpr int kSmemKb = kSmemKa + kKStages * kKStageBytes;
constexpr int kSmemV = kSmemKb + kBStages * kAtomBytes;
constexpr int kSmemP = kSmemV + kVStages * 16384;
constexpr int kSmemAlpha = kSmemP + 2 * kPBytes;
constexpr int kSmemQ = kSmemAlpha + 2 * kMaxGQ * 4;
constexpr int kSmemBase = kSmemQ + 128 * kMaxGQ * 4;
constexpr int kSmemRot = kSmemBase + kTileChunks * kRopeStride * 4;
constexpr int kSmemFt = kSmemRot + 8 * kRopeStride * 4;
constexpr int kSmemRed = kSmemFt + 64 * 8;
constexpr int kSmemSpart = kSmemRed + 64 * 4;                         // [128][8] partial scores of half 1
constexpr int kSmemBars = kSmemSpart + 128 * kMaxGQ * 4;
constexpr int kNumBars = 2 * kKStages + 2 * kBStages + 2 * kVStages + 14;
constexpr int kSmemEnd = kSmemBars + kNumBars * 8 + 16;
constexpr int kVAccCol = 256;  // TMEM columns of the value accumulators (2 x 64)

// Warp roles: 0-7 key epilogue (warp w reads TMEM lane quarter w % 4 and the
// frequency pairs of half w / 4), 8-11 value epilogue, 12 key TMA producer,
// 13 value TMA producer, 14 key MMA issuer (TMEM owner), 15 value MMA issuer.
// The two issuers run independently, so the key gathers of later tiles never
// wait behind the value products of earlier ones.
// ------------------------------------------------------ merge of a unit
// Final output of one unit (the combine step) by one CTA, for output columns
// [j0, j1).  Each phase issues all of its loads before using them (one memory
// round trip per phase):
//   A  (m, l) of the unit's partial slots and of its window partial;
//   C  M_g, the slot factors 2^(m - M_g) and L_g (warp per query head);
//   D  U_g = sum over slots of u 2^(m - M_g), kept in shared memory in an
//      order where lane-consecutive 8-column groups are word-consecutive;
//   E  o_g[j] = (U_g . Bt_V[h hd + j] + 2^(m_w - M_g) o_w,g[j]) / L_g for the
//      split's columns (a warp per 4 columns, whose Bt_V rows were staged in
//      shared memory by cp.async or are loaded 16 bytes a lane; the warp's 32
//      sums are reduce-scattered so each lane stores one).  With uncompressed
//      values (xK-SR) U_g is already o_g's value sum and E is a scaled copy.
constexpr int kCombineSplit = 4;
constexpr int kCombineThreads = 512;
constexpr int kMaxSlots = 64;
constexpr int kCombineColsPerWarp = 4;
constexpr int kCombineStageBytes = 64 * 1024;  // Bt_V rows staged for E, when they fit

// Partials are read through L2 (__ldcg): they may have been written by other
// CTAs of the same launch.  smf: (gq rV + 64 * 24 + 32 + gq (j1 - j0) + 2 + 128)
// floats, 16-byte aligned.
template <typename T>
__device__ void merge_unit(const T* __restrict__ BtV, const float* __restrict__ win, const AttendArgs& args, int hd,
                           float* __restrict__ out, int u, int j0, int j1, float* smf) {
  const int gq = args.Hq / args.Hkv;
  const int b = u / args.Hkv, h = u % args.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  const int tpu = args.tiles_per_unit;
  const int rV = args.rV;
  // bf16 rows with 8-column groups: U stored as [g][e][v] for column 8v + e
  const bool vec = !args.v_raw && sizeof(T) == 2 && rV % 8 == 0 && args.sbv % 8 == 0;
  const int nv = rV / 8;
  float* Us = smf;                              // [gq][rV] (permuted when vec)
  float* ml = Us + gq * rV;                     // [slots][16] partial m, l
  float* sc = ml + kMaxSlots * 16;              // [slots][8] slot factors
  float* wml = sc + kMaxSlots * kMaxGQ;         // [16] window m, l
  float* Lg = wml + 16;                         // [8] 1 / L_g
  float* fw = Lg + kMaxGQ;                      // [8] window factors
  float* wo = fw + kMaxGQ;                      // [gq][j1 - j0] window value sums of the columns
  const float* wslot = win + static_cast<int64_t>(u) * (16 + gq * hd);
  const int fc = cta_of_tile(u * tpu, args.n_tiles, args.ctas);
  const int lc = cta_of_tile((u + 1) * tpu - 1, args.n_tiles, args.ctas);
  const int nslots = lc - fc + 1;
  // slot i of the unit belongs to CTA fc + i; its offset is computed once
  int64_t* soff = reinterpret_cast<int64_t*>(wo + gq * (j1 - j0) + 1) ;
  soff = reinterpret_cast<int64_t*>((reinterpret_cast<uintptr_t>(soff) + 7) & ~uintptr_t(7));
  for (int i = tid; i < nslots; i += blockDim.x) {
    const int c = fc + i;
    const int uf = tile_begin(c, args.n_tiles, args.ctas) / tpu;
    soff[i] = (static_cast<int64_t>(c) * args.max_units + (u - uf)) * args.slot_floats;
  }
  __syncthreads();
  auto slot_ptr = [&](int c) -> const float* { return args.part + soff[c - fc]; };
  // E's Bt_V rows depend on nothing: cp.async stages them in shared memory
  // while the partials are merged (when they fit; else E loads them itself)
  const int ncols = j1 - j0;
  uint4* Bs = reinterpret_cast<uint4*>((reinterpret_cast<uintptr_t>(soff + kMaxSlots) + 15) & ~uintptr_t(15));
  const bool staged = vec && static_cast<int64_t>(ncols) * rV * 2 <= kCombineStageBytes;
  if (staged) {
    for (int i = tid; i < ncols * nv; i += blockDim.x) {
      const int cc = i / nv, v = i - cc * nv;
      cp_async16(Bs + i, BtV + b * args.sbv + static_cast<int64_t>(h * hd + j0 + cc) * rV + 8 * v);
    }
  }
  cp_async_commit();
  wait_prior_grid();  // the partial slots (and, through the attend grid's own wait, the window partials)
  // ---- A
  for (int i = tid; i < nslots * 16; i += blockDim.x) ml[i] = __ldcg(slot_ptr(fc + i / 16) + i % 16);
  if (tid < 16) wml[tid] = __ldcg(wslot + tid);
  for (int i = tid; i < gq * (j1 - j0); i += blockDim.x)
    wo[i] = __ldcg(wslot + 16 + (i / (j1 - j0)) * hd + j0 + i % (j1 - j0));
  __syncthreads();
  // ---- C
  for (int g = warp; g < gq; g += nwarps) {
    float M = lane == 0 ? wml[g] : -INFINITY;
    for (int i = lane; i < nslots; i += 32) M = fmaxf(M, ml[i * 16 + g]);
    M = warp_max(M);
    // M = -inf: no kept row and no window row for this head (a token shard
    // whose chunks were all selected elsewhere): every factor and the output
    // are 0, and (M, L) = (-inf, 0) tells the caller's merge to skip it
    const bool none = M == -INFINITY;
    float L = 0.f;
    for (int i = lane; i < nslots; i += 32) {
      const float f = none ? 0.f : exp2f(ml[i * 16 + g] - M);
      sc[i * kMaxGQ + g] = f;
      L = fmaf(ml[i * 16 + 8 + g], f, L);
    }
    L = warp_sum(L);
    if (lane == 0) {
      const float f = none ? 0.f : exp2f(wml[g] - M);
      fw[g] = f;
      const float Lt = fmaf(wml[8 + g], f, L);
      Lg[g] = Lt > 0.f ? 1.f / Lt : 0.f;
      if (args.ml_out && j0 == 0) {
        float* mo = args.ml_out + (static_cast<int64_t>(b) * args.Hq + h * gq + g) * 2;
        mo[0] = M;
        mo[1] = Lt;
      }
    }
  }
  __syncthreads();
  // ---- D (float4 over rank columns, 16 slots' loads in flight; a float4
  // must not span two heads, whose slot factors differ: rV % 4 == 0)
  {
    const int n4 = rV % 4 == 0 ? gq * rV / 4 : 0;
    for (int i4 = tid; i4 < n4; i4 += blockDim.x) {
      const int g = (4 * i4) / rV;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int c0 = 0; c0 < nslots; c0 += 16) {
        float4 v[16];
#pragma unroll
        for (int t = 0; t < 16; ++t)
          v[t] = c0 + t < nslots ? __ldcg(reinterpret_cast<const float4*>(slot_ptr(fc + c0 + t) + 16) + i4)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          if (c0 + t < nslots) {
            const float f = sc[(c0 + t) * kMaxGQ + g];
            acc.x = fmaf(v[t].x, f, acc.x);
            acc.y = fmaf(v[t].y, f, acc.y);
            acc.z = fmaf(v[t].z, f, acc.z);
            acc.w = fmaf(v[t].w, f, acc.w);
          }
        }
      }
      if (vec) {
        const int c = 4 * i4 - g * rV, vv = c >> 3, e = c & 7;  // rV % 8 == 0: no float4 spans two heads
        float* dst = Us + (g * 8 + e) * nv + vv;
        dst[0] = acc.x;
        dst[nv] = acc.y;
        dst[2 * nv] = acc.z;
        dst[3 * nv] = acc.w;
      } else {
        reinterpret_cast<float4*>(Us)[i4] = acc;
      }
    }
    // other value ranks entry by entry (never the permuted layout: there rV % 8 == 0)
    for (int i = 4 * n4 + tid; i < gq * rV; i += blockDim.x) {
      const int g = i / rV;
      float acc = 0.f;
      for (int c = 0; c < nslots; ++c) acc = fmaf(__ldcg(slot_ptr(fc + c) + 16 + i), sc[c * kMaxGQ + g], acc);
      Us[i] = acc;
    }
  }
  cp_async_wait_all();
  __syncthreads();
  if (args.v_raw) {
    // values were not compressed: U_g is already the kept rows' value sum
    for (int i = tid; i < gq * ncols; i += blockDim.x) {
      const int g = i / ncols, j = j0 + i % ncols;
      out[(static_cast<int64_t>(b) * args.Hq + h * gq + g) * hd + j] = fmaf(fw[g], wo[i], Us[g * rV + j]) * Lg[g];
    }
    return;
  }
  // ---- E
  for (int jb = j0 + warp * kCombineColsPerWarp; jb < j1; jb += nwarps * kCombineColsPerWarp) {
    const int ncol = min(kCombineColsPerWarp, j1 - jb);
    float acc[kCombineColsPerWarp][kMaxGQ];
#pragma unroll
    for (int cc = 0; cc < kCombineColsPerWarp; ++cc)
#pragma unroll
      for (int g = 0; g < kMaxGQ; ++g) acc[cc][g] = 0.f;
    if (vec) {
      auto fold = [&](const uint4* w, int v) {
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          float2 f[kCombineColsPerWarp];
#pragma unroll
          for (int cc = 0; cc < kCombineColsPerWarp; ++cc)
            f[cc] = bf2_to_f2(e2 == 0 ? w[cc].x : e2 == 1 ? w[cc].y : e2 == 2 ? w[cc].z : w[cc].w);
#pragma unroll
          for (int g = 0; g < kMaxGQ; ++g) {
            if (g < gq) {
              const float u0 = Us[(g * 8 + 2 * e2) * nv + v], u1 = Us[(g * 8 + 2 * e2 + 1) * nv + v];
#pragma unroll
              for (int cc = 0; cc < kCombineColsPerWarp; ++cc) acc[cc][g] = fmaf(u0, f[cc].x, fmaf(u1, f[cc].y, acc[cc][g]));
            }
          }
        }
      };
      for (int v0 = 0; v0 < nv; v0 += 32) {
        const int v = v0 + lane;
        uint4 w[kCombineColsPerWarp];
#pragma unroll
        for (int cc = 0; cc < kCombineColsPerWarp; ++cc) {
          if (cc < ncol && v < nv)
            w[cc] = staged ? Bs[(jb - j0 + cc) * nv + v]
                           : *reinterpret_cast<const uint4*>(BtV + b * args.sbv +
                                                             static_cast<int64_t>(h * hd + jb + cc) * rV + 8 * v);
          else
            w[cc] = make_uint4(0, 0, 0, 0);
        }
        if (v < nv) fold(w, v);
      }
    } else {
      for (int c = lane; c < rV; c += 32) {
        float bv[kCombineColsPerWarp];
#pragma unroll
        for (int cc = 0; cc < kCombineColsPerWarp; ++cc)
          bv[cc] = cc < ncol ? to_f(BtV[b * args.sbv + static_cast<int64_t>(h * hd + jb + cc) * rV + c]) : 0.f;
#pragma unroll
        for (int g = 0; g < kMaxGQ; ++g)
          if (g < gq) {
            const float uu = Us[g * rV + c];
#pragma unroll
            for (int cc = 0; cc < kCombineColsPerWarp; ++cc) acc[cc][g] = fmaf(uu, bv[cc], acc[cc][g]);
          }
      }
    }
    // reduce-scatter of the 32 sums over the warp: lane l ends with the
    // total of entry l = (column cc, head g) = (l / 8, l % 8)
    static_assert(kCombineColsPerWarp * kMaxGQ == 32, "one entry per lane");
    float* a = &acc[0][0];
#pragma unroll
    for (int st = 16; st >= 1; st >>= 1) {
      const bool up = (lane & st) != 0;
#pragma unroll
      for (int i = 0; i < st; ++i) {
        const float keep = up ? a[i + st] : a[i];
        const float send = up ? a[i] : a[i + st];
        a[i] = keep + __shfl_xor_sync(0xffffffffu, send, st);
      }
    }
    const int cc = lane / kMaxGQ, g = lane % kMaxGQ;
    if (g < gq && cc < ncol) {
      const int j = jb + cc;
      out[(static_cast<int64_t>(b) * args.Hq + h * gq + g) * hd + j] = fmaf(fw[g], wo[g * (j1 - j0) + j - j0], a[0]) * Lg[g];
    }
  }
}

template <int GQ>
__global__ void __launch_bounds__(kAttendThreads, 1)
    sr_attend_tc_kernel(const __grid_constant__ CUtensorMap mapAK, const __grid_constant__ CUtensorMap mapBK,
                        const __grid_constant__ CUtensorMap mapAV, const AttendArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int NKA = args.rK / 64;
  const int NKS = (NKA + kKAtoms - 1) / kKAtoms;  // key stages per tile
  const int NMB = (args.rV + 127) / 128;  // value M-blocks of 128 rank columns
  const int NAVp = 2 * NMB;               // 64-column atoms per value slab (zero-padded)
  const int NAV = args.rV / 64;           // atoms actually loaded
  uint8_t* Ka = smem + kSmemKa;
  uint8_t* Kb = smem + kSmemKb;
  uint8_t* Vs = smem + kSmemV;
  uint8_t* Ps = smem + kSmemP;
  float* alpha_s = reinterpret_cast<float*>(smem + kSmemAlpha);
  float* q_s = reinterpret_cast<float*>(smem + kSmemQ);
  float* base_s = reinterpret_cast<float*>(smem + kSmemBase);
  float* rot_s = reinterpret_cast<float*>(smem + kSmemRot);
  double* ft = reinterpret_cast<double*>(smem + kSmemFt);
  float* red = reinterpret_cast<float*>(smem + kSmemRed);
  float* spart = reinterpret_cast<float*>(smem + kSmemSpart);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSmemBars);
  uint64_t* kfull = bars;
  uint64_t* kempty = kfull + kKStages;
  uint64_t* bfull = kempty + kKStages;
  uint64_t* bempty = bfull + kBStages;
  uint64_t* vfull = bempty + kBStages;
  uint64_t* vempty = vfull + kVStages;
  uint64_t* accfull = vempty + kVStages;
  uint64_t* accempty = accfull + 2;
  uint64_t* pfull = accempty + 2;
  uint64_t* pempty = pfull + 2;
  uint64_t* vaccfull = pempty + 2;
  uint64_t* vaccempty = vaccfull + 2;
  uint64_t* drain = vaccempty + 2;  // [2] last commit of each MMA issuer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x;
  const int tb = tile_begin(cta, args.n_tiles, args.ctas), te = tile_begin(cta + 1, args.n_tiles, args.ctas);
  const int tpu = args.tiles_per_unit, k = args.k;

  if (tid == 0) {
    for (int i = 0; i < kKStages; ++i) { mbar_init(&kfull[i], 1); mbar_init(&kempty[i], 1); }
    for (int i = 0; i < kBStages; ++i) { mbar_init(&bfull[i], 1); mbar_init(&bempty[i], 1); }
    for (int i = 0; i < kVStages; ++i) { mbar_init(&vfull[i], 1); mbar_init(&vempty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accfull[i], 1);
      mbar_init(&accempty[i], 256);
      mbar_init(&pfull[i], 128);
      mbar_init(&pempty[i], 129);
      mbar_init(&vaccfull[i], 1);
      mbar_init(&vaccempty[i], 128);
      mbar_init(&drain[i], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (tid < 64) ft[tid] = args.ft[tid];
  // rows of P beyond the query group, and value atoms past the rank (when it
  // is not a multiple of 128), are never loaded and stay zero
  for (int i = tid; i < 2 * kPBytes / 16; i += blockDim.x) reinterpret_cast<uint4*>(Ps)[i] = make_uint4(0, 0, 0, 0);
  for (int i = tid; i < kVStages * 16384 / 16; i += blockDim.x) reinterpret_cast<uint4*>(Vs)[i] = make_uint4(0, 0, 0, 0);
  __syncthreads();
  for (int i = tid; i < 8 * 64; i += blockDim.x) {
    const int e = i >> 6, j = i & 63;
    float c, sn;
    rope_cs(ft[j], static_cast<double>(e), &c, &sn);
    rot_s[e * kRopeStride + 2 * j] = c;
    rot_s[e * kRopeStride + 2 * j + 1] = sn;
  }
  if (warp == 14) tmem_alloc(tmem_slot, 512);
  if (warp == 12 && lane == 0) {
    prefetch_tmap(&mapAK);
    prefetch_tmap(&mapBK);
    prefetch_tmap(&mapAV);
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  allow_next_grid();
  // The first stage's Bt_K atoms depend on the CTA's first unit only, not on
  // the selection the previous kernel writes: issue them before waiting.
  int b_pre = 0;
  if (warp == 12 && lane == 0 && te > tb) {
    const int u = tb / tpu, b = u / args.Hkv, h = u % args.Hkv;
    b_pre = min(kKAtoms, NKA);
    for (int a = 0; a < b_pre; ++a) {
      mbar_arrive_expect_tx(&bfull[a], kAtomBytes);
      tma_load_3d(Kb + a * kAtomBytes, &mapBK, &bfull[a], a * 64, h * 128, args.sbk ? b : 0);
    }
  }
  wait_prior_grid();  // the selection

  if (warp == 12) {
    // ------------------------------------------------------ TMA producer (keys)
    if (lane == 0) {
      uint32_t ks = 0, bs = 0;
      for (int x = tb; x < te && !*abort_flag; ++x) {
        const int u = x / tpu, ti = x % tpu;
        const int b = u / args.Hkv, h = u % args.Hkv;
        const int nch = min(kTileChunks, k - ti * kTileChunks);
        const int32_t* su = args.sel + static_cast<int64_t>(u) * k + ti * kTileChunks;
        int rows[kTileChunks];
#pragma unroll
        for (int ch = 0; ch < kTileChunks; ++ch)
          rows[ch] = ch < nch && kept_here(args, su[ch]) ? args.sink + (su[ch] - args.c_lo) * 8 : 0;
        // one 4-D box per chunk covers kKAtoms atoms (8 rows x 128 columns);
        // the Bt_K atoms of the stage follow on their own ring (L2 hits)
        // (an odd atom count leaves the last box half out of range: TMA fills
        // it with zeros and still delivers the whole box; it gets no MMA)
        bool ok = true;
        for (int sk = 0; sk < NKS && ok; ++sk, ++ks) {
          const int slot = ks % kKStages;
          if (!mbar_wait(&kempty[slot], ((ks / kKStages) & 1) ^ 1, args.status)) { *abort_flag = 1; ok = false; break; }
          mbar_arrive_expect_tx(&kfull[slot], nch * kKAtoms * 1024);
          for (int ch = 0; ch < nch; ++ch)
            tma_load_4d(Ka + slot * kKStageBytes + ch * kKAtoms * 1024, &mapAK, &kfull[slot], 0, rows[ch],
                        sk * kKAtoms, b);
          const int na = min(kKAtoms, NKA - sk * kKAtoms);
          for (int a = 0; a < na; ++a, ++bs) {
            if (static_cast<int>(bs) < b_pre) continue;  // issued before the wait
            const int bslot = bs % kBStages;
            if (!mbar_wait(&bempty[bslot], ((bs / kBStages) & 1) ^ 1, args.status)) { *abort_flag = 1; ok = false; break; }
            mbar_arrive_expect_tx(&bfull[bslot], kAtomBytes);
            tma_load_3d(Kb + bslot * kAtomBytes, &mapBK, &bfull[bslot], (sk * kKAtoms + a) * 64, h * 128,
                        args.sbk ? b : 0);
          }
        }
      }
      // on abort, the copies already issued still land in Ka / Kb: wait for
      // them before the CTA releases its shared memory
      if (*abort_flag) {
        drain_ring(kfull, kKStages, ks, args.status);
        drain_ring(bfull, kBStages, max(bs, static_cast<uint32_t>(b_pre)), args.status);
      }
    }
  } else if (warp == 13) {
    // ---------------------------------------------------- TMA producer (values)
    // a stage holds two chunks (16 rows); a missing second chunk is replaced by
    // the first (finite data; its softmax weights are zero)
    if (lane == 0) {
      uint32_t vsn = 0;
      // values are needed only once the first tile's softmax weights exist:
      // start after the first key stage has landed, so that the key path's
      // first loads are not queued behind the value ring's
      if (te > tb && !mbar_wait(&kfull[0], 0, args.status)) *abort_flag = 1;
      for (int x = tb; x < te && !*abort_flag; ++x) {
        const int u = x / tpu, ti = x % tpu;
        // batch coordinate, first 64-column atom and row of each chunk's value
        // rows: the unit's rank columns; head h's columns of V when values are
        // uncompressed; the staged rows of selection position c when they were
        // gathered from host memory
        const int b = args.v_raw == 2 ? u : u / args.Hkv;
        const int vz = args.v_raw == 1 ? (u % args.Hkv) * NAV : 0;
        const int nch = min(kTileChunks, k - ti * kTileChunks);
        const int32_t* su = args.sel + static_cast<int64_t>(u) * k + ti * kTileChunks;
        const int pos0 = ti * kTileChunks;
        int rows[kTileChunks];
#pragma unroll
        for (int ch = 0; ch < kTileChunks; ++ch)
          rows[ch] = ch < nch ? (args.v_raw == 2 ? (pos0 + ch) * 8
                                                 : kept_here(args, su[ch]) ? args.sink + (su[ch] - args.c_lo) * 8 : 0)
                              : 0;
        for (int v = 0; v < (nch + 1) / 2 && !*abort_flag; ++v, ++vsn) {
          const int slot = vsn % kVStages;
          if (!mbar_wait(&vempty[slot], ((vsn / kVStages) & 1) ^ 1, args.status)) { *abort_flag = 1; break; }
          mbar_arrive_expect_tx(&vfull[slot], 2 * NAV * 1024);
          for (int c2 = 0; c2 < 2; ++c2) {
            const int ch = (2 * v + c2 < nch) ? 2 * v + c2 : 2 * v;
            tma_load_4d(Vs + slot * 16384 + c2 * NAVp * 1024, &mapAV, &vfull[slot], 0, rows[ch], vz, b);
          }
        }
      }
      if (*abort_flag) drain_ring(vfull, kVStages, vsn, args.status);
    }
  } else if (warp == 14) {
    // -------------------------------------------------------- key MMA issuer
    if (lane == 0) {
      const uint32_t idk = umma_idesc_bf16(128, 128);
      uint32_t ks = 0, bs = 0;
      auto issue_keys = [&](int j) -> bool {
        const int buf = j & 1;
        if (!mbar_wait(&accempty[buf], ((j >> 1) & 1) ^ 1, args.status)) return false;
        tc_fence_after();
        const uint32_t dtm = tmem + buf * 128;
        for (int sk = 0; sk < NKS; ++sk, ++ks) {
          const int slot = ks % kKStages;
          if (!mbar_wait(&kfull[slot], (ks / kKStages) & 1, args.status)) return false;
          const int na = min(kKAtoms, NKA - sk * kKAtoms);
          for (int a = 0; a < na; ++a, ++bs) {
            const int bslot = bs % kBStages;
            if (!mbar_wait(&bfull[bslot], (bs / kBStages) & 1, args.status)) return false;
            tc_fence_after();
            const uint64_t ad = umma_desc_sw128(smem_u32(Ka + slot * kKStageBytes + a * 1024), kKAtoms * 1024);
            const uint64_t bd = umma_desc_sw128(smem_u32(Kb + bslot * kAtomBytes));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16(dtm, ad + 2 * kk, bd + 2 * kk, idk, (sk | a | kk) ? 1u : 0u);
            umma_commit(&bempty[bslot]);
          }
          umma_commit(&kempty[slot]);
        }
        umma_commit(&accfull[buf]);
        return true;
      };
      bool ok = true;
      int j = 0;
      for (int x = tb; x < te && ok && !*abort_flag; ++x, ++j) ok = issue_keys(j);
      if (!ok) *abort_flag = 1;
      // every MMA issued by this thread has finished before TMEM is released
      umma_commit(&drain[0]);
      (void)mbar_wait(&drain[0], 0, args.status);
    }
  } else if (warp == 15) {
    // ------------------------------------------------------ value MMA issuer
    if (lane == 0) {
      const uint32_t idv = umma_idesc_bf16(128, 16, true, false);
      uint32_t vsn = 0;
      auto issue_values = [&](int j, int x) -> bool {
        const int pb = j & 1;
        const int ti = x % tpu;
        const int nch = min(kTileChunks, k - ti * kTileChunks);
        if (!mbar_wait(&pfull[pb], (j >> 1) & 1, args.status)) return false;
        if (!mbar_wait(&vaccempty[pb], ((j >> 1) & 1) ^ 1, args.status)) return false;
        tc_fence_after();
        const uint32_t dtm = tmem + kVAccCol + pb * 64;
        for (int v = 0; v < (nch + 1) / 2; ++v, ++vsn) {
          const int slot = vsn % kVStages;
          if (!mbar_wait(&vfull[slot], (vsn / kVStages) & 1, args.status)) return false;
          tc_fence_after();
          const uint64_t pd = umma_desc_sw128(smem_u32(Ps + pb * kPBytes + (v >> 2) * 2048 + (v & 3) * 32));
          for (int mb = 0; mb < NMB; ++mb) {
            const uint64_t ad = umma_desc_sw128_mn(smem_u32(Vs + slot * 16384 + 2 * mb * 1024), 1024, NAVp * 1024);
            umma_bf16(dtm + mb * 16, ad, pd, idv, v > 0 ? 1u : 0u);
          }
          umma_commit(&vempty[slot]);
        }
        umma_commit(&vaccfull[pb]);
        umma_commit(&pempty[pb]);
        return true;
      };
      bool ok = true;
      int j = 0;
      for (int x = tb; x < te && ok && !*abort_flag; ++x, ++j) ok = issue_values(j, x);
      if (!ok) *abort_flag = 1;
      umma_commit(&drain[1]);
      (void)mbar_wait(&drain[1], 0, args.status);
    }
  } else if (warp < 8) {
    // --------------------------------------- key epilogue: RoPE, q.k, softmax
    const int lq = warp & 3, hf = warp >> 2;  // lane quarter, frequency half
    const int row = lq * 32 + lane;
    const int et = tid;                       // 0..255
    const float qscale = rsqrtf(128.0f) * kLog2e;
    float m[GQ], l[GQ];
    int cur_u = -1, j = 0;
    for (int x = tb; x < te && !*abort_flag; ++x, ++j) {
      const int u = x / tpu, ti = x % tpu;
      const int nch = min(kTileChunks, k - ti * kTileChunks);
      const int32_t* su = args.sel + static_cast<int64_t>(u) * k + ti * kTileChunks;
      named_bar_sync(1, 256);  // the previous tile's readers of q_s / base_s / spart are done
      if (u != cur_u) {
        const int b = u / args.Hkv, h = u % args.Hkv;
        for (int i = et; i < 128 * kMaxGQ; i += 256) {
          const int jj = i / kMaxGQ, g = i % kMaxGQ;
          q_s[i] = g < GQ ? to_f(reinterpret_cast<const __nv_bfloat16*>(args.q)[(static_cast<int64_t>(b) * args.Hq +
                                                                                 h * GQ + g) * 128 + jj]) * qscale
                          : 0.f;
        }
        cur_u = u;
#pragma unroll
        for (int g = 0; g < GQ; ++g) { m[g] = -INFINITY; l[g] = 0.f; }
      }
      // base angle of every chunk of the tile: (cos, sin)(t0 f_j), t0 = first token
      for (int i = et; i < kTileChunks * 64; i += 256) {
        const int ch = i >> 6, jj = i & 63;
        float c = 1.f, sn = 0.f;
        if (ch < nch && kept_here(args, su[ch]))
          rope_cs(ft[jj], static_cast<double>(args.pos_off + args.sink + static_cast<int64_t>(su[ch] - args.c_lo) * 8),
                  &c, &sn);
        base_s[ch * kRopeStride + 2 * jj] = c;
        base_s[ch * kRopeStride + 2 * jj + 1] = sn;
      }
      named_bar_sync(1, 256);
      const int ch = row >> 3, e = row & 7;
      const bool valid = ch < nch && kept_here(args, su[ch]);
      const float2* bse = reinterpret_cast<const float2*>(base_s + ch * kRopeStride);
      const float2* rte = reinterpret_cast<const float2*>(rot_s + e * kRopeStride);
      const int buf = j & 1;
      if (!mbar_wait(&accfull[buf], (j >> 1) & 1, args.status)) { *abort_flag = 1; break; }
      __syncwarp();  // converged for the warp-wide tcgen05.ld
      tc_fence_after();
      const uint32_t taddr = tmem + (static_cast<uint32_t>(lq * 32) << 16) + buf * 128;
      float s0[GQ], s1[GQ];
#pragma unroll
      for (int g = 0; g < GQ; ++g) { s0[g] = 0.f; s1[g] = 0.f; }
#pragma unroll 1
      for (int jb = 2 * hf; jb < 2 * hf + 2; ++jb) {
        float lo[16], hi[16];
        tmem_ld16(taddr + jb * 16, lo);
        tmem_ld16(taddr + 64 + jb * 16, hi);
        tmem_ld_wait();
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const int jx = jb * 16 + jj;
          const float2 b0 = bse[jx], r0 = rte[jx];
          const float c = b0.x * r0.x - b0.y * r0.y;
          const float sn = b0.y * r0.x + b0.x * r0.y;
          const float y0 = lo[jj] * c - hi[jj] * sn;
          const float y1 = hi[jj] * c + lo[jj] * sn;
          const float4* q0 = reinterpret_cast<const float4*>(q_s + jx * kMaxGQ);
          const float4* q1 = reinterpret_cast<const float4*>(q_s + (64 + jx) * kMaxGQ);
          float qa[8], qb[8];
          *reinterpret_cast<float4*>(qa) = q0[0];
          *reinterpret_cast<float4*>(qb) = q1[0];
          if (GQ > 4) {
            *reinterpret_cast<float4*>(qa + 4) = q0[1];
            *reinterpret_cast<float4*>(qb + 4) = q1[1];
          }
#pragma unroll
          for (int g = 0; g < GQ; ++g) {
            if (jj & 1) s1[g] = fmaf(qa[g], y0, fmaf(qb[g], y1, s1[g]));
            else s0[g] = fmaf(qa[g], y0, fmaf(qb[g], y1, s0[g]));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&accempty[buf]);
      if (hf == 1) {
#pragma unroll
        for (int g = 0; g < GQ; ++g) spart[row * kMaxGQ + g] = s0[g] + s1[g];
      }
      named_bar_sync(1, 256);
      if (hf == 1) continue;
      float s[GQ];
#pragma unroll
      for (int g = 0; g < GQ; ++g) s[g] = s0[g] + s1[g] + spart[row * kMaxGQ + g];
      // tile maximum per query head (the 128 threads of half 0)
      float tmax[GQ];
#pragma unroll
      for (int g = 0; g < GQ; ++g) {
        if (!valid) s[g] = -INFINITY;
        const float w = warp_max(s[g]);
        if (lane == 0) red[lq * 8 + g] = w;
      }
      named_bar_sync(2, 128);
#pragma unroll
      for (int g = 0; g < GQ; ++g)
        tmax[g] = fmaxf(fmaxf(red[0 * 8 + g], red[1 * 8 + g]), fmaxf(red[2 * 8 + g], red[3 * 8 + g]));
      float alpha[GQ];
      __nv_bfloat16 pbf[GQ];
#pragma unroll
      for (int g = 0; g < GQ; ++g) {
        const float mn = fmaxf(m[g], tmax[g]);
        // (no kept row yet: mn = -inf, nothing to rescale)
        alpha[g] = mn == -INFINITY ? 1.f : exp2f(m[g] - mn);
        // the weights enter the value MMA as bf16: the sum uses the same values
        pbf[g] = __float2bfloat16_rn(valid && mn != -INFINITY ? exp2f(s[g] - mn) : 0.f);
        m[g] = mn;
        const float w = warp_sum(__bfloat162float(pbf[g]));
        if (lane == 0) red[32 + lq * 8 + g] = w;
      }
      named_bar_sync(2, 128);
#pragma unroll
      for (int g = 0; g < GQ; ++g)
        l[g] = l[g] * alpha[g] + (red[32 + g] + red[40 + g] + red[48 + g] + red[56 + g]);
      const int pb = j & 1;
      if (!mbar_wait(&pempty[pb], ((j >> 1) & 1) ^ 1, args.status)) { *abort_flag = 1; break; }
      // P[g][t] (K-major, 128-byte swizzle): row g of the K-atom t / 64
      {
        const int katom = row >> 6, kin = row & 63;
        uint8_t* pbase = Ps + pb * kPBytes + katom * 2048;
#pragma unroll
        for (int g = 0; g < GQ; ++g) {
          const int off = (g >> 3) * 1024 + (g & 7) * 128 + ((((kin * 2) >> 4) ^ (g & 7)) << 4) + ((kin * 2) & 15);
          *reinterpret_cast<__nv_bfloat16*>(pbase + off) = pbf[g];
        }
      }
      if (et == 0)
#pragma unroll
        for (int g = 0; g < GQ; ++g) alpha_s[pb * kMaxGQ + g] = alpha[g];
      fence_proxy_async();
      mbar_arrive(&pfull[pb]);
      const bool seg_end = (x + 1 == te) || ((x + 1) / tpu != u);
      if (seg_end && et == 0) {
        const int u_first = tb / tpu;
        float* slot = args.part + (static_cast<int64_t>(cta) * args.max_units + (u - u_first)) * args.slot_floats;
#pragma unroll
        for (int g = 0; g < GQ; ++g) { slot[g] = m[g]; slot[8 + g] = l[g]; }
      }
    }
  } else if (warp < 12) {
    // ------------------------- value epilogue: u_g = u_g alpha + P A_V (TMEM)
    const int lq = warp & 3;
    float acc[4][GQ];
#pragma unroll
    for (int mb = 0; mb < 4; ++mb)
#pragma unroll
      for (int g = 0; g < GQ; ++g) acc[mb][g] = 0.f;
    int cur_u = -1, j = 0;
    for (int x = tb; x < te && !*abort_flag; ++x, ++j) {
      const int u = x / tpu;
      if (u != cur_u) {
        cur_u = u;
#pragma unroll
        for (int mb = 0; mb < 4; ++mb)
#pragma unroll
          for (int g = 0; g < GQ; ++g) acc[mb][g] = 0.f;
      }
      const int pb = j & 1;
      if (!mbar_wait(&vaccfull[pb], (j >> 1) & 1, args.status)) { *abort_flag = 1; break; }
      __syncwarp();  // converged for the warp-wide tcgen05.ld
      tc_fence_after();
      float al[GQ];
#pragma unroll
      for (int g = 0; g < GQ; ++g) al[g] = alpha_s[pb * kMaxGQ + g];
      const uint32_t taddr = tmem + (static_cast<uint32_t>(lq * 32) << 16) + kVAccCol + pb * 64;
#pragma unroll
      for (int mb = 0; mb < 4; ++mb) {
        if (mb < NMB) {
          float v[16];
          tmem_ld16(taddr + mb * 16, v);
          tmem_ld_wait();
#pragma unroll
          for (int g = 0; g < GQ; ++g) acc[mb][g] = fmaf(acc[mb][g], al[g], v[g]);
        }
      }
      tc_fence_before();
      mbar_arrive(&vaccempty[pb]);
      mbar_arrive(&pempty[pb]);
      const bool seg_end = (x + 1 == te) || ((x + 1) / tpu != u);
      if (seg_end) {
        const int u_first = tb / tpu;
        float* slot = args.part + (static_cast<int64_t>(cta) * args.max_units + (u - u_first)) * args.slot_floats;
#pragma unroll
        for (int mb = 0; mb < 4; ++mb) {
          const int c = mb * 128 + lq * 32 + lane;
          if (mb < NMB && c < args.rV)
#pragma unroll
            for (int g = 0; g < GQ; ++g) slot[16 + g * args.rV + c] = acc[mb][g];
        }
      }
    }
  }
  // lane 0 of the role warps may still be in its loop: reconverge every warp
  // before the block-wide barrier, so that the barrier cannot complete (and
  // TMEM be released) while a role thread is still issuing
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 14) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

size_t attend_tc_smem() { return 1024 + kSmemEnd; }

// ----------------------------------------------------------- sr_combine
// Grid (unit, column split of kCombineSplit), 512 threads.
template <typename T>
__global__ void __launch_bounds__(kCombineThreads) sr_combine_kernel(const T* __restrict__ BtV,
                                                                     const float* __restrict__ win,
                                                                     const AttendArgs args, int hd,
                                                                     float* __restrict__ out) {
  extern __shared__ float4 smf4[];
  const int cols = (hd + kCombineSplit - 1) / kCombineSplit, j0 = blockIdx.y * cols, j1 = min(hd, j0 + cols);
  merge_unit<T>(BtV, win, args, hd, out, blockIdx.x, j0, j1, reinterpret_cast<float*>(smf4));
}


// ---------------------------------------------------- sr_attend (SIMT)
// Same schedule and partial format; rebuilds both K and the value basis sums on
// CUDA cores.  Tiles are 16 chunks of `chunk` rows, handled 32 rows at a time.
template <typename T>
__global__ void __launch_bounds__(256) sr_attend_simt_kernel(const T* __restrict__ q, const T* __restrict__ AK,
                                                             const T* __restrict__ BtK, const T* __restrict__ AV,
                                                             const AttendArgs args, int hd, int chunk,
                                                             int64_t sak, int64_t sav) {
  extern __shared__ double smd[];
  const int gq = args.Hq / args.Hkv;
  double* ft = smd;                                        // [hd/2]
  float* qs = reinterpret_cast<float*>(smd + hd / 2);      // [gq][hd] scaled
  float* Ks = qs + gq * hd;             // [32][hd]
  float* us = Ks + 32 * hd;             // [gq][rV]
  float* ps = us + gq * args.rV;        // [32][gq]
  float* ms = ps + 32 * gq;             // [gq] running max
  float* ls = ms + kMaxGQ;              // [gq] running sum
  float* al = ls + kMaxGQ;              // [gq] rescale
  const int tid = threadIdx.x;
  const int cta = blockIdx.x;
  const int tb = tile_begin(cta, args.n_tiles, args.ctas), te = tile_begin(cta + 1, args.n_tiles, args.ctas);
  const int tpu = args.tiles_per_unit, k = args.k, half = hd / 2;
  const int d = args.Hkv * hd;
  const float qscale = rsqrtf(static_cast<float>(hd)) * kLog2e;
  for (int j = tid; j < half; j += blockDim.x) ft[j] = args.ft[j];
  wait_prior_grid();  // the selection
  int cur_u = -1;
  for (int x = tb; x < te; ++x) {
    const int u = x / tpu, ti = x % tpu;
    const int b = u / args.Hkv, h = u % args.Hkv;
    __syncthreads();
    if (u != cur_u) {
      cur_u = u;
      for (int i = tid; i < gq * hd; i += blockDim.x)
        qs[i] = to_f(q[(static_cast<int64_t>(b) * args.Hq + h * gq) * hd + i]) * qscale;
      for (int i = tid; i < gq * args.rV; i += blockDim.x) us[i] = 0.f;
      if (tid < gq) { ms[tid] = -INFINITY; ls[tid] = 0.f; }
    }
    __syncthreads();
    const int nch = min(kTileChunks, k - ti * kTileChunks);
    const int rows = nch * chunk;
    for (int rb = 0; rb < rows; rb += 32) {
      const int nr = min(32, rows - rb);
      // rebuilt, rotated keys of this row block
      for (int i = tid; i < nr * half; i += blockDim.x) {
        const int r = i / half, jj = i % half;
        const int rr = rb + r;
        const int cc = args.sel[static_cast<int64_t>(u) * k + ti * kTileChunks + rr / chunk];
        const bool kept = kept_here(args, cc);
        const int64_t t = args.sink + static_cast<int64_t>(kept ? cc - args.c_lo : 0) * chunk + rr % chunk;
        const T* a = AK + b * sak + t * args.rK;
        const T* b0 = BtK + b * args.sbk + static_cast<int64_t>(h * hd + jj) * args.rK;
        const T* b1 = BtK + b * args.sbk + static_cast<int64_t>(h * hd + jj + half) * args.rK;
        float y0 = 0.f, y1 = 0.f;
        for (int c = 0; c < args.rK; ++c) {
          const float av = to_f(a[c]);
          y0 = fmaf(av, to_f(b0[c]), y0);
          y1 = fmaf(av, to_f(b1[c]), y1);
        }
        float cs, sn;
        rope_cs(ft[jj], static_cast<double>(args.pos_off + t), &cs, &sn);
        Ks[r * hd + jj] = kept ? y0 * cs - y1 * sn : 0.f;
        Ks[r * hd + jj + half] = kept ? y1 * cs + y0 * sn : 0.f;
      }
      __syncthreads();
      for (int i = tid; i < nr * gq; i += blockDim.x) {
        const int r = i / gq, g = i % gq;
        const int rr = rb + r;
        float s = 0.f;
        for (int jj = 0; jj < hd; ++jj) s = fmaf(qs[g * hd + jj], Ks[r * hd + jj], s);
        const bool kept = kept_here(args, args.sel[static_cast<int64_t>(u) * k + ti * kTileChunks + rr / chunk]);
        ps[r * gq + g] = kept ? s : -INFINITY;
      }
      __syncthreads();
      if (tid < gq) {
        const int g = tid;
        float mx = ms[g];
        for (int r = 0; r < nr; ++r) mx = fmaxf(mx, ps[r * gq + g]);
        al[g] = mx == -INFINITY ? 1.f : exp2f(ms[g] - mx);
        float sum = 0.f;
        for (int r = 0; r < nr; ++r) {
          const float pv = mx == -INFINITY ? 0.f : exp2f(ps[r * gq + g] - mx);
          ps[r * gq + g] = pv;
          sum += pv;
        }
        ls[g] = ls[g] * al[g] + sum;
        ms[g] = mx;
      }
      __syncthreads();
      // value rows: A_V [t][rV]; head h's columns of V [t][d] when uncompressed;
      // the unit's staged rows [k][chunk][hd] when gathered from host memory
      const int64_t vld = args.v_raw == 1 ? d : args.rV;
      const T* avb = args.v_raw == 2 ? AV + static_cast<int64_t>(u) * k * chunk * hd
                                      : AV + b * sav + (args.v_raw ? h * hd : 0);
      for (int i = tid; i < gq * args.rV; i += blockDim.x) {
        const int g = i / args.rV, c = i % args.rV;
        float acc = us[i] * al[g];
        for (int r = 0; r < nr; ++r) {
          const int rr = rb + r;
          const int64_t t =
              args.v_raw == 2
                  ? static_cast<int64_t>(ti * kTileChunks + rr / chunk) * chunk + rr % chunk
                  : args.sink +
                        static_cast<int64_t>(kept_here(args, args.sel[static_cast<int64_t>(u) * k + ti * kTileChunks + rr / chunk])
                                                 ? args.sel[static_cast<int64_t>(u) * k + ti * kTileChunks + rr / chunk] - args.c_lo
                                                 : 0) * chunk + rr % chunk;
          acc = fmaf(ps[r * gq + g], to_f(avb[t * vld + c]), acc);
        }
        us[i] = acc;
      }
      __syncthreads();
    }
    const bool seg_end = (x + 1 == te) || ((x + 1) / tpu != u);
    if (seg_end) {
      const int u_first = tb / tpu;
      float* slot = args.part + (static_cast<int64_t>(cta) * args.max_units + (u - u_first)) * args.slot_floats;
      for (int i = tid; i < gq * args.rV; i += blockDim.x) slot[16 + i] = us[i];
      if (tid < gq) { slot[tid] = ms[tid]; slot[8 + tid] = ls[tid]; }
    }
  }
}


// ------------------------------------------------ host-resident values
// xK-SR with the uncompressed values off the GPU (the xKV explainer,
// "选择性重建": the value cache stays in host memory and only the selected
// tokens' rows are fetched): the kept chunks' rows of head h, read from
// page-locked host memory over the host link with 16-byte loads, land in a
// device staging buffer [units][k][chunk][hd] that the attend kernels read.
template <typename T>
__global__ void __launch_bounds__(256) gather_host_values_kernel(const T* __restrict__ V, int64_t vbs,
                                                                 const int32_t* __restrict__ sel, int k, int Hkv,
                                                                 int hd, int chunk, int sink, T* __restrict__ stage) {
  allow_next_grid();
  wait_prior_grid();  // the selection
  constexpr int kVec = 16 / sizeof(T);
  constexpr int kUnroll = 4;
  const int u = blockIdx.y, b = u / Hkv, h = u % Hkv;
  const int64_t d = static_cast<int64_t>(Hkv) * hd;
  const int per_row = hd / kVec;
  const int64_t total = static_cast<int64_t>(k) * chunk * per_row;  // 16-byte pieces of the unit
  const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i0 < total; i0 += kUnroll * step) {
    uint4 v[kUnroll];
    int64_t dst[kUnroll];
#pragma unroll
    for (int r = 0; r < kUnroll; ++r) {
      const int64_t i = i0 + r * step;
      dst[r] = -1;
      if (i < total) {
        const int piece = static_cast<int>(i % per_row);
        const int64_t rr = i / per_row;  // staged row of the unit
        const int pos = static_cast<int>(rr / chunk), e = static_cast<int>(rr % chunk);
        const int64_t t = sink + static_cast<int64_t>(sel[static_cast<int64_t>(u) * k + pos]) * chunk + e;
        v[r] = *reinterpret_cast<const uint4*>(V + b * vbs + t * d + h * hd + piece * kVec);
        dst[r] = ((static_cast<int64_t>(u) * k + pos) * chunk + e) * hd + piece * kVec;
      }
    }
#pragma unroll
    for (int r = 0; r < kUnroll; ++r)
      if (dst[r] >= 0) *reinterpret_cast<uint4*>(stage + dst[r]) = v[r];
  }
}

size_t combine_smem(int gq, int rV, int hd) {
  const int cols = (hd + kCombineSplit - 1) / kCombineSplit;
  const size_t stage = static_cast<size_t>(cols) * rV * 2;
  return (static_cast<size_t>(gq) * rV + kMaxSlots * 16 + kMaxSlots * kMaxGQ + 16 + 2 * kMaxGQ +
          static_cast<size_t>(gq) * cols + 2 + 2 * kMaxSlots) * 4 + 16 + 16 +
         (stage <= static_cast<size_t>(kCombineStageBytes) ? stage : 0);
}

size_t simt_smem(int gq, int rV, int hd) {
  return (static_cast<size_t>(gq) * hd + 32 * hd + gq * rV + 32 * gq + 3 * kMaxGQ + 8) * 4 + (hd / 2) * 8 + 16;
}

bool tc_shape_ok(const xkv_sr_params* p) {
  const int gq = p->n_q_heads / p->n_kv_heads;
  return p->dtype == XKV_BF16 && p->head_dim == 128 && p->chunk == 8 && p->rank_k % 64 == 0 &&
         p->rank_v % 64 == 0 && p->rank_k <= 2048 && p->rank_v <= 512 && gq <= kMaxGQ &&
         p->a_k_batch_stride % 8 == 0 && p->a_v_batch_stride % 8 == 0 && p->bt_k_batch_stride % 8 == 0 &&
         !force_simt();
}

}  // namespace

xkv_status sr_plan(const xkv_sr_params* p, SRPlan* plan) {
  const int64_t n_mid = (p->T - p->sink - p->recent) / p->chunk;
  const int gq = p->n_q_heads / p->n_kv_heads;
  plan->units = p->batch * p->n_kv_heads;
  plan->tiles_per_unit = (p->topk + kTileChunks - 1) / kTileChunks;
  plan->total_tiles = plan->units * plan->tiles_per_unit;
  plan->tc = tc_shape_ok(p);
  const int sms = num_sms();
  plan->ctas = std::min(plan->total_tiles, plan->tc ? sms : 2 * sms);
  int mx = 1;
  for (int c = 0; c < plan->ctas; ++c) {
    const int tb = tile_begin(c, plan->total_tiles, plan->ctas), te = tile_begin(c + 1, plan->total_tiles, plan->ctas);
    if (te > tb) mx = std::max(mx, (te - 1) / plan->tiles_per_unit - tb / plan->tiles_per_unit + 1);
  }
  plan->max_units_per_cta = mx;
  // a multiple of 4 floats, so that every slot's float4 reads stay aligned
  plan->slot_floats = (16 + static_cast<size_t>(std::max(gq, 1)) * p->rank_v + 3) & ~size_t(3);
  size_t off = 0;
  plan->off_scores = off;  // rows padded to a multiple of 4 floats
  off = align_up(off + static_cast<size_t>(plan->units) * ((n_mid + 3) & ~int64_t(3)) * 4);
  plan->off_sel = off;
  off = align_up(off + static_cast<size_t>(plan->units) * p->topk * 4);
  plan->off_part = off;
  off = align_up(off + static_cast<size_t>(plan->ctas) * mx * plan->slot_floats * 4);
  plan->off_win = off;
  off = align_up(off + static_cast<size_t>(plan->units) * (16 + static_cast<size_t>(gq) * p->head_dim) * 4);
  plan->bytes = off;
  return XKV_OK;
}

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel in the stream drains and waits for it in
// wait_prior_grid before reading its output.
template <typename... KArgs, typename... Args>
cudaError_t launch_after_prior(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                               Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// stage-timing events (see xkv_sr_profile_enable)
struct SRProfile {
  bool on = false, recorded = false;
  int device = -1;
  cudaEvent_t ev[5] = {};
};
SRProfile g_prof;

inline void prof_mark(int i, cudaStream_t st) {
  int dev = -1;
  if (g_prof.on && cudaGetDevice(&dev) == cudaSuccess && dev == g_prof.device) {
    cudaEventRecord(g_prof.ev[i], st);
    if (i == 4) g_prof.recorded = true;
  }
}

template <typename T>
static xkv_status sr_launch_t(const xkv_sr_params* p, const SRPlan& plan, const void* q, const void* A_K,
                              const void* Bt_K, const void* A_V, const void* Bt_V, const void* lm,
                              const void* sr_K, const void* sr_V, float* out, int32_t* sel_out, void* ws,
                              const void* v_host, void* stage, const SRShard* shard, cudaStream_t st) {
  const int64_t n_mid = (p->T - p->sink - p->recent) / p->chunk;
  const int gq = p->n_q_heads / p->n_kv_heads;
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* scores = reinterpret_cast<float*>(w + plan.off_scores);
  int32_t* sel = reinterpret_cast<int32_t*>(w + plan.off_sel);
  float* part = reinterpret_cast<float*>(w + plan.off_part);
  float* win = reinterpret_cast<float*>(w + plan.off_win);
  prof_mark(0, st);
  // 1. chunk scores
  {
    const int cpb = 512;
    dim3 grid(static_cast<unsigned>((n_mid + cpb - 1) / cpb), static_cast<unsigned>(plan.units));
    const int64_t lm_cap = p->landmark_capacity > 0 ? p->landmark_capacity : n_mid;
    if (!shard)
      sr_score_kernel<T><<<grid, 256, 0, st>>>(static_cast<const T*>(q), static_cast<const T*>(lm), scores,
                                               p->n_q_heads, p->n_kv_heads, p->head_dim, n_mid, lm_cap,
                                               (n_mid + 3) & ~int64_t(3), cpb);
    if (cudaPeekAtLastError() != cudaSuccess) return XKV_ERR_CUDA;
  }
  prof_mark(1, st);
  // 2. exact top-k (blocks [0, units)) and the raw window partials (blocks [units, 2 units))
  {
    WinArgs wa;
    wa.q = q;
    wa.srK = sr_K;
    wa.srV = sr_V;
    wa.win = win;
    wa.T = p->T;
    wa.wbs = p->window_batch_stride > 0 ? p->window_batch_stride
                                        : static_cast<int64_t>(p->sink + p->recent) * p->n_kv_heads * p->head_dim;
    wa.Hq = p->n_q_heads;
    wa.Hkv = p->n_kv_heads;
    wa.hd = p->head_dim;
    wa.sink = p->sink;
    wa.recent = p->recent;
    wa.pos_off = shard ? shard->pos_off : 0;
    for (int j = 0; j < 128; ++j) wa.ft[j] = j < p->head_dim / 2 ? rope_turns(p->rope_theta, j, p->head_dim) : 0.0;
    const int nsr = p->sink + p->recent;
    const int64_t per = (n_mid + kTopkThreads - 1) / kTopkThreads;
    const size_t smem = std::max(static_cast<size_t>(per * kTopkThreads + n_mid) * 4 + static_cast<size_t>(n_mid) + 16,
                                 window_smem(gq, p->head_dim, nsr));
    // the opt-in covers static + dynamic shared memory above 48 KiB
    cudaFuncSetAttribute(sr_topk_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    const int64_t ld = (n_mid + 3) & ~int64_t(3);
    // with a given selection only the window blocks run (top-k units = 0)
    const int topk_units = shard ? 0 : static_cast<int>(plan.units);
    if (launch_after_prior(sr_topk_kernel<T>, dim3(topk_units + plan.units), dim3(kTopkThreads), smem, st,
                           static_cast<const float*>(scores), ld, sel, sel_out, n_mid, static_cast<int>(p->topk),
                           topk_units, wa) != cudaSuccess)
      return XKV_ERR_CUDA;
  }
  prof_mark(2, st);
  AttendArgs a;
  a.sel = shard ? shard->sel : sel;
  a.pos_off = shard ? shard->pos_off : 0;
  a.c_lo = shard ? shard->c_lo : 0;
  a.c_hi = shard ? shard->c_hi : static_cast<int>(n_mid);
  a.ml_out = shard ? shard->ml_out : nullptr;
  a.q = q;
  a.part = part;
  a.status = device_status_ptr();
  a.T = p->T;
  a.sbk = p->bt_k_batch_stride;
  // Bt_V absent: the xK-SR mode, A_V is the uncompressed V [B][T][d] and rank_v = hd;
  // with v_host, that V is in page-locked host memory and the kept rows are
  // first gathered into the staging buffer
  a.v_raw = v_host ? 2 : (Bt_V == nullptr ? 1 : 0);
  if (v_host) {
    dim3 grid(static_cast<unsigned>(std::max(1, std::min(64, p->topk / 4))), static_cast<unsigned>(plan.units));
    if (launch_after_prior(gather_host_values_kernel<T>, grid, dim3(256), 0, st, static_cast<const T*>(v_host),
                           p->a_v_batch_stride, static_cast<const int32_t*>(sel), static_cast<int>(p->topk),
                           static_cast<int>(p->n_kv_heads), static_cast<int>(p->head_dim),
                           static_cast<int>(p->chunk), static_cast<int>(p->sink), static_cast<T*>(stage)) !=
        cudaSuccess)
      return XKV_ERR_CUDA;
    A_V = stage;
  }
  a.sbv = a.v_raw ? 0 : p->bt_v_batch_stride;
  a.Hq = p->n_q_heads;
  a.Hkv = p->n_kv_heads;
  a.k = p->topk;
  a.sink = p->sink;
  a.recent = p->recent;
  a.rK = p->rank_k;
  a.rV = p->rank_v;
  a.tiles_per_unit = plan.tiles_per_unit;
  a.n_tiles = plan.total_tiles;
  a.ctas = plan.ctas;
  a.max_units = plan.max_units_per_cta;
  a.slot_floats = static_cast<int>(plan.slot_floats);
  a.theta = p->rope_theta;
  for (int j = 0; j < 128; ++j) a.ft[j] = j < p->head_dim / 2 ? rope_turns(p->rope_theta, j, p->head_dim) : 0.0;
  // 3. selective reconstruction + attention partials
  if (plan.tc) {
    CUtensorMap mAK, mBK, mAV;
    const int d = p->n_kv_heads * p->head_dim;
    {
      // (64 columns, token rows, 64-column atoms, batch): one box = 8 rows x kKAtoms atoms
      const uint64_t dims[4] = {64, static_cast<uint64_t>(p->T), static_cast<uint64_t>(p->rank_k / 64),
                                static_cast<uint64_t>(p->batch)};
      const uint64_t str[3] = {static_cast<uint64_t>(p->rank_k) * 2, 128, static_cast<uint64_t>(p->a_k_batch_stride) * 2};
      const uint32_t box[4] = {64, 8, static_cast<uint32_t>(kKAtoms), 1};
      if (!make_tmap(&mAK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, A_K, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
        return XKV_ERR_CUDA;
    }
    {
      const bool batched = p->bt_k_batch_stride != 0;
      const uint64_t dims[3] = {static_cast<uint64_t>(p->rank_k), static_cast<uint64_t>(d),
                                static_cast<uint64_t>(batched ? p->batch : 1)};
      const uint64_t str[2] = {static_cast<uint64_t>(p->rank_k) * 2,
                               static_cast<uint64_t>(batched ? p->bt_k_batch_stride : int64_t(d) * p->rank_k) * 2};
      const uint32_t box[3] = {64, 128, 1};
      if (!make_tmap(&mBK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, Bt_K, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
        return XKV_ERR_CUDA;
    }
    {
      // (64 columns, token rows, atoms, batch): one box = 8 rows x the full rank;
      // uncompressed values: rows of d columns, one box = 8 rows x head h's hd columns;
      // staged values: (64 columns, staged rows k chunk, atoms, units)
      const int vcols = a.v_raw == 1 ? d : p->rank_v;
      const bool staged = a.v_raw == 2;
      const uint64_t dims[4] = {64, static_cast<uint64_t>(staged ? static_cast<int64_t>(p->topk) * 8 : p->T),
                                static_cast<uint64_t>(vcols / 64),
                                static_cast<uint64_t>(staged ? plan.units : p->batch)};
      const uint64_t str[3] = {static_cast<uint64_t>(vcols) * 2, 128,
                               static_cast<uint64_t>(staged ? static_cast<int64_t>(p->topk) * 8 * vcols
                                                            : p->a_v_batch_stride) * 2};
      const uint32_t box[4] = {64, 8, static_cast<uint32_t>(p->rank_v / 64), 1};
      if (!make_tmap(&mAV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, A_V, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
        return XKV_ERR_CUDA;
    }
    const size_t smem = attend_tc_smem();
    void (*kern)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const AttendArgs) = nullptr;
    switch (gq) {
      case 1: kern = sr_attend_tc_kernel<1>; break;
      case 2: kern = sr_attend_tc_kernel<2>; break;
      case 3: kern = sr_attend_tc_kernel<3>; break;
      case 4: kern = sr_attend_tc_kernel<4>; break;
      case 5: kern = sr_attend_tc_kernel<5>; break;
      case 6: kern = sr_attend_tc_kernel<6>; break;
      case 7: kern = sr_attend_tc_kernel<7>; break;
      default: kern = sr_attend_tc_kernel<8>; break;
    }
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (launch_after_prior(kern, dim3(plan.ctas), dim3(kAttendThreads), smem, st, mAK, mBK, mAV, a) != cudaSuccess)
      return XKV_ERR_CUDA;
  } else {
    const size_t smem = simt_smem(gq, p->rank_v, p->head_dim);
    cudaFuncSetAttribute(sr_attend_simt_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem));
    if (launch_after_prior(sr_attend_simt_kernel<T>, dim3(plan.ctas), dim3(256), smem, st, static_cast<const T*>(q),
                           static_cast<const T*>(A_K), static_cast<const T*>(Bt_K), static_cast<const T*>(A_V), a,
                           static_cast<int>(p->head_dim), static_cast<int>(p->chunk), p->a_k_batch_stride,
                           p->a_v_batch_stride) != cudaSuccess)
      return XKV_ERR_CUDA;
  }
  if (cudaPeekAtLastError() != cudaSuccess) return XKV_ERR_CUDA;
  prof_mark(3, st);
  // 4. combine
  {
    const size_t smem = combine_smem(gq, p->rank_v, p->head_dim);
    cudaFuncSetAttribute(sr_combine_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(smem));
    if (launch_after_prior(sr_combine_kernel<T>, dim3(plan.units, kCombineSplit), dim3(kCombineThreads), smem, st,
                           static_cast<const T*>(Bt_V), static_cast<const float*>(win), a,
                           static_cast<int>(p->head_dim), out) != cudaSuccess)
      return XKV_ERR_CUDA;
  }
  prof_mark(4, st);
  return cudaPeekAtLastError() == cudaSuccess ? XKV_OK : XKV_ERR_CUDA;
}

// ------------------------------------------------------- token sharding
xkv_status sr_scores_launch(const xkv_sr_params* p, const void* q, const void* lm, float* scores, int64_t ld,
                            cudaStream_t st) {
  const int64_t n_mid = (p->T - p->sink - p->recent) / p->chunk;
  const int units = p->batch * p->n_kv_heads;
  const int cpb = 512;
  const int64_t lm_cap = p->landmark_capacity > 0 ? p->landmark_capacity : n_mid;
  dim3 grid(static_cast<unsigned>((n_mid + cpb - 1) / cpb), static_cast<unsigned>(units));
  if (p->dtype == XKV_BF16)
    sr_score_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(q),
                                                          static_cast<const __nv_bfloat16*>(lm), scores, p->n_q_heads,
                                                          p->n_kv_heads, p->head_dim, n_mid, lm_cap, ld, cpb);
  else
    sr_score_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(q), static_cast<const float*>(lm), scores,
                                                  p->n_q_heads, p->n_kv_heads, p->head_dim, n_mid, lm_cap, ld, cpb);
  return cudaPeekAtLastError() == cudaSuccess ? XKV_OK : XKV_ERR_CUDA;
}

xkv_status sr_topk_launch(const float* scores, int64_t ld, int units, int64_t n, int k, int32_t* sel,
                          cudaStream_t st) {
  const int64_t per = (n + kTopkThreads - 1) / kTopkThreads;
  const size_t smem = static_cast<size_t>(per * kTopkThreads + n) * 4 + static_cast<size_t>(n) + 16;
  cudaFuncSetAttribute(sr_topk_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  WinArgs wa{};
  sr_topk_kernel<float><<<units, kTopkThreads, smem, st>>>(scores, ld, sel, nullptr, n, k, units, wa);
  return cudaPeekAtLastError() == cudaSuccess ? XKV_OK : XKV_ERR_CUDA;
}

// Merge of per-shard decode partials: row i (sequence, query head) of shard r
// holds the output o_r normalised by its own softmax sum L_r and the running
// maximum M_r (log2 units); the whole-sequence output is
//   sum_r 2^(M_r - M) L_r o_r / sum_r 2^(M_r - M) L_r,  M = max_r M_r,
// shards with L_r = 0 (nothing of theirs kept) contributing nothing.
__global__ void merge_partials_kernel(const float* __restrict__ o, const float* __restrict__ ml, int R, int rows,
                                      int hd, float* __restrict__ out) {
  const int i = blockIdx.x;
  float M = -INFINITY;
  for (int r = 0; r < R; ++r) {
    const float* m = ml + (static_cast<int64_t>(r) * rows + i) * 2;
    if (m[1] > 0.f) M = fmaxf(M, m[0]);
  }
  float den = 0.f;
  for (int r = 0; r < R; ++r) {
    const float* m = ml + (static_cast<int64_t>(r) * rows + i) * 2;
    if (m[1] > 0.f) den += exp2f(m[0] - M) * m[1];
  }
  for (int j = threadIdx.x; j < hd; j += blockDim.x) {
    float num = 0.f;
    for (int r = 0; r < R; ++r) {
      const float* m = ml + (static_cast<int64_t>(r) * rows + i) * 2;
      if (m[1] > 0.f) num = fmaf(exp2f(m[0] - M) * m[1], o[(static_cast<int64_t>(r) * rows + i) * hd + j], num);
    }
    out[static_cast<int64_t>(i) * hd + j] = den > 0.f ? num / den : 0.f;
  }
}

xkv_status merge_partials_launch(const float* o, const float* ml, int R, int rows, int hd, float* out,
                                 cudaStream_t st) {
  merge_partials_kernel<<<rows, 128, 0, st>>>(o, ml, R, rows, hd, out);
  return cudaPeekAtLastError() == cudaSuccess ? XKV_OK : XKV_ERR_CUDA;
}

xkv_status sr_profile_enable(int enable) {
  if (!enable) {
    g_prof.on = false;
    return XKV_OK;
  }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return XKV_ERR_CUDA;
  if (g_prof.device != dev) {
    for (cudaEvent_t& e : g_prof.ev) {
      if (e) cudaEventDestroy(e);
      e = nullptr;
    }
    for (cudaEvent_t& e : g_prof.ev)
      if (cudaEventCreate(&e) != cudaSuccess) return XKV_ERR_CUDA;
    g_prof.device = dev;
  }
  g_prof.recorded = false;
  g_prof.on = true;
  return XKV_OK;
}

xkv_status sr_profile_read(float* stage_ms) {
  if (!stage_ms || !g_prof.recorded) return XKV_ERR_INVALID_ARG;
  if (cudaEventSynchronize(g_prof.ev[4]) != cudaSuccess) return XKV_ERR_CUDA;
  for (int i = 0; i < 4; ++i)
    if (cudaEventElapsedTime(&stage_ms[i], g_prof.ev[i], g_prof.ev[i + 1]) != cudaSuccess) return XKV_ERR_CUDA;
  return XKV_OK;
}

xkv_status sr_launch(const xkv_sr_params* p, const SRPlan& plan, const void* q, const void* A_K, const void* Bt_K,
                     const void* A_V, const void* Bt_V, const void* landmarks, const void* sr_K, const void* sr_V,
                     float* out, int32_t* sel_out, void* ws, cudaStream_t st, const void* v_host, void* stage,
                     const SRShard* shard) {
  if (p->dtype == XKV_BF16)
    return sr_launch_t<__nv_bfloat16>(p, plan, q, A_K, Bt_K, A_V, Bt_V, landmarks, sr_K, sr_V, out, sel_out, ws,
                                      v_host, stage, shard, st);
  return sr_launch_t<float>(p, plan, q, A_K, Bt_K, A_V, Bt_V, landmarks, sr_K, sr_V, out, sel_out, ws, v_host,
                            stage, shard, st);
}

}  // namespace xkv
