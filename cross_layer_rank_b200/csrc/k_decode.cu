// Decode-time Selective Reconstruction (xKV explainer, "仅仅压缩还不够，xKV 还做了
// “选择性重建”"; xKV abstract): landmark scoring, exact top-k chunk selection,
// reconstruction of only the selected rows of K and V from the shared basis A
// and the layer's B_l, RoPE on the rebuilt keys, and online-softmax GQA
// attention (KQ-SVD page, 3.2) over them plus the raw sink/recent window.
//
// Kernels (one decode step of one layer = 4 launches):
//   sr_score   : s_c = (sum_g q_g) . landmark_c            (HBM stream of landmarks)
//   sr_topk    : exact radix select of the k best chunks, ascending output
//   sr_attend  : persistent CTAs over (unit, 128-row tile) ranges.  tcgen05
//                path: TMA gathers the selected 8-row chunk slabs of A_K
//                (8 x 64 bf16 = one 1 KiB swizzle atom each) and the head's
//                Bt_K slice, tcgen05.mma rebuilds the 128 x 128 key tile in
//                TMEM, the epilogue applies RoPE and the q . k products, and
//                256 threads fold p into u_g = sum_t p_gt A_V[t] (the value
//                path is re-associated: o_g = (u_g / l_g) Bt_V^T, exact up to
//                rounding).  A SIMT path covers f32 and other shapes.
//   sr_combine : merges the per-CTA (m, l, u) partials with the sink/recent
//                rows and applies Bt_V.
#include <float.h>

#include <algorithm>

#include "xkv_common.cuh"
#include "xkv_internal.h"

namespace xkv {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kTileChunks = 16;   // chunks of 8 rows per 128-row tile (tcgen05 path)
constexpr int kMaxGQ = 8;
constexpr int kKStages = 4;
constexpr int kVStages = 4;
constexpr int kAtomBytes = 16384;  // 128 rows x 64 bf16
constexpr int kAttendThreads = 448;  // 14 warps: TMA, MMA, 4 epilogue, 8 value

// ----------------------------------------------------------------- helpers
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
                                                       int64_t n_mid, int chunks_per_block) {
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
  const T* base = lm + static_cast<int64_t>(unit) * n_mid * hd;
  float* out = scores + static_cast<int64_t>(unit) * n_mid;
  if (sizeof(T) == 2 && hd == 128) {
    // 16 lanes x 16 B cover one 256-B landmark row; a warp scores 2 rows per load.
    const int half = lane >> 4, hl = lane & 15;
    float qv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) qv[i] = qbar[hl * 8 + i];
    for (int64_t c = c0 + warp * 2 + half; c < c1; c += 16) {
      const uint4 w = *reinterpret_cast<const uint4*>(base + c * 128 + hl * 8);
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = bf2_to_f2(ww[i]);
        s = fmaf(qv[2 * i], f.x, s);
        s = fmaf(qv[2 * i + 1], f.y, s);
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (hl == 0) out[c] = s;
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
// Exact top-k of one unit's chunk scores (1024 threads): radix select of the
// k-th largest key over 4 passes of 8 bits, then an ordered compaction that
// keeps every key above it and the lowest-index ties.
__global__ void __launch_bounds__(1024) sr_topk_kernel(const float* __restrict__ scores, int32_t* __restrict__ sel,
                                                        int32_t* __restrict__ sel_out, int64_t n_mid, int k) {
  extern __shared__ uint32_t keys[];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t warp_tot[32];
  __shared__ uint32_t s_digit, s_kk, s_total;
  const int unit = blockIdx.x;
  const int n = static_cast<int>(n_mid);
  const float* sc = scores + static_cast<int64_t>(unit) * n_mid;
  for (int i = threadIdx.x; i < n; i += blockDim.x) keys[i] = order_key(sc[i]);
  uint32_t prefix = 0, pmask = 0;
  if (threadIdx.x == 0) s_kk = static_cast<uint32_t>(k);
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const uint32_t key = keys[i];
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // lane l owns digits 255-8l .. 248-8l (descending)
      const int lane = threadIdx.x;
      uint32_t loc = 0;
      for (int i = 0; i < 8; ++i) loc += hist[255 - 8 * lane - i];
      uint32_t incl = loc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t kk = s_kk;
      const uint32_t excl = incl - loc;
      const bool mine = excl < kk && incl >= kk;
      const uint32_t ballot = __ballot_sync(0xffffffffu, mine);
      if (mine) {
        uint32_t cum = excl;
        int dsel = 255 - 8 * lane;
        for (int i = 0; i < 8; ++i) {
          const int dgt = 255 - 8 * lane - i;
          if (cum + hist[dgt] >= kk) { dsel = dgt; break; }
          cum += hist[dgt];
        }
        s_digit = static_cast<uint32_t>(dsel);
        s_kk = kk - cum;
      }
      (void)ballot;
    }
    __syncthreads();
    prefix |= s_digit << shift;
    pmask |= 255u << shift;
  }
  const uint32_t tau = prefix;     // key of the k-th largest score
  const uint32_t need_eq = s_kk;   // how many keys equal to tau are kept
  // ordered compaction over contiguous per-thread segments
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int i0 = min(n, static_cast<int>(threadIdx.x) * per), i1 = min(n, i0 + per);
  uint32_t n_eq = 0;
  for (int i = i0; i < i1; ++i) n_eq += (keys[i] == tau);
  uint32_t eq_before = block_exclusive_scan(n_eq, warp_tot, &s_total);
  uint32_t n_sel = 0;
  {
    uint32_t e = eq_before;
    for (int i = i0; i < i1; ++i) {
      const uint32_t key = keys[i];
      if (key > tau) ++n_sel;
      else if (key == tau) { if (e < need_eq) ++n_sel; ++e; }
    }
  }
  uint32_t pos = block_exclusive_scan(n_sel, warp_tot, &s_total);
  {
    uint32_t e = eq_before;
    int32_t* o = sel + static_cast<int64_t>(unit) * k;
    int32_t* o2 = sel_out ? sel_out + static_cast<int64_t>(unit) * k : nullptr;
    for (int i = i0; i < i1; ++i) {
      const uint32_t key = keys[i];
      bool take = false;
      if (key > tau) take = true;
      else if (key == tau) { take = e < need_eq; ++e; }
      if (take) {
        o[pos] = i;
        if (o2) o2[pos] = i;
        ++pos;
      }
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
  int tiles_per_unit, n_tiles, ctas, max_units;
  int slot_floats;
  float theta;
};

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                            int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

template <int GQ>
__global__ void __launch_bounds__(kAttendThreads, 1)
    sr_attend_tc_kernel(const __grid_constant__ CUtensorMap mapAK, const __grid_constant__ CUtensorMap mapBK,
                        const __grid_constant__ CUtensorMap mapAV, const AttendArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int NKA = args.rK / 64, NAV = args.rV / 64;
  const int vstage_bytes = 2 * NAV * 1024;
  uint8_t* Ka = smem;
  uint8_t* Kb = Ka + kKStages * kAtomBytes;
  uint8_t* Vs = Kb + kKStages * kAtomBytes;
  float* p_s = reinterpret_cast<float*>(Vs + kVStages * 16384);  // [2][128][8]
  float* alpha_s = p_s + 2 * 128 * kMaxGQ;                          // [2][8]
  float* q_s = alpha_s + 2 * kMaxGQ;                                // [GQ][128]
  double* ft = reinterpret_cast<double*>(q_s + kMaxGQ * 128);       // [64]
  float* red = reinterpret_cast<float*>(ft + 64);                   // [2][4][8]
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + 64);
  uint64_t* kfull = bars;
  uint64_t* kempty = kfull + kKStages;
  uint64_t* vfull = kempty + kKStages;
  uint64_t* vempty = vfull + kVStages;
  uint64_t* accfull = vempty + kVStages;
  uint64_t* accempty = accfull + 2;
  uint64_t* pfull = accempty + 2;
  uint64_t* pempty = pfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x;
  const int tb = tile_begin(cta, args.n_tiles, args.ctas), te = tile_begin(cta + 1, args.n_tiles, args.ctas);
  const int tpu = args.tiles_per_unit, k = args.k;

  if (tid == 0) {
    for (int i = 0; i < kKStages; ++i) { mbar_init(&kfull[i], 1); mbar_init(&kempty[i], 1); }
    for (int i = 0; i < kVStages; ++i) { mbar_init(&vfull[i], 1); mbar_init(&vempty[i], 256); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accfull[i], 1);
      mbar_init(&accempty[i], 128);
      mbar_init(&pfull[i], 128);
      mbar_init(&pempty[i], 256);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (tid < 64) ft[tid] = rope_turns(static_cast<double>(args.theta), tid, 128);
  if (warp == 1) tmem_alloc(tmem_slot, 256);
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&mapAK);
    prefetch_tmap(&mapBK);
    prefetch_tmap(&mapAV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t ks = 0, vsn = 0;
      for (int x = tb; x < te && !*abort_flag; ++x) {
        const int u = x / tpu, ti = x % tpu;
        const int b = u / args.Hkv, h = u % args.Hkv;
        const int nch = min(kTileChunks, k - ti * kTileChunks);
        const int32_t* su = args.sel + static_cast<int64_t>(u) * k + ti * kTileChunks;
        int rows[kTileChunks];
#pragma unroll
        for (int ch = 0; ch < kTileChunks; ++ch) rows[ch] = ch < nch ? args.sink + su[ch] * 8 : 0;
        for (int a = 0; a < NKA; ++a, ++ks) {
          const int slot = ks % kKStages;
          if (!mbar_wait(&kempty[slot], ((ks / kKStages) & 1) ^ 1, args.status)) { *abort_flag = 1; break; }
          mbar_arrive_expect_tx(&kfull[slot], nch * 1024 + kAtomBytes);
          for (int ch = 0; ch < nch; ++ch)
            tma_load_3d(Ka + slot * kAtomBytes + ch * 1024, &mapAK, &kfull[slot], a * 64, rows[ch], b);
          tma_load_3d(Kb + slot * kAtomBytes, &mapBK, &kfull[slot], a * 64, h * 128, args.sbk ? b : 0);
        }
        for (int v = 0; v < (nch + 1) / 2 && !*abort_flag; ++v, ++vsn) {
          const int slot = vsn % kVStages;
          if (!mbar_wait(&vempty[slot], ((vsn / kVStages) & 1) ^ 1, args.status)) { *abort_flag = 1; break; }
          const int nv = min(2, nch - 2 * v);
          mbar_arrive_expect_tx(&vfull[slot], nv * NAV * 1024);
          for (int c2 = 0; c2 < nv; ++c2)
            for (int a = 0; a < NAV; ++a)
              tma_load_3d(Vs + slot * 16384 + (c2 * NAV + a) * 1024, &mapAV, &vfull[slot], a * 64,
                          rows[2 * v + c2], b);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(128, 128);
      uint32_t ks = 0;
      int j = 0;
      for (int x = tb; x < te && !*abort_flag; ++x, ++j) {
        const int buf = j & 1;
        if (!mbar_wait(&accempty[buf], ((j >> 1) & 1) ^ 1, args.status)) { *abort_flag = 1; break; }
        tc_fence_after();
        const uint32_t dtm = tmem + buf * 128;
        for (int a = 0; a < NKA; ++a, ++ks) {
          const int slot = ks % kKStages;
          if (!mbar_wait(&kfull[slot], (ks / kKStages) & 1, args.status)) { *abort_flag = 1; break; }
          tc_fence_after();
          const uint64_t ad = umma_desc_sw128(smem_u32(Ka + slot * kAtomBytes));
          const uint64_t bd = umma_desc_sw128(smem_u32(Kb + slot * kAtomBytes));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) umma_bf16(dtm, ad + 2 * kk, bd + 2 * kk, idesc, (a | kk) ? 1u : 0u);
          umma_commit(&kempty[slot]);
        }
        umma_commit(&accfull[buf]);
      }
    }
  } else if (warp < 6) {
    // --------------------------------------- key epilogue: RoPE, q.k, softmax
    const int lq = warp & 3;
    const int row = lq * 32 + lane;
    const int et = tid - 64;
    const float qscale = rsqrtf(128.0f) * kLog2e;
    // queries of the unit are (re)loaded when the unit changes
    float m[GQ], l[GQ];
    int cur_u = -1, j = 0;
    for (int x = tb; x < te && !*abort_flag; ++x, ++j) {
      const int u = x / tpu, ti = x % tpu;
      if (u != cur_u) {
        named_bar_sync(1, 128);
        const int b = u / args.Hkv, h = u % args.Hkv;
        for (int i = et; i < GQ * 128; i += 128) {
          const int g = i / 128, jj = i % 128;
          q_s[g * 128 + jj] =
              to_f(reinterpret_cast<const __nv_bfloat16*>(args.q)[(static_cast<int64_t>(b) * args.Hq + h * GQ + g) * 128 + jj]) *
              qscale;
        }
        named_bar_sync(1, 128);
        cur_u = u;
#pragma unroll
        for (int g = 0; g < GQ; ++g) { m[g] = -INFINITY; l[g] = 0.f; }
      }
      const int ch = row >> 3, e = row & 7;
      const bool valid = ti * kTileChunks + ch < k;
      const double pos =
          valid ? static_cast<double>(args.sink + static_cast<int64_t>(args.sel[static_cast<int64_t>(u) * k + ti * kTileChunks + ch]) * 8 + e)
                : 0.0;
      const int buf = j & 1;
      if (!mbar_wait(&accfull[buf], (j >> 1) & 1, args.status)) { *abort_flag = 1; break; }
      tc_fence_after();
      const uint32_t taddr = tmem + (static_cast<uint32_t>(lq * 32) << 16) + buf * 128;
      float s[GQ];
#pragma unroll
      for (int g = 0; g < GQ; ++g) s[g] = 0.f;
#pragma unroll 1
      for (int jb = 0; jb < 4; ++jb) {
        float lo[16], hi[16];
        tmem_ld16(taddr + jb * 16, lo);
        tmem_ld16(taddr + 64 + jb * 16, hi);
        tmem_ld_wait();
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const int jx = jb * 16 + jj;
          float c, sn;
          rope_cs(ft[jx], pos, &c, &sn);
          const float y0 = lo[jj] * c - hi[jj] * sn;
          const float y1 = hi[jj] * c + lo[jj] * sn;
#pragma unroll
          for (int g = 0; g < GQ; ++g) s[g] = fmaf(q_s[g * 128 + jx], y0, fmaf(q_s[g * 128 + 64 + jx], y1, s[g]));
        }
      }
      tc_fence_before();
      mbar_arrive(&accempty[buf]);
      // tile maximum per query head
      float tmax[GQ];
#pragma unroll
      for (int g = 0; g < GQ; ++g) {
        if (!valid) s[g] = -INFINITY;
        const float w = warp_max(s[g]);
        if (lane == 0) red[(lq)*8 + g] = w;
      }
      named_bar_sync(1, 128);
#pragma unroll
      for (int g = 0; g < GQ; ++g)
        tmax[g] = fmaxf(fmaxf(red[0 * 8 + g], red[1 * 8 + g]), fmaxf(red[2 * 8 + g], red[3 * 8 + g]));
      float alpha[GQ], p[GQ];
#pragma unroll
      for (int g = 0; g < GQ; ++g) {
        const float mn = fmaxf(m[g], tmax[g]);
        alpha[g] = exp2f(m[g] - mn);
        p[g] = valid ? exp2f(s[g] - mn) : 0.f;
        m[g] = mn;
        const float w = warp_sum(p[g]);
        if (lane == 0) red[32 + lq * 8 + g] = w;
      }
      named_bar_sync(1, 128);
#pragma unroll
      for (int g = 0; g < GQ; ++g)
        l[g] = l[g] * alpha[g] + (red[32 + g] + red[40 + g] + red[48 + g] + red[56 + g]);
      const int pb = j & 1;
      if (!mbar_wait(&pempty[pb], ((j >> 1) & 1) ^ 1, args.status)) { *abort_flag = 1; break; }
#pragma unroll
      for (int g = 0; g < GQ; ++g) p_s[(pb * 128 + row) * kMaxGQ + g] = p[g];
      if (et == 0)
#pragma unroll
        for (int g = 0; g < GQ; ++g) alpha_s[pb * kMaxGQ + g] = alpha[g];
      mbar_arrive(&pfull[pb]);
      const bool seg_end = (x + 1 == te) || ((x + 1) / tpu != u);
      if (seg_end && et == 0) {
        const int u_first = tb / tpu;
        float* slot = args.part + (static_cast<int64_t>(cta) * args.max_units + (u - u_first)) * args.slot_floats;
#pragma unroll
        for (int g = 0; g < GQ; ++g) { slot[g] = m[g]; slot[8 + g] = l[g]; }
      }
    }
  } else {
    // ------------------------------------- value path: u_g += p_gt A_V[t]
    const int vt = tid - 192;
    const int cp = vt;
    const bool act = cp < args.rV / 2;
    const int atom = cp >> 5, wrd = cp & 31;
    float acc[GQ][2];
    int cur_u = -1, j = 0;
    uint32_t vsn = 0;
    for (int x = tb; x < te && !*abort_flag; ++x, ++j) {
      const int u = x / tpu, ti = x % tpu;
      if (u != cur_u) {
        cur_u = u;
#pragma unroll
        for (int g = 0; g < GQ; ++g) acc[g][0] = acc[g][1] = 0.f;
      }
      const int pb = j & 1;
      if (!mbar_wait(&pfull[pb], (j >> 1) & 1, args.status)) { *abort_flag = 1; break; }
#pragma unroll
      for (int g = 0; g < GQ; ++g) {
        const float a = alpha_s[pb * kMaxGQ + g];
        acc[g][0] *= a;
        acc[g][1] *= a;
      }
      const int nch = min(kTileChunks, k - ti * kTileChunks);
      bool ok = true;
      for (int v = 0; v < (nch + 1) / 2; ++v, ++vsn) {
        const int slot = vsn % kVStages;
        if (!mbar_wait(&vfull[slot], (vsn / kVStages) & 1, args.status)) { *abort_flag = 1; ok = false; break; }
        const int nr = min(2, nch - 2 * v) * 8;
        if (act) {
          const uint8_t* base = Vs + slot * 16384;
          const float* pr = p_s + (pb * 128 + v * 16) * kMaxGQ;
#pragma unroll 4
          for (int r = 0; r < nr; ++r) {
            const int c2 = r >> 3, rr = r & 7;
            const uint32_t w = *reinterpret_cast<const uint32_t*>(base + ((c2 * NAV + atom) * 8 + rr) * 128 + wrd * 4);
            const float2 a = bf2_to_f2(w);
#pragma unroll
            for (int g = 0; g < GQ; ++g) {
              const float pg = pr[r * kMaxGQ + g];
              acc[g][0] = fmaf(pg, a.x, acc[g][0]);
              acc[g][1] = fmaf(pg, a.y, acc[g][1]);
            }
          }
        }
        fence_proxy_async();
        mbar_arrive(&vempty[slot]);
      }
      if (!ok) break;
      mbar_arrive(&pempty[pb]);
      const bool seg_end = (x + 1 == te) || ((x + 1) / tpu != u);
      if (seg_end && act) {
        const int u_first = tb / tpu;
        float* slot = args.part + (static_cast<int64_t>(cta) * args.max_units + (u - u_first)) * args.slot_floats;
#pragma unroll
        for (int g = 0; g < GQ; ++g) {
          slot[16 + g * args.rV + 2 * cp] = acc[g][0];
          slot[16 + g * args.rV + 2 * cp + 1] = acc[g][1];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

size_t attend_tc_smem() {
  return 1024 + 2 * kKStages * kAtomBytes + kVStages * 16384 + (2 * 128 * kMaxGQ + 2 * kMaxGQ + kMaxGQ * 128) * 4 +
         64 * 8 + 64 * 4 + (2 * kKStages + 2 * kVStages + 8) * 8 + 16;
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
  for (int j = tid; j < half; j += blockDim.x) ft[j] = rope_turns(static_cast<double>(args.theta), j, hd);
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
        const int64_t t = args.sink + static_cast<int64_t>(args.sel[static_cast<int64_t>(u) * k + ti * kTileChunks + rr / chunk]) * chunk + rr % chunk;
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
        rope_cs(ft[jj], static_cast<double>(t), &cs, &sn);
        Ks[r * hd + jj] = y0 * cs - y1 * sn;
        Ks[r * hd + jj + half] = y1 * cs + y0 * sn;
      }
      __syncthreads();
      for (int i = tid; i < nr * gq; i += blockDim.x) {
        const int r = i / gq, g = i % gq;
        float s = 0.f;
        for (int jj = 0; jj < hd; ++jj) s = fmaf(qs[g * hd + jj], Ks[r * hd + jj], s);
        ps[r * gq + g] = s;
      }
      __syncthreads();
      if (tid < gq) {
        const int g = tid;
        float mx = ms[g];
        for (int r = 0; r < nr; ++r) mx = fmaxf(mx, ps[r * gq + g]);
        al[g] = exp2f(ms[g] - mx);
        float sum = 0.f;
        for (int r = 0; r < nr; ++r) {
          const float pv = exp2f(ps[r * gq + g] - mx);
          ps[r * gq + g] = pv;
          sum += pv;
        }
        ls[g] = ls[g] * al[g] + sum;
        ms[g] = mx;
      }
      __syncthreads();
      for (int i = tid; i < gq * args.rV; i += blockDim.x) {
        const int g = i / args.rV, c = i % args.rV;
        float acc = us[i] * al[g];
        for (int r = 0; r < nr; ++r) {
          const int rr = rb + r;
          const int64_t t = args.sink + static_cast<int64_t>(args.sel[static_cast<int64_t>(u) * k + ti * kTileChunks + rr / chunk]) * chunk + rr % chunk;
          acc = fmaf(ps[r * gq + g], to_f(AV[b * sav + t * args.rV + c]), acc);
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
  (void)d;
}

// ----------------------------------------------------------- sr_combine
// One block per unit: merge the partials of every CTA that covered the unit,
// add the raw sink/recent rows, and map the value-basis sums through Bt_V:
//   o_g = (sum_c U_g[c] Bt_V[h hd + j][c] + sum_t p_gt V_t[j]) / L_g.
template <typename T>
__global__ void __launch_bounds__(256) sr_combine_kernel(const T* __restrict__ q, const T* __restrict__ BtV,
                                                         const T* __restrict__ srK, const T* __restrict__ srV,
                                                         const AttendArgs args, int hd, float* __restrict__ out) {
  extern __shared__ double smd[];
  const int gq = args.Hq / args.Hkv;
  const int nsr = args.sink + args.recent;
  const int u = blockIdx.x, b = u / args.Hkv, h = u % args.Hkv;
  const int tid = threadIdx.x;
  const int tpu = args.tiles_per_unit;
  const int d = args.Hkv * hd, half = hd / 2;
  double* ft = smd;                        // [half]
  float* Us = reinterpret_cast<float*>(smd + half);  // [gq][rV]
  float* Ws = Us + gq * args.rV;           // [gq][hd]
  float* qs = Ws + gq * hd;                // [gq][hd]
  float* srs = qs + gq * hd;               // [nsr][gq] scores, then weights
  float* Mg = srs + nsr * gq;              // [gq]
  float* Lg = Mg + kMaxGQ;                 // [gq]
  float* sc = Lg + kMaxGQ;                 // [slots][gq] partial rescale factors (slots <= 64)
  const int fc = cta_of_tile(u * tpu, args.n_tiles, args.ctas);
  const int lc = cta_of_tile((u + 1) * tpu - 1, args.n_tiles, args.ctas);
  const int nslots = lc - fc + 1;
  const float qscale = rsqrtf(static_cast<float>(hd)) * kLog2e;
  for (int i = tid; i < gq * hd; i += blockDim.x)
    qs[i] = to_f(q[(static_cast<int64_t>(b) * args.Hq + h * gq) * hd + i]) * qscale;
  for (int j = tid; j < half; j += blockDim.x) ft[j] = rope_turns(static_cast<double>(args.theta), j, hd);
  __syncthreads();
  // scores of the raw window rows (row i < sink is token i, else T - recent + i - sink)
  for (int i = tid; i < nsr * gq; i += blockDim.x) {
    const int r = i / gq, g = i % gq;
    const int64_t t = r < args.sink ? r : args.T - args.recent + (r - args.sink);
    const T* kr = srK + (static_cast<int64_t>(b) * nsr + r) * d + h * hd;
    float s = 0.f;
    for (int jj = 0; jj < half; ++jj) {
      float cs, sn;
      rope_cs(ft[jj], static_cast<double>(t), &cs, &sn);
      const float x0 = to_f(kr[jj]), x1 = to_f(kr[jj + half]);
      s = fmaf(qs[g * hd + jj], x0 * cs - x1 * sn, s);
      s = fmaf(qs[g * hd + jj + half], x1 * cs + x0 * sn, s);
    }
    srs[r * gq + g] = s;
  }
  __syncthreads();
  if (tid < gq) {
    const int g = tid;
    const int u_first0 = 0;
    (void)u_first0;
    float M = -INFINITY;
    for (int c = fc; c <= lc; ++c) {
      const int uf = tile_begin(c, args.n_tiles, args.ctas) / tpu;
      const float* slot = args.part + (static_cast<int64_t>(c) * args.max_units + (u - uf)) * args.slot_floats;
      M = fmaxf(M, slot[g]);
    }
    for (int r = 0; r < nsr; ++r) M = fmaxf(M, srs[r * gq + g]);
    float L = 0.f;
    for (int c = fc; c <= lc; ++c) {
      const int uf = tile_begin(c, args.n_tiles, args.ctas) / tpu;
      const float* slot = args.part + (static_cast<int64_t>(c) * args.max_units + (u - uf)) * args.slot_floats;
      const float f = exp2f(slot[g] - M);
      sc[(c - fc) * kMaxGQ + g] = f;
      L += slot[8 + g] * f;
    }
    for (int r = 0; r < nsr; ++r) {
      const float w = exp2f(srs[r * gq + g] - M);
      srs[r * gq + g] = w;
      L += w;
    }
    Mg[g] = M;
    Lg[g] = L;
  }
  __syncthreads();
  for (int i = tid; i < gq * args.rV; i += blockDim.x) {
    const int g = i / args.rV, c = i % args.rV;
    float acc = 0.f;
    for (int cc = fc; cc <= lc; ++cc) {
      const int uf = tile_begin(cc, args.n_tiles, args.ctas) / tpu;
      const float* slot = args.part + (static_cast<int64_t>(cc) * args.max_units + (u - uf)) * args.slot_floats;
      acc = fmaf(slot[16 + g * args.rV + c], sc[(cc - fc) * kMaxGQ + g], acc);
    }
    Us[i] = acc;
  }
  for (int i = tid; i < gq * hd; i += blockDim.x) {
    const int g = i / hd, j = i % hd;
    float acc = 0.f;
    for (int r = 0; r < nsr; ++r)
      acc = fmaf(srs[r * gq + g], to_f(srV[(static_cast<int64_t>(b) * nsr + r) * d + h * hd + j]), acc);
    Ws[i] = acc;
  }
  __syncthreads();
  for (int j = tid; j < hd; j += blockDim.x) {
    const T* br = BtV + b * args.sbv + static_cast<int64_t>(h * hd + j) * args.rV;
    float acc[kMaxGQ];
#pragma unroll
    for (int g = 0; g < kMaxGQ; ++g) acc[g] = 0.f;
    for (int c = 0; c < args.rV; ++c) {
      const float bv = to_f(br[c]);
#pragma unroll
      for (int g = 0; g < kMaxGQ; ++g)
        if (g < gq) acc[g] = fmaf(Us[g * args.rV + c], bv, acc[g]);
    }
#pragma unroll
    for (int g = 0; g < kMaxGQ; ++g)
      if (g < gq)
        out[(static_cast<int64_t>(b) * args.Hq + h * gq + g) * hd + j] = (acc[g] + Ws[g * hd + j]) / Lg[g];
  }
  (void)nslots;
}

size_t combine_smem(int gq, int rV, int hd, int nsr) {
  return (static_cast<size_t>(gq) * rV + 2 * gq * hd + nsr * gq + 2 * kMaxGQ + 64 * kMaxGQ + 8) * 4 +
         (hd / 2) * 8 + 16;
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
  plan->slot_floats = 16 + static_cast<size_t>(std::max(gq, 1)) * p->rank_v;
  size_t off = 0;
  plan->off_scores = off;
  off = align_up(off + static_cast<size_t>(plan->units) * n_mid * 4);
  plan->off_sel = off;
  off = align_up(off + static_cast<size_t>(plan->units) * p->topk * 4);
  plan->off_part = off;
  off = align_up(off + static_cast<size_t>(plan->ctas) * mx * plan->slot_floats * 4);
  plan->bytes = off;
  return XKV_OK;
}

template <typename T>
static xkv_status sr_launch_t(const xkv_sr_params* p, const SRPlan& plan, const void* q, const void* A_K,
                              const void* Bt_K, const void* A_V, const void* Bt_V, const void* lm,
                              const void* sr_K, const void* sr_V, float* out, int32_t* sel_out, void* ws,
                              cudaStream_t st) {
  const int64_t n_mid = (p->T - p->sink - p->recent) / p->chunk;
  const int gq = p->n_q_heads / p->n_kv_heads;
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* scores = reinterpret_cast<float*>(w + plan.off_scores);
  int32_t* sel = reinterpret_cast<int32_t*>(w + plan.off_sel);
  float* part = reinterpret_cast<float*>(w + plan.off_part);
  // 1. chunk scores
  {
    const int cpb = 512;
    dim3 grid(static_cast<unsigned>((n_mid + cpb - 1) / cpb), static_cast<unsigned>(plan.units));
    sr_score_kernel<T><<<grid, 256, 0, st>>>(static_cast<const T*>(q), static_cast<const T*>(lm), scores,
                                             p->n_q_heads, p->n_kv_heads, p->head_dim, n_mid, cpb);
  }
  // 2. exact top-k
  {
    const size_t smem = static_cast<size_t>(n_mid) * 4;
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(sr_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    sr_topk_kernel<<<plan.units, 1024, smem, st>>>(scores, sel, sel_out, n_mid, p->topk);
  }
  AttendArgs a;
  a.sel = sel;
  a.q = q;
  a.part = part;
  a.status = device_status_ptr();
  a.T = p->T;
  a.sbk = p->bt_k_batch_stride;
  a.sbv = p->bt_v_batch_stride;
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
  // 3. selective reconstruction + attention partials
  if (plan.tc) {
    CUtensorMap mAK, mBK, mAV;
    const int d = p->n_kv_heads * p->head_dim;
    {
      const uint64_t dims[3] = {static_cast<uint64_t>(p->rank_k), static_cast<uint64_t>(p->T),
                                static_cast<uint64_t>(p->batch)};
      const uint64_t str[2] = {static_cast<uint64_t>(p->rank_k) * 2, static_cast<uint64_t>(p->a_k_batch_stride) * 2};
      const uint32_t box[3] = {64, 8, 1};
      if (!make_tmap(&mAK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, A_K, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
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
      const uint64_t dims[3] = {static_cast<uint64_t>(p->rank_v), static_cast<uint64_t>(p->T),
                                static_cast<uint64_t>(p->batch)};
      const uint64_t str[2] = {static_cast<uint64_t>(p->rank_v) * 2, static_cast<uint64_t>(p->a_v_batch_stride) * 2};
      const uint32_t box[3] = {64, 8, 1};
      if (!make_tmap(&mAV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, A_V, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
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
    kern<<<plan.ctas, kAttendThreads, smem, st>>>(mAK, mBK, mAV, a);
  } else {
    const size_t smem = simt_smem(gq, p->rank_v, p->head_dim);
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(sr_attend_simt_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
    sr_attend_simt_kernel<T><<<plan.ctas, 256, smem, st>>>(
        static_cast<const T*>(q), static_cast<const T*>(A_K), static_cast<const T*>(Bt_K),
        static_cast<const T*>(A_V), a, p->head_dim, p->chunk, p->a_k_batch_stride, p->a_v_batch_stride);
  }
  // 4. combine
  {
    const size_t smem = combine_smem(gq, p->rank_v, p->head_dim, p->sink + p->recent);
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(sr_combine_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
    sr_combine_kernel<T><<<plan.units, 256, smem, st>>>(static_cast<const T*>(q), static_cast<const T*>(Bt_V),
                                                         static_cast<const T*>(sr_K), static_cast<const T*>(sr_V),
                                                         a, p->head_dim, out);
  }
  return cudaPeekAtLastError() == cudaSuccess ? XKV_OK : XKV_ERR_CUDA;
}

xkv_status sr_launch(const xkv_sr_params* p, const SRPlan& plan, const void* q, const void* A_K, const void* Bt_K,
                     const void* A_V, const void* Bt_V, const void* landmarks, const void* sr_K, const void* sr_V,
                     float* out, int32_t* sel_out, void* ws, cudaStream_t st) {
  if (p->dtype == XKV_BF16)
    return sr_launch_t<__nv_bfloat16>(p, plan, q, A_K, Bt_K, A_V, Bt_V, landmarks, sr_K, sr_V, out, sel_out, ws, st);
  return sr_launch_t<float>(p, plan, q, A_K, Bt_K, A_V, Bt_V, landmarks, sr_K, sr_V, out, sel_out, ws, st);
}

}  // namespace xkv
