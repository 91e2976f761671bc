// Prefill-time cross-layer factorisation of one group of G layers (xKV
// explainer, "xKV 到底做了什么"; xKV abstract) with the incremental covariance
// of KV-CoRE (2.A):
//   1. C = sum over token shards of X_s^T X_s, X = [X_1 | ... | X_G] read through
//      the G layer pointers (never concatenated).  bf16: each shard is
//      transposed to a K-major copy and multiplied on tcgen05 tensor cores:
//      upper-triangular 128 x 256 tiles when G d is a multiple of 256 (else
//      128 x 128), 256-row chunks accumulated in TMEM and summed in fp32
//      registers, and a mirrored fp32 epilogue.
//   2. top-r subspace: block subspace iteration Y = C Q, Q = qr(Y) (shifted
//      Cholesky QR, fp64 small factors with a blocked Cholesky; one pass per
//      iteration, two for the basis that enters Rayleigh-Ritz),
//      started from a Gaussian block (Philox4x32-10 + Box-Muller on the
//      device); Rayleigh-Ritz: H = Q^T C Q, eigenpairs of H by one-sided block
//      Jacobi, V_r = Q U[:, top r].
//   3. A = X V_r: tcgen05 GEMM over the layer tensor maps with V_r split into a
//      bf16 hi/lo pair (two MMAs per step keep ~16 significant bits of V_r);
//      Bt = V_r stored in the cache dtype (layer l owns rows l d .. l d + d - 1).
#include <algorithm>

#include "k_gemm_tc.cuh"
#include "xkv_common.cuh"
#include "xkv_internal.h"
#include "xkv_linalg.cuh"

namespace xkv {
namespace {

// X_s (rows x d per layer, row stride ldx) -> Xt (n x ldt), Xt[l d + c][t] = X_l[t][c].
struct LayerPtrs {
  const void* p[8];
};

// One 64 (rows t) x 64 (columns c) tile per CTA, moved in 16-byte vectors
// both ways: row t's 8-column vectors land in shared memory at granule
// (c / 8) ^ (t / 8 mod 8), so that the column reads of the store phase (8
// values of t for one c) fall in different banks; each warp then writes 128
// contiguous bytes of 4 rows of Xt.  Requires 16-byte aligned layers, ldx and
// ldt multiples of 8.
__global__ void __launch_bounds__(256) transpose_layers_kernel(const LayerPtrs X, int d, int64_t ldx, int64_t rows,
                                                               __nv_bfloat16* __restrict__ Xt, int64_t ldt) {
  __shared__ uint4 tile[64][8];
  const int l = blockIdx.z;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * 64;
  const int c0 = blockIdx.y * 64;
  const int tid = threadIdx.x;
  const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(X.p[l]);
  for (int v = tid; v < 512; v += 256) {
    const int r = v >> 3, cv = v & 7;
    const int64_t t = t0 + r;
    const uint4 val = t < rows ? *reinterpret_cast<const uint4*>(src + t * ldx + c0 + 8 * cv) : make_uint4(0, 0, 0, 0);
    tile[r][cv ^ ((r >> 3) & 7)] = val;
  }
  __syncthreads();
  const uint16_t* th = reinterpret_cast<const uint16_t*>(&tile[0][0]);
  for (int v = tid; v < 512; v += 256) {
    const int c = v >> 3, tv = v & 7;  // column c, rows 8 tv .. 8 tv + 7
    const int g = (c >> 3) ^ tv;       // (8 tv + e) / 8 = tv
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      const uint32_t lo = th[(8 * tv + e) * 64 + g * 8 + (c & 7)];
      const uint32_t hi = th[(8 * tv + e + 1) * 64 + g * 8 + (c & 7)];
      w[e / 2] = lo | (hi << 16);
    }
    const int64_t t = t0 + 8 * tv;
    if (t < ldt)
      *reinterpret_cast<uint4*>(Xt + static_cast<int64_t>(l * d + c0 + c) * ldt + t) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// Philox4x32-10 (Salmon et al., SC'11) keyed by the seed; Box-Muller pairs.
__device__ __forceinline__ void philox10(uint32_t c[4], uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c[0];
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c[2];
    const uint32_t n0 = static_cast<uint32_t>(p1 >> 32) ^ c[1] ^ k0;
    const uint32_t n2 = static_cast<uint32_t>(p0 >> 32) ^ c[3] ^ k1;
    c[1] = static_cast<uint32_t>(p1);
    c[3] = static_cast<uint32_t>(p0);
    c[0] = n0;
    c[2] = n2;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
}

__global__ void gaussian_kernel(float* __restrict__ out, int64_t count, uint64_t seed) {
  for (int64_t blk = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; blk * 4 < count;
       blk += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    uint32_t c[4] = {static_cast<uint32_t>(blk), static_cast<uint32_t>(blk >> 32), 0u, 0u};
    philox10(c, static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float u1 = (static_cast<float>(c[2 * h] >> 8) + 0.5f) * (1.0f / 16777216.0f);
      const float u2 = (static_cast<float>(c[2 * h + 1] >> 8) + 0.5f) * (1.0f / 16777216.0f);
      const float rad = sqrtf(-2.0f * logf(u1));
      float s, co;
      sincospif(2.0f * u2, &s, &co);
      const int64_t e = blk * 4 + 2 * h;
      if (e < count) out[e] = rad * co;
      if (e + 1 < count) out[e + 1] = rad * s;
    }
  }
}

// Ur[k][i] = U[order[i]][k]  (U column-major b x b: column c at U + c b)
__global__ void gather_ritz_kernel(const double* __restrict__ U, const int* __restrict__ order, int b, int r,
                                   float* __restrict__ Ur, const double* __restrict__ lam, float* __restrict__ eig) {
  const int64_t total = static_cast<int64_t>(b) * r;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int k = static_cast<int>(i / r), c = static_cast<int>(i % r);
    Ur[i] = static_cast<float>(U[static_cast<int64_t>(order[c]) * b + k]);
  }
  if (eig && blockIdx.x == 0)
    for (int c = threadIdx.x; c < r; c += blockDim.x) eig[c] = static_cast<float>(lam[order[c]]);
}

// Bt (n x r, dtype) = Vr; Vt hi/lo (r x n bf16) = transposed split of Vr.
template <typename T>
__global__ void emit_factors_kernel(const float* __restrict__ Vr, int n, int r, T* __restrict__ Bt,
                                    __nv_bfloat16* __restrict__ vhi, __nv_bfloat16* __restrict__ vlo) {
  const int64_t total = static_cast<int64_t>(n) * r;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float v = Vr[i];
    store_f(Bt + i, v);
    if (vhi) {
      const int k = static_cast<int>(i / r), c = static_cast<int>(i % r);
      const __nv_bfloat16 h = __float2bfloat16_rn(v);
      vhi[static_cast<int64_t>(c) * n + k] = h;
      vlo[static_cast<int64_t>(c) * n + k] = __float2bfloat16_rn(v - __bfloat162float(h));
    }
  }
}

// Gram tile C[tm-block][tn-block] += X_s^T X_s (upper-triangular tile list),
// operands from the K-major transposed shard Xt.  The tensor cores accumulate
// only kGramChunk rows into a TMEM buffer (two buffers, double-buffered); the
// epilogue warps add each chunk's tile into fp32 registers with IEEE adds.
// Keeping the in-MMA accumulation chain short (16 MMAs of 16 rows) removes the
// drift a long chain of tensor-core accumulations shows over thousands of
// rows; the outer sum is an ordinary round-to-nearest fp32 chain.
constexpr int kGramChunkStages = 4;  // 4 x 64 rows per TMEM chunk
constexpr int kGramStages = 4;
constexpr int kGramThreads = 320;  // producer, MMA issuer, 8 epilogue warps (2 per TMEM lane quarter)

inline size_t gram_tc_smem() { return 1024 + kGramStages * 2 * 16384 + (2 * kGramStages + 4) * 8 + 16; }

__global__ void __launch_bounds__(kGramThreads, 1)
    gram_tc_kernel(const __grid_constant__ CUtensorMap xmap, int nk, int tiles_n, float* __restrict__ C, int64_t ldc,
                   int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGramStages * 2 * 16384);
  uint64_t* empty = full + kGramStages;
  uint64_t* accfull = empty + kGramStages;
  uint64_t* accempty = accfull + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(accempty + 2);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int idx = blockIdx.x, tm = 0, len = tiles_n;
  while (idx >= len) { idx -= len; ++tm; --len; }
  const int tn = tm + idx;
  const int m0 = tm * 128, n0 = tn * 128;
  const int nchunks = (nk + kGramChunkStages - 1) / kGramChunkStages;
  if (tid == 0) {
    for (int i = 0; i < kGramStages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&accfull[i], 1); mbar_init(&accempty[i], 256); }
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tslot, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  if (warp == 0) {
    if (lane == 0) {
      for (int a = 0; a < nk; ++a) {
        const int slot = a % kGramStages;
        if (!mbar_wait(&empty[slot], ((a / kGramStages) & 1) ^ 1, status)) break;
        uint8_t* st = smem + slot * 2 * 16384;
        mbar_arrive_expect_tx(&full[slot], 2 * 16384);
        tma_load_2d(st, &xmap, &full[slot], a * 64, m0);
        tma_load_2d(st + 16384, &xmap, &full[slot], a * 64, n0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(128, 128);
      int a = 0;
      bool ok = true;
      for (int c = 0; c < nchunks && ok; ++c) {
        const int buf = c & 1;
        if (!mbar_wait(&accempty[buf], ((c >> 1) & 1) ^ 1, status)) break;
        tc_fence_after();
        for (int s = 0; s < kGramChunkStages && a < nk; ++s, ++a) {
          const int slot = a % kGramStages;
          if (!mbar_wait(&full[slot], (a / kGramStages) & 1, status)) { ok = false; break; }
          tc_fence_after();
          uint8_t* st = smem + slot * 2 * 16384;
          const uint64_t ad = umma_desc_sw128(smem_u32(st));
          const uint64_t bd = umma_desc_sw128(smem_u32(st + 16384));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tmem + buf * 128, ad + 2 * kk, bd + 2 * kk, idesc, (s | kk) ? 1u : 0u);
          umma_commit(&empty[slot]);
        }
        umma_commit(&accfull[buf]);
      }
    }
  } else {
    // warp w reads TMEM lane quarter w % 4; warps 2-5 own columns 0-63 of the
    // tile, warps 6-9 columns 64-127
    const int lq = warp & 3, half = (warp - 2) >> 2;
    const int row = lq * 32 + lane;
    const uint32_t tbase = tmem + (static_cast<uint32_t>(lq * 32) << 16) + half * 64;
    float acc[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) acc[i] = 0.f;
    bool ok = true;
    for (int c = 0; c < nchunks; ++c) {
      const int buf = c & 1;
      if (!mbar_wait(&accfull[buf], (c >> 1) & 1, status)) { ok = false; break; }
      __syncwarp();  // converged for the warp-wide tcgen05.ld
      tc_fence_after();
      float v[64];
#pragma unroll
      for (int jb = 0; jb < 4; ++jb) tmem_ld16(tbase + buf * 128 + jb * 16, v + jb * 16);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&accempty[buf]);
#pragma unroll
      for (int i = 0; i < 64; ++i) acc[i] += v[i];
    }
    if (ok) {
      // read-modify-write of C in batches whose loads are all issued before
      // any of their stores (C is read and written through one pointer, so a
      // plain += loop would wait for every load in turn)
      const int m = m0 + row;
      const int nb = n0 + half * 64;
      float* crow = C + static_cast<int64_t>(m) * ldc + nb;
#pragma unroll
      for (int i0 = 0; i0 < 64; i0 += 32) {
        float4 cv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) cv[u] = *reinterpret_cast<const float4*>(crow + i0 + 4 * u);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = i0 + 4 * u;
          cv[u].x += acc[i];
          cv[u].y += acc[i + 1];
          cv[u].z += acc[i + 2];
          cv[u].w += acc[i + 3];
          *reinterpret_cast<float4*>(crow + i) = cv[u];
        }
      }
      if (tm != tn) {
        // the mirrored tile: lanes hold consecutive m, so each access is one
        // 128-byte row segment per warp
#pragma unroll
        for (int i0 = 0; i0 < 64; i0 += 16) {
          float w[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) w[u] = C[static_cast<int64_t>(nb + i0 + u) * ldc + m];
#pragma unroll
          for (int u = 0; u < 16; ++u) C[static_cast<int64_t>(nb + i0 + u) * ldc + m] = w[u] + acc[i0 + u];
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
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}


// Wide variant for n % 256 == 0: tiles of 128 rows x 256 columns (row block tm,
// column block tn >= tm / 2, so every upper-triangular entry belongs to exactly
// one tile), fp32 accumulators of 256 TMEM columns, double-buffered (all 512
// columns).  Per 64-row step the MMA reads 12 KB of operands for twice the
// work of a 128 x 128 tile, which leaves shared-memory bandwidth for the TMA
// writes.  Entries left of the diagonal in a straddling tile are skipped; the
// others are added to C and (off the diagonal) mirrored.
constexpr int kGramWStages = 4;
constexpr int kGramWStage = 16384 + 32768;  // A: 128 x 64, B: 256 x 64 bf16
constexpr int kGramWThreads = 576;          // producer, MMA issuer, 16 epilogue warps

inline size_t gram_tc256_smem() { return 1024 + kGramWStages * kGramWStage + (2 * kGramWStages + 4) * 8 + 16; }

__global__ void __launch_bounds__(kGramWThreads, 1)
    gram_tc256_kernel(const __grid_constant__ CUtensorMap xmap, int nk, int tiles_m, int tiles_w, float* __restrict__ C,
                      int64_t ldc, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGramWStages * kGramWStage);
  uint64_t* empty = full + kGramWStages;
  uint64_t* accfull = empty + kGramWStages;
  uint64_t* accempty = accfull + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(accempty + 2);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // tile list: row block tm holds column blocks tn = tm / 2 .. tiles_w - 1
  int idx = blockIdx.x, tm = 0;
  while (tm < tiles_m && idx >= tiles_w - tm / 2) { idx -= tiles_w - tm / 2; ++tm; }
  const int tn = tm / 2 + idx;
  const int m0 = tm * 128, n0 = tn * 256;
  const int nchunks = (nk + kGramChunkStages - 1) / kGramChunkStages;
  if (tid == 0) {
    for (int i = 0; i < kGramWStages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&accfull[i], 1); mbar_init(&accempty[i], 512); }
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  if (warp == 0) {
    if (lane == 0) {
      for (int a = 0; a < nk; ++a) {
        const int slot = a % kGramWStages;
        if (!mbar_wait(&empty[slot], ((a / kGramWStages) & 1) ^ 1, status)) break;
        uint8_t* st = smem + slot * kGramWStage;
        mbar_arrive_expect_tx(&full[slot], kGramWStage);
        tma_load_2d(st, &xmap, &full[slot], a * 64, m0);
        tma_load_2d(st + 16384, &xmap, &full[slot], a * 64, n0);
        tma_load_2d(st + 32768, &xmap, &full[slot], a * 64, n0 + 128);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(128, 256);
      int a = 0;
      bool ok = true;
      for (int c = 0; c < nchunks && ok; ++c) {
        const int buf = c & 1;
        if (!mbar_wait(&accempty[buf], ((c >> 1) & 1) ^ 1, status)) break;
        tc_fence_after();
        for (int s = 0; s < kGramChunkStages && a < nk; ++s, ++a) {
          const int slot = a % kGramWStages;
          if (!mbar_wait(&full[slot], (a / kGramWStages) & 1, status)) { ok = false; break; }
          tc_fence_after();
          uint8_t* st = smem + slot * kGramWStage;
          const uint64_t ad = umma_desc_sw128(smem_u32(st));
          const uint64_t bd = umma_desc_sw128(smem_u32(st + 16384));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tmem + buf * 256, ad + 2 * kk, bd + 2 * kk, idesc, (s | kk) ? 1u : 0u);
          umma_commit(&empty[slot]);
        }
        umma_commit(&accfull[buf]);
      }
    }
  } else {
    // warp w reads TMEM lane quarter w % 4; warps 2-5, 6-9, 10-13, 14-17 own
    // columns 0-63, 64-127, 128-191, 192-255 of the tile
    const int lq = warp & 3, quarter = (warp - 2) >> 2;
    const int row = lq * 32 + lane;
    const uint32_t tbase = tmem + (static_cast<uint32_t>(lq * 32) << 16) + quarter * 64;
    float acc[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) acc[i] = 0.f;
    bool ok = true;
    for (int c = 0; c < nchunks; ++c) {
      const int buf = c & 1;
      if (!mbar_wait(&accfull[buf], (c >> 1) & 1, status)) { ok = false; break; }
      __syncwarp();  // converged for the warp-wide tcgen05.ld
      tc_fence_after();
#pragma unroll
      for (int jb = 0; jb < 4; ++jb) {
        float v[16];
        tmem_ld16(tbase + buf * 256 + jb * 16, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[jb * 16 + i] += v[i];
      }
      tc_fence_before();
      mbar_arrive(&accempty[buf]);
    }
    if (ok) {
      const int m = m0 + row;
      const int nb = n0 + quarter * 64;
      if (nb > m) {
        // whole column block right of the diagonal: batched read-modify-write
        // (loads of a batch before its stores, C read and written through one
        // pointer), then the mirrored entries
        float* crow = C + static_cast<int64_t>(m) * ldc + nb;
#pragma unroll
        for (int i0 = 0; i0 < 64; i0 += 16) {
          float4 cv[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) cv[u] = *reinterpret_cast<const float4*>(crow + i0 + 4 * u);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = i0 + 4 * u;
            cv[u].x += acc[i];
            cv[u].y += acc[i + 1];
            cv[u].z += acc[i + 2];
            cv[u].w += acc[i + 3];
            *reinterpret_cast<float4*>(crow + i) = cv[u];
          }
        }
#pragma unroll
        for (int i0 = 0; i0 < 64; i0 += 8) {
          float w[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) w[u] = C[static_cast<int64_t>(nb + i0 + u) * ldc + m];
#pragma unroll
          for (int u = 0; u < 8; ++u) C[static_cast<int64_t>(nb + i0 + u) * ldc + m] = w[u] + acc[i0 + u];
        }
      } else if (nb + 63 >= m) {
        // the block meets the diagonal: entries j >= m, mirrored when j > m
        // (predicated batches, loads before stores)
        float* crow = C + static_cast<int64_t>(m) * ldc + nb;
#pragma unroll
        for (int i0 = 0; i0 < 64; i0 += 8) {
          float w[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) w[u] = nb + i0 + u >= m ? crow[i0 + u] : 0.f;
#pragma unroll
          for (int u = 0; u < 8; ++u)
            if (nb + i0 + u >= m) crow[i0 + u] = w[u] + acc[i0 + u];
        }
#pragma unroll
        for (int i0 = 0; i0 < 64; i0 += 8) {
          float w[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) w[u] = nb + i0 + u > m ? C[static_cast<int64_t>(nb + i0 + u) * ldc + m] : 0.f;
#pragma unroll
          for (int u = 0; u < 8; ++u)
            if (nb + i0 + u > m) C[static_cast<int64_t>(nb + i0 + u) * ldc + m] = w[u] + acc[i0 + u];
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
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

bool gram_tc_ok(int G, int d, xkv_dtype dt) { return dt == XKV_BF16 && (G * d) % 128 == 0 && !force_simt(); }

}  // namespace

size_t gram_workspace(int G, int64_t rows, int d, xkv_dtype dt) {
  if (!gram_tc_ok(G, d, dt)) return kAlign;
  const int64_t ldt = (rows + 7) / 8 * 8;
  return align_up(static_cast<size_t>(G) * d * ldt * 2);
}

xkv_status gram_launch(const void* const* X, int G, int64_t rows, int d, int64_t ldx, xkv_dtype dt, float* C,
                       void* ws, cudaStream_t st) {
  const int n = G * d;
  if (rows <= 0) return XKV_OK;
  // the vectorised transpose reads 16-byte aligned layers and rows
  bool vec_ok = ldx % 8 == 0 && d % 64 == 0;
  for (int l = 0; l < G; ++l) vec_ok = vec_ok && (reinterpret_cast<uintptr_t>(X[l]) & 15) == 0;
  if (gram_tc_ok(G, d, dt) && vec_ok) {
    const int64_t ldt = (rows + 7) / 8 * 8;
    __nv_bfloat16* Xt = static_cast<__nv_bfloat16*>(ws);
    LayerPtrs lp;
    for (int l = 0; l < 8; ++l) lp.p[l] = l < G ? X[l] : nullptr;
    dim3 tg(static_cast<unsigned>((ldt + 63) / 64), d / 64, G);
    transpose_layers_kernel<<<tg, 256, 0, st>>>(lp, d, ldx, rows, Xt, ldt);
    CUtensorMap xm;
    const uint64_t dims[2] = {static_cast<uint64_t>(rows), static_cast<uint64_t>(n)};
    const uint64_t str[1] = {static_cast<uint64_t>(ldt) * 2};
    const uint32_t box[2] = {64, 128};
    if (!make_tmap(&xm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Xt, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return XKV_ERR_CUDA;
    const int tiles_n = n / 128;
    const int nk = static_cast<int>((rows + 63) / 64);
    if (n % 256 == 0) {
      const int tiles_w = n / 256;
      int tiles = 0;
      for (int tm = 0; tm < tiles_n; ++tm) tiles += tiles_w - tm / 2;
      const size_t smem = gram_tc256_smem();
      cudaFuncSetAttribute(gram_tc256_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      gram_tc256_kernel<<<tiles, kGramWThreads, smem, st>>>(xm, nk, tiles_n, tiles_w, C, n, device_status_ptr());
    } else {
      const size_t smem = gram_tc_smem();
      cudaFuncSetAttribute(gram_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      gram_tc_kernel<<<tiles_n * (tiles_n + 1) / 2, kGramThreads, smem, st>>>(xm, nk, tiles_n, C, n,
                                                                               device_status_ptr());
    }
  } else {
    for (int li = 0; li < G; ++li)
      for (int lj = 0; lj < G; ++lj) {
        float* Cb = C + static_cast<int64_t>(li) * d * n + static_cast<int64_t>(lj) * d;
        if (dt == XKV_BF16)
          gemm_simt<__nv_bfloat16, __nv_bfloat16, float, float>(
              static_cast<const __nv_bfloat16*>(X[li]), 1, ldx, static_cast<const __nv_bfloat16*>(X[lj]), ldx, 1, Cb,
              n, d, d, static_cast<int>(rows), 1.0, 1.0, st);
        else
          gemm_simt<float, float, float, float>(static_cast<const float*>(X[li]), 1, ldx,
                                                static_cast<const float*>(X[lj]), ldx, 1, Cb, n, d, d,
                                                static_cast<int>(rows), 1.0, 1.0, st);
      }
  }
  return cudaPeekAtLastError() == cudaSuccess ? XKV_OK : XKV_ERR_CUDA;
}

// ------------------------------------------- subspace iteration on tcgen05
// Y = C Q for the symmetric Gram C (n x n f32) and the block Q (n x b f32),
// both split into bf16 hi/lo pairs (x = hi + lo keeps ~16 significant bits):
// Y = Chi Qhi + Chi Qlo + Clo Qhi, the three products accumulated in fp32 in
// TMEM (the dropped lo lo term and the split are of the order of the fp32
// rounding of a 4096-term dot product).  Used for the iterations, which need
// only the span of C Q.  C's pair is K-major (rows of C are
// its columns: C is symmetric), Q's pair is MN-major (Q row-major).  One
// 128 x bn output tile per CTA; warp 0 loads, warp 1 issues, warps 2-5 store.
constexpr int kCqStages = 3;
constexpr int kCqThreads = 192;

inline size_t cq_smem(int bn) { return 1024 + kCqStages * (32768 + 2 * bn * 128) + (2 * kCqStages + 2) * 8 + 16; }

__global__ void __launch_bounds__(kCqThreads, 1)
    cq_tc_kernel(const __grid_constant__ CUtensorMap chi, const __grid_constant__ CUtensorMap clo,
                 const __grid_constant__ CUtensorMap qhi, const __grid_constant__ CUtensorMap qlo, int n, int b,
                 int bn, float* __restrict__ Y, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int SB = 32768 + 2 * bn * 128;  // A hi, A lo (128 x 64), B hi, B lo (64 x bn)
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kCqStages * SB);
  uint64_t* empty = full + kCqStages;
  uint64_t* accbar = empty + kCqStages;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(accbar + 2);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * 128, n0 = blockIdx.y * bn;
  const int nk = n / 64;
  if (tid == 0) {
    for (int i = 0; i < kCqStages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    mbar_init(&accbar[0], 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tslot, 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  if (warp == 0) {
    if (lane == 0) {
      for (int a = 0; a < nk; ++a) {
        const int slot = a % kCqStages;
        if (!mbar_wait(&empty[slot], ((a / kCqStages) & 1) ^ 1, status)) break;
        uint8_t* st = smem + slot * SB;
        mbar_arrive_expect_tx(&full[slot], SB);
        tma_load_2d(st, &chi, &full[slot], a * 64, m0);
        tma_load_2d(st + 16384, &clo, &full[slot], a * 64, m0);
        for (int j = 0; j < bn / 64; ++j) {
          tma_load_2d(st + 32768 + j * 8192, &qhi, &full[slot], n0 + 64 * j, a * 64);
          tma_load_2d(st + 32768 + bn * 128 + j * 8192, &qlo, &full[slot], n0 + 64 * j, a * 64);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(128, bn, false, true);
      for (int a = 0; a < nk; ++a) {
        const int slot = a % kCqStages;
        if (!mbar_wait(&full[slot], (a / kCqStages) & 1, status)) break;
        tc_fence_after();
        uint8_t* st = smem + slot * SB;
        const uint64_t ah = umma_desc_sw128(smem_u32(st));
        const uint64_t al = umma_desc_sw128(smem_u32(st + 16384));
        const uint64_t bh = umma_desc_sw128_mn(smem_u32(st + 32768), 8192, 1024);
        const uint64_t bl = umma_desc_sw128_mn(smem_u32(st + 32768 + bn * 128), 8192, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          umma_bf16(tmem, ah + 2 * kk, bh + 128 * kk, idesc, (a | kk) ? 1u : 0u);
          umma_bf16(tmem, ah + 2 * kk, bl + 128 * kk, idesc, 1u);
          umma_bf16(tmem, al + 2 * kk, bh + 128 * kk, idesc, 1u);
        }
        umma_commit(&empty[slot]);
      }
      umma_commit(&accbar[0]);
    }
  } else {
    const int lq = warp & 3;
    const int m = m0 + lq * 32 + lane;
    const bool ok = mbar_wait(&accbar[0], 0, status);
    __syncwarp();  // converged for the warp-wide tcgen05.ld
    tc_fence_after();
    const uint32_t taddr = tmem + (static_cast<uint32_t>(lq * 32) << 16);
    if (ok) {
      for (int jb = 0; jb < bn / 16; ++jb) {
        float v[16];
        tmem_ld16(taddr + jb * 16, v);
        tmem_ld_wait();
        float4* yrow = reinterpret_cast<float4*>(Y + static_cast<int64_t>(m) * b + n0 + jb * 16);
#pragma unroll
        for (int i = 0; i < 4; ++i) yrow[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      }
    }
  }
  // reconverge the role warps before the block-wide barrier (TMEM release)
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// x (f32) -> hi = bf16(x), lo = bf16(x - hi), same layout
__global__ void split_hilo_kernel(const float* __restrict__ x, int64_t count, __nv_bfloat16* __restrict__ hi,
                                  __nv_bfloat16* __restrict__ lo) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float v = x[i];
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    hi[i] = h;
    lo[i] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
}

bool cq_tc_ok(int n, int b) { return n % 128 == 0 && b % 64 == 0 && n >= 128 && !force_simt(); }

// Y = C Q on tensor cores; chl / qhl: the bf16 hi/lo pairs of C (n x n, split
// once per factorisation) and of Q (n x b, split here)
xkv_status cq_launch(const __nv_bfloat16* chl, const float* Q, __nv_bfloat16* qhl, float* Y, int n, int b,
                     cudaStream_t st) {
  const int64_t nb = static_cast<int64_t>(n) * b;
  split_hilo_kernel<<<512, 256, 0, st>>>(Q, nb, qhl, qhl + nb);
  const int64_t nn = static_cast<int64_t>(n) * n;
  CUtensorMap mh, ml, bh, bl;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(n), static_cast<uint64_t>(n)};
    const uint64_t str[1] = {static_cast<uint64_t>(n) * 2};
    const uint32_t box[2] = {64, 128};
    if (!make_tmap(&mh, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, chl, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap(&ml, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, chl + nn, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return XKV_ERR_CUDA;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(b), static_cast<uint64_t>(n)};
    const uint64_t str[1] = {static_cast<uint64_t>(b) * 2};
    const uint32_t box[2] = {64, 64};
    if (!make_tmap(&bh, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, qhl, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap(&bl, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, qhl + nb, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return XKV_ERR_CUDA;
  }
  const int bn = b % 128 == 0 ? 128 : 64;
  const size_t smem = cq_smem(bn);
  cudaFuncSetAttribute(cq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  cq_tc_kernel<<<dim3(n / 128, b / bn), kCqThreads, smem, st>>>(mh, ml, bh, bl, n, b, bn, Y, device_status_ptr());
  return XKV_OK;
}

// ---------------------------------------------------------- factorisation
// Block width of the subspace iteration: b = min(rank + oversample, G d, rows).
xkv_status factor_plan(int n, int64_t rows, int rank, int oversample, FactorPlan* p) {
  const int64_t b = std::min<int64_t>(std::min<int64_t>(static_cast<int64_t>(rank) + std::max(oversample, 0), n), rows);
  p->n = n;
  p->b = static_cast<int>(b);
  p->rank = rank;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes);
    return o;
  };
  p->off_Q = take(static_cast<size_t>(n) * b * 4);
  p->off_Y = take(static_cast<size_t>(n) * b * 4);
  p->off_W = take(static_cast<size_t>(b) * b * 8);
  p->off_H = take(static_cast<size_t>(b) * b * 8);
  p->off_U = take(static_cast<size_t>(b) * b * 8);
  p->off_lam = take(static_cast<size_t>(b) * 8 + 64);
  p->off_ord = take(static_cast<size_t>(b) * 4);
  p->off_Ur = take(static_cast<size_t>(b) * rank * 4);
  p->off_Vr = take(static_cast<size_t>(n) * rank * 4);
  p->off_jac = take(jacobi_workspace(static_cast<int>(b), 1));
  p->off_dblk = take(cholqr_dblk_bytes(static_cast<int>(b)));
  p->off_part = take(cholqr_part_bytes(n, static_cast<int>(b)));
  // bf16 hi/lo pairs of C and of the block for the tensor-core C Q
  const bool tc = cq_tc_ok(n, static_cast<int>(b));
  p->off_chl = take(tc ? static_cast<size_t>(n) * n * 4 : 0);
  p->off_qhl = take(tc ? static_cast<size_t>(n) * b * 4 : 0);
  p->bytes = off;
  return XKV_OK;
}

// Steps 2 of the factorisation on a given Gram C (n x n f32): subspace
// iteration, Rayleigh-Ritz, V_r (f32, left in the workspace and optionally
// copied to Vr_out), the Ritz values, and Bt = V_r in the cache dtype.
xkv_status factor_launch(const FactorPlan& P, const float* C, xkv_dtype dt, int iters, uint64_t seed, void* Bt,
                         float* Vr_out, float* eigvals, void* ws, cudaStream_t st) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  const int n = P.n, b = P.b, r = P.rank;
  float* Q = reinterpret_cast<float*>(w + P.off_Q);
  float* Y = reinterpret_cast<float*>(w + P.off_Y);
  double* W = reinterpret_cast<double*>(w + P.off_W);
  double* H = reinterpret_cast<double*>(w + P.off_H);
  double* U = reinterpret_cast<double*>(w + P.off_U);
  double* lam = reinterpret_cast<double*>(w + P.off_lam);
  double* scal = lam + b;
  int* order = reinterpret_cast<int*>(w + P.off_ord);
  float* Ur = reinterpret_cast<float*>(w + P.off_Ur);
  float* Vr = reinterpret_cast<float*>(w + P.off_Vr);
  int* status = device_status_ptr();
  if (!status) return XKV_ERR_CUDA;
  double* part = gemm_splits(b, b, n) > 1 ? reinterpret_cast<double*>(w + P.off_part) : nullptr;
  const CholQRScratch cs{W, H, reinterpret_cast<double*>(w + P.off_dblk), part, scal};
  const bool tc = cq_tc_ok(n, b);
  __nv_bfloat16* chl = reinterpret_cast<__nv_bfloat16*>(w + P.off_chl);
  __nv_bfloat16* qhl = reinterpret_cast<__nv_bfloat16*>(w + P.off_qhl);
  if (tc) split_hilo_kernel<<<512, 256, 0, st>>>(C, static_cast<int64_t>(n) * n, chl, chl + static_cast<int64_t>(n) * n);
  // Y = C Q: on tensor cores (bf16 hi/lo splits) while iterating, where only
  // the span matters; in fp32 on CUDA cores for the Rayleigh-Ritz product, whose
  // Ritz values (eigvals, and the energy they leave out) need the full fp32
  // accuracy of C Q
  auto apply_c = [&](bool exact) -> xkv_status {
    if (tc && !exact) return cq_launch(chl, Q, qhl, Y, n, b, st);
    gemm_simt<float, float, float, float>(C, n, 1, Q, b, 1, Y, b, n, b, n, 1.0, 0.0, st);
    return XKV_OK;
  };
  gaussian_kernel<<<256, 256, 0, st>>>(Y, static_cast<int64_t>(n) * b, seed);
  // Q <- an orthonormal basis of span(src).  The iterations only need a
  // well-conditioned basis of the right span (the span is what converges), so
  // they take one shifted CholQR pass (orthogonal to ~1e-7 in fp32); the basis
  // that enters Rayleigh-Ritz takes a second, plain pass (CholQR2).
  auto orthonormalise = [&](float* src, bool twice) {
    cholqr_pass(src, Q, n, b, 1e-13, cs, status, st);
    if (!twice) return;
    cholqr_pass(Q, src, n, b, 0.0, cs, status, st);
    cudaMemcpyAsync(Q, src, static_cast<size_t>(n) * b * 4, cudaMemcpyDeviceToDevice, st);
  };
  orthonormalise(Y, iters == 0);
  for (int it = 0; it < iters; ++it) {
    xkv_status s = apply_c(false);
    if (s != XKV_OK) return s;
    orthonormalise(Y, it == iters - 1);
  }
  // Rayleigh-Ritz
  if (xkv_status s = apply_c(true); s != XKV_OK) return s;
  gemm_simt_split<float, float, double, double>(Q, 1, b, Y, b, 1, H, b, b, b, n, 1.0, 0.0, part, false, st);
  xkv_status s = jacobi_launch(H, U, lam, b, 1, w + P.off_jac, st);
  if (s != XKV_OK) return s;
  order_desc(lam, b, order, st);
  gather_ritz_kernel<<<64, 256, 0, st>>>(U, order, b, r, Ur, lam, eigvals);
  gemm_simt<float, float, float, float>(Q, b, 1, Ur, r, 1, Vr, r, n, r, b, 1.0, 0.0, st);
  if (dt == XKV_BF16)
    emit_factors_kernel<__nv_bfloat16><<<256, 256, 0, st>>>(Vr, n, r, static_cast<__nv_bfloat16*>(Bt), nullptr,
                                                            nullptr);
  else
    emit_factors_kernel<float><<<256, 256, 0, st>>>(Vr, n, r, static_cast<float*>(Bt), nullptr, nullptr);
  if (Vr_out && cudaMemcpyAsync(Vr_out, Vr, static_cast<size_t>(n) * r * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return XKV_ERR_CUDA;
  return cudaPeekAtLastError() == cudaSuccess ? XKV_OK : XKV_ERR_CUDA;
}

// ------------------------------------------------------------- projection
bool project_tc_ok(int d, int rank, xkv_dtype dt) { return dt == XKV_BF16 && rank % 64 == 0 && d % 64 == 0 && !force_simt(); }

size_t project_workspace(int n, int rank) { return align_up(static_cast<size_t>(2) * rank * n * 2); }

// V (n x rank, f32 or bf16) -> Vt hi (and lo for f32) (rank x n bf16)
template <typename TV>
__global__ void split_basis_kernel(const TV* __restrict__ V, int n, int r, __nv_bfloat16* __restrict__ vhi,
                                   __nv_bfloat16* __restrict__ vlo) {
  const int64_t total = static_cast<int64_t>(n) * r;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float v = to_f(V[i]);
    const int k = static_cast<int>(i / r), c = static_cast<int>(i % r);
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    vhi[static_cast<int64_t>(c) * n + k] = h;
    if (vlo) vlo[static_cast<int64_t>(c) * n + k] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
}

// A (T x rank, row stride lda) = X V, X = [X_1 | ... | X_G] through the layer
// pointers.  bf16 caches: tcgen05 GEMM; an f32 basis is split into a bf16
// hi/lo pair (two products per step keep ~16 significant bits), a bf16 basis
// is used as is.  f32 caches: CUDA-core GEMM per layer (f32 basis only).
xkv_status project_launch(const void* const* X, int G, int64_t T, int d, int64_t ldx, xkv_dtype dt, const void* V,
                          xkv_dtype v_dt, int r, void* A, int64_t lda, void* ws, cudaStream_t st) {
  const int n = G * d;
  if (T <= 0) return XKV_OK;
  int* status = device_status_ptr();
  if (!status) return XKV_ERR_CUDA;
  if (project_tc_ok(d, r, dt)) {
    __nv_bfloat16* vhi = static_cast<__nv_bfloat16*>(ws);
    __nv_bfloat16* vlo = vhi + static_cast<int64_t>(r) * n;
    const bool two = v_dt == XKV_F32;
    if (two)
      split_basis_kernel<float><<<256, 256, 0, st>>>(static_cast<const float*>(V), n, r, vhi, vlo);
    else
      split_basis_kernel<__nv_bfloat16><<<256, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(V), n, r, vhi, nullptr);
    TmapSet am;
    CUtensorMap bh, bl;
    for (int l = 0; l < G; ++l) {
      const uint64_t dims[2] = {static_cast<uint64_t>(d), static_cast<uint64_t>(T)};
      const uint64_t str[1] = {static_cast<uint64_t>(ldx) * 2};
      const uint32_t box[2] = {64, 128};
      if (!make_tmap(&am.m[l], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X[l], dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
        return XKV_ERR_CUDA;
    }
    const int bn = r % 128 == 0 ? 128 : 64;
    const uint64_t dims[2] = {static_cast<uint64_t>(n), static_cast<uint64_t>(r)};
    const uint64_t str[1] = {static_cast<uint64_t>(n) * 2};
    const uint32_t box[2] = {64, static_cast<uint32_t>(bn)};
    if (!make_tmap(&bh, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, vhi, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap(&bl, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, vlo, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return XKV_ERR_CUDA;
    GemmArgs g{};
    g.M = static_cast<int>(T);
    g.N = r;
    g.K = n;
    g.bn = bn;
    g.layer_cols = d;
    g.two_b = two ? 1 : 0;
    g.out = A;
    g.ldo = lda;
    g.status = status;
    const size_t smem = gemm_smem_bytes<kProj>();
    cudaFuncSetAttribute(gemm_tc_kernel<kProj>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if ((T + 127) / 128 > 65535) return XKV_ERR_UNSUPPORTED;  // row tiles on grid.y
    dim3 grid(r / bn, static_cast<unsigned>((T + 127) / 128));
    gemm_tc_kernel<kProj><<<grid, kGemmThreads, smem, st>>>(am, bh, bl, g);
  } else if (dt == XKV_F32 && v_dt == XKV_F32) {
    const float* Vf = static_cast<const float*>(V);
    for (int l = 0; l < G; ++l)
      gemm_simt<float, float, float, float>(static_cast<const float*>(X[l]), ldx, 1, Vf + static_cast<int64_t>(l) * d * r,
                                            r, 1, static_cast<float*>(A), lda, static_cast<int>(T), r, d, 1.0,
                                            l > 0 ? 1.0 : 0.0, st);
  } else {
    return XKV_ERR_UNSUPPORTED;
  }
  return cudaPeekAtLastError() == cudaSuccess ? XKV_OK : XKV_ERR_CUDA;
}

// ------------------------------------------------------------ whole group
xkv_status compress_plan(int G, int64_t T, int d, int rank, int oversample, int64_t shard_rows, xkv_dtype dt,
                         CompressPlan* p) {
  const int n = G * d;
  factor_plan(n, T, rank, oversample, &p->f);
  p->shard = shard_rows > 0 ? std::min<int64_t>(shard_rows, T) : T;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes);
    return o;
  };
  p->off_gram = take(static_cast<size_t>(n) * n * 4);
  p->off_gramws = take(gram_workspace(G, p->shard, d, dt));
  p->off_factor = take(p->f.bytes);
  p->off_proj = take(project_workspace(n, rank));
  p->bytes = off;
  return XKV_OK;
}

xkv_status compress_launch(const CompressPlan& P, const void* const* X, int G, int64_t T, int d, int64_t ldx,
                           xkv_dtype dt, int iters, uint64_t seed, void* A, void* Bt, float* eigvals,
                           float* gram_out, void* ws, cudaStream_t st) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  const int n = P.f.n, r = P.f.rank;
  const size_t es = dt == XKV_BF16 ? 2 : 4;
  float* C = gram_out ? gram_out : reinterpret_cast<float*>(w + P.off_gram);
  // 1. Gram over token shards
  if (cudaMemsetAsync(C, 0, static_cast<size_t>(n) * n * 4, st) != cudaSuccess) return XKV_ERR_CUDA;
  for (int64_t t0 = 0; t0 < T; t0 += P.shard) {
    const int64_t rows = std::min<int64_t>(P.shard, T - t0);
    const void* Xs[8];
    for (int l = 0; l < G; ++l) Xs[l] = static_cast<const uint8_t*>(X[l]) + t0 * ldx * es;
    const xkv_status s = gram_launch(Xs, G, rows, d, ldx, dt, C, w + P.off_gramws, st);
    if (s != XKV_OK) return s;
  }
  // 2. top-r subspace, Ritz values, Bt
  xkv_status s = factor_launch(P.f, C, dt, iters, seed, Bt, nullptr, eigvals, w + P.off_factor, st);
  if (s != XKV_OK) return s;
  // 3. A = X V_r from the f32 basis left in the factor workspace
  const float* Vr = reinterpret_cast<const float*>(w + P.off_factor + P.f.off_Vr);
  return project_launch(X, G, T, d, ldx, dt, Vr, XKV_F32, r, A, r, w + P.off_proj, st);
}

}  // namespace xkv
