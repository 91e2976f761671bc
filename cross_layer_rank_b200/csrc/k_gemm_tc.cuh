// tcgen05 GEMM tile kernel: D[m][n] = sum_k A[m][k] B[n][k] for one 128 x BN
// output tile per CTA (grid: column tiles x row tiles), both operands K-major bf16 loaded by TMA with the
// 128-byte swizzle, fp32 accumulation in TMEM.  Warp 0 issues TMA, warp 1
// issues tcgen05.mma, warps 2..5 drain TMEM through a mode-specific epilogue:
//   kRecon : bf16 store of A Bt^T with optional RoPE per head (position = row)
//   kProj  : A operand split over up to 8 layer tensor maps along K; B given
//            as a bf16 hi/lo pair (two MMAs per step) for ~16-bit coefficients,
//            or as one bf16 operand; bf16 store with row stride ldo
#pragma once

#include "xkv_common.cuh"

namespace xkv {

enum GemmMode { kRecon = 0, kProj = 1 };

struct TmapSet {
  CUtensorMap m[8];
};

struct GemmArgs {
  int M, N, K;          // K multiple of 64
  int bn;               // 64 or 128
  int layer_cols;       // kProj: columns per layer map (d)
  int two_b;            // kProj: B given as a hi/lo pair (1) or a single bf16 operand (0)
  void* out;            // bf16 [M][ldo]
  int64_t ldo;
  int hd;               // kRecon RoPE head size (0 = no RoPE)
  float theta;
  int* status;
};

// ring depth: the projection streams a long K (G d); the reconstruction's K is
// the rank, so two stages suffice and several CTAs share an SM (one's
// epilogue overlaps another's MMAs)
template <int MODE>
__host__ __device__ constexpr int gemm_stages() {
  return MODE == kProj ? 4 : 2;
}
constexpr int kGemmThreads = 192;

template <int MODE>
__host__ __device__ constexpr int gemm_stage_bytes() {
  return MODE == kProj ? 3 * 16384 : 2 * 16384;
}

template <int MODE>
inline size_t gemm_smem_bytes() {
  return 1024 + gemm_stages<MODE>() * gemm_stage_bytes<MODE>() + 64 * 8 + (2 * gemm_stages<MODE>() + 2) * 8 + 16;
}

template <int MODE>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ TmapSet amaps, const __grid_constant__ CUtensorMap bmap,
                   const __grid_constant__ CUtensorMap bmap_lo, const GemmArgs g) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int SB = gemm_stage_bytes<MODE>();
  constexpr int kGemmStages = gemm_stages<MODE>();
  double* ft = reinterpret_cast<double*>(smem + kGemmStages * SB);
  uint64_t* full = reinterpret_cast<uint64_t*>(ft + 64);
  uint64_t* empty = full + kGemmStages;
  uint64_t* accbar = empty + kGemmStages;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(accbar + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // the column tiles of one row tile are neighbours in launch order, so the
  // row tile's A operand is read from DRAM once and from L2 after
  const int tn = blockIdx.x, tm = blockIdx.y;
  const int m0 = tm * 128, n0 = tn * g.bn;
  const int nk = g.K / 64;

  if (tid == 0) {
    for (int i = 0; i < kGemmStages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    mbar_init(&accbar[0], 1);
    fence_mbar_init();
  }
  if (MODE == kRecon && g.hd > 0 && tid < g.hd / 2) ft[tid] = rope_turns(static_cast<double>(g.theta), tid, g.hd);
  if (warp == 1) tmem_alloc(tslot, 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == 0) {
    if (lane == 0) {
      const uint32_t bytes = 16384 + (MODE == kProj && g.two_b ? 2 : 1) * g.bn * 128;
      for (int a = 0; a < nk; ++a) {
        const int slot = a % kGemmStages;
        if (!mbar_wait(&empty[slot], ((a / kGemmStages) & 1) ^ 1, g.status)) break;
        uint8_t* st = smem + slot * SB;
        mbar_arrive_expect_tx(&full[slot], bytes);
        if (MODE == kProj) {
          const int kc = a * 64;
          const int layer = kc / g.layer_cols;
          tma_load_2d(st, &amaps.m[layer], &full[slot], kc - layer * g.layer_cols, m0);
        } else {
          tma_load_2d(st, &amaps.m[0], &full[slot], a * 64, m0);
        }
        tma_load_2d(st + 16384, &bmap, &full[slot], a * 64, n0);
        if (MODE == kProj && g.two_b) tma_load_2d(st + 2 * 16384, &bmap_lo, &full[slot], a * 64, n0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(128, g.bn);
      for (int a = 0; a < nk; ++a) {
        const int slot = a % kGemmStages;
        if (!mbar_wait(&full[slot], (a / kGemmStages) & 1, g.status)) break;
        tc_fence_after();
        uint8_t* st = smem + slot * SB;
        const uint64_t ad = umma_desc_sw128(smem_u32(st));
        const uint64_t bd = umma_desc_sw128(smem_u32(st + 16384));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) umma_bf16(tmem, ad + 2 * kk, bd + 2 * kk, idesc, (a | kk) ? 1u : 0u);
        if (MODE == kProj && g.two_b) {
          const uint64_t bl = umma_desc_sw128(smem_u32(st + 2 * 16384));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) umma_bf16(tmem, ad + 2 * kk, bl + 2 * kk, idesc, 1u);
        }
        umma_commit(&empty[slot]);
      }
      umma_commit(&accbar[0]);
    }
  } else {
    const int lq = warp & 3;
    const int row = lq * 32 + lane;
    const int m = m0 + row;
    const bool ok = mbar_wait(&accbar[0], 0, g.status);
    __syncwarp();  // converged for the warp-wide tcgen05.ld
    tc_fence_after();
    const uint32_t taddr = tmem + (static_cast<uint32_t>(lq * 32) << 16);
    if (ok) {
      if (MODE == kRecon && g.hd > 0) {
        __nv_bfloat16* O = static_cast<__nv_bfloat16*>(g.out);
        const int half = g.hd / 2;
        for (int hb = 0; hb < g.bn / g.hd; ++hb) {
          for (int jb = 0; jb < half / 16; ++jb) {
            float lo[16], hi[16];
            tmem_ld16(taddr + hb * g.hd + jb * 16, lo);
            tmem_ld16(taddr + hb * g.hd + half + jb * 16, hi);
            tmem_ld_wait();
            if (m < g.M) {
              uint32_t w0[8], w1[8];
#pragma unroll
              for (int i = 0; i < 16; i += 2) {
                float c0, s0, c1, s1;
                rope_cs(ft[jb * 16 + i], static_cast<double>(m), &c0, &s0);
                rope_cs(ft[jb * 16 + i + 1], static_cast<double>(m), &c1, &s1);
                w0[i / 2] = f2_to_bf2(lo[i] * c0 - hi[i] * s0, lo[i + 1] * c1 - hi[i + 1] * s1);
                w1[i / 2] = f2_to_bf2(hi[i] * c0 + lo[i] * s0, hi[i + 1] * c1 + lo[i + 1] * s1);
              }
              __nv_bfloat16* orow = O + static_cast<int64_t>(m) * g.ldo + n0 + hb * g.hd + jb * 16;
              *reinterpret_cast<uint4*>(orow) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
              *reinterpret_cast<uint4*>(orow + 8) = make_uint4(w0[4], w0[5], w0[6], w0[7]);
              *reinterpret_cast<uint4*>(orow + half) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
              *reinterpret_cast<uint4*>(orow + half + 8) = make_uint4(w1[4], w1[5], w1[6], w1[7]);
            }
          }
        }
      } else {
        __nv_bfloat16* O = static_cast<__nv_bfloat16*>(g.out);
        for (int jb = 0; jb < g.bn / 16; ++jb) {
          float v[16];
          tmem_ld16(taddr + jb * 16, v);
          tmem_ld_wait();
          if (m < g.M) {
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) w[i] = f2_to_bf2(v[2 * i], v[2 * i + 1]);
            __nv_bfloat16* orow = O + static_cast<int64_t>(m) * g.ldo + n0 + jb * 16;
            *reinterpret_cast<uint4*>(orow) = make_uint4(w[0], w[1], w[2], w[3]);
            *reinterpret_cast<uint4*>(orow + 8) = make_uint4(w[4], w[5], w[6], w[7]);
          }
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
    tmem_dealloc(tmem, 128);
  }
}

}  // namespace xkv
