// Host-side launchers shared between the C-ABI layer and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/xkv.h"

namespace xkv {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }

// Per-device status word (device address), created on first use.
int* device_status_ptr();
int num_sms();
bool force_simt();

// TMA descriptor creation through the driver entry point.
bool make_tmap(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
               const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz);

// ------------------------------------------------------------ SR decode
struct SRPlan {
  int units;        // B * Hkv
  int tiles_per_unit;
  int total_tiles;
  int ctas;         // attention CTAs (persistent ranges of tiles)
  int max_units_per_cta;
  bool tc;          // tcgen05 path
  size_t off_scores, off_sel, off_part, off_win, slot_floats, bytes;
};
// top-k shared memory: 9 bytes per chunk (+ padding) must stay under the
// 227 KiB opt-in with the kernel's static arrays
constexpr int64_t kMaxMidChunks = 24576;
xkv_status sr_plan(const xkv_sr_params* p, SRPlan* plan);
xkv_status sr_profile_enable(int enable);
xkv_status sr_profile_read(float* stage_ms);
// A token shard of the sequence: the selection is given (global chunk
// indices), only chunks in [c_lo, c_hi) are kept here, local row 0 sits at
// global position pos_off, and (M, L) per query head are written to ml_out.
struct SRShard {
  const int32_t* sel;
  int64_t pos_off;
  int c_lo, c_hi;
  float* ml_out;
};
// v_host (optional): the xK-SR value cache in page-locked host memory (device
// address); its kept rows are gathered into `stage` [units][k][chunk][hd].
xkv_status sr_launch(const xkv_sr_params* p, const SRPlan& plan, const void* q, const void* A_K,
                     const void* Bt_K, const void* A_V, const void* Bt_V, const void* landmarks,
                     const void* sr_K, const void* sr_V, float* out, int32_t* sel_out, void* ws,
                     cudaStream_t st, const void* v_host = nullptr, void* stage = nullptr,
                     const SRShard* shard = nullptr);
xkv_status sr_scores_launch(const xkv_sr_params* p, const void* q, const void* lm, float* scores, int64_t ld,
                            cudaStream_t st);
xkv_status sr_topk_launch(const float* scores, int64_t ld, int units, int64_t n, int k, int32_t* sel,
                          cudaStream_t st);
xkv_status merge_partials_launch(const float* o, const float* ml, int R, int rows, int hd, float* out,
                                 cudaStream_t st);

// --------------------------------------------------------- dense / recon
size_t dense_workspace(const xkv_dense_params* p);
xkv_status dense_launch(const xkv_dense_params* p, const void* q, const void* K, const void* V, float* out,
                        void* ws, cudaStream_t st);
xkv_status recon_launch(const void* A, const void* Bt, int64_t T, int rank, int d, int hkv, int hd,
                        int apply_rope, float theta, xkv_dtype dt, void* out, cudaStream_t st);

// ------------------------------------------------------------ landmarks
xkv_status landmarks_launch(const void* K, int64_t T, int64_t ldk, int hkv, int hd, xkv_dtype dt, int chunk,
                            int sink, int recent, float theta, void* out, cudaStream_t st);

// ---------------------------------------------------------- compression
size_t gram_workspace(int G, int64_t rows, int d, xkv_dtype dt);
xkv_status gram_launch(const void* const* X, int G, int64_t rows, int d, int64_t ldx, xkv_dtype dt, float* C,
                       void* ws, cudaStream_t st);
struct FactorPlan {
  int n, b, rank;
  size_t off_Q, off_Y, off_W, off_H, off_U, off_lam, off_ord, off_Ur, off_Vr, off_jac, off_dblk, off_part, off_chl,
      off_qhl, bytes;
};
xkv_status factor_plan(int n, int64_t rows, int rank, int oversample, FactorPlan* plan);
xkv_status factor_launch(const FactorPlan& plan, const float* C, xkv_dtype dt, int iters, uint64_t seed, void* Bt,
                         float* Vr_out, float* eigvals, void* ws, cudaStream_t st);
bool project_tc_ok(int d, int rank, xkv_dtype dt);
size_t project_workspace(int n, int rank);
xkv_status project_launch(const void* const* X, int G, int64_t T, int d, int64_t ldx, xkv_dtype dt, const void* V,
                          xkv_dtype v_dt, int rank, void* A, int64_t lda, void* ws, cudaStream_t st);
struct CompressPlan {
  FactorPlan f;
  int64_t shard;
  size_t off_gram, off_gramws, off_factor, off_proj, bytes;
};
xkv_status compress_plan(int G, int64_t T, int d, int rank, int oversample, int64_t shard_rows, xkv_dtype dt,
                         CompressPlan* plan);
xkv_status compress_launch(const CompressPlan& plan, const void* const* X, int G, int64_t T, int d,
                           int64_t ldx, xkv_dtype dt, int iters, uint64_t seed, void* A, void* Bt,
                           float* eigvals, float* gram_out, void* ws, cudaStream_t st);

// ---------------------------------------------------- multi-step decode
size_t append_workspace(const xkv_append_params* p);
xkv_status append_launch(const xkv_append_params* p, const void* const* k_new, const void* const* v_new,
                         void* const* win_K, void* const* win_V, const void* Bt_K, const void* Bt_V, void* A_K,
                         void* A_V, void* const* landmarks, int* rolled, void* ws, cudaStream_t st);

// ------------------------------------------------------------------ NER
size_t ner_workspace(int n, int block);
xkv_status energy_rank_launch(const float* gram, int n, int block, double energy, int32_t* rank, float* lam_out,
                               void* ws, cudaStream_t st);
xkv_status ner_launch(const float* gram, int n, int block, double tol, float* ner, float* erank, int32_t* rank,
                      void* ws, cudaStream_t st);

// Symmetric eigen-solver shared by Rayleigh-Ritz and NER (one-sided block Jacobi,
// fp64).  Operates on `count` independent n x n problems stored column-major
// at W (+ count * n * n each); V (optional) receives eigenvectors; lam the
// eigenvalues (unsorted, |lambda| from column norms).
size_t jacobi_workspace(int n, int count);
xkv_status jacobi_launch(double* W, double* V, double* lam, int n, int count, void* ws, cudaStream_t st);

// Eigenvalues only of `count` symmetric n x n problems (row-major fp64 at W,
// overwritten): Householder tridiagonalisation and bisection; lam receives
// each problem's eigenvalues in ascending order.
size_t spectrum_workspace(int n, int count);
xkv_status spectrum_launch(double* W, double* lam, int n, int count, void* ws, cudaStream_t st);

}  // namespace xkv
