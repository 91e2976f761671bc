/*
 * xKV CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 restatement of what the xKV hot path computes, written
 * from the published descriptions.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg load this library; the product never does, and
 * this file shares no code, header, table or constant with the CUDA library.
 *
 * Sources (page title -- section):
 *   [xKV-blog]  "xKV大模型压缩秘籍：跨层共享，小白也能轻松上手，收藏必备！"
 *               -- "xKV 到底做了什么？" (grouping, horizontal concatenation, one
 *               SVD, shared basis A and per-layer B_l) and "仅仅压缩还不够，xKV
 *               还做了“选择性重建”" (landmark-guided top-k chunk selection,
 *               reconstruct only the selected rows).
 *   [xKV-abs]   "xKV: Cross-Layer KV-Cache Compression via Aligned Singular
 *               Vector Extraction" -- abstract (joint factorisation of grouped
 *               layers into a shared low-rank subspace; Selective Reconstruction).
 *   [KV-CoRE]   "KV-CoRE: Benchmarking Data-Dependent Low-Rank Compressibility of
 *               KV-Caches in LLMs" -- 2.A (streamed covariance C = sum_t k_t^T k_t,
 *               eigen-decomposition) and 2.B (effective rank, NER = erank / r).
 *   [KQ-SVD]    "KQ-SVD: KV cache compression with provable guarantees on
 *               attention fidelity" -- 3.2 (multi-head attention, decode with a
 *               cache: h_T = softmax(q_T K^T / sqrt(d)) V) and 3.3 (truncated SVD
 *               is the Frobenius-optimal rank-R approximation, P = V V^T).
 *
 * Readings where the pages leave a step open: the Gram is uncentred; factors
 * are A = X V_r and B = V_r^T (stored transposed, Bt = V_r); keys are
 * factorised before RoPE and RoPE (rotate-half,
 * inv_freq_j = theta^(-2j/hd)) is applied to rebuilt keys at their absolute
 * position; a landmark is the mean of a chunk's post-RoPE keys; the chunk score
 * of a KV head is the sum over its GQA query heads of q_g . l_c; top-k breaks
 * ties toward the lower chunk index; sink and recent windows are kept raw; the
 * effective rank is the exponential of the entropy of the normalised singular
 * values sigma_i = sqrt(lambda_i) over the numerical rank r = #{lambda_i >
 * tol * lambda_max}.
 *
 * Every input is float32 (bf16 values arrive exactly widened); every
 * intermediate and output is double unless stated.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define XO_EXPORT __attribute__((visibility("default")))

XO_EXPORT int xo_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ---------------------------------------------------------------- storage */
/* Round a double to the nearest bfloat16 (ties to even), returned widened.
 * Values are first rounded to float (the intermediate an fp32 accumulator
 * holds); bfloat16 keeps the top 16 bits of the float encoding. */
static float xo_round_bf16(double x) {
  float f = (float)x;
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u) return f; /* inf / nan unchanged */
  uint32_t lsb = (u >> 16) & 1u;
  u = (u + 0x7FFFu + lsb) & 0xFFFF0000u;
  memcpy(&f, &u, 4);
  return f;
}

XO_EXPORT void xo_round_bf16_array(const double* x, float* y, int64_t n) {
  for (int64_t i = 0; i < n; ++i) y[i] = xo_round_bf16(x[i]);
}

/* ------------------------------------------------------------------ Gram */
/* [KV-CoRE] 2.A: C += sum_{t in [t0,t1)} x_t^T x_t, where x_t is row t of the
 * horizontal concatenation X = [K_1 | ... | K_G] of [xKV-blog] "xKV 到底做了什么".
 * layers[l] points at a T x d matrix with row stride ldx; C is (G d) x (G d). */
XO_EXPORT void xo_gram_accumulate(const float* const* layers, int G, int64_t T, int d,
                                  int64_t ldx, int64_t t0, int64_t t1, double* C) {
  const int n = G * d;
  const int64_t rows = t1 - t0;
  (void)T;
  if (rows <= 0) return;
  /* Column i of X copied out contiguously (a change of layout only: each entry
   * below is still the ascending-t sum of x_t[i] x_t[j]). */
  float* cols = (float*)malloc(sizeof(float) * (size_t)n * (size_t)rows);
#pragma omp parallel for schedule(static)
  for (int i = 0; i < n; ++i) {
    const float* Li = layers[i / d];
    const int ci = i % d;
    for (int64_t t = 0; t < rows; ++t) cols[(int64_t)i * rows + t] = Li[(t0 + t) * ldx + ci];
  }
#pragma omp parallel for schedule(dynamic, 8)
  for (int i = 0; i < n; ++i) {
    const float* xi = cols + (int64_t)i * rows;
    for (int j = i; j < n; ++j) {
      const float* xj = cols + (int64_t)j * rows;
      double s = 0.0;
      for (int64_t t = 0; t < rows; ++t) s += (double)xi[t] * (double)xj[t];
      C[(int64_t)i * n + j] += s;
      if (j != i) C[(int64_t)j * n + i] += s;
    }
  }
  free(cols);
}

/* --------------------------------------------------------------- Jacobi */
/* Cyclic Jacobi eigen-decomposition of a symmetric matrix, visiting all pairs
 * once per sweep in round-robin ("parallel") order so that the n/2 rotations of
 * one step touch disjoint rows and columns.  Each rotation is the symmetric
 * Schur rotation that zeroes a_pq:
 *   tau = (a_qq - a_pp) / (2 a_pq),  t = sign(tau) / (|tau| + sqrt(1 + tau^2)),
 *   c = 1 / sqrt(1 + t^2),  s = t c,  A <- J^T A J,  V <- V J.
 * Pairs with |a_pq| <= 1e-15 ||A||_F are not rotated.  Stops when
 * off(A) <= tol * ||A||_F or when a whole sweep rotated nothing.  A (row-major
 * n x n) is overwritten.
 * On return w[0..n) holds the eigenvalues in descending order and column k of V
 * (row-major n x n) the matching unit eigenvector.  Returns the sweep count, or
 * -1 if max_sweeps was reached. */
XO_EXPORT int xo_jacobi_eigh(double* A, int n, double* w, double* V, double tol, int max_sweeps) {
  const int m = n + (n & 1); /* players in the round-robin; index n is a bye */
  int* play = (int*)malloc(sizeof(int) * m);
  double* cs = (double*)malloc(sizeof(double) * m);
  double* sn = (double*)malloc(sizeof(double) * m);
  int* pp = (int*)malloc(sizeof(int) * m);
  int* qq = (int*)malloc(sizeof(int) * m);
  for (int i = 0; i < n; ++i)
    for (int j = 0; j < n; ++j) V[(int64_t)i * n + j] = (i == j) ? 1.0 : 0.0;
  double fro = 0.0;
  for (int64_t i = 0; i < (int64_t)n * n; ++i) fro += A[i] * A[i];
  fro = sqrt(fro);
  const double skip = 1e-15 * fro;
  int sweep = 0, converged = 0;
  long rotations = 0;
  for (sweep = 0; sweep < max_sweeps; ++sweep) {
    double off = 0.0;
    for (int i = 0; i < n; ++i)
      for (int j = 0; j < n; ++j)
        if (i != j) off += A[(int64_t)i * n + j] * A[(int64_t)i * n + j];
    if (sqrt(off) <= tol * fro || fro == 0.0 || (sweep > 0 && rotations == 0)) { converged = 1; break; }
    rotations = 0;
    for (int i = 0; i < m; ++i) play[i] = i;
    for (int step = 0; step < m - 1; ++step) {
      int np = 0;
      for (int k = 0; k < m / 2; ++k) {
        int p = play[k], q = play[m - 1 - k];
        if (p >= n || q >= n) continue;
        if (p > q) { int tmp = p; p = q; q = tmp; }
        pp[np] = p; qq[np] = q; ++np;
      }
      /* rotation of each pair from the current 2x2 block */
      for (int k = 0; k < np; ++k) {
        const int p = pp[k], q = qq[k];
        const double apq = A[(int64_t)p * n + q];
        const double app = A[(int64_t)p * n + p], aqq = A[(int64_t)q * n + q];
        /* entries at the rounding level of ||A||_F are left alone: rotating
         * them only reshuffles rounding noise (e.g. inside a null space) */
        if (fabs(apq) <= skip) { cs[k] = 1.0; sn[k] = 0.0; continue; }
        ++rotations;
        const double tau = (aqq - app) / (2.0 * apq);
        const double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
        cs[k] = 1.0 / sqrt(1.0 + t * t);
        sn[k] = t * cs[k];
      }
      /* A <- A J (columns), V <- V J */
#pragma omp parallel for schedule(static)
      for (int i = 0; i < n; ++i) {
        double* Ai = A + (int64_t)i * n;
        double* Vi = V + (int64_t)i * n;
        for (int k = 0; k < np; ++k) {
          const int p = pp[k], q = qq[k];
          const double c = cs[k], s = sn[k];
          const double ap = Ai[p], aq = Ai[q];
          Ai[p] = c * ap - s * aq;
          Ai[q] = s * ap + c * aq;
          const double vp = Vi[p], vq = Vi[q];
          Vi[p] = c * vp - s * vq;
          Vi[q] = s * vp + c * vq;
        }
      }
      /* A <- J^T A (rows) */
#pragma omp parallel for schedule(static)
      for (int k = 0; k < np; ++k) {
        double* Ap = A + (int64_t)pp[k] * n;
        double* Aq = A + (int64_t)qq[k] * n;
        const double c = cs[k], s = sn[k];
        for (int j = 0; j < n; ++j) {
          const double ap = Ap[j], aq = Aq[j];
          Ap[j] = c * ap - s * aq;
          Aq[j] = s * ap + c * aq;
        }
      }
      /* next round-robin arrangement: player 0 fixed, the others rotate */
      const int last = play[m - 1];
      for (int i = m - 1; i > 1; --i) play[i] = play[i - 1];
      play[1] = last;
    }
  }
  /* eigenvalues from the diagonal, sorted descending (ties: lower index first) */
  int* order = pp;
  int* tmpi = qq;
  for (int i = 0; i < n; ++i) order[i] = i;
  for (int i = 1; i < n; ++i) { /* insertion sort: stable, exact */
    int key = order[i], j = i - 1;
    const double kv = A[(int64_t)key * n + key];
    while (j >= 0 && A[(int64_t)order[j] * n + order[j]] < kv) { order[j + 1] = order[j]; --j; }
    order[j + 1] = key;
  }
  double* Vs = (double*)malloc(sizeof(double) * (size_t)n * n);
  for (int k = 0; k < n; ++k) {
    w[k] = A[(int64_t)order[k] * n + order[k]];
    for (int i = 0; i < n; ++i) Vs[(int64_t)i * n + k] = V[(int64_t)i * n + order[k]];
  }
  memcpy(V, Vs, sizeof(double) * (size_t)n * n);
  (void)tmpi;
  free(Vs); free(play); free(cs); free(sn); free(pp); free(qq);
  return converged ? sweep : -1;
}

/* ---------------------------------------------------------- compression */
/* [xKV-blog] "xKV 到底做了什么": one decomposition of the horizontally
 * concatenated group, a shared token basis A and per-layer reconstruction
 * matrices B_l; [KQ-SVD] 3.3: the rank-r truncation X V_r V_r^T is optimal.
 *   C = X^T X (uncentred), C = V diag(lambda) V^T (cyclic Jacobi),
 *   A = X V_r (T x r), Bt = V_r ((G d) x r; layer l owns rows l d .. l d + d - 1).
 * stats[0] = ||X - A V_r^T||_F (subspace error),
 * stats[1] = ||X - bf16(A) bf16(V_r)^T||_F (stored-factor error),
 * stats[2] = sum_{i >= r} lambda_i (discarded energy),
 * stats[3] = ||X||_F^2, stats[4] = Jacobi sweeps.
 * lam receives all G d eigenvalues, descending.  Returns 0, or -1 if Jacobi did
 * not converge. */
XO_EXPORT int xo_compress_group(const float* const* layers, int G, int64_t T, int d, int64_t ldx,
                                int r, double* A, double* Bt, double* lam, double* stats) {
  const int n = G * d;
  double* C = (double*)calloc((size_t)n * n, sizeof(double));
  double* Vf = (double*)malloc(sizeof(double) * (size_t)n * n);
  xo_gram_accumulate(layers, G, T, d, ldx, 0, T, C);
  const int sweeps = xo_jacobi_eigh(C, n, lam, Vf, 1e-14, 60);
  for (int i = 0; i < n; ++i)
    for (int k = 0; k < r; ++k) Bt[(int64_t)i * r + k] = Vf[(int64_t)i * n + k];
  free(Vf);
  free(C);
  /* A = X V_r */
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    for (int k = 0; k < r; ++k) {
      double s = 0.0;
      for (int i = 0; i < n; ++i)
        s += (double)layers[i / d][t * ldx + (i % d)] * Bt[(int64_t)i * r + k];
      A[t * r + k] = s;
    }
  }
  /* errors of the subspace approximation and of the bf16-stored factors */
  float* Ab = (float*)malloc(sizeof(float) * (size_t)T * r);
  float* Bb = (float*)malloc(sizeof(float) * (size_t)n * r);
  xo_round_bf16_array(A, Ab, T * r);
  xo_round_bf16_array(Bt, Bb, (int64_t)n * r);
  double e_sub = 0.0, e_sto = 0.0, xx = 0.0;
#pragma omp parallel for schedule(static) reduction(+ : e_sub, e_sto, xx)
  for (int64_t t = 0; t < T; ++t) {
    for (int i = 0; i < n; ++i) {
      const double x = (double)layers[i / d][t * ldx + (i % d)];
      double y = 0.0, yb = 0.0;
      for (int k = 0; k < r; ++k) {
        y += A[t * r + k] * Bt[(int64_t)i * r + k];
        yb += (double)Ab[t * r + k] * (double)Bb[(int64_t)i * r + k];
      }
      e_sub += (x - y) * (x - y);
      e_sto += (x - yb) * (x - yb);
      xx += x * x;
    }
  }
  double tail = 0.0;
  for (int i = r; i < n; ++i) tail += lam[i];
  stats[0] = sqrt(e_sub);
  stats[1] = sqrt(e_sto);
  stats[2] = tail;
  stats[3] = xx;
  stats[4] = (double)sweeps;
  free(Ab);
  free(Bb);
  return sweeps < 0 ? -1 : 0;
}

/* ------------------------------------------------------------------ RoPE */
/* Rotary position embedding, rotate-half pairing (j, j + hd/2) at absolute
 * position pos with inv_freq_j = theta^(-2j/hd):
 *   y_j        = x_j cos(pos f_j) - x_{j+h} sin(pos f_j)
 *   y_{j+h}    = x_{j+h} cos(pos f_j) + x_j sin(pos f_j). */
XO_EXPORT void xo_rope(const double* x, double* y, int hd, double pos, double theta) {
  const int h = hd / 2;
  for (int j = 0; j < h; ++j) {
    const double f = pow(theta, -2.0 * (double)j / (double)hd);
    const double a = pos * f;
    const double c = cos(a), s = sin(a);
    const double x0 = x[j], x1 = x[j + h];
    y[j] = x0 * c - x1 * s;
    y[j + h] = x1 * c + x0 * s;
  }
}

/* ------------------------------------------------------------- landmarks */
/* [xKV-blog] "选择性重建": chunk landmarks guide the top-k chunk selector.
 * Landmark of (KV head h, middle chunk c) = mean over the chunk's tokens
 * t in [sink + c C, sink + (c+1) C) of RoPE_t(K[t, h hd : (h+1) hd]).
 * K is T x d (pre-RoPE, row stride ldk); out is [Hkv][n_mid][hd]. */
XO_EXPORT void xo_landmarks(const float* K, int64_t T, int64_t ldk, int Hkv, int hd, int C, int sink,
                            int recent, double theta, double* out) {
  const int64_t n_mid = (T - sink - recent) / C;
#pragma omp parallel for collapse(2) schedule(static)
  for (int h = 0; h < Hkv; ++h) {
    for (int64_t c = 0; c < n_mid; ++c) {
      double x[512], y[512], acc[512];
      for (int j = 0; j < hd; ++j) acc[j] = 0.0;
      for (int i = 0; i < C; ++i) {
        const int64_t t = sink + c * C + i;
        for (int j = 0; j < hd; ++j) x[j] = (double)K[t * ldk + h * hd + j];
        xo_rope(x, y, hd, (double)t, theta);
        for (int j = 0; j < hd; ++j) acc[j] += y[j];
      }
      for (int j = 0; j < hd; ++j) out[((int64_t)h * n_mid + c) * hd + j] = acc[j] / (double)C;
    }
  }
}

/* ----------------------------------------------------- reconstruction */
/* [xKV-blog] "xKV 到底做了什么": K_l ~= A B_l, i.e. out[t][c] = sum_i A[t][i] Bt[c][i]
 * for all T rows, optionally followed by RoPE per head at position t.
 * A is T x r, Bt is d x r, out is T x d. */
XO_EXPORT void xo_full_reconstruct(const float* A, const float* Bt, int64_t T, int r, int d, int Hkv,
                                   int hd, int apply_rope, double theta, double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    double row[8192];
    for (int c = 0; c < d; ++c) {
      double s = 0.0;
      for (int i = 0; i < r; ++i) s += (double)A[t * r + i] * (double)Bt[(int64_t)c * r + i];
      row[c] = s;
    }
    for (int h = 0; h < Hkv; ++h) {
      if (apply_rope) xo_rope(row + h * hd, out + t * d + h * hd, hd, (double)t, theta);
      else for (int j = 0; j < hd; ++j) out[t * d + h * hd + j] = row[h * hd + j];
    }
  }
}

/* ------------------------------------------------------------ attention */
/* [KQ-SVD] 3.2 decode step: o = softmax(q K^T / sqrt(hd)) V over the n given
 * keys (already rotated) and values, each row hd long.  Written with the
 * maximum subtracted, which leaves the softmax unchanged. */
static void xo_attend(const double* q, const double* Kr, const double* Vr, int64_t n, int hd,
                      double* o) {
  double* s = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  double mx = -INFINITY;
  const double scale = 1.0 / sqrt((double)hd);
  for (int64_t t = 0; t < n; ++t) {
    double dot = 0.0;
    for (int j = 0; j < hd; ++j) dot += q[j] * Kr[t * hd + j];
    s[t] = dot * scale;
    if (s[t] > mx) mx = s[t];
  }
  double den = 0.0;
  for (int64_t t = 0; t < n; ++t) { s[t] = exp(s[t] - mx); den += s[t]; }
  for (int j = 0; j < hd; ++j) o[j] = 0.0;
  for (int64_t t = 0; t < n; ++t)
    for (int j = 0; j < hd; ++j) o[j] += s[t] * Vr[t * hd + j];
  for (int j = 0; j < hd; ++j) o[j] /= den;
  free(s);
}

/* Dense decode attention over a full cache (the comparison path of
 * [xKV-blog] Fig. 6: reconstruct everything, then attend).  K holds post-RoPE
 * keys.  q [B][Hq][hd], K,V [B][T][d], out [B][Hq][hd]; query head j reads KV
 * head j / (Hq / Hkv).  units (b * Hkv + h) restricts the work (NULL: all). */
XO_EXPORT void xo_dense_decode(int B, int Hq, int Hkv, int hd, int64_t T, const float* q,
                               const float* K, const float* V, const int32_t* units, int n_units,
                               double* out) {
  const int gq = Hq / Hkv, d = Hkv * hd;
  const int nu = units ? n_units : B * Hkv;
#pragma omp parallel for schedule(dynamic, 1)
  for (int u = 0; u < nu; ++u) {
    const int unit = units ? units[u] : u;
    const int b = unit / Hkv, h = unit % Hkv;
    double* Kr = (double*)malloc(sizeof(double) * (size_t)T * hd);
    double* Vr = (double*)malloc(sizeof(double) * (size_t)T * hd);
    for (int64_t t = 0; t < T; ++t)
      for (int j = 0; j < hd; ++j) {
        Kr[t * hd + j] = K[((int64_t)b * T + t) * d + h * hd + j];
        Vr[t * hd + j] = V[((int64_t)b * T + t) * d + h * hd + j];
      }
    for (int g = 0; g < gq; ++g) {
      const int qh = h * gq + g;
      double qq[512];
      for (int j = 0; j < hd; ++j) qq[j] = q[((int64_t)b * Hq + qh) * hd + j];
      xo_attend(qq, Kr, Vr, T, hd, out + ((int64_t)b * Hq + qh) * hd);
    }
    free(Kr);
    free(Vr);
  }
}

/* -------------------------------------------------------- SR decode */
typedef struct {
  int batch, n_q_heads, n_kv_heads, head_dim;
  int64_t T;
  int rank_k, rank_v;
  int chunk, topk, sink, recent;
  double rope_theta;
} xo_sr_params;

typedef struct { double s; int64_t c; } xo_scored;

/* exact order: larger score first; equal scores -> lower chunk index first */
static int xo_cmp_scored(const void* a, const void* b) {
  const xo_scored* x = (const xo_scored*)a;
  const xo_scored* y = (const xo_scored*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return (x->c < y->c) ? -1 : (x->c > y->c);
}

static int xo_cmp_i32(const void* a, const void* b) {
  const int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

/* One decode step of Selective Reconstruction ([xKV-blog] "选择性重建",
 * [xKV-abs]) for the units listed (b * Hkv + h; NULL: all):
 *   1. s_c = sum_{g in group(h)} q_g . l_c for every middle chunk c;
 *   2. keep the top-k chunks (exact sort; ties -> lower c), ascending by c,
 *      unless sel_in supplies the selection;
 *   3. rebuild rows t of the kept chunks: K_t = RoPE_t(A_K[t] B_K), V_t = A_V[t] B_V
 *      (B_K restricted to head h's hd columns; Bt stores B transposed).  In the
 *      xK-SR mode ([xKV-blog] "选择性重建": keys compressed, values kept whole)
 *      Bt_V is NULL and A_V is the uncompressed value cache [B][T][d]: V_t is
 *      read as is, head h's hd columns of row t;
 *   4. raw sink rows [0, sink) and recent rows [T - recent, T) (RoPE on K);
 *   5. o_g = softmax(q_g K^T / sqrt(hd)) V over sink, kept and recent rows.
 * Shapes: q [B][Hq][hd]; A_K [B][T][rK] (batch stride sak); Bt_K [B][d][rK]
 * (batch stride sbk; 0 = one Bt for the batch); A_V [B][T][rV] (sav); Bt_V
 * [B][d][rV] (sbv), or NULL with A_V [B][T][d] (sav; rank_v unused); lm
 * [B][Hkv][n_mid][hd]; srK, srV
 * [B][sink+recent][d]; out [B][Hq][hd]; sel_out [B][Hkv][k];
 * scores_out [B][Hkv][n_mid] (optional). */
XO_EXPORT int xo_sr_decode(const xo_sr_params* p, const float* q, const float* A_K, int64_t sak,
                           const float* Bt_K, int64_t sbk, const float* A_V, int64_t sav, const float* Bt_V,
                           int64_t sbv,
                           const float* lm, const float* srK, const float* srV,
                           const int32_t* sel_in, const int32_t* units, int n_units, double* out,
                           int32_t* sel_out, double* scores_out) {
  const int Hq = p->n_q_heads, Hkv = p->n_kv_heads, hd = p->head_dim, gq = Hq / Hkv;
  const int d = Hkv * hd, C = p->chunk, k = p->topk, sw = p->sink + p->recent;
  const int64_t T = p->T, n_mid = (T - p->sink - p->recent) / C;
  const int rK = p->rank_k, rV = p->rank_v;
  if (k > n_mid || (T - p->sink - p->recent) % C != 0) return -1;
  const int nu = units ? n_units : p->batch * Hkv;
#pragma omp parallel for schedule(dynamic, 1)
  for (int u = 0; u < nu; ++u) {
    const int unit = units ? units[u] : u;
    const int b = unit / Hkv, h = unit % Hkv;
    /* 1. chunk scores */
    xo_scored* sc = (xo_scored*)malloc(sizeof(xo_scored) * (size_t)n_mid);
    for (int64_t c = 0; c < n_mid; ++c) {
      const float* l = lm + (((int64_t)b * Hkv + h) * n_mid + c) * hd;
      double s = 0.0;
      for (int g = 0; g < gq; ++g) {
        const float* qg = q + ((int64_t)b * Hq + h * gq + g) * hd;
        for (int j = 0; j < hd; ++j) s += (double)qg[j] * (double)l[j];
      }
      sc[c].s = s;
      sc[c].c = c;
      if (scores_out) scores_out[((int64_t)b * Hkv + h) * n_mid + c] = s;
    }
    /* 2. top-k */
    int32_t* sel = (int32_t*)malloc(sizeof(int32_t) * (size_t)(k > 0 ? k : 1));
    if (sel_in) {
      for (int i = 0; i < k; ++i) sel[i] = sel_in[((int64_t)b * Hkv + h) * k + i];
    } else {
      qsort(sc, (size_t)n_mid, sizeof(xo_scored), xo_cmp_scored);
      for (int i = 0; i < k; ++i) sel[i] = (int32_t)sc[i].c;
    }
    qsort(sel, (size_t)k, sizeof(int32_t), xo_cmp_i32);
    if (sel_out)
      for (int i = 0; i < k; ++i) sel_out[((int64_t)b * Hkv + h) * k + i] = sel[i];
    /* 3-4. the attended rows */
    const int64_t n = (int64_t)sw + (int64_t)k * C;
    double* Kr = (double*)malloc(sizeof(double) * (size_t)n * hd);
    double* Vr = (double*)malloc(sizeof(double) * (size_t)n * hd);
    double x[512];
    int64_t row = 0;
    for (int i = 0; i < p->sink; ++i, ++row) {
      const int64_t t = i;
      for (int j = 0; j < hd; ++j) x[j] = srK[((int64_t)b * sw + i) * d + h * hd + j];
      xo_rope(x, Kr + row * hd, hd, (double)t, p->rope_theta);
      for (int j = 0; j < hd; ++j) Vr[row * hd + j] = srV[((int64_t)b * sw + i) * d + h * hd + j];
    }
    for (int i = 0; i < k; ++i) {
      for (int e = 0; e < C; ++e, ++row) {
        const int64_t t = p->sink + (int64_t)sel[i] * C + e;
        const float* ak = A_K + b * sak + t * rK;
        for (int j = 0; j < hd; ++j) {
          const float* bk = Bt_K + b * sbk + (int64_t)(h * hd + j) * rK;
          double sk = 0.0, sv = 0.0;
          for (int a = 0; a < rK; ++a) sk += (double)ak[a] * (double)bk[a];
          if (Bt_V) {
            const float* av = A_V + b * sav + t * rV;
            const float* bv = Bt_V + b * sbv + (int64_t)(h * hd + j) * rV;
            for (int a = 0; a < rV; ++a) sv += (double)av[a] * (double)bv[a];
          } else {
            sv = A_V[b * sav + t * d + h * hd + j];
          }
          x[j] = sk;
          Vr[row * hd + j] = sv;
        }
        xo_rope(x, Kr + row * hd, hd, (double)t, p->rope_theta);
      }
    }
    for (int i = 0; i < p->recent; ++i, ++row) {
      const int64_t t = T - p->recent + i;
      const int64_t srow = (int64_t)b * sw + p->sink + i;
      for (int j = 0; j < hd; ++j) x[j] = srK[srow * d + h * hd + j];
      xo_rope(x, Kr + row * hd, hd, (double)t, p->rope_theta);
      for (int j = 0; j < hd; ++j) Vr[row * hd + j] = srV[srow * d + h * hd + j];
    }
    /* 5. attention per query head of the group */
    for (int g = 0; g < gq; ++g) {
      const int qh = h * gq + g;
      double qq[512];
      for (int j = 0; j < hd; ++j) qq[j] = q[((int64_t)b * Hq + qh) * hd + j];
      xo_attend(qq, Kr, Vr, n, hd, out + ((int64_t)b * Hq + qh) * hd);
    }
    free(Kr); free(Vr); free(sel); free(sc);
  }
  return 0;
}

/* ------------------------------------------------------------------ NER */
/* [KV-CoRE] 2.B: for each diagonal block C_ll (block x block) of the Gram:
 * eigenvalues lambda (Jacobi), numerical rank r = #{lambda_i > tol lambda_max},
 * sigma_i = sqrt(lambda_i) over those r, p_i = sigma_i / sum sigma,
 * erank = exp(-sum p_i ln p_i), NER = erank / r in [1/r, 1].
 * A block with lambda_max <= 0 gets rank 0, erank 0, NER 0.
 * eig_out (optional) receives each block's eigenvalues, descending. */
XO_EXPORT int xo_ner(const double* C, int n, int block, double rel_tol, double* ner, double* erank,
                     int32_t* rank, double* eig_out) {
  const int nb = n / block;
  int status = 0;
  for (int b = 0; b < nb; ++b) {
    double* Ab = (double*)malloc(sizeof(double) * (size_t)block * block);
    double* Vb = (double*)malloc(sizeof(double) * (size_t)block * block);
    double* w = (double*)malloc(sizeof(double) * (size_t)block);
    for (int i = 0; i < block; ++i)
      for (int j = 0; j < block; ++j)
        Ab[(int64_t)i * block + j] = C[(int64_t)(b * block + i) * n + b * block + j];
    if (xo_jacobi_eigh(Ab, block, w, Vb, 1e-14, 60) < 0) status = -1;
    const double lmax = w[0];
    int r = 0;
    double ssum = 0.0;
    for (int i = 0; i < block; ++i)
      if (lmax > 0.0 && w[i] > rel_tol * lmax) { ++r; ssum += sqrt(w[i]); }
    double H = 0.0;
    for (int i = 0; i < block; ++i)
      if (lmax > 0.0 && w[i] > rel_tol * lmax) {
        const double pi = sqrt(w[i]) / ssum;
        if (pi > 0.0) H -= pi * log(pi);
      }
    const double er = r > 0 ? exp(H) : 0.0;
    ner[b] = r > 0 ? er / (double)r : 0.0;
    if (erank) erank[b] = er;
    if (rank) rank[b] = r;
    if (eig_out) memcpy(eig_out + (int64_t)b * block, w, sizeof(double) * block);
    free(Ab); free(Vb); free(w);
  }
  return status;
}

/* ---------------------------------------------------- multi-step decode */
/* [xKV-blog] (the editor's note after "仅仅压缩还不够，xKV 还做了“选择性重建”"):
 * the factorisation covers the long prefill; tokens generated afterwards stay
 * raw in the recent window until a whole chunk of them can join the
 * compressed cache.  Two steps of that roll, restated plainly:
 *
 * Projection of `rows` token rows onto a stored group basis V ((G d) x r):
 *   A[t][k] = sum_i x_t[i] V[i][k],  x_t = [K_1[t] | ... | K_G[t]]
 * (the same A = X V_r as the prefill factorisation, "xKV 到底做了什么").
 * layers[l] is rows x d with row stride ldx; A is rows x r. */
XO_EXPORT void xo_project_rows(const float* const* layers, int G, int64_t rows, int d, int64_t ldx,
                               const float* V, int r, double* A) {
  const int n = G * d;
  for (int64_t t = 0; t < rows; ++t)
    for (int k = 0; k < r; ++k) {
      double s = 0.0;
      for (int i = 0; i < n; ++i) s += (double)layers[i / d][t * ldx + (i % d)] * (double)V[(int64_t)i * r + k];
      A[t * r + k] = s;
    }
}

/* Landmark of one chunk whose C rows sit at absolute positions t0 .. t0+C-1
 * ([xKV-blog] "选择性重建"): for KV head h, the mean over i of
 * RoPE_{t0+i}(K[i, h hd : (h+1) hd]).  K rows have stride ldk; out is
 * [Hkv][hd]. */
XO_EXPORT void xo_chunk_landmark(const float* K, int64_t ldk, int Hkv, int hd, int C, int64_t t0, double theta,
                                 double* out) {
  double x[512], y[512];
  for (int h = 0; h < Hkv; ++h) {
    for (int j = 0; j < hd; ++j) out[h * hd + j] = 0.0;
    for (int i = 0; i < C; ++i) {
      for (int j = 0; j < hd; ++j) x[j] = (double)K[i * ldk + h * hd + j];
      xo_rope(x, y, hd, (double)(t0 + i), theta);
      for (int j = 0; j < hd; ++j) out[h * hd + j] += y[j];
    }
    for (int j = 0; j < hd; ++j) out[h * hd + j] /= (double)C;
  }
}
