/*
 * xkv.h -- C ABI of the B200 (sm_100a) xKV hot path.
 *
 * The library computes, on one GPU, the two halves of xKV:
 *   - prefill-time cross-layer factorisation of a group of G adjacent layers
 *     (Gram -> top-r subspace -> shared basis A and per-layer B_l) and KV-CoRE's
 *     normalised effective rank from the same Gram;
 *   - decode-time Selective Reconstruction (SR) attention: landmark-guided top-k
 *     chunk selection, reconstruction of only the selected rows, RoPE, and
 *     online-softmax GQA attention over them plus a raw sink/recent window;
 *     and its xK-SR mode, where only the keys are compressed and the selected
 *     rows' values are read from the uncompressed cache.
 *
 * Sources (page title -- section):
 *   [xKV-blog] "xKV大模型压缩秘籍：跨层共享，小白也能轻松上手，收藏必备！" --
 *              "xKV 到底做了什么？" and "仅仅压缩还不够，xKV 还做了“选择性重建”";
 *              Fig. 6 (full reconstruction vs selective reconstruction).
 *   [xKV-abs]  "xKV: Cross-Layer KV-Cache Compression via Aligned Singular Vector
 *              Extraction" -- abstract.
 *   [KV-CoRE]  "KV-CoRE: Benchmarking Data-Dependent Low-Rank Compressibility of
 *              KV-Caches in LLMs" -- 2.A (incremental covariance), 2.B (NER).
 *   [KQ-SVD]   "KQ-SVD: KV cache compression with provable guarantees on attention
 *              fidelity" -- 3.2 (decode attention), 3.3 (truncated SVD).
 *
 * Conventions shared by every call:
 *   - Every data pointer is a DEVICE pointer owned by the caller, 16-byte
 *     aligned; the library never allocates device memory.  Scratch space is a
 *     caller-provided `workspace` whose size the matching *_workspace_size()
 *     call reports (256-byte alignment required).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls only
 *     enqueue work; they return before the GPU finishes.
 *   - Matrices are row-major; sizes are in elements.  bf16 data is IEEE
 *     bfloat16; f32 data is IEEE binary32.  Outputs of attention are f32.
 *   - Errors: each call returns an xkv_status.  On XKV_ERR_INVALID_ARG /
 *     XKV_ERR_UNSUPPORTED / XKV_ERR_WORKSPACE nothing was launched and nothing
 *     was written.  XKV_ERR_CUDA means a launch or runtime call failed.  Errors
 *     detected on the device (a bounded wait that expired, a non-finite or
 *     non-positive pivot) are recorded in a per-device status word that
 *     xkv_get_device_status() returns and clears.  No C++ exception crosses
 *     this interface.
 *   - Compressed-cache layout: A is T x r per (batch, group); B_l is stored
 *     TRANSPOSED, Bt_l = d x r (row c holds the r coefficients of output column
 *     c), which for layer l of a group equals rows l d .. l d + d - 1 of V_r.
 *   - RoPE is rotate-half: pairs (j, j + hd/2) turn by pos * theta^(-2j/hd).
 *     Token t of the cache sits at position t; the decode query sits at T.
 */
#ifndef XKV_H_
#define XKV_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define XKV_API __attribute__((visibility("default")))
#else
#define XKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum xkv_status {
  XKV_OK = 0,
  XKV_ERR_INVALID_ARG = 1,    /* null pointer, misalignment, inconsistent sizes */
  XKV_ERR_UNSUPPORTED = 2,    /* valid request outside what this build implements */
  XKV_ERR_WORKSPACE = 3,      /* workspace missing or smaller than required */
  XKV_ERR_CUDA = 4,           /* a CUDA runtime/driver call failed */
  XKV_ERR_NUMERICAL = 5,      /* device detected a numerical breakdown */
  XKV_ERR_DEVICE_TIMEOUT = 6  /* a bounded device-side wait expired */
} xkv_status;

typedef enum xkv_dtype { XKV_F32 = 0, XKV_BF16 = 1 } xkv_dtype;

/* Static description of a status code (never NULL). */
XKV_API const char* xkv_status_string(xkv_status status);

/* Library ABI version: (major << 16) | minor. */
XKV_API int xkv_version(void);

/* Synchronises `stream`, then returns and clears the calling device's deferred
 * status word (XKV_OK if no device-side error was recorded).  The word is
 * taken out and reset to zero in one atomic device operation, so a code that
 * a kernel on another stream records meanwhile is kept for the next call.
 * Concurrent calls from several host threads for the same device share one
 * small device slot for the value taken out; serialise them. */
XKV_API xkv_status xkv_get_device_status(void* stream);

/* ------------------------------------------------------------------ Gram */
/* [KV-CoRE] 2.A incremental covariance over the horizontal concatenation of
 * [xKV-blog] "xKV 到底做了什么":  C += X^T X,  X = [X_1 | ... | X_G] (rows x G d).
 *   X_layers : host array of G device pointers; X_layers[l] is rows x d with row
 *              stride ldx (elements, >= d, multiple of 8).
 *   C        : (G d) x (G d) f32, accumulated in place (zero it before the first
 *              shard).  Both triangles are written.
 *   d must be a multiple of 64.  Workspace: xkv_gram_workspace_size(). */
XKV_API xkv_status xkv_gram_workspace_size(int G, int64_t rows, int d, xkv_dtype dt, size_t* bytes);
XKV_API xkv_status xkv_gram_accumulate(const void* const* X_layers, int G, int64_t rows, int d, int64_t ldx,
                               xkv_dtype dt, float* C, void* workspace, size_t ws_bytes, void* stream);

/* --------------------------------------------------------- compression */
/* Cross-layer factorisation of one group ([xKV-blog] "xKV 到底做了什么",
 * [xKV-abs]; optimality of the truncation: [KQ-SVD] 3.3):
 *   1. C = X^T X accumulated over token shards of `shard_rows` rows;
 *   2. top-r subspace of C: `iters` block subspace iterations Y = C Q, Q = qr(Y)
 *      with block width b = min(rank + oversample, G d, T), started from a
 *      Gaussian block drawn from `seed`; then Rayleigh-Ritz: H = Q^T C Q,
 *      H = U diag(lambda) U^T, V_r = Q U[:, 1..rank];
 *   3. A = X V_r (T x rank) and Bt = V_r ((G d) x rank; layer l = rows l d..).
 * Arguments: X_layers as for xkv_gram_accumulate (T rows each); A (T x rank) and
 * Bt (G d x rank) in `dt`; eigvals (rank f32, descending Ritz values) and
 * gram_out ((G d)^2 f32, the full Gram, e.g. for xkv_ner) may be NULL.
 * Requires d % 64 == 0, rank % 16 == 0, 1 <= rank <= min(T, G d), iters >= 1
 * (XKV_ERR_INVALID_ARG otherwise); a bf16 group also needs rank % 64 == 0 (the
 * tensor-core projection), and the block width b may not exceed 3584 (the
 * widest block the factorisation is built for: the Rayleigh-Ritz Jacobi's
 * b / 32 pair CTAs then still run as one cooperative launch), else
 * XKV_ERR_UNSUPPORTED.  At most G = 8 layers. */
XKV_API xkv_status xkv_compress_workspace_size(int G, int64_t T, int d, int rank, int oversample,
                                       int64_t shard_rows, xkv_dtype dt, size_t* bytes);
XKV_API xkv_status xkv_compress_group(const void* const* X_layers, int G, int64_t T, int d, int64_t ldx,
                              xkv_dtype dt, int rank, int iters, int oversample, int64_t shard_rows,
                              uint64_t seed, void* A, void* Bt, float* eigvals, float* gram_out,
                              void* workspace, size_t ws_bytes, void* stream);

/* The two halves of xkv_compress_group, for callers that accumulate the Gram
 * themselves (e.g. over token shards held by several GPUs, whose partial Grams
 * are summed by an all-reduce, [KV-CoRE] 2.A) or that project rows onto an
 * existing basis (e.g. a chunk of generated tokens leaving the raw window).
 *
 * xkv_factor_gram: steps 2 of xkv_compress_group on a given Gram.
 *   gram    : (G d) x (G d) f32, the uncentred Gram of `rows` token rows
 *             (rows only caps the block width: b = min(rank + oversample, G d,
 *             rows)).
 *   Bt      : (G d) x rank in `dt`, the stored basis V_r.
 *   Vr_out  : (G d) x rank f32 copy of V_r (may be NULL).
 *   eigvals : rank f32 Ritz values, descending (may be NULL).
 *   Same seed and Gram give the same bits, so ranks that factor one summed
 *   Gram obtain one basis.  Argument rules as for xkv_compress_group.
 *
 * xkv_project: A = X V for X = [X_1 | ... | X_G] (T x G d through the layer
 *   pointers, as for xkv_gram_accumulate) and V ((G d) x rank) in v_dtype:
 *   an f32 basis enters the bf16 tensor-core product as a bf16 hi/lo pair,
 *   a bf16 basis (e.g. a stored Bt) as is.  A is T x rank in `dt` with row
 *   stride lda (elements; a multiple of 8 for bf16).  bf16 caches need
 *   rank % 64 == 0; f32 caches need an f32 basis (XKV_ERR_UNSUPPORTED
 *   otherwise).  Workspace: xkv_project_workspace_size (bf16 caches only). */
XKV_API xkv_status xkv_factor_workspace_size(int G, int d, int64_t rows, int rank, int oversample, xkv_dtype dt,
                                     size_t* bytes);
XKV_API xkv_status xkv_factor_gram(const float* gram, int G, int d, int64_t rows, xkv_dtype dt, int rank,
                           int iters, int oversample, uint64_t seed, void* Bt, float* Vr_out,
                           float* eigvals, void* workspace, size_t ws_bytes, void* stream);
XKV_API xkv_status xkv_project_workspace_size(int G, int d, int rank, size_t* bytes);
XKV_API xkv_status xkv_project(const void* const* X_layers, int G, int64_t T, int d, int64_t ldx, xkv_dtype dt,
                       const void* V, xkv_dtype v_dtype, int rank, void* A, int64_t lda, void* workspace,
                       size_t ws_bytes, void* stream);

/* ------------------------------------------------------------ landmarks */
/* Chunk landmarks for the top-k selector of [xKV-blog] "选择性重建": for KV head
 * h and middle chunk c (tokens sink + c chunk .. sink + (c+1) chunk - 1),
 *   landmark[h][c] = mean over the chunk of RoPE_t(K[t, h hd : (h+1) hd]).
 *   K         : T x (n_kv_heads head_dim) pre-RoPE keys, row stride ldk.
 *   landmarks : [n_kv_heads][n_mid][head_dim] in `dt`, n_mid = (T-sink-recent)/chunk.
 * Requires (T - sink - recent) % chunk == 0 and head_dim even. */
XKV_API xkv_status xkv_build_landmarks(const void* K, int64_t T, int64_t ldk, int n_kv_heads, int head_dim,
                               xkv_dtype dt, int chunk, int sink, int recent, float rope_theta,
                               void* landmarks, void* stream);

/* ------------------------------------------------------------ SR decode */
typedef struct xkv_sr_params {
  int batch;              /* B */
  int n_q_heads;          /* Hq (multiple of n_kv_heads) */
  int n_kv_heads;         /* Hkv */
  int head_dim;           /* hd (even) */
  int64_t T;              /* cached tokens; the query sits at position T */
  int rank_k, rank_v;     /* columns of A_K, A_V */
  int chunk;              /* tokens per chunk */
  int topk;               /* chunks kept per (batch, KV head), <= n_mid and <= 1024;
                             n_mid = (T - sink - recent) / chunk <= 24576 */
  int sink, recent;       /* raw windows [0, sink) and [T - recent, T) */
  float rope_theta;
  xkv_dtype dtype;        /* of q, A, Bt, landmarks, sink/recent */
  int64_t a_k_batch_stride, a_v_batch_stride;   /* elements between batches of A_K / A_V */
  int64_t bt_k_batch_stride, bt_v_batch_stride; /* elements between batches of Bt_K / Bt_V;
                                                   0 = one Bt shared by the batch */
  int64_t window_batch_stride; /* elements between sequences of sr_K / sr_V; 0 = (sink + recent) d.
                                  A window buffer with room for recent + chunk rows (multi-step
                                  decode, xkv_sr_append) passes (sink + recent + chunk) d. */
  int64_t landmark_capacity;   /* chunks allocated per (sequence, KV head) in landmarks; 0 = n_mid */
} xkv_sr_params;

/* One decode step of xKV-SR for one layer ([xKV-blog] "选择性重建", [xKV-abs];
 * attention as in [KQ-SVD] 3.2), for every (batch b, KV head h):
 *   s_c = sum_{g in group(h)} q_g . landmark[b][h][c]; keep the top-k chunks
 *   (ties -> lower c; sel_out ascending);  rebuild rows t of the kept chunks:
 *   K_t = RoPE_t(A_K[b][t] Bt_K[h hd : (h+1) hd]^T),  V_t = A_V[b][t] Bt_V[...]^T;
 *   o_g = softmax(q_g K^T / sqrt(hd)) V over sink, kept and recent rows.
 *   q         : [B][Hq][hd] post-RoPE queries (query head j uses KV head j/(Hq/Hkv)).
 *   A_K, A_V  : [B][T][rank] (batch strides in params).   Bt_K, Bt_V : [d][rank] per
 *               batch element (batch strides in params; each sequence has its own
 *               factorisation, or 0 to share one).
 *   landmarks : [B][Hkv][cap][hd], cap = landmark_capacity (or n_mid); chunk c < n_mid
 *               of (b, h) at [b][h][c].   sr_K, sr_V : [B][rows][d] with batch stride
 *               window_batch_stride; row i < sink is token i, row sink + i is token
 *               T - recent + i; keys pre-RoPE.
 *   out       : [B][Hq][hd] f32.   sel_out : [B][Hkv][topk] int32, or NULL. */
XKV_API xkv_status xkv_sr_workspace_size(const xkv_sr_params* p, size_t* bytes);
XKV_API xkv_status xkv_sr_attention_decode(const xkv_sr_params* p, const void* q, const void* A_K,
                                   const void* Bt_K, const void* A_V, const void* Bt_V,
                                   const void* landmarks, const void* sr_K, const void* sr_V,
                                   float* out, int32_t* sel_out, void* workspace, size_t ws_bytes,
                                   void* stream);

/* The same decode step without a caller workspace (an interface convenience;
 * the pages have no counterpart).  Its scratch is a fixed device array of
 * XKV_SR_STATIC_SCRATCH_BYTES inside the loaded library, so the call performs
 * no device allocation of any kind; it serves callers that cannot allocate or
 * hold a workspace, e.g. a plain C host program without a device allocator of
 * its own, or a decode loop that must run under a fixed memory budget.
 *   - Requests whose scratch (xkv_sr_workspace_size) exceeds the array return
 *     XKV_ERR_UNSUPPORTED and launch nothing.
 *   - The array's device address is looked up once per device and CUDA
 *     context, on the first call made with that device current (after
 *     cudaDeviceReset the new context's module is looked up afresh); make that
 *     first call before any stream capture that includes this entry point.
 *   - Nothing in the scratch needs to start at zero: every word the kernels
 *     read is written earlier in the same call.
 *   - Every call on a device shares the one array: calls that overlap in time
 *     (on different streams or from different host threads) race on it and
 *     corrupt each other's results.  Order them, e.g. on one stream.
 * Arguments, layouts and errors are otherwise those of xkv_sr_attention_decode. */
#define XKV_SR_STATIC_SCRATCH_BYTES (8u << 20)
XKV_API xkv_status xkv_sr_attention_decode_noalloc(const xkv_sr_params* p, const void* q, const void* A_K,
                                           const void* Bt_K, const void* A_V, const void* Bt_V,
                                           const void* landmarks, const void* sr_K, const void* sr_V,
                                           float* out, int32_t* sel_out, void* stream);

/* One decode step of the xK-SR mode ([xKV-blog] "选择性重建": only the keys are
 * compressed; the values stay whole).  Chunk scores, the exact top-k and the
 * key rows K_t = RoPE_t(A_K[b][t] Bt_K[h hd : (h+1) hd]^T) are those of
 * xkv_sr_attention_decode; the value of a kept row t is read from the
 * uncompressed cache, V_t = V[b][t][h hd : (h+1) hd].
 *   V         : [B][T][d] in p->dtype, 16-byte aligned; p->a_v_batch_stride is its
 *               batch stride in elements (>= T d).  p->rank_v and
 *               p->bt_v_batch_stride are ignored.
 *   workspace : at least xkv_xk_sr_workspace_size bytes, 256-byte aligned.
 * Every other argument, layout and error is that of xkv_sr_attention_decode. */
XKV_API xkv_status xkv_xk_sr_workspace_size(const xkv_sr_params* p, size_t* bytes);
XKV_API xkv_status xkv_xk_sr_attention_decode(const xkv_sr_params* p, const void* q, const void* A_K,
                                              const void* Bt_K, const void* V, const void* landmarks,
                                              const void* sr_K, const void* sr_V, float* out, int32_t* sel_out,
                                              void* workspace, size_t ws_bytes, void* stream);

/* Failure-detection self-test (the pages have no counterpart).  Launches one
 * CTA whose mbarrier wait nothing ever completes, through the same bounded wait
 * every kernel of the library uses: after its limit (about one second) the
 * wait gives up, records XKV_ERR_DEVICE_TIMEOUT in the device status word and
 * the kernel returns, leaving the context usable.  Returns the launch status;
 * xkv_get_device_status(stream) then reports (and clears) the timeout. */
XKV_API xkv_status xkv_selftest_expired_wait(void* stream);

/* Stage timing (measurement aid; the method has no counterpart).  While
 * enabled, every xkv_sr_attention_decode call records CUDA events on its
 * stream around its four launches: chunk scores, top-k (+ raw window
 * partials), selective reconstruction + attention partials, combine.
 * xkv_sr_profile_read waits for the most recent call's last event and writes
 * the four durations in milliseconds to stage_ms[0..3].  The events belong to
 * the device current at enable time; calls on another device are not timed.
 * Not for use while a stream is being captured.  Process-wide state, not
 * thread-safe.  Errors: XKV_ERR_CUDA (event creation or query failed),
 * XKV_ERR_INVALID_ARG (stage_ms NULL, or nothing recorded yet). */
XKV_API xkv_status xkv_sr_profile_enable(int enable);
XKV_API xkv_status xkv_sr_profile_read(float* stage_ms);

/* ---------------------------------------------------- multi-step decode */
/* Appends one generated token per layer of a group to the raw recent window
 * and, when the window then holds recent + chunk rows, rolls its oldest chunk
 * into the compressed cache.  [xKV-blog] (the editor's note after
 * "仅仅压缩还不够，xKV 还做了“选择性重建”") compresses only the long prefill;
 * here tokens generated afterwards stay raw until a chunk of them is complete,
 * then join the compressed cache exactly as prefill tokens did:
 *   - A_K / A_V rows of the chunk = x V on the group's stored bases Bt_K / Bt_V
 *     (x = the chunk's rows of all G layers side by side, [xKV-blog]
 *     "xKV 到底做了什么"), rounded to the cache dtype;
 *   - landmark[l][b][h][n_mid] = mean over the chunk of RoPE_t(K_l[t, h]) at
 *     the tokens' absolute positions ([xKV-blog] "选择性重建");
 *   - the window moves down by one chunk.
 * The state is a function of the length T before the call: with
 * n0 = T - sink - recent, the window holds w = recent + n0 % chunk rows after
 * the sink rows, n_mid = n0 / chunk chunks are compressed, and the new token
 * goes to window row sink + w.  A decode at length T passes recent = w and
 * the strides below in xkv_sr_params.
 *   k_new, v_new : host arrays of G device pointers, each [B][d] (keys pre-RoPE).
 *   win_K, win_V : host arrays of G device pointers, each [B][rows][d], rows >=
 *                  sink + recent + chunk, batch stride window_batch_stride.
 *   Bt_K, Bt_V   : group bases [B][G d][rank] (batch strides; 0 = shared), the
 *                  Bt that xkv_compress_group returned; layer l owns rows l d...
 *   A_K, A_V     : [B][capacity][rank] (batch strides >= (T + 1) rank).
 *   landmarks    : host array of G device pointers, each [B][Hkv][cap][hd],
 *                  cap = landmark_capacity >= n_mid + 1.
 *   rolled       : host int, set to 1 when a chunk was rolled (may be NULL).
 * bf16 caches need d % 64 == 0 and ranks % 64 == 0; f32 caches use CUDA cores.
 * Workspace: xkv_sr_append_workspace_size.  Calls are stream-ordered; a decode
 * of any layer of the group after the call sees the new state. */
typedef struct xkv_append_params {
  int batch;                   /* B */
  int group;                   /* G <= 8 */
  int n_kv_heads, head_dim;    /* d = n_kv_heads head_dim */
  int chunk, sink, recent;
  float rope_theta;
  xkv_dtype dtype;
  int64_t T;                   /* tokens cached before this append, >= sink + recent */
  int rank_k, rank_v;
  int64_t a_k_batch_stride, a_v_batch_stride;
  int64_t bt_k_batch_stride, bt_v_batch_stride;
  int64_t window_batch_stride; /* elements, >= (sink + recent + chunk) d, multiple of 8 */
  int64_t landmark_capacity;   /* chunks per (sequence, KV head) */
} xkv_append_params;
XKV_API xkv_status xkv_sr_append_workspace_size(const xkv_append_params* p, size_t* bytes);
XKV_API xkv_status xkv_sr_append(const xkv_append_params* p, const void* const* k_new, const void* const* v_new,
                         void* const* win_K, void* const* win_V, const void* Bt_K, const void* Bt_V,
                         void* A_K, void* A_V, void* const* landmarks, int* rolled, void* workspace,
                         size_t ws_bytes, void* stream);

/* The xK-SR step with the uncompressed values in host memory, where the
 * explainer ([xKV-blog] "选择性重建") keeps them: scores, the exact top-k and
 * the rebuilt keys are those of xkv_xk_sr_attention_decode; then, for every
 * (sequence b, KV head h), the kept chunks' rows of head h's columns are read
 * from V_host over the host link into a device staging buffer (only those
 * k chunk rows cross, never the whole cache), and attention proceeds as in
 * the HBM-resident mode.
 *   V_host    : [B][T][d] in p->dtype, page-locked host memory mapped for the
 *               device (e.g. cudaHostAlloc / cudaHostRegister), 16-byte
 *               aligned, batch stride p->a_v_batch_stride; anything else
 *               (device or pageable memory) returns XKV_ERR_INVALID_ARG.
 *   workspace : xkv_xk_sr_host_workspace_size bytes (the SR scratch plus the
 *               staging buffer, B Hkv k chunk hd elements).
 * head_dim times the element size must be a multiple of 16 bytes.  Every other
 * argument, layout and error is that of xkv_xk_sr_attention_decode. */
XKV_API xkv_status xkv_xk_sr_host_workspace_size(const xkv_sr_params* p, size_t* bytes);
XKV_API xkv_status xkv_xk_sr_attention_decode_host_values(const xkv_sr_params* p, const void* q, const void* A_K,
                                                  const void* Bt_K, const void* V_host, const void* landmarks,
                                                  const void* sr_K, const void* sr_V, float* out,
                                                  int32_t* sel_out, void* workspace, size_t ws_bytes,
                                                  void* stream);

/* --------------------------------------------------- token sharding */
/* The path split over devices by tokens.  Prefill: [KV-CoRE] 2.A accumulates
 * the covariance over streamed token rows, so per-device Grams add up: each
 * device runs xkv_gram_accumulate on its rows, an all-reduce sums the Grams,
 * every device runs xkv_factor_gram on the sum (same Gram and seed, same
 * basis) and xkv_project on its own rows.  Decode: each device holds a
 * contiguous slice of the token sequence (the sink on the first, the recent
 * window on the last, whole middle chunks in between); per step
 *   1. xkv_sr_scores   : chunk scores of the local middle chunks;
 *   2. (all-gather of the scores, laid out chunk-major per (b, h))
 *      xkv_sr_topk     : the exact top-k over all chunks, the same on every
 *                        device ([xKV-blog] "选择性重建");
 *   3. xkv_sr_attention_partial : attention over the kept chunks that are held
 *                        here plus the local window rows, as a partial
 *                        (o normalised by its own softmax sum L, and M);
 *   4. (all-gather of the partials) xkv_merge_partials : the exact softmax
 *                        combination of the partials.
 * One device with the whole sequence gives xkv_sr_attention_decode's result. */
typedef struct xkv_sr_shard {
  int64_t position_offset; /* global position of local token row 0 */
  int64_t chunk_begin;     /* global index of the first middle chunk held here */
} xkv_sr_shard;

/* Chunk scores s_c = sum_{g in group(h)} q_g . landmark[b][h][c] of the local
 * middle chunks (n_mid = (T - sink - recent) / chunk of p); scores is
 * [B][Hkv] rows of n_mid f32 with row stride ld (>= n_mid, multiple of 4). */
XKV_API xkv_status xkv_sr_scores(const xkv_sr_params* p, const void* q, const void* landmarks, float* scores,
                         int64_t ld, void* stream);
/* Exact top-k of each of `rows` score rows of n entries (row stride ld, a
 * multiple of 4, >= n): the k largest, ties to the lower index, ascending.
 * n <= 24576, 1 <= k <= min(n, 1024). */
XKV_API xkv_status xkv_sr_topk(const float* scores, int64_t ld, int rows, int64_t n, int k, int32_t* sel_out,
                       void* stream);
/* Attention of one device's token slice for a given selection.  p describes
 * the local slice (T local rows, its own sink / recent rows, topk = the global
 * k); sel [B][Hkv][topk] holds global chunk indices, of which those in
 * [chunk_begin, chunk_begin + n_mid) are attended here (row sink + (c -
 * chunk_begin) chunk, RoPE at position_offset + row).  out [B][Hq][hd] is the
 * partial normalised by its own sum L; ml_out [B][Hq][2] = (M, L), M the
 * running maximum of the scores scaled by log2(e)/sqrt(hd), (-inf, 0) when
 * nothing is held here.  Workspace: xkv_sr_partial_workspace_size. */
XKV_API xkv_status xkv_sr_partial_workspace_size(const xkv_sr_params* p, size_t* bytes);
XKV_API xkv_status xkv_sr_attention_partial(const xkv_sr_params* p, const xkv_sr_shard* shard, const int32_t* sel,
                                    const void* q, const void* A_K, const void* Bt_K, const void* A_V,
                                    const void* Bt_V, const void* sr_K, const void* sr_V, float* out,
                                    float* ml_out, void* workspace, size_t ws_bytes, void* stream);
/* out[i] = sum_r 2^(M_ri - M_i) L_ri o_ri / sum_r 2^(M_ri - M_i) L_ri over R
 * partials (o [R][rows][hd], ml [R][rows][2]); rows = B Hq. */
XKV_API xkv_status xkv_merge_partials(const float* o, const float* ml, int R, int rows, int hd, float* out,
                              void* stream);

/* -------------------------------------------------- full reconstruction */
/* The comparison path of [xKV-blog] Fig. 6: rebuild every row,
 *   out[t][c] = sum_i A[t][i] Bt[c][i]   (T x d, `dt`),
 * then, if apply_rope, RoPE per head at position t.  A is T x rank, Bt d x rank.
 * Requires rank % 16 == 0 and d % head_dim == 0. */
XKV_API xkv_status xkv_full_reconstruct(const void* A, const void* Bt, int64_t T, int rank, int d,
                                int n_kv_heads, int head_dim, int apply_rope, float rope_theta,
                                xkv_dtype dt, void* out, void* stream);

/* Dense decode attention over a full cache ([KQ-SVD] 3.2), the second half of
 * the comparison path:  o_g = softmax(q_g K^T / sqrt(hd)) V over all T rows.
 *   q [B][Hq][hd], K (post-RoPE) and V [B][T][d] in `dtype`, out [B][Hq][hd] f32. */
typedef struct xkv_dense_params {
  int batch, n_q_heads, n_kv_heads, head_dim;
  int64_t T;
  xkv_dtype dtype;
} xkv_dense_params;
XKV_API xkv_status xkv_dense_workspace_size(const xkv_dense_params* p, size_t* bytes);
XKV_API xkv_status xkv_dense_attention_decode(const xkv_dense_params* p, const void* q, const void* K,
                                      const void* V, float* out, void* workspace, size_t ws_bytes,
                                      void* stream);

/* ------------------------------------------------------------------ NER */
/* [KV-CoRE] 2.B per diagonal block C_ll (block x block) of an n x n f32 Gram:
 * eigenvalues lambda, numerical rank r = #{lambda_i > rank_rel_tol lambda_max},
 * sigma_i = sqrt(lambda_i) over those r, p_i = sigma_i / sum sigma,
 * erank = exp(-sum p_i ln p_i), NER = erank / r (in [1/r, 1]).  A block with
 * lambda_max <= 0 reports rank 0, erank 0, NER 0.
 *   ner_out [n/block] f32; erank_out [n/block] f32 or NULL; rank_out [n/block]
 *   int32 or NULL.  Requires n % block == 0, block even. */
XKV_API xkv_status xkv_ner_workspace_size(int n, int block, size_t* bytes);
XKV_API xkv_status xkv_ner(const float* gram, int n, int block, double rank_rel_tol, float* ner_out,
                   float* erank_out, int32_t* rank_out, void* workspace, size_t ws_bytes,
                   void* stream);

/* Energy rank per diagonal block ([xKV-blog] Fig. 2(c): the rank that keeps a
 * given share of a layer's cache energy).  Eigenvalues lambda of C_ll, with
 * values below zero (rounding only) counted as 0, sorted descending; rank =
 * the smallest k with lambda_1 + ... + lambda_k >= energy * sum_i lambda_i, or
 * 0 for a zero block.
 *   rank_out [n/block] int32; lambda_out [n/block][block] f32 descending, or NULL.
 *   energy in (0, 1]; n % block == 0, block even and <= 8192 (else
 *   XKV_ERR_UNSUPPORTED).  Workspace: xkv_ner_workspace_size(n, block). */
XKV_API xkv_status xkv_energy_rank(const float* gram, int n, int block, double energy, int32_t* rank_out,
                                   float* lambda_out, void* workspace, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* XKV_H_ */
