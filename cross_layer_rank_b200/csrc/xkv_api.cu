// C-ABI entry points of libxkv (declared in include/xkv.h): argument
// validation (nothing is launched on a bad argument), workspace sizing, TMA
// descriptor creation and the per-device status word.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "xkv_common.cuh"
#include "xkv_internal.h"

namespace xkv {

static __device__ int g_device_status;
// Where xkv_get_device_status's exchange kernel leaves the value it took out.
static __device__ int g_device_status_taken;

// Scratch of xkv_sr_attention_decode_noalloc: a fixed device array that is part
// of the loaded module, so that entry point never allocates.
static __device__ __align__(256) unsigned char g_sr_static_scratch[XKV_SR_STATIC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
int g_sms[kMaxDevices] = {0};
std::mutex g_mu;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CtxGetCurrentFn g_ctx_current = nullptr;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

// Device addresses of the module's __device__ symbols, looked up with
// cudaGetSymbolAddress once per (device, context) with that device current.
// A context created after cudaDeviceReset holds a freshly loaded module, so
// the addresses are looked up again for it.
struct SymbolCache {
  CUcontext ctx = nullptr;
  bool valid = false;
  int* status = nullptr;
  int* status_taken = nullptr;
  void* scratch = nullptr;
};
SymbolCache g_sym[kMaxDevices];

const SymbolCache* symbols() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_ctx_current) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return nullptr;
    g_ctx_current = reinterpret_cast<CtxGetCurrentFn>(fn);
  }
  // no context is current before the runtime's first call on this thread
  CUcontext ctx = nullptr;
  if (g_ctx_current(&ctx) != CUDA_SUCCESS) return nullptr;
  SymbolCache& c = g_sym[dev];
  if (!ctx || !c.valid || c.ctx != ctx) {
    void* a = nullptr;
    void* b = nullptr;
    void* sc = nullptr;
    // (the first lookup also makes the device's primary context current)
    if (cudaGetSymbolAddress(&a, g_device_status) != cudaSuccess ||
        cudaGetSymbolAddress(&b, g_device_status_taken) != cudaSuccess ||
        cudaGetSymbolAddress(&sc, g_sr_static_scratch) != cudaSuccess)
      return nullptr;
    if (g_ctx_current(&ctx) != CUDA_SUCCESS || !ctx) return nullptr;
    c.status = static_cast<int*>(a);
    c.status_taken = static_cast<int*>(b);
    c.scratch = sc;
    c.ctx = ctx;
    c.valid = true;
  }
  return &c;
}
}  // namespace

int* device_status_ptr() {
  const SymbolCache* c = symbols();
  return c ? c->status : nullptr;
}

// Device address of g_sr_static_scratch on the current device and context.
void* static_scratch_ptr() {
  const SymbolCache* c = symbols();
  return c ? c->scratch : nullptr;
}

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  if (!g_sms[dev]) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    g_sms[dev] = v;
  }
  return g_sms[dev];
}

bool force_simt() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("XKV_FORCE_SIMT");
    v = (e && e[0] == '1') ? 1 : 0;
  }
  return v == 1;
}

bool make_tmap(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
               const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return false;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
  }
  cuuint64_t d[5];
  cuuint64_t s[4];
  cuuint32_t b[5], e[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    e[i] = 1;
    if (i + 1 < rank) s[i] = strides_bytes[i];
  }
  const CUresult r = g_encode(map, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), d, s, b, e,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace xkv

using namespace xkv;

extern "C" {

const char* xkv_status_string(xkv_status s) {
  switch (s) {
    case XKV_OK: return "ok";
    case XKV_ERR_INVALID_ARG: return "invalid argument";
    case XKV_ERR_UNSUPPORTED: return "unsupported configuration";
    case XKV_ERR_WORKSPACE: return "workspace missing or too small";
    case XKV_ERR_CUDA: return "CUDA error";
    case XKV_ERR_NUMERICAL: return "numerical breakdown detected on the device";
    case XKV_ERR_DEVICE_TIMEOUT: return "bounded device-side wait expired";
  }
  return "unknown status";
}

int xkv_version(void) { return (1 << 16) | 0; }

// Takes the status word out and leaves 0 in one atomic step, so that a code
// recorded by a kernel on another stream is either returned now or kept for
// the next call, never lost between a read and a clear.
__global__ void take_status_kernel(int* status, int* taken) { *taken = atomicExch(status, 0); }

xkv_status xkv_get_device_status(void* stream) {
  const SymbolCache* c = symbols();
  if (!c) return XKV_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return XKV_ERR_CUDA;
  take_status_kernel<<<1, 1, 0, st>>>(c->status, c->status_taken);
  if (cudaPeekAtLastError() != cudaSuccess) return XKV_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyAsync(&v, c->status_taken, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return XKV_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return XKV_ERR_CUDA;
  return static_cast<xkv_status>(v);
}

// ------------------------------------------------ bounded-wait self-test
// One CTA waits on an mbarrier that nothing completes: mbar_wait gives up
// after kWaitLimitNs, records kDevTimeout and the kernel returns.
__global__ void selftest_expired_wait_kernel(int* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, status);
  __syncthreads();
}

xkv_status xkv_selftest_expired_wait(void* stream) {
  int* status = device_status_ptr();
  if (!status) return XKV_ERR_CUDA;
  selftest_expired_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status);
  return cudaPeekAtLastError() == cudaSuccess ? XKV_OK : XKV_ERR_CUDA;
}

// ------------------------------------------------------------------- Gram
static xkv_status check_layers(const void* const* X, int G, int d, int64_t ldx, xkv_dtype dt) {
  if (!X || G < 1 || G > 8 || d < 64 || d % 64 != 0 || ldx < d || ldx % 8 != 0) return XKV_ERR_INVALID_ARG;
  if (dt != XKV_F32 && dt != XKV_BF16) return XKV_ERR_INVALID_ARG;
  for (int l = 0; l < G; ++l)
    if (!X[l] || !aligned16(X[l])) return XKV_ERR_INVALID_ARG;
  return XKV_OK;
}

xkv_status xkv_gram_workspace_size(int G, int64_t rows, int d, xkv_dtype dt, size_t* bytes) {
  if (!bytes || G < 1 || G > 8 || d < 64 || d % 64 != 0 || rows < 0) return XKV_ERR_INVALID_ARG;
  *bytes = gram_workspace(G, rows, d, dt);
  return XKV_OK;
}

xkv_status xkv_gram_accumulate(const void* const* X_layers, int G, int64_t rows, int d, int64_t ldx, xkv_dtype dt,
                               float* C, void* workspace, size_t ws_bytes, void* stream) {
  xkv_status s = check_layers(X_layers, G, d, ldx, dt);
  if (s != XKV_OK) return s;
  if (!C || !aligned16(C) || rows < 0) return XKV_ERR_INVALID_ARG;
  const size_t need = gram_workspace(G, rows, d, dt);
  if (need > kAlign && (!workspace || ws_bytes < need || !aligned256(workspace))) return XKV_ERR_WORKSPACE;
  return gram_launch(X_layers, G, rows, d, ldx, dt, C, workspace, static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------ compression
static xkv_status check_compress(int G, int64_t T, int d, int rank, int iters, int oversample, int64_t shard_rows,
                                 xkv_dtype dt) {
  if (G < 1 || G > 8 || T < 1 || d < 64 || d % 64 != 0 || rank < 1 || rank % 16 != 0 || iters < 1 ||
      oversample < 0 || shard_rows < 0 || T > (int64_t(1) << 31) - 1)
    return XKV_ERR_INVALID_ARG;
  if (rank > G * d || rank > T) return XKV_ERR_INVALID_ARG;
  if (dt != XKV_F32 && dt != XKV_BF16) return XKV_ERR_INVALID_ARG;
  if (dt == XKV_BF16 && rank % 64 != 0) return XKV_ERR_UNSUPPORTED;
  // block width of the subspace iteration: the widest the factorisation is
  // built for (the Rayleigh-Ritz Jacobi's b / 32 pair CTAs in one cooperative
  // launch)
  const int64_t b = std::min<int64_t>(std::min<int64_t>(static_cast<int64_t>(rank) + oversample, int64_t(G) * d), T);
  if (b > 3584) return XKV_ERR_UNSUPPORTED;
  return XKV_OK;
}

xkv_status xkv_compress_workspace_size(int G, int64_t T, int d, int rank, int oversample, int64_t shard_rows,
                                       xkv_dtype dt, size_t* bytes) {
  if (!bytes) return XKV_ERR_INVALID_ARG;
  xkv_status s = check_compress(G, T, d, rank, 1, oversample, shard_rows, dt);
  if (s != XKV_OK) return s;
  CompressPlan p;
  compress_plan(G, T, d, rank, oversample, shard_rows, dt, &p);
  *bytes = p.bytes;
  return XKV_OK;
}

xkv_status xkv_compress_group(const void* const* X_layers, int G, int64_t T, int d, int64_t ldx, xkv_dtype dt,
                              int rank, int iters, int oversample, int64_t shard_rows, uint64_t seed, void* A, void* Bt,
                              float* eigvals, float* gram_out, void* workspace, size_t ws_bytes, void* stream) {
  xkv_status s = check_compress(G, T, d, rank, iters, oversample, shard_rows, dt);
  if (s != XKV_OK) return s;
  s = check_layers(X_layers, G, d, ldx, dt);
  if (s != XKV_OK) return s;
  if (!A || !Bt || !aligned16(A) || !aligned16(Bt)) return XKV_ERR_INVALID_ARG;
  if ((eigvals && !aligned16(eigvals)) || (gram_out && !aligned16(gram_out))) return XKV_ERR_INVALID_ARG;
  CompressPlan p;
  compress_plan(G, T, d, rank, oversample, shard_rows, dt, &p);
  if (!workspace || ws_bytes < p.bytes || !aligned256(workspace)) return XKV_ERR_WORKSPACE;
  return compress_launch(p, X_layers, G, T, d, ldx, dt, iters, seed, A, Bt, eigvals, gram_out, workspace,
                         static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------- factorisation pieces
static xkv_status check_factor(int G, int d, int64_t rows, int rank, int iters, int oversample, xkv_dtype dt) {
  if (G < 1 || G > 8 || d < 64 || d % 64 != 0 || rows < 1 || rank < 1 || rank % 16 != 0 || iters < 1 ||
      oversample < 0)
    return XKV_ERR_INVALID_ARG;
  if (rank > G * d || rank > rows) return XKV_ERR_INVALID_ARG;
  if (dt != XKV_F32 && dt != XKV_BF16) return XKV_ERR_INVALID_ARG;
  const int64_t b = std::min<int64_t>(std::min<int64_t>(static_cast<int64_t>(rank) + oversample, int64_t(G) * d), rows);
  if (b > 3584) return XKV_ERR_UNSUPPORTED;
  return XKV_OK;
}

xkv_status xkv_factor_workspace_size(int G, int d, int64_t rows, int rank, int oversample, xkv_dtype dt,
                                     size_t* bytes) {
  if (!bytes) return XKV_ERR_INVALID_ARG;
  const xkv_status s = check_factor(G, d, rows, rank, 1, oversample, dt);
  if (s != XKV_OK) return s;
  FactorPlan p;
  factor_plan(G * d, rows, rank, oversample, &p);
  *bytes = p.bytes;
  return XKV_OK;
}

xkv_status xkv_factor_gram(const float* gram, int G, int d, int64_t rows, xkv_dtype dt, int rank, int iters,
                           int oversample, uint64_t seed, void* Bt, float* Vr_out, float* eigvals, void* workspace,
                           size_t ws_bytes, void* stream) {
  const xkv_status s = check_factor(G, d, rows, rank, iters, oversample, dt);
  if (s != XKV_OK) return s;
  if (!gram || !Bt || !aligned16(gram) || !aligned16(Bt)) return XKV_ERR_INVALID_ARG;
  if ((Vr_out && !aligned16(Vr_out)) || (eigvals && !aligned16(eigvals))) return XKV_ERR_INVALID_ARG;
  FactorPlan p;
  factor_plan(G * d, rows, rank, oversample, &p);
  if (!workspace || ws_bytes < p.bytes || !aligned256(workspace)) return XKV_ERR_WORKSPACE;
  return factor_launch(p, gram, dt, iters, seed, Bt, Vr_out, eigvals, workspace, static_cast<cudaStream_t>(stream));
}

xkv_status xkv_project_workspace_size(int G, int d, int rank, size_t* bytes) {
  if (!bytes || G < 1 || G > 8 || d < 64 || d % 64 != 0 || rank < 1) return XKV_ERR_INVALID_ARG;
  *bytes = project_workspace(G * d, rank);
  return XKV_OK;
}

xkv_status xkv_project(const void* const* X_layers, int G, int64_t T, int d, int64_t ldx, xkv_dtype dt,
                       const void* V, xkv_dtype v_dtype, int rank, void* A, int64_t lda, void* workspace,
                       size_t ws_bytes, void* stream) {
  xkv_status s = check_layers(X_layers, G, d, ldx, dt);
  if (s != XKV_OK) return s;
  if (!V || !A || !aligned16(V) || !aligned16(A) || T < 0 || rank < 1 || rank > G * d || lda < rank ||
      (v_dtype != XKV_F32 && v_dtype != XKV_BF16))
    return XKV_ERR_INVALID_ARG;
  if (T > (int64_t(1) << 31) - 1) return XKV_ERR_UNSUPPORTED;
  const bool tc = project_tc_ok(d, rank, dt);
  if (!tc && !(dt == XKV_F32 && v_dtype == XKV_F32)) return XKV_ERR_UNSUPPORTED;
  if (tc && lda % 8 != 0) return XKV_ERR_INVALID_ARG;
  if (tc && (!workspace || ws_bytes < project_workspace(G * d, rank) || !aligned256(workspace)))
    return XKV_ERR_WORKSPACE;
  return project_launch(X_layers, G, T, d, ldx, dt, V, v_dtype, rank, A, lda, workspace,
                        static_cast<cudaStream_t>(stream));
}

// -------------------------------------------------------------- landmarks
xkv_status xkv_build_landmarks(const void* K, int64_t T, int64_t ldk, int n_kv_heads, int head_dim, xkv_dtype dt,
                               int chunk, int sink, int recent, float rope_theta, void* landmarks, void* stream) {
  if (!K || !landmarks || !aligned16(K) || !aligned16(landmarks)) return XKV_ERR_INVALID_ARG;
  if (n_kv_heads < 1 || head_dim < 2 || head_dim % 2 != 0 || head_dim > 256 || chunk < 1 || sink < 0 || recent < 0)
    return XKV_ERR_INVALID_ARG;
  if (dt != XKV_F32 && dt != XKV_BF16) return XKV_ERR_INVALID_ARG;
  if (ldk < static_cast<int64_t>(n_kv_heads) * head_dim || T < sink + recent) return XKV_ERR_INVALID_ARG;
  if ((T - sink - recent) % chunk != 0 || !(rope_theta > 1.0f)) return XKV_ERR_INVALID_ARG;
  return landmarks_launch(K, T, ldk, n_kv_heads, head_dim, dt, chunk, sink, recent, rope_theta, landmarks,
                          static_cast<cudaStream_t>(stream));
}

// -------------------------------------------------------------- SR decode
static xkv_status check_sr(const xkv_sr_params* p) {
  if (!p) return XKV_ERR_INVALID_ARG;
  if (p->batch < 1 || p->n_kv_heads < 1 || p->n_q_heads < p->n_kv_heads || p->n_q_heads % p->n_kv_heads != 0)
    return XKV_ERR_INVALID_ARG;
  if (p->head_dim < 2 || p->head_dim % 2 != 0 || p->chunk < 1 || p->sink < 0 || p->recent < 0 || p->topk < 1)
    return XKV_ERR_INVALID_ARG;
  if (p->rank_k < 1 || p->rank_v < 1 || p->T < p->sink + p->recent + p->chunk) return XKV_ERR_INVALID_ARG;
  if ((p->T - p->sink - p->recent) % p->chunk != 0) return XKV_ERR_INVALID_ARG;
  const int64_t n_mid = (p->T - p->sink - p->recent) / p->chunk;
  if (p->topk > n_mid) return XKV_ERR_INVALID_ARG;
  if (p->a_k_batch_stride < p->T * p->rank_k || p->a_v_batch_stride < p->T * p->rank_v) return XKV_ERR_INVALID_ARG;
  const int64_t d = static_cast<int64_t>(p->n_kv_heads) * p->head_dim;
  if ((p->bt_k_batch_stride != 0 && p->bt_k_batch_stride < d * p->rank_k) ||
      (p->bt_v_batch_stride != 0 && p->bt_v_batch_stride < d * p->rank_v) || p->bt_k_batch_stride < 0 ||
      p->bt_v_batch_stride < 0)
    return XKV_ERR_INVALID_ARG;
  if (p->dtype != XKV_F32 && p->dtype != XKV_BF16) return XKV_ERR_INVALID_ARG;
  if (!(p->rope_theta > 1.0f)) return XKV_ERR_INVALID_ARG;
  if (p->window_batch_stride < 0 ||
      (p->window_batch_stride != 0 && p->window_batch_stride < static_cast<int64_t>(p->sink + p->recent) * d) ||
      p->window_batch_stride % 8 != 0)
    return XKV_ERR_INVALID_ARG;
  if (p->landmark_capacity < 0 || (p->landmark_capacity != 0 && p->landmark_capacity < n_mid))
    return XKV_ERR_INVALID_ARG;
  const int gq = p->n_q_heads / p->n_kv_heads;
  if (gq > 8 || p->head_dim > 256 || p->sink + p->recent > 64 || n_mid > kMaxMidChunks || p->rank_v > 4096 ||
      p->topk > 1024)
    return XKV_ERR_UNSUPPORTED;
  if (p->T > (int64_t(1) << 30)) return XKV_ERR_UNSUPPORTED;
  return XKV_OK;
}

xkv_status xkv_sr_profile_enable(int enable) { return sr_profile_enable(enable); }

xkv_status xkv_sr_profile_read(float* stage_ms) { return sr_profile_read(stage_ms); }

xkv_status xkv_sr_workspace_size(const xkv_sr_params* p, size_t* bytes) {
  if (!bytes) return XKV_ERR_INVALID_ARG;
  xkv_status s = check_sr(p);
  if (s != XKV_OK) return s;
  SRPlan plan;
  sr_plan(p, &plan);
  *bytes = plan.bytes;
  return XKV_OK;
}

xkv_status xkv_sr_attention_decode(const xkv_sr_params* p, const void* q, const void* A_K, const void* Bt_K,
                                   const void* A_V, const void* Bt_V, const void* landmarks, const void* sr_K,
                                   const void* sr_V, float* out, int32_t* sel_out, void* workspace, size_t ws_bytes,
                                   void* stream) {
  xkv_status s = check_sr(p);
  if (s != XKV_OK) return s;
  const void* ptrs[] = {q, A_K, Bt_K, A_V, Bt_V, landmarks, out};
  for (const void* x : ptrs)
    if (!x || !aligned16(x)) return XKV_ERR_INVALID_ARG;
  if (p->sink + p->recent > 0 && (!sr_K || !sr_V || !aligned16(sr_K) || !aligned16(sr_V))) return XKV_ERR_INVALID_ARG;
  if (sel_out && !aligned16(sel_out)) return XKV_ERR_INVALID_ARG;
  SRPlan plan;
  sr_plan(p, &plan);
  if (!workspace || ws_bytes < plan.bytes || !aligned256(workspace)) return XKV_ERR_WORKSPACE;
  return sr_launch(p, plan, q, A_K, Bt_K, A_V, Bt_V, landmarks, sr_K, sr_V, out, sel_out, workspace,
                   static_cast<cudaStream_t>(stream));
}

xkv_status xkv_sr_attention_decode_noalloc(const xkv_sr_params* p, const void* q, const void* A_K,
                                           const void* Bt_K, const void* A_V, const void* Bt_V, const void* landmarks,
                                           const void* sr_K, const void* sr_V, float* out, int32_t* sel_out,
                                           void* stream) {
  xkv_status s = check_sr(p);
  if (s != XKV_OK) return s;
  const void* ptrs[] = {q, A_K, Bt_K, A_V, Bt_V, landmarks, out};
  for (const void* x : ptrs)
    if (!x || !aligned16(x)) return XKV_ERR_INVALID_ARG;
  if (p->sink + p->recent > 0 && (!sr_K || !sr_V || !aligned16(sr_K) || !aligned16(sr_V))) return XKV_ERR_INVALID_ARG;
  if (sel_out && !aligned16(sel_out)) return XKV_ERR_INVALID_ARG;
  SRPlan plan;
  sr_plan(p, &plan);
  if (plan.bytes > static_cast<size_t>(XKV_SR_STATIC_SCRATCH_BYTES)) return XKV_ERR_UNSUPPORTED;
  void* scratch = static_scratch_ptr();
  if (!scratch) return XKV_ERR_CUDA;
  return sr_launch(p, plan, q, A_K, Bt_K, A_V, Bt_V, landmarks, sr_K, sr_V, out, sel_out, scratch,
                   static_cast<cudaStream_t>(stream));
}

// ------------------------------------------- xK-SR decode (values uncompressed)
// The SR kernels with the uncompressed value cache as their value operand:
// rank_v = head_dim, no Bt_V, A_V = V [B][T][d] (head h at columns h hd).
static xkv_status xk_params(const xkv_sr_params* p, xkv_sr_params* pv) {
  if (!p) return XKV_ERR_INVALID_ARG;
  *pv = *p;
  pv->rank_v = p->head_dim;
  pv->bt_v_batch_stride = 0;
  const xkv_status s = check_sr(pv);
  if (s != XKV_OK) return s;
  if (p->a_v_batch_stride < p->T * p->n_kv_heads * p->head_dim) return XKV_ERR_INVALID_ARG;
  return XKV_OK;
}

xkv_status xkv_xk_sr_workspace_size(const xkv_sr_params* p, size_t* bytes) {
  if (!bytes) return XKV_ERR_INVALID_ARG;
  xkv_sr_params pv;
  const xkv_status s = xk_params(p, &pv);
  if (s != XKV_OK) return s;
  SRPlan plan;
  sr_plan(&pv, &plan);
  *bytes = plan.bytes;
  return XKV_OK;
}

xkv_status xkv_xk_sr_attention_decode(const xkv_sr_params* p, const void* q, const void* A_K, const void* Bt_K,
                                      const void* V, const void* landmarks, const void* sr_K, const void* sr_V,
                                      float* out, int32_t* sel_out, void* workspace, size_t ws_bytes, void* stream) {
  xkv_sr_params pv;
  const xkv_status s = xk_params(p, &pv);
  if (s != XKV_OK) return s;
  const void* ptrs[] = {q, A_K, Bt_K, V, landmarks, out};
  for (const void* x : ptrs)
    if (!x || !aligned16(x)) return XKV_ERR_INVALID_ARG;
  if (p->sink + p->recent > 0 && (!sr_K || !sr_V || !aligned16(sr_K) || !aligned16(sr_V))) return XKV_ERR_INVALID_ARG;
  if (sel_out && !aligned16(sel_out)) return XKV_ERR_INVALID_ARG;
  SRPlan plan;
  sr_plan(&pv, &plan);
  if (!workspace || ws_bytes < plan.bytes || !aligned256(workspace)) return XKV_ERR_WORKSPACE;
  return sr_launch(&pv, plan, q, A_K, Bt_K, V, nullptr, landmarks, sr_K, sr_V, out, sel_out, workspace,
                   static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------ multi-step decode
static xkv_status check_append(const xkv_append_params* p) {
  if (!p || p->batch < 1 || p->group < 1 || p->group > 8 || p->n_kv_heads < 1 || p->head_dim < 2 ||
      p->head_dim % 2 != 0 || p->head_dim > 256 || p->chunk < 1 || p->sink < 0 || p->recent < 0 ||
      p->T < p->sink + p->recent || p->rank_k < 1 || p->rank_v < 1 || !(p->rope_theta > 1.0f))
    return XKV_ERR_INVALID_ARG;
  if (p->dtype != XKV_F32 && p->dtype != XKV_BF16) return XKV_ERR_INVALID_ARG;
  const int64_t d = static_cast<int64_t>(p->n_kv_heads) * p->head_dim;
  const int64_t n = d * p->group;
  if (p->rank_k > n || p->rank_v > n) return XKV_ERR_INVALID_ARG;
  const int64_t n0 = p->T - p->sink - p->recent;
  const int64_t n_mid = n0 / p->chunk;
  const bool roll = n0 % p->chunk == p->chunk - 1;
  const int64_t rows_needed = p->sink + (n_mid + (roll ? 1 : 0)) * p->chunk;
  if (p->window_batch_stride < (p->sink + p->recent + p->chunk) * d || p->window_batch_stride % 8 != 0)
    return XKV_ERR_INVALID_ARG;
  if (p->landmark_capacity < n_mid + (roll ? 1 : 0)) return XKV_ERR_INVALID_ARG;
  if (p->a_k_batch_stride < rows_needed * p->rank_k || p->a_v_batch_stride < rows_needed * p->rank_v)
    return XKV_ERR_INVALID_ARG;
  if ((p->bt_k_batch_stride != 0 && p->bt_k_batch_stride < n * p->rank_k) ||
      (p->bt_v_batch_stride != 0 && p->bt_v_batch_stride < n * p->rank_v) || p->bt_k_batch_stride < 0 ||
      p->bt_v_batch_stride < 0)
    return XKV_ERR_INVALID_ARG;
  if (p->dtype == XKV_BF16 && (!project_tc_ok(static_cast<int>(d), p->rank_k, XKV_BF16) ||
                               !project_tc_ok(static_cast<int>(d), p->rank_v, XKV_BF16)))
    return XKV_ERR_UNSUPPORTED;
  if (p->recent > 56) return XKV_ERR_UNSUPPORTED;
  return XKV_OK;
}

xkv_status xkv_sr_append_workspace_size(const xkv_append_params* p, size_t* bytes) {
  if (!bytes) return XKV_ERR_INVALID_ARG;
  const xkv_status s = check_append(p);
  if (s != XKV_OK) return s;
  *bytes = append_workspace(p);
  return XKV_OK;
}

xkv_status xkv_sr_append(const xkv_append_params* p, const void* const* k_new, const void* const* v_new,
                         void* const* win_K, void* const* win_V, const void* Bt_K, const void* Bt_V, void* A_K,
                         void* A_V, void* const* landmarks, int* rolled, void* workspace, size_t ws_bytes,
                         void* stream) {
  const xkv_status s = check_append(p);
  if (s != XKV_OK) return s;
  if (!k_new || !v_new || !win_K || !win_V || !landmarks) return XKV_ERR_INVALID_ARG;
  for (int l = 0; l < p->group; ++l)
    if (!k_new[l] || !v_new[l] || !win_K[l] || !win_V[l] || !landmarks[l] || !aligned16(k_new[l]) ||
        !aligned16(v_new[l]) || !aligned16(win_K[l]) || !aligned16(win_V[l]) || !aligned16(landmarks[l]))
      return XKV_ERR_INVALID_ARG;
  const void* ptrs[] = {Bt_K, Bt_V, A_K, A_V};
  for (const void* x : ptrs)
    if (!x || !aligned16(x)) return XKV_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < append_workspace(p) || !aligned256(workspace)) return XKV_ERR_WORKSPACE;
  return append_launch(p, k_new, v_new, win_K, win_V, Bt_K, Bt_V, A_K, A_V, landmarks, rolled, workspace,
                       static_cast<cudaStream_t>(stream));
}

// ------------------------------------ xK-SR decode, values in host memory
static size_t host_stage_bytes(const xkv_sr_params* pv) {
  const size_t es = pv->dtype == XKV_BF16 ? 2 : 4;
  return align_up(static_cast<size_t>(pv->batch) * pv->n_kv_heads * pv->topk * pv->chunk * pv->head_dim * es);
}

xkv_status xkv_xk_sr_host_workspace_size(const xkv_sr_params* p, size_t* bytes) {
  if (!bytes) return XKV_ERR_INVALID_ARG;
  xkv_sr_params pv;
  const xkv_status s = xk_params(p, &pv);
  if (s != XKV_OK) return s;
  SRPlan plan;
  sr_plan(&pv, &plan);
  *bytes = align_up(plan.bytes) + host_stage_bytes(&pv);
  return XKV_OK;
}

xkv_status xkv_xk_sr_attention_decode_host_values(const xkv_sr_params* p, const void* q, const void* A_K,
                                                  const void* Bt_K, const void* V_host, const void* landmarks,
                                                  const void* sr_K, const void* sr_V, float* out, int32_t* sel_out,
                                                  void* workspace, size_t ws_bytes, void* stream) {
  xkv_sr_params pv;
  const xkv_status s = xk_params(p, &pv);
  if (s != XKV_OK) return s;
  const void* ptrs[] = {q, A_K, Bt_K, V_host, landmarks, out};
  for (const void* x : ptrs)
    if (!x || !aligned16(x)) return XKV_ERR_INVALID_ARG;
  if (p->sink + p->recent > 0 && (!sr_K || !sr_V || !aligned16(sr_K) || !aligned16(sr_V))) return XKV_ERR_INVALID_ARG;
  if (sel_out && !aligned16(sel_out)) return XKV_ERR_INVALID_ARG;
  const size_t es = p->dtype == XKV_BF16 ? 2 : 4;
  if ((p->head_dim * es) % 16 != 0 || (p->a_v_batch_stride * es) % 16 != 0) return XKV_ERR_UNSUPPORTED;
  // the values must be page-locked host memory mapped for the device
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, V_host) != cudaSuccess || attr.type != cudaMemoryTypeHost) {
    cudaGetLastError();
    return XKV_ERR_INVALID_ARG;
  }
  void* v_dev = nullptr;
  if (cudaHostGetDevicePointer(&v_dev, const_cast<void*>(V_host), 0) != cudaSuccess || !v_dev) {
    cudaGetLastError();
    return XKV_ERR_INVALID_ARG;
  }
  SRPlan plan;
  sr_plan(&pv, &plan);
  const size_t need = align_up(plan.bytes) + host_stage_bytes(&pv);
  if (!workspace || ws_bytes < need || !aligned256(workspace)) return XKV_ERR_WORKSPACE;
  void* stage = static_cast<uint8_t*>(workspace) + align_up(plan.bytes);
  return sr_launch(&pv, plan, q, A_K, Bt_K, stage, nullptr, landmarks, sr_K, sr_V, out, sel_out, workspace,
                   static_cast<cudaStream_t>(stream), v_dev, stage);
}

// ------------------------------------------------------- token sharding
// the local slice of a token-sharded decode: p's own checks, with the global
// k (topk) allowed above the local chunk count
static xkv_status check_partial(const xkv_sr_params* p, xkv_sr_params* loc);

xkv_status xkv_sr_scores(const xkv_sr_params* p, const void* q, const void* landmarks, float* scores, int64_t ld,
                         void* stream) {
  xkv_sr_params loc;
  xkv_status s = check_partial(p, &loc);
  if (s != XKV_OK) return s;
  const int64_t n_mid = (p->T - p->sink - p->recent) / p->chunk;
  if (!q || !landmarks || !scores || !aligned16(q) || !aligned16(landmarks) || !aligned16(scores) || ld < n_mid ||
      ld % 4 != 0)
    return XKV_ERR_INVALID_ARG;
  return sr_scores_launch(p, q, landmarks, scores, ld, static_cast<cudaStream_t>(stream));
}

xkv_status xkv_sr_topk(const float* scores, int64_t ld, int rows, int64_t n, int k, int32_t* sel_out, void* stream) {
  if (!scores || !sel_out || !aligned16(scores) || !aligned16(sel_out) || rows < 1 || n < 1 || k < 1 || k > n ||
      ld < n || ld % 4 != 0)
    return XKV_ERR_INVALID_ARG;
  if (n > kMaxMidChunks || k > 1024) return XKV_ERR_UNSUPPORTED;
  return sr_topk_launch(scores, ld, rows, n, k, sel_out, static_cast<cudaStream_t>(stream));
}

static xkv_status check_partial(const xkv_sr_params* p, xkv_sr_params* loc) {
  if (!p) return XKV_ERR_INVALID_ARG;
  *loc = *p;
  if (p->chunk < 1 || p->T < p->sink + p->recent + p->chunk) return XKV_ERR_INVALID_ARG;
  const int64_t n_mid = (p->T - p->sink - p->recent) / p->chunk;
  if (p->topk < 1 || p->topk > 1024) return p->topk < 1 ? XKV_ERR_INVALID_ARG : XKV_ERR_UNSUPPORTED;
  loc->topk = static_cast<int>(std::min<int64_t>(p->topk, n_mid));
  const xkv_status s = check_sr(loc);
  *loc = *p;
  return s;
}

xkv_status xkv_sr_partial_workspace_size(const xkv_sr_params* p, size_t* bytes) {
  if (!bytes) return XKV_ERR_INVALID_ARG;
  xkv_sr_params loc;
  const xkv_status s = check_partial(p, &loc);
  if (s != XKV_OK) return s;
  SRPlan plan;
  sr_plan(&loc, &plan);
  *bytes = plan.bytes;
  return XKV_OK;
}

xkv_status xkv_sr_attention_partial(const xkv_sr_params* p, const xkv_sr_shard* shard, const int32_t* sel,
                                    const void* q, const void* A_K, const void* Bt_K, const void* A_V,
                                    const void* Bt_V, const void* sr_K, const void* sr_V, float* out, float* ml_out,
                                    void* workspace, size_t ws_bytes, void* stream) {
  xkv_sr_params loc;
  const xkv_status s = check_partial(p, &loc);
  if (s != XKV_OK) return s;
  if (!shard || shard->position_offset < 0 || shard->chunk_begin < 0 || shard->chunk_begin > (int64_t(1) << 30))
    return XKV_ERR_INVALID_ARG;
  const void* ptrs[] = {sel, q, A_K, Bt_K, A_V, Bt_V, out, ml_out};
  for (const void* x : ptrs)
    if (!x || !aligned16(x)) return XKV_ERR_INVALID_ARG;
  if (p->sink + p->recent > 0 && (!sr_K || !sr_V || !aligned16(sr_K) || !aligned16(sr_V))) return XKV_ERR_INVALID_ARG;
  SRPlan plan;
  sr_plan(&loc, &plan);
  if (!workspace || ws_bytes < plan.bytes || !aligned256(workspace)) return XKV_ERR_WORKSPACE;
  const int64_t n_mid = (p->T - p->sink - p->recent) / p->chunk;
  SRShard sh;
  sh.sel = sel;
  sh.pos_off = shard->position_offset;
  sh.c_lo = static_cast<int>(shard->chunk_begin);
  sh.c_hi = static_cast<int>(shard->chunk_begin + n_mid);
  sh.ml_out = ml_out;
  return sr_launch(&loc, plan, q, A_K, Bt_K, A_V, Bt_V, nullptr, sr_K, sr_V, out, nullptr, workspace,
                   static_cast<cudaStream_t>(stream), nullptr, nullptr, &sh);
}

xkv_status xkv_merge_partials(const float* o, const float* ml, int R, int rows, int hd, float* out, void* stream) {
  if (!o || !ml || !out || R < 1 || rows < 1 || hd < 1) return XKV_ERR_INVALID_ARG;
  return merge_partials_launch(o, ml, R, rows, hd, out, static_cast<cudaStream_t>(stream));
}

// --------------------------------------------------- full reconstruction
xkv_status xkv_full_reconstruct(const void* A, const void* Bt, int64_t T, int rank, int d, int n_kv_heads,
                                int head_dim, int apply_rope, float rope_theta, xkv_dtype dt, void* out, void* stream) {
  if (!A || !Bt || !out || !aligned16(A) || !aligned16(Bt) || !aligned16(out)) return XKV_ERR_INVALID_ARG;
  if (T < 0 || rank < 1 || rank % 16 != 0 || d < 1 || n_kv_heads < 1 || head_dim < 2 || head_dim % 2 != 0 ||
      n_kv_heads * head_dim != d)
    return XKV_ERR_INVALID_ARG;
  if (dt != XKV_F32 && dt != XKV_BF16) return XKV_ERR_INVALID_ARG;
  if (apply_rope && !(rope_theta > 1.0f)) return XKV_ERR_INVALID_ARG;
  if (T > (int64_t(1) << 31) - 1) return XKV_ERR_UNSUPPORTED;
  return recon_launch(A, Bt, T, rank, d, n_kv_heads, head_dim, apply_rope, rope_theta, dt, out,
                      static_cast<cudaStream_t>(stream));
}

static xkv_status check_dense(const xkv_dense_params* p) {
  if (!p || p->batch < 1 || p->n_kv_heads < 1 || p->n_q_heads % p->n_kv_heads != 0 || p->n_q_heads < 1 ||
      p->head_dim < 2 || p->head_dim % 2 != 0 || p->T < 1)
    return XKV_ERR_INVALID_ARG;
  if (p->dtype != XKV_F32 && p->dtype != XKV_BF16) return XKV_ERR_INVALID_ARG;
  if (p->n_q_heads / p->n_kv_heads > 8 || p->head_dim > 256 || 256 % (p->head_dim / 2) != 0) return XKV_ERR_UNSUPPORTED;
  return XKV_OK;
}

xkv_status xkv_dense_workspace_size(const xkv_dense_params* p, size_t* bytes) {
  if (!bytes) return XKV_ERR_INVALID_ARG;
  xkv_status s = check_dense(p);
  if (s != XKV_OK) return s;
  *bytes = dense_workspace(p);
  return XKV_OK;
}

xkv_status xkv_dense_attention_decode(const xkv_dense_params* p, const void* q, const void* K, const void* V, float* out,
                                      void* workspace, size_t ws_bytes, void* stream) {
  xkv_status s = check_dense(p);
  if (s != XKV_OK) return s;
  if (!q || !K || !V || !out || !aligned16(q) || !aligned16(K) || !aligned16(V) || !aligned16(out))
    return XKV_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < dense_workspace(p) || !aligned256(workspace)) return XKV_ERR_WORKSPACE;
  return dense_launch(p, q, K, V, out, workspace, static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------- NER
xkv_status xkv_ner_workspace_size(int n, int block, size_t* bytes) {
  if (!bytes || n < 2 || block < 2 || block % 2 != 0 || n % block != 0) return XKV_ERR_INVALID_ARG;
  *bytes = ner_workspace(n, block);
  return XKV_OK;
}

xkv_status xkv_ner(const float* gram, int n, int block, double rank_rel_tol, float* ner_out, float* erank_out,
                   int32_t* rank_out, void* workspace, size_t ws_bytes, void* stream) {
  if (!gram || !ner_out || !aligned16(gram) || n < 2 || block < 2 || block % 2 != 0 || n % block != 0)
    return XKV_ERR_INVALID_ARG;
  if (!(rank_rel_tol >= 0.0) || !(rank_rel_tol < 1.0)) return XKV_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < ner_workspace(n, block) || !aligned256(workspace)) return XKV_ERR_WORKSPACE;
  return ner_launch(gram, n, block, rank_rel_tol, ner_out, erank_out, rank_out, workspace,
                    static_cast<cudaStream_t>(stream));
}

xkv_status xkv_energy_rank(const float* gram, int n, int block, double energy, int32_t* rank_out, float* lambda_out,
                           void* workspace, size_t ws_bytes, void* stream) {
  if (!gram || !rank_out || !aligned16(gram) || n < 2 || block < 2 || block % 2 != 0 || n % block != 0)
    return XKV_ERR_INVALID_ARG;
  if (!(energy > 0.0) || !(energy <= 1.0)) return XKV_ERR_INVALID_ARG;
  if (block > 8192) return XKV_ERR_UNSUPPORTED;
  if (!workspace || ws_bytes < ner_workspace(n, block) || !aligned256(workspace)) return XKV_ERR_WORKSPACE;
  return energy_rank_launch(gram, n, block, energy, rank_out, lambda_out, workspace, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
