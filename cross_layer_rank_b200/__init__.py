"""B200 (sm_100a) xKV hot path: thin Python binding of libxkv.so.

Every call below marshals torch tensors into the C ABI declared in
include/xkv.h and returns; all arithmetic runs in the library's CUDA kernels.
There is no CPU or PyTorch fallback: importing this package fails loudly when
libxkv.so has not been built (``python cross_layer_rank_b200/build.py``).

Functions keep the C names (xkv_compress_group, xkv_build_landmarks,
xkv_sr_attention_decode, xkv_full_reconstruct, xkv_ner, ...).  Tensors must be
CUDA tensors, contiguous, of the dtype named by the call; errors raise
XKVError carrying the library's status code.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libxkv.so")

XKV_OK = 0
XKV_ERR_INVALID_ARG = 1
XKV_ERR_UNSUPPORTED = 2
XKV_ERR_WORKSPACE = 3
XKV_ERR_CUDA = 4
XKV_ERR_NUMERICAL = 5
XKV_ERR_DEVICE_TIMEOUT = 6
XKV_F32 = 0
XKV_BF16 = 1

EXPORTS = (
    "xkv_status_string", "xkv_version", "xkv_get_device_status",
    "xkv_gram_workspace_size", "xkv_gram_accumulate",
    "xkv_compress_workspace_size", "xkv_compress_group",
    "xkv_factor_workspace_size", "xkv_factor_gram", "xkv_project_workspace_size", "xkv_project",
    "xkv_build_landmarks",
    "xkv_sr_workspace_size", "xkv_sr_attention_decode",
    "xkv_sr_attention_decode_noalloc",
    "xkv_xk_sr_workspace_size", "xkv_xk_sr_attention_decode",
    "xkv_xk_sr_host_workspace_size", "xkv_xk_sr_attention_decode_host_values",
    "xkv_sr_profile_enable", "xkv_sr_profile_read",
    "xkv_sr_append_workspace_size", "xkv_sr_append",
    "xkv_sr_scores", "xkv_sr_topk", "xkv_sr_partial_workspace_size", "xkv_sr_attention_partial",
    "xkv_merge_partials",
    "xkv_selftest_expired_wait",
    "xkv_full_reconstruct",
    "xkv_dense_workspace_size", "xkv_dense_attention_decode",
    "xkv_ner_workspace_size", "xkv_ner", "xkv_energy_rank",
)


class XKVError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class SRParams(C.Structure):
    """Mirror of xkv_sr_params."""
    _fields_ = [("batch", C.c_int), ("n_q_heads", C.c_int), ("n_kv_heads", C.c_int), ("head_dim", C.c_int),
                ("T", C.c_int64), ("rank_k", C.c_int), ("rank_v", C.c_int), ("chunk", C.c_int),
                ("topk", C.c_int), ("sink", C.c_int), ("recent", C.c_int), ("rope_theta", C.c_float),
                ("dtype", C.c_int), ("a_k_batch_stride", C.c_int64), ("a_v_batch_stride", C.c_int64),
                ("bt_k_batch_stride", C.c_int64), ("bt_v_batch_stride", C.c_int64),
                ("window_batch_stride", C.c_int64), ("landmark_capacity", C.c_int64)]


class AppendParams(C.Structure):
    """Mirror of xkv_append_params."""
    _fields_ = [("batch", C.c_int), ("group", C.c_int), ("n_kv_heads", C.c_int), ("head_dim", C.c_int),
                ("chunk", C.c_int), ("sink", C.c_int), ("recent", C.c_int), ("rope_theta", C.c_float),
                ("dtype", C.c_int), ("T", C.c_int64), ("rank_k", C.c_int), ("rank_v", C.c_int),
                ("a_k_batch_stride", C.c_int64), ("a_v_batch_stride", C.c_int64),
                ("bt_k_batch_stride", C.c_int64), ("bt_v_batch_stride", C.c_int64),
                ("window_batch_stride", C.c_int64), ("landmark_capacity", C.c_int64)]


class ShardParams(C.Structure):
    """Mirror of xkv_sr_shard."""
    _fields_ = [("position_offset", C.c_int64), ("chunk_begin", C.c_int64)]


class DenseParams(C.Structure):
    """Mirror of xkv_dense_params."""
    _fields_ = [("batch", C.c_int), ("n_q_heads", C.c_int), ("n_kv_heads", C.c_int), ("head_dim", C.c_int),
                ("T", C.c_int64), ("dtype", C.c_int)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libxkv.so not built ({LIB_PATH}); run `python cross_layer_rank_b200/build.py`")
    lib = C.CDLL(LIB_PATH)
    vp, i64, sz = C.c_void_p, C.c_int64, C.c_size_t
    sig = {
        "xkv_status_string": (C.c_char_p, [C.c_int]),
        "xkv_version": (C.c_int, []),
        "xkv_get_device_status": (C.c_int, [vp]),
        "xkv_gram_workspace_size": (C.c_int, [C.c_int, i64, C.c_int, C.c_int, C.POINTER(sz)]),
        "xkv_gram_accumulate": (C.c_int, [vp, C.c_int, i64, C.c_int, i64, C.c_int, vp, vp, sz, vp]),
        "xkv_compress_workspace_size": (C.c_int, [C.c_int, i64, C.c_int, C.c_int, C.c_int, i64, C.c_int,
                                                  C.POINTER(sz)]),
        "xkv_compress_group": (C.c_int, [vp, C.c_int, i64, C.c_int, i64, C.c_int, C.c_int, C.c_int, C.c_int, i64,
                                         C.c_uint64, vp, vp, vp, vp, vp, sz, vp]),
        "xkv_factor_workspace_size": (C.c_int, [C.c_int, C.c_int, i64, C.c_int, C.c_int, C.c_int, C.POINTER(sz)]),
        "xkv_factor_gram": (C.c_int, [vp, C.c_int, C.c_int, i64, C.c_int, C.c_int, C.c_int, C.c_int, C.c_uint64,
                                      vp, vp, vp, vp, sz, vp]),
        "xkv_project_workspace_size": (C.c_int, [C.c_int, C.c_int, C.c_int, C.POINTER(sz)]),
        "xkv_project": (C.c_int, [vp, C.c_int, i64, C.c_int, i64, C.c_int, vp, C.c_int, C.c_int, vp, i64, vp, sz,
                                  vp]),
        "xkv_build_landmarks": (C.c_int, [vp, i64, i64, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                          C.c_float, vp, vp]),
        "xkv_sr_workspace_size": (C.c_int, [C.POINTER(SRParams), C.POINTER(sz)]),
        "xkv_sr_attention_decode": (C.c_int, [C.POINTER(SRParams), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                                              vp]),
        "xkv_sr_attention_decode_noalloc": (C.c_int, [C.POINTER(SRParams), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                                      vp]),
        "xkv_xk_sr_workspace_size": (C.c_int, [C.POINTER(SRParams), C.POINTER(sz)]),
        "xkv_xk_sr_attention_decode": (C.c_int, [C.POINTER(SRParams), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                                                 vp]),
        "xkv_xk_sr_host_workspace_size": (C.c_int, [C.POINTER(SRParams), C.POINTER(sz)]),
        "xkv_xk_sr_attention_decode_host_values": (C.c_int, [C.POINTER(SRParams), vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                                             vp, sz, vp]),
        "xkv_sr_scores": (C.c_int, [C.POINTER(SRParams), vp, vp, vp, i64, vp]),
        "xkv_sr_topk": (C.c_int, [vp, i64, C.c_int, i64, C.c_int, vp, vp]),
        "xkv_sr_partial_workspace_size": (C.c_int, [C.POINTER(SRParams), C.POINTER(sz)]),
        "xkv_sr_attention_partial": (C.c_int, [C.POINTER(SRParams), C.POINTER(ShardParams), vp, vp, vp, vp, vp, vp,
                                               vp, vp, vp, vp, vp, sz, vp]),
        "xkv_merge_partials": (C.c_int, [vp, vp, C.c_int, C.c_int, C.c_int, vp, vp]),
        "xkv_selftest_expired_wait": (C.c_int, [vp]),
        "xkv_sr_append_workspace_size": (C.c_int, [C.POINTER(AppendParams), C.POINTER(sz)]),
        "xkv_sr_append": (C.c_int, [C.POINTER(AppendParams), vp, vp, vp, vp, vp, vp, vp, vp, vp, C.POINTER(C.c_int),
                                    vp, sz, vp]),
        "xkv_sr_profile_enable": (C.c_int, [C.c_int]),
        "xkv_sr_profile_read": (C.c_int, [C.POINTER(C.c_float)]),
        "xkv_full_reconstruct": (C.c_int, [vp, vp, i64, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_float,
                                           C.c_int, vp, vp]),
        "xkv_dense_workspace_size": (C.c_int, [C.POINTER(DenseParams), C.POINTER(sz)]),
        "xkv_dense_attention_decode": (C.c_int, [C.POINTER(DenseParams), vp, vp, vp, vp, vp, sz, vp]),
        "xkv_ner_workspace_size": (C.c_int, [C.c_int, C.c_int, C.POINTER(sz)]),
        "xkv_ner": (C.c_int, [vp, C.c_int, C.c_int, C.c_double, vp, vp, vp, vp, sz, vp]),
        "xkv_energy_rank": (C.c_int, [vp, C.c_int, C.c_int, C.c_double, vp, vp, vp, sz, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()


def status_string(status: int) -> str:
    return lib.xkv_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != XKV_OK:
        raise XKVError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return C.c_void_p(t.data_ptr())


def _stream(stream) -> C.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return XKV_BF16
    if t == torch.float32:
        return XKV_F32
    raise ValueError(f"unsupported dtype {t}")


def workspace(nbytes: int, device=None) -> torch.Tensor:
    """Caller-owned scratch (256-byte aligned, as torch's allocator guarantees)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


def _wsize(fn, *args) -> int:
    n = C.c_size_t(0)
    _check(fn(*args, C.byref(n)), fn.__name__)
    return int(n.value)


def get_device_status(stream=None) -> int:
    """Deferred device-side status (synchronises the stream), cleared on read."""
    return int(lib.xkv_get_device_status(_stream(stream)))


# ------------------------------------------------------------------- Gram
def xkv_gram_workspace_size(G: int, rows: int, d: int, dtype: torch.dtype) -> int:
    return _wsize(lib.xkv_gram_workspace_size, G, rows, d, dtype_code(dtype))


def xkv_gram_accumulate(layers: Sequence[torch.Tensor], C_out: torch.Tensor, ws: Optional[torch.Tensor] = None,
                        stream=None):
    """C_out += X^T X over X = [layers...] (each rows x d)."""
    G = len(layers)
    rows, d = layers[0].shape
    ldx = layers[0].stride(0)
    ptrs = (C.c_void_p * G)(*[t.data_ptr() for t in layers])
    nbytes = xkv_gram_workspace_size(G, rows, d, layers[0].dtype)
    ws = ws if ws is not None else workspace(nbytes, layers[0].device)
    _check(lib.xkv_gram_accumulate(ptrs, G, rows, d, ldx, dtype_code(layers[0].dtype), _ptr(C_out), _ptr(ws),
                                   ws.numel(), _stream(stream)), "xkv_gram_accumulate")


# ------------------------------------------------------------ compression
def xkv_compress_workspace_size(G, T, d, rank, oversample, shard_rows, dtype: torch.dtype) -> int:
    return _wsize(lib.xkv_compress_workspace_size, G, T, d, rank, oversample, shard_rows, dtype_code(dtype))


def xkv_compress_group(layers: Sequence[torch.Tensor], rank: int, A: torch.Tensor, Bt: torch.Tensor,
                       iters: int = 8, oversample: int = 64, shard_rows: int = 8192, seed: int = 0x784B56,
                       eigvals: Optional[torch.Tensor] = None, gram_out: Optional[torch.Tensor] = None,
                       ws: Optional[torch.Tensor] = None, stream=None):
    """Cross-layer factorisation of one group into A (T x rank) and Bt (G d x rank)."""
    G = len(layers)
    T, d = layers[0].shape
    ldx = layers[0].stride(0)
    for t in layers:
        if t.shape != layers[0].shape or t.stride(0) != ldx or t.stride(1) != 1:
            raise ValueError("layers must share shape and row stride")
    dt = dtype_code(layers[0].dtype)
    nbytes = xkv_compress_workspace_size(G, T, d, rank, oversample, shard_rows, layers[0].dtype)
    ws = ws if ws is not None else workspace(nbytes, layers[0].device)
    ptrs = (C.c_void_p * G)(*[t.data_ptr() for t in layers])
    _check(lib.xkv_compress_group(ptrs, G, T, d, ldx, dt, rank, iters, oversample, shard_rows, seed, _ptr(A),
                                  _ptr(Bt), _ptr(eigvals), _ptr(gram_out), _ptr(ws), ws.numel(), _stream(stream)),
           "xkv_compress_group")


def xkv_factor_workspace_size(G, d, rows, rank, oversample, dtype: torch.dtype) -> int:
    return _wsize(lib.xkv_factor_workspace_size, G, d, rows, rank, oversample, dtype_code(dtype))


def xkv_factor_gram(gram: torch.Tensor, G: int, d: int, rows: int, rank: int, Bt: torch.Tensor,
                    iters: int = 8, oversample: int = 64, seed: int = 0x784B56, Vr_out: Optional[torch.Tensor] = None,
                    eigvals: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None, stream=None):
    """Top-r basis of a given (G d)^2 f32 Gram: Bt (G d x rank, Bt's dtype), optional f32 V_r and Ritz values."""
    nbytes = xkv_factor_workspace_size(G, d, rows, rank, oversample, Bt.dtype)
    ws = ws if ws is not None else workspace(nbytes, gram.device)
    _check(lib.xkv_factor_gram(_ptr(gram), G, d, rows, dtype_code(Bt.dtype), rank, iters, oversample, seed, _ptr(Bt),
                               _ptr(Vr_out), _ptr(eigvals), _ptr(ws), ws.numel(), _stream(stream)), "xkv_factor_gram")


def xkv_project_workspace_size(G, d, rank) -> int:
    return _wsize(lib.xkv_project_workspace_size, G, d, rank)


def xkv_project(layers: Sequence[torch.Tensor], V: torch.Tensor, A: torch.Tensor, ws: Optional[torch.Tensor] = None,
                stream=None):
    """A = [layers...] V; A may be a row-strided view (rows of rank elements)."""
    G = len(layers)
    T, d = layers[0].shape
    ldx = layers[0].stride(0)
    for t in layers:
        if t.shape != layers[0].shape or t.stride(0) != ldx or t.stride(1) != 1:
            raise ValueError("layers must share shape and row stride")
    rank = V.shape[1]
    if A.shape[-1] != rank or A.stride(-1) != 1 or not A.is_cuda:
        raise ValueError("A must be T x rank with contiguous rows")
    ws = ws if ws is not None else workspace(xkv_project_workspace_size(G, d, rank), layers[0].device)
    ptrs = (C.c_void_p * G)(*[t.data_ptr() for t in layers])
    _check(lib.xkv_project(ptrs, G, T, d, ldx, dtype_code(layers[0].dtype), _ptr(V), dtype_code(V.dtype), rank,
                           C.c_void_p(A.data_ptr()), A.stride(0), _ptr(ws), ws.numel(), _stream(stream)),
           "xkv_project")


# -------------------------------------------------------------- landmarks
def xkv_build_landmarks(K: torch.Tensor, n_kv_heads: int, head_dim: int, chunk: int, sink: int, recent: int,
                        rope_theta: float, out: torch.Tensor, stream=None):
    T = K.shape[0]
    if K.stride(1) != 1:
        raise ValueError("K rows must be contiguous")
    _check(lib.xkv_build_landmarks(C.c_void_p(K.data_ptr()), T, K.stride(0), n_kv_heads, head_dim,
                                   dtype_code(K.dtype), chunk, sink, recent, rope_theta, _ptr(out), _stream(stream)),
           "xkv_build_landmarks")


# -------------------------------------------------------------- SR decode
def sr_params(batch, n_q_heads, n_kv_heads, head_dim, T, rank_k, rank_v, chunk, topk, sink, recent, rope_theta,
              dtype: torch.dtype, a_k_batch_stride=None, a_v_batch_stride=None, bt_k_batch_stride=None,
              bt_v_batch_stride=None, window_batch_stride=0, landmark_capacity=0) -> SRParams:
    """Batch strides default to dense [B][T][r] A and per-batch dense [B][d][r] Bt;
    window and landmark strides default to the exact sizes (0)."""
    d = n_kv_heads * head_dim
    return SRParams(batch, n_q_heads, n_kv_heads, head_dim, T, rank_k, rank_v, chunk, topk, sink, recent,
                    float(rope_theta), dtype_code(dtype),
                    T * rank_k if a_k_batch_stride is None else a_k_batch_stride,
                    T * rank_v if a_v_batch_stride is None else a_v_batch_stride,
                    d * rank_k if bt_k_batch_stride is None else bt_k_batch_stride,
                    d * rank_v if bt_v_batch_stride is None else bt_v_batch_stride,
                    window_batch_stride, landmark_capacity)


def xkv_sr_workspace_size(p: SRParams) -> int:
    return _wsize(lib.xkv_sr_workspace_size, C.byref(p))


def _addr(t: Optional[torch.Tensor]):
    """Device address of a tensor whose layout the call's strides describe (a
    view such as one layer's rows of a group basis is accepted)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if t.numel() > 0 and t.shape[-1] > 1 and t.stride(-1) != 1:
        raise ValueError("expected contiguous rows")
    return C.c_void_p(t.data_ptr())


def xkv_sr_attention_decode(p: SRParams, q, A_K, Bt_K, A_V, Bt_V, landmarks, sr_K, sr_V, out,
                            sel_out=None, ws=None, stream=None):
    """One SR decode step of one layer; writes out [B][Hq][hd] f32 (and sel_out).
    A, Bt, landmarks and windows may be views: their strides come from p."""
    ws = ws if ws is not None else workspace(xkv_sr_workspace_size(p), q.device)
    _check(lib.xkv_sr_attention_decode(C.byref(p), _ptr(q), _addr(A_K), _addr(Bt_K), _addr(A_V), _addr(Bt_V),
                                       _addr(landmarks), _addr(sr_K), _addr(sr_V), _ptr(out), _ptr(sel_out),
                                       _ptr(ws), ws.numel(), _stream(stream)), "xkv_sr_attention_decode")


SR_STATIC_SCRATCH_BYTES = 8 << 20


def xkv_sr_attention_decode_noalloc(p: SRParams, q, A_K, Bt_K, A_V, Bt_V, landmarks, sr_K, sr_V, out,
                                    sel_out=None, stream=None):
    """One SR decode step with the library's fixed scratch array (no workspace,
    no allocation); calls that overlap in time race on that array."""
    _check(lib.xkv_sr_attention_decode_noalloc(C.byref(p), _ptr(q), _ptr(A_K), _ptr(Bt_K), _ptr(A_V), _ptr(Bt_V),
                                               _ptr(landmarks), _ptr(sr_K), _ptr(sr_V), _ptr(out), _ptr(sel_out),
                                               _stream(stream)), "xkv_sr_attention_decode_noalloc")


def xk_sr_params(batch, n_q_heads, n_kv_heads, head_dim, T, rank_k, chunk, topk, sink, recent, rope_theta,
                 dtype: torch.dtype, a_k_batch_stride=None, v_batch_stride=None, bt_k_batch_stride=None) -> SRParams:
    """Parameters of the xK-SR mode: keys as in sr_params, values an uncompressed
    [B][T][d] cache (batch stride defaults to T d)."""
    d = n_kv_heads * head_dim
    return SRParams(batch, n_q_heads, n_kv_heads, head_dim, T, rank_k, head_dim, chunk, topk, sink, recent,
                    float(rope_theta), dtype_code(dtype),
                    T * rank_k if a_k_batch_stride is None else a_k_batch_stride,
                    T * d if v_batch_stride is None else v_batch_stride,
                    d * rank_k if bt_k_batch_stride is None else bt_k_batch_stride, 0, 0, 0)


def xkv_xk_sr_host_workspace_size(p: SRParams) -> int:
    return _wsize(lib.xkv_xk_sr_host_workspace_size, C.byref(p))


def xkv_xk_sr_attention_decode_host_values(p: SRParams, q, A_K, Bt_K, V_host: torch.Tensor, landmarks, sr_K, sr_V,
                                           out, sel_out=None, ws=None, stream=None):
    """xK-SR step with V [B][T][d] in pinned host memory (V_host.is_pinned());
    only the kept chunks' rows are read over the host link."""
    if V_host.is_cuda or not V_host.is_pinned():
        raise ValueError("V_host must be a pinned host tensor")
    ws = ws if ws is not None else workspace(xkv_xk_sr_host_workspace_size(p), q.device)
    _check(lib.xkv_xk_sr_attention_decode_host_values(C.byref(p), _ptr(q), _addr(A_K), _addr(Bt_K),
                                                      C.c_void_p(V_host.data_ptr()), _addr(landmarks), _addr(sr_K),
                                                      _addr(sr_V), _ptr(out), _ptr(sel_out), _ptr(ws), ws.numel(),
                                                      _stream(stream)), "xkv_xk_sr_attention_decode_host_values")


def xkv_xk_sr_workspace_size(p: SRParams) -> int:
    return _wsize(lib.xkv_xk_sr_workspace_size, C.byref(p))


def xkv_xk_sr_attention_decode(p: SRParams, q, A_K, Bt_K, V, landmarks, sr_K, sr_V, out, sel_out=None, ws=None,
                               stream=None):
    """One xK-SR decode step of one layer (values read from the uncompressed V
    [B][T][d]); writes out [B][Hq][hd] f32 (and sel_out)."""
    ws = ws if ws is not None else workspace(xkv_xk_sr_workspace_size(p), q.device)
    _check(lib.xkv_xk_sr_attention_decode(C.byref(p), _ptr(q), _ptr(A_K), _ptr(Bt_K), _ptr(V), _ptr(landmarks),
                                          _ptr(sr_K), _ptr(sr_V), _ptr(out), _ptr(sel_out), _ptr(ws), ws.numel(),
                                          _stream(stream)), "xkv_xk_sr_attention_decode")


def xkv_selftest_expired_wait(stream=None) -> None:
    """Launch the bounded-wait self-test (a wait that runs out after about one
    second); read the outcome with get_device_status()."""
    _check(lib.xkv_selftest_expired_wait(_stream(stream)), "xkv_selftest_expired_wait")


def xkv_sr_profile_enable(enable: bool = True) -> None:
    """Record CUDA events around the four launches of each later SR decode call."""
    _check(lib.xkv_sr_profile_enable(int(bool(enable))), "xkv_sr_profile_enable")


def xkv_sr_profile_read() -> list:
    """Durations (ms) of the last timed call: scores, top-k + window, attend, combine."""
    buf = (C.c_float * 4)()
    _check(lib.xkv_sr_profile_read(buf), "xkv_sr_profile_read")
    return [float(x) for x in buf]


# --------------------------------------------------- full reconstruction
def xkv_full_reconstruct(A, Bt, n_kv_heads: int, head_dim: int, apply_rope: bool, rope_theta: float, out,
                         stream=None):
    T, r = A.shape
    d = Bt.shape[0]
    _check(lib.xkv_full_reconstruct(_ptr(A), _ptr(Bt), T, r, d, n_kv_heads, head_dim, int(bool(apply_rope)),
                                    float(rope_theta), dtype_code(A.dtype), _ptr(out), _stream(stream)),
           "xkv_full_reconstruct")


def dense_params(batch, n_q_heads, n_kv_heads, head_dim, T, dtype: torch.dtype) -> DenseParams:
    return DenseParams(batch, n_q_heads, n_kv_heads, head_dim, T, dtype_code(dtype))


def xkv_dense_workspace_size(p: DenseParams) -> int:
    return _wsize(lib.xkv_dense_workspace_size, C.byref(p))


def xkv_dense_attention_decode(p: DenseParams, q, K, V, out, ws=None, stream=None):
    ws = ws if ws is not None else workspace(xkv_dense_workspace_size(p), q.device)
    _check(lib.xkv_dense_attention_decode(C.byref(p), _ptr(q), _ptr(K), _ptr(V), _ptr(out), _ptr(ws), ws.numel(),
                                          _stream(stream)), "xkv_dense_attention_decode")


# -------------------------------------------------------------------- NER
def xkv_ner_workspace_size(n: int, block: int) -> int:
    return _wsize(lib.xkv_ner_workspace_size, n, block)


def xkv_ner(gram: torch.Tensor, block: int, ner_out, erank_out=None, rank_out=None, rank_rel_tol: float = 1e-9,
            ws=None, stream=None):
    n = gram.shape[0]
    ws = ws if ws is not None else workspace(xkv_ner_workspace_size(n, block), gram.device)
    _check(lib.xkv_ner(_ptr(gram), n, block, rank_rel_tol, _ptr(ner_out), _ptr(erank_out), _ptr(rank_out), _ptr(ws),
                       ws.numel(), _stream(stream)), "xkv_ner")


def xkv_energy_rank(gram, block: int, energy: float = 0.95, rank_out=None, lambda_out=None, ws=None, stream=None):
    """Per diagonal block: the rank keeping `energy` of the block's eigenvalue
    total, and optionally its eigenvalues in descending order."""
    n = gram.shape[0]
    count = n // block
    rank_out = rank_out if rank_out is not None else torch.empty(count, dtype=torch.int32, device=gram.device)
    ws = ws if ws is not None else workspace(xkv_ner_workspace_size(n, block), gram.device)
    _check(lib.xkv_energy_rank(_ptr(gram), n, block, float(energy), _ptr(rank_out), _ptr(lambda_out), _ptr(ws),
                               ws.numel(), _stream(stream)), "xkv_energy_rank")
    return rank_out


# ------------------------------------------------------- multi-step decode
def decode_layout(T: int, sink: int, recent: int, chunk: int):
    """(n_mid, window rows) of a cache of T tokens built by prefill plus appends:
    n0 = T - sink - recent; n_mid = n0 // chunk; the window holds recent + n0 % chunk rows."""
    n0 = T - sink - recent
    return n0 // chunk, recent + n0 % chunk


def append_params(batch, group, n_kv_heads, head_dim, chunk, sink, recent, rope_theta, dtype: torch.dtype, T,
                  rank_k, rank_v, a_k_batch_stride, a_v_batch_stride, bt_k_batch_stride, bt_v_batch_stride,
                  window_batch_stride, landmark_capacity) -> AppendParams:
    return AppendParams(batch, group, n_kv_heads, head_dim, chunk, sink, recent, float(rope_theta), dtype_code(dtype),
                        T, rank_k, rank_v, a_k_batch_stride, a_v_batch_stride, bt_k_batch_stride, bt_v_batch_stride,
                        window_batch_stride, landmark_capacity)


def xkv_sr_append(p: AppendParams, k_new, v_new, win_K, win_V, Bt_K, Bt_V, A_K, A_V, landmarks, ws=None,
                  stream=None) -> bool:
    """Append one token per layer (lists of G tensors); returns True when a chunk was rolled."""
    G = p.group
    arr = lambda ts: (C.c_void_p * G)(*[t.data_ptr() for t in ts])
    n = C.c_size_t(0)
    _check(lib.xkv_sr_append_workspace_size(C.byref(p), C.byref(n)), "xkv_sr_append_workspace_size")
    ws = ws if ws is not None else workspace(n.value, A_K.device)
    rolled = C.c_int(0)
    _check(lib.xkv_sr_append(C.byref(p), arr(k_new), arr(v_new), arr(win_K), arr(win_V), _ptr(Bt_K), _ptr(Bt_V),
                             _ptr(A_K), _ptr(A_V), arr(landmarks), C.byref(rolled), _ptr(ws), ws.numel(),
                             _stream(stream)), "xkv_sr_append")
    return bool(rolled.value)


# ------------------------------------------------------- token sharding
def xkv_sr_scores(p: SRParams, q, landmarks, scores, stream=None):
    """scores [B][Hkv][ld] f32 (ld >= n_mid, a multiple of 4): the local chunk scores."""
    _check(lib.xkv_sr_scores(C.byref(p), _ptr(q), _addr(landmarks), _addr(scores), scores.stride(-2),
                             _stream(stream)), "xkv_sr_scores")


def xkv_sr_topk(scores, n: int, k: int, sel_out, stream=None):
    """Exact top-k of each row of scores [..., ld] over its first n entries."""
    rows = scores.numel() // scores.shape[-1]
    _check(lib.xkv_sr_topk(_addr(scores), scores.stride(-2), rows, n, k, _ptr(sel_out), _stream(stream)),
           "xkv_sr_topk")


def xkv_sr_attention_partial(p: SRParams, shard: ShardParams, sel, q, A_K, Bt_K, A_V, Bt_V, sr_K, sr_V, out, ml_out,
                             ws=None, stream=None):
    """Attention of this device's token slice for the global selection sel; out
    normalised by its own sum, ml_out = (M, L) per (sequence, query head)."""
    if ws is None:
        n = C.c_size_t(0)
        _check(lib.xkv_sr_partial_workspace_size(C.byref(p), C.byref(n)), "xkv_sr_partial_workspace_size")
        ws = workspace(n.value, q.device)
    _check(lib.xkv_sr_attention_partial(C.byref(p), C.byref(shard), _ptr(sel), _ptr(q), _addr(A_K), _addr(Bt_K),
                                        _addr(A_V), _addr(Bt_V), _addr(sr_K), _addr(sr_V), _ptr(out), _ptr(ml_out),
                                        _ptr(ws), ws.numel(), _stream(stream)), "xkv_sr_attention_partial")


def xkv_merge_partials(o, ml, out, stream=None):
    """o [R][rows][hd], ml [R][rows][2] -> out [rows][hd] (the exact softmax combination)."""
    R, rows, hd = o.shape[0], o.numel() // (o.shape[0] * o.shape[-1]), o.shape[-1]
    _check(lib.xkv_merge_partials(_ptr(o), _ptr(ml), R, rows, hd, _ptr(out), _stream(stream)), "xkv_merge_partials")

