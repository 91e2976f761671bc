"""xKV CPU oracle -- TEST INFRASTRUCTURE ONLY.

A plain, slow fp64 CPU implementation of the xKV hot path (see xkv_oracle.c for
the passages each function follows).  Only tests/, __graft_entry__.smoke() and
bench.py's CPU-baseline / reference legs may import this package; the product
library never does, and the two share no code.  Inputs come from numpy arrays
(bf16 data widened exactly to float32); results are float64.

Every function here is pinned by tests/test_oracle_*.py against closed forms,
invariants, brute force and LAPACK; none is "parity unpinned".
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "xkv_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (-O2, OpenMP, IEEE arithmetic)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        _lib.xo_num_threads.restype = C.c_int
        _lib.xo_jacobi_eigh.restype = C.c_int
        _lib.xo_compress_group.restype = C.c_int
        _lib.xo_sr_decode.restype = C.c_int
        _lib.xo_ner.restype = C.c_int
    return _lib


class _SRParams(C.Structure):
    _fields_ = [("batch", C.c_int), ("n_q_heads", C.c_int), ("n_kv_heads", C.c_int),
                ("head_dim", C.c_int), ("T", C.c_int64), ("rank_k", C.c_int), ("rank_v", C.c_int),
                ("chunk", C.c_int), ("topk", C.c_int), ("sink", C.c_int), ("recent", C.c_int),
                ("rope_theta", C.c_double)]


def _p(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def num_threads() -> int:
    return int(lib().xo_num_threads())


def round_bf16(x) -> np.ndarray:
    """Round to bfloat16 (nearest, ties to even), returned as float32."""
    x = _f64(x)
    y = np.empty(x.shape, dtype=np.float32)
    lib().xo_round_bf16_array(_p(x), _p(y), C.c_int64(x.size))
    return y


def _layer_ptrs(layers: Sequence[np.ndarray]):
    arr = (C.c_void_p * len(layers))(*[l.ctypes.data for l in layers])
    return arr


def gram(layers: Sequence[np.ndarray], t0: int = 0, t1: Optional[int] = None,
         C_in: Optional[np.ndarray] = None) -> np.ndarray:
    """C (+)= sum_{t0<=t<t1} x_t^T x_t over X = [K_1 | ... | K_G] (fp64)."""
    layers = [_f32(l) for l in layers]
    G = len(layers)
    T, d = layers[0].shape
    t1 = T if t1 is None else t1
    n = G * d
    Cm = np.zeros((n, n), dtype=np.float64) if C_in is None else _f64(C_in).copy()
    lib().xo_gram_accumulate(_layer_ptrs(layers), C.c_int(G), C.c_int64(T), C.c_int(d),
                             C.c_int64(d), C.c_int64(t0), C.c_int64(t1), _p(Cm))
    return Cm


def jacobi_eigh(A: np.ndarray, tol: float = 1e-14, max_sweeps: int = 60):
    """(eigenvalues descending, eigenvectors as columns, sweeps) by cyclic Jacobi."""
    A = _f64(A).copy()
    n = A.shape[0]
    w = np.empty(n, dtype=np.float64)
    V = np.empty((n, n), dtype=np.float64)
    sweeps = lib().xo_jacobi_eigh(_p(A), C.c_int(n), _p(w), _p(V), C.c_double(tol), C.c_int(max_sweeps))
    return w, V, int(sweeps)


def compress_group(layers: Sequence[np.ndarray], rank: int):
    """Cross-layer factorisation of one group.

    Returns dict: A (T x r), Bt ((G d) x r, = V_r), lam (all eigenvalues,
    descending), err_subspace, err_stored (bf16 factors), tail, xx, sweeps.
    """
    layers = [_f32(l) for l in layers]
    G = len(layers)
    T, d = layers[0].shape
    n = G * d
    A = np.empty((T, rank), dtype=np.float64)
    Bt = np.empty((n, rank), dtype=np.float64)
    lam = np.empty(n, dtype=np.float64)
    st = np.zeros(5, dtype=np.float64)
    rc = lib().xo_compress_group(_layer_ptrs(layers), C.c_int(G), C.c_int64(T), C.c_int(d),
                                 C.c_int64(d), C.c_int(rank), _p(A), _p(Bt), _p(lam), _p(st))
    if rc != 0:
        raise RuntimeError("oracle Jacobi did not converge")
    return dict(A=A, Bt=Bt, lam=lam, err_subspace=st[0], err_stored=st[1], tail=st[2], xx=st[3],
                sweeps=int(st[4]))


def rope(x, pos: float, theta: float) -> np.ndarray:
    """Rotate-half RoPE of one head vector at absolute position pos."""
    x = _f64(x)
    y = np.empty_like(x)
    lib().xo_rope(_p(x), _p(y), C.c_int(x.size), C.c_double(pos), C.c_double(theta))
    return y


def landmarks(K: np.ndarray, n_kv_heads: int, head_dim: int, chunk: int, sink: int, recent: int,
              theta: float) -> np.ndarray:
    """[Hkv][n_mid][hd] chunk means of post-RoPE keys (fp64)."""
    K = _f32(K)
    T = K.shape[0]
    n_mid = (T - sink - recent) // chunk
    out = np.empty((n_kv_heads, n_mid, head_dim), dtype=np.float64)
    lib().xo_landmarks(_p(K), C.c_int64(T), C.c_int64(K.shape[1]), C.c_int(n_kv_heads),
                       C.c_int(head_dim), C.c_int(chunk), C.c_int(sink), C.c_int(recent),
                       C.c_double(theta), _p(out))
    return out


def full_reconstruct(A, Bt, n_kv_heads: int, head_dim: int, apply_rope: bool, theta: float):
    """T x d rebuilt cache A Bt^T (+ RoPE per head at position t)."""
    A = _f32(A)
    Bt = _f32(Bt)
    T, r = A.shape
    d = Bt.shape[0]
    out = np.empty((T, d), dtype=np.float64)
    lib().xo_full_reconstruct(_p(A), _p(Bt), C.c_int64(T), C.c_int(r), C.c_int(d),
                              C.c_int(n_kv_heads), C.c_int(head_dim), C.c_int(int(apply_rope)),
                              C.c_double(theta), _p(out))
    return out


def dense_decode(q, K, V, n_kv_heads: int, units: Optional[Sequence[int]] = None):
    """Decode attention over full caches. q [B][Hq][hd]; K (post-RoPE), V [B][T][d]."""
    q = _f32(q)
    K = _f32(K)
    V = _f32(V)
    B, Hq, hd = q.shape
    T = K.shape[1]
    out = np.full((B, Hq, hd), np.nan, dtype=np.float64)
    u = None if units is None else np.ascontiguousarray(units, dtype=np.int32)
    lib().xo_dense_decode(C.c_int(B), C.c_int(Hq), C.c_int(n_kv_heads), C.c_int(hd), C.c_int64(T),
                          _p(q), _p(K), _p(V), None if u is None else _p(u),
                          C.c_int(0 if u is None else u.size), _p(out))
    return out


def sr_decode(w, q, A_K, Bt_K, A_V, Bt_V, landmarks, sr_K, sr_V, T: Optional[int] = None,
              sel_in=None, units: Optional[Sequence[int]] = None):
    """One Selective-Reconstruction decode step (fp64).

    w: a synth.Workload (shape fields).  Bt_K / Bt_V are [d][r] (shared by the
    batch) or [B][d][r] (one factorisation per sequence).  Returns (out [B][Hq][hd], sel [B][Hkv][k],
    scores [B][Hkv][n_mid]).  Rows of units not listed are NaN / -1.
    """
    T = T or w.T
    q, A_K, Bt_K, A_V, Bt_V, lm, sr_K, sr_V = (_f32(a) for a in (q, A_K, Bt_K, A_V, Bt_V, landmarks, sr_K, sr_V))
    B = q.shape[0]
    p = _SRParams(B, w.n_q_heads, w.n_kv_heads, w.head_dim, T, A_K.shape[-1], A_V.shape[-1],
                  w.chunk, w.topk, w.sink, w.recent, float(w.rope_theta))
    n_mid = (T - w.sink - w.recent) // w.chunk
    out = np.full((B, w.n_q_heads, w.head_dim), np.nan, dtype=np.float64)
    sel = np.full((B, w.n_kv_heads, w.topk), -1, dtype=np.int32)
    scores = np.full((B, w.n_kv_heads, n_mid), np.nan, dtype=np.float64)
    si = None if sel_in is None else np.ascontiguousarray(sel_in, dtype=np.int32)
    u = None if units is None else np.ascontiguousarray(units, dtype=np.int32)
    sbk = Bt_K.shape[-2] * Bt_K.shape[-1] if Bt_K.ndim == 3 else 0
    sbv = Bt_V.shape[-2] * Bt_V.shape[-1] if Bt_V.ndim == 3 else 0
    rc = lib().xo_sr_decode(C.byref(p), _p(q), _p(A_K), C.c_int64(T * A_K.shape[-1]), _p(Bt_K), C.c_int64(sbk),
                            _p(A_V), C.c_int64(T * A_V.shape[-1]), _p(Bt_V), C.c_int64(sbv), _p(lm), _p(sr_K),
                            _p(sr_V),
                            None if si is None else _p(si), None if u is None else _p(u),
                            C.c_int(0 if u is None else u.size), _p(out), _p(sel), _p(scores))
    if rc != 0:
        raise ValueError("invalid SR decode shape")
    return out, sel, scores


def xk_sr_decode(w, q, A_K, Bt_K, V, landmarks, sr_K, sr_V, T: Optional[int] = None,
                 sel_in=None, units: Optional[Sequence[int]] = None):
    """One decode step of the xK-SR mode (fp64): keys as in sr_decode (landmark
    top-k, rows rebuilt from A_K Bt_K^T with RoPE), values read uncompressed
    from V [B][T][d] for the same rows.  Returns (out, sel, scores) like
    sr_decode."""
    T = T or w.T
    q, A_K, Bt_K, V, lm, sr_K, sr_V = (_f32(a) for a in (q, A_K, Bt_K, V, landmarks, sr_K, sr_V))
    B = q.shape[0]
    if V.shape[-1] != w.d or V.shape[-2] != T:
        raise ValueError("V must be [B][T][d]")
    p = _SRParams(B, w.n_q_heads, w.n_kv_heads, w.head_dim, T, A_K.shape[-1], 0,
                  w.chunk, w.topk, w.sink, w.recent, float(w.rope_theta))
    n_mid = (T - w.sink - w.recent) // w.chunk
    out = np.full((B, w.n_q_heads, w.head_dim), np.nan, dtype=np.float64)
    sel = np.full((B, w.n_kv_heads, w.topk), -1, dtype=np.int32)
    scores = np.full((B, w.n_kv_heads, n_mid), np.nan, dtype=np.float64)
    si = None if sel_in is None else np.ascontiguousarray(sel_in, dtype=np.int32)
    u = None if units is None else np.ascontiguousarray(units, dtype=np.int32)
    sbk = Bt_K.shape[-2] * Bt_K.shape[-1] if Bt_K.ndim == 3 else 0
    rc = lib().xo_sr_decode(C.byref(p), _p(q), _p(A_K), C.c_int64(T * A_K.shape[-1]), _p(Bt_K), C.c_int64(sbk),
                            _p(V), C.c_int64(T * w.d), None, C.c_int64(0), _p(lm), _p(sr_K), _p(sr_V),
                            None if si is None else _p(si), None if u is None else _p(u),
                            C.c_int(0 if u is None else u.size), _p(out), _p(sel), _p(scores))
    if rc != 0:
        raise ValueError("invalid SR decode shape")
    return out, sel, scores


def ner(Cm: np.ndarray, block: int, rel_tol: float = 1e-9):
    """Per diagonal block: (NER, erank, rank, eigenvalues) of KV-CoRE."""
    Cm = _f64(Cm)
    n = Cm.shape[0]
    nb = n // block
    nr = np.empty(nb, dtype=np.float64)
    er = np.empty(nb, dtype=np.float64)
    rk = np.empty(nb, dtype=np.int32)
    ev = np.empty((nb, block), dtype=np.float64)
    rc = lib().xo_ner(_p(Cm), C.c_int(n), C.c_int(block), C.c_double(rel_tol), _p(nr), _p(er), _p(rk), _p(ev))
    if rc != 0:
        raise RuntimeError("oracle Jacobi did not converge")
    return nr, er, rk, ev


def energy_rank(Cm: np.ndarray, block: int, energy: float = 0.95):
    """[xKV-blog] Fig. 2(c): per diagonal block C_ll, the smallest k whose k
    largest eigenvalues hold `energy` of the block's total (eigenvalues below
    zero, which only rounding produces, count as 0; 0 for a zero block).
    Eigenvalues from the oracle's Jacobi; returns (ranks, eigenvalues sorted
    descending)."""
    _, _, _, ev = ner(Cm, block)
    lam = np.sort(np.maximum(ev, 0.0), axis=1)[:, ::-1]
    ranks = np.zeros(lam.shape[0], dtype=np.int32)
    for i, l in enumerate(lam):
        total = l.sum()
        if total > 0.0:
            cum = np.cumsum(l)
            ranks[i] = int(np.searchsorted(cum, energy * total, side="left")) + 1
    return ranks, lam


# ------------------------------------------------------------ multi-step decode
def project_rows(layers: Sequence[np.ndarray], V: np.ndarray) -> np.ndarray:
    """A = [layers...] V for a few token rows (fp64); V is (G d) x r."""
    layers = [_f32(l) for l in layers]
    G = len(layers)
    rows, d = layers[0].shape
    V = _f32(V)
    r = V.shape[1]
    A = np.empty((rows, r), dtype=np.float64)
    lib().xo_project_rows(_layer_ptrs(layers), C.c_int(G), C.c_int64(rows), C.c_int(d), C.c_int64(d), _p(V),
                          C.c_int(r), _p(A))
    return A


def chunk_landmark(K_rows: np.ndarray, n_kv_heads: int, head_dim: int, t0: int, theta: float) -> np.ndarray:
    """[Hkv][hd] mean of RoPE_{t0+i}(K_rows[i]) over the chunk's rows (fp64)."""
    K_rows = _f32(K_rows)
    Cn = K_rows.shape[0]
    out = np.empty((n_kv_heads, head_dim), dtype=np.float64)
    lib().xo_chunk_landmark(_p(K_rows), C.c_int64(K_rows.shape[1]), C.c_int(n_kv_heads), C.c_int(head_dim),
                            C.c_int(Cn), C.c_int64(t0), C.c_double(theta), _p(out))
    return out


class SRState:
    """Host-side state of one layer group for multi-step decode (test
    infrastructure): the compressed rows A_K / A_V [B][T_cap][r], the group
    bases Bt_K / Bt_V [B][G d][r], per layer the landmarks [B][Hkv][cap][hd] and
    the raw window K / V [B][sink + recent + chunk][d] (sink rows first, then the
    current recent rows), the length T, the middle-chunk count n_mid and the
    number of recent rows w_cur.  Stored values are bf16 numbers held in
    float32, as the library stores them."""

    def __init__(self, w, A_K, A_V, Bt_K, Bt_V, lms, win_K, win_V, T, n_mid, w_cur):
        self.w, self.A_K, self.A_V, self.Bt_K, self.Bt_V = w, A_K, A_V, Bt_K, Bt_V
        self.lms, self.win_K, self.win_V = lms, win_K, win_V
        self.T, self.n_mid, self.w_cur = T, n_mid, w_cur

    def append(self, k_new: Sequence[np.ndarray], v_new: Sequence[np.ndarray]):
        """One generated token for every layer of the group: k_new[l], v_new[l]
        are [B][d] (pre-RoPE keys).  The rows join the raw window; when the
        window holds recent + chunk rows, its oldest chunk is rolled into the
        compressed cache: A rows by projection onto the stored bases, one
        landmark per layer and KV head, and the window moves down by a chunk."""
        w = self.w
        s, Cn, G = w.sink, w.chunk, w.group
        row = s + self.w_cur
        for l in range(G):
            self.win_K[l][:, row] = k_new[l]
            self.win_V[l][:, row] = v_new[l]
        self.w_cur += 1
        self.T += 1
        if self.w_cur < w.recent + Cn:
            return False
        t0 = s + self.n_mid * Cn
        for b in range(self.A_K.shape[0]):
            for X, A, Bt in ((self.win_K, self.A_K, self.Bt_K), (self.win_V, self.A_V, self.Bt_V)):
                rows = [X[l][b, s:s + Cn] for l in range(G)]
                A[b, t0:t0 + Cn] = round_bf16(project_rows(rows, Bt[b]))
            for l in range(G):
                lm = chunk_landmark(self.win_K[l][b, s:s + Cn], w.n_kv_heads, w.head_dim, t0, w.rope_theta)
                self.lms[l][b, :, self.n_mid] = round_bf16(lm)
        for X in (self.win_K, self.win_V):
            for l in range(G):
                X[l][:, s:s + w.recent] = X[l][:, s + Cn:s + Cn + w.recent].copy()
        self.n_mid += 1
        self.w_cur = w.recent
        return True

