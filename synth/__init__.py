"""Seeded synthetic inputs for the xKV hot path.

This module is the ONLY code shared by the CUDA path's tests/bench and the CPU
oracle.  It draws random numbers and shapes them into K/V caches, queries and
compressed-cache stand-ins; it holds none of the method's arithmetic (no Gram,
no eigenvectors, no RoPE, no landmarks, no attention).

Random numbers
--------------
* Philox4x32-10, the counter-based generator of Salmon, Moraes, Dror and Shaw,
  "Parallel random numbers: as easy as 1, 2, 3" (SC'11): a 128-bit counter and a
  64-bit key pass through ten rounds of two 32x32->64 multiplies and xors, the
  key being bumped by the Weyl constants between rounds.
* Stream keys are made with the SplitMix64 finaliser (Steele, Lea, Flood,
  "Fast splittable pseudorandom number generators", OOPSLA'14) folded over the
  integer identifiers of the stream.
* Gaussians come from the Box-Muller transform (Box & Muller 1958) applied to
  pairs of uniforms u = (x + 0.5) / 2**32 taken from consecutive Philox words.

Synthetic caches (the workloads of the xKV explainer page, "xKV 到底做了什么",
and its RULER/Llama-3.1-8B/Qwen2.5-7B setting, which are not available here)
are drawn as

    K_l = Z (W_s + 0.1 E_l) + 0.01 N

with Z a T x m Gaussian matrix whose column i is scaled by i^-alpha, W_s and E_l
m x d Gaussian matrices (W_s shared by the group, E_l per layer) and N a T x d
Gaussian noise matrix.  V is drawn the same way from independent streams.

A CPU (numpy, float64 transform) and a CUDA (torch) implementation of the same
integer stream are provided; the float transform on the device may differ from
the CPU one in the last bit, so every oracle parity input is drawn on the CPU.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import numpy as np

BASE_SEED = 0x784B56  # ASCII "xKV"

_M0 = 0xD2511F53
_M1 = 0xCD9E8D57
_W0 = 0x9E3779B9
_W1 = 0xBB67AE85
_MASK32 = 0xFFFFFFFF
_MASK64 = 0xFFFFFFFFFFFFFFFF


# ----------------------------------------------------------------------------- keys
def _splitmix64_mix(z: int) -> int:
    z = (z + 0x9E3779B97F4A7C15) & _MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


_TAGS = {
    "Z": 1, "W": 2, "E": 3, "N": 4, "q": 5, "A": 6, "B": 7, "L": 8, "SK": 9, "SV": 10,
    "K": 100, "V": 200, "Q0": 11, "X": 12,
}


def stream_key(*ids) -> int:
    """64-bit Philox key for a named stream; ids are ints or short tag strings."""
    h = _splitmix64_mix(BASE_SEED)
    for v in ids:
        if isinstance(v, str):
            v = _TAGS.get(v, None) if v in _TAGS else int.from_bytes(v.encode()[:8].ljust(8, b"\0"), "little")
        h = _splitmix64_mix(h ^ (int(v) & _MASK64))
    return h


# --------------------------------------------------------------------------- philox
def philox4x32_10(counter: np.ndarray, key: Sequence[int]) -> np.ndarray:
    """Philox4x32-10 on an (n, 4) uint32 counter array with a 2-word key."""
    c = np.asarray(counter, dtype=np.uint64) & _MASK32
    c0, c1, c2, c3 = (c[:, i].copy() for i in range(4))
    k0 = np.uint64(int(key[0]) & _MASK32)
    k1 = np.uint64(int(key[1]) & _MASK32)
    m0 = np.uint64(_M0)
    m1 = np.uint64(_M1)
    mask = np.uint64(_MASK32)
    s32 = np.uint64(32)
    for rnd in range(10):
        if rnd:
            k0 = np.uint64((int(k0) + _W0) & _MASK32)
            k1 = np.uint64((int(k1) + _W1) & _MASK32)
        p0 = m0 * c0
        p1 = m1 * c2
        hi0, lo0 = p0 >> s32, p0 & mask
        hi1, lo1 = p1 >> s32, p1 & mask
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return np.stack([c0, c1, c2, c3], axis=1).astype(np.uint32)


def uniform_words(key64: int, n_words: int, offset_blocks: int = 0) -> np.ndarray:
    """n_words uint32 values from stream key64 (block i -> counter (i, 0, 0, 0))."""
    n_blocks = (n_words + 3) // 4
    idx = np.arange(offset_blocks, offset_blocks + n_blocks, dtype=np.uint64)
    ctr = np.zeros((n_blocks, 4), dtype=np.uint64)
    ctr[:, 0] = idx & np.uint64(_MASK32)
    ctr[:, 1] = idx >> np.uint64(32)
    out = philox4x32_10(ctr, (key64 & _MASK32, key64 >> 32))
    return out.reshape(-1)[:n_words]


def normal(key64: int, n: int) -> np.ndarray:
    """n standard normals (float64) from stream key64, Box-Muller on word pairs."""
    n_pairs = (n + 1) // 2
    w = uniform_words(key64, 2 * n_pairs).astype(np.float64)
    u1 = (w[0::2] + 0.5) * (1.0 / 4294967296.0)
    u2 = (w[1::2] + 0.5) * (1.0 / 4294967296.0)
    rad = np.sqrt(-2.0 * np.log(u1))
    ang = 2.0 * math.pi * u2
    z = np.empty(2 * n_pairs, dtype=np.float64)
    z[0::2] = rad * np.cos(ang)
    z[1::2] = rad * np.sin(ang)
    return z[:n]


def normal_chunked(key64: int, n: int, chunk: int = 1 << 24) -> np.ndarray:
    """Same values as normal(key64, n) drawn in bounded-memory pieces."""
    out = np.empty(n, dtype=np.float32)
    chunk -= chunk % 4
    for s in range(0, n, chunk):
        m = min(chunk, n - s)
        n_pairs = (m + 1) // 2
        w = uniform_words(key64, 2 * n_pairs, offset_blocks=s // 2 // 2).astype(np.float64)
        u1 = (w[0::2] + 0.5) * (1.0 / 4294967296.0)
        u2 = (w[1::2] + 0.5) * (1.0 / 4294967296.0)
        rad = np.sqrt(-2.0 * np.log(u1))
        ang = 2.0 * math.pi * u2
        z = np.empty(2 * n_pairs, dtype=np.float64)
        z[0::2] = rad * np.cos(ang)
        z[1::2] = rad * np.sin(ang)
        out[s:s + m] = z[:m]
    return out


# ------------------------------------------------------------------ torch (device)
def _mulhilo32_torch(a: int, b):
    """(hi, lo) of a*b for a 32-bit constant a and an int64 tensor b of u32 values."""
    ah, al = a >> 16, a & 0xFFFF
    p1 = b * ah            # < 2^48
    p0 = b * al            # < 2^48
    t = p0 + ((p1 & 0xFFFF) << 16)
    lo = t & _MASK32
    hi = (p1 >> 16) + (t >> 32)
    return hi & _MASK32, lo


def normal_torch(key64: int, n: int, device, dtype=None):
    """Device twin of normal(): same Philox words; float transform on the device."""
    import torch
    n_pairs = (n + 1) // 2
    n_blocks = (2 * n_pairs + 3) // 4
    idx = torch.arange(n_blocks, dtype=torch.int64, device=device)
    c0 = idx & _MASK32
    c1 = idx >> 32
    c2 = torch.zeros_like(idx)
    c3 = torch.zeros_like(idx)
    k0 = key64 & _MASK32
    k1 = key64 >> 32
    for rnd in range(10):
        if rnd:
            k0 = (k0 + _W0) & _MASK32
            k1 = (k1 + _W1) & _MASK32
        hi0, lo0 = _mulhilo32_torch(_M0, c0)
        hi1, lo1 = _mulhilo32_torch(_M1, c2)
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    w = torch.stack([c0, c1, c2, c3], dim=1).reshape(-1)[: 2 * n_pairs].to(torch.float64)
    u1 = (w[0::2] + 0.5) * (1.0 / 4294967296.0)
    u2 = (w[1::2] + 0.5) * (1.0 / 4294967296.0)
    rad = torch.sqrt(-2.0 * torch.log(u1))
    ang = 2.0 * math.pi * u2
    z = torch.stack([rad * torch.cos(ang), rad * torch.sin(ang)], dim=1).reshape(-1)[:n]
    return z.to(dtype or torch.float32)


# -------------------------------------------------------------------- workloads
@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape of one synthetic xKV workload (one decode step per layer)."""
    name: str
    batch: int
    n_layers: int
    group: int            # G, layers per group
    n_kv_heads: int
    head_dim: int
    n_q_heads: int
    T: int
    latent: int           # m
    alpha: float
    rank_k: int
    rank_v: int
    chunk: int = 8
    topk: int = 16
    sink: int = 8
    recent: int = 32
    rope_theta: float = 500000.0
    dtype: str = "bf16"   # "f32" | "bf16"

    @property
    def d(self) -> int:
        return self.n_kv_heads * self.head_dim

    @property
    def gq(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def n_groups(self) -> int:
        return self.n_layers // self.group

    @property
    def n_mid(self) -> int:
        return (self.T - self.sink - self.recent) // self.chunk

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads: a tiny fp32 single group; a Llama-3.1-8B-shaped group at
# 16K; the full 32-layer Llama-3.1-8B shape at 64K, batch 4; a Qwen2.5-7B shape
# at 128K, batch 2; and the prefill-compression sweep (d=1024, T=32K, G=1..8).
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 4, 4, 2, 64, 8, 1024, 96, 0.8, 64, 64,
                         topk=16, dtype="f32"),
    "llama_group_16k": Workload("llama_group_16k", 1, 4, 4, 8, 128, 32, 16384, 768, 0.8,
                                512, 512, topk=256),
    "llama8b_64k_b4": Workload("llama8b_64k_b4", 4, 32, 4, 8, 128, 32, 65536, 768, 0.8,
                               512, 512, topk=256),
    "qwen7b_128k_b2": Workload("qwen7b_128k_b2", 2, 28, 4, 4, 128, 28, 131072, 512, 1.0,
                               256, 384, topk=512),
}


def compression_sweep(G: int) -> Workload:
    """Prefill sweep point: d=1024 (8 x 128), T=32768, rank 128*G, 4 shards of 8192."""
    return Workload(f"compress_sweep_g{G}", 1, G, G, 8, 128, 32, 32768, 768, 0.8,
                    128 * G, 128 * G, topk=256)


def oversample(rank: int) -> int:
    """Oversampling p for block subspace iteration: max(64, r/4)."""
    return max(64, rank // 4)


# ------------------------------------------------------------------ generators
def _bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even), kept as float32."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = ((u >> np.uint64(16)) & np.uint64(1)) + np.uint64(0x7FFF)
    r = ((u + bias) >> np.uint64(16)) << np.uint64(16)
    return (r & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def to_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """float32 values as they are stored for the workload dtype (bf16 -> rounded)."""
    x = np.asarray(x, dtype=np.float32)
    return _bf16_round(x) if dtype == "bf16" else x


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of float32 values that are exact bfloat16 numbers."""
    return (np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def kv_group(w: Workload, batch: int, group: int, kind: str, T: Optional[int] = None,
             layers: Optional[Sequence[int]] = None) -> List[np.ndarray]:
    """Per-layer caches (T x d, float32, in storage precision) for one group.

    kind is "K" (pre-RoPE keys) or "V"; layers defaults to all G layers.
    """
    T = T or w.T
    m, d = w.latent, w.d
    scales = np.arange(1, m + 1, dtype=np.float64) ** (-w.alpha)
    Z = normal_chunked(stream_key(w.name, batch, group, kind, "Z"), T * m).reshape(T, m)
    Z = (Z * scales[None, :].astype(np.float32)).astype(np.float32)
    Ws = normal(stream_key(w.name, batch, group, kind, "W"), m * d).reshape(m, d)
    out = []
    for l in (range(w.group) if layers is None else layers):
        E = normal(stream_key(w.name, batch, group, kind, "E", l), m * d).reshape(m, d)
        Wl = (Ws + 0.1 * E).astype(np.float32)
        N = normal_chunked(stream_key(w.name, batch, group, kind, "N", l), T * d).reshape(T, d)
        X = Z @ Wl + np.float32(0.01) * N
        out.append(to_storage(X, w.dtype))
    return out


def kv_group_torch(w: Workload, batch: int, group: int, kind: str, device, T: Optional[int] = None):
    """Device twin of kv_group (bench set-up): same streams, values in torch dtype."""
    import torch
    T = T or w.T
    m, d = w.latent, w.d
    scales = torch.arange(1, m + 1, dtype=torch.float64, device=device) ** (-w.alpha)
    Z = normal_torch(stream_key(w.name, batch, group, kind, "Z"), T * m, device).view(T, m)
    Z = Z * scales.to(torch.float32)[None, :]
    Ws = normal_torch(stream_key(w.name, batch, group, kind, "W"), m * d, device, torch.float64).view(m, d)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    out = []
    for l in range(w.group):
        E = normal_torch(stream_key(w.name, batch, group, kind, "E", l), m * d, device, torch.float64).view(m, d)
        Wl = (Ws + 0.1 * E).to(torch.float32)
        X = Z @ Wl
        X += 0.01 * normal_torch(stream_key(w.name, batch, group, kind, "N", l), T * d, device).view(T, d)
        out.append(X.to(tdt))
        del X
    return out


def queries(w: Workload, layer: int) -> np.ndarray:
    """Decode queries q ~ N(0,1), [B][Hq][hd] float32 in storage precision."""
    q = normal(stream_key(w.name, "q", layer), w.batch * w.n_q_heads * w.head_dim)
    return to_storage(q.reshape(w.batch, w.n_q_heads, w.head_dim), w.dtype)


def raw_values(w: Workload, layer: int, T: Optional[int] = None) -> np.ndarray:
    """An uncompressed value cache V ~ N(0,1), [B][T][d] float32 in storage
    precision (the xK-SR mode keeps values whole)."""
    T = T or w.T
    v = normal_chunked(stream_key(w.name, "Vraw", layer, T), w.batch * T * w.d)
    return to_storage(v.reshape(w.batch, T, w.d), w.dtype)


def compressed_cache(w: Workload, layer: int, T: Optional[int] = None):
    """Stand-ins for a compressed layer, drawn directly (decode-only tests).

    Returns dict with A_K [B][T][rK], A_V [B][T][rV] (columns scaled like U*Sigma
    of the synthetic spectrum), Bt_K [B][d][rK], Bt_V [B][d][rV] (one per
    sequence, entries ~ N(0, 1/r)),
    landmarks [B][Hkv][n_mid][hd] (~ N(0,1)), sink/recent K and V [B][s+w][d],
    and q [B][Hq][hd]; all float32 in storage precision.
    """
    T = T or w.T
    n_mid = (T - w.sink - w.recent) // w.chunk
    out = {}
    for kind, r in (("K", w.rank_k), ("V", w.rank_v)):
        sc = (np.arange(1, r + 1, dtype=np.float64) ** (-w.alpha)) * 3.0
        A = normal_chunked(stream_key(w.name, "A", kind, layer, T), w.batch * T * r)
        A = A.reshape(w.batch, T, r) * sc[None, None, :].astype(np.float32)
        out["A_" + kind] = to_storage(A, w.dtype)
        Bt = normal(stream_key(w.name, "B", kind, layer), w.batch * w.d * r).reshape(w.batch, w.d, r) / math.sqrt(r)
        out["Bt_" + kind] = to_storage(Bt, w.dtype)
    L = normal_chunked(stream_key(w.name, "L", layer, T), w.batch * w.n_kv_heads * n_mid * w.head_dim)
    out["landmarks"] = to_storage(L.reshape(w.batch, w.n_kv_heads, n_mid, w.head_dim), w.dtype)
    sw = w.sink + w.recent
    out["sr_K"] = to_storage(normal(stream_key(w.name, "SK", layer, T), w.batch * sw * w.d)
                             .reshape(w.batch, sw, w.d), w.dtype)
    out["sr_V"] = to_storage(normal(stream_key(w.name, "SV", layer, T), w.batch * sw * w.d)
                             .reshape(w.batch, sw, w.d), w.dtype)
    out["q"] = queries(w, layer)
    return out
