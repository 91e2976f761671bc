"""Token-sharded xKV across GPUs (one process per GPU, torch.distributed).

Each device holds a contiguous slice of the token sequence: the sink rows on
the first, the recent window on the last, whole middle chunks in between.

Prefill (KV-CoRE 2.A: the covariance is a sum over token rows, so the Grams of
the slices add up):
    local Gram -> all-reduce (sum) -> the same factorisation on every device
    (same Gram and seed, same basis) -> projection of the local rows.
Decode, one step (the xKV explainer's "选择性重建" over the whole sequence):
    local chunk scores -> all-gather -> exact top-k over all chunks (the same
    on every device) -> attention over the kept chunks held locally plus the
    local window rows, as a partial (o, M, L) -> all-gather -> exact merge.

The arithmetic runs in the library's kernels (the `ops` object, LibraryOps by
default); this module moves tensors between devices with torch.distributed and
lays them out.  Tests may pass other ops and collectives (for example CPU
stand-ins under the gloo backend) to exercise the same orchestration.
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import torch

from . import (ShardParams, XKVError, sr_params, workspace, xkv_factor_gram, xkv_gram_accumulate,
               xkv_gram_workspace_size, xkv_merge_partials, xkv_project, xkv_sr_attention_partial, xkv_sr_scores,
               xkv_sr_topk)


# ------------------------------------------------------------- collectives
class Collectives:
    """torch.distributed collectives over `group` (all ranks by default)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def all_reduce_sum(self, t: torch.Tensor) -> torch.Tensor:
        self.dist.all_reduce(t, op=self.dist.ReduceOp.SUM, group=self.group)
        return t

    def all_gather(self, t: torch.Tensor) -> torch.Tensor:
        """[R, *t.shape], rank r's tensor at index r."""
        t = t.contiguous()
        out = torch.empty((self.world * t.shape[0],) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
        self.dist.all_gather_into_tensor(out, t, group=self.group)
        return out.view((self.world,) + tuple(t.shape))


# --------------------------------------------------------------------- ops
class LibraryOps:
    """The library's kernels (CUDA tensors)."""

    def gram(self, X: Sequence[torch.Tensor], shard_rows: int) -> torch.Tensor:
        G = len(X)
        rows, d = X[0].shape
        C = torch.zeros((G * d, G * d), dtype=torch.float32, device=X[0].device)
        ws = workspace(xkv_gram_workspace_size(G, min(shard_rows, max(rows, 1)), d, X[0].dtype), X[0].device)
        for s in range(0, rows, shard_rows):
            xkv_gram_accumulate([x[s:s + shard_rows] for x in X], C, ws)
        return C

    def factor(self, C: torch.Tensor, G: int, d: int, rows: int, rank: int, iters: int, oversample: int, seed: int,
               dtype: torch.dtype):
        n = G * d
        Bt = torch.empty((n, rank), dtype=dtype, device=C.device)
        Vr = torch.empty((n, rank), dtype=torch.float32, device=C.device)
        ev = torch.empty((rank,), dtype=torch.float32, device=C.device)
        xkv_factor_gram(C, G, d, rows, rank, Bt, iters=iters, oversample=oversample, seed=seed, Vr_out=Vr,
                        eigvals=ev)
        return Bt, Vr, ev

    def project(self, X: Sequence[torch.Tensor], Vr: torch.Tensor) -> torch.Tensor:
        A = torch.empty((X[0].shape[0], Vr.shape[1]), dtype=X[0].dtype, device=X[0].device)
        xkv_project(X, Vr, A)
        return A

    def scores(self, p, q, landmarks, n_mid: int) -> torch.Tensor:
        B, Hkv = p.batch, p.n_kv_heads
        ld = (n_mid + 3) // 4 * 4
        s = torch.empty((B, Hkv, ld), dtype=torch.float32, device=q.device)
        xkv_sr_scores(p, q, landmarks, s)
        return s[..., :n_mid]

    def topk(self, scores: torch.Tensor, k: int) -> torch.Tensor:
        B, Hkv, n = scores.shape
        ld = (n + 3) // 4 * 4
        buf = torch.full((B, Hkv, ld), float("-inf"), dtype=torch.float32, device=scores.device)
        buf[..., :n] = scores
        sel = torch.empty((B, Hkv, k), dtype=torch.int32, device=scores.device)
        xkv_sr_topk(buf, n, k, sel)
        return sel

    def partial(self, p, shard, sel, q, A_K, Bt_K, A_V, Bt_V, sr_K, sr_V):
        out = torch.empty((p.batch, p.n_q_heads, p.head_dim), dtype=torch.float32, device=q.device)
        ml = torch.empty((p.batch, p.n_q_heads, 2), dtype=torch.float32, device=q.device)
        xkv_sr_attention_partial(p, shard, sel, q, A_K, Bt_K, A_V, Bt_V, sr_K, sr_V, out, ml)
        return out, ml

    def merge(self, o_all: torch.Tensor, ml_all: torch.Tensor) -> torch.Tensor:
        out = torch.empty(o_all.shape[1:], dtype=torch.float32, device=o_all.device)
        xkv_merge_partials(o_all, ml_all, out)
        return out


# ----------------------------------------------------------------- prefill
def compress_group_sharded(X_local: Sequence[torch.Tensor], rank: int, coll, iters: int = 8,
                           oversample: Optional[int] = None, shard_rows: int = 8192, seed: int = 0x784B56, ops=None):
    """Factorise one group whose token rows are split across the ranks.

    X_local: this rank's rows of every layer (T_r x d each).  Returns
    (A_local (T_r x rank), Bt ((G d) x rank), Ritz values).  The Gram of the
    local rows is summed over the ranks by an all-reduce; every rank then runs
    the same factorisation, and projects its own rows."""
    ops = ops or LibraryOps()
    G = len(X_local)
    T_r, d = X_local[0].shape
    p = max(64, rank // 4) if oversample is None else oversample
    C = ops.gram(X_local, shard_rows)
    coll.all_reduce_sum(C)
    T_all = coll.all_reduce_sum(torch.tensor([T_r], dtype=torch.float64, device=C.device))
    Bt, Vr, ev = ops.factor(C, G, d, int(T_all.item()), rank, iters, p, seed, X_local[0].dtype)
    return ops.project(X_local, Vr), Bt, ev


# ------------------------------------------------------------------ decode
def global_topk(scores_all: torch.Tensor, k: int, ops=None) -> torch.Tensor:
    """scores_all [R][B][Hkv][n_r] (rank r holds chunks r n_r ... (r+1) n_r - 1)
    -> the exact top-k global chunk indices [B][Hkv][k], ascending."""
    ops = ops or LibraryOps()
    R, B, Hkv, n_r = scores_all.shape
    s = scores_all.permute(1, 2, 0, 3).reshape(B, Hkv, R * n_r)
    return ops.topk(s, k)


def sr_decode_sharded(coll, p_local, shard: ShardParams, n_mid_per_rank: int, k: int, q, A_K, Bt_K, A_V, Bt_V,
                      landmarks, sr_K, sr_V, ops=None):
    """One SR decode step of one layer over a token-sharded cache.

    p_local describes this rank's slice (T local rows, its own sink / recent
    rows, topk = k); every rank holds n_mid_per_rank middle chunks, the slice of
    rank r starting at global chunk r n_mid_per_rank.  Returns (out
    [B][Hq][hd] f32, the global selection [B][Hkv][k])."""
    ops = ops or LibraryOps()
    s_local = ops.scores(p_local, q, landmarks, n_mid_per_rank)
    sel = global_topk(coll.all_gather(s_local.contiguous()), k, ops)
    o, ml = ops.partial(p_local, shard, sel, q, A_K, Bt_K, A_V, Bt_V, sr_K, sr_V)
    return ops.merge(coll.all_gather(o), coll.all_gather(ml)), sel


def local_params(w, rank: int, world: int, n_mid_per_rank: int, batch: int, dtype: torch.dtype, **strides):
    """(xkv_sr_params, xkv_sr_shard) of rank `rank`'s slice of a sequence with
    world * n_mid_per_rank middle chunks: rank 0 holds the sink rows, the last
    rank the recent rows."""
    sink = w.sink if rank == 0 else 0
    recent = w.recent if rank == world - 1 else 0
    T_local = sink + n_mid_per_rank * w.chunk + recent
    pos_off = 0 if rank == 0 else w.sink + rank * n_mid_per_rank * w.chunk
    p = sr_params(batch, w.n_q_heads, w.n_kv_heads, w.head_dim, T_local, w.rank_k, w.rank_v, w.chunk, w.topk, sink,
                  recent, w.rope_theta, dtype, **strides)
    return p, ShardParams(pos_off, rank * n_mid_per_rank)
