"""Token-sharded xKV (cross_layer_rank_b200.sharded) on two gloo ranks (CPU).

The orchestration under test is the product's: which rows and chunks each rank
holds, the all-reduce of the Gram, the replicated factorisation, the all-gather
and chunk-major layout of the scores, the global top-k, the positions and chunk
ranges of each rank's partial, and the exact merge of the partials.  The
per-rank arithmetic, which runs in CUDA kernels on GPUs, is done here by CPU
stand-ins in fp64 (the oracle's Gram, Jacobi and projection; plain numpy for
scores, top-k and partial attention).  Checked against the single-rank oracle:
  * prefill: the reconstruction A Bt^T of the sharded factorisation equals the
    oracle's on all rows (KV-CoRE 2.A: the Grams of the slices add up);
  * decode: the global selection is the exact top-k of the oracle's scores and
    the merged output equals the oracle's SR decode on that selection.
"""
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

LOG2E = 1.4426950408889634


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class CpuOps:
    """fp64 CPU stand-ins for the library kernels (torch CPU tensors)."""

    def __init__(self, oracle, w):
        self.oracle = oracle
        self.w = w

    def gram(self, X, shard_rows):
        return torch.from_numpy(self.oracle.gram([x.numpy() for x in X]))

    def factor(self, C, G, d, rows, rank, iters, oversample, seed, dtype):
        lam, V, _ = self.oracle.jacobi_eigh(C.numpy())
        Vr = V[:, :rank].copy()
        Vr *= np.sign(Vr[np.abs(Vr).argmax(axis=0), np.arange(rank)])  # a fixed sign per column
        return torch.from_numpy(Vr), torch.from_numpy(Vr), torch.from_numpy(lam[:rank].copy())

    def project(self, X, Vr):
        return torch.from_numpy(self.oracle.project_rows([x.numpy() for x in X], Vr.numpy()))

    def scores(self, p, q, landmarks, n_mid):
        q, lm = q.numpy(), landmarks.numpy()
        gq = p.n_q_heads // p.n_kv_heads
        qbar = q.reshape(p.batch, p.n_kv_heads, gq, p.head_dim).astype(np.float64).sum(axis=2)
        return torch.from_numpy(np.einsum("bhd,bhcd->bhc", qbar, lm[:, :, :n_mid].astype(np.float64)))

    def topk(self, scores, k):
        s = scores.numpy()
        B, H, n = s.shape
        sel = np.empty((B, H, k), np.int32)
        for b in range(B):
            for h in range(H):
                sel[b, h] = np.sort(np.lexsort((np.arange(n), -s[b, h]))[:k])
        return torch.from_numpy(sel)

    def partial(self, p, shard, sel, q, A_K, Bt_K, A_V, Bt_V, sr_K, sr_V):
        w, rope = self.w, self.oracle.rope
        q, A_K, Bt_K, A_V, Bt_V = (x.numpy().astype(np.float64) for x in (q, A_K, Bt_K, A_V, Bt_V))
        srK, srV, sel = sr_K.numpy().astype(np.float64), sr_V.numpy().astype(np.float64), sel.numpy()
        hd, C, gq = p.head_dim, p.chunk, p.n_q_heads // p.n_kv_heads
        n_mid = (p.T - p.sink - p.recent) // C
        c_lo = shard.chunk_begin
        out = np.zeros((p.batch, p.n_q_heads, hd))
        ml = np.zeros((p.batch, p.n_q_heads, 2))
        for b in range(p.batch):
            for h in range(p.n_kv_heads):
                cols = slice(h * hd, (h + 1) * hd)
                K, V = [], []
                for i in range(p.sink):  # window rows: local row i, then T - recent + i
                    K.append(rope(srK[b, i, cols], shard.position_offset + i, p.rope_theta))
                    V.append(srV[b, i, cols])
                for c in sel[b, h]:
                    if c_lo <= c < c_lo + n_mid:
                        for e in range(C):
                            t = p.sink + (c - c_lo) * C + e
                            K.append(rope(A_K[b, t] @ Bt_K[b, cols].T, shard.position_offset + t, p.rope_theta))
                            V.append(A_V[b, t] @ Bt_V[b, cols].T)
                for i in range(p.recent):
                    t = p.T - p.recent + i
                    K.append(rope(srK[b, p.sink + i, cols], shard.position_offset + t, p.rope_theta))
                    V.append(srV[b, p.sink + i, cols])
                for g in range(gq):
                    j = h * gq + g
                    if not K:
                        ml[b, j] = (-np.inf, 0.0)
                        continue
                    s = np.array(K) @ q[b, j] / math.sqrt(hd) * LOG2E
                    M = s.max()
                    e2 = np.exp2(s - M)
                    ml[b, j] = (M, e2.sum())
                    out[b, j] = e2 @ np.array(V) / e2.sum()
        return torch.from_numpy(out), torch.from_numpy(ml)

    def merge(self, o_all, ml_all):
        o, ml = o_all.numpy(), ml_all.numpy()
        M = np.where(ml[..., 1] > 0, ml[..., 0], -np.inf).max(axis=0)
        wgt = np.where(ml[..., 1] > 0, np.exp2(ml[..., 0] - M) * ml[..., 1], 0.0)
        return torch.from_numpy((wgt[..., None] * o).sum(axis=0) / wgt.sum(axis=0)[..., None])


def _workload():
    import synth
    # 2 sequences, 2 KV heads of 32, GQA 2, 10 middle chunks per rank
    return synth.Workload("sharded", 2, 2, 2, 2, 32, 4, 8 + 32 + 8 * 20, 24, 0.8, 16, 24, topk=7, dtype="f32")


def _slices(w, inp, world):
    """Each rank's slice of the whole compressed cache."""
    n_r = w.n_mid // world
    T, s, C = w.T, w.sink, w.chunk
    out = []
    for r in range(world):
        lo = 0 if r == 0 else s + r * n_r * C
        hi = T if r == world - 1 else s + (r + 1) * n_r * C
        win = list(range(s)) if r == 0 else []
        if r == world - 1:
            win += list(range(s, s + w.recent))
        sl = {"q": inp["q"], "Bt_K": inp["Bt_K"], "Bt_V": inp["Bt_V"],
              "A_K": np.ascontiguousarray(inp["A_K"][:, lo:hi]), "A_V": np.ascontiguousarray(inp["A_V"][:, lo:hi]),
              "landmarks": np.ascontiguousarray(inp["landmarks"][:, :, r * n_r:(r + 1) * n_r]),
              "sr_K": np.ascontiguousarray(inp["sr_K"][:, win]), "sr_V": np.ascontiguousarray(inp["sr_V"][:, win])}
        out.append(sl)
    return out, n_r


def _rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        import synth
        from cross_layer_rank_b200 import sharded
        w = _workload()
        ops = CpuOps(oracle, w)
        coll = sharded.Collectives()
        # prefill: this rank's half of the token rows of every layer
        layers = synth.kv_group(w, 0, 0, "K", T=w.T)
        half = w.T // 2
        X = [torch.from_numpy(l[rank * half:(rank + 1) * half]) for l in layers]
        A, Bt, ev = sharded.compress_group_sharded(X, 16, coll, ops=ops)
        out[("A", rank)] = A.numpy()
        out[("Bt", rank)] = Bt.numpy()
        # decode
        inp = synth.compressed_cache(w, 1)
        sl, n_r = _slices(w, inp, world)
        mine = sl[rank]
        p, shard = sharded.local_params(w, rank, world, n_r, w.batch, torch.float32)
        T = {k: torch.from_numpy(v) for k, v in mine.items()}
        o, sel = sharded.sr_decode_sharded(coll, p, shard, n_r, w.topk, T["q"], T["A_K"], T["Bt_K"], T["A_V"],
                                           T["Bt_V"], T["landmarks"], T["sr_K"], T["sr_V"], ops=ops)
        out[("o", rank)] = o.numpy()
        out[("sel", rank)] = sel.numpy()
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_token_sharded_prefill_and_decode_match_the_single_rank_oracle():
    sys.path.insert(0, ROOT)
    import oracle
    import synth
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        res = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, res)) for r in range(world)]
        for pr in procs:
            pr.start()
        for pr in procs:
            pr.join(300)
            assert pr.exitcode == 0
        res = dict(res)
    w = _workload()
    # prefill: every rank holds the same basis; the sharded reconstruction is the oracle's
    assert np.array_equal(res[("Bt", 0)], res[("Bt", 1)])
    layers = synth.kv_group(w, 0, 0, "K", T=w.T)
    ref = oracle.compress_group(layers, 16)
    A = np.concatenate([res[("A", 0)], res[("A", 1)]])
    rec = A @ res[("Bt", 0)].T
    rec_ref = ref["A"] @ ref["Bt"].T
    X = np.concatenate([l.astype(np.float64) for l in layers], axis=1)
    # the Grams are summed in another order: the basis moves by rounding over a
    # small eigen-gap, while the error (Eckart-Young) is fixed to second order
    assert abs(np.linalg.norm(X - rec) - ref["err_subspace"]) <= 1e-10 * ref["err_subspace"]
    assert np.abs(rec - rec_ref).max() <= 1e-6 * np.abs(rec_ref).max()
    # decode: same selection and output on both ranks, equal to the oracle's
    assert np.array_equal(res[("sel", 0)], res[("sel", 1)])
    assert np.array_equal(res[("o", 0)], res[("o", 1)])
    inp = synth.compressed_cache(w, 1)
    out_o, sel_o, scores = oracle.sr_decode(w, **inp)
    sel = res[("sel", 0)]
    for b in range(w.batch):
        for h in range(w.n_kv_heads):
            s = scores[b, h]
            kth = np.sort(s)[::-1][w.topk - 1]
            for c in set(sel[b, h].tolist()) ^ set(sel_o[b, h].tolist()):
                assert abs(s[c] - kth) <= 1e-9 * abs(kth)
    ref_o, _, _ = oracle.sr_decode(w, sel_in=sel, **inp)
    assert np.abs(res[("o", 0)] - ref_o).max() <= 1e-9
