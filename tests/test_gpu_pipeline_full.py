"""The whole path at full size on the Llama-3.1-8B-shaped 16K group (G = 4
layers of 8 x 128 keys and values, T = 16384, r = 512, k = 256): the GPU
compresses the group's keys and values (xkv_compress_group), builds layer 2's
landmarks from its original keys (xkv_build_landmarks) and runs one SR decode
step of layer 2 (xkv_sr_attention_decode) on its own factors, so selection and
output are checked on the score distribution that real factors produce
(the xKV explainer, "选择性重建").

What comes from where:
  * the caches and queries come from the seeded generators, identical on both
    sides;
  * the factorisation is not unique (rotations inside the flat part of the
    spectrum around r; Eckart-Young fixes only its error, KQ-SVD 3.3), so the
    GPU's bf16 factors are first validated as a correct result, their stored
    error within 1e-3 of the oracle's (tests/golden/compress_oracle.json,
    written by the oracle), and the oracle's decode then runs on them;
  * the landmarks are unique: the oracle computes its own from the original
    keys (rounded to bf16 like the stored ones), and the GPU's must lie within
    one bf16 ulp of them;
  * the selection is an integer decision on floating-point scores: the GPU's
    set equals the oracle's exact top-k except chunks within 1e-3 of the k-th
    score, and the output equals the oracle's on that selection within 1e-2.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import check_selection, host, ulp_bf16

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "compress_oracle.json")
LAYER = 2


def _compress(xkv, X, rank):
    T, d = X[0].shape
    A = torch.empty((T, rank), dtype=torch.bfloat16, device="cuda")
    Bt = torch.empty((len(X) * d, rank), dtype=torch.bfloat16, device="cuda")
    xkv.xkv_compress_group(X, rank, A, Bt, iters=8, oversample=synth.oversample(rank), shard_rows=8192)
    return A, Bt


def _stored_error(X, A, Bt):
    Xd = torch.cat([x.double() for x in X], dim=1)
    return float(torch.linalg.vector_norm(Xd - A.double() @ Bt.double().T).item())


def test_compress_landmarks_decode_pipeline_at_16k(xkv):
    w = synth.WORKLOADS["llama_group_16k"]
    with open(GOLDEN) as f:
        gold = json.load(f)
    d, T, hd = w.d, w.T, w.head_dim
    bf = torch.bfloat16
    raw = {kind: synth.kv_group(w, 0, 0, kind) for kind in ("K", "V")}
    fac = {}
    for kind, rank, key in (("K", w.rank_k, "llama16k_k"), ("V", w.rank_v, "llama16k_v")):
        X = [torch.from_numpy(l).cuda().to(bf) for l in raw[kind]]
        A, Bt = _compress(xkv, X, rank)
        torch.cuda.synchronize()
        assert xkv.get_device_status() == 0
        sto = _stored_error(X, A, Bt)
        ref = gold[key]["err_stored"]
        assert abs(sto - ref) <= 1e-3 * ref, (kind, sto, ref)
        fac[kind] = (A, Bt[LAYER * d:(LAYER + 1) * d].contiguous())
        del X
    K2, V2 = raw["K"][LAYER], raw["V"][LAYER]
    # landmarks of layer 2 from its original keys
    lm = torch.empty((w.n_kv_heads, w.n_mid, hd), dtype=bf, device="cuda")
    xkv.xkv_build_landmarks(torch.from_numpy(K2).cuda().to(bf), w.n_kv_heads, hd, w.chunk, w.sink, w.recent,
                            w.rope_theta, lm)
    # the raw window: sink rows, then the recent rows
    win = np.r_[0:w.sink, T - w.recent:T]
    sr_K = np.ascontiguousarray(K2[win][None])
    sr_V = np.ascontiguousarray(V2[win][None])
    q = synth.queries(w, LAYER)
    p = xkv.sr_params(1, w.n_q_heads, w.n_kv_heads, hd, T, w.rank_k, w.rank_v, w.chunk, w.topk, w.sink, w.recent,
                      w.rope_theta, bf)
    out = torch.full((1, w.n_q_heads, hd), float("nan"), dtype=torch.float32, device="cuda")
    sel = torch.full((1, w.n_kv_heads, w.topk), -1, dtype=torch.int32, device="cuda")
    on = lambda x: torch.from_numpy(x).cuda().to(bf).contiguous()
    xkv.xkv_sr_attention_decode(p, on(q), fac["K"][0][None], fac["K"][1][None], fac["V"][0][None],
                                fac["V"][1][None], lm[None], on(sr_K), on(sr_V), out, sel)
    torch.cuda.synchronize()
    assert xkv.get_device_status() == 0
    # landmarks: unique, so checked against the oracle's own
    lm_o = oracle.landmarks(K2, w.n_kv_heads, hd, w.chunk, w.sink, w.recent, w.rope_theta)
    floor = 1e-6 * np.abs(K2).max()
    excess = np.abs(host(lm).astype(np.float64) - lm_o) / (ulp_bf16(lm_o) + floor)
    assert excess.max() <= 1.0, excess.max()
    # decode: the oracle on the validated factors and its own bf16 landmarks
    fo = {k: (host(A)[None], host(Bt)[None]) for k, (A, Bt) in fac.items()}
    inp = dict(q=q, A_K=fo["K"][0], Bt_K=fo["K"][1], A_V=fo["V"][0], Bt_V=fo["V"][1],
               landmarks=oracle.round_bf16(lm_o)[None], sr_K=sr_K, sr_V=sr_V)
    _, _, scores = oracle.sr_decode(w, **inp)
    sel_g = sel.cpu().numpy()
    check_selection(sel_g, scores, w.topk)
    ref, _, _ = oracle.sr_decode(w, sel_in=sel_g, **inp)
    o = host(out)
    assert np.isfinite(o).all()
    assert np.abs(o - ref).max() <= 1e-2, np.abs(o - ref).max()
    # the selection is not degenerate: real factors concentrate the scores, so
    # the kept chunks are not a prefix, and they span the sequence
    assert not np.array_equal(sel_g[0, 0], np.arange(w.topk))
