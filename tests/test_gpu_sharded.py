"""Token-sharded xKV on one GPU: two shards of the sequence processed one after
the other by the library's kernels (xkv_sr_scores, xkv_sr_topk,
xkv_sr_attention_partial, xkv_merge_partials; xkv_gram_accumulate,
xkv_factor_gram, xkv_project), with the collectives done in the process
(stacking the shards' tensors stands in for the all-gather, adding the Grams
for the all-reduce).  No kernel waits on another shard's.

Checked: the global selection equals the single-device decode's bit for bit
(the same score arithmetic per chunk); the merged output equals the
single-device output within 1e-4 and the oracle's within the decode tolerance;
the sharded factorisation's errors equal the oracle's within 1e-3 (KQ-SVD 3.3).
The multi-process orchestration itself is covered on CPU by
tests/test_sharded_gloo.py.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from cross_layer_rank_b200 import sharded
from gpu_helpers import dev, host, run_sr, sr_inputs_on_device, tdtype

pytestmark = pytest.mark.gpu


def _shard_inputs(w, inp, world):
    n_r = w.n_mid // world
    T, s, C = w.T, w.sink, w.chunk
    out = []
    for r in range(world):
        lo = 0 if r == 0 else s + r * n_r * C
        hi = T if r == world - 1 else s + (r + 1) * n_r * C
        win = list(range(s)) if r == 0 else []
        if r == world - 1:
            win += list(range(s, s + w.recent))
        out.append({"q": inp["q"], "Bt_K": inp["Bt_K"], "Bt_V": inp["Bt_V"],
                    "A_K": np.ascontiguousarray(inp["A_K"][:, lo:hi]),
                    "A_V": np.ascontiguousarray(inp["A_V"][:, lo:hi]),
                    "landmarks": np.ascontiguousarray(inp["landmarks"][:, :, r * n_r:(r + 1) * n_r]),
                    "sr_K": np.ascontiguousarray(inp["sr_K"][:, win]),
                    "sr_V": np.ascontiguousarray(inp["sr_V"][:, win])})
    return out, n_r


@pytest.mark.parametrize("case", ["bf16", "f32", "llama_group_16k"])
def test_sharded_decode_matches_single_device_and_oracle(xkv, case):
    world = 2
    if case == "bf16":
        w = synth.Workload("shd_bf16", 2, 4, 4, 2, 128, 8, 8 + 32 + 8 * 160, 96, 0.8, 128, 192, topk=37)
        tol = 1e-2
    elif case == "f32":
        w = synth.Workload("shd_f32", 2, 4, 4, 3, 64, 6, 5 + 7 + 4 * 90, 48, 0.8, 48, 80, chunk=4, topk=23, sink=5,
                           recent=7, dtype="f32")
        tol = 2e-4
    else:
        w = synth.WORKLOADS["llama_group_16k"].replace(T=8 + 32 + 8 * 2046)
        tol = 1e-2
    dt = tdtype(w)
    inp = synth.compressed_cache(w, 1)
    d_inp = sr_inputs_on_device(w, inp)
    ref_out, ref_sel = run_sr(xkv, w, d_inp)
    ops = sharded.LibraryOps()
    slices, n_r = _shard_inputs(w, inp, world)
    scores = []
    for r, sl in enumerate(slices):
        p, _ = sharded.local_params(w, r, world, n_r, w.batch, dt)
        scores.append(ops.scores(p, dev(sl["q"], dt), dev(sl["landmarks"], dt), n_r))
    sel = sharded.global_topk(torch.stack(scores), w.topk, ops)
    parts, mls = [], []
    for r, sl in enumerate(slices):
        p, shard = sharded.local_params(w, r, world, n_r, w.batch, dt)
        D = {k: dev(v, dt) for k, v in sl.items()}
        o, ml = ops.partial(p, shard, sel, D["q"], D["A_K"], D["Bt_K"], D["A_V"], D["Bt_V"], D["sr_K"], D["sr_V"])
        parts.append(o)
        mls.append(ml)
    out = ops.merge(torch.stack(parts), torch.stack(mls))
    torch.cuda.synchronize()
    assert xkv.get_device_status() == 0
    assert torch.equal(sel, ref_sel)
    out, ref_out = host(out), host(ref_out)
    assert np.isfinite(out).all()
    assert np.abs(out - ref_out).max() <= 1e-4
    ref, _, _ = oracle.sr_decode(w, sel_in=sel.cpu().numpy(), **inp)
    assert np.abs(out - ref).max() <= tol


def test_shard_holding_no_kept_chunk_contributes_nothing(xkv):
    # every kept chunk lies in shard 0's half: shard 1 (no window, no kept
    # chunk) reports (M, L) = (-inf, 0) and the merge ignores it
    w = synth.Workload("shd_empty", 1, 4, 4, 2, 128, 8, 8 + 8 * 64, 96, 0.8, 128, 128, topk=16, recent=0)
    dt = tdtype(w)
    inp = synth.compressed_cache(w, 0)
    slices, n_r = _shard_inputs(w, inp, 2)
    ops = sharded.LibraryOps()
    p1, sh1 = sharded.local_params(w, 1, 2, n_r, w.batch, dt)
    sel = torch.arange(w.topk, dtype=torch.int32, device="cuda").repeat(w.batch, w.n_kv_heads, 1).contiguous()
    D = {k: dev(v, dt) for k, v in slices[1].items()}
    o, ml = ops.partial(p1, sh1, sel, D["q"], D["A_K"], D["Bt_K"], D["A_V"], D["Bt_V"], D["sr_K"], D["sr_V"])
    torch.cuda.synchronize()
    assert xkv.get_device_status() == 0
    ml = host(ml)
    assert np.all(np.isneginf(ml[..., 0])) and np.all(ml[..., 1] == 0.0)
    assert np.all(host(o) == 0.0)


def test_sharded_prefill_matches_oracle_errors(xkv):
    # two halves of the token rows: Gram per half, summed (the all-reduce), one
    # factorisation, each half projected
    w = synth.WORKLOADS["tiny_f32"].replace(name="shd_cmp", group=4, n_layers=4, dtype="bf16", n_kv_heads=2,
                                             head_dim=64, latent=256)
    T, rank = 1536, 128
    layers = synth.kv_group(w, 0, 0, "K", T=T)
    ref = oracle.compress_group(layers, rank)
    ops = sharded.LibraryOps()
    X = [dev(l, torch.bfloat16) for l in layers]
    halves = [[x[:T // 2] for x in X], [x[T // 2:] for x in X]]
    C = ops.gram(halves[0], 512) + ops.gram(halves[1], 512)
    Bt, Vr, ev = ops.factor(C, 4, w.d, T, rank, 8, synth.oversample(rank), 0x784B56, torch.bfloat16)
    A = torch.cat([ops.project(h, Vr) for h in halves])
    torch.cuda.synchronize()
    assert xkv.get_device_status() == 0
    Xd = np.concatenate([l.astype(np.float64) for l in layers], axis=1)
    V = host(Vr).astype(np.float64)
    sub = np.linalg.norm(Xd - (Xd @ V) @ V.T)
    sto = np.linalg.norm(Xd - host(A).astype(np.float64) @ host(Bt).astype(np.float64).T)
    assert abs(sub - ref["err_subspace"]) <= 1e-3 * ref["err_subspace"]
    assert abs(sto - ref["err_stored"]) <= 1e-3 * ref["err_stored"]
