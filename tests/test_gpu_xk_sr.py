"""GPU parity: one decode step of the xK-SR mode (xkv_xk_sr_attention_decode:
keys compressed and rebuilt as in SR, values read from the uncompressed
[B][T][d] cache) against the oracle's xk_sr_decode on identical seeded inputs.

The selection rule and the tolerances are those of the SR parity tests: the
top-k set equals the exact one except near-ties (1e-3 relative of the k-th
score); outputs within 1e-2 max-abs (bf16 storage) or 2e-4 (f32) of the oracle
run on the GPU's own selection.  Shapes: a small bf16 case on the tensor-core
path with a ragged last tile, the f32 CUDA-core path with odd sizes, no raw
window, one layer of the Llama-3.1-8B group at 16K and one layer of the
Qwen2.5-7B shape at 128K, batch 2 (sampled units).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import check_selection, dev, host, tdtype

pytestmark = pytest.mark.gpu


def _xk_inputs(w, layer=0):
    inp = synth.compressed_cache(w, layer)
    V = synth.raw_values(w, layer)
    rows = list(range(w.sink)) + list(range(w.T - w.recent, w.T))
    x = {k: inp[k] for k in ("q", "A_K", "Bt_K", "landmarks", "sr_K")}
    x["sr_V"] = np.ascontiguousarray(V[:, rows])  # the raw window is the same cache's rows
    return x, V


def _run_xk(xkv, w, x, V):
    dt = tdtype(w)
    d = {k: dev(v, dt) for k, v in x.items()}
    dV = dev(V, dt)
    B = x["q"].shape[0]
    p = xkv.xk_sr_params(B, w.n_q_heads, w.n_kv_heads, w.head_dim, w.T, w.rank_k, w.chunk, w.topk, w.sink,
                         w.recent, w.rope_theta, dt)
    out = torch.full((B, w.n_q_heads, w.head_dim), float("nan"), device="cuda", dtype=torch.float32)
    sel = torch.full((B, w.n_kv_heads, w.topk), -1, device="cuda", dtype=torch.int32)
    xkv.xkv_xk_sr_attention_decode(p, d["q"], d["A_K"], d["Bt_K"], dV, d["landmarks"], d["sr_K"], d["sr_V"], out,
                                   sel)
    torch.cuda.synchronize()
    assert xkv.get_device_status() == 0
    return host(out), sel.cpu().numpy()


def _xk_parity(xkv, w, tol=1e-2, layer=0, units=None):
    x, V = _xk_inputs(w, layer)
    out_g, sel_g = _run_xk(xkv, w, x, V)
    _, _, scores = oracle.xk_sr_decode(w, V=V, units=units, **x)
    check_selection(sel_g, scores, w.topk, units=units)
    ref, _, _ = oracle.xk_sr_decode(w, V=V, sel_in=sel_g, units=units, **x)
    rows = np.zeros(out_g.shape[:2], dtype=bool)
    for u in (units if units is not None else range(x["q"].shape[0] * w.n_kv_heads)):
        b, h = divmod(u, w.n_kv_heads)
        rows[b, h * w.gq:(h + 1) * w.gq] = True
    assert np.isfinite(out_g[rows]).all()
    err = np.abs(out_g[rows] - ref[rows]).max()
    assert err <= tol, err
    return err


def test_xk_sr_bf16_tensor_core_ragged_tile(xkv):
    w = synth.Workload("xk_bf16_small", 2, 4, 4, 2, 128, 8, 8 + 32 + 8 * 150, 96, 0.8, 128, 192, topk=37)
    _xk_parity(xkv, w)


def test_xk_sr_f32_general_shape(xkv):
    w = synth.Workload("xk_f32_general", 2, 4, 4, 3, 64, 6, 5 + 7 + 4 * 90, 48, 0.8, 48, 80, chunk=4, topk=23,
                       sink=5, recent=7, dtype="f32")
    _xk_parity(xkv, w, tol=2e-4)


def test_xk_sr_full_size_llama_group_16k(xkv):
    _xk_parity(xkv, synth.WORKLOADS["llama_group_16k"])


def test_xk_sr_without_sink_or_recent_window(xkv):
    w = synth.Workload("xk_nowin", 2, 4, 4, 2, 128, 8, 8 * 150, 96, 0.8, 128, 128, topk=37, sink=0, recent=0)
    _xk_parity(xkv, w)


def test_xk_sr_full_size_qwen7b_128k_batch2_layer(xkv):
    # values whole: 2 x 131072 x 512 bf16 (268 MB) for the layer
    _xk_parity(xkv, synth.WORKLOADS["qwen7b_128k_b2"], layer=3, units=[0, 3, 5, 6])
