"""Integer parity of the chunk selection, taken in the kernel's precision.

The score launch writes each unit's fp32 chunk scores at the start of the
decode workspace (one row of n_mid entries, padded to a multiple of 4 floats,
per unit).  On those very values the selection must be the exact top-k with
ties to the lower chunk index, ascending, bit for bit; and the fp32 scores
themselves must agree with the oracle's fp64 scores within an fp32 rounding
bound of the dot products (sum over the GQA group of q_g . landmark_c).
Cases: one layer of the Llama-3.1-8B group at 16K, and crafted scores with 800
and 2000 chunks tied at the boundary (counting and radix paths).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import sr_inputs_on_device, tdtype

pytestmark = pytest.mark.gpu


def _tied_inputs(w, n_tied):
    # three exact score levels (as in the tied-boundary decode test)
    inp = synth.compressed_cache(w, 0)
    rng = np.random.default_rng(7)
    q = inp["q"].reshape(1, w.n_kv_heads, w.gq, w.head_dim)
    lm = np.empty_like(inp["landmarks"])
    for h in range(w.n_kv_heads):
        qbar = q[0, h].astype(np.float64).sum(axis=0)
        u = np.where(qbar >= 0, 1.0, -1.0) / 16.0
        perm = rng.permutation(w.n_mid)
        a = np.full(w.n_mid, 0.5)
        a[perm[:300]] = 2.0
        a[perm[300:300 + n_tied]] = 1.0
        lm[0, h] = (a[:, None] * u[None, :]).astype(np.float32)
    inp["landmarks"] = lm
    return inp


def _check(xkv, w, inp):
    d = sr_inputs_on_device(w, inp)
    B, units, n, k = inp["q"].shape[0], inp["q"].shape[0] * w.n_kv_heads, w.n_mid, w.topk
    p = xkv.sr_params(B, w.n_q_heads, w.n_kv_heads, w.head_dim, w.T, w.rank_k, w.rank_v, w.chunk, k, w.sink,
                      w.recent, w.rope_theta, tdtype(w))
    ws = xkv.workspace(xkv.xkv_sr_workspace_size(p))
    out = torch.empty((B, w.n_q_heads, w.head_dim), dtype=torch.float32, device="cuda")
    sel = torch.full((B, w.n_kv_heads, k), -1, dtype=torch.int32, device="cuda")
    xkv.xkv_sr_attention_decode(p, d["q"], d["A_K"], d["Bt_K"], d["A_V"], d["Bt_V"], d["landmarks"], d["sr_K"],
                                d["sr_V"], out, sel, ws=ws)
    torch.cuda.synchronize()
    assert xkv.get_device_status() == xkv.XKV_OK
    ld = (n + 3) & ~3
    s32 = ws[:units * ld * 4].view(torch.float32).view(units, ld)[:, :n].cpu().numpy()
    sel = sel.cpu().numpy().reshape(units, k)
    _, _, s64 = oracle.sr_decode(w, **inp)
    s64 = s64.reshape(units, n)
    q = inp["q"].astype(np.float64).reshape(units, w.gq, w.head_dim)
    lm = inp["landmarks"].astype(np.float64).reshape(units, n, w.head_dim)
    for u in range(units):
        exact = np.sort(np.lexsort((np.arange(n), -s32[u]))[:k])
        assert np.array_equal(sel[u], exact), u
        bound = 2e-5 * (np.abs(lm[u]) @ np.abs(q[u]).sum(axis=0)) + 1e-6
        assert np.all(np.abs(s32[u] - s64[u]) <= bound), u


def test_topk_bit_exact_on_kernel_scores_llama_group_16k(xkv):
    w = synth.WORKLOADS["llama_group_16k"]
    _check(xkv, w, synth.compressed_cache(w, 0))


@pytest.mark.parametrize("n_tied", [800, 2000])
def test_topk_bit_exact_on_tied_scores(xkv, n_tied):
    w = synth.Workload("topk_ties_exact", 1, 4, 4, 2, 128, 8, 8 + 32 + 8 * 3000, 96, 0.8, 64, 64, topk=600)
    _check(xkv, w, _tied_inputs(w, n_tied))
