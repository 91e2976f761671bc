"""GPU parity: one SR decode step (xkv_sr_attention_decode) against the oracle on
identical seeded inputs.

Selection: the GPU's top-k set must equal the exact one except chunks whose
score lies within 1e-3 (relative) of the k-th score.  Output: max-abs error
<= 1e-2 against the oracle run on the GPU's own (valid) selection; the f32
path is held to 2e-4.  Shapes cover the tiny f32 workload, small bf16 cases on
the tensor-core path (ragged last tile, GQA group of 7, odd atom counts,
every chunk kept) and,
at full size, one layer launch of the Llama-3.1-8B group (16K), the 32-layer
Llama-3.1-8B shape (64K, batch 4, sampled units) and the Qwen2.5-7B shape
(128K, batch 2).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import check_selection, host, run_sr, sr_inputs_on_device

pytestmark = pytest.mark.gpu


def _parity(xkv, w, layer=0, T=None, units=None, tol=1e-2, inp=None):
    T = T or w.T
    inp = inp if inp is not None else synth.compressed_cache(w, layer, T=T)
    d_inp = sr_inputs_on_device(w, inp)
    out_g, sel_g = run_sr(xkv, w, d_inp, T=T)
    out_g, sel_g = host(out_g), sel_g.cpu().numpy()
    _, sel_o, scores = oracle.sr_decode(w, T=T, units=units, **inp)
    check_selection(sel_g, scores, w.topk, units=units)
    ref, _, _ = oracle.sr_decode(w, T=T, sel_in=sel_g, units=units, **inp)
    B = inp["q"].shape[0]
    rows = np.zeros((B, w.n_q_heads), dtype=bool)
    for u in (units if units is not None else range(B * w.n_kv_heads)):
        b, h = divmod(u, w.n_kv_heads)
        rows[b, h * w.gq:(h + 1) * w.gq] = True
    err = np.abs(out_g[rows] - ref[rows]).max()
    assert np.isfinite(out_g[rows]).all()
    assert err <= tol, err
    return err, sel_g


def test_sr_tiny_f32(xkv):
    w = synth.WORKLOADS["tiny_f32"]
    err, _ = _parity(xkv, w, tol=2e-4)


def test_sr_bf16_tensor_core_ragged_tile(xkv):
    w = synth.Workload("sr_bf16_small", 2, 4, 4, 2, 128, 8, 8 + 32 + 8 * 150, 96, 0.8, 128, 192, topk=37)
    _parity(xkv, w)


def test_sr_bf16_gqa7_single_tile(xkv):
    w = synth.Workload("sr_bf16_gq7", 1, 4, 4, 2, 128, 14, 8 + 32 + 8 * 100, 96, 1.0, 64, 128, topk=16)
    _parity(xkv, w)


@pytest.mark.parametrize("n_q_heads", [2, 16])
def test_sr_bf16_gqa_group_extremes(xkv, n_q_heads):
    # 2 KV heads: one query head per KV head (plain multi-head attention) and
    # the largest group the kernels take (8)
    w = synth.Workload(f"sr_bf16_hq{n_q_heads}", 1, 4, 4, 2, 128, n_q_heads, 8 + 32 + 8 * 100, 96, 0.8, 128, 128,
                       topk=21)
    _parity(xkv, w)


def test_sr_bf16_odd_key_atom_count(xkv):
    # key rank 192 = three 64-column atoms: the last key stage is half empty;
    # value rank 320 leaves the last 128-column value block half empty
    w = synth.Workload("sr_bf16_odd_atoms", 1, 4, 4, 2, 128, 8, 8 + 32 + 8 * 120, 96, 0.8, 192, 320, topk=33)
    _parity(xkv, w)


@pytest.mark.parametrize("n_tied", [800, 2000])
def test_sr_topk_tied_boundary_bucket(xkv, n_tied):
    # landmarks l_c = a_c u with u = sign(qbar) / 16 and a_c in {2, 1, 1/2}
    # (all bf16-exact), so the scores take three exact values.  300 chunks
    # score highest, n_tied share the boundary score and the rest score lower;
    # with k = 600 the selection is the 300 high chunks plus the 300 tied
    # chunks of lowest index (ties go to the lower index).  800 tied chunks
    # are ranked by counting, 2000 by the radix passes.
    n_mid = 3000
    w = synth.Workload("sr_topk_ties", 1, 4, 4, 2, 128, 8, 8 + 32 + 8 * n_mid, 96, 0.8, 64, 64, topk=600)
    inp = synth.compressed_cache(w, 0)
    rng = np.random.default_rng(5)
    q = inp["q"].reshape(1, w.n_kv_heads, w.gq, w.head_dim)
    lm = np.empty_like(inp["landmarks"])
    expect = []
    for h in range(w.n_kv_heads):
        qbar = q[0, h].astype(np.float64).sum(axis=0)
        u = np.where(qbar >= 0, 1.0, -1.0) / 16.0
        perm = rng.permutation(n_mid)
        high, tied = np.sort(perm[:300]), np.sort(perm[300:300 + n_tied])
        a = np.full(n_mid, 0.5)
        a[high] = 2.0
        a[tied] = 1.0
        lm[0, h] = (a[:, None] * u[None, :]).astype(np.float32)
        expect.append(np.sort(np.concatenate([high, tied[:300]])))
    inp["landmarks"] = lm
    out_g, sel_g = run_sr(xkv, w, sr_inputs_on_device(w, inp))
    sel_g = sel_g.cpu().numpy()
    for h in range(w.n_kv_heads):
        assert np.array_equal(sel_g[0, h], expect[h])
    ref, _, _ = oracle.sr_decode(w, sel_in=sel_g, **inp)
    assert np.abs(host(out_g) - ref).max() <= 1e-2


def test_sr_bf16_odd_value_rank(xkv):
    # value rank 51 with a GQA group of 3: partial slots of 16 + 153 floats are
    # padded to a multiple of 4 and the merge folds the last entry on its own
    w = synth.Workload("sr_bf16_odd_rank", 1, 4, 4, 2, 128, 6, 8 + 32 + 8 * 90, 96, 0.8, 64, 51, topk=19)
    _parity(xkv, w)


def test_sr_f32_general_shape(xkv):
    # f32, hd 64, chunk 4, odd ranks: the CUDA-core path
    w = synth.Workload("sr_f32_general", 2, 4, 4, 3, 64, 6, 5 + 7 + 4 * 90, 48, 0.8, 48, 80, chunk=4, topk=23,
                       sink=5, recent=7, dtype="f32")
    _parity(xkv, w, tol=2e-4)


def test_sr_every_chunk_kept_equals_dense_attention(xkv):
    # KQ-SVD page 3.2: with k = n_mid, SR is dense decode attention over the
    # cache [raw sink | A Bt^T rows | raw recent]
    w = synth.Workload("sr_all_chunks", 1, 4, 4, 2, 128, 8, 8 + 32 + 8 * 40, 96, 0.8, 64, 64, topk=40)
    inp = synth.compressed_cache(w, 0)
    d_inp = sr_inputs_on_device(w, inp)
    out_g, sel_g = run_sr(xkv, w, d_inp)
    assert np.array_equal(sel_g.cpu().numpy()[0, 0], np.arange(40))
    T, hd = w.T, w.head_dim
    Km = oracle.full_reconstruct(inp["A_K"][0], inp["Bt_K"][0], w.n_kv_heads, hd, True, w.rope_theta)
    Vm = oracle.full_reconstruct(inp["A_V"][0], inp["Bt_V"][0], w.n_kv_heads, hd, False, w.rope_theta)
    rows = list(range(w.sink)) + list(range(T - w.recent, T))
    for i, t in enumerate(rows):
        for h in range(w.n_kv_heads):
            sl = slice(h * hd, (h + 1) * hd)
            Km[t, sl] = oracle.rope(inp["sr_K"][0, i, sl], t, w.rope_theta)
        Vm[t] = inp["sr_V"][0, i]
    ref = oracle.dense_decode(inp["q"], Km[None], Vm[None], w.n_kv_heads)
    assert np.abs(host(out_g) - ref).max() <= 1e-2


def test_sr_deterministic(xkv):
    w = synth.Workload("sr_det", 2, 4, 4, 2, 128, 8, 8 + 32 + 8 * 120, 96, 0.8, 128, 128, topk=40)
    d_inp = sr_inputs_on_device(w, synth.compressed_cache(w, 0))
    o1, s1 = run_sr(xkv, w, d_inp)
    o2, s2 = run_sr(xkv, w, d_inp)
    assert np.array_equal(host(o1), host(o2)) and np.array_equal(s1.cpu().numpy(), s2.cpu().numpy())


def test_sr_full_size_llama_group_16k(xkv):
    _parity(xkv, synth.WORKLOADS["llama_group_16k"])


def test_sr_full_size_llama8b_64k_batch4_layer(xkv):
    w = synth.WORKLOADS["llama8b_64k_b4"]
    _parity(xkv, w, layer=5, units=[0, 9, 18, 27, 31])


def test_sr_full_size_qwen7b_128k_batch2_layer(xkv):
    _parity(xkv, synth.WORKLOADS["qwen7b_128k_b2"], layer=3)


def test_stage_timing_reports_every_launch(xkv):
    # xkv_sr_profile_enable / xkv_sr_profile_read: four non-negative stage
    # durations of the last call; the attend stage did work
    w = synth.Workload("sr_profile", 2, 4, 4, 2, 128, 8, 8 + 32 + 8 * 150, 96, 0.8, 128, 192, topk=37)
    d_inp = sr_inputs_on_device(w, synth.compressed_cache(w, 0))
    xkv.xkv_sr_profile_enable(True)
    try:
        run_sr(xkv, w, d_inp)
        ms = xkv.xkv_sr_profile_read()
    finally:
        xkv.xkv_sr_profile_enable(False)
    assert len(ms) == 4 and all(np.isfinite(ms)) and min(ms) >= 0.0 and ms[2] > 0.0


def test_sr_without_sink_or_recent_window(xkv):
    # degenerate window: no raw rows at all, attention over the kept chunks only
    w = synth.Workload("sr_nowin", 2, 4, 4, 2, 128, 8, 8 * 150, 96, 0.8, 128, 128, topk=37, sink=0, recent=0)
    _parity(xkv, w)


def test_sr_single_chunk_kept(xkv):
    w = synth.Workload("sr_k1", 2, 4, 4, 2, 128, 8, 8 + 32 + 8 * 90, 96, 0.8, 128, 128, topk=1)
    _parity(xkv, w)


def test_sr_factors_shared_by_the_batch(xkv):
    # Bt_K and Bt_V given once for the whole batch (batch stride 0)
    w = synth.Workload("sr_shared_bt", 3, 4, 4, 2, 128, 8, 8 + 32 + 8 * 120, 96, 0.8, 128, 192, topk=33)
    inp = synth.compressed_cache(w, 0)
    inp["Bt_K"], inp["Bt_V"] = inp["Bt_K"][0], inp["Bt_V"][0]
    d_inp = sr_inputs_on_device(w, inp)
    B = w.batch
    p = xkv.sr_params(B, w.n_q_heads, w.n_kv_heads, w.head_dim, w.T, w.rank_k, w.rank_v, w.chunk, w.topk, w.sink,
                      w.recent, w.rope_theta, torch.bfloat16, bt_k_batch_stride=0, bt_v_batch_stride=0)
    out = torch.full((B, w.n_q_heads, w.head_dim), float("nan"), device="cuda", dtype=torch.float32)
    sel = torch.full((B, w.n_kv_heads, w.topk), -1, device="cuda", dtype=torch.int32)
    xkv.xkv_sr_attention_decode(p, d_inp["q"], d_inp["A_K"], d_inp["Bt_K"], d_inp["A_V"], d_inp["Bt_V"],
                                d_inp["landmarks"], d_inp["sr_K"], d_inp["sr_V"], out, sel)
    torch.cuda.synchronize()
    sel = sel.cpu().numpy()
    _, _, scores = oracle.sr_decode(w, **inp)
    check_selection(sel, scores, w.topk)
    ref, _, _ = oracle.sr_decode(w, sel_in=sel, **inp)
    assert np.abs(host(out) - ref).max() <= 1e-2


def test_sr_largest_supported_chunk_count(xkv):
    # n_mid = 24576 middle chunks (the top-k shared-memory limit), one unit
    w = synth.Workload("sr_max_chunks", 1, 4, 4, 1, 128, 4, 8 + 32 + 8 * 24576, 96, 0.8, 128, 128, topk=96)
    _parity(xkv, w)
