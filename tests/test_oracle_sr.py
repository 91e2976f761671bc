"""Oracle pins: Selective-Reconstruction decode (xKV explainer, "选择性重建").

* the top-k chunk selection equals a brute-force library sort (ties -> lower
  chunk index), and is returned ascending;
* with k = every middle chunk, SR equals dense decode attention (KQ-SVD page,
  3.2) over the cache [raw sink | A B rows | raw recent];
* with full rank and every chunk kept, SR on the factors equals dense attention
  over the ORIGINAL cache (exact reconstruction, KQ-SVD page 3.3);
* a chunk planted to match the query is selected and dominates the output.

xK-SR mode (same explainer: keys compressed, values kept whole):
* with values equal to the rebuilt A_V Bt_V^T rows it reduces to SR;
* with every chunk kept it is dense attention over rebuilt keys and raw values;
* values outside the selected chunks and the window are never read.
"""
import numpy as np
import pytest

import oracle
import synth

W = synth.WORKLOADS["tiny_f32"].replace(name="oracle_sr_pin", T=8 + 32 + 20 * 8, topk=5)


def _inputs(w=W, seed_layer=0):
    return synth.compressed_cache(w, seed_layer)


def _dense_cache(w, inp, K_mid, V_mid):
    """[B][T][d] post-RoPE keys and values with raw sink/recent rows."""
    B, T, d, hd = w.batch, w.T, w.d, w.head_dim
    K = np.empty((B, T, d)); V = np.empty((B, T, d))
    for b in range(B):
        K[b], V[b] = K_mid[b], V_mid[b]
        rows = list(range(w.sink)) + list(range(T - w.recent, T))
        for i, t in enumerate(rows):
            for h in range(w.n_kv_heads):
                sl = slice(h * hd, (h + 1) * hd)
                K[b, t, sl] = oracle.rope(inp["sr_K"][b, i, sl], t, w.rope_theta)
            V[b, t] = inp["sr_V"][b, i]
    return K, V


def test_selection_is_exact_topk_with_low_index_ties():
    inp = _inputs()
    # quantise landmarks so that exact score ties occur
    inp["landmarks"] = np.round(inp["landmarks"] * 2) / 2
    inp["q"] = np.round(inp["q"])
    _, sel, scores = oracle.sr_decode(W, **inp)
    for b in range(W.batch):
        for h in range(W.n_kv_heads):
            s = scores[b, h]
            order = np.lexsort((np.arange(s.size), -s))  # by -score, then index
            assert list(sel[b, h]) == sorted(order[: W.topk].tolist())
    # scores are sum_g q_g . l_c over the GQA group of KV head h
    q = inp["q"].astype(np.float64); lm = inp["landmarks"].astype(np.float64)
    gq = W.gq
    ref = np.einsum("bhgj,bhcj->bhc", q.reshape(W.batch, W.n_kv_heads, gq, -1), lm)
    assert np.abs(scores - ref).max() < 1e-12


def test_all_chunks_equals_dense_over_rebuilt_cache():
    w = W.replace(topk=W.n_mid)
    inp = _inputs(w)
    out, sel, _ = oracle.sr_decode(w, **inp)
    assert np.array_equal(sel[0, 0], np.arange(w.n_mid))
    Km = np.stack([oracle.full_reconstruct(inp["A_K"][b], inp["Bt_K"][b], w.n_kv_heads, w.head_dim, True,
                                           w.rope_theta) for b in range(w.batch)])
    Vm = np.stack([oracle.full_reconstruct(inp["A_V"][b], inp["Bt_V"][b], w.n_kv_heads, w.head_dim, False,
                                           w.rope_theta) for b in range(w.batch)])
    K, V = _dense_cache(w, inp, Km, Vm)
    ref = oracle.dense_decode(inp["q"], K, V, w.n_kv_heads)
    # the dense path takes the rebuilt cache through float32: agreement to that rounding
    assert np.abs(out - ref).max() < 1e-6


def test_full_rank_all_chunks_equals_dense_over_original():
    w = synth.WORKLOADS["tiny_f32"].replace(name="oracle_sr_fullrank", T=8 + 32 + 8 * 8, topk=8,
                                            rank_k=4 * 128, rank_v=4 * 128)
    layer = 2
    Ks = synth.kv_group(w, 0, 0, "K", T=w.T)
    Vs = synth.kv_group(w, 0, 0, "V", T=w.T)
    ck = oracle.compress_group(Ks, w.rank_k)
    cv = oracle.compress_group(Vs, w.rank_v)
    d = w.d
    sw_rows = list(range(w.sink)) + list(range(w.T - w.recent, w.T))
    inp = dict(q=synth.queries(w, layer),
               A_K=ck["A"][None], Bt_K=ck["Bt"][layer * d:(layer + 1) * d],
               A_V=cv["A"][None], Bt_V=cv["Bt"][layer * d:(layer + 1) * d],
               landmarks=oracle.landmarks(Ks[layer], w.n_kv_heads, w.head_dim, w.chunk, w.sink, w.recent,
                                   w.rope_theta)[None],
               sr_K=Ks[layer][sw_rows][None], sr_V=Vs[layer][sw_rows][None])
    out, _, _ = oracle.sr_decode(w, **inp)
    Kr = np.empty((w.T, d))
    for t in range(w.T):
        for h in range(w.n_kv_heads):
            sl = slice(h * w.head_dim, (h + 1) * w.head_dim)
            Kr[t, sl] = oracle.rope(Ks[layer][t, sl], t, w.rope_theta)
    ref = oracle.dense_decode(inp["q"], Kr[None], Vs[layer][None], w.n_kv_heads)
    # A, Bt are passed through float32: agreement to float32 rounding
    assert np.abs(out - ref).max() < 1e-4


def test_planted_chunk_is_selected_and_dominates():
    w = W.replace(batch=1)
    inp = _inputs(w)
    b, h, c_star = 0, 1, 13
    g_q = inp["q"][b, h * w.gq:(h + 1) * w.gq].astype(np.float64)
    # landmark of chunk c_star points along the group's mean query
    inp["landmarks"] = inp["landmarks"].copy()
    inp["landmarks"][b, h, c_star] = (50 * g_q.mean(0) / np.linalg.norm(g_q.mean(0))).astype(np.float32)
    _, sel, _ = oracle.sr_decode(w, **inp)
    assert c_star in sel[b, h]


def test_sel_in_overrides_selection():
    inp = _inputs()
    _, sel, _ = oracle.sr_decode(W, **inp)
    alt = np.sort(np.stack([np.arange(W.topk)] * (W.batch * W.n_kv_heads)).reshape(sel.shape), axis=-1).astype(np.int32)
    out2, sel2, _ = oracle.sr_decode(W, **inp, sel_in=alt)
    assert np.array_equal(sel2, alt)


def test_unit_subset_matches_full_run():
    inp = _inputs()
    out, sel, _ = oracle.sr_decode(W, **inp)
    out1, sel1, _ = oracle.sr_decode(W, **inp, units=[1])
    b, h = divmod(1, W.n_kv_heads)
    rows = slice(h * W.gq, (h + 1) * W.gq)
    assert np.array_equal(out1[b, rows], out[b, rows]) and np.array_equal(sel1[b, h], sel[b, h])
    assert np.isnan(out1[0, 0]).all()


def test_rejects_ragged_middle():
    w = W.replace(T=W.T + 3)
    with pytest.raises(ValueError):
        oracle.sr_decode(w, **_inputs(w))


# ---------------------------------------------------------------- xK-SR mode
# Keys compressed and selected as above; values read uncompressed ([B][T][d]).

def _xk_inputs(w=W, layer=0):
    inp = _inputs(w, layer)
    V = synth.raw_values(w, layer)
    rows = list(range(w.sink)) + list(range(w.T - w.recent, w.T))
    # the raw window is the same cache's rows
    inp["sr_V"] = np.ascontiguousarray(V[:, rows])
    x = {k: inp[k] for k in ("q", "A_K", "Bt_K", "landmarks", "sr_K", "sr_V")}
    x["V"] = V
    return x, inp


def test_xk_values_from_factors_reduce_to_sr():
    # V = A_V Bt_V^T (one factorisation per sequence, so every head's columns
    # differ): xK-SR must give SR's output on the same selection
    inp = _inputs()
    V = np.stack([oracle.full_reconstruct(inp["A_V"][b], inp["Bt_V"][b], W.n_kv_heads, W.head_dim, False,
                                          W.rope_theta) for b in range(W.batch)]).astype(np.float32)
    x = {k: inp[k] for k in ("q", "A_K", "Bt_K", "landmarks", "sr_K", "sr_V")}
    out_x, sel_x, sc_x = oracle.xk_sr_decode(W, V=V, **x)
    out_s, sel_s, sc_s = oracle.sr_decode(W, **inp)
    assert np.array_equal(sel_x, sel_s) and np.array_equal(sc_x, sc_s)
    # V went through float32 once: agreement to that rounding
    assert np.abs(out_x - out_s).max() < 1e-6


def test_xk_all_chunks_equals_dense_over_rebuilt_keys_and_raw_values():
    w = W.replace(topk=W.n_mid)
    x, inp = _xk_inputs(w)
    out, sel, _ = oracle.xk_sr_decode(w, **x)
    assert np.array_equal(sel[0, 0], np.arange(w.n_mid))
    Km = np.stack([oracle.full_reconstruct(inp["A_K"][b], inp["Bt_K"][b], w.n_kv_heads, w.head_dim, True,
                                           w.rope_theta) for b in range(w.batch)])
    K, V = _dense_cache(w, inp, Km, x["V"].astype(np.float64))
    ref = oracle.dense_decode(inp["q"], K, V, w.n_kv_heads)
    assert np.abs(out - ref).max() < 1e-6


def test_xk_reads_only_selected_rows_and_window():
    x, _ = _xk_inputs()
    out, sel, _ = oracle.xk_sr_decode(W, **x)
    b, h = 0, 1
    hd, C = W.head_dim, W.chunk
    chosen = set(sel[b, h].tolist())
    skipped = next(c for c in range(W.n_mid) if c not in chosen)
    kept = sel[b, h, 0]
    # a middle chunk that was not selected: its values are never read
    V2 = x["V"].copy()
    t0 = W.sink + skipped * C
    V2[b, t0:t0 + C, h * hd:(h + 1) * hd] += 100.0
    out2, _, _ = oracle.xk_sr_decode(W, **{**x, "V": V2})
    assert np.array_equal(out2, out)
    # one row of a selected chunk: the unit's outputs move, the others do not
    V3 = x["V"].copy()
    V3[b, W.sink + kept * C, h * hd:(h + 1) * hd] += 100.0
    out3, _, _ = oracle.xk_sr_decode(W, **{**x, "V": V3})
    rows = slice(h * W.gq, (h + 1) * W.gq)
    assert np.abs(out3[b, rows] - out[b, rows]).max() > 1e-6
    mask = np.ones(out.shape[:2], dtype=bool)
    mask[b, rows] = False
    assert np.array_equal(out3[mask], out[mask])
