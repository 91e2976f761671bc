"""GPU parity of multi-step decode (xkv_sr_append + xkv_sr_attention_decode)
against the oracle's state machine (oracle.SRState) on identical inputs.

Each step appends one token per layer of the group to the raw window (the
xKV explainer's editor's note: only the prefill is compressed, generated
tokens stay raw), rolls a full chunk into the compressed cache when the window
holds recent + chunk rows (A rows = x V on the stored bases, one landmark per
layer and head), then decodes one layer at the new length.  Checked every step:
the roll decision, the selection (exact top-k up to near-ties, on the oracle's
scores) and the output (max-abs 1e-2, on the GPU's own selection).  At the end:
the windows bit for bit, the rolled A rows and landmarks within one bf16 ulp
(landmarks: plus the cancellation floor of the prefill landmarks).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import check_selection, host, ulp_bf16

pytestmark = pytest.mark.gpu


def _bf(x):
    return synth.to_storage(np.asarray(x, np.float32), "bf16")


@pytest.mark.parametrize("B,G,Hkv,Hq,rk,rv,k,steps", [(2, 2, 2, 8, 128, 192, 16, 21), (1, 4, 1, 7, 64, 64, 9, 12)])
def test_multistep_decode_matches_oracle(xkv, B, G, Hkv, Hq, rk, rv, k, steps):
    hd, C, s, wr = 128, 8, 8, 32
    d = Hkv * hd
    n = G * d
    n_mid0 = 60
    T0 = s + wr + C * n_mid0
    cap_chunks = n_mid0 + steps // C + 2
    T_cap = s + cap_chunks * C + wr + C
    w = synth.Workload("multistep", B, G, G, Hkv, hd, Hq, T0, 96, 0.8, rk, rv, topk=k)
    rng = np.random.default_rng(B * 100 + G)
    sc = lambda r: (np.arange(1, r + 1) ** -0.8 * 3.0).astype(np.float32)
    A_K = np.zeros((B, T_cap, rk), np.float32)
    A_V = np.zeros((B, T_cap, rv), np.float32)
    A_K[:, :T0] = _bf(rng.standard_normal((B, T0, rk)) * sc(rk))
    A_V[:, :T0] = _bf(rng.standard_normal((B, T0, rv)) * sc(rv))
    Bt_K = _bf(rng.standard_normal((B, n, rk)) / math.sqrt(rk))
    Bt_V = _bf(rng.standard_normal((B, n, rv)) / math.sqrt(rv))
    lms, wk, wv = [], [], []
    for _ in range(G):
        lm = np.zeros((B, Hkv, cap_chunks, hd), np.float32)
        lm[:, :, :n_mid0] = _bf(rng.standard_normal((B, Hkv, n_mid0, hd)))
        lms.append(lm)
        for lst in (wk, wv):
            win = np.zeros((B, s + wr + C, d), np.float32)
            win[:, :s + wr] = _bf(rng.standard_normal((B, s + wr, d)))
            lst.append(win)
    st = oracle.SRState(w, A_K.copy(), A_V.copy(), Bt_K, Bt_V, [l.copy() for l in lms], [x.copy() for x in wk],
                        [x.copy() for x in wv], T0, n_mid0, wr)
    bf = torch.bfloat16
    D = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda().to(bf)
    gA_K, gA_V, gBt_K, gBt_V = D(A_K), D(A_V), D(Bt_K), D(Bt_V)
    glms = [D(x) for x in lms]
    gwk, gwv = [D(x) for x in wk], [D(x) for x in wv]
    wbs = (s + wr + C) * d
    T = T0
    rolls = 0
    for step in range(steps):
        k_new = [_bf(rng.standard_normal((B, d))) for _ in range(G)]
        v_new = [_bf(rng.standard_normal((B, d))) for _ in range(G)]
        ap = xkv.append_params(B, G, Hkv, hd, C, s, wr, w.rope_theta, bf, T, rk, rv, T_cap * rk, T_cap * rv, n * rk,
                               n * rv, wbs, cap_chunks)
        rolled = xkv.xkv_sr_append(ap, [D(x) for x in k_new], [D(x) for x in v_new], gwk, gwv, gBt_K, gBt_V, gA_K,
                                   gA_V, glms)
        assert rolled == st.append(k_new, v_new)
        rolls += rolled
        T += 1
        n_mid, w_cur = xkv.decode_layout(T, s, wr, C)
        assert (n_mid, w_cur, T) == (st.n_mid, st.w_cur, st.T)
        # decode one layer of the group at the new length
        l = step % G
        q = _bf(rng.standard_normal((B, Hq, hd)))
        p = xkv.sr_params(B, Hq, Hkv, hd, T, rk, rv, C, k, s, w_cur, w.rope_theta, bf, a_k_batch_stride=T_cap * rk,
                          a_v_batch_stride=T_cap * rv, bt_k_batch_stride=n * rk, bt_v_batch_stride=n * rv,
                          window_batch_stride=wbs, landmark_capacity=cap_chunks)
        out = torch.full((B, Hq, hd), float("nan"), device="cuda")
        sel = torch.full((B, Hkv, k), -1, device="cuda", dtype=torch.int32)
        xkv.xkv_sr_attention_decode(p, D(q), gA_K, gBt_K[:, l * d:(l + 1) * d], gA_V, gBt_V[:, l * d:(l + 1) * d],
                                    glms[l], gwk[l], gwv[l], out, sel)
        torch.cuda.synchronize()
        assert xkv.get_device_status() == 0
        wd = w.replace(T=T, recent=w_cur)
        args = (q, st.A_K[:, :T], st.Bt_K[:, l * d:(l + 1) * d], st.A_V[:, :T], st.Bt_V[:, l * d:(l + 1) * d],
                np.ascontiguousarray(st.lms[l][:, :, :n_mid]), np.ascontiguousarray(st.win_K[l][:, :s + w_cur]),
                np.ascontiguousarray(st.win_V[l][:, :s + w_cur]))
        _, _, scores = oracle.sr_decode(wd, *args, T=T)
        sel_h = sel.cpu().numpy()
        check_selection(sel_h, scores, k)
        ref, _, _ = oracle.sr_decode(wd, *args, T=T, sel_in=sel_h)
        assert np.abs(host(out) - ref).max() <= 1e-2, step
    assert rolls == (steps + (T0 - s - wr) % C) // C
    # final state: windows exact; rolled A rows and landmarks within a bf16 ulp
    for l in range(G):
        assert np.array_equal(host(gwk[l])[:, :s + st.w_cur], st.win_K[l][:, :s + st.w_cur])
        assert np.array_equal(host(gwv[l])[:, :s + st.w_cur], st.win_V[l][:, :s + st.w_cur])
    t1 = s + st.n_mid * C
    for g, o in ((gA_K, st.A_K), (gA_V, st.A_V)):
        a, b = host(g)[:, T0 - wr:t1], o[:, T0 - wr:t1]
        assert np.all(np.abs(a - b) <= ulp_bf16(b) * 1.001 + 1e-30)
        assert np.array_equal(host(g)[:, :T0 - wr], o[:, :T0 - wr])
    for l in range(G):
        a, b = host(glms[l])[:, :, n_mid0:st.n_mid], st.lms[l][:, :, n_mid0:st.n_mid]
        floor = 1e-6 * max(np.abs(wk[l]).max(), 1.0)
        assert np.all(np.abs(a - b) <= ulp_bf16(b) * 1.001 + floor)
