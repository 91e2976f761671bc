"""GPU parity of the xK-SR step with the uncompressed values in pinned host
memory (xkv_xk_sr_attention_decode_host_values), the placement of the xKV
explainer's "选择性重建" section: only the kept chunks' value rows cross the
host link.

Against the HBM-resident xK-SR entry point on identical inputs: the same
selection and the same outputs (the attend kernels read the same rows, from a
staging buffer instead of the cache); against the oracle's xk_sr_decode on the
GPU's selection within the decode tolerance (1e-2 bf16, 2e-4 f32).  A device
pointer in place of host memory is refused before anything runs.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import check_selection, dev, host, tdtype

pytestmark = pytest.mark.gpu


def _inputs(w, layer=0):
    inp = synth.compressed_cache(w, layer)
    V = synth.raw_values(w, layer)
    rows = list(range(w.sink)) + list(range(w.T - w.recent, w.T))
    x = {k: inp[k] for k in ("q", "A_K", "Bt_K", "landmarks", "sr_K")}
    x["sr_V"] = np.ascontiguousarray(V[:, rows])
    return x, V


def _both(xkv, w, layer=0):
    dt = tdtype(w)
    x, V = _inputs(w, layer)
    d = {k: dev(v, dt) for k, v in x.items()}
    B = x["q"].shape[0]
    p = xkv.xk_sr_params(B, w.n_q_heads, w.n_kv_heads, w.head_dim, w.T, w.rank_k, w.chunk, w.topk, w.sink,
                         w.recent, w.rope_theta, dt)
    res = []
    for where in ("hbm", "host"):
        out = torch.full((B, w.n_q_heads, w.head_dim), float("nan"), device="cuda", dtype=torch.float32)
        sel = torch.full((B, w.n_kv_heads, w.topk), -1, device="cuda", dtype=torch.int32)
        if where == "hbm":
            xkv.xkv_xk_sr_attention_decode(p, d["q"], d["A_K"], d["Bt_K"], dev(V, dt), d["landmarks"], d["sr_K"],
                                           d["sr_V"], out, sel)
        else:
            Vh = torch.from_numpy(np.ascontiguousarray(V, dtype=np.float32)).to(dt).pin_memory()
            xkv.xkv_xk_sr_attention_decode_host_values(p, d["q"], d["A_K"], d["Bt_K"], Vh, d["landmarks"],
                                                       d["sr_K"], d["sr_V"], out, sel)
        torch.cuda.synchronize()
        assert xkv.get_device_status() == 0
        res.append((host(out), sel.cpu().numpy()))
    return x, V, res


@pytest.mark.parametrize("case", ["bf16_small", "f32_general", "llama_group_16k"])
def test_host_values_match_hbm_values_and_oracle(xkv, case):
    if case == "bf16_small":
        w = synth.Workload("xkh_bf16_small", 2, 4, 4, 2, 128, 8, 8 + 32 + 8 * 150, 96, 0.8, 128, 192, topk=37)
        tol = 1e-2
    elif case == "f32_general":
        w = synth.Workload("xkh_f32_general", 2, 4, 4, 3, 64, 6, 5 + 7 + 4 * 90, 48, 0.8, 48, 80, chunk=4, topk=23,
                           sink=5, recent=7, dtype="f32")
        tol = 2e-4
    else:
        w = synth.WORKLOADS["llama_group_16k"]
        tol = 1e-2
    x, V, ((o_hbm, s_hbm), (o_host, s_host)) = _both(xkv, w)
    assert np.array_equal(s_host, s_hbm)
    assert np.isfinite(o_host).all()
    assert np.abs(o_host - o_hbm).max() <= 1e-6
    _, _, scores = oracle.xk_sr_decode(w, V=V, **x)
    check_selection(s_host, scores, w.topk)
    ref, _, _ = oracle.xk_sr_decode(w, V=V, sel_in=s_host, **x)
    assert np.abs(o_host - ref).max() <= tol


def test_host_values_refuse_device_memory(xkv):
    w = synth.Workload("xkh_ref", 1, 4, 4, 2, 128, 8, 8 + 32 + 8 * 40, 96, 0.8, 128, 128, topk=16)
    x, V = _inputs(w)
    d = {k: dev(v, torch.bfloat16) for k, v in x.items()}
    p = xkv.xk_sr_params(1, w.n_q_heads, w.n_kv_heads, w.head_dim, w.T, w.rank_k, w.chunk, w.topk, w.sink,
                         w.recent, w.rope_theta, torch.bfloat16)
    dV = dev(V, torch.bfloat16)
    out = torch.empty((1, w.n_q_heads, w.head_dim), device="cuda", dtype=torch.float32)
    ws = xkv.workspace(xkv.xkv_xk_sr_host_workspace_size(p))
    P = lambda t: C.c_void_p(t.data_ptr())
    st = xkv.lib.xkv_xk_sr_attention_decode_host_values(C.byref(p), P(d["q"]), P(d["A_K"]), P(d["Bt_K"]), P(dV),
                                                        P(d["landmarks"]), P(d["sr_K"]), P(d["sr_V"]), P(out), None,
                                                        P(ws), ws.numel(), None)
    assert st == xkv.XKV_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert xkv.get_device_status() == 0
