"""Shared helpers of the GPU parity tests: moving seeded inputs to the device in
their storage dtype, and the comparison rules (selection tolerance, bf16 ulps)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth


def tdtype(w) -> torch.dtype:
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def dev(x: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    """float32 host array whose values are exact in `dtype` -> CUDA tensor."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to("cuda").to(dtype).contiguous()


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def sr_inputs_on_device(w, inp, T=None):
    dt = tdtype(w)
    return {k: dev(v, dt) for k, v in inp.items()}


def run_sr(xkv, w, d_inp, T=None, sel=True):
    T = T or w.T
    p = xkv.sr_params(d_inp["q"].shape[0], w.n_q_heads, w.n_kv_heads, w.head_dim, T, d_inp["A_K"].shape[-1],
                      d_inp["A_V"].shape[-1], w.chunk, w.topk, w.sink, w.recent, w.rope_theta, tdtype(w))
    B = d_inp["q"].shape[0]
    out = torch.full((B, w.n_q_heads, w.head_dim), float("nan"), device="cuda", dtype=torch.float32)
    sel_out = torch.full((B, w.n_kv_heads, w.topk), -1, device="cuda", dtype=torch.int32) if sel else None
    xkv.xkv_sr_attention_decode(p, d_inp["q"], d_inp["A_K"], d_inp["Bt_K"], d_inp["A_V"], d_inp["Bt_V"],
                                d_inp["landmarks"], d_inp["sr_K"], d_inp["sr_V"], out, sel_out)
    torch.cuda.synchronize()
    return out, sel_out


def check_selection(sel_gpu: np.ndarray, scores: np.ndarray, k: int, rel: float = 1e-3, units=None):
    """GPU top-k set equals the exact one except chunks scoring within rel of the
    k-th score (ties and near-ties may go either way)."""
    B, H, _ = sel_gpu.shape
    for b in range(B):
        for h in range(H):
            if units is not None and b * H + h not in units:
                continue
            s = scores[b, h]
            g = sel_gpu[b, h]
            assert np.all(np.diff(g) > 0), "selection must be strictly ascending"
            assert g.min() >= 0 and g.max() < s.size
            kth = np.sort(s)[::-1][k - 1]
            exact = set(np.lexsort((np.arange(s.size), -s))[:k].tolist())
            diff = set(g.tolist()) ^ exact
            band = rel * max(abs(kth), 1e-30)
            for c in diff:
                assert abs(s[c] - kth) <= band, (b, h, c, s[c], kth)


def ulp_bf16(x: np.ndarray) -> np.ndarray:
    ax = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)
