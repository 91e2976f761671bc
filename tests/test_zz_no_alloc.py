"""xkv_sr_attention_decode_noalloc: the decode step with the library's fixed
scratch array instead of a caller workspace.  It must give the workspace
entry point's results (within the decode tolerance: output max-abs 1e-2,
same selection) on two calls in a row, and reject requests whose scratch
exceeds the array before launching anything.

The file name keeps it last in collection; every test here also passes alone.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import synth
from gpu_helpers import host, run_sr, sr_inputs_on_device, tdtype


def _noalloc(xkv, w, d_inp, T=None):
    T = T or w.T
    p = xkv.sr_params(d_inp["q"].shape[0], w.n_q_heads, w.n_kv_heads, w.head_dim, T, d_inp["A_K"].shape[-1],
                      d_inp["A_V"].shape[-1], w.chunk, w.topk, w.sink, w.recent, w.rope_theta, tdtype(w))
    B = d_inp["q"].shape[0]
    out = torch.full((B, w.n_q_heads, w.head_dim), float("nan"), device="cuda", dtype=torch.float32)
    sel = torch.full((B, w.n_kv_heads, w.topk), -1, device="cuda", dtype=torch.int32)
    xkv.xkv_sr_attention_decode_noalloc(p, d_inp["q"], d_inp["A_K"], d_inp["Bt_K"], d_inp["A_V"], d_inp["Bt_V"],
                                        d_inp["landmarks"], d_inp["sr_K"], d_inp["sr_V"], out, sel)
    torch.cuda.synchronize()
    assert xkv.get_device_status() == 0
    return host(out), sel.cpu().numpy()


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["ragged_bf16", "llama_group_16k"])
def test_noalloc_matches_workspace_entry_point_twice(xkv, name):
    if name == "ragged_bf16":
        w = synth.Workload("sr_bf16_small", 2, 4, 4, 2, 128, 8, 8 + 32 + 8 * 150, 96, 0.8, 128, 192, topk=37)
    else:
        w = synth.WORKLOADS["llama_group_16k"]
    d_inp = sr_inputs_on_device(w, synth.compressed_cache(w, 1))
    ref_out, ref_sel = run_sr(xkv, w, d_inp)
    ref_out, ref_sel = host(ref_out), ref_sel.cpu().numpy()
    for _ in range(2):
        out, sel = _noalloc(xkv, w, d_inp)
        assert np.isfinite(out).all()
        assert np.abs(out - ref_out).max() <= 1e-2
        assert np.array_equal(sel, ref_sel)


def test_noalloc_rejects_scratch_beyond_the_array(xkv):
    # batch 64 at 64K tokens needs far more than the fixed array; the call must
    # return XKV_ERR_UNSUPPORTED before touching any pointer (none is real here)
    p = xkv.sr_params(64, 32, 8, 128, 65536, 512, 512, 8, 256, 8, 32, 5e5, torch.bfloat16)
    need = xkv.xkv_sr_workspace_size(p)
    assert need > xkv.SR_STATIC_SCRATCH_BYTES
    fake = [C.c_void_p(0x10000 * (i + 1)) for i in range(10)]
    st = xkv.lib.xkv_sr_attention_decode_noalloc(C.byref(p), *fake, None)
    assert st == xkv.XKV_ERR_UNSUPPORTED
