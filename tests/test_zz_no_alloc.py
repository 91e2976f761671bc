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


def _reject_oversized(xkv):
    # batch 64 at 64K tokens needs far more than the fixed array; the call must
    # return XKV_ERR_UNSUPPORTED before touching any pointer (none is real here)
    p = xkv.sr_params(64, 32, 8, 128, 65536, 512, 512, 8, 256, 8, 32, 5e5, torch.bfloat16)
    need = xkv.xkv_sr_workspace_size(p)
    assert need > xkv.SR_STATIC_SCRATCH_BYTES
    fake = [C.c_void_p(0x10000 * (i + 1)) for i in range(10)]
    st = xkv.lib.xkv_sr_attention_decode_noalloc(C.byref(p), *fake, None)
    assert st == xkv.XKV_ERR_UNSUPPORTED


def test_noalloc_rejects_scratch_beyond_the_array(xkv):
    _reject_oversized(xkv)


@pytest.mark.gpu
def test_noalloc_rejects_scratch_beyond_the_array_on_the_gpu(xkv):
    # the same refusal with a device present (the plan then reads the real SM count)
    _reject_oversized(xkv)
    torch.cuda.synchronize()
    assert xkv.get_device_status() == 0


_PLAN_SCRIPT = r"""
import sys
sys.path.insert(0, {root!r})
import torch
import cross_layer_rank_b200 as xkv
import synth
for name in ("llama8b_64k_b4", "qwen7b_128k_b2"):
    w = synth.WORKLOADS[name]
    p = xkv.sr_params(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.T, w.rank_k, w.rank_v, w.chunk, w.topk,
                      w.sink, w.recent, w.rope_theta, torch.bfloat16)
    print(name, xkv.xkv_sr_workspace_size(p), xkv.SR_STATIC_SCRATCH_BYTES)
"""


@pytest.mark.gpu
@pytest.mark.parametrize("force_simt", ["0", "1"])
def test_noalloc_array_covers_the_benchmark_layers(xkv, force_simt):
    # one decode layer of the 64K batch-4 Llama shape and of the 128K batch-2
    # Qwen shape fits the fixed array, for the tensor-core plan and for the
    # CUDA-core plan (XKV_FORCE_SIMT=1 is read once per process, hence the
    # child process); the plan depends on the device's SM count
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, XKV_FORCE_SIMT=force_simt)
    r = subprocess.run([sys.executable, "-c", _PLAN_SCRIPT.format(root=root)], env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [l.split() for l in r.stdout.strip().splitlines()]
    assert [l[0] for l in lines] == ["llama8b_64k_b4", "qwen7b_128k_b2"]
    for _, need, cap in lines:
        assert 0 < int(need) <= int(cap)
