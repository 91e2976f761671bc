"""GPU parity: full reconstruction (xkv_full_reconstruct), dense decode
attention (the comparison path of the xKV explainer's Fig. 6) and chunk
landmarks (xkv_build_landmarks) against the oracle on identical inputs.

bf16 outputs may differ from the fp64 oracle by at most one bf16 ulp of the
oracle value (the GPU accumulates in fp32 and rounds once) plus a floor for
fp32 cancellation (1e-4 of the largest magnitude for the r-term products, 1e-6
of the largest key for the 8-term landmark means); f32 outputs to 1e-5
relative; attention to max-abs 1e-2."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import dev, host, ulp_bf16

pytestmark = pytest.mark.gpu


def _rand(key, shape, scale=1.0):
    return (synth.normal(synth.stream_key(*key), int(np.prod(shape))).reshape(shape) * scale).astype(np.float32)


@pytest.mark.parametrize("T,Hkv,hd,r,rope", [(1000, 2, 128, 128, True), (1000, 2, 128, 128, False),
                                             (777, 4, 64, 192, True), (256, 8, 128, 512, True)])
def test_full_reconstruct_bf16(xkv, T, Hkv, hd, r, rope):
    d = Hkv * hd
    A = synth.to_storage(_rand(("recA", T, r), (T, r), 0.5), "bf16")
    Bt = synth.to_storage(_rand(("recB", d, r), (d, r), 1 / np.sqrt(r)), "bf16")
    out = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    xkv.xkv_full_reconstruct(dev(A, torch.bfloat16), dev(Bt, torch.bfloat16), Hkv, hd, rope, 5e5, out)
    torch.cuda.synchronize()
    ref = oracle.full_reconstruct(A, Bt, Hkv, hd, rope, 5e5)
    g = host(out).astype(np.float64)
    assert np.all(np.abs(g - ref) <= ulp_bf16(ref) + 1e-4 * np.abs(ref).max())


@pytest.mark.parametrize("rope", [True, False])
def test_full_reconstruct_f32(xkv, rope):
    T, Hkv, hd, r = 1024, 2, 64, 64
    d = Hkv * hd
    A = _rand(("recA32",), (T, r))
    Bt = _rand(("recB32",), (d, r), 1 / np.sqrt(r))
    out = torch.empty((T, d), dtype=torch.float32, device="cuda")
    xkv.xkv_full_reconstruct(dev(A, torch.float32), dev(Bt, torch.float32), Hkv, hd, rope, 5e5, out)
    torch.cuda.synchronize()
    ref = oracle.full_reconstruct(A, Bt, Hkv, hd, rope, 5e5)
    assert np.abs(host(out) - ref).max() <= 1e-5 * np.abs(ref).max()


@pytest.mark.parametrize("dtype,hd,T,gq", [("bf16", 128, 3000, 4), ("f32", 64, 1111, 2), ("bf16", 128, 200, 7)])
def test_dense_decode(xkv, dtype, hd, T, gq):
    B, Hkv = 2, 2
    Hq = Hkv * gq
    d = Hkv * hd
    q = synth.to_storage(_rand(("dq", dtype, T), (B, Hq, hd)), dtype)
    K = synth.to_storage(_rand(("dK", dtype, T), (B, T, d)), dtype)
    V = synth.to_storage(_rand(("dV", dtype, T), (B, T, d)), dtype)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    p = xkv.dense_params(B, Hq, Hkv, hd, T, tdt)
    out = torch.empty((B, Hq, hd), dtype=torch.float32, device="cuda")
    xkv.xkv_dense_attention_decode(p, dev(q, tdt), dev(K, tdt), dev(V, tdt), out)
    torch.cuda.synchronize()
    ref = oracle.dense_decode(q, K, V, Hkv)
    assert np.abs(host(out) - ref).max() <= (1e-2 if dtype == "bf16" else 2e-5)


def test_landmarks_f32_tiny(xkv):
    w = synth.WORKLOADS["tiny_f32"]
    K = synth.kv_group(w, 0, 0, "K", layers=[1])[0]
    out = torch.empty((w.n_kv_heads, w.n_mid, w.head_dim), dtype=torch.float32, device="cuda")
    xkv.xkv_build_landmarks(dev(K, torch.float32), w.n_kv_heads, w.head_dim, w.chunk, w.sink, w.recent,
                            w.rope_theta, out)
    torch.cuda.synchronize()
    ref = oracle.landmarks(K, w.n_kv_heads, w.head_dim, w.chunk, w.sink, w.recent, w.rope_theta)
    assert np.abs(host(out) - ref).max() <= 1e-5 * np.abs(ref).max()


@pytest.mark.parametrize("T", [8 + 32 + 8 * 512, 8 + 32 + 8 * 2043])
def test_landmarks_bf16_within_one_ulp(xkv, T):
    w = synth.WORKLOADS["llama_group_16k"]
    K = synth.kv_group(w, 0, 0, "K", T=T, layers=[2])[0]
    out = torch.empty((w.n_kv_heads, (T - 40) // 8, w.head_dim), dtype=torch.bfloat16, device="cuda")
    xkv.xkv_build_landmarks(dev(K, torch.bfloat16), w.n_kv_heads, w.head_dim, w.chunk, w.sink, w.recent,
                            w.rope_theta, out)
    torch.cuda.synchronize()
    ref = oracle.landmarks(K, w.n_kv_heads, w.head_dim, w.chunk, w.sink, w.recent, w.rope_theta)
    g = host(out).astype(np.float64)
    # a chunk mean can cancel: fp32 summation then leaves an absolute error of
    # a few fp32 ulps of the summed keys, which exceeds a bf16 ulp of a tiny mean
    floor = 1e-6 * np.abs(K).max()
    excess = np.abs(g - ref) / (ulp_bf16(ref) + floor)
    assert excess.max() <= 1.0, (excess.max(), np.unravel_index(excess.argmax(), excess.shape))
