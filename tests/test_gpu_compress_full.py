"""GPU parity of the cross-layer factorisation at the full sizes of the five
workloads, against the CPU oracle's statistics in tests/golden/compress_oracle.json
(written by tests/golden/make_compress_golden.py, which calls only the oracle and
the input generator; the oracle's Jacobi on a 8192 x 8192 Gram takes hours).

Cases: the prefill sweep (d = 1024, T = 32768 in four 8192-row shards, G = 1, 2,
4, 8, r = 128 G), the Qwen2.5-7B-shaped group (T = 131072, d = 512, keys at
r = 256, values at r = 384) and the Llama-3.1-8B-shaped 16K group (r = 512,
keys and values).

Criteria (the synthetic spectra have no gap at r, so factors are compared
through their errors, never elementwise; Eckart-Young, KQ-SVD 3.3):
  * subspace error ||X - X V_r V_r^T||_F of the GPU's f32 basis, evaluated in
    fp64, within 1e-3 (relative) of the oracle's;
  * stored-factor error ||X - A Bt^T||_F of the GPU's bf16 factors within 1e-3
    of the oracle's own bf16-rounded stored-factor error;
  * where r exceeds the generator's latent dimension m (the G = 8 sweep point,
    r = 1024, m = 768), the directions past m are a noise floor below fp32
    resolution: both squared errors may then exceed the oracle's by at most
    the energy the exact subspace keeps in directions m .. r - 1 (stored by the
    oracle script), and never fall below the oracle's subspace error;
  * xkv_compress_group gives the same bits as its pieces (Gram over shards,
    xkv_factor_gram, xkv_project);
  * for the Llama keys, KV-CoRE's NER of every 1024-wide layer block within
    1e-3 with the same numerical rank, and the 95 % energy rank within one.
"""
import json
import os

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "compress_oracle.json")
CASES = ["sweep_g1", "sweep_g2", "sweep_g4", "sweep_g8", "qwen_k", "qwen_v", "llama16k_k", "llama16k_v"]


def _golden(name):
    with open(GOLDEN) as f:
        data = json.load(f)
    if name not in data:
        pytest.fail(f"{name} missing from {GOLDEN}; run tests/golden/make_compress_golden.py {name}")
    return data[name]


def _workload(rec):
    if rec["workload"].startswith("compress_sweep_g"):
        return synth.compression_sweep(rec["G"])
    return synth.WORKLOADS[rec["workload"]]


def _fro64(M):
    return float(torch.linalg.vector_norm(M.double()).item())


@pytest.mark.parametrize("name", CASES)
def test_compress_matches_oracle_at_full_size(xkv, name):
    rec = _golden(name)
    w = _workload(rec)
    layers = synth.kv_group(w, rec["batch"], rec["group"], rec["kind"])
    G, r = len(layers), rec["rank"]
    T, d = layers[0].shape
    assert (G, int(T), int(d)) == (rec["G"], rec["T"], rec["d"])
    n = G * d
    bf = torch.bfloat16
    X = [torch.from_numpy(l).cuda().to(bf) for l in layers]
    del layers
    p = synth.oversample(r)
    # the pieces: Gram over 8192-row shards, factor, project
    Cg = torch.zeros((n, n), dtype=torch.float32, device="cuda")
    wsg = xkv.workspace(xkv.xkv_gram_workspace_size(G, 8192, d, bf))
    for s in range(0, T, 8192):
        xkv.xkv_gram_accumulate([x[s:s + 8192] for x in X], Cg, wsg)
    Bt = torch.empty((n, r), dtype=bf, device="cuda")
    Vr = torch.empty((n, r), dtype=torch.float32, device="cuda")
    ev = torch.empty((r,), dtype=torch.float32, device="cuda")
    xkv.xkv_factor_gram(Cg, G, d, T, r, Bt, iters=8, oversample=p, Vr_out=Vr, eigvals=ev)
    A = torch.empty((T, r), dtype=bf, device="cuda")
    xkv.xkv_project(X, Vr, A)
    torch.cuda.synchronize()
    assert xkv.get_device_status() == 0
    # the whole entry point gives the same bits
    A2 = torch.empty_like(A)
    Bt2 = torch.empty_like(Bt)
    ev2 = torch.empty_like(ev)
    xkv.xkv_compress_group(X, r, A2, Bt2, iters=8, oversample=p, shard_rows=8192, eigvals=ev2)
    torch.cuda.synchronize()
    assert xkv.get_device_status() == 0
    assert torch.equal(A2, A) and torch.equal(Bt2, Bt) and torch.equal(ev2, ev)
    del A2, Bt2, Cg
    # errors in fp64 on the device
    Xd = torch.cat([x.double() for x in X], dim=1)
    del X
    V = Vr.double()
    sub = _fro64(Xd - (Xd @ V) @ V.T)
    sto = _fro64(Xd - A.double() @ Bt.double().T)
    del Xd
    if r <= w.latent:
        assert abs(sub - rec["err_subspace"]) <= 1e-3 * rec["err_subspace"], (sub, rec["err_subspace"])
        assert abs(sto - rec["err_stored"]) <= 1e-3 * rec["err_stored"], (sto, rec["err_stored"])
    else:
        # the rank reaches past the generator's latent dimension m into the flat
        # noise floor, whose eigenvalues (about 6.7 here) lie below the fp32
        # rounding of the largest (2.5e8 x 6e-8): there the fp32 Gram does not
        # determine which noise directions are the top ones.  The basis must
        # hold every direction above m (missing one costs thousands), and it
        # may lose at most the energy the exact top-r subspace keeps past m
        extra = rec["energy_latent_to_rank"] * (1 + 1e-3)
        assert sub ** 2 <= rec["err_subspace"] ** 2 + extra, (sub, rec["err_subspace"], extra)
        assert sto ** 2 <= rec["err_stored"] ** 2 + extra, (sto, rec["err_stored"], extra)
        # every direction above m is held: the Ritz values at m - 4 .. m - 1 are
        # the oracle's eigenvalues there (a missed one would leave a noise-level
        # Ritz value, 55 times smaller, among them)
        m = rec["latent"]
        evm = ev.double().cpu().numpy()
        assert np.allclose(evm[m - 4:m], rec["lam_at_latent"][:4], rtol=1e-3), (evm[m - 4:m + 4], rec["lam_at_latent"])
    # Eckart-Young: no rank-r basis beats the oracle's (up to its rounding)
    assert sub >= rec["err_subspace"] * (1 - 1e-6)
    # the leading Ritz values are the leading eigenvalues
    evh = ev.double().cpu().numpy()
    lam = np.array(rec["lam_top"])
    assert np.allclose(evh[:len(lam)], lam, rtol=1e-4)
    assert np.all(np.diff(evh) <= 1e-6 * evh[0])


def test_ner_and_energy_rank_of_the_llama_16k_key_blocks(xkv):
    rec = _golden("llama16k_k")
    w = _workload(rec)
    layers = synth.kv_group(w, 0, 0, "K")
    G, d = len(layers), rec["d"]
    n = G * d
    X = [torch.from_numpy(l).cuda().to(torch.bfloat16) for l in layers]
    Cg = torch.zeros((n, n), dtype=torch.float32, device="cuda")
    xkv.xkv_gram_accumulate(X, Cg)
    ner = torch.empty(G, dtype=torch.float32, device="cuda")
    er = torch.empty(G, dtype=torch.float32, device="cuda")
    rk = torch.empty(G, dtype=torch.int32, device="cuda")
    xkv.xkv_ner(Cg, d, ner, er, rk)
    e95 = xkv.xkv_energy_rank(Cg, d, 0.95)
    torch.cuda.synchronize()
    assert xkv.get_device_status() == 0
    assert rk.cpu().tolist() == rec["ner_rank"]
    assert np.abs(ner.cpu().numpy() - np.array(rec["ner"])).max() <= 1e-3
    assert np.abs(e95.cpu().numpy() - np.array(rec["energy_rank_95"])).max() <= 1
