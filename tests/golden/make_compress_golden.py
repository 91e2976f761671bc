"""Write tests/golden/compress_oracle.json: the CPU oracle's factorisation
statistics for the full-size compression cases, which take the oracle minutes to
hours (cyclic Jacobi on a 8192 x 8192 Gram is the longest), so the GPU tests
read them instead of recomputing them.

Only the oracle (oracle/) and the seeded input generator (synth/) are called.
Inputs are drawn on the CPU, so a GPU test that draws the same workload gets
bit-identical bf16 caches.

Cases (name: workload, tensor, rank):
  sweep_g1 .. sweep_g8  prefill compression sweep, d = 1024, T = 32768, G = 1, 2,
                        4, 8, r = 128 G, keys of sequence 0, group 0;
  qwen_k, qwen_v        Qwen2.5-7B shape, T = 131072, G = 4, d = 512, keys at
                        r = 256 and values at r = 384, sequence 0, group 0;
  llama16k_k, _v        Llama-3.1-8B shape, T = 16384, G = 4, d = 1024, r = 512;
                        the key case also stores KV-CoRE's NER and the 95 %
                        energy rank of each 1024-wide layer block.

Usage: python tests/golden/make_compress_golden.py [--spectrum] [case ...]
Each finished case is merged into the JSON file at once, so an interrupted run
keeps what it has.  --spectrum adds, for a case whose rank exceeds the
generator's latent dimension m (sweep_g8), the energy that the exact top-rank
subspace keeps in the directions m .. rank - 1 (eigenvalues of the oracle's
fp64 Gram), without recomputing the factorisation.
"""
from __future__ import annotations

import json
import os
import sys
import time

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import synth  # noqa: E402

OUT = os.path.join(HERE, "compress_oracle.json")


def cases():
    q = synth.WORKLOADS["qwen7b_128k_b2"]
    l16 = synth.WORKLOADS["llama_group_16k"]
    out = {}
    for G in (1, 2, 4, 8):
        w = synth.compression_sweep(G)
        out[f"sweep_g{G}"] = (w, "K", w.rank_k)
    out["qwen_k"] = (q, "K", q.rank_k)
    out["qwen_v"] = (q, "V", q.rank_v)
    out["llama16k_k"] = (l16, "K", l16.rank_k)
    out["llama16k_v"] = (l16, "V", l16.rank_v)
    return out


ORDER = ["sweep_g1", "sweep_g2", "qwen_k", "qwen_v", "llama16k_k", "llama16k_v", "sweep_g4", "sweep_g8"]


def run_case(name, w, kind, rank):
    t0 = time.time()
    layers = synth.kv_group(w, 0, 0, kind)
    t_in = time.time() - t0
    T, d = layers[0].shape
    t0 = time.time()
    res = oracle.compress_group(layers, rank)
    t_cmp = time.time() - t0
    lam = res["lam"]
    rec = dict(workload=w.name, kind=kind, batch=0, group=0, T=int(T), G=len(layers), d=int(d), rank=int(rank),
               err_subspace=float(res["err_subspace"]), err_stored=float(res["err_stored"]),
               tail=float(res["tail"]), xx=float(res["xx"]), sweeps=int(res["sweeps"]),
               lam_top=[float(x) for x in lam[:16]],
               lam_at_rank=[float(x) for x in lam[max(rank - 4, 0):rank + 4]],
               oracle_seconds=round(t_cmp, 1), input_seconds=round(t_in, 1), threads=oracle.num_threads())
    del res
    if name == "llama16k_k":
        t0 = time.time()
        Cm = oracle.gram(layers)
        ner, er, rk, _ = oracle.ner(Cm, d)
        ranks95, _ = oracle.energy_rank(Cm, d, 0.95)
        rec["ner_block"] = int(d)
        rec["ner"] = [float(x) for x in ner]
        rec["erank"] = [float(x) for x in er]
        rec["ner_rank"] = [int(x) for x in rk]
        rec["energy_rank_95"] = [int(x) for x in ranks95]
        rec["ner_seconds"] = round(time.time() - t0, 1)
    return rec


def spectrum_fields(w, kind, rank):
    """For a rank past the generator's latent dimension m: the energy of the
    eigen-directions m .. rank - 1 that the exact top-rank subspace keeps,
    sum of those eigenvalues of the oracle's fp64 Gram (LAPACK eigvalsh as a
    library step), and the eigenvalues around m."""
    layers = synth.kv_group(w, 0, 0, kind)
    Cm = oracle.gram(layers)
    lam = np.linalg.eigvalsh(Cm)[::-1]
    m = int(w.latent)
    return dict(latent=m, energy_latent_to_rank=float(lam[m:rank].sum()),
                lam_at_latent=[float(x) for x in lam[max(m - 4, 0):m + 4]])


def save(name, fields, replace):
    data = {}
    if os.path.exists(OUT):
        with open(OUT) as f:
            data = json.load(f)
    data[name] = fields if replace else {**data.get(name, {}), **fields}
    tmp = OUT + ".tmp"
    with open(tmp, "w") as f:
        json.dump(data, f, indent=1, sort_keys=True)
        f.write("\n")
    os.replace(tmp, OUT)


def main(argv):
    spectrum = "--spectrum" in argv
    todo = [a for a in argv if not a.startswith("--")] or ORDER
    allc = cases()
    for name in todo:
        w, kind, rank = allc[name]
        print(f"[{time.strftime('%H:%M:%S')}] {name}: {w.name} {kind} r={rank}", flush=True)
        if spectrum:
            if rank <= w.latent:
                print("  rank within the latent dimension: nothing to add", flush=True)
                continue
            fields = spectrum_fields(w, kind, rank)
            save(name, fields, replace=False)
            print(f"  done: energy of directions {fields['latent']} .. {rank - 1}: "
                  f"{fields['energy_latent_to_rank']:.6g}", flush=True)
            continue
        rec = run_case(name, w, kind, rank)
        save(name, rec, replace=True)
        print(f"  done: sweeps {rec['sweeps']}, {rec['oracle_seconds']} s, err_sub {rec['err_subspace']:.6g}, "
              f"err_sto {rec['err_stored']:.6g}", flush=True)


if __name__ == "__main__":
    main(sys.argv[1:])
