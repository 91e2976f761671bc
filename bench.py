"""Benchmark of the xKV hot path on B200.

One step = one decode step of Selective-Reconstruction attention over every
layer of the model for the whole batch (32 layers x batch 4 at 64K context for
the Llama-3.1-8B shape), captured in one CUDA graph: per layer the library
scores landmarks, selects the top-k chunks, rebuilds the selected K/V rows from
the shared basis and attends.  Metric: decode tokens/s (batch / step time) and
the HBM bandwidth implied by the step's algorithmic bytes.

The compressed caches are produced on the GPU by the library itself before
timing (synthetic K/V -> xkv_compress_group -> xkv_build_landmarks); that
prefill work is timed separately and reported under "prefill".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the CPU oracle, bounded sample

Multi-GPU (torchrun): every rank runs its own batch (independent sequences, no
data-path collective: "scaling": "weak"); the step time is the maximum over
ranks of the device-timed region.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "SR-attn decode tokens/s & HBM GB/s (% of peak), Llama-8B shape, 64K ctx"


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def sr_bytes_per_unit(w) -> int:
    """Algorithmic HBM bytes of one (batch, layer, KV head) SR decode unit."""
    el = 2 if w.dtype == "bf16" else 4
    n_mid = w.n_mid
    return (n_mid * w.head_dim * el                                  # landmarks
            + w.topk * w.chunk * (w.rank_k + w.rank_v) * el          # selected A slabs
            + (w.rank_k + w.rank_v) * w.head_dim * el                # Bt slices
            + (w.sink + w.recent) * w.head_dim * 2 * el              # raw sink/recent K and V
            + 2 * w.gq * w.head_dim * el)                            # queries in, outputs out


def attend_bytes_per_unit(w) -> int:
    """Algorithmic HBM bytes of the attend stage for one unit: the selected
    A_K and A_V chunk rows, the head's Bt_K slice and the group's queries."""
    el = 2 if w.dtype == "bf16" else 4
    return (w.topk * w.chunk * (w.rank_k + w.rank_v) * el + w.rank_k * w.head_dim * el
            + w.gq * w.head_dim * el)


def code_digest(text: str) -> str:
    """sha1 of C/C++/CUDA source with comments and blank lines removed and runs
    of white space folded (string and character literals kept), so that the
    digest changes with the code and not with its comments or layout."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = [" ".join(ln.split()) for ln in "".join(out).splitlines()]
    return hashlib.sha1("\n".join(ln for ln in lines if ln).encode()).hexdigest()


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary (profiles/traffic.json), or None unless the kernel source's code
    (comments aside) is still the code that was profiled."""
    tp = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        ent = json.load(open(tp)).get(workload)
        src = open(os.path.join(ROOT, ent["source"]), encoding="utf-8").read()
        if code_digest(src) == ent["source_code_sha1"]:
            return ent["bytes_per_launch"]
    except Exception:
        pass
    return None


def cache_ratio(w, values_compressed: bool = True):
    """Dense K+V cache bytes of a layer over the compressed cache's bytes per
    layer: the group's shared A_K and A_V plus its per-layer Bt slices, alone
    and with the landmarks.  Uncompressed values (the xK-SR mode) count T d
    elements instead of A_V and Bt_V.  The raw sink/recent rows are left out."""
    el = 2 if w.dtype == "bf16" else 4
    dense = 2 * w.T * w.d * el
    rv = w.rank_v if values_compressed else 0
    ab = (w.T * (w.rank_k + rv) + w.group * w.d * (w.rank_k + rv)) * el / w.group
    if not values_compressed:
        ab += w.T * w.d * el
    lm = w.n_kv_heads * w.n_mid * w.head_dim * el
    return round(dense / ab, 3), round(dense / (ab + lm), 3)


def xk_attend_bytes_per_unit(w) -> int:
    """The attend stage's algorithmic bytes per unit in the xK-SR mode: the
    selected A_K rows, the selected rows' hd value columns of the head, the
    Bt_K head slice and the group's queries."""
    el = 2 if w.dtype == "bf16" else 4
    return (w.topk * w.chunk * (w.rank_k + w.head_dim) * el + w.rank_k * w.head_dim * el
            + w.gq * w.head_dim * el)


def stage_rooflines(w, stage_ms, peak_gbs):
    """Achieved GB/s of each decode launch of one layer call (whole batch)
    against the HBM peak, from its algorithmic bytes:
      score   the landmarks and the queries;
      top-k   the chunk scores (fp32) and, for the window blocks, the raw
              sink/recent K and V rows (latency-bound: few bytes);
      attend  the selected A rows, the Bt_K head slices and the queries;
      combine the Bt_V head slices and the outputs (plus partials in L2)."""
    el = 2 if w.dtype == "bf16" else 4
    units = w.batch * w.n_kv_heads
    byts = {
        "score": units * (w.n_mid * w.head_dim * el + w.gq * w.head_dim * el),
        "topk_window": units * (w.n_mid * 4 + (w.sink + w.recent) * w.head_dim * 2 * el),
        "attend": units * attend_bytes_per_unit(w),
        "combine": units * (w.rank_v * w.head_dim * el + w.gq * w.head_dim * 4),
    }
    out = {}
    for (name, b), ms in zip(byts.items(), stage_ms):
        gbs = b / (ms / 1e3) / 1e9 if ms > 0 else 0.0
        out[name] = {"bytes": int(b), "achieved_gbs": round(gbs, 1), "frac": round(gbs / peak_gbs, 4)}
    return out


def landmark_bytes(w) -> int:
    """xkv_build_landmarks for one layer and sequence: T rows of K read, the
    middle chunks' landmarks written."""
    el = 2 if w.dtype == "bf16" else 4
    return w.T * w.d * el + w.n_kv_heads * w.n_mid * w.head_dim * el


def sr_flops_per_unit(w) -> int:
    rows = w.topk * w.chunk
    return (2 * rows * w.rank_k * w.head_dim                 # K rebuild
            + 2 * w.gq * w.n_mid * w.head_dim                # landmark scores
            + 4 * w.gq * (rows + w.sink + w.recent) * w.head_dim
            + 2 * w.gq * rows * w.rank_v + 2 * w.gq * w.rank_v * w.head_dim)


class Clocks:
    """nvidia-smi sampling during the timed region."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"xkv_bench_clocks_rank{index}.csv")

    def __enter__(self):
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        try:
            rows = [l.strip().split(",") for l in open(self.path) if l.strip()]
        except Exception:
            rows = []
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
                for nm, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(nm)
            except (ValueError, IndexError):
                continue
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------- set-up
def build_model(xkv, w, device, groups=None, log=print):
    """Compressed caches of every layer: A_K/A_V per group, Bt per layer,
    landmarks and raw sink/recent rows per layer, q per layer."""
    import torch
    bf = torch.bfloat16
    G, d, T, B = w.group, w.d, w.T, w.batch
    n_groups = groups or w.n_groups
    sw_rows = torch.tensor(list(range(w.sink)) + list(range(T - w.recent, T)), device=device)
    model = {"A_K": [], "A_V": [], "Bt_K": [], "Bt_V": [], "lm": [], "srK": [], "srV": [], "q": []}
    ws_bytes = xkv.xkv_compress_workspace_size(G, T, d, w.rank_k, synth.oversample(w.rank_k), 8192, bf)
    ws_bytes = max(ws_bytes, xkv.xkv_compress_workspace_size(G, T, d, w.rank_v, synth.oversample(w.rank_v), 8192, bf))
    ws = xkv.workspace(ws_bytes, device)
    prefill = {"compress_ms": [], "landmarks_ms": []}
    for g in range(n_groups):
        AK = torch.empty((B, T, w.rank_k), dtype=bf, device=device)
        AV = torch.empty((B, T, w.rank_v), dtype=bf, device=device)
        BtK = torch.empty((B, G * d, w.rank_k), dtype=bf, device=device)
        BtV = torch.empty((B, G * d, w.rank_v), dtype=bf, device=device)
        lms = [torch.empty((B, w.n_kv_heads, w.n_mid, w.head_dim), dtype=bf, device=device) for _ in range(G)]
        srK = [torch.empty((B, w.sink + w.recent, d), dtype=bf, device=device) for _ in range(G)]
        srV = [torch.empty((B, w.sink + w.recent, d), dtype=bf, device=device) for _ in range(G)]
        for b in range(B):
            # each sequence of the batch is factorised on its own
            for kind, A, Bt, r in (("K", AK, BtK, w.rank_k), ("V", AV, BtV, w.rank_v)):
                X = synth.kv_group_torch(w, b, g, kind, device)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                xkv.xkv_compress_group(X, r, A[b], Bt[b], iters=8, oversample=synth.oversample(r), shard_rows=8192,
                                       ws=ws)
                e1.record()
                e1.synchronize()
                prefill["compress_ms"].append(e0.elapsed_time(e1))
                for l in range(G):
                    if kind == "K":
                        e0.record()
                        xkv.xkv_build_landmarks(X[l], w.n_kv_heads, w.head_dim, w.chunk, w.sink, w.recent,
                                                w.rope_theta, lms[l][b])
                        e1.record()
                        e1.synchronize()
                        prefill["landmarks_ms"].append(e0.elapsed_time(e1))
                        srK[l][b].copy_(X[l].index_select(0, sw_rows))
                    else:
                        srV[l][b].copy_(X[l].index_select(0, sw_rows))
                del X
        for l in range(G):
            model["A_K"].append(AK)
            model["A_V"].append(AV)
            # per-layer factors [B][d][r] (batch stride d r)
            model["Bt_K"].append(BtK[:, l * d:(l + 1) * d].contiguous())
            model["Bt_V"].append(BtV[:, l * d:(l + 1) * d].contiguous())
            model["lm"].append(lms[l])
            model["srK"].append(srK[l])
            model["srV"].append(srV[l])
        del BtK, BtV
        log(f"group {g + 1}/{n_groups} compressed")
    for layer in range(n_groups * G):
        q = synth.normal_torch(synth.stream_key(w.name, "q", layer), B * w.n_q_heads * w.head_dim, device)
        model["q"].append(q.view(B, w.n_q_heads, w.head_dim).to(bf))
    return model, prefill


def compress_profile(w):
    """xkv_compress_group (r = rank_k, p = max(64, r/4), 8 iterations,
    8192-row shards) and xkv_ner on its Gram for the (batch 0, group 0) keys;
    the second call pair runs between cudaProfilerStart and cudaProfilerStop."""
    import torch
    import cross_layer_rank_b200 as xkv
    device = torch.device("cuda", 0)
    X = synth.kv_group_torch(w, 0, 0, "K", device)
    r, G, d = w.rank_k, w.group, w.d
    A = torch.empty((w.T, r), dtype=torch.bfloat16, device=device)
    Bt = torch.empty((G * d, r), dtype=torch.bfloat16, device=device)
    C = torch.empty((G * d, G * d), dtype=torch.float32, device=device)
    ner = torch.empty(G, dtype=torch.float32, device=device)

    def once():
        xkv.xkv_compress_group(X, r, A, Bt, iters=8, oversample=synth.oversample(r), shard_rows=8192, gram_out=C)
        xkv.xkv_ner(C, d, ner)

    once()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.cudart().cudaProfilerStart()
    e0.record()
    once()
    e1.record()
    torch.cuda.synchronize()
    torch.cuda.cudart().cudaProfilerStop()
    assert xkv.get_device_status() == 0
    return {"workload": w.name, "compress_and_ner_ms": round(e0.elapsed_time(e1), 3)}


def measure_gram(xkv, w, device, spectra=True):
    """Device time of the Gram of one (batch 0, group 0) K shard set (T rows),
    of KV-CoRE's NER and energy rank on it (spectra=True) and of A = X V_r."""
    import torch
    X = synth.kv_group_torch(w, 0, 0, "K", device)
    n = w.group * w.d
    C = torch.zeros((n, n), dtype=torch.float32, device=device)
    ws = xkv.workspace(xkv.xkv_gram_workspace_size(w.group, 8192, w.d, torch.bfloat16), device)
    for _ in range(2):
        for s in range(0, w.T, 8192):
            xkv.xkv_gram_accumulate([x[s:s + 8192] for x in X], C, ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 3
    e0.record()
    for _ in range(reps):
        for s in range(0, w.T, 8192):
            xkv.xkv_gram_accumulate([x[s:s + 8192] for x in X], C, ws)
    e1.record()
    e1.synchronize()
    ms = e0.elapsed_time(e1) / reps
    flops = n * (n + 1) * w.T  # unique entries of the symmetric product, 2 T flops each
    # KV-CoRE's NER and the energy rank of every layer of the group, from this
    # Gram (the diagonal d x d blocks; scale-invariant, so the repeated sums do)
    ner = torch.empty(w.group, dtype=torch.float32, device=device)
    wsn = xkv.workspace(xkv.xkv_ner_workspace_size(n, w.d), device)
    todo = (("ner", lambda: xkv.xkv_ner(C, w.d, ner, ws=wsn)),
            ("energy_rank_95", lambda: xkv.xkv_energy_rank(C, w.d, 0.95, ws=wsn))) if spectra else ()
    spectra = {}
    for name, fn in todo:
        fn()
        torch.cuda.synchronize()
        e0.record()
        fn()
        e1.record()
        e1.synchronize()
        spectra[name + "_ms"] = round(e0.elapsed_time(e1), 3)
    assert xkv.get_device_status() == 0
    spectra["blocks"] = f"{w.group} x {w.d} x {w.d}"
    proj_ms, proj_flops = measure_projection(xkv, X, w.rank_k, device)
    return ms, flops, spectra, proj_ms, proj_flops


def _time_ms(fn, reps=3):
    """Mean device time of fn() over reps calls (after one untimed call)."""
    import torch
    fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    e1.synchronize()
    return e0.elapsed_time(e1) / reps


def measure_projection(xkv, X, rank, device):
    """Device time of A = X V_r (xkv_project, f32 basis as a bf16 hi/lo pair)
    for X = the given layers; algorithmic flops 2 T (G d) r (the hi/lo pair's
    second product is not counted)."""
    import torch
    G = len(X)
    T, d = X[0].shape
    n = G * d
    V = torch.randn((n, rank), dtype=torch.float32, device=device) / math.sqrt(n)
    A = torch.empty((T, rank), dtype=torch.bfloat16, device=device)
    ws = xkv.workspace(xkv.xkv_project_workspace_size(G, d, rank), device)
    ms = _time_ms(lambda: xkv.xkv_project(X, V, A, ws))
    flops = 2.0 * T * n * rank
    return ms, flops


def measure_compress_sweep(xkv, device, bf16_peak, log):
    """The prefill compression sweep: d = 1024 (8 x 128), T = 32768 in four
    8192-row shards, G = 1, 2, 4, 8 layers, r = 128 G.  Per G: the Gram over the
    shards, the projection, and the whole xkv_compress_group call."""
    import torch
    out = {}
    for G in (1, 2, 4, 8):
        w = synth.compression_sweep(G)
        X = synth.kv_group_torch(w, 0, 0, "K", device)
        n, r, T = G * w.d, w.rank_k, w.T
        C = torch.zeros((n, n), dtype=torch.float32, device=device)
        wsg = xkv.workspace(xkv.xkv_gram_workspace_size(G, 8192, w.d, torch.bfloat16), device)

        def gram():
            for s0 in range(0, T, 8192):
                xkv.xkv_gram_accumulate([x[s0:s0 + 8192] for x in X], C, wsg)
        g_ms = _time_ms(gram)
        g_fl = n * (n + 1) * T
        p_ms, p_fl = measure_projection(xkv, X, r, device)
        A = torch.empty((T, r), dtype=torch.bfloat16, device=device)
        Bt = torch.empty((n, r), dtype=torch.bfloat16, device=device)
        p = synth.oversample(r)
        wsc = xkv.workspace(xkv.xkv_compress_workspace_size(G, T, w.d, r, p, 8192, torch.bfloat16), device)
        c_ms = _time_ms(lambda: xkv.xkv_compress_group(X, r, A, Bt, iters=8, oversample=p, shard_rows=8192, ws=wsc),
                        reps=1)
        assert xkv.get_device_status() == 0
        out[f"G{G}"] = {"n": n, "rank": r, "gram_ms": round(g_ms, 4),
                        "gram_tflops": round(g_fl / (g_ms / 1e3) / 1e12, 1),
                        "gram_frac_of_bf16_peak": round(g_fl / (g_ms / 1e3) / 1e12 / bf16_peak, 4),
                        "projection_ms": round(p_ms, 4),
                        "projection_tflops": round(p_fl / (p_ms / 1e3) / 1e12, 1),
                        "projection_frac_of_bf16_peak": round(p_fl / (p_ms / 1e3) / 1e12 / bf16_peak, 4),
                        "compress_group_ms": round(c_ms, 3)}
        log(f"compression sweep G={G}: {out[f'G{G}']}")
        del X, C, A, Bt, wsc, wsg
        torch.cuda.empty_cache()
    out["shape"] = "d = 1024, T = 32768 (4 shards of 8192), r = 128 G; flops: Gram n (n+1) T, projection 2 T n r"
    return out


# --------------------------------------------------------- multi-rank
def max_over_ranks(values, world: int, device=None):
    """Element-wise maximum over all ranks of per-rank device times (every
    rank calls it, in the same order); the identity for one rank."""
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def job_throughput(batch_per_rank: int, world: int, ms_step: float):
    """Whole-job tokens per step and tokens/s: every rank decodes its own
    batch (independent sequences), the step lasts as long as the slowest rank."""
    tokens = batch_per_rank * world
    return tokens, tokens / (ms_step / 1e3)


# ------------------------------------------------------------------- arms
def run_cuda(args, rank, world, log):
    import torch
    import torch.distributed as dist
    import cross_layer_rank_b200 as xkv

    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(device)
    w = synth.WORKLOADS[args.workload]
    if args.batch:
        w = w.replace(batch=args.batch)
    n_groups = args.groups or w.n_groups
    L = n_groups * w.group
    bf = torch.bfloat16
    model, prefill = build_model(xkv, w, device, n_groups, log)
    gram_ms, gram_flops, spectra, proj_ms, proj_flops = (measure_gram(xkv, w, device) if args.prefill
                                                         else (None,) * 5)

    p = xkv.sr_params(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.T, w.rank_k, w.rank_v, w.chunk, w.topk,
                      w.sink, w.recent, w.rope_theta, bf)
    ws = xkv.workspace(xkv.xkv_sr_workspace_size(p), device)
    outs = [torch.empty((w.batch, w.n_q_heads, w.head_dim), dtype=torch.float32, device=device) for _ in range(L)]
    stream = torch.cuda.Stream(device)

    def layer_call(l, st):
        xkv.xkv_sr_attention_decode(p, model["q"][l], model["A_K"][l], model["Bt_K"][l], model["A_V"][l],
                                    model["Bt_V"][l], model["lm"][l], model["srK"][l], model["srV"][l], outs[l],
                                    None, ws, st)

    # warm-up (also loads the kernels) then capture one step in a CUDA graph
    with torch.cuda.stream(stream):
        for l in range(L):
            layer_call(l, stream)
    stream.synchronize()
    assert xkv.get_device_status(stream) == 0
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for l in range(L):
            layer_call(l, stream)
    # one graph per single layer for the per-call roofline timing
    g1 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g1, stream=stream):
        layer_call(0, stream)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    with Clocks(device.index) as clk:
        with torch.cuda.stream(stream):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record(stream)
            for _ in range(args.steps):
                graph.replay()
            e1.record(stream)
            e1.synchronize()
        ms_total = e0.elapsed_time(e1)
        if world > 1:
            dist.barrier()
        # per-call timing of one layer of SR decode (graph of one call), live
        with torch.cuda.stream(stream):
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(20)]
            for a, b_ in ev:
                a.record(stream)
                g1.replay()
                b_.record(stream)
            torch.cuda.synchronize()
        call_ms = statistics.median(a.elapsed_time(b_) for a, b_ in ev)
        # per-launch durations of the four stages (CUDA events recorded by the
        # library on the launching stream), layers in turn so caches are cold
        xkv.xkv_sr_profile_enable(True)
        stages = []
        with torch.cuda.stream(stream):
            for i in range(2 * L):
                layer_call(i % L, stream)
                stages.append(xkv.xkv_sr_profile_read())
        xkv.xkv_sr_profile_enable(False)
        stage_ms = [statistics.median(s_[j] for s_ in stages) for j in range(4)]
        # end to end through the C ABI: per step, pinned-host queries in, one
        # library call per layer, outputs back to pinned host memory
        q_host = [model["q"][l].cpu().pin_memory() for l in range(L)]
        o_host = [torch.empty_like(outs[l], device="cpu").pin_memory() for l in range(L)]
        with torch.cuda.stream(stream):
            e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e2.record(stream)
            for _ in range(args.steps):
                for l in range(L):
                    model["q"][l].copy_(q_host[l], non_blocking=True)
                for l in range(L):
                    layer_call(l, stream)
                for l in range(L):
                    o_host[l].copy_(outs[l], non_blocking=True)
            e3.record(stream)
            e3.synchronize()
        e2e_ms = e2.elapsed_time(e3)
    assert xkv.get_device_status(stream) == 0
    clocks = clk.summary()
    # secondary measurements: a failure there is logged and leaves the headline intact
    comparison = xk = None
    if args.comparison:
        try:
            comparison = measure_full_reconstruction(xkv, w, model, device, stream, call_ms)
        except Exception as e:  # noqa: BLE001
            log(f"comparison path not measured: {e!r}")
    if args.xk and world == 1:
        del graph, g1
        torch.cuda.empty_cache()
        try:
            xk = measure_xk_sr(xkv, w, model, device, stream, L, args.steps, args.warmup, _peaks()[0])
        except Exception as e:  # noqa: BLE001
            log(f"xK-SR mode not measured: {e!r}")
        try:
            if xk is not None:
                xk["host_values"] = measure_xk_sr_host(xkv, w, model, device, stream)
        except Exception as e:  # noqa: BLE001
            log(f"xK-SR with host values not measured: {e!r}")
    appended = None
    if world == 1 and args.xk:
        try:
            appended = measure_append(xkv, w, device, stream)
        except Exception as e:  # noqa: BLE001
            log(f"append not measured: {e!r}")

    ms_total, e2e_ms = max_over_ranks([ms_total, e2e_ms], world, device)
    ms_step = ms_total / args.steps
    tokens, value = job_throughput(w.batch, world, ms_step)
    units_step = w.batch * L * w.n_kv_heads
    bytes_step = sr_bytes_per_unit(w) * units_step
    hbm_gbs_peak, bf16_peak, _, peak_kind = _peaks()
    achieved_step = bytes_step / (ms_step / 1e3) / 1e9
    bytes_call = sr_bytes_per_unit(w) * w.batch * w.n_kv_heads
    achieved_call = bytes_call / (call_ms / 1e3) / 1e9
    # dominant kernel: selective reconstruction + attention (sr_attend)
    bytes_attend = attend_bytes_per_unit(w) * w.batch * w.n_kv_heads
    achieved_attend = bytes_attend / (stage_ms[2] / 1e3) / 1e9
    traffic = profiled_traffic(args.workload)
    q_bytes = sum(t.numel() * t.element_size() for t in model["q"])
    o_bytes = sum(t.numel() * t.element_size() for t in outs)
    res = {
        "metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "global_batch": tokens, "seq_len": w.T, "layers": L,
                   "kv_heads": w.n_kv_heads, "q_heads": w.n_q_heads, "head_dim": w.head_dim,
                   "rank_k": w.rank_k, "rank_v": w.rank_v, "topk": w.topk, "chunk": w.chunk, "sink": w.sink,
                   "recent": w.recent, "parallelism": f"dp{world}",
                   "l2": "inputs larger than L2 (%.1f GB touched per step)" % (bytes_step / 1e9)},
        "hbm_gbs": round(achieved_step, 1),
        "hbm_frac_of_peak": round(achieved_step / hbm_gbs_peak, 4),
        "roofline": {"bound": "hbm", "kernel": "sr_attend_tc (selective reconstruction + attention partials)",
                     "achieved": round(achieved_attend, 1), "peak": hbm_gbs_peak, "unit": "GB/s",
                     "frac": round(achieved_attend / hbm_gbs_peak, 4), "traffic": traffic,
                     "peak_source": f"{peak_kind} hbm_gbs (burst copy)", "bytes_per_launch": bytes_attend,
                     "launch_ms": round(stage_ms[2], 5)},
        "stages_ms": {"score": round(stage_ms[0], 5), "topk_window": round(stage_ms[1], 5),
                      "attend": round(stage_ms[2], 5), "combine": round(stage_ms[3], 5)},
        "stage_rooflines": stage_rooflines(w, stage_ms, hbm_gbs_peak),
        "layer_call": {"ms": round(call_ms, 5), "bytes": bytes_call, "achieved_gbs": round(achieved_call, 1),
                       "frac": round(achieved_call / hbm_gbs_peak, 4)},
        "e2e": {"value": round(tokens / (e2e_ms / args.steps / 1e3), 2), "unit": "tokens/s",
                "h2d_bytes_per_step": q_bytes, "d2h_bytes_per_step": o_bytes},
        "gpu_launches": 4 * L * args.steps,
        "cache_ratio": dict(zip(("a_b", "with_landmarks"), cache_ratio(w))),
        "clocks": clocks,
        "flops_per_step": sr_flops_per_unit(w) * units_step,
    }
    if comparison is not None:
        res["comparison"] = comparison
    if xk is not None:
        res["xk_sr"] = xk
    if appended is not None:
        res["multistep_append"] = appended
    if args.prefill:
        cm = prefill["compress_ms"]
        res["prefill"] = {"compress_group_ms_median": round(statistics.median(cm), 3), "groups_compressed": len(cm),
                          "landmarks_ms_median": round(statistics.median(prefill["landmarks_ms"]), 4),
                          "landmarks_frac_of_hbm": round(landmark_bytes(w) / (statistics.median(prefill["landmarks_ms"]) /
                                                                               1e3) / 1e9 / hbm_gbs_peak, 4),
                          "gram_ms": round(gram_ms, 4),
                          "gram_tflops": round(gram_flops / (gram_ms / 1e3) / 1e12, 1),
                          "gram_frac_of_bf16_peak": round(gram_flops / (gram_ms / 1e3) / 1e12 / bf16_peak, 4),
                          "projection_ms": round(proj_ms, 4),
                          "projection_tflops": round(proj_flops / (proj_ms / 1e3) / 1e12, 1),
                          "projection_frac_of_bf16_peak": round(proj_flops / (proj_ms / 1e3) / 1e12 / bf16_peak, 4),
                          "spectra": spectra,
                          "sweep": measure_compress_sweep(xkv, device, bf16_peak, log)}
    return res, w


def measure_xk_sr(xkv, w, model, device, stream, L, steps, warmup, peak_gbs):
    """The xK-SR mode on the same compressed keys, landmarks and queries: values
    read from an uncompressed [B][T][d] cache per layer (seeded normals, bf16).
    Device time of `steps` replays of one CUDA graph of L layer calls, and the
    attend launch's achieved GB/s from the library's stage events."""
    import torch
    bf = torch.bfloat16
    Vs = []
    for l in range(L):
        Vs.append(synth.normal_torch(synth.stream_key(w.name, "Vraw", l, w.T), w.batch * w.T * w.d, device,
                                     bf).view(w.batch, w.T, w.d))
        torch.cuda.empty_cache()
    p = xkv.xk_sr_params(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.T, w.rank_k, w.chunk, w.topk, w.sink,
                         w.recent, w.rope_theta, bf)
    ws = xkv.workspace(xkv.xkv_xk_sr_workspace_size(p), device)
    outs = [torch.empty((w.batch, w.n_q_heads, w.head_dim), dtype=torch.float32, device=device) for _ in range(L)]

    def call(l):
        xkv.xkv_xk_sr_attention_decode(p, model["q"][l], model["A_K"][l], model["Bt_K"][l], Vs[l], model["lm"][l],
                                       model["srK"][l], model["srV"][l], outs[l], None, ws, stream)

    with torch.cuda.stream(stream):
        for l in range(L):
            call(l)
    stream.synchronize()
    assert xkv.get_device_status(stream) == 0
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for l in range(L):
            call(l)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            graph.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(steps):
            graph.replay()
        e1.record(stream)
        e1.synchronize()
    ms_step = e0.elapsed_time(e1) / steps
    xkv.xkv_sr_profile_enable(True)
    stages = []
    with torch.cuda.stream(stream):
        for i in range(2 * L):
            call(i % L)
            stages.append(xkv.xkv_sr_profile_read())
    xkv.xkv_sr_profile_enable(False)
    assert xkv.get_device_status(stream) == 0
    st = [statistics.median(s_[j] for s_ in stages) for j in range(4)]
    bytes_attend = xk_attend_bytes_per_unit(w) * w.batch * w.n_kv_heads
    gbs = bytes_attend / (st[2] / 1e3) / 1e9
    del graph, Vs
    torch.cuda.empty_cache()
    return {"path": "xkv_xk_sr_attention_decode (keys compressed, values uncompressed in HBM)",
            "value": round(w.batch / (ms_step / 1e3), 2), "unit": "tokens/s", "ms_per_step": round(ms_step, 4),
            "stages_ms": {"score": round(st[0], 5), "topk_window": round(st[1], 5), "attend": round(st[2], 5),
                          "combine": round(st[3], 5)},
            "attend_roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak_gbs, "unit": "GB/s",
                                "frac": round(gbs / peak_gbs, 4), "bytes_per_launch": bytes_attend},
            "value_cache_gb": round(L * w.batch * w.T * w.d * 2 / 1e9, 2),
            "cache_ratio": dict(zip(("a_b", "with_landmarks"), cache_ratio(w, values_compressed=False)))}


def measure_xk_sr_host(xkv, w, model, device, stream, layers=4):
    """The xK-SR step with the uncompressed values in pinned host memory (the
    explainer's placement): per layer call only the kept chunks' value rows
    (B Hkv k chunk hd elements) cross the host link.  Device time per layer call
    (eager, median over calls) and the host-link bytes per call."""
    import torch
    bf = torch.bfloat16
    Vh = torch.empty((w.batch, w.T, w.d), dtype=bf).pin_memory()
    Vh.copy_(synth.normal_torch(synth.stream_key(w.name, "Vraw", 0, w.T), w.batch * w.T * w.d, device, bf)
             .view(w.batch, w.T, w.d).cpu())
    p = xkv.xk_sr_params(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.T, w.rank_k, w.chunk, w.topk, w.sink,
                         w.recent, w.rope_theta, bf)
    ws = xkv.workspace(xkv.xkv_xk_sr_host_workspace_size(p), device)
    out = torch.empty((w.batch, w.n_q_heads, w.head_dim), dtype=torch.float32, device=device)
    times = []
    with torch.cuda.stream(stream):
        for i in range(3 * layers):
            l = i % layers
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            xkv.xkv_xk_sr_attention_decode_host_values(p, model["q"][l], model["A_K"][l], model["Bt_K"][l], Vh,
                                                       model["lm"][l], model["srK"][l], model["srV"][l], out, None,
                                                       ws, stream)
            e1.record(stream)
            e1.synchronize()
            if i >= layers:
                times.append(e0.elapsed_time(e1))
    assert xkv.get_device_status(stream) == 0
    ms = statistics.median(times)
    link = w.batch * w.n_kv_heads * w.topk * w.chunk * w.head_dim * 2
    return {"path": "xkv_xk_sr_attention_decode_host_values (values in pinned host memory)",
            "ms_per_layer_call": round(ms, 4), "host_link_bytes_per_call": link,
            "host_link_gbs": round(link / (ms / 1e3) / 1e9, 2),
            "note": "eager calls; the value rows cross the host link, the rest is the HBM-resident xK-SR step"}


def measure_append(xkv, w, device, stream):
    """xkv_sr_append for one group of the workload (batch, G layers): the device
    time of an append that only writes the window, and of one that rolls a
    chunk into the compressed cache (landmarks, projection of x onto the
    stored bases, window move)."""
    import torch
    bf = torch.bfloat16
    B, G, d, C = w.batch, w.group, w.d, w.chunk
    n = G * d
    T0 = w.sink + w.recent + C * 64
    cap = 80
    Tcap = w.sink + cap * C + w.recent + C
    A_K = torch.zeros((B, Tcap, w.rank_k), dtype=bf, device=device)
    A_V = torch.zeros((B, Tcap, w.rank_v), dtype=bf, device=device)
    Bt_K = torch.randn((B, n, w.rank_k), device=device).to(bf)
    Bt_V = torch.randn((B, n, w.rank_v), device=device).to(bf)
    lms = [torch.zeros((B, w.n_kv_heads, cap, w.head_dim), dtype=bf, device=device) for _ in range(G)]
    wk = [torch.randn((B, w.sink + w.recent + C, d), device=device).to(bf) for _ in range(G)]
    wv = [torch.randn((B, w.sink + w.recent + C, d), device=device).to(bf) for _ in range(G)]
    kn = [torch.randn((B, d), device=device).to(bf) for _ in range(G)]
    vn = [torch.randn((B, d), device=device).to(bf) for _ in range(G)]
    wbs = (w.sink + w.recent + C) * d
    times = {False: [], True: []}
    T = T0
    with torch.cuda.stream(stream):
        for _ in range(4 * C):
            ap = xkv.append_params(B, G, w.n_kv_heads, w.head_dim, C, w.sink, w.recent, w.rope_theta, bf, T,
                                   w.rank_k, w.rank_v, Tcap * w.rank_k, Tcap * w.rank_v, n * w.rank_k, n * w.rank_v,
                                   wbs, cap)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            rolled = xkv.xkv_sr_append(ap, kn, vn, wk, wv, Bt_K, Bt_V, A_K, A_V, lms, stream=stream)
            e1.record(stream)
            e1.synchronize()
            times[rolled].append(e0.elapsed_time(e1))
            T += 1
    assert xkv.get_device_status(stream) == 0
    return {"path": "xkv_sr_append (one token per layer of a group; a chunk rolled every chunk steps)",
            "append_ms": round(statistics.median(times[False]), 4),
            "append_with_roll_ms": round(statistics.median(times[True]), 4),
            "group": f"batch {B}, G = {G}, d = {d}, ranks {w.rank_k} / {w.rank_v}"}


def measure_full_reconstruction(xkv, w, model, device, stream, sr_call_ms):
    """The comparison path of one layer for the whole batch: every K row
    rebuilt (A_K Bt_K^T + RoPE) and every V row rebuilt (A_V Bt_V^T), then
    dense decode attention over the T rebuilt rows; device time per layer,
    median over eager runs with L2 flushed in between, beside the SR call."""
    import torch
    bf = torch.bfloat16
    B, T, d = w.batch, w.T, w.d
    K = torch.empty((B, T, d), dtype=bf, device=device)
    V = torch.empty((B, T, d), dtype=bf, device=device)
    out = torch.empty((B, w.n_q_heads, w.head_dim), dtype=torch.float32, device=device)
    dp = xkv.dense_params(B, w.n_q_heads, w.n_kv_heads, w.head_dim, T, bf)
    dws = xkv.workspace(xkv.xkv_dense_workspace_size(dp), device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    times = []
    with torch.cuda.stream(stream):
        for it in range(6):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for b in range(B):
                xkv.xkv_full_reconstruct(model["A_K"][0][b], model["Bt_K"][0][b], w.n_kv_heads, w.head_dim, True,
                                         w.rope_theta, K[b], stream)
                xkv.xkv_full_reconstruct(model["A_V"][0][b], model["Bt_V"][0][b], w.n_kv_heads, w.head_dim, False,
                                         w.rope_theta, V[b], stream)
            xkv.xkv_dense_attention_decode(dp, model["q"][0], K, V, out, dws, stream)
            e1.record(stream)
            e1.synchronize()
            if it > 0:
                times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    del K, V, flush
    el = 2
    # algorithmic bytes: A and Bt read, rebuilt K and V written, then read by the dense pass
    byts = B * (T * (w.rank_k + w.rank_v) * el + d * (w.rank_k + w.rank_v) * el + 2 * 2 * T * d * el)
    return {"path": "xkv_full_reconstruct (K with RoPE, V) for every row + xkv_dense_attention_decode",
            "ms_per_layer": round(ms, 4), "sr_ms_per_layer": round(sr_call_ms, 4),
            "sr_speedup": round(ms / sr_call_ms, 2), "bytes_per_layer": int(byts),
            "achieved_gbs": round(byts / (ms / 1e3) / 1e9, 1),
            "note": "comparison kernels untuned: the ratio overstates SR's advantage"}


def cpu_baseline(w, budget_s: float, log):
    """The oracle (fp64 C, OpenMP) on a bounded sample of the same decode step."""
    import oracle
    wb = w.replace(batch=1)
    inp = synth.compressed_cache(wb, 0)
    units_per_layer = wb.n_kv_heads
    t0 = time.time()
    done = 0
    while time.time() - t0 < budget_s and done < 64:
        oracle.sr_decode(wb, units=list(range(units_per_layer)), **inp)
        done += units_per_layer
    dt = time.time() - t0
    units_step = w.batch * w.n_layers * w.n_kv_heads
    step_s = dt / done * units_step
    return {"value": round(w.batch / step_s, 4), "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle", "wall_s": round(dt, 3),
            "sample": f"{done} (layer, KV-head) units of one decode step (batch 1, T={w.T}), oracle SR decode in "
                      f"fp64, scaled to the full {w.n_layers}-layer batch-{w.batch} step ({units_step} units)"}


def run_reference(args, log):
    w = synth.WORKLOADS[args.workload]
    if args.batch:
        w = w.replace(batch=args.batch)
    import oracle
    oracle.build()
    budget = max(2.0, min(20.0, 60.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_baseline(w, budget / 4, log)
    vals = [cpu_baseline(w, budget, log) for _ in range(args.steps)]
    v = statistics.median(x["value"] for x in vals)
    cb = dict(vals[0])
    cb["value"] = v
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(w.batch / v * 1e3, 3),
            "sampled": True, "sample_wall_s_per_step": round(statistics.median(x["wall_s"] for x in vals), 3),
            "note": "each step runs the oracle on a bounded sample of (layer, KV head) units and scales its time "
                    "to the whole step; ms_per_step is that scaled time, not the wall time of the sample",
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "global_batch": w.batch, "seq_len": w.T, "layers": w.n_layers},
            "cpu_baseline": cb, "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                                        "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--workload", default="llama8b_64k_b4", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--batch", type=int, default=0, help="override the batch per GPU")
    ap.add_argument("--groups", type=int, default=0, help="build only this many layer groups")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", dest="prefill", action="store_false")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-xk", dest="xk", action="store_false",
                    help="skip the xK-SR measurement (values uncompressed; one GPU only)")
    ap.add_argument("--also", default="qwen7b_128k_b2",
                    help="comma-separated further workloads measured on one GPU (empty string: none)")
    ap.add_argument("--no-comparison", dest="comparison", action="store_false",
                    help="skip timing the full-reconstruction comparison path")
    ap.add_argument("--prefill-only", action="store_true",
                    help="time only the compression kernels (Gram, projection, the compression sweep) and print "
                         "them; no decode step (a profiling aid)")
    ap.add_argument("--compress-profile", action="store_true",
                    help="one xkv_compress_group + xkv_ner on the workload's (batch 0, group 0) keys, run once "
                         "untimed and once between cudaProfilerStart / Stop (for ncu --profile-from-start off); "
                         "prints the second run's device time")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    log = (lambda *a: print(*a, file=sys.stderr, flush=True)) if rank == 0 else (lambda *a: None)

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, log)), flush=True)
        return
    if args.compress_profile:
        print(json.dumps(compress_profile(synth.WORKLOADS[args.workload])), flush=True)
        return
    if args.prefill_only:
        import torch
        import cross_layer_rank_b200 as xkv
        device = torch.device("cuda", 0)
        w = synth.WORKLOADS[args.workload]
        _, bf16_peak, _, _ = _peaks()
        gram_ms, gram_flops, _, proj_ms, proj_flops = measure_gram(xkv, w, device, spectra=False)
        res = {"workload": w.name, "gram_ms": round(gram_ms, 4),
               "gram_frac_of_bf16_peak": round(gram_flops / (gram_ms / 1e3) / 1e12 / bf16_peak, 4),
               "projection_ms": round(proj_ms, 4),
               "projection_frac_of_bf16_peak": round(proj_flops / (proj_ms / 1e3) / 1e12 / bf16_peak, 4),
               "sweep": measure_compress_sweep(xkv, device, bf16_peak, log)}
        print(json.dumps(res), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    res, w = run_cuda(args, rank, world, log)
    if world == 1 and args.also:
        # the other shapes the decode path is reported on (same step, same
        # timing; no prefill, comparison or CPU legs)
        import copy
        import torch
        for name in [x for x in args.also.split(",") if x and x != args.workload]:
            torch.cuda.empty_cache()
            a2 = copy.copy(args)
            a2.workload, a2.prefill, a2.comparison, a2.xk, a2.batch, a2.groups = name, False, False, False, 0, 0
            try:
                r2, _ = run_cuda(a2, rank, world, log)
            except Exception as e:  # noqa: BLE001
                log(f"{name} not measured: {e!r}")
                continue
            res.setdefault("other_workloads", {})[name] = {
                k: r2[k] for k in ("value", "unit", "ms_per_step", "steps", "roofline", "stage_rooflines", "e2e",
                                   "config", "clocks", "cache_ratio")}
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        res["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds, log)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
