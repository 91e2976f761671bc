"""The bench's algorithmic counts against figures worked out by hand from the
per-unit byte formula, for the three decode shapes (Llama-3.1-8B group at 16K,
the 32-layer Llama-3.1-8B at 64K batch 4, the 28-layer Qwen2.5-7B at 128K
batch 2): bytes per decode step
(landmarks + selected A rows + Bt slices + raw window + queries/outputs) and
the cache compression ratios (A+B alone, and with the landmarks)."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
import synth  # noqa: E402


@pytest.mark.parametrize("name, layers, gb", [("llama_group_16k", 4, 0.160), ("llama8b_64k_b4", 32, 6.73),
                                              ("qwen7b_128k_b2", 28, 2.16)])
def test_bytes_per_step(name, layers, gb):
    w = synth.WORKLOADS[name]
    step = bench.sr_bytes_per_unit(w) * w.batch * w.n_kv_heads * layers
    assert abs(step / 1e9 - gb) < 0.005 * gb


@pytest.mark.parametrize("name, ab, lm", [("llama_group_16k", 6.40, 4.57), ("llama8b_64k_b4", 7.53, 5.12),
                                          ("qwen7b_128k_b2", 6.30, 4.52)])
def test_cache_ratio(name, ab, lm):
    r_ab, r_lm = bench.cache_ratio(synth.WORKLOADS[name])
    assert abs(r_ab - ab) < 0.01 and abs(r_lm - lm) < 0.01


def test_cache_ratio_with_uncompressed_values():
    # xK-SR: K at rank 512 plus whole V: (2 T d) / (T d + (T + G d) r_K / G)
    w = synth.WORKLOADS["llama8b_64k_b4"]
    r_ab, _ = bench.cache_ratio(w, values_compressed=False)
    T, d, G, r = w.T, w.d, w.group, w.rank_k
    assert abs(r_ab - 2 * T * d / (T * d + (T + G * d) * r / G)) < 1e-3
    assert 1.0 < r_ab < 2.0


def test_code_digest_ignores_comments_only():
    a = 'int f(int x) {  // add one\n  /* block\n comment */ return x + 1;\n}\nconst char* s = "a // b";\n'
    b = 'int f(int x) {  // plus one\n\n  return x + 1;   \n}\nconst char* s = "a // b";\n'
    c = 'int f(int x) {\n  return x + 2;\n}\nconst char* s = "a // b";\n'
    d = 'int f(int x) {\n  return x + 1;\n}\nconst char* s = "a // c";\n'
    assert bench.code_digest(a) == bench.code_digest(b)
    assert bench.code_digest(a) != bench.code_digest(c)
    assert bench.code_digest(a) != bench.code_digest(d)


def test_attend_bytes_per_unit_llama():
    # per (sequence, layer, KV head) at the Llama shape: the selected A rows are
    # k C (r_K + r_V) 2 = 4 MiB, the head's Bt_K slice r_K hd 2 = 128 KiB, the
    # group's queries Gq hd 2 = 1 KiB; xK-SR swaps r_V for hd
    w = synth.WORKLOADS["llama8b_64k_b4"]
    assert bench.attend_bytes_per_unit(w) == 4 * 2**20 + 128 * 2**10 + 2**10
    assert bench.xk_attend_bytes_per_unit(w) == 256 * 8 * (512 + 128) * 2 + 128 * 2**10 + 2**10
    # launch totals used by the roofline lines: 32 units
    assert bench.attend_bytes_per_unit(w) * w.batch * w.n_kv_heads == 138444800
    assert bench.xk_attend_bytes_per_unit(w) * w.batch * w.n_kv_heads == 88113152
