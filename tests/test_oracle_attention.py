"""Oracle pins: decode attention (KQ-SVD page, 3.2: h_T = softmax(q K^T / sqrt(d)) V),
by cases with closed forms: one token, equal keys (uniform weights), two tokens
(logistic weight with the 1/sqrt(hd) scale), GQA head mapping, a dominant key."""
import numpy as np

import oracle


def test_single_token_returns_its_value():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((1, 2, 8)).astype(np.float32)
    K = rng.standard_normal((1, 1, 8)).astype(np.float32)
    V = rng.standard_normal((1, 1, 8)).astype(np.float32)
    out = oracle.dense_decode(q, K, V, 1)
    assert np.abs(out - V[0, 0]).max() < 1e-15


def test_equal_keys_average_values():
    rng = np.random.default_rng(1)
    T, hd = 37, 16
    q = rng.standard_normal((1, 1, hd)).astype(np.float32)
    K = np.tile(rng.standard_normal((1, 1, hd)), (1, T, 1)).astype(np.float32)
    V = rng.standard_normal((1, T, hd)).astype(np.float32)
    out = oracle.dense_decode(q, K, V, 1)
    assert np.abs(out[0, 0] - V[0].astype(np.float64).mean(0)).max() < 1e-14


def test_two_tokens_logistic_weight_with_scale():
    hd = 64
    q = np.zeros((1, 1, hd), dtype=np.float32); q[0, 0, 0] = 2.0
    K = np.zeros((1, 2, hd), dtype=np.float32); K[0, 0, 0] = 3.0; K[0, 1, 0] = -1.0
    V = np.zeros((1, 2, hd), dtype=np.float32); V[0, 0, 5] = 1.0; V[0, 1, 6] = 1.0
    out = oracle.dense_decode(q, K, V, 1)
    # logits 6/8 and -2/8: weight of token 0 = 1 / (1 + e^(-1))
    p0 = 1.0 / (1.0 + np.exp(-1.0))
    assert abs(out[0, 0, 5] - p0) < 1e-15 and abs(out[0, 0, 6] - (1 - p0)) < 1e-15


def test_gqa_query_head_reads_kv_head_j_div_gq():
    B, Hkv, gq, hd, T = 2, 3, 4, 8, 5
    q = np.random.default_rng(2).standard_normal((B, Hkv * gq, hd)).astype(np.float32)
    K = np.zeros((B, T, Hkv * hd), dtype=np.float32)
    V = np.zeros((B, T, Hkv * hd), dtype=np.float32)
    for b in range(B):
        for h in range(Hkv):
            V[b, :, h * hd:(h + 1) * hd] = 10 * b + h + 1
    out = oracle.dense_decode(q, K, V, Hkv)
    for b in range(B):
        for j in range(Hkv * gq):
            assert np.allclose(out[b, j], 10 * b + j // gq + 1, atol=1e-13)


def test_dominant_key_selects_its_value():
    rng = np.random.default_rng(4)
    T, hd = 50, 32
    q = rng.standard_normal((1, 1, hd)).astype(np.float32)
    K = (0.01 * rng.standard_normal((1, T, hd))).astype(np.float32)
    K[0, 17] = 40 * q[0, 0]
    V = rng.standard_normal((1, T, hd)).astype(np.float32)
    out = oracle.dense_decode(q, K, V, 1)
    assert np.abs(out[0, 0] - V[0, 17]).max() < 1e-6
