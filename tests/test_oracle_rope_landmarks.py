"""Oracle pins: rotary embedding and chunk landmarks.

RoPE (rotate-half, inv_freq_j = theta^(-2j/hd)) is pinned by rotations whose
angles are known, by norm preservation and by the relative-position identity
R_m(q) . R_n(k) = q . R_(n-m)(k).  A landmark (mean of a chunk's post-RoPE keys;
the xKV explainer's "landmark-guided" selector) is pinned by the closed form of
a chunk whose pre-RoPE key is constant: sum_{t=t0}^{t0+C-1} e^{i t f} =
e^{i (t0 + (C-1)/2) f} sin(C f / 2) / sin(f / 2).
"""
import numpy as np
import pytest

import oracle


def test_rope_hd2_is_rotation_by_position_radians():
    for t in (0.0, 1.0, 2.5, 1000.0):
        y = oracle.rope([1.0, 0.0], t, 500000.0)
        assert np.allclose(y, [np.cos(t), np.sin(t)], atol=1e-12)


def test_rope_pairs_j_with_j_plus_half():
    # hd = 4, theta = 1e4: pair (1, 3) turns at 1e4^(-1/2) = 0.01 rad per position
    y = oracle.rope([0.0, 1.0, 0.0, 0.0], 300.0, 1e4)
    assert np.allclose(y, [0.0, np.cos(3.0), 0.0, np.sin(3.0)], atol=1e-12)
    assert np.array_equal(oracle.rope([1, 2, 3, 4], 0.0, 1e4), [1, 2, 3, 4])


def test_rope_norm_and_relative_position():
    rng = np.random.default_rng(0)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    for m, n in ((5, 17), (1000, 65000), (131071, 3)):
        qm, kn = oracle.rope(q, m, 5e5), oracle.rope(k, n, 5e5)
        assert abs(np.linalg.norm(qm) - np.linalg.norm(q)) < 1e-12 * np.linalg.norm(q)
        assert abs(qm @ kn - q @ oracle.rope(k, n - m, 5e5)) < 1e-9


@pytest.mark.parametrize("hd,chunk,theta", [(8, 8, 500000.0), (64, 4, 1e4), (128, 8, 500000.0)])
def test_landmark_closed_form_for_constant_chunk(hd, chunk, theta):
    rng = np.random.default_rng(hd)
    H, sink, recent, n_mid = 2, 3, 5, 6
    T = sink + recent + n_mid * chunk
    K = np.zeros((T, H * hd), dtype=np.float32)
    keys = rng.standard_normal((H, n_mid, hd)).astype(np.float32)
    for c in range(n_mid):
        t0 = sink + c * chunk
        for h in range(H):
            K[t0:t0 + chunk, h * hd:(h + 1) * hd] = keys[h, c]
    L = oracle.landmarks(K, H, hd, chunk, sink, recent, theta)
    assert L.shape == (H, n_mid, hd)
    half = hd // 2
    f = theta ** (-2.0 * np.arange(half) / hd)
    for h in range(H):
        for c in range(n_mid):
            t0 = sink + c * chunk
            amp = np.sin(chunk * f / 2) / np.sin(f / 2) / chunk
            ph = (t0 + (chunk - 1) / 2.0) * f
            mc, ms = amp * np.cos(ph), amp * np.sin(ph)
            k = keys[h, c].astype(np.float64)
            exp = np.concatenate([k[:half] * mc - k[half:] * ms, k[half:] * mc + k[:half] * ms])
            assert np.abs(L[h, c] - exp).max() < 1e-9


def test_landmarks_ignore_sink_and_recent_rows():
    rng = np.random.default_rng(3)
    T, d = 8 + 32 + 4 * 8, 16
    K = rng.standard_normal((T, d)).astype(np.float32)
    L1 = oracle.landmarks(K, 2, 8, 8, 8, 32, 5e5)
    K2 = K.copy()
    K2[:8] = 100.0
    K2[-32:] = -100.0
    assert np.array_equal(L1, oracle.landmarks(K2, 2, 8, 8, 8, 32, 5e5))
