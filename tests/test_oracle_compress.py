"""Oracle pins: the cross-layer factorisation.

Pinned against LAPACK's SVD of the concatenation X (its singular values squared
are the Gram's eigenvalues; its truncation is the Frobenius-optimal rank-r
approximation, Eckart-Young-Mirsky, as the KQ-SVD page's section 3.3 states),
against exactness at full rank, and against per-layer SVD for G = 1 (the
"Single SVD" case of the xKV explainer's Table 2).
"""
import numpy as np
import pytest

import oracle
import synth


def _group(T=192, d=32, G=3, m=20, seed=0):
    rng = np.random.default_rng(seed)
    Z = rng.standard_normal((T, m)) * (np.arange(1, m + 1) ** -0.8)
    Ws = rng.standard_normal((m, d))
    return [(Z @ (Ws + 0.1 * rng.standard_normal((m, d))) + 0.01 * rng.standard_normal((T, d)))
            .astype(np.float32) for _ in range(G)]


def _concat(layers):
    return np.concatenate([l.astype(np.float64) for l in layers], axis=1)


@pytest.mark.parametrize("r", [1, 8, 20])
def test_eckart_young_against_lapack_svd(r):
    layers = _group()
    X = _concat(layers)
    res = oracle.compress_group(layers, r)
    U, s, Vt = np.linalg.svd(X, full_matrices=False)
    # eigenvalues of X^T X are the squared singular values
    assert np.allclose(res["lam"][: s.size], s ** 2, rtol=1e-10, atol=1e-10 * s[0] ** 2)
    # squared subspace error = discarded energy = LAPACK's truncation error
    opt = np.sum(s[r:] ** 2)
    assert abs(res["err_subspace"] ** 2 - opt) <= 1e-9 * res["xx"]
    assert abs(res["tail"] - opt) <= 1e-9 * res["xx"]
    # the rebuilt matrix equals the truncated SVD (unique: there is a gap at r)
    ref = (U[:, :r] * s[:r]) @ Vt[:r]
    got = res["A"] @ res["Bt"].T
    assert np.abs(got - ref).max() < 1e-8 * np.abs(X).max()
    # A = X V_r and V_r has orthonormal columns
    assert np.abs(res["A"] - X @ res["Bt"]).max() < 1e-9 * np.abs(res["A"]).max()
    assert np.abs(res["Bt"].T @ res["Bt"] - np.eye(r)).max() < 1e-12


def test_full_rank_is_exact():
    layers = _group(T=80, d=8, G=2)
    X = _concat(layers)
    res = oracle.compress_group(layers, 16)
    assert res["err_subspace"] <= 1e-10 * np.linalg.norm(X)


def test_single_layer_group_is_per_layer_svd():
    layers = _group(G=1)
    X = layers[0].astype(np.float64)
    r = 6
    res = oracle.compress_group(layers, r)
    U, s, Vt = np.linalg.svd(X, full_matrices=False)
    assert np.abs(res["A"] @ res["Bt"].T - (U[:, :r] * s[:r]) @ Vt[:r]).max() < 1e-8 * np.abs(X).max()


def test_stored_error_is_bf16_of_own_factors():
    layers = _group()
    X = _concat(layers)
    r = 8
    res = oracle.compress_group(layers, r)
    Ab = synth.to_storage(res["A"].astype(np.float32), "bf16").astype(np.float64)
    Bb = synth.to_storage(res["Bt"].astype(np.float32), "bf16").astype(np.float64)
    # synth rounds via float32 exactly as the oracle does (fp64 -> fp32 -> bf16)
    e = np.linalg.norm(X - Ab @ Bb.T)
    assert abs(e - res["err_stored"]) < 1e-9 * e
    assert res["err_stored"] >= res["err_subspace"] * (1 - 1e-12)


def test_shared_basis_beats_per_layer_at_equal_storage_on_aligned_layers():
    # the xKV explainer's central observation: when the layers' dominant
    # subspaces align, one shared basis of rank r for G layers keeps more energy
    # than G separate rank-(r/G) bases (equal A storage).
    layers = _group(T=256, d=32, G=4, m=12)
    X = _concat(layers)
    shared = oracle.compress_group(layers, 12)
    per = sum(oracle.compress_group([l], 3)["err_subspace"] ** 2 for l in layers)
    assert shared["err_subspace"] ** 2 < per
    assert shared["err_subspace"] ** 2 < 1e-2 * np.sum(X ** 2)


def test_full_reconstruct_at_full_rank_returns_each_layer():
    # full_reconstruct (the comparison path's rebuild) of layer l from the
    # group's factors: at full rank A Bt_l^T is X_l itself, and with RoPE every
    # head's row is X_l's row turned by its position (the rotation pinned in
    # the RoPE tests)
    n_kv, hd = 2, 8
    layers = _group(T=40, d=n_kv * hd, G=2)
    d = n_kv * hd
    res = oracle.compress_group(layers, 2 * d)
    A = res["A"].astype(np.float32)
    for l, X in enumerate(layers):
        Bt = res["Bt"][l * d:(l + 1) * d].astype(np.float32)
        plain = oracle.full_reconstruct(A, Bt, n_kv, hd, False, 500000.0)
        assert np.abs(plain - X).max() <= 1e-5 * np.abs(X).max()
        rot = oracle.full_reconstruct(A, Bt, n_kv, hd, True, 500000.0)
        for t in (0, 1, 17, 39):
            for h in range(n_kv):
                sl = slice(h * hd, (h + 1) * hd)
                ref = oracle.rope(X[t, sl], t, 500000.0)
                assert np.abs(rot[t, sl] - ref).max() <= 1e-5 * np.abs(X).max()
