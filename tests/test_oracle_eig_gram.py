"""Oracle pins: cyclic Jacobi and the streamed Gram.

The Jacobi eigensolver is pinned against LAPACK (numpy.linalg.eigh) and against
matrices whose spectrum is fixed by construction; the Gram accumulation of
KV-CoRE 2.A ("C = sum_t k_t^T k_t" over streamed tokens) is pinned against
numpy's matrix product and against the one-shot sum (sharding changes nothing).
"""
import numpy as np
import pytest

import oracle


@pytest.mark.parametrize("n", [1, 2, 7, 64, 129])
def test_jacobi_matches_lapack(n):
    rng = np.random.default_rng(n)
    X = rng.standard_normal((n, n))
    A = X + X.T
    w, V, sweeps = oracle.jacobi_eigh(A)
    assert sweeps >= 0
    ref = np.linalg.eigh(A)[0][::-1]
    assert np.allclose(w, ref, rtol=0, atol=1e-12 * max(1.0, np.abs(ref).max()))
    assert np.abs(V.T @ V - np.eye(n)).max() < 1e-12
    assert np.abs(A @ V - V * w).max() < 1e-11 * max(1.0, np.abs(ref).max())


def test_jacobi_known_spectrum_and_vectors():
    rng = np.random.default_rng(1)
    n = 40
    Q, _ = np.linalg.qr(rng.standard_normal((n, n)))
    lam = np.linspace(10.0, 1.0, n) ** 2  # distinct
    A = (Q * lam) @ Q.T
    w, V, _ = oracle.jacobi_eigh(A)
    assert np.allclose(w, lam, rtol=1e-12)
    # eigenvectors equal Q's columns up to sign
    s = np.sign(np.sum(V * Q, axis=0))
    assert np.abs(V - Q * s).max() < 1e-10


def test_jacobi_degenerate_cases():
    w, V, _ = oracle.jacobi_eigh(np.zeros((5, 5)))
    assert np.all(w == 0) and np.array_equal(V, np.eye(5))
    D = np.diag([3.0, -1.0, 7.0, 7.0])
    w, V, sweeps = oracle.jacobi_eigh(D)
    assert sweeps == 0 and list(w) == [7.0, 7.0, 3.0, -1.0]


def test_gram_matches_matmul_and_streaming():
    rng = np.random.default_rng(2)
    T, d, G = 301, 24, 3
    layers = [rng.standard_normal((T, d)).astype(np.float32) for _ in range(G)]
    X = np.concatenate([l.astype(np.float64) for l in layers], axis=1)
    Cm = oracle.gram(layers)
    assert np.abs(Cm - X.T @ X).max() < 1e-10 * np.abs(X.T @ X).max()
    # streamed over ragged shards, the covariance is the same sum
    Cs = None
    for t0, t1 in ((0, 128), (128, 256), (256, 301)):
        Cs = oracle.gram(layers, t0, t1, C_in=Cs)
    assert np.abs(Cs - Cm).max() < 1e-10 * np.abs(Cm).max()
    assert np.array_equal(Cm, Cm.T)
    # layer order: the (0,1) block is K_1^T K_2, not K_2^T K_1
    blk = Cm[:d, d:2 * d]
    assert np.abs(blk - layers[0].astype(np.float64).T @ layers[1]).max() < 1e-10 * np.abs(blk).max()
