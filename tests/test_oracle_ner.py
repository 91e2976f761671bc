"""Oracle pins: KV-CoRE's normalised effective rank (section 2.B).

Hand-worked examples (tests/golden/ner_examples.txt), the range [1/r, 1], the
limits (flat spectrum -> 1; one dominant singular value -> 1/r), exact numerical
rank detection and the per-layer (diagonal block) reading."""
import os

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden", "ner_examples.txt")


def _gold():
    out = []
    for line in open(GOLD):
        if line.startswith("#") or not line.strip():
            continue
        sig, r, er, ner = (p.strip() for p in line.split("|"))
        out.append(([float(x) for x in sig.split()], int(r), float(er), float(ner)))
    return out


@pytest.mark.parametrize("sig,r,er,nr", _gold())
def test_worked_examples(sig, r, er, nr):
    X = np.diag(sig)  # singular values sig -> Gram eigenvalues sig^2
    ner, erank, rank, _ = oracle.ner(X.T @ X, len(sig))
    assert rank[0] == r and abs(erank[0] - er) < 1e-12 and abs(ner[0] - nr) < 1e-12


def test_flat_and_dominant_limits():
    n = 64
    ner, _, rank, _ = oracle.ner(3.7 * np.eye(n), n)
    assert rank[0] == n and abs(ner[0] - 1.0) < 1e-12
    lam = np.full(n, 1e-8); lam[0] = 1.0  # sigma: 1 and 1e-4 (x63)
    ner, _, rank, _ = oracle.ner(np.diag(lam), n)
    assert rank[0] == n and 1.0 / n <= ner[0] < 1.1 / n


def test_rank_detection_and_range():
    rng = np.random.default_rng(0)
    X = rng.standard_normal((200, 5)) @ rng.standard_normal((5, 32))
    ner, erank, rank, ev = oracle.ner(X.T @ X, 32)
    assert rank[0] == 5 and 1.0 / 5 <= ner[0] <= 1.0
    Y = rng.standard_normal((300, 48)) * (np.arange(1, 49) ** -0.8)
    ner, _, rank, _ = oracle.ner(Y.T @ Y, 48)
    assert rank[0] == 48 and 1.0 / 48 <= ner[0] <= 1.0


def test_per_block_reading_and_zero_block():
    rng = np.random.default_rng(1)
    A = rng.standard_normal((100, 8))
    Cm = np.zeros((16, 16))
    Cm[:8, :8] = A.T @ A
    Cm[:8, 8:] = 5.0  # off-diagonal blocks are ignored
    Cm[8:, :8] = 5.0
    ner, erank, rank, _ = oracle.ner(Cm, 8)
    ref, _, _, _ = oracle.ner(A.T @ A, 8)
    assert abs(ner[0] - ref[0]) < 1e-14
    assert ner[1] == 0.0 and rank[1] == 0 and erank[1] == 0.0


# --------------------------------------------------------- energy rank
def _diag_gram(blocks):
    n = sum(len(b) for b in blocks)
    C = np.zeros((n, n))
    o = 0
    for b in blocks:
        C[o:o + len(b), o:o + len(b)] = np.diag(b)
        o += len(b)
    return C


def test_energy_rank_closed_forms():
    # flat: 16 equal eigenvalues need ceil(0.95 * 16) = 16; geometric 2^-i,
    # i = 0..15: 2 - 2^(1-k) >= 0.95 (2 - 2^-15) first holds at k = 5; one
    # dominant value: 1; a zero block: 0
    flat = np.ones(64)
    geo = 0.5 ** np.arange(16)
    dom = np.concatenate([[1.0], np.full(15, 1e-9)])
    zero = np.zeros(16)
    C = _diag_gram([flat[:16], geo, dom, zero])
    ranks, lam = oracle.energy_rank(C, 16, 0.95)
    assert list(ranks) == [16, 5, 1, 0]
    assert np.all(np.diff(lam, axis=1) <= 0)


def test_energy_rank_rotation_invariant_and_matches_lapack():
    # a rotated spectrum gives the same rank; eigenvalues agree with LAPACK
    rng = np.random.default_rng(3)
    d = 32
    Q, _ = np.linalg.qr(rng.standard_normal((d, d)))
    lam = np.sort(rng.uniform(0, 1, d) ** 4)[::-1]
    M = Q @ np.diag(lam) @ Q.T
    for e in (0.5, 0.9, 0.99):
        r_rot, l_rot = oracle.energy_rank(M, d, e)
        r_diag, _ = oracle.energy_rank(np.diag(lam), d, e)
        assert r_rot[0] == r_diag[0] == int(np.searchsorted(np.cumsum(lam), e * lam.sum())) + 1
        assert np.allclose(l_rot[0], np.sort(np.linalg.eigvalsh(M))[::-1], atol=1e-12)

