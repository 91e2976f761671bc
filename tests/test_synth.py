"""Seeded input generator: Philox4x32-10 known answers, Box-Muller moments,
stream independence and the device twin's integer stream."""
import os

import numpy as np
import pytest

import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")


def _kat():
    rows = []
    for line in open(GOLD):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        v = [int(x, 16) for x in line.split()]
        rows.append((v[0:4], v[4:6], v[6:10]))
    return rows


@pytest.mark.parametrize("ctr,key,out", _kat())
def test_philox_known_answers(ctr, key, out):
    got = synth.philox4x32_10(np.array([ctr], dtype=np.uint64), key)[0]
    assert [int(x) for x in got] == out


def test_normal_moments_and_determinism():
    k = synth.stream_key("moments")
    z = synth.normal(k, 400_000)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1.0) < 0.01
    # fourth moment of a standard normal is 3
    assert abs((z ** 4).mean() - 3.0) < 0.1
    assert np.array_equal(z, synth.normal(k, 400_000))
    assert not np.array_equal(z[:1000], synth.normal(synth.stream_key("other"), 1000))


def test_chunked_equals_whole():
    k = synth.stream_key("chunk")
    a = synth.normal(k, 100_003).astype(np.float32)
    b = synth.normal_chunked(k, 100_003, chunk=4096)
    assert np.array_equal(a, b)


def test_torch_twin_same_stream():
    torch = pytest.importorskip("torch")
    k = synth.stream_key("twin")
    a = synth.normal(k, 10_001)
    b = synth.normal_torch(k, 10_001, "cpu", torch.float64).numpy()
    assert np.abs(a - b).max() < 1e-12


def test_bf16_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1e-40], dtype=np.float32)
    y = synth.to_storage(x, "bf16")
    # 1 + 2^-8 is the midpoint between 1 and 1 + 2^-7: ties go to the even one (1.0)
    assert y[0] == 1.0 and y[1] == 1.0 and y[2] == np.float32(1.0 + 2 ** -6)
    assert y[3] == -2.5


def test_workload_shapes():
    w = synth.WORKLOADS["llama8b_64k_b4"]
    assert w.d == 1024 and w.gq == 4 and w.n_groups == 8 and w.n_mid == 8187
    w3 = synth.WORKLOADS["qwen7b_128k_b2"]
    assert w3.d == 512 and w3.gq == 7 and w3.n_mid == 16379
    assert synth.WORKLOADS["tiny_f32"].n_mid == 123
    assert synth.compression_sweep(8).rank_k == 1024


def test_kv_group_structure():
    w = synth.WORKLOADS["tiny_f32"]
    Ks = synth.kv_group(w, 0, 0, "K", T=256)
    assert len(Ks) == 4 and Ks[0].shape == (256, 128)
    # layers of a group share W_s: their column spaces are close; layers differ
    assert not np.allclose(Ks[0], Ks[1])
    Vs = synth.kv_group(w, 0, 0, "V", T=256)
    assert not np.allclose(Ks[0], Vs[0])


def test_group_spectrum_has_no_gap_at_the_rank_and_a_gap_at_the_latent_dimension():
    # the recipe's spectra: eigenvalues of the group Gram decay like i^(-2 alpha)
    # with no gap at the compression rank (so a subspace projector is not
    # unique there) and a sharp drop after the latent dimension m, where only
    # the 0.01 N noise remains
    w = synth.WORKLOADS["tiny_f32"]
    X = np.concatenate([k.astype(np.float64) for k in synth.kv_group(w, 0, 0, "K")], axis=1)
    lam = np.linalg.eigvalsh(X.T @ X)[::-1]
    r, m = w.rank_k, w.latent
    assert lam[r - 1] / lam[r] < 1.1
    assert lam[m - 1] / lam[m] > 20.0
    assert np.all(lam[m:] < 1e-3 * lam[0])
