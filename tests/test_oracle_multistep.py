"""Oracle pins for multi-step decode: the projection of new rows onto a stored
group basis, the landmark of one chunk at absolute positions, and the roll of a
full chunk out of the raw window (oracle.SRState.append).

The xKV explainer's editor's note says the factorisation covers the long
prefill only; here generated tokens stay raw in the recent window, and once a
chunk's worth (recent + chunk rows) has accumulated, its oldest chunk joins
the compressed cache (A rows = x V, one landmark per layer and KV head).
"""
import numpy as np

import oracle
import synth


def test_project_rows_hand_worked():
    # x = [1 2 | 3 4] over two layers of d = 2; V is 4 x 2:
    # A = [1 + 3 + 8, 2 + 3 - 4] = [12, 1]
    layers = [np.array([[1.0, 2.0]], np.float32), np.array([[3.0, 4.0]], np.float32)]
    V = np.array([[1, 0], [0, 1], [1, 1], [2, -1]], np.float32)
    assert np.array_equal(oracle.project_rows(layers, V), np.array([[12.0, 1.0]]))


def test_project_rows_onto_a_full_orthogonal_basis_reconstructs_the_rows():
    rng = np.random.default_rng(3)
    G, d, rows = 3, 8, 5
    layers = [rng.standard_normal((rows, d)).astype(np.float32) for _ in range(G)]
    Q, _ = np.linalg.qr(rng.standard_normal((G * d, G * d)))
    V = Q.astype(np.float32)
    A = oracle.project_rows(layers, V)
    X = np.concatenate(layers, axis=1).astype(np.float64)
    assert np.abs(A @ V.astype(np.float64).T - X).max() < 1e-5
    # a sub-basis gives the leading columns
    assert np.abs(oracle.project_rows(layers, V[:, :4]) - A[:, :4]).max() == 0.0


def test_chunk_landmark_of_a_constant_key_is_the_rotation_mean():
    # key k constant over the chunk: for pair j the mean of the rotations by
    # (t0 + i) f_j, i < C, is the geometric sum e^{i t0 f}(1 - e^{i C f}) / (C (1 - e^{i f}))
    hd, C, t0, theta = 8, 8, 1234, 500000.0
    rng = np.random.default_rng(5)
    k = rng.standard_normal(hd)
    K = np.tile(k.astype(np.float32), (C, 1))
    out = oracle.chunk_landmark(K, 1, hd, t0, theta)[0]
    h = hd // 2
    for j in range(h):
        f = theta ** (-2.0 * j / hd)
        m = np.exp(1j * t0 * f) * (1 - np.exp(1j * C * f)) / (C * (1 - np.exp(1j * f)))
        z = (np.float32(k[j]) + 1j * np.float32(k[j + h])) * m
        assert abs(out[j] - z.real) < 1e-12 and abs(out[j + h] - z.imag) < 1e-12


def test_chunk_landmark_agrees_with_the_prefill_landmarks():
    w = synth.WORKLOADS["tiny_f32"]
    K = synth.kv_group(w, 0, 0, "K", T=w.T)[1]
    lm = oracle.landmarks(K, w.n_kv_heads, w.head_dim, w.chunk, w.sink, w.recent, w.rope_theta)
    for c in (0, 7, w.n_mid - 1):
        t0 = w.sink + c * w.chunk
        one = oracle.chunk_landmark(K[t0:t0 + w.chunk], w.n_kv_heads, w.head_dim, t0, w.rope_theta)
        assert np.abs(one - lm[:, c]).max() < 1e-12


def _state(w, T0, rank):
    """A prefill state of one sequence: full-rank orthonormal bases, A = X V,
    landmarks of the middle chunks, and the raw sink / recent rows."""
    G, d, s, Cn = w.group, w.d, w.sink, w.chunk
    Ks = synth.kv_group(w, 0, 0, "K", T=T0)
    Vs = synth.kv_group(w, 0, 0, "V", T=T0)
    n = G * d
    rng = np.random.default_rng(11)
    bases = [oracle.round_bf16(np.linalg.qr(rng.standard_normal((n, n)))[0][:, :rank]) for _ in range(2)]
    cap = T0 + 4 * Cn
    A = []
    for X, Bt in ((Ks, bases[0]), (Vs, bases[1])):
        a = np.zeros((1, cap, rank), np.float32)
        a[0, :T0] = oracle.round_bf16(oracle.project_rows(X, Bt))
        A.append(a)
    n_mid = (T0 - s - w.recent) // Cn
    lms, wk, wv = [], [], []
    for l in range(G):
        lm = np.zeros((1, w.n_kv_heads, n_mid + 4, w.head_dim), np.float32)
        lm[0, :, :n_mid] = oracle.round_bf16(oracle.landmarks(Ks[l], w.n_kv_heads, w.head_dim, Cn, s, w.recent,
                                                              w.rope_theta))
        lms.append(lm)
        for src, dst in ((Ks[l], wk), (Vs[l], wv)):
            win = np.zeros((1, s + w.recent + Cn, d), np.float32)
            win[0, :s] = src[:s]
            win[0, s:s + w.recent] = src[T0 - w.recent:]
            dst.append(win)
    st = oracle.SRState(w, A[0], A[1], bases[0][None], bases[1][None], lms, wk, wv, T0, n_mid, w.recent)
    return st, Ks, Vs


def test_roll_moves_one_chunk_and_keeps_the_last_recent_rows():
    w = synth.WORKLOADS["tiny_f32"].replace(name="roll", batch=1)
    T0 = w.sink + w.recent + 8 * w.chunk
    st, Ks, Vs = _state(w, T0, 64)
    rng = np.random.default_rng(2)
    new_k = [[rng.standard_normal((1, w.d)).astype(np.float32) for _ in range(w.group)]
             for _ in range(2 * w.chunk + 3)]
    new_v = [[rng.standard_normal((1, w.d)).astype(np.float32) for _ in range(w.group)] for _ in new_k]
    rolls = [st.append(k, v) for k, v in zip(new_k, new_v)]
    # a roll every chunk appends, starting once the window holds recent + chunk rows
    assert [i for i, r in enumerate(rolls) if r] == [w.chunk - 1, 2 * w.chunk - 1]
    assert st.T == T0 + len(new_k) and st.n_mid == 10 and st.w_cur == w.recent + 3
    # the window holds the last w_cur tokens of the stream in order
    hist = [np.concatenate([Ks[l][T0 - w.recent:]] + [k[l] for k in new_k]) for l in range(w.group)]
    for l in range(w.group):
        assert np.array_equal(st.win_K[l][0, w.sink:w.sink + st.w_cur], hist[l][-st.w_cur:])
        assert np.array_equal(st.win_K[l][0, :w.sink], Ks[l][:w.sink])
    # the rolled chunk at positions t0..t0+C-1 got A = round(x V) and its landmark
    t0 = w.sink + 9 * w.chunk
    rows = [hist[l][len(hist[l]) - st.w_cur - w.chunk:len(hist[l]) - st.w_cur] for l in range(w.group)]
    assert np.array_equal(st.A_K[0, t0:t0 + w.chunk], oracle.round_bf16(oracle.project_rows(rows, st.Bt_K[0])))
    lm = oracle.chunk_landmark(rows[2], w.n_kv_heads, w.head_dim, t0, w.rope_theta)
    assert np.array_equal(st.lms[2][0, :, 9], oracle.round_bf16(lm))


def test_decode_after_rolls_at_full_rank_and_every_chunk_kept_is_dense_attention():
    # with a full-rank basis and every middle chunk kept, SR decode over the
    # rolled state is dense attention over the whole token history (up to the
    # bf16 storage of A)
    w = synth.WORKLOADS["tiny_f32"].replace(name="roll2", batch=1, n_kv_heads=1, n_q_heads=2, head_dim=32, group=2,
                                            n_layers=2, latent=24)
    T0 = w.sink + w.recent + 4 * w.chunk
    n = w.group * w.d
    st, Ks, Vs = _state(w, T0, n)
    rng = np.random.default_rng(4)
    hk = [list(Ks[l]) for l in range(w.group)]
    hv = [list(Vs[l]) for l in range(w.group)]
    for _ in range(2 * w.chunk + 5):
        k = [rng.standard_normal((1, w.d)).astype(np.float32) for _ in range(w.group)]
        v = [rng.standard_normal((1, w.d)).astype(np.float32) for _ in range(w.group)]
        st.append(k, v)
        for l in range(w.group):
            hk[l].append(k[l][0])
            hv[l].append(v[l][0])
    T = st.T
    layer = 1
    wd = w.replace(T=T, recent=st.w_cur, topk=st.n_mid)
    q = rng.standard_normal((1, w.n_q_heads, w.head_dim)).astype(np.float32)
    lm = np.ascontiguousarray(st.lms[layer][:, :, :st.n_mid])
    srK = np.ascontiguousarray(st.win_K[layer][:, :w.sink + st.w_cur])
    srV = np.ascontiguousarray(st.win_V[layer][:, :w.sink + st.w_cur])
    d = w.d
    BtK = st.Bt_K[:, layer * d:(layer + 1) * d]
    BtV = st.Bt_V[:, layer * d:(layer + 1) * d]
    out, _, _ = oracle.sr_decode(wd, q, st.A_K[:, :T], BtK, st.A_V[:, :T], BtV, lm, srK, srV)
    Kh = np.array(hk[layer], np.float32)
    Kr = np.stack([oracle.rope(Kh[t], t, w.rope_theta) for t in range(T)]).astype(np.float32)
    ref = oracle.dense_decode(q, Kr[None], np.array(hv[layer], np.float32)[None], w.n_kv_heads)
    assert np.abs(out - ref).max() < 2e-2
