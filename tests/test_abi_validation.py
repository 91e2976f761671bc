"""Host-side argument checks of the calls beyond the five hot-path ones: the
multi-step append, the token-sharding pieces (scores, top-k, partial
attention, merge), the factorisation of a given Gram, the projection and the
xK-SR step with values in host memory.  Every case returns its status before
any CUDA call, so no GPU is needed: the fake, aligned addresses below are
never dereferenced."""
import ctypes as C

import pytest
import torch

FAKE = C.c_void_p(1 << 20)
MIS = C.c_void_p((1 << 20) + 4)  # 4-byte aligned only
CHUNK, SINK, RECENT, HKV, HD, RANK, G = 8, 8, 32, 2, 64, 64, 2
D = HKV * HD


def _append(xkv, **kw):
    T = SINK + RECENT + CHUNK * 10  # ten middle chunks, no roll on the next token
    base = dict(batch=1, group=G, n_kv_heads=HKV, head_dim=HD, chunk=CHUNK, sink=SINK, recent=RECENT,
                rope_theta=5e5, dtype=torch.float32, T=T, rank_k=RANK, rank_v=RANK,
                a_k_batch_stride=(T + CHUNK) * RANK, a_v_batch_stride=(T + CHUNK) * RANK, bt_k_batch_stride=0,
                bt_v_batch_stride=0, window_batch_stride=(SINK + RECENT + CHUNK) * D, landmark_capacity=11)
    base.update(kw)
    return xkv.append_params(**base)


def _append_ws(xkv, p):
    n = C.c_size_t(0)
    return xkv.lib.xkv_sr_append_workspace_size(C.byref(p), C.byref(n)), n.value


def test_append_parameter_checks(xkv):
    s, n = _append_ws(xkv, _append(xkv))
    assert s == xkv.XKV_OK and n > 0
    T = SINK + RECENT + CHUNK * 10
    for bad in (dict(group=9), dict(T=SINK + RECENT - 1), dict(rank_k=G * D + 16), dict(rope_theta=1.0),
                dict(window_batch_stride=(SINK + RECENT + CHUNK) * D + 4),  # not a multiple of 8
                dict(window_batch_stride=(SINK + RECENT) * D),              # no room for a chunk more
                dict(landmark_capacity=9),                                   # below the chunks held
                dict(a_k_batch_stride=(SINK + CHUNK * 10) * RANK - 1),     # A holds sink + middle rows
                dict(bt_v_batch_stride=-1), dict(head_dim=63)):
        assert _append_ws(xkv, _append(xkv, **bad))[0] == xkv.XKV_ERR_INVALID_ARG, bad
    # a token that completes a chunk rolls it: the landmark capacity must hold one more
    roll = dict(T=SINK + RECENT + CHUNK * 10 + CHUNK - 1, a_k_batch_stride=(T + 2 * CHUNK) * RANK,
                a_v_batch_stride=(T + 2 * CHUNK) * RANK)
    assert _append_ws(xkv, _append(xkv, landmark_capacity=11, **roll))[0] == xkv.XKV_OK
    assert _append_ws(xkv, _append(xkv, landmark_capacity=10, **roll))[0] == xkv.XKV_ERR_INVALID_ARG
    # the recent window beyond 56 rows, and bf16 ranks off the tensor-core grid
    assert _append_ws(xkv, _append(xkv, recent=64, T=SINK + 64 + CHUNK * 10,
                                   window_batch_stride=(SINK + 64 + CHUNK) * D))[0] == xkv.XKV_ERR_UNSUPPORTED
    assert _append_ws(xkv, _append(xkv, dtype=torch.bfloat16, rank_k=48))[0] == xkv.XKV_ERR_UNSUPPORTED


def test_append_pointer_and_workspace_checks(xkv):
    p = _append(xkv)
    _, need = _append_ws(xkv, p)
    arr = lambda *x: (C.c_void_p * G)(*x)  # noqa: E731
    ok = arr(FAKE, FAKE)
    f = xkv.lib.xkv_sr_append
    rolled = C.c_int(0)
    assert f(C.byref(p), None, ok, ok, ok, FAKE, FAKE, FAKE, FAKE, ok, C.byref(rolled), FAKE, need, None) == \
        xkv.XKV_ERR_INVALID_ARG                      # no k_new array
    assert f(C.byref(p), arr(FAKE, None), ok, ok, ok, FAKE, FAKE, FAKE, FAKE, ok, C.byref(rolled), FAKE, need,
             None) == xkv.XKV_ERR_INVALID_ARG          # a layer's pointer missing
    assert f(C.byref(p), ok, ok, arr(FAKE, MIS), ok, FAKE, FAKE, FAKE, FAKE, ok, C.byref(rolled), FAKE, need,
             None) == xkv.XKV_ERR_INVALID_ARG          # a window misaligned
    assert f(C.byref(p), ok, ok, ok, ok, FAKE, None, FAKE, FAKE, ok, C.byref(rolled), FAKE, need, None) == \
        xkv.XKV_ERR_INVALID_ARG                      # no Bt_V
    assert f(C.byref(p), ok, ok, ok, ok, FAKE, FAKE, FAKE, FAKE, ok, C.byref(rolled), FAKE, need - 1, None) == \
        xkv.XKV_ERR_WORKSPACE
    assert f(C.byref(p), ok, ok, ok, ok, FAKE, FAKE, FAKE, FAKE, ok, C.byref(rolled), MIS, need, None) == \
        xkv.XKV_ERR_WORKSPACE                        # workspace not 256-byte aligned


def _sr(xkv, **kw):
    base = dict(batch=1, n_q_heads=8, n_kv_heads=HKV, head_dim=HD, T=1024, rank_k=RANK, rank_v=RANK, chunk=CHUNK,
                topk=16, sink=SINK, recent=RECENT, rope_theta=5e5)
    base.update(kw)
    return xkv.sr_params(dtype=torch.float32, **base)


def test_topk_checks(xkv):
    f = xkv.lib.xkv_sr_topk
    assert f(None, 2048, 1, 2000, 16, FAKE, None) == xkv.XKV_ERR_INVALID_ARG
    assert f(FAKE, 2048, 1, 2000, 16, MIS, None) == xkv.XKV_ERR_INVALID_ARG
    assert f(FAKE, 2048, 0, 2000, 16, FAKE, None) == xkv.XKV_ERR_INVALID_ARG     # no rows
    assert f(FAKE, 2048, 1, 2000, 2001, FAKE, None) == xkv.XKV_ERR_INVALID_ARG   # k > n
    assert f(FAKE, 2048, 1, 2000, 0, FAKE, None) == xkv.XKV_ERR_INVALID_ARG      # k < 1
    assert f(FAKE, 1999, 1, 2000, 16, FAKE, None) == xkv.XKV_ERR_INVALID_ARG     # ld < n
    assert f(FAKE, 2002, 1, 2000, 16, FAKE, None) == xkv.XKV_ERR_INVALID_ARG     # ld not a multiple of 4
    assert f(FAKE, 24580, 1, 24577, 16, FAKE, None) == xkv.XKV_ERR_UNSUPPORTED   # n above the chunk limit
    assert f(FAKE, 2048, 1, 2000, 1025, FAKE, None) == xkv.XKV_ERR_UNSUPPORTED   # k above 1024


def test_scores_partial_and_merge_checks(xkv):
    p = _sr(xkv)
    n_mid = (1024 - SINK - RECENT) // CHUNK
    ld = (n_mid + 3) // 4 * 4
    f = xkv.lib.xkv_sr_scores
    assert f(C.byref(p), None, FAKE, FAKE, ld, None) == xkv.XKV_ERR_INVALID_ARG
    assert f(C.byref(p), FAKE, FAKE, FAKE, n_mid - 1, None) == xkv.XKV_ERR_INVALID_ARG
    assert f(C.byref(p), FAKE, FAKE, FAKE, ld + 2, None) == xkv.XKV_ERR_INVALID_ARG
    n = C.c_size_t(0)
    ws = xkv.lib.xkv_sr_partial_workspace_size
    assert ws(C.byref(p), C.byref(n)) == xkv.XKV_OK and n.value > 0
    need = n.value
    # the global k may exceed the local chunks, but not 1024
    assert ws(C.byref(_sr(xkv, topk=n_mid + 50)), C.byref(n)) == xkv.XKV_OK
    assert ws(C.byref(_sr(xkv, topk=1025)), C.byref(n)) == xkv.XKV_ERR_UNSUPPORTED
    assert ws(C.byref(_sr(xkv, topk=0)), C.byref(n)) == xkv.XKV_ERR_INVALID_ARG
    part = xkv.lib.xkv_sr_attention_partial
    sh = xkv.ShardParams(0, 0)
    args = [FAKE] * 7  # sel, q, A_K, Bt_K, A_V, Bt_V, then sr_K
    assert part(C.byref(p), None, *args, FAKE, FAKE, FAKE, FAKE, need, None) == xkv.XKV_ERR_INVALID_ARG
    assert part(C.byref(p), C.byref(xkv.ShardParams(-1, 0)), *args, FAKE, FAKE, FAKE, FAKE, need, None) == \
        xkv.XKV_ERR_INVALID_ARG                      # negative position offset
    assert part(C.byref(p), C.byref(sh), None, *args[1:], FAKE, FAKE, FAKE, FAKE, need, None) == \
        xkv.XKV_ERR_INVALID_ARG                      # no selection
    assert part(C.byref(p), C.byref(sh), *args, FAKE, FAKE, None, FAKE, need, None) == \
        xkv.XKV_ERR_INVALID_ARG                      # no (M, L) output
    assert part(C.byref(p), C.byref(sh), *args, FAKE, FAKE, FAKE, FAKE, need - 1, None) == xkv.XKV_ERR_WORKSPACE
    m = xkv.lib.xkv_merge_partials
    assert m(FAKE, FAKE, 0, 8, 64, FAKE, None) == xkv.XKV_ERR_INVALID_ARG
    assert m(FAKE, None, 2, 8, 64, FAKE, None) == xkv.XKV_ERR_INVALID_ARG
    assert m(FAKE, FAKE, 2, 8, 0, FAKE, None) == xkv.XKV_ERR_INVALID_ARG


def test_factor_and_project_checks(xkv):
    n = C.c_size_t(0)
    fw = xkv.lib.xkv_factor_workspace_size
    assert fw(G, D, 1000, RANK, 64, xkv.XKV_F32, C.byref(n)) == xkv.XKV_OK and n.value > 0
    need = n.value
    assert fw(G, D, 50, RANK, 64, xkv.XKV_F32, C.byref(n)) == xkv.XKV_ERR_INVALID_ARG      # rank > rows
    assert fw(G, 96, 1000, RANK, 64, xkv.XKV_F32, C.byref(n)) == xkv.XKV_ERR_INVALID_ARG   # d % 64
    assert fw(G, D, 1000, 40, 64, xkv.XKV_F32, C.byref(n)) == xkv.XKV_ERR_INVALID_ARG      # rank % 16
    assert fw(8, 1024, 1 << 20, 3520, 65, xkv.XKV_F32, C.byref(n)) == xkv.XKV_ERR_UNSUPPORTED  # b > 3584
    f = xkv.lib.xkv_factor_gram
    assert f(MIS, G, D, 1000, xkv.XKV_F32, RANK, 8, 64, 1, FAKE, None, None, FAKE, need, None) == \
        xkv.XKV_ERR_INVALID_ARG
    assert f(FAKE, G, D, 1000, xkv.XKV_F32, RANK, 8, 64, 1, FAKE, MIS, None, FAKE, need, None) == \
        xkv.XKV_ERR_INVALID_ARG                      # misaligned V_r output
    assert f(FAKE, G, D, 1000, xkv.XKV_F32, RANK, 0, 64, 1, FAKE, None, None, FAKE, need, None) == \
        xkv.XKV_ERR_INVALID_ARG                      # no iteration
    assert f(FAKE, G, D, 1000, xkv.XKV_F32, RANK, 8, 64, 1, FAKE, None, None, FAKE, need - 1, None) == \
        xkv.XKV_ERR_WORKSPACE
    pw = xkv.lib.xkv_project_workspace_size
    assert pw(G, D, RANK, C.byref(n)) == xkv.XKV_OK and n.value > 0
    pneed = n.value
    assert pw(9, D, RANK, C.byref(n)) == xkv.XKV_ERR_INVALID_ARG
    p = xkv.lib.xkv_project
    layers = (C.c_void_p * G)(FAKE, FAKE)
    assert p(layers, G, 1000, D, D, xkv.XKV_BF16, FAKE, xkv.XKV_F32, G * D + 64, FAKE, G * D + 64, FAKE, pneed,
             None) == xkv.XKV_ERR_INVALID_ARG       # rank > G d
    assert p(layers, G, 1000, D, D, xkv.XKV_BF16, FAKE, xkv.XKV_F32, RANK, FAKE, RANK - 1, FAKE, pneed,
             None) == xkv.XKV_ERR_INVALID_ARG       # lda < rank
    assert p(layers, G, 1000, D, D, xkv.XKV_BF16, FAKE, xkv.XKV_F32, RANK, FAKE, RANK, FAKE, pneed - 1,
             None) == xkv.XKV_ERR_WORKSPACE
    assert p(layers, G, 1000, D, D, xkv.XKV_BF16, FAKE, xkv.XKV_F32, 48, FAKE, 48, FAKE, pneed, None) == \
        xkv.XKV_ERR_UNSUPPORTED                      # bf16 off the tensor-core grid, f32 basis
    assert p((C.c_void_p * G)(FAKE, None), G, 1000, D, D, xkv.XKV_BF16, FAKE, xkv.XKV_F32, RANK, FAKE, RANK, FAKE,
             pneed, None) == xkv.XKV_ERR_INVALID_ARG


def test_host_value_step_checks(xkv):
    p = xkv.xk_sr_params(1, 8, HKV, HD, 1024, RANK, CHUNK, 16, SINK, RECENT, 5e5, torch.float32)
    n = C.c_size_t(0)
    assert xkv.lib.xkv_xk_sr_host_workspace_size(C.byref(p), C.byref(n)) == xkv.XKV_OK
    base = n.value
    assert xkv.lib.xkv_xk_sr_workspace_size(C.byref(p), C.byref(n)) == xkv.XKV_OK
    assert base > n.value  # the staging area for the kept value rows comes on top
    bad = xkv.xk_sr_params(1, 8, HKV, HD, 1024, RANK, CHUNK, 124, SINK, RECENT, 5e5, torch.float32)
    assert xkv.lib.xkv_xk_sr_host_workspace_size(C.byref(bad), C.byref(n)) == xkv.XKV_ERR_INVALID_ARG
    f = xkv.lib.xkv_xk_sr_attention_decode_host_values
    # q, A_K, Bt_K, V_host, landmarks, sr_K, sr_V, out, sel_out, workspace
    assert f(C.byref(p), FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, None, FAKE, base, None) == \
        xkv.XKV_ERR_INVALID_ARG                      # no values
    assert f(C.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, None, FAKE, base, None) == \
        xkv.XKV_ERR_INVALID_ARG                      # no raw window keys
    assert f(C.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, MIS, FAKE, base, None) == \
        xkv.XKV_ERR_INVALID_ARG                      # misaligned selection output


@pytest.mark.parametrize("fn", ["xkv_sr_append_workspace_size", "xkv_sr_partial_workspace_size",
                                "xkv_xk_sr_host_workspace_size"])
def test_size_queries_reject_null_outputs(xkv, fn):
    p = _append(xkv) if fn == "xkv_sr_append_workspace_size" else _sr(xkv)
    assert getattr(xkv.lib, fn)(C.byref(p), None) == xkv.XKV_ERR_INVALID_ARG
