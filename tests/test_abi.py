"""The C-ABI library loads, exports every symbol include/xkv.h declares, and
rejects bad arguments on the host (no GPU needed: validation happens before any
CUDA call and nothing is launched)."""
import ctypes as C
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "xkv.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"XKV_API\s+[\w\s\*]+?\b(xkv_\w+)\s*\(", src)))


def test_header_declares_the_five_hot_path_calls():
    names = _declared()
    for n in ("xkv_compress_group", "xkv_build_landmarks", "xkv_sr_attention_decode", "xkv_full_reconstruct",
              "xkv_ner"):
        assert n in names


def test_every_declared_symbol_is_exported(xkv):
    lib = C.CDLL(xkv.LIB_PATH)
    for n in _declared():
        assert hasattr(lib, n), n
    assert set(_declared()) == set(xkv.EXPORTS)


def test_status_strings_and_version(xkv):
    for s in range(7):
        assert xkv.status_string(s)
    assert xkv.lib.xkv_version() >> 16 == 1


def _sr(xkv, **kw):
    base = dict(batch=1, n_q_heads=8, n_kv_heads=2, head_dim=64, T=1024, rank_k=64, rank_v=64, chunk=8, topk=16,
                sink=8, recent=32, rope_theta=500000.0)
    base.update(kw)
    import torch
    return xkv.sr_params(dtype=torch.float32, **base)


@pytest.mark.parametrize("bad", [dict(topk=124), dict(T=1027), dict(n_q_heads=7), dict(chunk=0), dict(rank_k=0),
                                 dict(rope_theta=0.0), dict(head_dim=63), dict(batch=0)])
def test_sr_rejects_bad_shapes(xkv, bad):
    p = _sr(xkv, **bad)
    n = C.c_size_t(0)
    assert xkv.lib.xkv_sr_workspace_size(C.byref(p), C.byref(n)) == xkv.XKV_ERR_INVALID_ARG
    z = None
    assert xkv.lib.xkv_sr_attention_decode(C.byref(p), z, z, z, z, z, z, z, z, z, z, z, 0, z) == \
        xkv.XKV_ERR_INVALID_ARG


def test_sr_reports_unsupported_beyond_the_chunk_limit(xkv):
    # n_mid = 24577: one middle chunk more than the top-k's shared memory holds
    p = _sr(xkv, T=8 + 32 + 8 * 24577)
    n = C.c_size_t(0)
    assert xkv.lib.xkv_sr_workspace_size(C.byref(p), C.byref(n)) == xkv.XKV_ERR_UNSUPPORTED
    p = _sr(xkv, T=8 + 32 + 8 * 24576)
    assert xkv.lib.xkv_sr_workspace_size(C.byref(p), C.byref(n)) == xkv.XKV_OK


def test_sr_rejects_null_and_misaligned_pointers_and_small_workspace(xkv):
    p = _sr(xkv)
    n = C.c_size_t(0)
    assert xkv.lib.xkv_sr_workspace_size(C.byref(p), C.byref(n)) == xkv.XKV_OK and n.value > 0
    fake = C.c_void_p(1 << 20)  # aligned, never dereferenced: validation fails first
    mis = C.c_void_p((1 << 20) + 4)
    args = [fake] * 9
    assert xkv.lib.xkv_sr_attention_decode(C.byref(p), None, *args[1:], None, None, 0, None) == \
        xkv.XKV_ERR_INVALID_ARG
    assert xkv.lib.xkv_sr_attention_decode(C.byref(p), mis, *args[1:], None, None, 0, None) == \
        xkv.XKV_ERR_INVALID_ARG
    assert xkv.lib.xkv_sr_attention_decode(C.byref(p), *args, None, fake, 16, None) == xkv.XKV_ERR_WORKSPACE


def test_xk_sr_validation(xkv):
    import torch
    T, d = 1024, 2 * 64

    def xk(**kw):
        base = dict(batch=1, n_q_heads=8, n_kv_heads=2, head_dim=64, T=T, rank_k=64, chunk=8, topk=16, sink=8,
                    recent=32, rope_theta=500000.0, dtype=torch.float32)
        base.update(kw)
        return xkv.xk_sr_params(**base)

    n = C.c_size_t(0)
    p = xk()
    p.rank_v = 0  # ignored: the value rows are the uncompressed cache
    assert xkv.lib.xkv_xk_sr_workspace_size(C.byref(p), C.byref(n)) == xkv.XKV_OK and n.value > 0
    # a value batch stride below T d
    assert xkv.lib.xkv_xk_sr_workspace_size(C.byref(xk(v_batch_stride=T * 64)), C.byref(n)) == \
        xkv.XKV_ERR_INVALID_ARG
    assert xkv.lib.xkv_xk_sr_workspace_size(C.byref(xk(topk=124)), C.byref(n)) == xkv.XKV_ERR_INVALID_ARG
    fake = C.c_void_p(1 << 20)
    f = xkv.lib.xkv_xk_sr_attention_decode
    assert f(C.byref(p), fake, fake, fake, None, fake, fake, fake, fake, None, fake, 1 << 30, None) == \
        xkv.XKV_ERR_INVALID_ARG  # no V
    assert f(C.byref(p), fake, fake, fake, fake, fake, fake, fake, fake, None, fake, 16, None) == \
        xkv.XKV_ERR_WORKSPACE
    assert T * d == p.a_v_batch_stride


def test_compress_and_gram_validation(xkv):
    n = C.c_size_t(0)
    assert xkv.lib.xkv_compress_workspace_size(4, 1024, 128, 64, 64, 8192, xkv.XKV_F32, C.byref(n)) == xkv.XKV_OK
    assert n.value > 4 * 128 * 4 * 128 * 4
    # rank above G d, rank not a multiple of 16, d not a multiple of 64, G > 8
    for args in ((1, 1024, 128, 256), (4, 1024, 128, 40), (4, 1024, 96, 64), (9, 1024, 64, 64)):
        assert xkv.lib.xkv_compress_workspace_size(*args, 64, 0, xkv.XKV_F32, C.byref(n)) == xkv.XKV_ERR_INVALID_ARG
    # bf16 needs rank % 64 == 0
    assert xkv.lib.xkv_compress_workspace_size(4, 1024, 128, 48, 64, 0, xkv.XKV_BF16, C.byref(n)) == \
        xkv.XKV_ERR_UNSUPPORTED
    # block width b = min(rank + oversample, G d, T) up to 3584 (the compression
    # sweep's largest case, G = 8 at rank 1024 with p = 256, is far inside)
    f = xkv.lib.xkv_compress_workspace_size
    assert f(8, 32768, 1024, 1024, 256, 8192, xkv.XKV_BF16, C.byref(n)) == xkv.XKV_OK
    assert f(8, 32768, 1024, 3520, 64, 8192, xkv.XKV_F32, C.byref(n)) == xkv.XKV_OK
    assert f(8, 32768, 1024, 3520, 65, 8192, xkv.XKV_F32, C.byref(n)) == xkv.XKV_ERR_UNSUPPORTED
    assert f(8, 32768, 1024, 4096, 1024, 8192, xkv.XKV_BF16, C.byref(n)) == xkv.XKV_ERR_UNSUPPORTED
    assert f(8, 3000, 1024, 2048, 4096, 0, xkv.XKV_BF16, C.byref(n)) == xkv.XKV_OK  # b capped by T
    ptrs = (C.c_void_p * 2)(None, None)
    assert xkv.lib.xkv_gram_accumulate(ptrs, 2, 100, 64, 64, xkv.XKV_F32, C.c_void_p(1 << 20), None, 0, None) == \
        xkv.XKV_ERR_INVALID_ARG


def test_landmarks_recon_dense_ner_validation(xkv):
    fake = C.c_void_p(1 << 20)
    assert xkv.lib.xkv_build_landmarks(fake, 1027, 128, 2, 64, xkv.XKV_F32, 8, 8, 32, 5e5, fake, None) == \
        xkv.XKV_ERR_INVALID_ARG
    assert xkv.lib.xkv_full_reconstruct(fake, fake, 100, 64, 128, 2, 32, 1, 5e5, xkv.XKV_F32, fake, None) == \
        xkv.XKV_ERR_INVALID_ARG  # Hkv * hd != d
    bad = xkv.DenseParams(1, 6, 4, 64, 100, xkv.XKV_F32)
    n = C.c_size_t(0)
    assert xkv.lib.xkv_dense_workspace_size(C.byref(bad), C.byref(n)) == xkv.XKV_ERR_INVALID_ARG
    assert xkv.lib.xkv_ner_workspace_size(100, 30, C.byref(n)) == xkv.XKV_ERR_INVALID_ARG
    assert xkv.lib.xkv_ner(fake, 128, 64, 1e-9, fake, None, None, None, 0, None) == xkv.XKV_ERR_WORKSPACE


def test_energy_rank_validation(xkv):
    # argument checks run before any device work: fake, aligned pointers suffice
    g, r, ws = C.c_void_p(0x10000), C.c_void_p(0x20000), C.c_void_p(0x30000)
    n = C.c_size_t(0)
    assert xkv.lib.xkv_ner_workspace_size(256, 128, C.byref(n)) == xkv.XKV_OK
    f = xkv.lib.xkv_energy_rank
    assert f(g, 256, 128, 0.0, r, None, ws, n.value, None) == xkv.XKV_ERR_INVALID_ARG     # energy <= 0
    assert f(g, 256, 128, 1.5, r, None, ws, n.value, None) == xkv.XKV_ERR_INVALID_ARG     # energy > 1
    assert f(g, 256, 100, 0.9, r, None, ws, n.value, None) == xkv.XKV_ERR_INVALID_ARG     # n % block
    assert f(g, 256, 128, 0.9, None, None, ws, n.value, None) == xkv.XKV_ERR_INVALID_ARG  # no rank output
    assert f(g, 256, 128, 0.9, r, None, ws, n.value - 1, None) == xkv.XKV_ERR_WORKSPACE
    assert f(g, 2 * 16384, 16384, 0.9, r, None, ws, 1 << 40, None) == xkv.XKV_ERR_UNSUPPORTED  # block > 8192


def test_plain_c_host_program(xkv, tmp_path):
    # the boundary is plain C: a C99 program that includes only xkv.h builds
    # against libxkv.so and sees the same validation results
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.dirname(xkv.LIB_PATH)
    exe = str(tmp_path / "abi_host_check")
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(root, "include"),
                           os.path.join(root, "tests", "abi_host_check.c"), "-L", libdir, "-lxkv",
                           "-Wl,-rpath," + libdir, "-o", exe])
    out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "ok"


def test_package_fails_loudly_without_the_library(tmp_path):
    # a copy of the binding with no libxkv.so beside it must refuse to import:
    # there is no CPU or PyTorch fallback
    pkg = tmp_path / "cross_layer_rank_b200"
    pkg.mkdir()
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = open(os.path.join(root, "cross_layer_rank_b200", "__init__.py")).read()
    (pkg / "__init__.py").write_text(src)
    code = "import sys; sys.path.insert(0, sys.argv[1]); import cross_layer_rank_b200"
    out = subprocess.run([sys.executable, "-c", code, str(tmp_path)], capture_output=True, text=True, timeout=300)
    assert out.returncode != 0
    assert "ImportError" in out.stderr and "libxkv.so not built" in out.stderr


def test_binding_rejects_host_and_strided_tensors(xkv):
    import torch
    with pytest.raises(ValueError):
        xkv._ptr(torch.zeros(4))  # host memory
    if torch.cuda.is_available():
        with pytest.raises(ValueError):
            xkv._ptr(torch.zeros((4, 4), device="cuda").t())  # not contiguous
