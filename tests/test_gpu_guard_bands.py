"""Out-of-bounds writes, checked without a memory checker: every output and
every workspace of the public calls is carved out of a larger device buffer
whose bands before and after hold a guard pattern (all bytes 0xFF: NaN for
floats, -1 for indices).  After each call the bands must be intact, and the
outputs must have been written everywhere the call defines them (no NaN or -1
left inside).  The shapes are small and ragged (a partial last tile, odd chunk
and row counts, shards that end mid-tile), where an index error would spill
over an edge.  Values are checked against the oracle by the parity tests; here
only the write footprint is checked.
"""
import math

import numpy as np
import pytest
import torch

import synth
from gpu_helpers import dev, sr_inputs_on_device, tdtype

pytestmark = pytest.mark.gpu

GUARD = 4096  # bytes on each side; a multiple of 256, so carved tensors keep their alignment
FILL = 0xFF


class Carved:
    """A tensor of `shape` inside a guarded byte buffer."""

    def __init__(self, shape, dtype):
        el = torch.empty((), dtype=dtype).element_size()
        nbytes = math.prod(shape) * el
        self.buf = torch.full((2 * GUARD + nbytes,), FILL, dtype=torch.uint8, device="cuda")
        self.t = self.buf[GUARD:GUARD + nbytes].view(dtype).view(shape)
        self.nbytes = nbytes

    def guards_intact(self) -> bool:
        b = self.buf.cpu().numpy()
        return bool((b[:GUARD] == FILL).all() and (b[GUARD + self.nbytes:] == FILL).all())


class CarvedWorkspace:
    """A workspace of `nbytes` followed by a guard band."""

    def __init__(self, nbytes):
        nbytes = max(int(nbytes), 256)
        self.buf = torch.full((nbytes + GUARD,), FILL, dtype=torch.uint8, device="cuda")
        self.t = self.buf[:nbytes]
        self.nbytes = nbytes

    def guard_intact(self) -> bool:
        return bool((self.buf[self.nbytes:].cpu().numpy() == FILL).all())


def _written(t: torch.Tensor) -> bool:
    x = t.detach().cpu()
    if x.dtype in (torch.int32, torch.int64):
        return bool((x != -1).all())
    return bool(torch.isfinite(x.float()).all())


def _sr_case(xkv, w, xk=False):
    inp = synth.compressed_cache(w, 0)
    d_inp = sr_inputs_on_device(w, inp)
    B = inp["q"].shape[0]
    out = Carved((B, w.n_q_heads, w.head_dim), torch.float32)
    sel = Carved((B, w.n_kv_heads, w.topk), torch.int32)
    if xk:
        V = dev(synth.raw_values(w, 0), tdtype(w))
        p = xkv.xk_sr_params(B, w.n_q_heads, w.n_kv_heads, w.head_dim, w.T, w.rank_k, w.chunk, w.topk, w.sink,
                             w.recent, w.rope_theta, tdtype(w))
        ws = CarvedWorkspace(xkv.xkv_xk_sr_workspace_size(p))
        xkv.xkv_xk_sr_attention_decode(p, d_inp["q"], d_inp["A_K"], d_inp["Bt_K"], V, d_inp["landmarks"],
                                       d_inp["sr_K"], d_inp["sr_V"], out.t, sel.t, ws=ws.t)
    else:
        p = xkv.sr_params(B, w.n_q_heads, w.n_kv_heads, w.head_dim, w.T, w.rank_k, w.rank_v, w.chunk, w.topk,
                          w.sink, w.recent, w.rope_theta, tdtype(w))
        ws = CarvedWorkspace(xkv.xkv_sr_workspace_size(p))
        xkv.xkv_sr_attention_decode(p, d_inp["q"], d_inp["A_K"], d_inp["Bt_K"], d_inp["A_V"], d_inp["Bt_V"],
                                    d_inp["landmarks"], d_inp["sr_K"], d_inp["sr_V"], out.t, sel.t, ws=ws.t)
    torch.cuda.synchronize()
    assert xkv.get_device_status() == 0
    assert out.guards_intact() and sel.guards_intact() and ws.guard_intact()
    assert _written(out.t) and _written(sel.t)


@pytest.mark.parametrize("name,args,kw", [
    # tensor-core path, ragged last tile (37 chunks = 296 rows)
    ("gb_bf16", (2, 4, 4, 2, 128, 8, 8 + 32 + 8 * 150, 96, 0.8, 128, 192), dict(topk=37)),
    # odd value rank (entry-by-entry merge), GQA group of 3
    ("gb_oddrank", (1, 4, 4, 2, 128, 6, 8 + 32 + 8 * 90, 96, 0.8, 64, 51), dict(topk=19)),
    # f32 SIMT path, chunk 4, 3 KV heads of 64
    ("gb_f32", (2, 4, 4, 3, 64, 6, 5 + 7 + 4 * 90, 48, 0.8, 48, 80),
     dict(chunk=4, topk=23, sink=5, recent=7, dtype="f32")),
])
def test_sr_decode_writes_only_its_outputs(xkv, name, args, kw):
    _sr_case(xkv, synth.Workload(name, *args, **kw))


def test_xk_sr_decode_writes_only_its_outputs(xkv):
    _sr_case(xkv, synth.Workload("gb_xk", 2, 4, 4, 2, 128, 8, 8 + 32 + 8 * 130, 96, 0.8, 128, 128, topk=29), xk=True)


def test_landmarks_write_only_their_rows(xkv):
    w = synth.Workload("gb_lm", 1, 4, 4, 2, 128, 8, 8 + 32 + 8 * 211, 96, 0.8, 64, 64)
    K = dev(synth.kv_group(w, 0, 0, "K")[0], torch.bfloat16)
    n_mid = (w.T - w.sink - w.recent) // w.chunk
    lm = Carved((w.n_kv_heads, n_mid, w.head_dim), torch.bfloat16)
    xkv.xkv_build_landmarks(K, w.n_kv_heads, w.head_dim, w.chunk, w.sink, w.recent, w.rope_theta, lm.t)
    torch.cuda.synchronize()
    assert lm.guards_intact() and _written(lm.t)


@pytest.mark.parametrize("dt,G,T,rank,shard", [("bf16", 2, 1000, 64, 384), ("bf16", 3, 777, 128, 512),
                                               ("f32", 2, 600, 48, 256)])
def test_compress_group_writes_only_its_factors(xkv, dt, G, T, rank, shard):
    w = synth.WORKLOADS["tiny_f32"].replace(name=f"gb_cmp{G}{dt}", group=G, n_layers=G, dtype=dt, n_kv_heads=2,
                                             head_dim=64)
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    X = [dev(l, tdt) for l in synth.kv_group(w, 0, 0, "K", T=T)]
    n = G * w.d
    A = Carved((T, rank), tdt)
    Bt = Carved((n, rank), tdt)
    ev = Carved((rank,), torch.float32)
    gram = Carved((n, n), torch.float32)
    over = synth.oversample(rank)
    ws = CarvedWorkspace(xkv.xkv_compress_workspace_size(G, T, w.d, rank, over, shard, tdt))
    xkv.xkv_compress_group(X, rank, A.t, Bt.t, oversample=over, shard_rows=shard, eigvals=ev.t, gram_out=gram.t,
                           ws=ws.t)
    torch.cuda.synchronize()
    assert xkv.get_device_status() == 0
    for c in (A, Bt, ev, gram):
        assert c.guards_intact() and _written(c.t)
    assert ws.guard_intact()


def test_full_reconstruct_writes_only_its_rows(xkv):
    T, r, Hkv, hd = 1000, 96, 2, 128
    g = torch.Generator(device="cpu").manual_seed(5)
    A = torch.randn((T, r), generator=g).to("cuda", torch.bfloat16)
    Bt = torch.randn((Hkv * hd, r), generator=g).to("cuda", torch.bfloat16)
    for rope in (False, True):
        out = Carved((T, Hkv * hd), torch.bfloat16)
        xkv.xkv_full_reconstruct(A, Bt, Hkv, hd, rope, 500000.0, out.t)
        torch.cuda.synchronize()
        assert out.guards_intact() and _written(out.t)


def test_ner_and_energy_rank_write_only_their_entries(xkv):
    n, block = 3 * 96, 96
    g = np.random.default_rng(11)
    X = g.standard_normal((700, n)).astype(np.float32)
    gram = torch.from_numpy(X.T.astype(np.float64) @ X.astype(np.float64)).float().cuda()
    count = n // block
    ner = Carved((count,), torch.float32)
    erank = Carved((count,), torch.float32)
    rank = Carved((count,), torch.int32)
    ws = CarvedWorkspace(xkv.xkv_ner_workspace_size(n, block))
    xkv.xkv_ner(gram, block, ner.t, erank.t, rank.t, ws=ws.t)
    torch.cuda.synchronize()
    assert xkv.get_device_status() == 0
    for c in (ner, erank, rank):
        assert c.guards_intact() and _written(c.t)
    assert ws.guard_intact()
    er = Carved((count,), torch.int32)
    lam = Carved((n,), torch.float32)
    ws2 = CarvedWorkspace(xkv.xkv_ner_workspace_size(n, block))
    xkv.xkv_energy_rank(gram, block, 0.95, er.t, lam.t, ws=ws2.t)
    torch.cuda.synchronize()
    assert er.guards_intact() and lam.guards_intact() and ws2.guard_intact()
    assert _written(er.t) and _written(lam.t)
