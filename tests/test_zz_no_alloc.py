"""The allocation-free attention entry point, zha_sparse_attn_static.

It exists for callers that cannot allocate device memory where they attend (their
device memory belongs to another allocator, or the loop cannot afford an allocation and
the synchronisation it may bring).  It must give the same output as zha_sparse_attn for
the same routed sets while using only its fixed static working array.  This file is
collected last so that a failure here never hides the other tests.
"""
import numpy as np
import pytest
import torch

from hierarchical_tree_indexed_build_b200 import inputs, zha
from oracle import oracle as O
import zha_testlib as TL

pytestmark = pytest.mark.gpu
needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
OUT_TOL = 2e-3


def _rel(a, b):
    a = a.double().reshape(-1, a.shape[-1])
    b = b.double().reshape(-1, b.shape[-1])
    return ((a - b).abs().max(dim=1).values / b.abs().max(dim=1).values).max().item()


@needs_cuda
def test_static_attention_matches_sparse_attn_on_two_calls_in_a_row():
    g = inputs.DEEP
    n = 4 * 4096 + 777                                  # 4 top nodes + a dense tail
    seq = inputs.make_sequence(g, n, n, seed=77)
    K, V, qr = seq.K.cuda(), seq.V.cuda(), seq.qref.cuda()
    Q, _ = inputs.make_queries(seq, 2, 8, n, np.random.default_rng(5))
    Q = Q[None].cuda().contiguous()                     # [1][2][16][128]
    tree = zha.Tree(g.C, g.L, g.R, g.d, g.Hq, g.Hkv, n)
    tree.build(K, n, qr)
    dec = zha.Decoder([tree], 2)
    stream = torch.cuda.current_stream().cuda_stream
    for p in (0.95, 0.7):                               # two calls, different routed sets
        ref = dec.decode([K], [V], Q, p)
        bits, _ = dec.export_kept(1)
        out = torch.full_like(ref, float("nan"))
        zha.zha_sparse_attn_static(K.data_ptr(), V.data_ptr(), n, n, g.C, g.L, g.Hq, g.Hkv, g.d,
                                   Q.data_ptr(), 2, bits.data_ptr(), bits.shape[1], out.data_ptr(), stream)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all()
        assert _rel(out, ref) <= OUT_TOL, p


@needs_cuda
def test_static_attention_rejects_calls_beyond_its_array():
    g = inputs.DEEP
    n = 1 << 20
    K = torch.zeros((g.Hkv, 16, g.d), dtype=torch.bfloat16, device="cuda")
    Q = torch.zeros((64, g.Hq, g.d), dtype=torch.bfloat16, device="cuda")
    bits = torch.zeros((64 * g.Hq, (n // 4 + 31) // 32), dtype=torch.int32, device="cuda")
    out = torch.zeros((64, g.Hq, g.d), dtype=torch.float32, device="cuda")
    with pytest.raises(zha.ZhaError) as ei:
        # 64 query tokens over 1M tokens need far more than the static array holds
        zha.zha_sparse_attn_static(K.data_ptr(), K.data_ptr(), n, n, 4, 6, g.Hq, g.Hkv, g.d, Q.data_ptr(), 64,
                                   bits.data_ptr(), bits.shape[1], out.data_ptr(), 0)
    assert ei.value.status == zha.ZHA_ERR_CAPACITY
    assert "bytes" in zha.lib().zha_last_error().decode()


def _static(K, V, n, g, Q, n_q, bits, words):
    out = torch.full((1, n_q, g.Hq, g.d), float("nan"), dtype=torch.float32, device="cuda")
    zha.zha_sparse_attn_static(K.data_ptr(), V.data_ptr(), K.shape[1], n, g.C, g.L, g.Hq, g.Hkv, g.d,
                               Q.data_ptr(), n_q, bits.data_ptr(), words, out.data_ptr(),
                               torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return out


def _oracle(seq, n, Q, bits_bool):
    """The oracle's attention of every lane over the attended set its level-1 bits give."""
    g = seq.geom
    q, lane_g, ids = TL.lanes_for(seq, Q[0].cpu(), range(Q.shape[1]))
    toks = [O.attended_set(bits_bool[x], n, g.C, g.L) for x in range(len(ids))]
    return O.attend_batch(TL.f64(seq.K), TL.f64(seq.V), q, lane_g, toks)


@needs_cuda
@pytest.mark.parametrize("geom,n,n_q", [
    (inputs.Geometry(C=4, L=4, R=16, d=64, Hq=16, Hkv=2), 9 * 256 + 130, 2),   # d = 64
    (inputs.DEEP, 3000, 2),                                                  # no complete top node
])
def test_static_attention_d64_and_without_top_nodes(geom, n, n_q):
    seq = inputs.make_sequence(geom, n, n, seed=13)
    K, V, qr = seq.K.cuda(), seq.V.cuda(), seq.qref.cuda()
    Q, _ = inputs.make_queries(seq, n_q, 8, n, np.random.default_rng(2))
    Q = Q[None].cuda().contiguous()
    tree = zha.Tree(geom.C, geom.L, geom.R, geom.d, geom.Hq, geom.Hkv, n)
    tree.build(K, n, qr)
    dec = zha.Decoder([tree], n_q)
    for _ in range(2):                                   # two calls in a row
        ref = dec.decode([K], [V], Q, 0.9)
        bits, _ = dec.export_kept(1)
        out = _static(K, V, n, geom, Q, n_q, bits, bits.shape[1])
        assert torch.isfinite(out).all()
        assert _rel(out, ref) <= OUT_TOL
        o = _oracle(seq, n, Q, TL.bits_to_bool(bits, n // geom.C))
        assert TL.rel_err(out.cpu().numpy().astype(np.float64).reshape(-1, geom.d), o).max() <= OUT_TOL
    dec.close()
    tree.close()


@needs_cuda
def test_static_attention_ignores_bits_outside_routed_chunks():
    """A caller's bitmap may hold more words per lane than the chunks need, and bits for
    chunks under the dense tail or past the last complete chunk: none of them changes the
    attended set (the tail is attended whole; there are no rows past n_tokens)."""
    g = inputs.DEEP
    n = 4 * 4096 + 777 + 2                               # T = 4 top nodes; tail 779 tokens
    seq = inputs.make_sequence(g, n, n, seed=78)
    K, V, qr = seq.K.cuda(), seq.V.cuda(), seq.qref.cuda()
    Q, _ = inputs.make_queries(seq, 2, 8, n, np.random.default_rng(6))
    Q = Q[None].cuda().contiguous()
    tree = zha.Tree(g.C, g.L, g.R, g.d, g.Hq, g.Hkv, n)
    tree.build(K, n, qr)
    dec = zha.Decoder([tree], 2)
    ref = dec.decode([K], [V], Q, 0.9)
    bits, _ = dec.export_kept(1)
    n1 = n // g.C                                        # 4,290 complete chunks
    first_tail = 4 * 4096 // g.C                         # 4,096: first chunk of the tail
    words = (n1 + 31) // 32                              # 135: the last word holds chunks 4,288..4,319
    wide = torch.full((bits.shape[0], words + 5), -1, dtype=torch.int32, device="cuda")   # ones past `words`
    wide[:, :bits.shape[1]] = bits
    wide[:, bits.shape[1]:words] = 0
    dirty = wide.clone()
    dirty[:, first_tail // 32] |= 1 << 7                 # a tail chunk (4,103)
    dirty[:, words - 1] = -1                             # every chunk of the last word, past n1 too
    clean = _static(K, V, n, g, Q, 2, wide, words + 5)
    stray = _static(K, V, n, g, Q, 2, dirty, words + 5)
    assert torch.equal(clean, stray)
    assert _rel(clean, ref) <= OUT_TOL
    o = _oracle(seq, n, Q, TL.bits_to_bool(bits, n1))
    assert TL.rel_err(stray.cpu().numpy().astype(np.float64).reshape(-1, g.d), o).max() <= OUT_TOL
    dec.close()
    tree.close()
