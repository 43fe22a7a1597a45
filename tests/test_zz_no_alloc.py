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
