"""Full-size parity in the benchmark's launch configuration.

* The 1M-token deep tree (C4 L6, R16, GQA 16/2, d128) built over 1,048,576 tokens, grown by a
  4,096-token append, then decoded for all 128 queries in one batch at p = 0.95 with the
  default kernel choice: exactly the step the benchmark times.  Sampled summaries of every
  level, and every lane of two queries, are replayed by the oracle; so is one query's dense
  attention over the whole grown cache (the benchmark's dense comparison).
* The batched workload: 32 sequences x 131,072 tokens, half C16 L3 and half C4 L6, one
  appended token and one query per sequence per step; two steps, four sequences compared.
"""
import numpy as np
import pytest
import torch

from hierarchical_tree_indexed_build_b200 import inputs, zha
from oracle import oracle as O
import zha_testlib as TL

pytestmark = pytest.mark.gpu

needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def _report(name, rep, e1, e2):
    TL.record(name, rep, e1, e2)


@needs_cuda
def test_full_size_deep1m_benchmark_step():
    wl = inputs.deep_1m()
    seq = wl.seqs[0]
    g = seq.geom
    n0, n_app = seq.n_tokens, wl.n_append
    K, V, qr = seq.K.cuda(), seq.V.cuda(), seq.qref.cuda()
    tree = zha.Tree(g.C, g.L, g.R, g.d, g.Hq, g.Hkv, seq.capacity)
    tree.build(K, n0, qr)
    tree.append(K, n0, n_app)
    n = n0 + n_app
    w = TL.compare_summaries(tree, seq, n, sample=48)
    print("[deep1m summaries] worst normalised errors %r" % w)
    assert max(w.values()) <= TL.SUM_TOL
    Q = wl.Q[0]                                   # [1][128][16][128]
    res = TL.gpu_decode([tree], [K], [V], Q, 0.95)
    assert res.stats.status == 0
    rep, e1, e2, _ = TL.check_decode(seq, n, Q[0], 0.95, res.out[0], res.kept[0], [0, 77])
    _report("deep1m full batch", rep, e1, e2)
    # the dense baseline of the same batch over the whole grown cache, one query's lanes
    # replayed by the oracle over all n tokens
    dec = zha.Decoder([tree], Q.shape[1])
    dense = dec.dense_attn([K], [V], Q.cuda().contiguous())
    torch.cuda.synchronize()
    q, lane_g, ids = TL.lanes_for(seq, Q[0], [5])
    o = O.attend_batch(TL.f64(seq.K), TL.f64(seq.V), q, lane_g, [np.arange(n)] * len(ids))
    e = TL.rel_err(dense.cpu().numpy().astype(np.float64).reshape(-1, g.d)[ids], o)
    print("[deep1m dense] max rel err %.2e" % e.max())
    assert e.max() <= TL.OUT_TOL
    dec.close()
    tree.close()


@needs_cuda
def test_full_size_batched_32x128k():
    wl = inputs.batched_32x128k(n_steps=2)
    trees, Ks, Vs = [], [], []
    for sq in wl.seqs:
        t, K, V, _ = TL.make_tree(sq, sq.n_tokens)
        trees.append(t)
        Ks.append(K)
        Vs.append(V)
    dec = zha.Decoder(trees, 1)
    for step in range(2):
        for s, sq in enumerate(wl.seqs):
            trees[s].append(Ks[s], sq.n_tokens + step, 1)
        res = TL.gpu_decode(trees, Ks, Vs, wl.Q[step], 0.95, dec=dec)
        for s in (0, 15, 16, 31):
            sq = wl.seqs[s]
            rep, e1, e2, _ = TL.check_decode(sq, sq.n_tokens + step + 1, wl.Q[step][s], 0.95, res.out[s],
                                             res.kept[s], [0])
            _report("batched step %d seq %d" % (step, s), rep, e1, e2)
    dec.close()
    for t in trees:
        t.close()
