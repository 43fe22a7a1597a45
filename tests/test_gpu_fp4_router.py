"""Trees whose node records store the slopes m_r as MXFP4 (ZHA_SUMMARY_FP4): E2M1 codes with
one E8M0 scale per 32 dims, about 1/7 of the two-plane bytes per scored node - the FP4 router
variant the pages report testing (wqu.guru, summary bullets).

* Summaries: level-1 slopes are the oracle's MXFP4 rounding (O.mxfp4, pinned in
  test_oracle_pins) of the exact slopes, where the float32 slope and the exact one fall on
  the same side of every rounding boundary (>= 99% of the values; the rest within the
  rounding's own error bound); every higher level is the MXFP4 rounding of the online-softmax
  merge of its stored (decoded) children, replayed in float64 from the exported children; lse
  keeps the float32 bar; b is computed from the stored slopes.
* Appends: a tree grown by appends is bit-identical to one built in one pass.
* Routing: replayed in float64 on the tree's own stored summaries, every kept set matches up
  to logged near-ties; outputs are exact attention over the GPU's attended sets.  The recall
  of the float32-grade router's attended tokens is measured and reported.
"""
import math

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

from hierarchical_tree_indexed_build_b200 import inputs, zha
from oracle import oracle as O
import zha_testlib as TL

pytestmark = pytest.mark.gpu
needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def _tree(seq, fmt=zha.ZHA_SUMMARY_FP4, n=None):
    g = seq.geom
    K, V, qr = seq.K.cuda(), seq.V.cuda(), seq.qref.cuda()
    t = zha.Tree(g.C, g.L, g.R, g.d, g.Hq, g.Hkv, seq.capacity, fmt)
    t.build(K, seq.n_tokens if n is None else n, qr)
    return t, K, V, qr


def _block_scale(v):
    """The oracle's MXFP4 scale of each 32-value block, broadcast over the block."""
    _, _, E = O.mxfp4(v)
    X = np.ldexp(1.0, E.astype(np.int64) - 127)
    return np.repeat(X, 32, axis=-1)


def _check_rounded(mg, target, what):
    """Stored slopes vs the MXFP4 rounding of a float64 target: equal for >= 99% of the values,
    everywhere within 4 X of the target (the rounding error is at most 2 X, saturation
    included, and a block whose float32 maximum crosses a power of two takes the next scale)."""
    v, _, _ = O.mxfp4(target)
    eq = (mg == v).mean()
    X = _block_scale(target)
    err = np.abs(mg - target) / X
    assert eq >= 0.99, (what, eq)
    assert err.max() <= 4.0, (what, err.max())
    return eq


@needs_cuda
@pytest.mark.parametrize("geom,n", [(inputs.DEEP, 3 * 4096 + 1234), (inputs.MID, 2 * 4096 + 700),
                                    (inputs.TINY, 4096 + 77)])
def test_fp4_summaries_are_mxfp4_of_the_exact_and_merged_slopes(geom, n):
    seq = inputs.make_sequence(geom, n, n, seed=12)
    tree, K, V, qr = _tree(seq)
    Kf, qf = TL.f64(seq.K), TL.f64(seq.qref)
    s = 1 / math.sqrt(geom.d)
    exp = {lev: [x.cpu().numpy().astype(np.float64) for x in tree.export(lev)] for lev in range(1, geom.L + 1)}
    eqs = []
    for lev in range(1, geom.L + 1):
        span = geom.C ** lev
        nl = n // span
        if nl == 0:
            continue
        m, lse, b = exp[lev]
        nodes = np.arange(nl) if nl <= 96 else np.sort(np.random.default_rng(lev).choice(nl, 96, replace=False))
        for h in range(geom.Hkv):
            mo, lo, bo = O.summaries(Kf[h, :n], qf[h], span, nodes)
            mg = m[h, nodes]
            if lev == 1:
                eqs.append(_check_rounded(mg, mo, "level 1"))
            else:
                # the merge of the stored children, in float64, then MXFP4
                cm, cl, _ = exp[lev - 1]
                ch = nodes[:, None] * geom.C + np.arange(geom.C)[None, :]
                lp = logsumexp(cl[h, ch], axis=1)                        # [nodes][R]
                w = np.exp(cl[h, ch] - lp[:, None, :])                   # [nodes][C][R]
                target = np.einsum("ncr,ncrd->nrd", w, cm[h, ch])
                eqs.append(_check_rounded(mg, target, "level %d" % lev))
            el = (np.abs(lse[h, nodes] - lo) / np.maximum(1.0, np.abs(lo))).max()
            assert el <= TL.SUM_TOL, (lev, el)
            bb = lse[h, nodes] - s * np.einsum("nrd,rd->nr", mg, qf[h])
            eb = np.abs(b[h, nodes] - bb) / np.maximum(1.0, np.abs(bb))
            assert eb.max() <= 1e-5, (lev, eb.max())
    TL.NOTES.append("fp4 summaries C%dL%d: stored slopes equal to the float64 MXFP4 rounding on %.4f of the "
                    "values (worst level)" % (geom.C, geom.L, min(eqs)))
    tree.close()


@needs_cuda
def test_fp4_append_is_bit_identical_to_rebuild():
    geom = inputs.DEEP
    n0, n1 = 2 * 4096 + 500, 3 * 4096 + 77
    seq = inputs.make_sequence(geom, n1, n1, seed=13)
    a, K, _, qr = _tree(seq, n=n0)
    a.append(K, n0, n1 - n0)
    b, _, _, _ = _tree(seq, n=n1)
    for lev in range(1, geom.L + 1):
        if n1 // geom.C ** lev == 0:
            continue
        for x, y in zip(a.export(lev), b.export(lev)):
            assert torch.equal(x, y), lev
    a.close()
    b.close()


@needs_cuda
@pytest.mark.parametrize("geom,n,n_q", [(inputs.DEEP, 8 * 4096 + 333, 8),    # 64 lanes: k_score
                                        (inputs.DEEP, 8 * 4096 + 333, 1),    # 8 lanes: k_score_few
                                        (inputs.MID, 3 * 4096 + 900, 2),
                                        (inputs.TINY, 4096 + 77, 4)])       # d = 64, R = 4
def test_fp4_router_matches_replay_on_its_stored_summaries(geom, n, n_q):
    seq = inputs.make_sequence(geom, n, n, seed=42)
    Q, _ = inputs.make_queries(seq, n_q, 8, n, np.random.default_rng(7))
    tree, K, V, qr = _tree(seq)
    dec = zha.Decoder([tree], n_q)
    with pytest.raises(zha.ZhaError):
        dec.set_kernels(zha.ZHA_KERNELS_TENSOR, zha.ZHA_KERNELS_AUTO)
    res = TL.gpu_decode([tree], [K], [V], Q[None], 0.9, dec=dec)
    assert res.stats.status == 0
    assert res.stats.node_bytes == geom.R * geom.d // 2 + geom.R * geom.d // 32 + geom.R * 4
    qs = [0, n_q - 1] if n_q > 1 else [0]
    q, lane_g, ids = TL.lanes_for(seq, Q, qs)
    gk = {lev: res.kept[0][lev - 1][ids] for lev in range(1, geom.L + 1)}
    rep = TL.replay_on_stored(tree, seq, n, q, lane_g, 0.9, gk)
    exact = ties = 0
    for (lev, x), (row, info, sc) in rep.items():
        if np.array_equal(row, gk[lev][x]):
            exact += 1
            continue
        if min(info[0], info[1]) < TL.MASS_MARGIN:
            ties += 1
            continue
        diff = np.flatnonzero(row != gk[lev][x])
        e_last = np.nanmin(sc[row])
        assert np.all(np.abs(sc[diff] - e_last) <= 2 * TL.SCORE_TIE_REL * max(1.0, abs(e_last))), (lev, x)
        ties += 1
    assert ties <= max(TL.TIE_FLOOR, TL.TIE_RATE_MAX * len(rep))
    toks = [O.attended_set(gk[1][i], n, geom.C, geom.L) for i in range(len(ids))]
    o = O.attend_batch(TL.f64(seq.K), TL.f64(seq.V), q, lane_g, toks)
    e1 = TL.rel_err(res.out[0].reshape(-1, geom.d)[ids], o)
    assert e1.max() <= TL.OUT_TOL
    TL.TIE_LOG.append(("fp4 %s q=%d vs stored" % ("C%dL%d" % (geom.C, geom.L), n_q), len(rep), exact,
                       0, ties, float(e1.max()), float("nan")))
    dec.close()
    tree.close()


@needs_cuda
def test_fp4_and_two_plane_trees_route_alike_on_the_64k_workload():
    """The 64K workload (8 query tokens x 16 heads, p = 0.95) routed through a two-plane tree
    and an MXFP4 tree: the share of the float32-grade router's attended tokens the FP4 router
    also attends (recall) is measured and reported.  The pages give no accuracy figure for
    their FP4 router, so the only bound is that the rounded slopes still carry the routing:
    on every lane the recall exceeds, by at least 0.2, the recall of a choice of the same
    number of tokens at random (its attended fraction of the cache)."""
    wl = inputs.deep_64k(n_q=8)
    seq = wl.seqs[0]
    g = seq.geom
    full, K, V, qr = _tree(seq, zha.ZHA_SUMMARY_F16X2)
    four, _, _, _ = _tree(seq, zha.ZHA_SUMMARY_FP4)
    a = TL.gpu_decode([full], [K], [V], wl.Q[0], 0.95)
    b = TL.gpu_decode([four], [K], [V], wl.Q[0], 0.95)
    lanes = a.kept[0][0].shape[0]
    n = seq.n_tokens
    recall, size, chance = [], [], []
    for x in range(lanes):
        ta = O.attended_set(a.kept[0][0][x], n, g.C, g.L)
        tb = O.attended_set(b.kept[0][0][x], n, g.C, g.L)
        recall.append(np.intersect1d(ta, tb).size / ta.size)
        size.append(tb.size / ta.size)
        chance.append(tb.size / n)
    line = ("fp4 vs two-plane router, 64K, p = 0.95: attended-token recall min %.4f mean %.4f (a random choice "
            "of as many tokens: mean %.4f); attended tokens fp4 / two-plane mean %.3f"
            % (min(recall), float(np.mean(recall)), float(np.mean(chance)), float(np.mean(size))))
    print(line)
    TL.NOTES.append(line)
    assert min(r - c for r, c in zip(recall, chance)) >= 0.2
    full.close()
    four.close()
