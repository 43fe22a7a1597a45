"""Trees whose node records store the slopes m_r as one bf16 plane (ZHA_SUMMARY_BF16): half
the bytes per scored node and one tensor-core pass, the reduced-precision router the pages
report testing next to the full one (wqu.guru, summary bullets).

* Summaries: every level-1 slope is the bf16 rounding (to nearest even) of the oracle's exact
  slope, up to one bf16 unit where the exact value sits at a rounding boundary (and the
  float32 computation's absolute error for slopes near zero); every level is
  within 2^-7 of the exact slopes; lse keeps the float32 bar; b is computed from the stored
  slopes (b = lse - s q_r.m_r exactly as stored).
* Routing: replayed in float64 on the tree's own stored summaries (plane estimates from the
  exported m and b, the oracle's top-p cut), every kept set must match, up to logged
  near-ties.  Against the float64 oracle on exact summaries, the rate of identical kept sets is
  measured and reported.
* Outputs: exact attention over the GPU's own attended sets, within 2e-3 of the oracle.
"""
import math

import numpy as np
import pytest
import torch

from hierarchical_tree_indexed_build_b200 import inputs, zha
from oracle import oracle as O
import zha_testlib as TL

pytestmark = pytest.mark.gpu
needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")

BF16_REL = 2.0 ** -7     # bound on |m - m*|_inf / |m*|_inf at any level (rounding 2^-9 per level)


def _bf16_round(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()


def _bf16_ulp(x: np.ndarray) -> np.ndarray:
    e = np.floor(np.log2(np.maximum(np.abs(x), 1e-30)))
    return 2.0 ** (e - 7)


def _tree(seq, fmt=zha.ZHA_SUMMARY_BF16, n=None):
    g = seq.geom
    K, V, qr = seq.K.cuda(), seq.V.cuda(), seq.qref.cuda()
    t = zha.Tree(g.C, g.L, g.R, g.d, g.Hq, g.Hkv, seq.capacity, fmt)
    t.build(K, seq.n_tokens if n is None else n, qr)
    return t, K, V, qr


@needs_cuda
@pytest.mark.parametrize("geom,n", [(inputs.DEEP, 3 * 4096 + 1234), (inputs.MID, 2 * 4096 + 700),
                                    (inputs.TINY, 4096 + 77)])
def test_bf16_summaries_are_rounded_exact_summaries(geom, n):
    seq = inputs.make_sequence(geom, n, n, seed=11)
    tree, K, V, qr = _tree(seq)
    Kf, qf = TL.f64(seq.K), TL.f64(seq.qref)
    s = 1 / math.sqrt(geom.d)
    for lev in range(1, geom.L + 1):
        span = geom.C ** lev
        nl = n // span
        if nl == 0:
            continue
        m, lse, b = [x.cpu().numpy().astype(np.float64) for x in tree.export(lev)]
        nodes = np.arange(nl) if nl <= 96 else np.sort(np.random.default_rng(lev).choice(nl, 96, replace=False))
        for h in range(geom.Hkv):
            mo, lo, bo = O.summaries(Kf[h, :n], qf[h], span, nodes)
            mg = m[h, nodes]
            if lev == 1:
                # one bf16 unit where the float32 slope and the exact one round differently,
                # plus the float32 computation's absolute error (relative to the row's largest
                # slope), which exceeds a unit only for slopes near zero
                d = np.abs(mg - _bf16_round(mo))
                tol = _bf16_ulp(mo) * 1.0001 + 1e-5 * np.abs(mo).max(axis=2, keepdims=True)
                assert (d <= tol).all(), (d - tol).max()
                assert (d == 0).mean() >= 0.99
            em = (np.abs(mg - mo).max(axis=2) / np.abs(mo).max(axis=2)).max()
            assert em <= BF16_REL, (lev, em)
            el = (np.abs(lse[h, nodes] - lo) / np.maximum(1.0, np.abs(lo))).max()
            assert el <= TL.SUM_TOL, (lev, el)
            # b from the stored slopes: the plane passes through (q_r, lse_r)
            bb = lse[h, nodes] - s * np.einsum("nrd,rd->nr", mg, qf[h])
            eb = np.abs(b[h, nodes] - bb) / np.maximum(1.0, np.abs(bb))
            assert eb.max() <= 1e-5, (lev, eb.max())
    tree.close()


@needs_cuda
@pytest.mark.parametrize("score,geom,n,n_q", [
    (zha.ZHA_KERNELS_TENSOR, inputs.DEEP, 8 * 4096 + 333, 8),   # 64 lanes per group: tcgen05, one bf16 pass
    (zha.ZHA_KERNELS_SIMT, inputs.DEEP, 8 * 4096 + 333, 8),     # CUDA-core scorer
    (zha.ZHA_KERNELS_SIMT, inputs.DEEP, 8 * 4096 + 333, 2),     # 16 lanes: the few-lane CUDA-core scorer
    (zha.ZHA_KERNELS_TENSOR, inputs.MID, 3 * 4096 + 900, 8),
])
def test_bf16_router_matches_replay_on_its_stored_summaries(score, geom, n, n_q):
    seq = inputs.make_sequence(geom, n, n, seed=41)
    Q, _ = inputs.make_queries(seq, n_q, 8, n, np.random.default_rng(7))
    tree, K, V, qr = _tree(seq)
    dec = zha.Decoder([tree], n_q)
    dec.set_kernels(score, zha.ZHA_KERNELS_AUTO)
    res = TL.gpu_decode([tree], [K], [V], Q[None], 0.9, dec=dec)
    assert res.stats.status == 0
    assert res.stats.node_bytes == geom.R * geom.d * 2 + geom.R * 4      # one bf16 plane + b
    qs = [0, n_q - 1]
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
    # outputs: exact attention over the GPU's own attended sets
    toks = [O.attended_set(gk[1][i], n, geom.C, geom.L) for i in range(len(ids))]
    o = O.attend_batch(TL.f64(seq.K), TL.f64(seq.V), q, lane_g, toks)
    e1 = TL.rel_err(res.out[0].reshape(-1, geom.d)[ids], o)
    assert e1.max() <= TL.OUT_TOL
    # against the float64 oracle on exact summaries: the rate of identical kept sets
    ro = O.route(TL.f64(seq.K), TL.f64(seq.qref), geom.C, geom.L, n, q, lane_g, 0.9,
                 forced=[gk[lev] for lev in range(1, geom.L + 1)])
    same = sum(int(np.array_equal(ro.kept[v][x], gk[v + 1][x])) for v in range(geom.L) for x in range(len(ids)))
    total = geom.L * len(ids)
    print("[bf16 %s score=%d] replay on stored summaries: %d exact, %d near-ties of %d; kept sets equal "
          "to the exact-summary oracle's on %d of %d lane-levels (%.1f%%); out/own max %.2e"
          % (geom, score, exact, ties, len(rep), same, total, 100.0 * same / total, e1.max()))
    TL.TIE_LOG.append(("bf16 %s score=%d vs stored" % ("C%dL%d" % (geom.C, geom.L), score), len(rep), exact,
                       0, ties, float(e1.max()), float("nan")))
    TL.NOTES.append("bf16 router C%dL%d score=%d: kept sets equal to the exact-summary float64 oracle's on "
                    "%d of %d lane-levels (%.1f%%)" % (geom.C, geom.L, score, same, total, 100.0 * same / total))
    assert same >= 0.5 * total
    dec.close()
    tree.close()


@needs_cuda
def test_bf16_and_two_plane_trees_route_alike_on_the_64k_workload():
    """The same 64K workload (8 query tokens x 16 heads, p = 0.95) routed through a two-plane
    tree and a bf16 tree.  Measured and reported: the (lane, level) decisions that agree, the
    share of the float32-grade router's attended tokens that the bf16 router also attends
    (recall), and the difference of the two decodes' outputs."""
    wl = inputs.deep_64k(n_q=8)
    seq = wl.seqs[0]
    g = seq.geom
    full, K, V, qr = _tree(seq, zha.ZHA_SUMMARY_F16X2)
    half, _, _, _ = _tree(seq, zha.ZHA_SUMMARY_BF16)
    a = TL.gpu_decode([full], [K], [V], wl.Q[0], 0.95)
    b = TL.gpu_decode([half], [K], [V], wl.Q[0], 0.95)
    lanes = a.kept[0][0].shape[0]
    agree = sum(int((~(x != y).any(axis=1)).sum()) for x, y in zip(a.kept[0], b.kept[0]))
    n = seq.n_tokens
    recall = []
    for x in range(lanes):
        ta = O.attended_set(a.kept[0][0][x], n, g.C, g.L)
        tb = O.attended_set(b.kept[0][0][x], n, g.C, g.L)
        recall.append(np.intersect1d(ta, tb).size / ta.size)
    e = TL.rel_err(b.out[0].reshape(-1, g.d), a.out[0].reshape(-1, g.d))
    line = ("bf16 vs two-plane router, 64K, p = 0.95: %d of %d (lane, level) decisions identical; attended-token "
            "recall min %.4f mean %.4f; output difference max %.2e median %.2e"
            % (agree, lanes * g.L, min(recall), float(np.mean(recall)), e.max(), float(np.median(e))))
    print(line)
    TL.NOTES.append(line)
    # the bf16 router attends at least 95 % of the tokens the float32-grade router attends, for
    # every lane; the outputs' max-relative difference is reported, not bounded: with attention
    # spread over half the cache an output's largest entry is small, so a few chunks swapped at
    # a cut move that ratio far more than they move the attention
    assert min(recall) >= 0.95
    full.close()
    half.close()
