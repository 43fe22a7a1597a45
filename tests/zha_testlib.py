"""Helpers for the GPU parity tests: run the CUDA path through the C ABI (via the ctypes
binding) and compare it with the float64 oracle on the same seeded inputs.

Comparison rules (tolerances from the method's parity contract):
* summaries: |lse - lse*| <= 1e-4 max(1, |lse*|) and |m - m*|_inf <= 1e-4 |m*|_inf per node
  and reference query; b within the error those two imply;
* kept sets: compared level by level in replay mode (the oracle cuts the frontier the GPU
  actually used).  A difference is accepted only as a logged near-tie:
    - mass tie: the oracle's cumulative mass at the cut is within 1e-5 of p
      (min(cum_k* - p, p - cum_{k*-1}) < 1e-5), or
    - score tie: every node in the symmetric difference has an oracle estimate within
      SCORE_TIE of the oracle's last kept estimate (a boundary swap caused by float32
      evaluation of nearly equal estimates);
  anything else fails;
* outputs: max_i |o_i - o*_i| / max_i |o*_i| <= 2e-3 per lane, against the oracle on the
  GPU's own attended set (every lane) and against the oracle end to end (lanes whose kept
  sets matched exactly at every level).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

from hierarchical_tree_indexed_build_b200 import zha
from oracle import oracle as O

SUM_TOL = 1e-4
OUT_TOL = 2e-3
MASS_MARGIN = 1e-5
SCORE_TIE_REL = 2e-5     # relative to max(1, |e|): float32 evaluation error of an estimate
# Logged near-ties may excuse at most this fraction of a check's (lane, level) decisions
# (and at least TIE_FLOOR of them): a higher rate would mean the excuse hides a real fault.
TIE_RATE_MAX = 0.05
TIE_FLOOR = 2

# Every parity check of the session: (name, lane-levels, exact, mass ties, score ties,
# max error vs the oracle on the GPU's set, max error end to end); printed as a table at
# the end of the run (tests/conftest.py), also under -q.
TIE_LOG: List[tuple] = []
# Free-form measured rates of the session, printed after that table.
NOTES: List[str] = []


def record(name: str, rep, e1, e2) -> str:
    """Log one parity check's decision and error counts; returns its one-line summary."""
    e1m = float(np.max(e1)) if np.size(e1) else float("nan")
    e2m = float(np.max(e2)) if np.size(e2) else float("nan")
    TIE_LOG.append((name, rep.levels, rep.exact, rep.mass_ties, rep.score_ties, e1m, e2m))
    line = ("[%s] levels=%d exact=%d mass_ties=%d score_ties=%d  out/own max=%.2e  out/e2e max=%s"
            % (name, rep.levels, rep.exact, rep.mass_ties, rep.score_ties, e1m,
               "%.2e" % e2m if np.size(e2) else "-"))
    print(line)
    return line


def f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).cpu().numpy()


def bits_to_bool(bits: torch.Tensor, n: int) -> np.ndarray:
    b = np.ascontiguousarray(bits.cpu().numpy()).view(np.uint8).reshape(bits.shape[0], -1)
    return np.unpackbits(b, axis=1, bitorder="little")[:, :n].astype(bool)


def make_tree(seq, n_tokens: Optional[int] = None):
    """Tree over a generated sequence; returns (Tree, K_dev, V_dev, qref_dev)."""
    g = seq.geom
    K = seq.K.cuda()
    V = seq.V.cuda()
    qr = seq.qref.cuda()
    t = zha.Tree(g.C, g.L, g.R, g.d, g.Hq, g.Hkv, seq.capacity)
    t.build(K, seq.n_tokens if n_tokens is None else n_tokens, qr)
    return t, K, V, qr


@dataclass
class GpuDecode:
    out: np.ndarray                      # [n_seq][n_q][Hq][d]
    kept: List[List[np.ndarray]]         # [seq][level-1] bool [n_q*Hq][n_l]
    counts: List[List[np.ndarray]]
    stats: object


def gpu_decode(trees, Ks, Vs, Q: torch.Tensor, p: float, dec: Optional[zha.Decoder] = None) -> GpuDecode:
    """Q bf16 [n_seq][n_q][Hq][d] (CPU or GPU)."""
    Qd = Q.cuda().contiguous()
    own = dec is None
    if own:
        dec = zha.Decoder(trees, Qd.shape[1])
    out = dec.decode(Ks, Vs, Qd, p)
    torch.cuda.synchronize()
    n_seq, n_q, Hq = Qd.shape[0], Qd.shape[1], Qd.shape[2]
    per = n_q * Hq
    Lmax = max(t.geom.L for t in trees)
    kept = [[None] * t.geom.L for t in trees]
    counts = [[None] * t.geom.L for t in trees]
    for lev in range(1, Lmax + 1):
        bits, cnt = dec.export_kept(lev)
        for s, t in enumerate(trees):
            if lev <= t.geom.L:
                n_l = t.level_nodes()[lev - 1]
                kept[s][lev - 1] = bits_to_bool(bits[s * per:(s + 1) * per], n_l)
                counts[s][lev - 1] = cnt[s * per:(s + 1) * per].cpu().numpy()
    st = dec.stats()
    res = GpuDecode(out.cpu().numpy().astype(np.float64), kept, counts, st)
    if own:
        dec.close()
    return res


def compare_summaries(tree: zha.Tree, seq, n_tokens: int, levels=None, sample: Optional[int] = None,
                      seed: int = 0) -> Dict[str, float]:
    """Tree export vs oracle summaries by definition.  Returns the worst normalised errors."""
    g = seq.geom
    K = f64(seq.K)
    qref = f64(seq.qref)
    worst = {"lse": 0.0, "m": 0.0, "b": 0.0}
    rng = np.random.default_rng(seed)
    for lev in (levels or range(1, g.L + 1)):
        span = g.C ** lev
        n_l = n_tokens // span
        if n_l == 0:
            continue
        m, lse, b = tree.export(lev)
        m, lse, b = m.cpu().numpy(), lse.cpu().numpy(), b.cpu().numpy()
        nodes = np.arange(n_l) if sample is None or sample >= n_l else np.sort(
            np.concatenate([[0, n_l - 1], rng.choice(n_l, sample, replace=False)]))
        for h in range(g.Hkv):
            mo, lo, bo = O.summaries(K[h, :n_tokens], qref[h], span, nodes)
            el = np.abs(lse[h, nodes] - lo) / np.maximum(1.0, np.abs(lo))
            em = np.abs(m[h, nodes] - mo).max(axis=2) / np.abs(mo).max(axis=2)
            # b = lse - s q_r.m_r: its error is bounded by the lse error plus s |q_r|_1 |dm|_inf
            s = 1 / np.sqrt(g.d)
            bbound = SUM_TOL * np.maximum(1.0, np.abs(lo)) + s * np.abs(qref[h]).sum(axis=1)[None, :] * \
                SUM_TOL * np.abs(mo).max(axis=2)
            eb = np.abs(b[h, nodes] - bo) / bbound
            worst["lse"] = max(worst["lse"], float(el.max()))
            worst["m"] = max(worst["m"], float(em.max()))
            worst["b"] = max(worst["b"], float(eb.max()) * SUM_TOL)
    return worst


@dataclass
class RouteReport:
    levels: int = 0
    exact: int = 0
    mass_ties: int = 0
    score_ties: int = 0
    failures: List[tuple] = field(default_factory=list)
    lane_exact: Optional[np.ndarray] = None   # lanes whose kept sets matched at every level


def compare_routing(seq, n_tokens: int, q: np.ndarray, lane_g: np.ndarray, p: float,
                    gpu_kept: List[np.ndarray]) -> (RouteReport, O.Route):
    """Oracle replay on the GPU's frontiers; classify every (level, lane) decision."""
    g = seq.geom
    K = f64(seq.K)
    qref = f64(seq.qref)
    r = O.route(K, qref, g.C, g.L, n_tokens, q, lane_g, p, forced=gpu_kept, return_scores=True)
    rep = RouteReport()
    n_lanes = q.shape[0]
    rep.lane_exact = np.ones(n_lanes, dtype=bool)
    for v in range(g.L):
        if r.kept[v].shape[1] == 0:
            continue
        for x in range(n_lanes):
            rep.levels += 1
            own, gk = r.kept[v][x], gpu_kept[v][x]
            if np.array_equal(own, gk):
                rep.exact += 1
                continue
            rep.lane_exact[x] = False
            info = r.info[v, x]
            if min(info[0], info[1]) < MASS_MARGIN:
                rep.mass_ties += 1
                continue
            diff = np.flatnonzero(own != gk)
            sc = r.scores[v][x]
            kept_sc = sc[own]
            e_last = kept_sc.min()
            tol = SCORE_TIE_REL * max(1.0, abs(e_last))
            if np.all(np.abs(sc[diff] - e_last) <= 2 * tol):
                rep.score_ties += 1
                continue
            rep.failures.append((v + 1, x, diff[:8].tolist(), sc[diff[:8]].tolist(), e_last, info.tolist()))
    return rep, r


def rel_err(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """max_i |a_i - b_i| / max_i |b_i| over the last axis."""
    return np.abs(a - b).max(axis=-1) / np.abs(b).max(axis=-1)


def lanes_for(seq, Q_seq: torch.Tensor, queries: Sequence[int]):
    """Oracle lanes (query i, head h) for the given queries of one sequence.
    Returns q [n][d] float64, lane_g [n] int32, and the GPU lane indices within the
    sequence (i*Hq + h)."""
    g = seq.geom
    Qf = f64(Q_seq)              # [n_q][Hq][d]
    qs, gs, ids = [], [], []
    for i in queries:
        for h in range(g.Hq):
            qs.append(Qf[i, h])
            gs.append(h * g.Hkv // g.Hq)
            ids.append(i * g.Hq + h)
    return np.array(qs), np.array(gs, dtype=np.int32), np.array(ids)


def check_decode(seq, n_tokens: int, Q_seq: torch.Tensor, p: float, res_out: np.ndarray,
                 res_kept: List[np.ndarray], queries: Sequence[int], end_to_end: bool = True):
    """Full parity check of one sequence's decode on a subset of queries.

    res_out [n_q][Hq][d] (GPU), res_kept per level bool [n_q*Hq][n_l] (GPU)."""
    g = seq.geom
    q, lane_g, ids = lanes_for(seq, Q_seq, queries)
    gk = [k[ids] for k in res_kept]
    rep, r = compare_routing(seq, n_tokens, q, lane_g, p, gk)
    assert not rep.failures, "unexplained kept-set differences: %r" % rep.failures[:5]
    ties = rep.mass_ties + rep.score_ties
    assert ties <= max(TIE_FLOOR, TIE_RATE_MAX * rep.levels), \
        "near-ties excuse %d of %d lane-levels" % (ties, rep.levels)
    K = f64(seq.K)
    V = f64(seq.V)
    gpu = res_out.reshape(-1, g.d)[ids]
    # (1) oracle attention over the GPU's own attended set
    toks = [O.attended_set(gk[0][x], n_tokens, g.C, g.L) for x in range(len(ids))]
    o_own = O.attend_batch(K, V, q, lane_g, toks)
    e1 = rel_err(gpu, o_own)
    assert e1.max() <= OUT_TOL, "output vs oracle on GPU's set: %g" % e1.max()
    e2 = np.zeros(0)
    if end_to_end:
        # (2) end to end, for lanes whose kept sets matched at every level
        r2, o_e2e, _ = O.decode(K, V, f64(seq.qref), g.C, g.L, n_tokens, q, lane_g, p)
        ok = rep.lane_exact
        if ok.any():
            e2 = rel_err(gpu[ok], o_e2e[ok])
            assert e2.max() <= OUT_TOL, "output vs end-to-end oracle: %g" % e2.max()
    return rep, e1, e2, toks


def replay_on_stored(tree, seq, n, q, lane_g, p, gk):
    """Float64 replay of the routing on the tree's stored summaries: at every level the
    frontier is the children of the GPU's kept set one level up; each frontier node's
    estimate max_r (s q.m_r + b_r) is taken from the exported record; the cut is the
    oracle's.  Returns per-(level, lane) (oracle kept bool row, info, estimates)."""
    g = seq.geom
    exp = {lev: [x.cpu().numpy().astype(np.float64) for x in tree.export(lev)] for lev in range(1, g.L + 1)}
    out = {}
    for lev in range(g.L, 0, -1):
        m, _, b = exp[lev]
        nl = n // g.C ** lev
        for x in range(q.shape[0]):
            h = lane_g[x]
            if lev == g.L:
                front = np.arange(nl)
            else:
                par = np.flatnonzero(gk[lev + 1][x])
                front = (par[:, None] * g.C + np.arange(g.C)[None, :]).ravel()
                front = front[front < nl]
            est = np.array([O.plane_estimate(m[h, j], b[h, j], q[x]) for j in front])
            keep, k, info = O.topp(est, front, p)
            row = np.zeros(nl, dtype=bool)
            row[front[keep]] = True
            sc = np.full(nl, np.nan)
            sc[front] = est
            out[(lev, x)] = (row, info, sc)
    return out
