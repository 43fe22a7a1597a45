"""Pins of the float64 oracle against what the pages and the mathematics fix.

None of these re-types the oracle's own formulas: they use closed forms worked by
hand, library routines (scipy logsumexp / softmax, torch SDPA), mathematical
identities (gradient of log-sum-exp, convexity, merge of disjoint sets), brute force
over all subsets, and the numbers the pages print (tests/golden/page_facts.json).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp, softmax

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")


def _lse_direct(K, q):
    """log sum_t exp(q.k_t / sqrt(d)) via scipy."""
    return float(logsumexp(K @ q / math.sqrt(K.shape[1])))


# ----------------------------------------------------------------------------- summaries

def test_summary_closed_form_two_tokens():
    """Hand-worked node of 2 tokens, d = 4 (s = 1/2), two reference queries.

    q_1 = e_0 gives scores (ln 3, 0): weights 3/4, 1/4, lse = ln 4,
    m_1 = 3/4 k_1 + 1/4 k_2, b_1 = ln 4 - (1/2)(q_1 . m_1) = ln 4 - (3/4) ln 3.
    q_2 = 2 e_1 gives scores (1, 0): weights e/(e+1), 1/(e+1), lse = ln(e+1),
    b_2 = ln(e+1) - e/(e+1)."""
    l3 = math.log(3.0)
    K = np.array([[2 * l3, 1.0, 0.0, 0.0], [0.0, 0.0, 1.0, 0.0]])
    qref = np.array([[1.0, 0.0, 0.0, 0.0], [0.0, 2.0, 0.0, 0.0]])
    m, lse, b = O.summaries(K, qref, span=2)
    E = math.e
    assert lse[0, 0] == pytest.approx(math.log(4.0), abs=1e-14)
    assert lse[0, 1] == pytest.approx(math.log(E + 1), abs=1e-14)
    np.testing.assert_allclose(m[0, 0], [1.5 * l3, 0.75, 0.25, 0.0], atol=1e-14)
    w = E / (E + 1)
    np.testing.assert_allclose(m[0, 1], [w * 2 * l3, w, 1 - w, 0.0], atol=1e-14)
    assert b[0, 0] == pytest.approx(math.log(4.0) - 0.75 * l3, abs=1e-14)
    assert b[0, 1] == pytest.approx(math.log(E + 1) - w, abs=1e-14)
    # plane estimate at q = 2 e_2: plane 1 = 1/4 + b_1, plane 2 = 1/(e+1) + b_2; max is plane 2;
    # the true log mass there is ln(1 + e)
    q = np.array([0.0, 0.0, 2.0, 0.0])
    est = O.plane_estimate(m[0], b[0], q)
    assert est == pytest.approx(max(0.25 + b[0, 0], (1 - w) + b[0, 1]), abs=1e-14)
    assert est == pytest.approx((1 - E) / (E + 1) + math.log(E + 1), abs=1e-14)
    assert est <= math.log(1 + E)


@pytest.mark.parametrize("span,R,d", [(1, 1, 8), (7, 3, 16), (64, 4, 64)])
def test_summary_matches_scipy(span, R, d):
    rng = np.random.default_rng(span * 100 + R)
    N = span * 5
    K = rng.standard_normal((N, d)) + 0.3
    qref = rng.standard_normal((R, d))
    m, lse, b = O.summaries(K, qref, span)
    s = 1 / math.sqrt(d)
    for i in range(N // span):
        Kc = K[i * span:(i + 1) * span]
        a = s * Kc @ qref.T                      # [span][R]
        np.testing.assert_allclose(lse[i], logsumexp(a, axis=0), rtol=0, atol=1e-12)
        w = softmax(a, axis=0)                   # [span][R]
        np.testing.assert_allclose(m[i], w.T @ Kc, rtol=0, atol=1e-12)
        np.testing.assert_allclose(b[i], lse[i] - s * np.sum(qref * m[i], axis=1), atol=1e-12)


def test_slope_is_gradient_of_log_mass():
    """The tangent plane at q_r has slope s*m_r = grad_q log sum_t exp(s q.k_t) at q_r.
    Checked by central differences of scipy's logsumexp (catches a transposed m, wrong
    weights or a wrong scale)."""
    rng = np.random.default_rng(7)
    d, R, span = 16, 3, 40
    K = rng.standard_normal((span, d))
    qref = rng.standard_normal((R, d))
    m, lse, b = O.summaries(K, qref, span)
    h = 1e-5
    s = 1 / math.sqrt(d)
    for r in range(R):
        grad = np.empty(d)
        for i in range(d):
            e = np.zeros(d); e[i] = h
            grad[i] = (_lse_direct(K, qref[r] + e) - _lse_direct(K, qref[r] - e)) / (2 * h)
        np.testing.assert_allclose(s * m[0, r], grad, atol=1e-8)
        assert lse[0, r] == pytest.approx(_lse_direct(K, qref[r]), abs=1e-12)


def test_plane_is_lower_bound_and_touches_at_reference():
    """Convexity: every tangent plane of a convex log-sum-exp lies below it, so the
    max-over-planes estimate never exceeds the node's true log mass; it is exact at q_r."""
    rng = np.random.default_rng(11)
    d, R, span = 32, 5, 50
    K = rng.standard_normal((span * 3, d)) + 0.2
    qref = rng.standard_normal((R, d))
    m, lse, b = O.summaries(K, qref, span)
    for i in range(3):
        Kc = K[i * span:(i + 1) * span]
        for _ in range(40):
            q = rng.standard_normal(d) * rng.uniform(0.1, 4.0)
            est = O.plane_estimate(m[i], b[i], q)
            assert est <= _lse_direct(Kc, q) + 1e-12
            assert est <= O.true_log_mass(Kc, 0, span, q) + 1e-12
        for r in range(R):
            est = O.plane_estimate(m[i], b[i], qref[r])
            assert est == pytest.approx(_lse_direct(Kc, qref[r]), abs=1e-12)


@pytest.mark.parametrize("C", [2, 4, 16])
def test_parent_summary_is_merge_of_children(C):
    """A parent's summary (by definition over its C*span tokens) equals the online-softmax
    merge of its children's summaries: lse_P = log sum_c exp(lse_c),
    m_P = sum_c exp(lse_c - lse_P) m_c.  Identity of log-sum-exp over a disjoint union."""
    rng = np.random.default_rng(C)
    d, R, span = 16, 4, 3
    K = rng.standard_normal((C * span * 2, d))
    qref = rng.standard_normal((R, d))
    mc, lc, bc = O.summaries(K, qref, span)
    mp, lp, bp = O.summaries(K, qref, span * C)
    s = 1 / math.sqrt(d)
    for P in range(2):
        ch = slice(P * C, (P + 1) * C)
        lse_m = logsumexp(lc[ch], axis=0)
        np.testing.assert_allclose(lp[P], lse_m, atol=1e-12)
        w = np.exp(lc[ch] - lse_m)                     # [C][R]
        np.testing.assert_allclose(mp[P], np.einsum("cr,crd->rd", w, mc[ch]), atol=1e-12)
        np.testing.assert_allclose(bp[P], lp[P] - s * np.sum(qref * mp[P], axis=1), atol=1e-12)


def test_top_node_covers_page_span():
    """The pages print: chunk size 4 and 6 levels give 4096 tokens per top node (and the
    wide tree 256).  The oracle's top-level summary must be the log mass of exactly those
    tokens, not one more or one less."""
    facts = json.load(open(GOLDEN))["top_node_coverage"]
    rng = np.random.default_rng(5)
    d = 8
    for f in facts:
        C, L, cover = f["C"], f["L"], f["tokens_per_top_node"]
        assert C ** L == cover
        K = rng.standard_normal((2 * cover + 3, d))
        qref = rng.standard_normal((1, d))
        m, lse, b = O.summaries(K, qref, C ** L, nodes=[1])
        assert lse[0, 0] == pytest.approx(_lse_direct(K[cover:2 * cover], qref[0]), abs=1e-11)
        assert abs(lse[0, 0] - _lse_direct(K[cover:2 * cover + 1], qref[0])) > 1e-6
        assert abs(lse[0, 0] - _lse_direct(K[cover + 1:2 * cover], qref[0])) > 1e-6
        assert O.level_sizes(2 * cover + 3, C, L)[-1] == 2


# ----------------------------------------------------------------------------- top-p

def test_topp_worked_example():
    """Scores ln4, ln2, ln1, ln1 (indices 10..13) have masses 1/2, 1/4, 1/8, 1/8.
    p = 0.7 -> {10, 11}; p = 0.8 -> 3 nodes and the tie at 1/8 goes to the lower index 12;
    p = 0.9 -> all four; p = 1 -> all; p tiny -> the single best node."""
    e = np.log([4.0, 2.0, 1.0, 1.0])
    idx = np.array([10, 11, 12, 13])
    for p, want in [(0.7, [1, 1, 0, 0]), (0.8, [1, 1, 1, 0]), (0.9, [1, 1, 1, 1]),
                    (1.0, [1, 1, 1, 1]), (1e-6, [1, 0, 0, 0])]:
        keep, k, info = O.topp(e, idx, p)
        assert keep.tolist() == [bool(x) for x in want], p
        assert k == sum(want)
    # same candidates presented in another order: same kept indices
    perm = np.array([3, 1, 2, 0])
    keep, k, _ = O.topp(e[perm], idx[perm], 0.8)
    assert sorted(idx[perm][keep].tolist()) == [10, 11, 12]


def test_topp_worked_example_margins():
    """The decision margins the parity tests use to excuse a near-tie, worked by hand on the
    masses 1/2, 1/4, 1/8, 1/8 (sorted order 10, 11, 12, 13; cumulative 1/2, 3/4, 7/8, 1):
      p = 0.7: k* = 2, cum_2 - p = 0.05, p - cum_1 = 0.2, P_(2) - P_(3) = 1/4 - 1/8,
               e_(2) - e_(3) = ln 2 - ln 1;
      p = 0.8: k* = 3, cum_3 - p = 0.075, p - cum_2 = 0.05, and the last kept and the first
               dropped node tie (both 1/8), so the last two margins are 0;
      p = 0.9: k* = 4 = n, cum_4 - p = 0.1, p - cum_3 = 0.025, no dropped node (+inf);
      p = 1:   every node kept without a cut: every margin +inf."""
    e = np.log([4.0, 2.0, 1.0, 1.0])
    idx = np.array([10, 11, 12, 13])
    inf = math.inf
    for p, want in [(0.7, (0.05, 0.2, 0.125, math.log(2.0))), (0.8, (0.075, 0.05, 0.0, 0.0)),
                    (0.9, (0.1, 0.025, inf, inf)), (1.0, (inf, inf, inf, inf))]:
        _, _, info = O.topp(e, idx, p)
        for got, w in zip(info, want):
            if w == inf:
                assert got == inf, (p, info)
            else:
                assert got == pytest.approx(w, abs=1e-15), (p, info)
    # the candidates in another order: the margins describe the sorted order, not the input's
    perm = np.array([2, 0, 3, 1])
    _, _, info2 = O.topp(e[perm], idx[perm], 0.7)
    np.testing.assert_allclose(info2, [0.05, 0.2, 0.125, math.log(2.0)], atol=1e-15)


def _bf_topp(e, p):
    """Brute force: the smallest k such that some k-subset holds mass >= p; returns k and a
    k-subset of maximal mass.  Up to 14 candidates every subset is enumerated; above that
    the maximal k-subset mass is taken as the sum of the k largest masses (numpy sort of
    the masses, not of the (score, index) keys the oracle sorts)."""
    P = softmax(e)
    n = len(e)
    if n > 14:
        order = np.argsort(-P, kind="stable")
        cum = np.cumsum(P[order])
        k = int(np.searchsorted(cum, p - 1e-15) + 1) if p < 1 else n
        k = min(k, n)
        return k, tuple(sorted(order[:k].tolist())), float(cum[k - 1])
    for k in range(1, n + 1):
        best, arg = -1.0, None
        for c in itertools.combinations(range(n), k):
            v = sum(P[list(c)])
            if v > best:
                best, arg = v, c
        if best >= p:
            return k, arg, best
    return n, tuple(range(n)), 1.0


def _bf_topp_size(e, k):
    """Brute force: the largest mass any k-subset of the candidates holds (every subset)."""
    P = softmax(e)
    best, arg = -1.0, None
    for c in itertools.combinations(range(len(e)), k):
        v = sum(P[list(c)])
        if v > best:
            best, arg = v, c
    return k, arg, best


@pytest.mark.parametrize("seed", range(12))
def test_topp_brute_force(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 11))
    e = rng.standard_normal(n) * rng.uniform(0.1, 3.0)
    idx = rng.permutation(100)[:n]
    for p in [0.3, 0.7, 0.9, 0.95, 0.99]:
        keep, k, info = O.topp(e, idx, p)
        kb, _, best = _bf_topp(e, p)
        P = softmax(e)
        assert k == kb == keep.sum()
        assert P[keep].sum() == pytest.approx(best, abs=1e-12)
        assert P[keep].sum() >= p - 1e-12
        # permutation of the candidates keeps the same set of node indices
        perm = rng.permutation(n)
        keep2, _, _ = O.topp(e[perm], idx[perm], p)
        assert set(idx[perm][keep2].tolist()) == set(idx[keep].tolist())
        # decision margins against brute force: the best k*-subset's mass and the best
        # (k*-1)-subset's mass (every subset enumerated), and the masses and scores on the
        # two sides of the cut from scipy's softmax sorted by numpy
        _, _, prev = _bf_topp_size(e, k - 1) if k > 1 else (0, (), 0.0)
        assert info[0] == pytest.approx(best - p, abs=1e-12)
        assert info[1] == pytest.approx(p - prev, abs=1e-12)
        if k < n:
            Ps = np.sort(P)[::-1]
            es = np.sort(e)[::-1]
            assert info[2] == pytest.approx(Ps[k - 1] - Ps[k], abs=1e-12)
            assert info[3] == pytest.approx(es[k - 1] - es[k], abs=1e-12)
        else:
            assert info[2] == math.inf and info[3] == math.inf


def test_topp_ties_prefer_lower_index():
    e = np.zeros(6)
    idx = np.array([5, 3, 9, 0, 7, 1])
    keep, k, _ = O.topp(e, idx, 0.5)         # uniform masses 1/6: 3 nodes
    assert k == 3
    assert sorted(idx[keep].tolist()) == [0, 1, 3]


# ----------------------------------------------------------------------------- routing

def _bf_route(K, qref, C, L, N, q, g, p, scores=None):
    """Independent router: scipy summaries per frontier node, brute-force top-p per level.
    With a dict ``scores``, scores[l] gets {node: plane estimate} of every frontier node."""
    d = K.shape[2]
    s = 1 / math.sqrt(d)
    front = list(range(N // C ** L))
    kept = {}
    for l in range(L, 0, -1):
        span = C ** l
        e = []
        for j in front:
            toks = K[g, j * span:(j + 1) * span]
            a = s * toks @ qref[g].T
            lse = logsumexp(a, axis=0)
            m = softmax(a, axis=0).T @ toks
            bb = lse - s * np.sum(qref[g] * m, axis=1)
            e.append(np.max(s * m @ q + bb))
        e = np.array(e)
        if scores is not None:
            scores[l] = dict(zip(front, e.tolist()))
        k, choice, best = _bf_topp(e, p)
        sel = sorted(front[i] for i in choice)
        kept[l] = sel
        front = [j * C + c for j in sel for c in range(C)]
    return kept


@pytest.mark.parametrize("C,L,N,p,seed", [
    (2, 3, 64, 0.8, 0), (4, 2, 200, 0.9, 1), (4, 3, 256, 0.7, 2), (2, 2, 37, 0.95, 3),
    (3, 2, 100, 0.6, 4)])
def test_route_matches_brute_force(C, L, N, p, seed):
    rng = np.random.default_rng(seed)
    Hkv, d, R = 2, 8, 3
    K = rng.standard_normal((Hkv, N, d)) + 0.3 * rng.standard_normal((Hkv, 1, d))
    qref = rng.standard_normal((Hkv, R, d))
    n_lanes = 4
    q = 2.0 * rng.standard_normal((n_lanes, d))
    lane_g = np.array([0, 1, 0, 1], dtype=np.int32)
    r = O.route(K, qref, C, L, N, q, lane_g, p, return_scores=True)
    for x in range(n_lanes):
        sc = {}
        bf = _bf_route(K, qref, C, L, N, q[x], lane_g[x], p, scores=sc)
        for l in range(1, L + 1):
            assert np.flatnonzero(r.kept[l - 1][x]).tolist() == bf[l], (x, l)
            # every frontier node's estimate at its own index; the others left untouched (NaN)
            row = r.scores[l - 1][x]
            front = sorted(sc[l])
            np.testing.assert_allclose(row[front], [sc[l][j] for j in front], rtol=0, atol=1e-12)
            off = np.setdiff1d(np.arange(row.size), front)
            assert np.isnan(row[off]).all(), (x, l)
            assert r.nfront[l - 1][x] == len(front)
            # the margins of this lane's cut from the brute-force estimates: cumulative masses
            # of the sorted softmax (scipy) on both sides of k*
            e = np.array([sc[l][j] for j in front])
            P = np.sort(softmax(e))[::-1]
            k = int(r.kstar[l - 1][x])
            cum = np.concatenate([[0.0], np.cumsum(P)])
            info = r.info[l - 1][x]
            if p < 1:
                assert info[0] == pytest.approx(cum[k] - p, abs=1e-12)
                assert info[1] == pytest.approx(p - cum[k - 1], abs=1e-12)


def test_route_replay_with_own_sets_is_identity():
    rng = np.random.default_rng(3)
    K = rng.standard_normal((1, 512, 8))
    qref = rng.standard_normal((1, 2, 8))
    q = rng.standard_normal((3, 8)) * 2
    g = np.zeros(3, dtype=np.int32)
    r1 = O.route(K, qref, 4, 3, 512, q, g, 0.8)
    r2 = O.route(K, qref, 4, 3, 512, q, g, 0.8, forced=r1.kept)
    for a, b in zip(r1.kept, r2.kept):
        assert np.array_equal(a, b)
    np.testing.assert_array_equal(r1.info, r2.info)


# ----------------------------------------------------------------------------- attention

def test_attended_set_sink_tail_and_union():
    """Token 0 is always attended ([wqu] top-p routing section), once even if its chunk is
    kept; tokens past the last complete top node are attended densely; with no complete
    top node everything is attended."""
    sink = json.load(open(GOLDEN))["sink_token"]["token"]
    C, L, N = 4, 2, 16 * 3 + 5                    # T = 3 top nodes of 16 tokens, tail of 5
    kept1 = np.zeros(N // C, dtype=bool)
    A = O.attended_set(kept1, N, C, L)
    assert A.tolist() == [sink] + list(range(48, N))
    kept1[0] = kept1[5] = True
    A = O.attended_set(kept1, N, C, L)
    assert A.tolist() == [0, 1, 2, 3, 20, 21, 22, 23] + list(range(48, N))
    assert O.attended_set(np.zeros(3, bool), 15, 4, 2).tolist() == list(range(15))


def test_attend_closed_form():
    """Scores (ln 3, 0) -> weights 3/4, 1/4 -> o = 3/4 v_1 + 1/4 v_2."""
    d = 4
    K = np.array([[2 * math.log(3.0), 0, 0, 0], [0, 0, 0, 0], [9, 9, 9, 9.0]])
    V = np.array([[1.0, 2, 3, 4], [-4.0, 0, 8, 1], [100.0, 100, 100, 100]])
    out = O.attend(K, V, np.array([1.0, 0, 0, 0]), np.array([0, 1]))
    np.testing.assert_allclose(out, 0.75 * V[0] + 0.25 * V[1], atol=1e-14)


def test_p1_routing_reduces_to_dense_attention_sdpa():
    """p = 1 keeps every node, so the attended set is [0, N) and the output is plain
    softmax attention - checked against torch's scaled_dot_product_attention in float64."""
    from hierarchical_tree_indexed_build_b200 import inputs
    wl = inputs.tiny_4k()
    seq = wl.seqs[0]
    g = seq.geom
    K = seq.K.to(torch.float64).numpy()
    V = seq.V.to(torch.float64).numpy()
    qref = seq.qref.to(torch.float64).numpy()
    Q = wl.Q[0, 0].to(torch.float64).numpy()[:, 0, :]      # [n_q][d], one head
    lane_g = np.zeros(Q.shape[0], dtype=np.int32)
    r, out, toks = O.decode(K, V, qref, g.C, g.L, seq.n_tokens, Q, lane_g, 1.0)
    for t in toks:
        assert t.tolist() == list(range(seq.n_tokens))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q)[None, :, None, :], torch.from_numpy(K[0])[None, None],
        torch.from_numpy(V[0])[None, None])[0, :, 0, :].numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_tiny_workload_routing_keeps_sink_and_is_sparse():
    """On the tiny workload at p = 0.9 every lane attends token 0, attends fewer tokens than
    the cache, and every level keeps at least one node."""
    from hierarchical_tree_indexed_build_b200 import inputs
    wl = inputs.tiny_4k()
    seq = wl.seqs[0]
    g = seq.geom
    K = seq.K.to(torch.float64).numpy()
    V = seq.V.to(torch.float64).numpy()
    qref = seq.qref.to(torch.float64).numpy()
    Q = wl.Q[0, 0].to(torch.float64).numpy()[:, 0, :]
    r, out, toks = O.decode(K, V, qref, g.C, g.L, seq.n_tokens, Q, np.zeros(16, np.int32), 0.9)
    assert all(t[0] == 0 for t in toks)
    assert all(t.size < seq.n_tokens for t in toks)
    assert (r.kstar >= 1).all()
    assert (r.nfront[-1] == seq.n_tokens // g.top_span).all()


# ----------------------------------------------------------------------------- MXFP4 rounding

def _nearest_e2m1_brute(y):
    """Nearest of the 15 signed E2M1 values to y by exhaustive search; a tie goes to the value
    whose code has mantissa bit 0 (codes 0, 2, 4, 6 in each sign)."""
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    cands = [(abs(y - s * m), code % 2, s * m) for code, m in enumerate(mags) for s in (1.0, -1.0)]
    best = min(c[0] for c in cands)
    ties = [c for c in cands if c[0] == best]
    ties.sort(key=lambda c: c[1])                   # even mantissa first
    return ties[0][2]


def test_mxfp4_hand_worked_block():
    """Block max 7.9: floor(log2 7.9) = 2, so X = 2^0 = 1 and the E8M0 byte is 127.
    1.0 -> 1; 0.3 -> 0.5; -0.76 -> -1 (nearer 1 than 0.5); 0.24 -> 0; 5.0 (tie 4|6) -> 4 (even);
    7.9 -> 6 (saturated); 2.5 (tie 2|3) -> 2; 3.5 (tie 3|4) -> 4; 0.25 (tie 0|0.5) -> 0;
    0.75 (tie 0.5|1) -> 1; -1.75 (tie 1.5|2) -> -2; 1.25 (tie 1|1.5) -> 1."""
    x = np.zeros(32)
    x[:12] = [1.0, 0.3, -0.76, 0.24, 5.0, 7.9, 2.5, 3.5, 0.25, 0.75, -1.75, 1.25]
    v, codes, E = O.mxfp4(x)
    assert E.tolist() == [127]
    assert v[:12].tolist() == [1.0, 0.5, -1.0, 0.0, 4.0, 6.0, 2.0, 4.0, 0.0, 1.0, -2.0, 1.0]
    assert codes[:12].tolist() == [2, 1, 8 + 2, 0, 6, 7, 4, 6, 0, 2, 8 + 4, 2]
    assert (v[12:] == 0).all()


def test_mxfp4_scale_is_the_blocks_binade():
    """max |x| = 0.1 = 1.6 x 2^-4: X = 2^(-4 - 2) = 2^-6; 0.1 / X = 6.4 saturates to 6, so the
    block maximum decodes to 6 / 64 = 0.09375.  An all-zero block has byte 0 and decodes to 0."""
    x = np.zeros((2, 32))
    x[0, 5] = 0.1
    x[0, 6] = -0.05                                  # 3.2 -> 3
    v, _, E = O.mxfp4(x)
    assert E.ravel().tolist() == [127 - 6, 0]
    assert v[0, 5] == 6 / 64 and v[0, 6] == -3 / 64
    assert (v[1] == 0).all()


def test_mxfp4_is_the_nearest_value_on_the_block_grid():
    """Brute force: every element is the nearest signed E2M1 value times the block's scale."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((40, 64)) * np.exp(rng.uniform(-8, 8, (40, 1)))
    x[:, ::7] *= 1e-3                                # small members of a block
    v, _, E = O.mxfp4(x)
    for i in range(x.shape[0]):
        for j in range(x.shape[1]):
            X = 2.0 ** (int(E[i, j // 32]) - 127)
            assert v[i, j] == _nearest_e2m1_brute(x[i, j] / X) * X
        for b in range(2):
            blk = x[i, 32 * b:32 * b + 32]
            X = 2.0 ** (int(E[i, b]) - 127)
            # the scale's binade: 4 X <= max |x| < 8 X
            assert 4 * X <= np.abs(blk).max() < 8 * X


def test_mxfp4_representable_blocks_round_trip():
    """A block of E2M1 values times 2^k whose maximum magnitude is 4 or 6 (times 2^k) decodes to
    itself, codes and all."""
    rng = np.random.default_rng(4)
    for k in (-10, -1, 0, 3, 9):
        idx = rng.integers(0, 8, 32)
        idx[0] = 7
        sgn = rng.choice([-1.0, 1.0], 32)
        x = sgn * O.E2M1_VALUES[idx] * 2.0 ** k
        v, codes, E = O.mxfp4(x)
        assert np.array_equal(v, x)
        assert E.tolist() == [127 + k]
        assert np.array_equal(codes & 7, idx)
