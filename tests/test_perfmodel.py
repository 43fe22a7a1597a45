"""The stage-wise B200 model (CPU): byte accounting, limiting cases and monotonicity."""
import pytest

from hierarchical_tree_indexed_build_b200 import perfmodel as P


def test_record_and_kv_bytes():
    # m as two fp16 planes of R x d, lse and b in f32 per reference query
    assert P.record_bytes(16, 128) == 16 * 128 * 4 + 16 * 8 == 8320
    # K and V, bf16, per KV head
    assert P.kv_bytes_per_token(128, 1) == 512
    assert P.kv_bytes_per_token(128, 2) == 1024


def test_dense_is_kv_bytes_over_bandwidth():
    N = 1 << 20
    assert P.dense_ms(N, 128, 2, bw_gbs=1000.0) == pytest.approx(N * 1024 / 1e12 * 1e3)


def test_levels_leave_a_small_top():
    for N in (1 << 16, 1 << 18, 1 << 20, 10 << 20):
        L = P.levels_for(N, 4)
        assert 256 <= N // 4 ** L < 1024 or L == 1
    assert P.levels_for(1 << 20, 4) == 6


def test_scoring_every_node_costs_more_bytes_than_dense():
    """At p = 1 the routed decode scores every node and attends every token: with C = 4 and
    R = 16 a level-1 record alone is 4x the K/V bytes of its 4 tokens, so routing cannot win
    on bytes unless the scored frontier is a small part of each level."""
    N, C, L, R, d, Hkv = 1 << 20, 4, 6, 16, 128, 2
    union = [n * Hkv for n in P.level_nodes(N, C, L)]
    rb = P.routed_bytes(union, N * Hkv, R, d, Hkv)
    assert rb > 4 * N * P.kv_bytes_per_token(d, Hkv)
    assert P.record_bytes(R, d) > 4 * P.kv_bytes_per_token(d, 1) * C


def test_fixed_budget_sizes_are_bounded_by_the_levels():
    N, C, L, k, G, Hkv = 1 << 20, 4, 6, 64, 8, 2
    union, tokens = P.fixed_budget_sizes(N, C, L, k, G, Hkv)
    n = P.level_nodes(N, C, L)
    assert union[0] == n[L - 1] * Hkv                      # the top level is scored whole
    for l, u in zip(range(L - 1, 0, -1), union[1:]):
        assert u == min(n[l - 1], G * k * C) * Hkv
    assert tokens == (G * k * C + 1) * Hkv                 # no tail: N is a multiple of C^L
    # a budget that covers everything scores every node
    union_all, tokens_all = P.fixed_budget_sizes(N, C, L, N, G, Hkv)
    assert union_all == [n[l - 1] * Hkv for l in range(L, 0, -1)]
    assert tokens_all == (N + 1) * Hkv


def test_speedup_grows_with_context_under_a_fixed_budget():
    rows = P.project([1 << 18, 1 << 20, 1 << 24, 1 << 27], k=64)
    sb = [r["speedup_bytes"] for r in rows]
    sm = [r["speedup"] for r in rows]
    assert all(a < b for a, b in zip(sb, sb[1:]))
    assert all(a < b for a, b in zip(sm, sm[1:]))
    for r in rows:                                          # latency only adds time
        assert r["routed_ms"] >= r["routed_bytes_ms"]
        assert r["speedup"] <= r["speedup_bytes"]


def test_latency_term_is_per_level():
    fit = P.Fit(level_ms=0.5)
    u = [10, 20, 30]
    assert P.routed_ms(u, 0, 16, 128, 2, fit) - P.routed_ms(u, 0, 16, 128, 2, fit, latency=False) \
        == pytest.approx(1.5)
