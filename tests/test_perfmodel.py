"""The stage-wise B200 model (CPU): byte accounting, each term's limiting cases, the fit and
the projections."""
import json
import math

import numpy as np
import pytest

from hierarchical_tree_indexed_build_b200 import perfmodel as P

PK = P.Peaks(hbm_gbs=1000.0, tensor_tflops=1000.0, fp32_tflops=50.0, source="test")


def test_record_and_kv_bytes():
    # m as two fp16 planes of R x d, lse and b in f32 per reference query
    assert P.record_bytes(16, 128) == 16 * 128 * 4 + 16 * 8 == 8320
    assert P.scored_bytes(16, 128) == 8256                 # the scorer reads m and b, not lse
    # K and V, bf16, per KV head
    assert P.kv_bytes_per_token(128, 1) == 512
    assert P.kv_bytes_per_token(128, 2) == 1024


def test_peaks_come_from_the_measured_file(tmp_path):
    f = tmp_path / "peaks.json"
    f.write_text(json.dumps({"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "sm_max_mhz": 1000.0}))
    pk = P.peaks(str(f))
    assert (pk.hbm_gbs, pk.tensor_tflops, pk.source) == (6000.0, 1500.0, "measured")
    assert pk.fp32_tflops == pytest.approx(148 * 128 * 2 * 1e9 / 1e12)
    fb = P.peaks(str(tmp_path / "missing.json"))
    assert (fb.hbm_gbs, fb.tensor_tflops, fb.source) == (6650.0, 1590.0, "fallback")


def test_wave_factor_limits():
    assert P.wave(148, 148) == 1.0                          # one full wave
    assert P.wave(148 * 5, 148) == 1.0                      # whole waves
    assert P.wave(37, 148) == pytest.approx(4.0)            # a quarter of the machine busy
    assert P.wave(148 * 1.5, 148) == pytest.approx(2 / 1.5) # a ragged last wave
    assert P.wave(1, 148) == 148.0
    # many waves: the ragged tail stops mattering
    assert P.wave(148 * 1000 + 1, 148) == pytest.approx(1.0, abs=2e-3)


def test_roofline_memory_and_compute_limits():
    # memory-bound: 1 GB at 1000 GB/s = 1 ms, the flops take 1 us
    w = P.StageWork(bytes=1e9, flops=1e9, tensor=True, units=148, slots=148, launches=0)
    assert w.roofline_ms(PK) == pytest.approx(1.0)
    # compute-bound on the tensor cores: 1e15 flop at 1000 TFLOP/s = 1000 ms
    w = P.StageWork(bytes=1e6, flops=1e15, tensor=True, units=148, slots=148, launches=0)
    assert w.roofline_ms(PK) == pytest.approx(1000.0)
    # the same flops on CUDA cores use the FP32 peak
    w = P.StageWork(bytes=1e6, flops=1e15, tensor=False, units=148, slots=148, launches=0)
    assert w.roofline_ms(PK) == pytest.approx(20000.0)
    # idle places stretch the bound by the wave factor
    w = P.StageWork(bytes=1e9, flops=0.0, tensor=False, units=74, slots=148, launches=0)
    assert w.roofline_ms(PK) == pytest.approx(2.0)


def test_latency_term_is_per_launch():
    f = P.Fit()
    f.beta["routing"] = 0.01
    w = P.StageWork(bytes=0.0, flops=0.0, tensor=False, units=1, slots=1, launches=21)
    assert f.predict("routing", w, PK) == pytest.approx(0.21)


def test_fit_recovers_known_constants():
    rng = np.random.default_rng(0)
    alpha = {"build": 2.0, "routing": 5.0, "node_scan": 1.5, "attention": 3.0}
    beta = {"build": 0.004, "routing": 0.02, "node_scan": 0.0, "attention": 0.01}
    pts = []
    for s in P.STAGES:
        for _ in range(6):
            w = P.StageWork(bytes=float(rng.uniform(1e7, 1e9)), flops=0.0, tensor=False,
                            units=148, slots=148, launches=float(rng.integers(1, 30)))
            pts.append((s, w, alpha[s] * w.roofline_ms(PK) + beta[s] * w.launches))
    f, resid = P.fit(pts, PK)
    for s in P.STAGES:
        assert f.alpha[s] == pytest.approx(alpha[s], rel=1e-9)
        assert f.beta[s] == pytest.approx(beta[s], rel=1e-9, abs=1e-12)
        assert max(abs(r) for r in resid[s]) < 1e-9


def test_stage_times_sum_the_kernels():
    st = P.stage_times({"k_build_stream": 2.0, "k_merge": 0.1, "k_union": 0.3, "k_member": 0.4,
                        "k_select": 2.5, "k_score_tc": 5.0, "k_attn_tc": 3.5, "k_combine": 0.2})
    assert st == pytest.approx({"build": 2.1, "routing": 3.2, "node_scan": 5.0, "attention": 3.7})


def test_build_work_counts_every_node_once():
    g = P.Geometry(C=4, L=6, R=16, d=128, Hq=16, Hkv=2)
    N = 1 << 20
    w = P.build_work(g, N)
    nodes = sum(N // 4 ** l for l in range(1, 7))
    assert w.bytes == 2 * (N * 256 + nodes * 8320)
    assert w.flops == 4.0 * N * 16 * 128 * 2
    assert w.units == 2 * N // 64                           # one worker per 64-token subtree


def test_decode_work_tensor_scan_counts_every_lane_and_union_node():
    g = P.Geometry(C=4, L=2, R=16, d=128, Hq=16, Hkv=2)
    st = {"union_nodes": [400, 64], "lane_nodes": [3000, 1024], "union_tokens": 5000, "lane_tokens": 40000}
    w = P.decode_work(g, 16, st, True, False)
    assert w["node_scan"].flops == 464 * 16 * 2 * 16 * 128 * 2
    assert w["node_scan"].bytes == 464 * 8256 + 464 * 16 * 4
    assert w["routing"].bytes == 4024 * 8
    assert w["attention"].flops == 40000 * 4 * 128           # CUDA cores: each lane's own tokens
    assert w["attention"].bytes >= 5000 * 512


def test_fixed_budget_stats_are_bounded_by_the_levels():
    N, C, L, k, G, Hkv = 1 << 20, 4, 6, 64, 8, 2
    st = P.fixed_budget_stats(N, C, L, k, G, Hkv)
    n = P.level_nodes(N, C, L)
    assert st["union_nodes"][L - 1] == n[L - 1] * Hkv       # the top level is scored whole
    for l in range(1, L):
        assert st["union_nodes"][l - 1] == min(n[l - 1], G * k * C) * Hkv
    assert st["union_tokens"] == (G * k * C + 1) * Hkv      # no tail: N is a multiple of C^L
    # a budget that covers everything scores every node
    all_ = P.fixed_budget_stats(N, C, L, N, G, Hkv)
    assert all_["union_nodes"] == [x * Hkv for x in n]
    assert all_["union_tokens"] == (N + 1) * Hkv


def test_speedup_grows_with_context_under_a_fixed_budget():
    f = P.Fit()
    f.beta = {s: 0.02 for s in P.STAGES}
    rows = P.project([1 << 18, 1 << 20, 1 << 24, 1 << 27], k=64, f=f, pk=PK)
    sb = [r["speedup_bytes"] for r in rows]
    sm = [r["speedup"] for r in rows]
    assert all(a < b for a, b in zip(sb, sb[1:]))
    assert all(a < b for a, b in zip(sm, sm[1:]))
    for r in rows:                                          # latency and waves only add time
        assert r["routed_ms"] >= r["routed_bytes_ms"]


def test_fit_to_the_recorded_measurements():
    """The constants fitted to the recorded stage sweeps (1M and 256K, several p, batch and
    one query token) explain every recorded stage time within a factor of two and have
    non-negative launch latency; every stage stays above its roofline (alpha >= 1)."""
    runs = P.load_measured()
    pts = P.points_from_runs(runs)
    f, resid = P.fit(pts, P.peaks())
    for s in P.STAGES:
        assert s in resid, s
        assert f.beta[s] >= 0.0
        assert np.max(np.abs(resid[s])) < 1.0, (s, resid[s])
    for s, w, t in pts:
        assert t >= w.roofline_ms(P.peaks()) * 0.9, (s, t, w.roofline_ms(P.peaks()))
