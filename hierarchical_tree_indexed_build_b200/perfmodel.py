"""Stage-wise B200 performance model of the tree build and the tree-routed decode.

The pages model latency in four stages - tree build, per-level routing, node scan and the
final exact attention - each with a three-term roofline and a worker-wave term for the
parallelism a pruned level leaves idle ("Zyphra ZHA 稀疏注意力…", fluxbbs.com, section
加速数字需要打折看待).  The pages give no formula; this module takes the plainest reading:

  t_stage = alpha * max(bytes / BW, flops / P) * wave(units, slots) + beta * launches

* bytes, flops: what the stage moves and multiplies (algorithmic bytes; the flops the
  kernels execute - the tensor-core scorer multiplies every lane of a group with every
  candidate of the group, in two fp16 passes);
* BW, P: the measured HBM copy bandwidth and tensor (or FP32) peak of MEASURED_PEAKS.json;
* wave(units, slots) = ceil(units / slots) * slots / units: the stage's independent work
  items (workers, node tiles, lanes, attention splits) fill `slots` concurrent places (SMs x
  resident items per SM); fewer items than slots, or a ragged last wave, leave SMs idle;
* launches: dependent kernel launches of the stage (levels are sequential);
* alpha (>= 1: how far the kernels stay from their roofline) and beta (ms per launch) are
  fitted per stage by non-negative least squares to measured stage times.

Stage times are measured by the library's own CUDA-event profile (bench.py --stage-sweep):
  build      k_build_stream + k_merge
  routing    k_union + k_member + k_select          (per level: union, lane masks, top-p cut)
  node scan  k_score / k_score_few / k_score_tc     (plane estimates of every scored node)
  attention  k_attn / k_attn_tc + k_combine         (exact attention over the kept tokens)
Nothing here runs on the GPU.
"""
from __future__ import annotations

import json
import math
import os
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
MEASURED = os.path.join(HERE, "perfmodel_measured.json")
SMS = 148
HBM_CAPACITY_GB = 180.0
FP32_LANES_PER_SM = 128

STAGES = ("build", "routing", "node_scan", "attention")
STAGE_KERNELS = {
    "build": ("k_build_stream", "k_build_tc", "k_merge"),
    "routing": ("k_union", "k_member", "k_select"),
    "node_scan": ("k_score", "k_score_few", "k_score_tc"),
    "attention": ("k_attn", "k_attn_tc", "k_combine"),
}


@dataclass
class Peaks:
    hbm_gbs: float
    tensor_tflops: float          # dense bf16 / f16 (measured burst figure)
    fp32_tflops: float            # CUDA-core FMA peak from the unit counts and the max clock
    source: str


def peaks(path: Optional[str] = None) -> Peaks:
    """Measured denominators (MEASURED_PEAKS.json at the repository root); the recorded
    fallback (6.65 TB/s, 1.59 PFLOP/s, 1965 MHz) when the file is absent."""
    path = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        mhz = float(pk.get("sm_max_mhz", 1965.0))
        return Peaks(float(pk["hbm_gbs"]), float(pk["bf16_tflops"]),
                     SMS * FP32_LANES_PER_SM * 2 * mhz * 1e6 / 1e12, "measured")
    except (OSError, KeyError, ValueError):
        return Peaks(6650.0, 1590.0, SMS * FP32_LANES_PER_SM * 2 * 1965e6 / 1e12, "fallback")


def record_bytes(R: int, d: int) -> int:
    """Bytes of one node as the build writes it: m as fp16 hi + lo planes [R][d] each, plus
    b and lse in f32 per reference query."""
    return R * d * 2 * 2 + 2 * R * 4


def scored_bytes(R: int, d: int) -> int:
    """Bytes the scorer reads per node: the two m planes and b (lse is not read)."""
    return R * d * 2 * 2 + R * 4


def kv_bytes_per_token(d: int, Hkv: int) -> int:
    """K and V bytes of one token over all KV heads (bf16)."""
    return 2 * Hkv * d * 2


def level_nodes(N: int, C: int, L: int) -> List[int]:
    """Complete nodes per level 1..L (only complete nodes exist)."""
    return [N // C ** l for l in range(1, L + 1)]


def levels_for(N: int, C: int, top_nodes: int = 256) -> int:
    """Tree depth that leaves about top_nodes complete nodes at the top (at least 1 level)."""
    L = 1
    while N // C ** (L + 1) >= top_nodes:
        L += 1
    return L


def wave(units: float, slots: float) -> float:
    """Worker-wave factor: time of `units` equal work items on `slots` concurrent places,
    relative to the same work spread perfectly over all places."""
    if units <= 0:
        return 1.0
    return math.ceil(units / slots) * slots / units


@dataclass
class StageWork:
    """What one stage of one call moves, multiplies and launches."""
    bytes: float
    flops: float
    tensor: bool                  # flops run on the tensor cores (else CUDA cores)
    units: float                  # independent work items
    slots: float                  # concurrent places for them
    launches: float

    def roofline_ms(self, pk: Peaks) -> float:
        peak = pk.tensor_tflops if self.tensor else pk.fp32_tflops
        t = max(self.bytes / (pk.hbm_gbs * 1e9), self.flops / (peak * 1e12) if self.flops else 0.0)
        return t * 1e3 * wave(self.units, self.slots)


@dataclass
class Geometry:
    C: int
    L: int
    R: int
    d: int
    Hq: int
    Hkv: int


def build_work(g: Geometry, N: int, n_append: int = 0) -> StageWork:
    """Tree build over N tokens (plus an append): K read once, every complete node written;
    flops 4 N R d per KV head (reference scores and the weighted key sums).  Units: the
    streaming build's workers (one 64-token subtree each); launches: the build kernel(s) and
    one merge per level above the streamed ones."""
    n = N + n_append
    nodes = sum(level_nodes(n, g.C, g.L))
    bts = g.Hkv * (n * 2 * g.d + nodes * record_bytes(g.R, g.d))
    flops = 4.0 * n * g.R * g.d * g.Hkv
    span = g.C
    k_emit = 1
    while k_emit < g.L and span * g.C <= 64:
        span *= g.C
        k_emit += 1
    units = g.Hkv * max(1, n // span)
    launches = 2 + (g.L - 1) + (g.L if n_append else 0)
    return StageWork(bts, flops, False, units, SMS * 16, launches)


def decode_work(g: Geometry, n_gl: int, stats: Dict, tensor_score: bool, tensor_attn: bool) -> Dict[str, StageWork]:
    """Routing, node scan and attention of one decode call from the decoder's work counters:
    union_nodes / lane_nodes per level (summed over the (sequence, KV head) groups),
    union_tokens / lane_tokens.  n_gl: lanes per group."""
    un = list(stats["union_nodes"])[:g.L]
    ln = list(stats["lane_nodes"])[:g.L]
    ut, lt = stats["union_tokens"], stats["lane_tokens"]
    lanes = n_gl * g.Hkv                                 # lanes of the call (one sequence)
    levels = sum(1 for u in un if u)
    # routing: each lane's scores read twice by the cut, plus its kept bitmap; one block per lane
    routing = StageWork(bytes=sum(ln) * 4 * 2, flops=0.0, tensor=False, units=lanes,
                        slots=SMS * 2, launches=4 * levels - 3)
    # node scan: every scored record read once per group, a score written per (lane, candidate)
    if tensor_score:
        flops = sum(un) * n_gl * 2.0 * g.R * g.d * 2      # every lane x every union node, hi + lo
        units = sum(un) / 8.0                            # node tiles of 8 nodes
        slots = SMS
    else:
        flops = sum(ln) * 2.0 * g.R * g.d
        units = sum(un)
        slots = SMS * 16
    scan = StageWork(bytes=sum(un) * scored_bytes(g.R, g.d) + sum(un) * n_gl * 4.0, flops=flops,
                     tensor=tensor_score, units=units, slots=slots, launches=levels)
    # attention: the union's K/V rows gathered once per group, 4d flops per (lane, token);
    # every (lane, split) partial record written once and read once by the combine
    split = 4096 if n_gl > 64 else (1024 if n_gl > 16 else 256)
    splits = max(1, math.ceil(ut / g.Hkv / split))       # splits per group
    units = splits * g.Hkv * max(1, math.ceil(n_gl / 128))
    if tensor_attn:
        aflops = ut * n_gl * 6.0 * g.d                   # Q K^T plus P V in two bf16 passes
    else:
        aflops = lt * 4.0 * g.d
    attn = StageWork(bytes=ut * 4.0 * g.d + lanes * splits * (g.d + 4) * 4.0 * 2, flops=aflops,
                     tensor=tensor_attn, units=units, slots=SMS, launches=3)
    return {"routing": routing, "node_scan": scan, "attention": attn}


@dataclass
class Fit:
    """alpha (dimensionless) and beta (ms per launch) per stage."""
    alpha: Dict[str, float] = field(default_factory=lambda: {s: 1.0 for s in STAGES})
    beta: Dict[str, float] = field(default_factory=lambda: {s: 0.0 for s in STAGES})

    def predict(self, stage: str, w: StageWork, pk: Peaks) -> float:
        return self.alpha[stage] * w.roofline_ms(pk) + self.beta[stage] * w.launches


def stage_times(kernel_ms: Dict[str, float]) -> Dict[str, float]:
    """Measured per-kernel device times (ms) summed into the four stages."""
    return {s: sum(kernel_ms.get(k, 0.0) for k in ks) for s, ks in STAGE_KERNELS.items()}


def fit(points: Sequence[Tuple[str, StageWork, float]], pk: Peaks) -> Tuple[Fit, Dict[str, List[float]]]:
    """Non-negative least squares per stage: measured_ms ~ alpha * roofline_ms + beta *
    launches over the given (stage, work, measured ms) points.  Returns the fit and, per
    stage, the relative residuals (predicted / measured - 1)."""
    from scipy.optimize import nnls
    f = Fit()
    resid: Dict[str, List[float]] = {}
    for s in STAGES:
        pts = [(w, t) for st, w, t in points if st == s and t > 0]
        if not pts:
            continue
        # weight rows by 1 / measured so that the fit minimises relative error
        A = np.array([[w.roofline_ms(pk) / t, w.launches / t] for w, t in pts])
        b = np.ones(len(pts))
        x, _ = nnls(A, b)
        f.alpha[s], f.beta[s] = float(x[0]), float(x[1])
        resid[s] = [f.predict(s, w, pk) / t - 1.0 for w, t in pts]
    return f, resid


def load_measured(path: str = MEASURED) -> List[Dict]:
    with open(path) as fh:
        return json.load(fh)["runs"]


def points_from_runs(runs: Sequence[Dict]) -> List[Tuple[str, StageWork, float]]:
    """(stage, work, measured ms) points of recorded stage-sweep lines."""
    pts = []
    for r in runs:
        g = Geometry(**r["geometry"])
        st = stage_times(r["kernel_ms"])
        if r["stage"] == "build":
            pts.append(("build", build_work(g, r["n_tokens"]), st["build"]))
            continue
        n_gl = r["n_q"] * g.Hq // g.Hkv
        ts = any(k == "k_score_tc" for k in r["kernel_ms"])
        ta = any(k == "k_attn_tc" for k in r["kernel_ms"])
        for s, w in decode_work(g, n_gl, r["stats"], ts, ta).items():
            pts.append((s, w, st[s]))
    return pts


def dense_ms(N: int, d: int, Hkv: int, bw_gbs: Optional[float] = None) -> float:
    """Dense flash-decode lower bound: K and V of all N tokens read once."""
    bw = bw_gbs if bw_gbs is not None else peaks().hbm_gbs
    return N * kv_bytes_per_token(d, Hkv) / (bw * 1e9) * 1e3


def fixed_budget_stats(N: int, C: int, L: int, k: int, lanes_per_group: int, Hkv: int) -> Dict:
    """Decoder statistics when every lane keeps k nodes per level: the top level is scored
    whole; below it each lane scores the C children of its k kept parents, and a group's
    union is at most its lanes times that (no overlap assumed, an upper bound) and at most
    the level.  Attended tokens per group: the lanes' kept chunks, the sink and the tail."""
    n = level_nodes(N, C, L)
    union, lane = [0] * L, [0] * L
    for l in range(L, 0, -1):
        per_lane = n[l - 1] if l == L else min(n[l - 1], k * C)
        per_group = n[l - 1] if l == L else min(n[l - 1], lanes_per_group * k * C)
        union[l - 1] = per_group * Hkv
        lane[l - 1] = per_lane * lanes_per_group * Hkv
    tail = N - n[L - 1] * C ** L
    tokens = (min(N, lanes_per_group * k * C) + 1 + tail) * Hkv
    ltok = (min(N, k * C) + 1 + tail) * lanes_per_group * Hkv
    return {"union_nodes": union, "lane_nodes": lane, "union_tokens": tokens, "lane_tokens": ltok}


def project(Ns: Sequence[int], C: int = 4, R: int = 16, d: int = 128, Hq: int = 16, Hkv: int = 2,
            k: int = 64, f: Optional[Fit] = None, pk: Optional[Peaks] = None) -> List[Dict[str, float]]:
    """One query token per step: dense lower bound against the modelled routed decode (node
    scan + routing + attention, CUDA-core kernels as the few-lane path uses) under a fixed
    kept budget of k nodes per lane per level, with the fitted stage constants."""
    pk = pk or peaks()
    f = f or Fit()
    G = Hq // Hkv
    rows = []
    for N in Ns:
        L = levels_for(N, C)
        g = Geometry(C, L, R, d, Hq, Hkv)
        st = fixed_budget_stats(N, C, L, k, G, Hkv)
        work = decode_work(g, G, st, False, False)
        rb = sum(w.bytes for w in work.values()) / (pk.hbm_gbs * 1e9) * 1e3
        rm = sum(f.predict(s, w, pk) for s, w in work.items())
        dn = dense_ms(N, d, Hkv, pk.hbm_gbs)
        rows.append({"N": N, "L": L, "kv_gb": N * kv_bytes_per_token(d, Hkv) / 1e9,
                     "fits_one_gpu": N * kv_bytes_per_token(d, Hkv) / 1e9 <= HBM_CAPACITY_GB,
                     "dense_ms": dn, "routed_bytes_ms": rb, "routed_ms": rm,
                     "speedup_bytes": dn / rb, "speedup": dn / rm})
    return rows


def main() -> None:
    import argparse
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--k", type=int, nargs="+", default=[64, 1024],
                    help="kept nodes per lane per level (fixed budget) for the projections")
    ap.add_argument("--record", nargs="+", metavar="LOG",
                    help="rewrite the recorded measurements from the JSON lines of `bench.py --stage-sweep` "
                         "logs (one per command in --commands), then fit")
    ap.add_argument("--commands", nargs="+", default=[], help="the commands that wrote the --record logs")
    args = ap.parse_args()
    if args.record:
        runs = []
        for path in args.record:
            with open(path) as fh:
                runs += [json.loads(l) for l in fh if l.startswith("{") and '"stage"' in l]
        with open(MEASURED, "w") as fh:
            json.dump({"what": "per-kernel device times (ms per call, the library's CUDA-event profile) and "
                               "decoder work counters of the build and of the decode at several p, one B200",
                       "commands": args.commands, "runs": runs}, fh, indent=1)
        print("recorded %d runs into %s" % (len(runs), MEASURED))
    pk = peaks()
    runs = load_measured()
    f, resid = fit(points_from_runs(runs), pk)
    print("peaks (%s): HBM %.0f GB/s, tensor %.0f TFLOP/s, FP32 %.1f TFLOP/s" %
          (pk.source, pk.hbm_gbs, pk.tensor_tflops, pk.fp32_tflops))
    print("%-10s %8s %12s %6s %22s" % ("stage", "alpha", "beta (us)", "pts", "residual median / max"))
    for s in STAGES:
        if s in resid:
            r = np.abs(resid[s])
            print("%-10s %8.2f %12.2f %6d %10.1f%% / %6.1f%%" % (s, f.alpha[s], f.beta[s] * 1e3, len(r),
                                                                100 * np.median(r), 100 * r.max()))
    for k in args.k:
        print("\nkept budget k = %d nodes per lane per level, one query token (16 heads, GQA 16/2)" % k)
        print("%12s %3s %9s %5s %11s %14s %11s %9s %9s" % ("N", "L", "KV GB", "1GPU", "dense ms",
                                                        "routed(bytes)", "routed ms", "x bytes", "x model"))
        for r in project([262144, 1 << 20, 10 << 20, 100 << 20, 1 << 30], k=k, f=f, pk=pk):
            print("%12d %3d %9.1f %5s %11.3f %14.3f %11.3f %9.2f %9.2f" % (
                r["N"], r["L"], r["kv_gb"], "yes" if r["fits_one_gpu"] else "no", r["dense_ms"],
                r["routed_bytes_ms"], r["routed_ms"], r["speedup_bytes"], r["speedup"]))


if __name__ == "__main__":
    main()
