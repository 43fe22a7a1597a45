"""Benchmark: ZHA tree build + append + tree-routed sparse decode on B200.

One step = the whole hot path over one batch of the 1M-token deep-tree workload:
  zha_build_tree over N = 1,048,576 tokens (chunk summaries + level merges),
  zha_append of 4,096 tokens, then
  zha_decode of the 128 needle queries (16 query heads / 2 KV heads each) at p = 0.95
  (routing level by level + exact attention over sink, kept chunks and tail).
value = decoded queries per second of device time (max over ranks, summed over ranks).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--p P] [--workload deep1m|deep256k|deep64k|wide256k] [--n-q N]
                  [--no-e2e] [--no-cpu-baseline] [--no-dense]
Under torchrun every rank runs an independent replica (no data-path collective).  After the
timed region the line also carries the end-to-end rate with host buffers (e2e), the dense
comparison (dense: zha_dense_attn against the routed decode, the batch and one query token)
and, on rank 0 at N = 1, the oracle timed on the host cores (cpu_baseline).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hierarchical_tree_indexed_build_b200 import inputs  # noqa: E402

METRIC = "ZHA decode queries/s at 256K & 1M ctx; achieved HBM GB/s vs peak"
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12   # SMs x FP32 lanes x FMA x max SM clock
TENSOR_KERNELS = {"k_score_tc": "f16", "k_attn_tc": "bf16"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--p", type=float, default=0.95)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense-attention comparison")
    ap.add_argument("--no-bf16", action="store_true", help="skip the bf16-record router measurement")
    ap.add_argument("--no-fp4", action="store_true", help="skip the MXFP4-record router measurement")
    ap.add_argument("--no-shard", action="store_true",
                    help="skip the sequence-sharded decode measurement (shards held on this one GPU)")
    ap.add_argument("--shards", type=int, default=2, help="shards of the sharded decode measurement")
    ap.add_argument("--shard", action="store_true",
                    help="under torchrun: one sequence split over the ranks (each rank builds its shard's "
                         "tree and the ranks decode the queries together over NCCL); strong scaling")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip the wide 256K and batched 32 x 128K measurements")
    ap.add_argument("--n-q", type=int, default=0, help="decode only the workload's first n query tokens (profiling)")
    ap.add_argument("--workload", default="deep1m", choices=["deep1m", "deep64k", "deep256k", "wide256k"],
                    help="deep1m is the benchmark; the smaller ones serve profiling runs")
    ap.add_argument("--stage-sweep", default="",
                    help="comma-separated p values: instead of the benchmark line, print one JSON line "
                         "per p with the decode's per-kernel device times and work counters (and one "
                         "for the build), the measurements the stage model is fitted to")
    return ap.parse_args()


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return pk["hbm_gbs"], "measured"
    except Exception:
        return 6650.0, "fallback"


# Kernel -> source file whose contents its DRAM-traffic record was taken against.
KERNEL_SOURCES = {
    "k_score_tc": "zha_score_tc.cu", "k_attn_tc": "zha_attn_tc.cu", "k_select": "zha_route.cu",
    "k_score": "zha_route.cu", "k_attn": "zha_attn.cu", "k_build_stream": "zha_build.cu", "k_build_tc": "zha_build_tc.cu",
}


def source_code_sha256(text: str) -> str:
    """SHA-256 of a C/CUDA source with its comments and blank lines removed, so a traffic
    record stays valid across comment edits but not across code changes."""
    import hashlib
    import re
    t = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    t = re.sub(r"//[^\n]*", "", t)
    lines = [l.rstrip() for l in t.splitlines() if l.strip()]
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()


def measured_traffic(name, workload):
    """DRAM bytes (read + write) per launch of `name` from profiles/traffic.txt, written from
    an ncu capture of this workload (JSON text); None when absent or when the kernel's source
    code has changed since (the record stores source_code_sha256 of the capture-time source)."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.txt")) as f:
            rec = json.load(f)[workload][name]
        src = os.path.join(ROOT, "hierarchical_tree_indexed_build_b200", "csrc", KERNEL_SOURCES[name])
        with open(src, encoding="utf-8") as f:
            if source_code_sha256(f.read()) != rec["source_code_sha256"]:
                return None
        return float(rec["bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def tensor_peak(dtype):
    """Dense tensor peak for the kernel's MMA dtype: the measured bf16 burst figure (fp16
    runs at the bf16 rate, tf32 at half of it)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            bf16, src = json.load(f)["bf16_tflops"], "measured"
    except (OSError, KeyError, ValueError):
        bf16, src = 1590.0, "fallback"
    if dtype == "tf32":
        return bf16 / 2, "%s bf16 x 1/2 (tf32)" % src
    return bf16, "%s bf16%s" % (src, " (f16 runs at the bf16 rate)" if dtype == "f16" else "")


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    def __init__(self, dev: int):
        self.proc = None
        self.path = None
        self.sel = []
        try:
            n = subprocess.run(["nvidia-smi", "-L"], capture_output=True, text=True, timeout=20).stdout
            if len([x for x in n.splitlines() if x.startswith("GPU ")]) > 1:
                self.sel = ["--id=GPU-%s" % str(torch.cuda.get_device_properties(dev).uuid)]
        except Exception:
            pass

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", *self.sel, "--query-gpu=" + q,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 8:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def kernel_algorithmic(name, st, geom, N, n_append, n_lanes, launches):
    """(bytes, flops) one launch of `name` must move/compute (per-unit figure x units),
    from the decoder's work counters of one step."""
    R, d = geom.R, geom.d
    if name in ("k_score", "k_score_tc"):
        nodes = sum(st.union_nodes)
        lane_nodes = sum(st.lane_nodes)
        return ((nodes * st.node_bytes + lane_nodes * 4) / launches, lane_nodes * R * d * 2 / launches)
    if name in ("k_attn", "k_attn_tc"):
        return st.union_tokens * 4 * d / launches, st.lane_tokens * 4 * d / launches
    if name == "k_select":
        return sum(st.lane_nodes) * 4 / launches, 0.0
    if name in ("k_build_tc", "k_build_stream", "k_merge"):
        nodes = sum((N + n_append) // geom.C ** l for l in range(1, geom.L + 1))
        rec = (R * d + 2 * R) * 4
        reads = geom.Hkv * (N + n_append) * 2 * d if name in ("k_build_tc", "k_build_stream") else 0
        return (reads + geom.Hkv * nodes * rec) / launches, 0.0
    return 0.0, 0.0


def kernel_executed_flops(name, st, geom, n_lanes_group, planes, launches):
    """Tensor work one launch of `name` executes: every lane of a (sequence, KV head) group
    against every union node (R rows of d, `planes` passes for the two-plane records), resp.
    every union token (Q K^T and the two P V passes, P = P_hi + P_lo)."""
    R, d = geom.R, geom.d
    if name == "k_score_tc":
        return sum(st.union_nodes) * n_lanes_group * R * d * 2 * planes / launches
    if name == "k_attn_tc":
        return st.union_tokens * n_lanes_group * d * 2 * 3 / launches
    return 0.0


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest of every rank's x (the job's time is its slowest rank's); x itself on one
    rank.  Every rank must call it at the same point."""
    if world <= 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, units_per_rank: int, ms_per_step: float) -> float:
    """Units per second of the whole job: every rank processes units_per_rank per step."""
    return world * units_per_rank / (ms_per_step / 1e3)


def run_ours(args, rank, world, dev):
    from hierarchical_tree_indexed_build_b200 import zha
    torch.cuda.set_device(dev)
    wl = load_workload(args.workload)
    seq = wl.seqs[0]
    g = seq.geom
    N0, n_app = seq.n_tokens, wl.n_append
    Q_host = wl.Q[0].contiguous()                    # [1][128][16][128] bf16
    if args.n_q > 0:
        Q_host = Q_host[:, :args.n_q].contiguous()
    n_q = Q_host.shape[1]
    K = seq.K.to(dev)
    V = seq.V.to(dev)
    qref = seq.qref.to(dev)
    Q = Q_host.to(dev)
    out = torch.empty(Q.shape, dtype=torch.float32, device=dev)
    tree = zha.Tree(g.C, g.L, g.R, g.d, g.Hq, g.Hkv, seq.capacity)
    dec = zha.Decoder([tree], n_q)
    stream = torch.cuda.current_stream()

    def step():
        tree.build(K, N0, qref)
        if n_app:
            tree.append(K, N0, n_app)
        dec.decode([K], [V], Q, args.p, out)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    zha.zha_profile_reset()
    clocks = Clocks(dev)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks.start()
    zha.zha_profile_enable(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    zha.zha_profile_enable(False)
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    prof = zha.zha_profile_read()
    st = dec.stats()
    ms = max_over_ranks(ms, world, dev)
    ms_step = ms / args.steps
    value = whole_job_rate(world, n_q, ms_step)

    # dominant kernel and its roofline
    n_lanes = n_q * g.Hq
    top = max(prof.items(), key=lambda kv: kv[1][1])
    name, (launches, tot_ms) = top
    per_step_launches = launches / args.steps
    nbytes, nflops = kernel_algorithmic(name, st, g, N0, n_app, n_lanes, per_step_launches)
    avg_ms = tot_ms / launches
    hbm_peak, peak_src = measured_peaks()
    intensity = nflops / nbytes if nbytes else 0.0
    if name in TENSOR_KERNELS:
        # executed tensor work: every lane of a group is scored against every union node
        # (resp. attends every union token); the algorithmic figure counts only each lane's
        # own frontier (resp. attended set)
        peak, src = tensor_peak(TENSOR_KERNELS[name])
        ach = nflops / (avg_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
                "traffic": None, "kernel": name, "peak_source": src}
        ex = kernel_executed_flops(name, st, g, n_q * (g.Hq // g.Hkv), 2 if name == "k_score_tc" else 1,
                                   per_step_launches)
        roof["executed_flops_per_launch"] = ex
        roof["executed_frac"] = ex / (avg_ms / 1e3) / 1e12 / peak
    elif nflops and intensity > FP32_PEAK_TFLOPS * 1e12 / (hbm_peak * 1e9):
        ach = nflops / (avg_ms / 1e3) / 1e12
        roof = {"bound": "alu", "achieved": ach, "peak": FP32_PEAK_TFLOPS, "unit": "TFLOP/s",
                "frac": ach / FP32_PEAK_TFLOPS, "traffic": None, "kernel": name,
                "peak_source": "derived: 148 SMs x 128 FP32 lanes x 2 x 1965 MHz"}
    else:
        ach = nbytes / (avg_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": hbm_peak, "unit": "GB/s", "frac": ach / hbm_peak,
                "traffic": None, "kernel": name, "peak_source": peak_src}
    roof["traffic"] = measured_traffic(name, wl.name)
    roof["algorithmic_bytes_per_launch"] = nbytes
    roof["algorithmic_flops_per_launch"] = nflops
    roof["avg_launch_ms"] = avg_ms
    roof["launches"] = launches

    # decode-only throughput and union bytes of the decode
    dec_ms = sum(v[1] for k, v in prof.items()
                 if k in ("k_union", "k_member", "k_score", "k_score_tc", "k_select", "k_attn", "k_attn_tc", "k_combine")) / args.steps
    union_bytes = sum(st.union_nodes) * st.node_bytes + st.union_tokens * 4 * g.d
    stages = {k: round(v[1] / args.steps, 4) for k, v in sorted(prof.items())}
    res = {
        "ms_per_step": ms_step, "value": value, "prof": prof, "roofline": roof, "clocks": clk,
        "gpu_launches": int(sum(v[0] for v in prof.values())),
        "decode_ms": dec_ms, "union_bytes": union_bytes, "n_q": n_q,
        "stats": {"union_nodes": list(st.union_nodes)[:g.L], "lane_nodes": list(st.lane_nodes)[:g.L],
                  "union_tokens": st.union_tokens, "lane_tokens": st.lane_tokens},
        "stages_ms": stages,
    }

    # The dense side of the pages' speedup comparison, after the timed region: exact attention
    # of the same queries over the whole grown cache (no routing) against the routed decode
    # (route + sparse attention) on the same tree, for the whole batch and for one query token.
    if not args.no_dense:
        def timed(fn):
            for _ in range(max(3, args.warmup)):
                fn()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(args.steps):
                fn()
            b.record(stream)
            torch.cuda.synchronize()
            return a.elapsed_time(b) / args.steps

        Q1 = Q[:, :1].contiguous()
        out1 = torch.empty(Q1.shape, dtype=torch.float32, device=dev)
        dense_ms = timed(lambda: dec.dense_attn([K], [V], Q, out))
        zha_ms = timed(lambda: dec.decode([K], [V], Q, args.p, out))
        dense1_ms = timed(lambda: dec.dense_attn([K], [V], Q1, out1))
        zha1_ms = timed(lambda: dec.decode([K], [V], Q1, args.p, out1))
        res["dense"] = {"n_tokens": N0 + n_app, "batch_queries": n_q,
                        "dense_ms": dense_ms, "zha_decode_ms": zha_ms, "speedup": dense_ms / zha_ms,
                        "one_query_dense_ms": dense1_ms, "one_query_zha_decode_ms": zha1_ms,
                        "one_query_speedup": dense1_ms / zha1_ms}

    # The reduced-precision router: the same grown cache indexed by a tree whose records hold
    # the slopes as one bf16 plane (half the bytes per scored node, one tensor-core pass), the
    # same queries decoded; per-kernel times from the library profile.
    if not args.no_bf16:
        tree16 = zha.Tree(g.C, g.L, g.R, g.d, g.Hq, g.Hkv, seq.capacity, zha.ZHA_SUMMARY_BF16)
        tree16.build(K, N0, qref)
        if n_app:
            tree16.append(K, N0, n_app)
        dec16 = zha.Decoder([tree16], n_q)
        out16 = torch.empty_like(out)
        for _ in range(max(3, args.warmup)):
            dec16.decode([K], [V], Q, args.p, out16)
        torch.cuda.synchronize()
        zha.zha_profile_reset()
        zha.zha_profile_enable(True)
        for _ in range(args.steps):
            dec16.decode([K], [V], Q, args.p, out16)
        torch.cuda.synchronize()
        zha.zha_profile_enable(False)
        pr16 = zha.zha_profile_read()
        st16 = dec16.stats()
        d16 = sum(v[1] for v in pr16.values()) / args.steps
        ub16 = sum(st16.union_nodes) * st16.node_bytes + st16.union_tokens * 4 * g.d
        hbm_peak, src = measured_peaks()
        obj = {"format": "bf16 slopes (one plane)", "node_bytes": st16.node_bytes, "decode_ms": d16,
               "queries_per_s": n_q / (d16 / 1e3), "union_gb": ub16 / 1e9,
               "union_frac_of_%s_hbm" % src: ub16 / (d16 / 1e3) / 1e9 / hbm_peak,
               "stages_ms": {k: round(v[1] / args.steps, 4) for k, v in sorted(pr16.items())},
               "max_abs_out_diff_vs_two_plane_tree": float((out16 - out).abs().max().item())}
        for kn in ("k_score_tc", "k_score", "k_score_few"):
            if kn in pr16:
                la, tms = pr16[kn]
                per = la / args.steps
                nb, nf = kernel_algorithmic(kn, st16, g, N0, n_app, n_q * g.Hq, per)
                avg = tms / la
                if kn == "k_score_tc":
                    peak, psrc = tensor_peak("bf16")
                    obj["roofline"] = {"kernel": kn, "bound": "tensor", "achieved": nf / (avg / 1e3) / 1e12,
                                       "peak": peak, "unit": "TFLOP/s", "frac": nf / (avg / 1e3) / 1e12 / peak,
                                       "hbm_frac": nb / (avg / 1e3) / 1e9 / hbm_peak, "avg_launch_ms": avg,
                                       "peak_source": psrc}
                else:
                    obj["roofline"] = {"kernel": kn, "bound": "hbm", "achieved": nb / (avg / 1e3) / 1e9,
                                       "peak": hbm_peak, "unit": "GB/s", "frac": nb / (avg / 1e3) / 1e9 / hbm_peak,
                                       "avg_launch_ms": avg, "peak_source": src}
                break
        res["bf16_router"] = obj
        dec16.close()
        tree16.close()

    # The reduced-precision records where their bytes matter most, the one-query-token decode
    # (16 lanes per sequence: the node scan is a byte stream): the same grown cache indexed by
    # two-plane, bf16 and MXFP4 trees, one query token decoded on each.
    if not args.no_fp4:
        res["fp4_router"] = fp4_measure(args, dev, stream, zha, seq, K, V, qref, Q, N0, n_app, dec, out)

    # The sequence-sharded decode (one sequence split over ranks): the same grown cache cut into
    # shards on whole top nodes, each with its own tree, decoded by the sharded protocol with
    # the shards held by this process on this GPU in lockstep (the collectives become copies
    # on the device); against the single-tree decode of the same queries.
    if not args.no_shard and args.shards >= 2:
        res["sharded"] = sharded_measure(args, dev, stream, zha, seq, K, V, qref, Q, N0 + n_app, dec, out)

    # end to end through the public API with host buffers
    if not args.no_e2e:
        Kh = seq.K.pin_memory()
        Vh = seq.V.pin_memory()
        qh = seq.qref.pin_memory()
        Qh = Q_host.pin_memory()
        outh = torch.empty(out.shape, dtype=torch.float32).pin_memory()

        def step_e2e():
            K.copy_(Kh, non_blocking=True)
            V.copy_(Vh, non_blocking=True)
            qref.copy_(qh, non_blocking=True)
            Q.copy_(Qh, non_blocking=True)
            step()
            outh.copy_(out, non_blocking=True)

        for _ in range(max(1, args.warmup)):
            step_e2e()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        e0.record(stream)
        for _ in range(args.steps):
            step_e2e()
        e1.record(stream)
        torch.cuda.synchronize()
        ems = e0.elapsed_time(e1)
        ems = max_over_ranks(ems, world, dev)
        h2d = sum(x.numel() * x.element_size() for x in (Kh, Vh, qh, Qh))
        res["e2e"] = {"value": whole_job_rate(world, n_q, ems / args.steps), "unit": "queries/s",
                      "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": outh.numel() * 4}
    # the build phase of the benchmark step: tokens/s and the fraction of HBM bandwidth its
    # algorithmic bytes (K read + every node record written) reach
    b_ms = sum(prof.get(k, (0, 0.0))[1] for k in ("k_build_tc", "k_build_stream", "k_merge")) / args.steps
    if b_ms > 0:
        hbm_peak, src = measured_peaks()
        bb = build_bytes(g, N0 + n_app)
        res["build"] = {"tokens": N0 + n_app, "ms": b_ms, "tokens_per_s": (N0 + n_app) / (b_ms / 1e3),
                        "algorithmic_gb": bb / 1e9, "hbm_frac_of_%s" % src: bb / (b_ms / 1e3) / 1e9 / hbm_peak}
    if not args.no_per_workload:
        res["per_workload"] = per_workload(args, dev, stream)
    res["wl"] = wl
    return res


def run_sharded(args, rank, world, dev):
    """One sequence split over the ranks: rank r holds its token range of the workload's cache
    (the last rank also takes the appended tokens), builds its shard's tree and decodes the
    workload's queries with the other ranks through the sharded protocol (NCCL collectives
    between the select phases and for the output merge; device copies when world is 1).
    Step = shard build + append + sharded decode; value = the job's queries per second
    (strong scaling: the work is one sequence whatever the number of ranks)."""
    from hierarchical_tree_indexed_build_b200 import zha
    torch.cuda.set_device(dev)
    wl = load_workload(args.workload)
    seq = wl.seqs[0]
    g = seq.geom
    N0, n_app = seq.n_tokens, wl.n_append
    n_all = N0 + n_app
    off, cnt = zha.shard_ranges(n_all, g.C, g.L, world)[rank]
    cnt0 = min(cnt, max(0, N0 - off))              # rows present before the append
    K = seq.K[:, off:off + cnt].contiguous().to(dev)
    V = seq.V[:, off:off + cnt].contiguous().to(dev)
    qref = seq.qref.to(dev)
    Q = wl.Q[0][0].contiguous().to(dev)           # [n_q][Hq][d]
    n_q = Q.shape[0]
    out = torch.empty((n_q, g.Hq, g.d), dtype=torch.float32, device=dev)
    tree = zha.Tree(g.C, g.L, g.R, g.d, g.Hq, g.Hkv, cnt)
    eng = zha.ShardedDecoder(tree, n_q, rank, world, off)
    coll = zha.TorchCollectives() if world > 1 else None
    stream = torch.cuda.current_stream()

    def step():
        tree.build(K, cnt0, qref)
        if cnt > cnt0:
            tree.append(K, cnt0, cnt - cnt0)
        if coll is None:
            zha.decode_local_shards([eng], [K], [V], Q, args.p, [out])
        else:
            zha.decode_sharded(eng, K, V, Q, args.p, out, coll=coll)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = Clocks(dev)
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / args.steps
    line = base_line(args, world, wl)
    line["config"].update({"parallelism": "sequence sharded over %d ranks" % world,
                           "step": "shard tree build + append + sharded decode of all queries",
                           "shard_tokens": [c for _, c in zha.shard_ranges(n_all, g.C, g.L, world)]})
    line.update({"scaling": "strong", "value": n_q / (ms / 1e3), "ms_per_step": ms, "clocks": clk,
                 "impl": "ours", "vs_baseline": None})
    eng.close()
    tree.close()
    return line


def fp4_measure(args, dev, stream, zha, seq, K, V, qref, Q, N0, n_app, dec, out):
    g = seq.geom
    Q1 = Q[:, :1].contiguous()
    out1 = torch.empty(Q1.shape, dtype=torch.float32, device=dev)
    trees = {"f16x2": None, "bf16": zha.ZHA_SUMMARY_BF16, "fp4": zha.ZHA_SUMMARY_FP4}
    decs, own = {"f16x2": dec}, []
    for name, fmt in trees.items():
        if fmt is None:
            continue
        t = zha.Tree(g.C, g.L, g.R, g.d, g.Hq, g.Hkv, seq.capacity, fmt)
        t.build(K, N0, qref)
        if n_app:
            t.append(K, N0, n_app)
        decs[name] = zha.Decoder([t], Q.shape[1])
        own.append((t, decs[name]))
    hbm_peak, src = measured_peaks()
    obj = {"format": "MXFP4 slopes (E2M1 codes, one E8M0 scale per 32 dims)", "query_tokens": 1,
           "one_query_decode_ms": {}, "node_bytes": {}, "scorer": {}}
    kept = {}
    for name, d in decs.items():
        for _ in range(max(3, args.warmup)):
            d.decode([K], [V], Q1, args.p, out1)
        torch.cuda.synchronize()
        zha.zha_profile_reset()
        zha.zha_profile_enable(True)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            d.decode([K], [V], Q1, args.p, out1)
        b.record(stream)
        torch.cuda.synchronize()
        zha.zha_profile_enable(False)
        pr = zha.zha_profile_read()
        st = d.stats()
        obj["one_query_decode_ms"][name] = a.elapsed_time(b) / args.steps
        obj["node_bytes"][name] = st.node_bytes
        for kn in ("k_score_tc", "k_score_few", "k_score"):
            if kn in pr:
                la, tms = pr[kn]
                nb = sum(st.union_nodes) * st.node_bytes
                obj["scorer"][name] = {"kernel": kn, "ms_per_decode": tms / args.steps,
                                       "union_node_gb": nb / 1e9,
                                       "hbm_frac_of_%s" % src: nb / (tms / args.steps / 1e3) / 1e9 / hbm_peak}
                break
        kept[name] = d.export_kept(1)[0].cpu().numpy()
    # the float32-grade router's attended level-1 chunks that each reduced router also attends
    base = np.unpackbits(np.ascontiguousarray(kept["f16x2"]).view(np.uint8), axis=1, bitorder="little").astype(bool)
    for name in ("bf16", "fp4"):
        other = np.unpackbits(np.ascontiguousarray(kept[name]).view(np.uint8), axis=1, bitorder="little").astype(bool)
        rec = [(base[x] & other[x]).sum() / max(1, base[x].sum()) for x in range(base.shape[0])]
        obj.setdefault("kept_chunk_recall_vs_f16x2", {})[name] = {"min": float(min(rec)), "mean": float(np.mean(rec))}
    for t, d in own:
        d.close()
        t.close()
    return obj


def sharded_measure(args, dev, stream, zha, seq, K, V, qref, Q, n_tok, dec, out):
    g = seq.geom
    world = args.shards
    ranges = zha.shard_ranges(n_tok, g.C, g.L, world)
    n_q = Q.shape[1]
    shards = []
    for r, (off, cnt) in enumerate(ranges):
        Ks = K[:, off:off + cnt].contiguous()
        Vs = V[:, off:off + cnt].contiguous()
        t = zha.Tree(g.C, g.L, g.R, g.d, g.Hq, g.Hkv, cnt)
        t.build(Ks, cnt, qref)
        shards.append((t, Ks, Vs, zha.ShardedDecoder(t, n_q, r, world, off)))
    outs = [torch.empty((n_q, g.Hq, g.d), dtype=torch.float32, device=dev) for _ in shards]
    Q3 = Q[0]

    def run():
        zha.decode_local_shards([s[3] for s in shards], [s[1] for s in shards], [s[2] for s in shards],
                                Q3, args.p, outs)

    def timed(fn):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / args.steps

    sh_ms = timed(run)
    one_ms = timed(lambda: dec.decode([K], [V], Q, args.p, out))
    diff = float((outs[0] - out[0]).abs().max().item())
    # kept sets of every shard against the single tree's, at every level (must be identical)
    same = True
    for lev in range(1, g.L + 1):
        bits1, _ = dec.export_kept(lev)
        span = g.C ** lev
        for (t, _, _, e), (off, cnt) in zip(shards, ranges):
            n_l = cnt // span
            b = e.export_kept(lev)[0]
            w1 = torch.from_numpy(_bits_slice(bits1.cpu().numpy(), off // span, n_l))
            w2 = torch.from_numpy(_bits_slice(b.cpu().numpy(), 0, n_l))
            same &= bool(torch.equal(w1, w2))
    lanes = n_q * g.Hq
    ex_level = lanes * (4 + 4 + zha.SHARD_BINS * 8 + world * (zha.SHARD_KEYS * 8 + 4))
    ex_attn = world * lanes * (g.d + 1) * 4
    obj = {"shards": world, "token_ranges": ranges, "decode_ms": sh_ms, "single_tree_decode_ms": one_ms,
           "overhead": sh_ms / one_ms, "kept_sets_identical_to_single_tree": same,
           "max_abs_out_diff_vs_single_tree": diff,
           "exchange_bytes_per_rank_per_decode": g.L * ex_level + ex_attn,
           "collectives_per_decode": 5 * g.L + 2,
           "note": "shards held by one process on one GPU in lockstep: the collectives are device copies"}
    for t, _, _, e in shards:
        e.close()
        t.close()
    return obj


def _bits_slice(bits, start, n):
    """Bits [start, start + n) of each row of a uint32-word bitmap, as a bool array."""
    b = np.ascontiguousarray(bits).view(np.uint8).reshape(bits.shape[0], -1)
    u = np.unpackbits(b, axis=1, bitorder="little")
    return u[:, start:start + n].astype(bool)


def build_bytes(g, n_tokens):
    """Bytes a build over n_tokens must move: K read (2d B per token per KV head) and every
    complete node's record written ((R d + 2R) 4 B: m and b, and lse)."""
    nodes = sum(n_tokens // g.C ** l for l in range(1, g.L + 1))
    return g.Hkv * (n_tokens * 2 * g.d + nodes * (g.R * g.d + 2 * g.R) * 4)


def per_workload(args, dev, stream):
    """The other geometries of the metric, each timed with CUDA events on its own (after the
    benchmark's timed region): the wide 256K tree (C256 L1) - build over the whole cache
    and the decode of its 64 queries - and the batched workload (32 x 131,072 tokens, half
    C16 L3, half C4 L6) - one appended token and one decoded query per sequence per step."""
    from hierarchical_tree_indexed_build_b200 import zha
    hbm_peak, src = measured_peaks()
    frac_key = "hbm_frac_of_%s" % src
    out = {}

    def timed(fn, reps):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    # wide 256K
    wl = inputs.wide_256k()
    seq = wl.seqs[0]
    g = seq.geom
    K, V, qr = seq.K.to(dev), seq.V.to(dev), seq.qref.to(dev)
    Q = wl.Q[0].to(dev).contiguous()
    tree = zha.Tree(g.C, g.L, g.R, g.d, g.Hq, g.Hkv, seq.capacity)
    n = seq.n_tokens
    bms = timed(lambda: tree.build(K, n, qr), args.steps)
    dec = zha.Decoder([tree], Q.shape[1])
    o = torch.empty(Q.shape, dtype=torch.float32, device=dev)
    dms = timed(lambda: dec.decode([K], [V], Q, args.p, o), args.steps)
    st = dec.stats()
    ub = sum(st.union_nodes) * st.node_bytes + st.union_tokens * 4 * g.d
    bb = build_bytes(g, n)
    out["wide_256k_C256L1"] = {
        "n_tokens": n, "queries": int(Q.shape[1]), "p": args.p,
        "decode_ms": dms, "queries_per_s": Q.shape[1] / (dms / 1e3),
        "union_gb": ub / 1e9, "union_" + frac_key: ub / (dms / 1e3) / 1e9 / hbm_peak,
        "keys_touched_frac": st.lane_tokens / (Q.shape[1] * g.Hq * n),
        "build_ms": bms, "build_tokens_per_s": n / (bms / 1e3), "build_" + frac_key: bb / (bms / 1e3) / 1e9 / hbm_peak}
    dec.close()
    tree.close()
    del K, V, qr, Q, o

    # batched 32 x 128K, mixed geometries, 1-token append + 1 query per sequence per step
    n_steps = max(3, args.warmup) + args.steps
    wl = inputs.batched_32x128k(n_steps=n_steps)
    trees, Ks, Vs = [], [], []
    for sq in wl.seqs:
        gg = sq.geom
        Kd, Vd = sq.K.to(dev), sq.V.to(dev)
        t = zha.Tree(gg.C, gg.L, gg.R, gg.d, gg.Hq, gg.Hkv, sq.capacity)
        t.build(Kd, sq.n_tokens, sq.qref.to(dev))
        trees.append(t)
        Ks.append(Kd)
        Vs.append(Vd)
    dec = zha.Decoder(trees, 1)
    Qs = wl.Q.to(dev)                               # [steps][32][1][16][128]
    o = torch.empty(Qs.shape[1:], dtype=torch.float32, device=dev)
    step = [0]

    def bstep():
        k = step[0]
        for s, sq in enumerate(wl.seqs):
            trees[s].append(Ks[s], sq.n_tokens + k, 1)
        dec.decode(Ks, Vs, Qs[k], args.p, o)
        step[0] += 1

    sms = timed(bstep, args.steps)
    st = dec.stats()
    ub = sum(st.union_nodes) * st.node_bytes + st.union_tokens * 4 * 128
    toks = sum(sq.n_tokens + step[0] for sq in wl.seqs)
    out[wl.name] = {
        "sequences": len(wl.seqs), "n_tokens_per_seq": wl.seqs[0].n_tokens, "queries_per_step": len(wl.seqs),
        "p": args.p, "step": "1-token append per sequence + decode of one query per sequence",
        "step_ms": sms, "queries_per_s": len(wl.seqs) / (sms / 1e3),
        "union_gb_last_step": ub / 1e9, "union_" + frac_key: ub / (sms / 1e3) / 1e9 / hbm_peak,
        "keys_touched_frac": st.lane_tokens / (16 * toks)}
    dec.close()
    for t in trees:
        t.close()
    return out


def stage_sweep(args, dev):
    """Per-kernel device times (library CUDA-event profile) and the decoder's work counters
    of the workload's build and of its decode at each p, one JSON line each."""
    from hierarchical_tree_indexed_build_b200 import zha
    torch.cuda.set_device(dev)
    wl = load_workload(args.workload)
    seq = wl.seqs[0]
    g = seq.geom
    N0, n_app = seq.n_tokens, wl.n_append
    K, V, qref = seq.K.to(dev), seq.V.to(dev), seq.qref.to(dev)
    Q = wl.Q[0].contiguous()
    if args.n_q > 0:
        Q = Q[:, :args.n_q].contiguous()
    Q = Q.to(dev)
    tree = zha.Tree(g.C, g.L, g.R, g.d, g.Hq, g.Hkv, seq.capacity)
    dec = zha.Decoder([tree], Q.shape[1])
    out = torch.empty(Q.shape, dtype=torch.float32, device=dev)
    geom = {"C": g.C, "L": g.L, "R": g.R, "d": g.d, "Hq": g.Hq, "Hkv": g.Hkv}

    def profiled(fn, reps):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize()
        zha.zha_profile_reset()
        zha.zha_profile_enable(True)
        for _ in range(reps):
            fn()
        torch.cuda.synchronize()
        zha.zha_profile_enable(False)
        pr = zha.zha_profile_read()
        return ({k: v[1] / reps for k, v in pr.items()}, {k: v[0] / reps for k, v in pr.items()})

    def build():
        tree.build(K, N0, qref)
        if n_app:
            tree.append(K, N0, n_app)

    ms, la = profiled(build, args.steps)
    print(json.dumps({"workload": wl.name, "stage": "build", "n_tokens": N0 + n_app, "geometry": geom,
                      "kernel_ms": ms, "kernel_launches": la}))
    for p in [float(x) for x in args.stage_sweep.split(",") if x]:
        for nq in sorted({int(Q.shape[1]), 1}):
            Qp = Q[:, :nq].contiguous()
            op = out[:, :nq].contiguous()
            ms, la = profiled(lambda: dec.decode([K], [V], Qp, p, op), args.steps)
            st = dec.stats()
            print(json.dumps({"workload": wl.name, "stage": "decode", "p": p, "n_q": nq, "n_tokens": N0 + n_app,
                              "geometry": geom, "kernel_ms": ms, "kernel_launches": la,
                              "stats": {"union_nodes": list(st.union_nodes)[:g.L],
                                        "lane_nodes": list(st.lane_nodes)[:g.L],
                                        "union_tokens": st.union_tokens, "lane_tokens": st.lane_tokens,
                                        "node_bytes": st.node_bytes}}))
    dec.close()
    tree.close()


def load_workload(name):
    if name == "deep64k":
        wl = inputs.deep_64k()
        wl.n_append = 0
        return wl
    if name == "wide256k":
        wl = inputs.wide_256k()
        wl.n_append = 0
        return wl
    if name == "deep256k":
        # the 1M workload's shapes over 262,144 tokens: K/V and tree (1.7 GB) exceed L2 while a
        # full ncu capture stays small
        wl = inputs.deep_1m(n_tokens=262144, n_append=0)
        wl.name = "deep_256k_C4L6"
        return wl
    return inputs.deep_1m()


def cpu_baseline(wl, p, min_s=10.0, max_queries=64):
    """The float64 oracle as it stands on a bounded sample of the same workload: query
    tokens (16 heads each) routed and attended one after another until about min_s
    seconds of CPU work have been spent."""
    from oracle import oracle as O
    seq = wl.seqs[0]
    g = seq.geom
    N = seq.n_tokens + wl.n_append
    K = seq.K.to(torch.float64).numpy()
    V = seq.V.to(torch.float64).numpy()
    qref = seq.qref.to(torch.float64).numpy()
    lane_g = np.array([h * g.Hkv // g.Hq for h in range(g.Hq)], dtype=np.int32)
    O.lib()
    done = 0
    t0 = time.perf_counter()
    while done < max_queries and (time.perf_counter() - t0) < min_s:
        q = wl.Q[0, 0, done].to(torch.float64).numpy()          # [Hq][d]
        O.decode(K, V, qref, g.C, g.L, N, q, lane_g, p)
        done += 1
    dt = time.perf_counter() - t0
    return {"value": done / dt, "unit": "queries/s", "cores": O.num_threads(), "kind": "oracle",
            "sample": "%d query tokens x %d heads of the %s workload (N=%d), float64 routing with "
                      "definition-level summaries + exact attention, %.1f s" % (done, g.Hq, wl.name, N, dt)}


def base_line(args, world, wl):
    seq = wl.seqs[0]
    g = seq.geom
    n = seq.n_tokens + wl.n_append
    kv_gb = 2 * g.Hkv * n * g.d * 2 / 1e9
    tree_gb = g.Hkv * sum(n // g.C ** l for l in range(1, g.L + 1)) * (g.R * g.d + 2 * g.R) * 4 / 1e9
    return {
        "metric": METRIC, "unit": "queries/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": wl.name, "n_tokens_build": seq.n_tokens, "n_append": wl.n_append,
                   "n_queries": int(wl.Q.shape[2]), "p": args.p, "C": g.C, "L": g.L, "R": g.R, "d": g.d,
                   "Hq": g.Hq, "Hkv": g.Hkv, "step": "build + append + decode of all queries",
                   "parallelism": "replicas" if world > 1 else "single",
                   "inputs": "bf16 K, V, Q and reference queries; f32 summaries, scores and outputs",
                   "l2": "inputs larger than L2 (K+V %.2f GB, tree %.2f GB; L2 126 MB), no flush" % (kv_gb, tree_gb)},
    }


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return
        wl = load_workload(args.workload)
        for _ in range(args.warmup):
            pass   # the oracle has no warm-up state; each step below is a full sample
        vals = [cpu_baseline(wl, args.p) for _ in range(args.steps)]
        v = statistics.median(x["value"] for x in vals)
        line = base_line(args, 1, wl)
        line.update({"impl": "reference", "value": v, "ms_per_step": 1e3 / v,
                     "cpu_baseline": dict(vals[0], value=v),
                     "e2e": {"value": v, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}})
        print(json.dumps(line))
        return
    if args.stage_sweep:
        if rank == 0:
            stage_sweep(args, local)
        return
    if world > 1:
        torch.distributed.init_process_group("nccl", device_id=torch.device("cuda", local),
                                             timeout=__import__("datetime").timedelta(seconds=120))
    if args.shard:
        line = run_sharded(args, rank, world, local)
        if rank == 0:
            print(json.dumps(line))
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        return
    res = run_ours(args, rank, world, local)
    wl = res.pop("wl")
    if rank == 0:
        line = base_line(args, world, wl)
        line.update({"value": res["value"], "ms_per_step": res["ms_per_step"], "roofline": res["roofline"],
                     "gpu_launches": res["gpu_launches"], "clocks": res["clocks"]})
        if "e2e" in res:
            line["e2e"] = res["e2e"]
        nq = res["n_q"]
        line["config"]["n_queries"] = nq
        hbm_peak, src = measured_peaks()
        line["decode"] = {"ms_per_step": res["decode_ms"],
                          "queries_per_s": nq / (res["decode_ms"] / 1e3),
                          "union_gb": res["union_bytes"] / 1e9,
                          "union_gbs": res["union_bytes"] / (res["decode_ms"] / 1e3) / 1e9,
                          "union_frac_of_%s_hbm" % src: res["union_bytes"] / (res["decode_ms"] / 1e3) / 1e9 / hbm_peak,
                          "keys_touched_frac": res["stats"]["lane_tokens"] / (
                              nq * wl.seqs[0].geom.Hq * (wl.seqs[0].n_tokens + wl.n_append))}
        line["stages_ms"] = res["stages_ms"]
        line["stats"] = res["stats"]
        if "dense" in res:
            line["dense"] = res["dense"]
        if "build" in res:
            line["build"] = res["build"]
        if "per_workload" in res:
            line["per_workload"] = res["per_workload"]
        if "bf16_router" in res:
            line["bf16_router"] = res["bf16_router"]
        if "sharded" in res:
            line["sharded"] = res["sharded"]
        if "fp4_router" in res:
            line["fp4_router"] = res["fp4_router"]
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl, args.p)
        print(json.dumps(line))
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
