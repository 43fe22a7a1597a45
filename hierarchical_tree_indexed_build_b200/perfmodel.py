"""Stage-wise B200 model of one decode step: dense flash-decode against the tree-routed decode.

The pages model their speedups with a three-term roofline per stage of the decode (tree
build, per-level routing, node scan, final exact attention) plus a worker-wave term for idle
parallelism ("Zyphra ZHA 稀疏注意力…", fluxbbs.com, section 加速数字需要打折看待).  This module
is that model with B200 numbers:

* a byte roofline for every stage at the measured HBM bandwidth (the decode of a few query
  tokens reads far more bytes than it multiplies: dense attention streams K and V, the router
  streams the scored nodes' records, the sparse attention gathers the kept tokens' K and V);
* a per-level latency term for the routed decode (its levels are dependent launches), fitted
  to this implementation's one-query decode at 1M tokens;
* routed sizes either given (the decoder's statistics of a real run) or from a fixed kept
  budget per level (each lane keeps k nodes per level, so the scored frontier does not grow
  with the context), the assumption under which routed attention beats dense at long context.

All times are per decode step of one layer, in milliseconds.  Nothing here runs on the GPU.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, List, Sequence

HBM_GBS = 6455.3            # measured STREAM-style copy on this machine's B200 (GB/s)
HBM_CAPACITY_GB = 180.0


def record_bytes(R: int, d: int) -> int:
    """Bytes of one node's record as stored: m as fp16 hi + lo planes [R][d] each, plus
    lse and b in f32 per reference query."""
    return R * d * 2 * 2 + 2 * R * 4


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


@dataclass
class Fit:
    """Per-level latency of the routed decode (ms): the part of the measured one-query decode
    that the byte roofline does not explain, divided by its levels.  Fitted to the 1M deep
    tree (C4 L6, R16, d128, GQA 16/2), one query token, p = 0.7: routed decode 1.826 ms with
    237,254 union nodes scored and 169,090 union tokens attended (bench `dense` object and
    decoder statistics)."""
    level_ms: float = 0.25


def dense_ms(N: int, d: int, Hkv: int, bw_gbs: float = HBM_GBS) -> float:
    """Dense flash-decode lower bound: K and V of all N tokens read once."""
    return N * kv_bytes_per_token(d, Hkv) / (bw_gbs * 1e9) * 1e3


def routed_bytes(union_nodes: Sequence[int], union_tokens: int, R: int, d: int, Hkv: int) -> float:
    """Bytes the routed decode must move: every scored node's record (union_nodes summed over
    the KV-head groups, as the decoder reports them) plus the gathered K/V rows of the union of
    attended tokens (summed over groups, one KV head each)."""
    return sum(union_nodes) * record_bytes(R, d) + union_tokens * kv_bytes_per_token(d, 1)


def routed_ms(union_nodes: Sequence[int], union_tokens: int, R: int, d: int, Hkv: int,
              fit: Fit = Fit(), bw_gbs: float = HBM_GBS, latency: bool = True) -> float:
    """Routed decode: byte roofline plus, with latency, the fitted per-level term."""
    t = routed_bytes(union_nodes, union_tokens, R, d, Hkv) / (bw_gbs * 1e9) * 1e3
    return t + (fit.level_ms * len(union_nodes) if latency else 0.0)


def fixed_budget_sizes(N: int, C: int, L: int, k: int, lanes_per_group: int, Hkv: int):
    """Routed sizes when every lane keeps k nodes per level: the top level is scored whole;
    below it each lane scores the C children of its k kept parents, and a group's union is at
    most its lanes times that (no overlap assumed, an upper bound) and at most the level.
    Attended tokens per group: the lanes' kept level-1 chunks, the sink and the tail."""
    n = level_nodes(N, C, L)
    union = []
    for l in range(L, 0, -1):
        per_group = n[l - 1] if l == L else min(n[l - 1], lanes_per_group * k * C)
        union.append(per_group * Hkv)
    tail = N - n[L - 1] * C ** L
    tokens = (min(N, lanes_per_group * k * C) + 1 + tail) * Hkv
    return union, tokens


def project(Ns: Sequence[int], C: int = 4, R: int = 16, d: int = 128, Hq: int = 16, Hkv: int = 2,
            k: int = 64, fit: Fit = Fit()) -> List[Dict[str, float]]:
    """One query token per step: dense lower bound against the routed decode under a fixed
    kept budget, with and without the fitted per-level latency."""
    G = Hq // Hkv
    rows = []
    for N in Ns:
        L = levels_for(N, C)
        union, tokens = fixed_budget_sizes(N, C, L, k, G, Hkv)
        dn = dense_ms(N, d, Hkv)
        rb = routed_ms(union, tokens, R, d, Hkv, fit, latency=False)
        rl = routed_ms(union, tokens, R, d, Hkv, fit, latency=True)
        rows.append({"N": N, "L": L, "kv_gb": N * kv_bytes_per_token(d, Hkv) / 1e9,
                     "fits_one_gpu": N * kv_bytes_per_token(d, Hkv) / 1e9 <= HBM_CAPACITY_GB,
                     "dense_ms": dn, "routed_bytes_ms": rb, "routed_ms": rl,
                     "speedup_bytes": dn / rb, "speedup": dn / rl})
    return rows


def main() -> None:
    import argparse
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--k", type=int, nargs="+", default=[64, 1024],
                    help="kept nodes per lane per level (fixed budget)")
    args = ap.parse_args()
    print("record bytes per node (R16, d128): %d; K+V bytes of its C = 4 tokens on one KV head: %d"
          % (record_bytes(16, 128), 4 * kv_bytes_per_token(128, 1)))
    for k in args.k:
        print("\nkept budget k = %d nodes per lane per level, one query token (16 heads, GQA 16/2)" % k)
        print("%12s %3s %9s %5s %11s %14s %11s %9s %9s" % ("N", "L", "KV GB", "1GPU", "dense ms",
                                                        "routed(bytes)", "routed ms", "x bytes", "x model"))
        for r in project([262144, 1 << 20, 10 << 20, 100 << 20, 1 << 30], k=k):
            print("%12d %3d %9.1f %5s %11.3f %14.3f %11.3f %9.2f %9.2f" % (
                r["N"], r["L"], r["kv_gb"], "yes" if r["fits_one_gpu"] else "no", r["dense_ms"],
                r["routed_bytes_ms"], r["routed_ms"], r["speedup_bytes"], r["speedup"]))


if __name__ == "__main__":
    main()
