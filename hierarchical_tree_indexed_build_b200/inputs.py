"""Seeded synthetic inputs for ZHA tree build and tree-routed decode.

This module only draws random numbers and rounds them to bf16.  It holds none
of the method's arithmetic (no summaries, no routing, no attention) and is the
one module shared by the CUDA path's tests/benchmark and by the float64 oracle.

Workloads stand in for the pages' long-context retrieval settings (needle
queries at 64K-256K, 1M projections); the evaluation suites themselves are not
used.  Recipe (one numpy ``Generator(PCG64)`` per purpose, spawned from the
workload seed):

* keys:    K[g, t] = mu_g + N(0, 1) per dimension, mu_g ~ N(0, 0.5^2) per KV head
           (the tiny case uses K ~ N(0, 1) with no mean);
* values:  V ~ N(0, 1);
* reference queries q_r ~ N(0, 1), R per KV head, shared by the sequences of
  one geometry;
* decode queries: for each query token draw needle positions uniformly over the
  cache, and for every query head h (KV head g = h * Hkv // Hq)
  q_h = mean_n(3 * K[g, needle_n]) + N(0, 1) noise, independently per head;
* everything is drawn in float32 and rounded once to bf16 (round to nearest
  even) - the exact bf16 values are what both sides consume.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np
import torch


@dataclass(frozen=True)
class Geometry:
    """Tree geometry: chunk size C, levels L, reference queries R, head dim d."""
    C: int
    L: int
    R: int
    d: int
    Hq: int
    Hkv: int

    @property
    def top_span(self) -> int:
        return self.C ** self.L


@dataclass
class Sequence:
    geom: Geometry
    n_tokens: int            # tokens present when the tree is built
    capacity: int            # rows allocated per KV head (n_tokens + appended)
    K: torch.Tensor          # bf16 [Hkv][capacity][d], CPU
    V: torch.Tensor          # bf16 [Hkv][capacity][d], CPU
    qref: torch.Tensor       # bf16 [Hkv][R][d], CPU


@dataclass
class Workload:
    name: str
    seqs: List[Sequence]
    Q: torch.Tensor                  # bf16 [n_steps][n_seq][n_q][Hq][d], CPU
    needles: List                    # per step, per seq, per query: np.ndarray of positions
    p_values: List[float]
    n_append: int = 0                # tokens appended per sequence before the queries
    append_per_step: int = 0         # tokens appended per sequence before each step
    meta: dict = field(default_factory=dict)


def _bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def _streams(seed: int, n: int):
    return [np.random.Generator(np.random.PCG64(s)) for s in np.random.SeedSequence(seed).spawn(n)]


def make_sequence(geom: Geometry, n_tokens: int, capacity: int, seed: int,
                  qref: Optional[torch.Tensor] = None, key_mean_std: float = 0.5) -> Sequence:
    rk, rv, rq = _streams(seed, 3)
    Hkv, d = geom.Hkv, geom.d
    K = rk.standard_normal((Hkv, capacity, d), dtype=np.float32)
    if key_mean_std > 0.0:
        mu = rk.standard_normal((Hkv, 1, d), dtype=np.float32) * np.float32(key_mean_std)
        K += mu
    V = rv.standard_normal((Hkv, capacity, d), dtype=np.float32)
    if qref is None:
        qref = _bf16(rq.standard_normal((Hkv, geom.R, d), dtype=np.float32))
    return Sequence(geom=geom, n_tokens=n_tokens, capacity=capacity, K=_bf16(K), V=_bf16(V), qref=qref)


def make_queries(seq: Sequence, n_q: int, n_needles, length: int, rng: np.random.Generator):
    """Needle queries against the first ``length`` tokens of ``seq``.

    ``n_needles`` is an int or a (lo, hi) inclusive range drawn uniformly per query.
    Returns (Q bf16 [n_q][Hq][d], list of needle arrays).
    """
    g = seq.geom
    Kf = seq.K  # bf16
    Q = np.empty((n_q, g.Hq, g.d), dtype=np.float32)
    needles = []
    for i in range(n_q):
        if isinstance(n_needles, tuple):
            cnt = int(rng.integers(n_needles[0], n_needles[1] + 1))
        else:
            cnt = int(n_needles)
        pos = rng.integers(0, length, size=cnt)
        needles.append(pos)
        for h in range(g.Hq):
            kv = h * g.Hkv // g.Hq
            keys = Kf[kv, torch.from_numpy(pos)].to(torch.float32).numpy()
            Q[i, h] = 3.0 * keys.mean(axis=0) + rng.standard_normal(g.d, dtype=np.float32)
    return _bf16(Q), needles


# --------------------------------------------------------------------------------------
# The five workloads.  Sizes default to the full configurations; tests pass smaller
# values (same shapes otherwise) where the oracle has to finish in seconds.
# --------------------------------------------------------------------------------------

TINY = Geometry(C=4, L=3, R=4, d=64, Hq=1, Hkv=1)
DEEP = Geometry(C=4, L=6, R=16, d=128, Hq=16, Hkv=2)
WIDE = Geometry(C=256, L=1, R=16, d=128, Hq=16, Hkv=2)
MID = Geometry(C=16, L=3, R=16, d=128, Hq=16, Hkv=2)


def tiny_4k(seed: int = 0, n_tokens: int = 4096, n_q: int = 16) -> Workload:
    """1 sequence, N=4096, 1/1 heads, d=64, K,V ~ N(0,1), R=4, C=4, L=3, p in {0.9, 1}."""
    seq = make_sequence(TINY, n_tokens, n_tokens, seed, key_mean_std=0.0)
    (rq,) = _streams(seed + 1000, 1)
    Q, nd = make_queries(seq, n_q, 1, n_tokens, rq)
    return Workload("tiny_4k_d64_C4L3", [seq], Q[None, None], [[nd]], [0.9, 1.0])


def deep_64k(seed: int = 1, n_tokens: int = 65536, n_q: int = 64) -> Workload:
    """Batch 1, N=65,536, GQA 16/2, d=128, R=16, C=4, L=6, p=0.95, 8 needles per query."""
    seq = make_sequence(DEEP, n_tokens, n_tokens, seed)
    (rq,) = _streams(seed + 1000, 1)
    Q, nd = make_queries(seq, n_q, 8, n_tokens, rq)
    return Workload("deep_64k_C4L6", [seq], Q[None, None], [[nd]], [0.95])


def wide_256k(seed: int = 2, n_tokens: int = 262144, n_q: int = 64) -> Workload:
    """Batch 1, N=262,144, GQA 16/2, d=128, R=16, C=256, L=1, p=0.95, 1..32 needles."""
    seq = make_sequence(WIDE, n_tokens, n_tokens, seed)
    (rq,) = _streams(seed + 1000, 1)
    Q, nd = make_queries(seq, n_q, (1, 32), n_tokens, rq)
    return Workload("wide_256k_C256L1", [seq], Q[None, None], [[nd]], [0.95])


def deep_1m(seed: int = 3, n_tokens: int = 1048576, n_q: int = 128, n_append: int = 4096) -> Workload:
    """Batch 1, N=1,048,576 (+4,096 appended), GQA 16/2, d=128, R=16, C=4, L=6,
    p in {0.7, 0.9, 0.95, 0.99}, 128 queries with 8 needles over the grown cache."""
    cap = n_tokens + n_append
    seq = make_sequence(DEEP, n_tokens, cap, seed)
    (rq,) = _streams(seed + 1000, 1)
    Q, nd = make_queries(seq, n_q, 8, cap, rq)
    return Workload("deep_1m_C4L6", [seq], Q[None, None], [[nd]], [0.7, 0.9, 0.95, 0.99],
                    n_append=n_append)


def batched_32x128k(seed: int = 4, n_seq: int = 32, n_tokens: int = 131072,
                    n_steps: int = 256) -> Workload:
    """n_seq independent sequences x N tokens, half C=16 L=3 and half C=4 L=6 (R=16,
    p=0.95); each step appends one token per sequence and then decodes one query per
    sequence with 8 needles over the current cache."""
    cap = n_tokens + n_steps
    streams = _streams(seed, 3)
    qref_mid = _bf16(streams[0].standard_normal((MID.Hkv, MID.R, MID.d), dtype=np.float32))
    qref_deep = _bf16(streams[1].standard_normal((DEEP.Hkv, DEEP.R, DEEP.d), dtype=np.float32))
    seqs = []
    for s in range(n_seq):
        geom, qr = (MID, qref_mid) if s < n_seq // 2 else (DEEP, qref_deep)
        seqs.append(make_sequence(geom, n_tokens, cap, seed * 1000 + s, qref=qr))
    rq = streams[2]
    Qs = np.empty((n_steps, n_seq, 1, DEEP.Hq, DEEP.d), dtype=np.float32)
    needles = []
    for t in range(n_steps):
        row = []
        for s, seq in enumerate(seqs):
            q, nd = make_queries(seq, 1, 8, n_tokens + t + 1, rq)
            Qs[t, s] = q.to(torch.float32).numpy()
            row.append(nd)
        needles.append(row)
    return Workload("batched_%dx%dk_mixed" % (n_seq, n_tokens // 1024), seqs, _bf16(Qs), needles,
                    [0.95], append_per_step=1)


WORKLOADS = {
    "tiny": tiny_4k,
    "deep64k": deep_64k,
    "wide256k": wide_256k,
    "deep1m": deep_1m,
    "batched": batched_32x128k,
}
