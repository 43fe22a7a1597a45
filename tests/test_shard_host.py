"""Host logic of the sequence-sharded decode on CPU.

* ``shard_ranges`` / ``check_shard_ranges``: the token ranges of the ranks.
* The protocol (``zha.shard_steps`` with ``zha.TorchCollectives``) over a world of 2 and 3
  gloo ranks, driving a test double of the shard engine that takes each phase in numpy
  (float64 estimates from the oracle's summaries, the fixed-point mass histogram, the
  boundary keys with global node indices, attention with its log-sum-exp).  The union of
  the ranks' kept nodes must equal, bit for bit, the same double's cut over the whole
  sequence as one shard (world 1), and the merged output must equal the oracle's attention
  over the attended set: this checks the order of the steps, what each collective does
  (MAX of ordered int32, SUM of 64-bit integers, rank-major gathers), the global node
  indices of the boundary keys, the sink on rank 0, the tail on the last rank and the
  log-sum-exp merge.
"""
import json
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from hierarchical_tree_indexed_build_b200 import zha
from oracle import oracle as O

BINS, KEYS = zha.SHARD_BINS, zha.SHARD_KEYS
C, L, R, D, HQ, HKV = 4, 2, 4, 16, 4, 2


def test_shard_ranges_tile_the_sequence():
    for n, world in [(10 * 4096 + 77, 3), (4 * 4096, 4), (4096 + 5, 1), (7 * 4096, 2), (100, 2)]:
        rs = zha.shard_ranges(n, 4, 6, world)
        assert len(rs) == world
        assert zha.check_shard_ranges(rs, 4, 6) == n
        assert all(c % 4096 == 0 for _, c in rs[:-1])
        # the non-last ranks hold as many whole top nodes as an even split allows
        assert all(c == rs[0][1] for _, c in rs[:-1])


def test_check_shard_ranges_rejects_bad_layouts():
    with pytest.raises(ValueError):
        zha.check_shard_ranges([(0, 4096), (4097, 100)], 4, 6)        # gap
    with pytest.raises(ValueError):
        zha.check_shard_ranges([(0, 4000), (4000, 100)], 4, 6)        # rank 0 splits a top node
    with pytest.raises(ValueError):
        zha.check_shard_ranges([(0, 4096 * 4096 * 4 + 4096), (4096 * 4096 * 4 + 4096, 8)], 4, 6)   # > 2^24 chunks
    assert zha.check_shard_ranges([(0, 4096), (4096, 5)], 4, 6) == 4101


# ------------------------------------------------------------------ the test double

def _ord_i32(e: float) -> int:
    u = int(np.float32(e).view(np.uint32))
    o = (~u & 0xFFFFFFFF) if (u & 0x80000000) else (u | 0x80000000)
    return int(np.uint32(o ^ 0x80000000).view(np.int32))


def _from_ord_i32(v: int) -> float:
    o = int(np.int32(v).view(np.uint32)) ^ 0x80000000
    u = (o ^ 0x80000000) if (o & 0x80000000) else (~o & 0xFFFFFFFF)
    return float(np.uint32(u).view(np.float32))


def _mass(e: float, M: float) -> int:
    return int(math.floor(float(np.float32(math.exp(e - M))) * 2.0 ** 39))


def _bin(e: float, M: float) -> int:
    return int(min(BINS - 1, max(0, np.rint((M - e) * 64.0))))


def _key(e: float, j: int) -> int:
    u = int(np.float32(e).view(np.uint32))
    o = (~u & 0xFFFFFFFF) if (u & 0x80000000) else (u | 0x80000000)
    return ((~o & 0xFFFFFFFF) << 32) | j


def _key_score(k: int) -> float:
    o = ~(k >> 32) & 0xFFFFFFFF
    u = (o ^ 0x80000000) if (o & 0x80000000) else (~o & 0xFFFFFFFF)
    return float(np.uint32(u).view(np.float32))


def _i64(u: int) -> int:
    return int(np.uint64(u).view(np.int64))


def _u64(i: int) -> int:
    return int(np.int64(i).view(np.uint64))


class FakeShard:
    """The shard engine's phases in numpy, over the oracle's summaries of this rank's tokens."""

    def __init__(self, K, V, qref, rank, world, off, cnt, n_q):
        self.K, self.V = K, V
        self.rank, self.world, self.off, self.cnt = rank, world, off, cnt
        self.L = L
        self.summ = {lev: [O.summaries(K[h, off:off + cnt], qref[h], C ** lev) for h in range(HKV)]
                     for lev in range(1, L + 1)}
        lanes = n_q * HQ
        z = lambda *s, dt: torch.zeros(s, dtype=dt)
        self.bufs = {"lane_max": z(lanes, dt=torch.int32), "lane_cnt": z(lanes, dt=torch.int32),
                     "hist": z(lanes, BINS, dt=torch.int64), "keys": z(lanes, KEYS, dt=torch.int64),
                     "nkeys": z(lanes, dt=torch.int32), "keys_all": z(world, lanes, KEYS, dt=torch.int64),
                     "nkeys_all": z(world, lanes, dt=torch.int32), "out": z(lanes, D, dt=torch.float32),
                     "lse": z(lanes, dt=torch.float32), "out_all": z(world, lanes, D, dt=torch.float32),
                     "lse_all": z(world, lanes, dt=torch.float32)}
        self.lanes = lanes

    def local(self, name):
        return self.bufs[name]

    def gathered(self, name):
        return self.bufs[name]

    def begin(self, Q, p):
        self.q = Q.to(torch.float64).numpy().reshape(-1, D)       # lane x = i*Hq + h
        self.p = p
        self.kept = {}

    def _g(self, x):
        return (x % HQ) * HKV // HQ

    def score(self, level):
        n_l = self.cnt // C ** level
        self.front = []
        for x in range(self.lanes):
            if level == L:
                fr = np.arange(n_l)
            else:
                par = np.flatnonzero(self.kept[level + 1][x])
                fr = (par[:, None] * C + np.arange(C)[None, :]).ravel()
                fr = fr[fr < n_l]
            m, _, b = self.summ[level][self._g(x)]
            e = np.array([float(np.float32(O.plane_estimate(m[j], b[j], self.q[x]))) for j in fr])
            self.front.append((fr, e))
            self.bufs["lane_max"][x] = _ord_i32(e.max()) if e.size else -2 ** 31
            self.bufs["lane_cnt"][x] = e.size

    def hist(self, level):
        self.M = [_from_ord_i32(int(v)) for v in self.bufs["lane_max"]]
        for x, (fr, e) in enumerate(self.front):
            h = np.zeros(BINS, dtype=np.int64)
            for v in e:
                h[_bin(v, self.M[x])] += _mass(v, self.M[x])
            self.bufs["hist"][x] = torch.from_numpy(h)

    def cut(self, level):
        n_l = self.cnt // C ** level
        off_l = self.off // C ** level
        self.kept[level] = np.zeros((self.lanes, n_l), dtype=bool)
        self.need = []
        for x, (fr, e) in enumerate(self.front):
            hist = [int(v) for v in self.bufs["hist"][x]]
            Z = sum(hist)
            keys = []
            if Z == 0 or self.bufs["lane_cnt"][x] == 0:
                self.need.append(0)
            else:
                target = min(Z, max(1, math.ceil(self.p * Z)))
                cum, bstar = 0, BINS - 1
                for i, hv in enumerate(hist):
                    if cum + hv >= target:
                        bstar = i
                        break
                    cum += hv
                self.need.append(target - cum)
                for j, v in zip(fr, e):
                    bn = _bin(v, self.M[x])
                    if bn < bstar:
                        self.kept[level][x, j] = True
                    elif bn == bstar:
                        keys.append(_key(v, int(j) + off_l))
            self.bufs["nkeys"][x] = len(keys)
            self.bufs["keys"][x, :len(keys)] = torch.tensor([_i64(k) for k in keys], dtype=torch.int64)

    def finish(self, level):
        n_l = self.cnt // C ** level
        off_l = self.off // C ** level
        for x in range(self.lanes):
            if self.need[x] == 0:
                continue
            ks = []
            for r in range(self.world):
                nr = int(self.bufs["nkeys_all"][r, x])
                ks += [_u64(int(v)) for v in self.bufs["keys_all"][r, x, :nr]]
            ks.sort()
            cum = 0
            for k in ks:
                cum += _mass(_key_score(k), self.M[x])
                jl = (k & 0xFFFFFFFF) - off_l
                if 0 <= jl < n_l:
                    self.kept[level][x, jl] = True
                if cum >= self.need[x]:
                    break

    def attend(self, K, V):
        top = C ** L
        T = self.cnt // top
        s = 1.0 / math.sqrt(D)
        for x in range(self.lanes):
            toks = []
            if T >= 1:
                if self.rank == 0:
                    toks.append(0)
                for c in np.flatnonzero(self.kept[1][x]):
                    toks += [t for t in range(c * C, c * C + C) if not (self.rank == 0 and t == 0)]
            toks += list(range(T * top, self.cnt))
            g = self._g(x)
            if not toks:
                self.bufs["out"][x] = 0.0
                self.bufs["lse"][x] = -math.inf
                continue
            kk = self.K[g, self.off + np.array(toks)]
            vv = self.V[g, self.off + np.array(toks)]
            sc = s * kk @ self.q[x]
            mx = sc.max()
            w = np.exp(sc - mx)
            self.bufs["out"][x] = torch.from_numpy(w @ vv / w.sum())
            self.bufs["lse"][x] = float(mx + math.log(w.sum()))

    def combine(self, out):
        lse = self.bufs["lse_all"].to(torch.float64)
        o = self.bufs["out_all"].to(torch.float64)
        M = lse.max(0).values
        c = torch.exp(lse - M)
        out.copy_(((c[:, :, None] * o).sum(0) / c.sum(0)[:, None]).to(torch.float32).reshape(out.shape))


class Identity:
    """The collectives of a world of one."""

    def run(self, engine, op):
        if op[0] == "gather":
            engine.gathered(op[1])[0].copy_(engine.local(op[2]))


def _inputs(n, n_q, seed=0):
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((HKV, n, D))
    V = rng.standard_normal((HKV, n, D))
    qref = rng.standard_normal((HKV, R, D))
    Q = torch.from_numpy(rng.standard_normal((n_q, HQ, D)) * 2.0)
    return K, V, qref, Q


def _decode(K, V, qref, Q, n, p, rank, world, coll):
    off, cnt = zha.shard_ranges(n, C, L, world)[rank]
    e = FakeShard(K, V, qref, rank, world, off, cnt, Q.shape[0])
    out = torch.zeros((Q.shape[0], HQ, D), dtype=torch.float32)
    zha.decode_sharded(e, None, None, Q, p, out, coll=coll)
    return e, out, off


def _rank_main(rank, world, port, n, p, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=120))
    try:
        K, V, qref, Q = _inputs(n, 3)
        e, out, off = _decode(K, V, qref, Q, n, p, rank, world, zha.TorchCollectives())
        kept = {str(lev): [np.flatnonzero(e.kept[lev][x]).tolist() for x in range(e.lanes)]
                for lev in range(1, L + 1)}
        with open(os.path.join(out_dir, "rank%d.json" % rank), "w") as f:
            json.dump({"off": off, "kept": kept, "out": out.numpy().tolist()}, f)
    finally:
        dist.destroy_process_group()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,n,p", [(2, 16 * 9 + 5, 0.9), (3, 16 * 10 + 3, 0.8)])
def test_sharded_protocol_over_gloo_equals_one_shard(tmp_path, world, n, p):
    mp.spawn(_rank_main, args=(world, _free_port(), n, p, str(tmp_path)), nprocs=world, join=True)
    got = [json.load(open(tmp_path / ("rank%d.json" % r))) for r in range(world)]
    K, V, qref, Q = _inputs(n, 3)
    whole, out1, _ = _decode(K, V, qref, Q, n, p, 0, 1, Identity())
    for lev in range(1, L + 1):
        span = C ** lev
        for x in range(whole.lanes):
            union = sorted(j + g["off"] // span for g in got for j in g["kept"][str(lev)][x])
            assert union == np.flatnonzero(whole.kept[lev][x]).tolist(), (lev, x)
    for g in got:
        assert np.array_equal(np.array(g["out"], dtype=np.float32), np.array(got[0]["out"], dtype=np.float32))
    # the merged output is the attention over the attended set
    o = np.array(got[0]["out"]).reshape(-1, D)
    for x in range(whole.lanes):
        toks = O.attended_set(whole.kept[1][x], n, C, L)
        ref = O.attend(K[(x % HQ) * HKV // HQ], V[(x % HQ) * HKV // HQ], whole.q[x], toks)
        assert np.abs(o[x] - ref).max() <= 1e-5 * np.abs(ref).max(), x
    assert np.abs(o - out1.numpy().reshape(-1, D)).max() <= 1e-5
