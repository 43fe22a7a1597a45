"""One sequence split over ranks (zha_shard_*), run as several shards of one process on one
GPU in lockstep (zha.decode_local_shards: every shard reaches its next collective, the
collective is taken over all of them with torch ops, then every shard resumes; no kernel
waits on another shard's kernel).

What must hold (the sharded cut is the single-tree cut over the union of the frontiers):
* kept sets: each shard's kept nodes at every level are bit for bit the single tree's kept
  nodes in the shard's range (the fixed-point histogram sums exactly in any order and the
  boundary bin is ordered by global node index);
* outputs: the merged output equals the single tree's decode up to float32 summation order
  (1e-4 relative), and the oracle's attention over the attended set (2e-3);
* the protocol: a call out of order, or a plain routing call on a shard decoder, is refused.
"""
import numpy as np
import pytest
import torch

from hierarchical_tree_indexed_build_b200 import inputs, zha
from oracle import oracle as O
import zha_testlib as TL

pytestmark = pytest.mark.gpu
needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def _shards(seq, n, world, fmt=zha.ZHA_SUMMARY_F16X2):
    """Per-rank trees over contiguous copies of the ranks' K/V rows."""
    g = seq.geom
    qr = seq.qref.cuda()
    out = []
    for r, (off, cnt) in enumerate(zha.shard_ranges(n, g.C, g.L, world)):
        K = seq.K[:, off:off + cnt].contiguous().cuda()
        V = seq.V[:, off:off + cnt].contiguous().cuda()
        t = zha.Tree(g.C, g.L, g.R, g.d, g.Hq, g.Hkv, max(cnt, 1), fmt)
        t.build(K, cnt, qr)
        out.append((off, cnt, t, K, V))
    return out


def _run(seq, n, Q, p, world, score=zha.ZHA_KERNELS_AUTO, attn=zha.ZHA_KERNELS_AUTO, fmt=zha.ZHA_SUMMARY_F16X2):
    g = seq.geom
    # the single tree over the whole sequence
    K, V, qr = seq.K.cuda(), seq.V.cuda(), seq.qref.cuda()
    full = zha.Tree(g.C, g.L, g.R, g.d, g.Hq, g.Hkv, seq.capacity, fmt)
    full.build(K, n, qr)
    dec = zha.Decoder([full], Q.shape[0])
    dec.set_kernels(score, attn)
    one = TL.gpu_decode([full], [K], [V], Q[None], p, dec=dec)
    # the shards
    sh = _shards(seq, n, world, fmt)
    engines = []
    for r, (off, cnt, t, _, _) in enumerate(sh):
        e = zha.ShardedDecoder(t, Q.shape[0], r, world, off)
        e.set_kernels(score, attn)
        e.set_sync(True)
        engines.append(e)
    Qd = Q.cuda().contiguous()
    outs = [torch.empty((Q.shape[0], g.Hq, g.d), dtype=torch.float32, device="cuda") for _ in engines]
    zha.decode_local_shards(engines, [s[3] for s in sh], [s[4] for s in sh], Qd, p, outs)
    torch.cuda.synchronize()
    return one, sh, engines, outs, (full, dec)


def _check_kept(seq, n, one, sh, engines):
    g = seq.geom
    for lev in range(1, g.L + 1):
        span = g.C ** lev
        for (off, cnt, t, _, _), e in zip(sh, engines):
            n_l = cnt // span
            bits, counts = e.export_kept(lev)
            mine = TL.bits_to_bool(bits, n_l)
            ref = one.kept[0][lev - 1][:, off // span:off // span + n_l]
            assert np.array_equal(mine, ref), (lev, off, int((mine != ref).sum()))
            assert np.array_equal(counts.cpu().numpy(), ref.sum(axis=1)), lev


@needs_cuda
@pytest.mark.parametrize("geom,n,n_q,world,score", [
    (inputs.DEEP, 3 * 4096 + 1234, 8, 2, zha.ZHA_KERNELS_AUTO),      # 64 lanes per group: tcgen05 scorer
    (inputs.DEEP, 5 * 4096 + 77, 8, 3, zha.ZHA_KERNELS_SIMT),        # CUDA-core scorer, 3 ranks
    (inputs.DEEP, 4 * 4096, 1, 4, zha.ZHA_KERNELS_SIMT),              # one query: few-lane scorer, no tail
    (inputs.MID, 3 * 4096 + 500, 4, 2, zha.ZHA_KERNELS_AUTO),        # C = 16
    (inputs.WIDE, 40 * 256 + 100, 4, 3, zha.ZHA_KERNELS_TENSOR),     # C = 256, L = 1
])
def test_sharded_decode_equals_single_tree(geom, n, n_q, world, score):
    seq = inputs.make_sequence(geom, n, n, seed=23)
    Q, _ = inputs.make_queries(seq, n_q, 6, n, np.random.default_rng(5))
    one, sh, engines, outs, keep = _run(seq, n, Q, 0.9, world, score=score)
    _check_kept(seq, n, one, sh, engines)
    # every shard produced the same merged output
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    got = outs[0].cpu().numpy().astype(np.float64).reshape(-1, geom.d)
    ref = one.out[0].reshape(-1, geom.d)
    e_one = TL.rel_err(got, ref)
    assert e_one.max() <= 1e-4, e_one.max()
    # against the oracle's attention over the attended set (sampled queries)
    qs = [0, n_q - 1]
    q, lane_g, ids = TL.lanes_for(seq, Q, qs)
    toks = [O.attended_set(one.kept[0][0][i], n, geom.C, geom.L) for i in ids]
    o = O.attend_batch(TL.f64(seq.K), TL.f64(seq.V), q, lane_g, toks)
    e_or = TL.rel_err(got[ids], o)
    assert e_or.max() <= TL.OUT_TOL, e_or.max()
    TL.NOTES.append("sharded C%dL%d over %d ranks, %d queries: kept sets identical to the single tree at "
                    "every level; output vs single tree max %.2e, vs oracle max %.2e"
                    % (geom.C, geom.L, world, n_q, e_one.max(), e_or.max()))
    for e in engines:
        e.close()
    keep[1].close()
    keep[0].close()


@needs_cuda
def test_sharded_decode_keeps_everything_at_p1():
    geom = inputs.DEEP
    n = 3 * 4096 + 99
    seq = inputs.make_sequence(geom, n, n, seed=3)
    Q, _ = inputs.make_queries(seq, 2, 4, n, np.random.default_rng(1))
    one, sh, engines, outs, keep = _run(seq, n, Q, 1.0, 2)
    _check_kept(seq, n, one, sh, engines)
    got = outs[0].cpu().numpy().astype(np.float64).reshape(-1, geom.d)
    q, lane_g, ids = TL.lanes_for(seq, Q, [0, 1])
    o = O.attend_batch(TL.f64(seq.K), TL.f64(seq.V), q, lane_g, [np.arange(n)] * len(ids))
    assert TL.rel_err(got[ids], o).max() <= TL.OUT_TOL


@needs_cuda
def test_sharded_bf16_trees_route_like_the_single_bf16_tree():
    geom = inputs.DEEP
    n = 3 * 4096 + 640
    seq = inputs.make_sequence(geom, n, n, seed=8)
    Q, _ = inputs.make_queries(seq, 8, 6, n, np.random.default_rng(2))
    one, sh, engines, outs, keep = _run(seq, n, Q, 0.9, 2, fmt=zha.ZHA_SUMMARY_BF16)
    _check_kept(seq, n, one, sh, engines)
    got = outs[0].cpu().numpy().astype(np.float64).reshape(-1, geom.d)
    assert TL.rel_err(got, one.out[0].reshape(-1, geom.d)).max() <= 1e-4


@needs_cuda
def test_shard_protocol_is_enforced():
    geom = inputs.DEEP
    n = 2 * 4096
    seq = inputs.make_sequence(geom, n, n, seed=4)
    Q, _ = inputs.make_queries(seq, 1, 2, n, np.random.default_rng(0))
    sh = _shards(seq, n, 2)
    e = zha.ShardedDecoder(sh[0][2], 1, 0, 2, 0)
    Qd = Q.cuda().contiguous()
    e.begin(Qd, 0.9)
    with pytest.raises(zha.ZhaError) as ei:
        e.hist(geom.L)                        # score first
    assert ei.value.status == zha.ZHA_ERR_STATE
    with pytest.raises(zha.ZhaError) as ei:
        e.score(geom.L - 1)                   # the top level first
    assert ei.value.status == zha.ZHA_ERR_STATE
    # a plain routing call on a shard decoder
    with pytest.raises(zha.ZhaError) as ei:
        zha.zha_route(e.handle, Qd.data_ptr(), 1, 0.9, zha._stream())
    assert ei.value.status == zha.ZHA_ERR_STATE
    # creation rules: rank 0 at token 0, offsets on whole top nodes
    with pytest.raises(zha.ZhaError):
        zha.ShardedDecoder(sh[1][2], 1, 1, 2, 0)
    with pytest.raises(zha.ZhaError):
        zha.ShardedDecoder(sh[1][2], 1, 1, 2, 100)
    # a non-last shard must hold whole top nodes
    K = seq.K[:, :5000].contiguous().cuda()
    t = zha.Tree(geom.C, geom.L, geom.R, geom.d, geom.Hq, geom.Hkv, 5000)
    t.build(K, 5000, seq.qref.cuda())
    e2 = zha.ShardedDecoder(t, 1, 0, 2, 0)
    with pytest.raises(zha.ZhaError) as ei:
        e2.begin(Qd, 0.9)
    assert ei.value.status == zha.ZHA_ERR_STATE
    for x in (e, e2):
        x.close()


@needs_cuda
def test_sharded_decode_through_nccl_collectives(tmp_path):
    """The protocol over torch.distributed with the NCCL backend (one rank: the whole sequence
    as one shard), so the collective calls themselves - in-place MAX / SUM all-reduces of int32
    and int64 buffers and rank-major all_gather_into_tensor - run on the device; the result
    must equal the single tree's decode."""
    import torch.distributed as dist
    geom = inputs.DEEP
    n = 3 * 4096 + 321
    seq = inputs.make_sequence(geom, n, n, seed=31)
    Q, _ = inputs.make_queries(seq, 4, 6, n, np.random.default_rng(3))
    one, sh, engines, outs, keep = _run(seq, n, Q, 0.9, 1)
    own = not dist.is_initialized()
    if own:
        dist.init_process_group("nccl", init_method="file://" + str(tmp_path / "pg"), rank=0, world_size=1)
    try:
        e = engines[0]
        out = torch.empty((Q.shape[0], geom.Hq, geom.d), dtype=torch.float32, device="cuda")
        zha.decode_sharded(e, sh[0][3], sh[0][4], Q.cuda().contiguous(), 0.9, out)
        torch.cuda.synchronize()
        for lev in range(1, geom.L + 1):
            n_l = n // geom.C ** lev
            assert np.array_equal(TL.bits_to_bool(e.export_kept(lev)[0], n_l), one.kept[0][lev - 1]), lev
        got = out.cpu().numpy().astype(np.float64).reshape(-1, geom.d)
        assert TL.rel_err(got, one.out[0].reshape(-1, geom.d)).max() <= 1e-4
    finally:
        if own:
            dist.destroy_process_group()
    for x in engines:
        x.close()
    keep[1].close()
    keep[0].close()
