"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on the same
seeded inputs.  Small cases run every lane; full-size cases run the batch the benchmark
times and compare sampled lanes."""
import numpy as np
import pytest
import torch

from hierarchical_tree_indexed_build_b200 import inputs, zha
from oracle import oracle as O
import zha_testlib as TL

pytestmark = pytest.mark.gpu

needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def _report(name, rep, e1, e2):
    TL.record(name, rep, e1, e2)


# ----------------------------------------------------------------------------- build

# Chunk sizes that neither divide nor are a multiple of the build's 8-token key groups, with
# 8 reference queries (one warp of tensor-core dot products per node).
ODD6 = inputs.Geometry(C=6, L=3, R=8, d=64, Hq=4, Hkv=2)
ODD12 = inputs.Geometry(C=12, L=2, R=8, d=64, Hq=4, Hkv=2)

@needs_cuda
@pytest.mark.parametrize("geom,n_tokens", [
    (inputs.TINY, 4096),                 # the tiny workload's tree
    (inputs.TINY, 4096 + 77),            # ragged: incomplete chunk and nodes at the end
    (inputs.DEEP, 3 * 4096 + 1234),      # C4 L6, ragged
    (inputs.MID, 2 * 4096 + 700),        # C16 L3, ragged
    (inputs.WIDE, 256 * 40 + 100),       # C256 L1, ragged
    (ODD6, 4096 + 333),                  # C6: key groups of 6 tokens
    (ODD12, 4096 + 333),                 # C12: chunks of 8 + 4 tokens
])
def test_build_summaries_match_oracle(geom, n_tokens):
    seq = inputs.make_sequence(geom, n_tokens, n_tokens, seed=11)
    tree, K, V, qr = TL.make_tree(seq)
    w = TL.compare_summaries(tree, seq, n_tokens)
    print("[build %s N=%d] worst lse %.2e m %.2e b %.2e" % (geom, n_tokens, w["lse"], w["m"], w["b"]))
    assert w["lse"] <= TL.SUM_TOL and w["m"] <= TL.SUM_TOL and w["b"] <= TL.SUM_TOL


@needs_cuda
def test_build_deep64k_all_nodes():
    wl = inputs.deep_64k()
    seq = wl.seqs[0]
    tree, K, V, qr = TL.make_tree(seq)
    w = TL.compare_summaries(tree, seq, seq.n_tokens)
    print("[build deep64k] worst", w)
    assert max(w.values()) <= TL.SUM_TOL


@needs_cuda
@pytest.mark.parametrize("geom", [inputs.DEEP, inputs.MID, inputs.WIDE, inputs.TINY, ODD6, ODD12])
def test_append_is_bit_identical_to_rebuild(geom):
    """Growing a tree by appends (single tokens, then a bulk range) gives exactly the
    summaries of a tree built over the final length in one pass."""
    n0, singles, bulk = 4096 * 2 + 13, 70, 4096 + 501
    cap = n0 + singles + bulk
    seq = inputs.make_sequence(geom, cap, cap, seed=5)
    K = seq.K.cuda(); qr = seq.qref.cuda()
    g = geom
    grown = zha.Tree(g.C, g.L, g.R, g.d, g.Hq, g.Hkv, cap)
    grown.build(K, n0, qr)
    n = n0
    for _ in range(singles):
        grown.append(K, n, 1)
        n += 1
    grown.append(K, n, bulk)
    n += bulk
    once = zha.Tree(g.C, g.L, g.R, g.d, g.Hq, g.Hkv, cap)
    once.build(K, n, qr)
    assert grown.n_tokens == once.n_tokens == cap
    for lev in range(1, g.L + 1):
        if grown.level_nodes()[lev - 1] == 0:
            continue
        a, b = grown.export(lev), once.export(lev)
        for x, y in zip(a, b):
            assert torch.equal(x, y), lev


# ----------------------------------------------------------------------------- decode

@needs_cuda
@pytest.mark.parametrize("p", [0.9, 1.0, 0.5])
def test_decode_tiny(p):
    wl = inputs.tiny_4k()
    seq = wl.seqs[0]
    tree, K, V, qr = TL.make_tree(seq)
    Q = wl.Q[0]                                   # [1][16][1][64]
    res = TL.gpu_decode([tree], [K], [V], Q, p)
    rep, e1, e2, toks = TL.check_decode(seq, seq.n_tokens, Q[0], p, res.out[0], res.kept[0], range(16))
    _report("tiny p=%g" % p, rep, e1, e2)
    if p == 1.0:
        assert all(t.size == seq.n_tokens for t in toks)
        dense = O.attend_batch(TL.f64(seq.K), TL.f64(seq.V), TL.lanes_for(seq, Q[0], range(16))[0],
                               np.zeros(16, np.int32), [np.arange(seq.n_tokens)] * 16)
        assert TL.rel_err(res.out[0].reshape(16, -1), dense).max() <= TL.OUT_TOL
    # sink always attended; per-lane token counts match the stats
    assert all(t[0] == 0 for t in toks)
    assert res.stats.lane_tokens == sum(t.size for t in toks)


@needs_cuda
def test_decode_deep_ragged_tail():
    """C4 L6 with 4 complete top nodes and a 1,500-token dense tail, 16 queries."""
    n = 4 * 4096 + 1500
    seq = inputs.make_sequence(inputs.DEEP, n, n, seed=21)
    rq = np.random.default_rng(3)
    Q, _ = inputs.make_queries(seq, 16, 8, n, rq)
    tree, K, V, qr = TL.make_tree(seq)
    res = TL.gpu_decode([tree], [K], [V], Q[None], 0.95)
    rep, e1, e2, toks = TL.check_decode(seq, n, Q, 0.95, res.out[0], res.kept[0], range(16))
    _report("deep ragged", rep, e1, e2)
    assert all(np.all(t[-1500:] == np.arange(n - 1500, n)) for t in toks)


@needs_cuda
def test_decode_no_complete_top_node_is_dense():
    n = 4000                                     # < 4096 = C^L: no top node, A = [0, N)
    seq = inputs.make_sequence(inputs.DEEP, n, n, seed=2)
    Q, _ = inputs.make_queries(seq, 2, 8, n, np.random.default_rng(0))
    tree, K, V, qr = TL.make_tree(seq)
    res = TL.gpu_decode([tree], [K], [V], Q[None], 0.95)
    q, lane_g, ids = TL.lanes_for(seq, Q, range(2))
    dense = O.attend_batch(TL.f64(seq.K), TL.f64(seq.V), q, lane_g, [np.arange(n)] * len(ids))
    assert TL.rel_err(res.out[0].reshape(-1, 128)[ids], dense).max() <= TL.OUT_TOL


@needs_cuda
def test_decode_deep64k_full_batch():
    """The 64K deep workload: all 64 queries routed in one batch, 16 compared lane by lane."""
    wl = inputs.deep_64k()
    seq = wl.seqs[0]
    tree, K, V, qr = TL.make_tree(seq)
    Q = wl.Q[0]
    res = TL.gpu_decode([tree], [K], [V], Q, 0.95)
    rep, e1, e2, _ = TL.check_decode(seq, seq.n_tokens, Q[0], 0.95, res.out[0], res.kept[0], range(0, 64, 4))
    _report("deep64k", rep, e1, e2)


@needs_cuda
def test_decode_wide256k():
    wl = inputs.wide_256k()
    seq = wl.seqs[0]
    tree, K, V, qr = TL.make_tree(seq)
    Q = wl.Q[0]
    res = TL.gpu_decode([tree], [K], [V], Q, 0.95)
    rep, e1, e2, _ = TL.check_decode(seq, seq.n_tokens, Q[0], 0.95, res.out[0], res.kept[0], [0, 9, 31, 63])
    _report("wide256k", rep, e1, e2)


@needs_cuda
@pytest.mark.parametrize("p", [0.7, 0.9, 0.99])
def test_decode_deep_p_sweep(p):
    n = 32 * 4096 + 333
    seq = inputs.make_sequence(inputs.DEEP, n, n, seed=31)
    Q, _ = inputs.make_queries(seq, 8, 8, n, np.random.default_rng(1))
    tree, K, V, qr = TL.make_tree(seq)
    res = TL.gpu_decode([tree], [K], [V], Q[None], p)
    rep, e1, e2, _ = TL.check_decode(seq, n, Q, p, res.out[0], res.kept[0], range(8))
    _report("deep128k p=%g" % p, rep, e1, e2)


@needs_cuda
def test_decode_batched_mixed_geometries_with_appends():
    """8 sequences (4 x C16 L3, 4 x C4 L6), ragged lengths, 3 decode steps each preceded
    by a one-token append; every lane compared."""
    seqs = []
    for s in range(8):
        geom = inputs.MID if s < 4 else inputs.DEEP
        n = 2 * 4096 + 97 * s + 5
        seqs.append(inputs.make_sequence(geom, n, n + 3, seed=100 + s))
    trees, Ks, Vs = [], [], []
    for sq in seqs:
        t, K, V, _ = TL.make_tree(sq, sq.n_tokens)
        trees.append(t); Ks.append(K); Vs.append(V)
    dec = zha.Decoder(trees, 1)
    rng = np.random.default_rng(9)
    for step in range(3):
        Qs = []
        for s, sq in enumerate(seqs):
            trees[s].append(Ks[s], sq.n_tokens + step, 1)
            q, _ = inputs.make_queries(sq, 1, 8, sq.n_tokens + step + 1, rng)
            Qs.append(q)
        Q = torch.stack(Qs)                      # [8][1][16][128]
        res = TL.gpu_decode(trees, Ks, Vs, Q, 0.95, dec=dec)
        for s, sq in enumerate(seqs):
            rep, e1, e2, _ = TL.check_decode(sq, sq.n_tokens + step + 1, Q[s], 0.95, res.out[s], res.kept[s], [0])
            _report("batched step %d seq %d" % (step, s), rep, e1, e2)


@needs_cuda
def test_decode_is_deterministic():
    wl = inputs.deep_64k(n_q=8)
    seq = wl.seqs[0]
    tree, K, V, qr = TL.make_tree(seq)
    a = TL.gpu_decode([tree], [K], [V], wl.Q[0], 0.95)
    b = TL.gpu_decode([tree], [K], [V], wl.Q[0], 0.95)
    assert np.array_equal(a.out, b.out)
    for x, y in zip(a.kept[0], b.kept[0]):
        assert np.array_equal(x, y)


@needs_cuda
def test_error_paths_on_device():
    seq = inputs.make_sequence(inputs.DEEP, 5000, 5000, seed=1)
    K = seq.K.cuda(); qr = seq.qref.cuda()
    g = inputs.DEEP
    t = zha.Tree(g.C, g.L, g.R, g.d, g.Hq, g.Hkv, 5000)
    with pytest.raises(zha.ZhaError) as ei:
        t.append(K, 0, 10)                        # before build
    assert ei.value.status == zha.ZHA_ERR_STATE
    t.build(K, 4000, qr)
    with pytest.raises(zha.ZhaError) as ei:
        t.append(K, 3999, 1)                      # wrong n_old
    assert ei.value.status == zha.ZHA_ERR_STATE
    with pytest.raises(zha.ZhaError) as ei:
        t.append(K, 4000, 1001)                   # past capacity
    assert ei.value.status == zha.ZHA_ERR_CAPACITY
    with pytest.raises(zha.ZhaError) as ei:
        t.build(K, 5001, qr)
    assert ei.value.status == zha.ZHA_ERR_CAPACITY
    dec = zha.Decoder([t], 2)
    Q = torch.zeros((1, 3, 16, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(zha.ZhaError) as ei:
        dec.route(Q, 0.9)                         # more queries than the decoder holds
    assert ei.value.status == zha.ZHA_ERR_CAPACITY
    with pytest.raises(zha.ZhaError) as ei:
        dec.route(Q[:, :2].contiguous(), 0.0)     # p must be > 0
    assert ei.value.status == zha.ZHA_ERR_ARG
    with pytest.raises(zha.ZhaError) as ei:
        dec.sparse_attn([K], [K], Q[:, :1].contiguous(), torch.zeros((1, 1, 16, 128), device="cuda"))
    assert ei.value.status == zha.ZHA_ERR_STATE   # attention before routing


@needs_cuda
@pytest.mark.parametrize("n_q", [1, 8, 20, 48, 64])
def test_tensor_core_and_cuda_core_scoring_agree(n_q):
    """The tcgen05 scorer (fp16 Q, summaries split into fp16 hi + lo passes) and the fp32
    CUDA-core scorer route the
    64K deep workload to the same kept sets (up to logged ties) and the same outputs; the
    tensor-core result is also checked against the oracle."""
    wl = inputs.deep_64k(n_q=n_q)
    seq = wl.seqs[0]
    tree, K, V, qr = TL.make_tree(seq)
    Q = wl.Q[0]
    res = {}
    for path in (zha.ZHA_KERNELS_SIMT, zha.ZHA_KERNELS_TENSOR):
        dec = zha.Decoder([tree], n_q)
        dec.set_kernels(score=path, attn=zha.ZHA_KERNELS_SIMT)
        res[path] = TL.gpu_decode([tree], [K], [V], Q, 0.95, dec=dec)
        dec.close()
    a, b = res[zha.ZHA_KERNELS_SIMT], res[zha.ZHA_KERNELS_TENSOR]
    differ = sum(int((x != y).any(axis=1).sum()) for x, y in zip(a.kept[0], b.kept[0]))
    lanes = a.kept[0][0].shape[0]
    print("[tc vs simt n_q=%d] lane-levels differing: %d of %d" % (n_q, differ, lanes * len(a.kept[0])))
    assert differ <= max(1, lanes * len(a.kept[0]) // 100)
    qs = list(range(min(n_q, 4)))
    rep, e1, e2, _ = TL.check_decode(seq, seq.n_tokens, Q[0], 0.95, b.out[0], b.kept[0], qs)
    _report("tensor n_q=%d" % n_q, rep, e1, e2)


@needs_cuda
def test_tensor_core_scoring_flags_inputs_outside_fp16_range():
    """A query entry beyond the fp16 range makes the tensor-core scorer raise status bit 8
    (its estimates are then not valid); the CUDA-core scorer takes the same input."""
    import ctypes
    wl = inputs.deep_64k(n_q=64)
    seq = wl.seqs[0]
    tree, K, V, qr = TL.make_tree(seq)
    Q = wl.Q[0].clone()
    Q[0, 3, 5, 7] = 1.0e5                          # bf16 holds it, fp16 does not
    Qd = Q.cuda()
    for path, want in ((zha.ZHA_KERNELS_TENSOR, 8), (zha.ZHA_KERNELS_SIMT, 0)):
        dec = zha.Decoder([tree], 64)
        dec.set_kernels(score=path, attn=zha.ZHA_KERNELS_SIMT)
        dec.route(Qd, 0.95)
        torch.cuda.synchronize()
        st = zha.DecodeStats()
        rc = zha.lib().zha_decoder_stats(dec.handle, ctypes.byref(st), 0)
        assert (st.status & 8) == want
        assert rc == (zha.ZHA_ERR_DEVICE if want else zha.ZHA_OK)
        dec.close()


@needs_cuda
def test_tensor_core_scoring_needs_r16():
    n = 4096 * 2
    seq = inputs.make_sequence(inputs.TINY, n, n, seed=3, key_mean_std=0.0)
    tree, K, V, qr = TL.make_tree(seq)
    dec = zha.Decoder([tree], 1)
    with pytest.raises(zha.ZhaError) as ei:
        dec.set_kernels(score=zha.ZHA_KERNELS_TENSOR)
    assert ei.value.status == zha.ZHA_ERR_ARG


@needs_cuda
@pytest.mark.parametrize("n_q,p", [(1, 0.95), (8, 0.9), (40, 0.9), (64, 0.95), (64, 1.0)])
def test_tensor_core_and_cuda_core_attention_agree(n_q, p):
    """The tcgen05 attention (exact QK^T, bf16 hi+lo P) and the CUDA-core attention give the
    same outputs on the same routed sets, and the tensor-core output matches the oracle."""
    wl = inputs.deep_64k(n_q=n_q)
    seq = wl.seqs[0]
    n = seq.n_tokens - 1234                        # ragged: dense tail after the last top node
    tree, K, V, qr = TL.make_tree(seq, n)
    Q = wl.Q[0]
    outs = {}
    for path in (zha.ZHA_KERNELS_SIMT, zha.ZHA_KERNELS_TENSOR):
        dec = zha.Decoder([tree], n_q)
        dec.set_kernels(score=zha.ZHA_KERNELS_SIMT, attn=path)
        outs[path] = TL.gpu_decode([tree], [K], [V], Q, p, dec=dec)
        dec.close()
    a, b = outs[zha.ZHA_KERNELS_SIMT], outs[zha.ZHA_KERNELS_TENSOR]
    for x, y in zip(a.kept[0], b.kept[0]):
        assert np.array_equal(x, y)               # same scorer: identical routing
    e = TL.rel_err(b.out.reshape(-1, 128), a.out.reshape(-1, 128)).max()
    print("[attn tc vs simt n_q=%d p=%g] max rel diff %.2e" % (n_q, p, e))
    assert e <= 1e-4
    rep, e1, e2, _ = TL.check_decode(seq, n, Q[0], p, b.out[0], b.kept[0], list(range(min(n_q, 3))))
    _report("attn tensor n_q=%d p=%g" % (n_q, p), rep, e1, e2)


# ----------------------------------------------------------------------------- dense baseline

@needs_cuda
@pytest.mark.parametrize("geom,n_tokens,n_q,attn", [
    (inputs.TINY, 4096 + 77, 16, zha.ZHA_KERNELS_SIMT),      # 16 lanes: CUDA-core split-KV
    (inputs.TINY, 4096 + 77, 16, zha.ZHA_KERNELS_AUTO),      # 16 lanes, d = 64: tcgen05 with a padded lane tile
    (inputs.DEEP, 3 * 4096 + 1234, 8, zha.ZHA_KERNELS_AUTO),  # 64 lanes per group: tcgen05
    (inputs.DEEP, 3 * 4096 + 1234, 8, zha.ZHA_KERNELS_SIMT),
    (inputs.MID, 2 * 4096 + 700, 3, zha.ZHA_KERNELS_TENSOR),  # 24 lanes: a ragged lane tile on tcgen05
])
def test_dense_attention_matches_oracle(geom, n_tokens, n_q, attn):
    """zha_dense_attn is exact softmax attention of every lane over all N tokens: the
    oracle's attention over the whole token range (pinned to float64 SDPA)."""
    seq = inputs.make_sequence(geom, n_tokens, n_tokens, seed=21)
    tree, K, V, qr = TL.make_tree(seq)
    rng = np.random.default_rng(3)
    Q = torch.from_numpy(rng.standard_normal((1, n_q, geom.Hq, geom.d), dtype=np.float32)).to(torch.bfloat16)
    dec = zha.Decoder([tree], n_q)
    dec.set_kernels(zha.ZHA_KERNELS_AUTO, attn)
    out = dec.dense_attn([K], [V], Q.cuda().contiguous())
    torch.cuda.synchronize()
    q, lane_g, ids = TL.lanes_for(seq, Q[0], range(n_q))
    o = O.attend_batch(TL.f64(seq.K), TL.f64(seq.V), q, lane_g, [np.arange(n_tokens)] * len(ids))
    e = TL.rel_err(out.cpu().numpy().astype(np.float64).reshape(-1, geom.d)[ids], o)
    print("[dense %s N=%d n_q=%d attn=%d] max rel err %.2e" % (geom, n_tokens, n_q, attn, e.max()))
    assert e.max() <= TL.OUT_TOL
    dec.close()
    tree.close()


@needs_cuda
def test_dense_attention_equals_routed_decode_at_p1():
    """At p = 1 every frontier node is kept at every level, so the routed set is every token
    and the routed decode computes dense attention (in another summation order); a dense
    call between a route and its sparse attention leaves the route's kept sets in place."""
    geom, n_tokens, n_q = inputs.DEEP, 3 * 4096 + 1234, 8
    seq = inputs.make_sequence(geom, n_tokens, n_tokens, seed=22)
    tree, K, V, qr = TL.make_tree(seq)
    rng = np.random.default_rng(4)
    Q = torch.from_numpy(rng.standard_normal((1, n_q, geom.Hq, geom.d), dtype=np.float32)).to(torch.bfloat16).cuda()
    dec = zha.Decoder([tree], n_q)
    routed = dec.decode([K], [V], Q, 1.0)
    dense = dec.dense_attn([K], [V], Q)
    torch.cuda.synchronize()
    e = TL.rel_err(dense.cpu().numpy().astype(np.float64).reshape(-1, geom.d),
                   routed.cpu().numpy().astype(np.float64).reshape(-1, geom.d))
    print("[dense vs routed p=1] max rel diff %.2e" % e.max())
    assert e.max() <= 1e-4
    dec.route(Q, 0.9)
    dense2 = dec.dense_attn([K], [V], Q)
    sparse = torch.empty_like(dense2)
    dec.sparse_attn([K], [V], Q, sparse)
    again = dec.decode([K], [V], Q, 0.9)
    torch.cuda.synchronize()
    assert torch.equal(dense, dense2)
    assert torch.equal(sparse, again)
    dec.close()
    tree.close()


# ----------------------------------------------------------------------------- kernel configurations

# Geometries that reach kernel variants the workloads above do not: d = 64 on both tensor-core
# kernels, chunk sizes that are not a multiple of 4 on the tensor scorer (one-node copies of
# each record instead of four-node runs), C = 16 on the tensor scorer, R = 32 (CUDA cores).
D64 = inputs.Geometry(C=4, L=4, R=16, d=64, Hq=16, Hkv=2)
C6R16 = inputs.Geometry(C=6, L=3, R=16, d=128, Hq=16, Hkv=2)
C2R16 = inputs.Geometry(C=2, L=7, R=16, d=128, Hq=16, Hkv=2)
R32 = inputs.Geometry(C=4, L=4, R=32, d=128, Hq=16, Hkv=2)


@needs_cuda
@pytest.mark.parametrize("name,geom,n_tokens,n_q,paths", [
    # 64 lanes per (sequence, KV head) group: the automatic choice takes both tcgen05 kernels
    ("d64 tensor", D64, 10 * 256 + 77, 8, (zha.ZHA_KERNELS_AUTO, zha.ZHA_KERNELS_AUTO)),
    ("C6 R16 tensor", C6R16, 14 * 216 + 101, 8, (zha.ZHA_KERNELS_AUTO, zha.ZHA_KERNELS_AUTO)),
    ("C2 R16 tensor", C2R16, 40 * 128 + 33, 8, (zha.ZHA_KERNELS_AUTO, zha.ZHA_KERNELS_AUTO)),
    ("C16 MID tensor", inputs.MID, 3 * 4096 + 900, 8, (zha.ZHA_KERNELS_AUTO, zha.ZHA_KERNELS_AUTO)),
    ("C16 MID tensor 24q", inputs.MID, 3 * 4096 + 900, 24, (zha.ZHA_KERNELS_TENSOR, zha.ZHA_KERNELS_TENSOR)),
    # more than 128 lanes per group: the attention pairs lane tiles in one CTA (320 lanes: one
    # full pair and one CTA holding a single lane tile)
    ("d64 tensor 40q", D64, 10 * 256 + 77, 40, (zha.ZHA_KERNELS_AUTO, zha.ZHA_KERNELS_AUTO)),
    ("C6 R16 tensor 40q", C6R16, 14 * 216 + 101, 40, (zha.ZHA_KERNELS_AUTO, zha.ZHA_KERNELS_AUTO)),
    # R = 32: scoring on CUDA cores (k_score), attention both ways
    ("R32 simt", R32, 12 * 256 + 5, 2, (zha.ZHA_KERNELS_AUTO, zha.ZHA_KERNELS_AUTO)),
    ("R32 simt score, tensor attn", R32, 12 * 256 + 5, 8, (zha.ZHA_KERNELS_AUTO, zha.ZHA_KERNELS_AUTO)),
])
def test_decode_kernel_configurations(name, geom, n_tokens, n_q, paths):
    seq = inputs.make_sequence(geom, n_tokens, n_tokens, seed=41)
    Q, _ = inputs.make_queries(seq, n_q, 8, n_tokens, np.random.default_rng(7))
    tree, K, V, qr = TL.make_tree(seq)
    w = TL.compare_summaries(tree, seq, n_tokens, sample=64)
    assert max(w.values()) <= TL.SUM_TOL, w
    dec = zha.Decoder([tree], n_q)
    dec.set_kernels(*paths)
    res = TL.gpu_decode([tree], [K], [V], Q[None], 0.9, dec=dec)
    assert res.stats.status == 0
    qs = sorted(set([0, n_q // 2, n_q - 1]))
    rep, e1, e2, _ = TL.check_decode(seq, n_tokens, Q, 0.9, res.out[0], res.kept[0], qs)
    _report(name, rep, e1, e2)
    # the CUDA-core kernels on the same tree agree (kept sets up to logged ties, outputs)
    ref_dec = zha.Decoder([tree], n_q)
    ref_dec.set_kernels(zha.ZHA_KERNELS_SIMT, zha.ZHA_KERNELS_SIMT)
    ref = TL.gpu_decode([tree], [K], [V], Q[None], 0.9, dec=ref_dec)
    differ = sum(int((x != y).any(axis=1).sum()) for x, y in zip(res.kept[0], ref.kept[0]))
    lanes = res.kept[0][0].shape[0]
    assert differ <= max(2, lanes * geom.L // 50), differ
    same = np.ones(lanes, dtype=bool)
    for x, y in zip(res.kept[0], ref.kept[0]):
        same &= ~(x != y).any(axis=1)
    e = TL.rel_err(res.out[0].reshape(-1, geom.d)[same], ref.out[0].reshape(-1, geom.d)[same])
    assert e.max() <= 1e-4, e.max()
    dec.close()
    ref_dec.close()
    tree.close()


# ----------------------------------------------------------------------------- device status at the boundary

def _range_case():
    """64 lanes per group (tensor-core scorer) with one query entry beyond the fp16 range."""
    wl = inputs.deep_64k(n_q=8)
    seq = wl.seqs[0]
    tree, K, V, qr = TL.make_tree(seq)
    Q = wl.Q[0].clone()
    good = Q.cuda().contiguous()
    Q[0, 3, 5, 7] = 1.0e5
    return tree, K, V, Q.cuda().contiguous(), good


@needs_cuda
def test_decode_reports_device_status_in_sync_mode():
    """A synchronous decoder returns ZHA_ERR_DEVICE from zha_decode itself when the tensor
    scorer flags an input outside the fp16 range (status bit 8), and ZHA_OK again for valid
    input."""
    tree, K, V, bad, good = _range_case()
    dec = zha.Decoder([tree], 8)
    dec.set_kernels(zha.ZHA_KERNELS_TENSOR, zha.ZHA_KERNELS_AUTO)
    dec.set_sync(True)
    with pytest.raises(zha.ZhaError) as ei:
        dec.decode([K], [V], bad, 0.95)
    assert ei.value.status == zha.ZHA_ERR_DEVICE
    assert "0x8" in str(ei.value) and "fp16" in str(ei.value)
    dec.decode([K], [V], good, 0.95)
    with pytest.raises(zha.ZhaError) as ei:
        dec.route(bad, 0.95)
    assert ei.value.status == zha.ZHA_ERR_DEVICE
    dec.close()


@needs_cuda
def test_decode_reports_device_status_on_the_next_call_when_async():
    """Asynchronous (default) decoder: the flagged call returns ZHA_OK; once its work has
    completed, the next call on the decoder returns ZHA_ERR_DEVICE and enqueues nothing; the
    call after that runs normally."""
    tree, K, V, bad, good = _range_case()
    dec = zha.Decoder([tree], 8)
    dec.set_kernels(zha.ZHA_KERNELS_TENSOR, zha.ZHA_KERNELS_AUTO)
    dec.decode([K], [V], bad, 0.95)
    torch.cuda.synchronize()
    out = torch.full((1, 8, 16, 128), 7.0, device="cuda")
    with pytest.raises(zha.ZhaError) as ei:
        dec.decode([K], [V], good, 0.95, out)
    assert ei.value.status == zha.ZHA_ERR_DEVICE
    torch.cuda.synchronize()
    assert (out == 7.0).all()                    # nothing was enqueued
    dec.decode([K], [V], good, 0.95, out)
    torch.cuda.synchronize()
    assert dec.stats().status == 0
    dec.close()
