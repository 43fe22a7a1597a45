"""ctypes binding of libzha (include/zha.h).

Argument marshalling only: every step of tree build, routing and attention runs in the
CUDA kernels of libzha.so.  Functions named ``zha_*`` mirror the C entry points one to
one; ``Tree`` and ``Decoder`` wrap them for torch tensors (device pointers and the
current CUDA stream).  There is no fallback: if libzha.so is missing or no CUDA device
is present, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libzha.so")
MAX_LEVELS = 16

ZHA_OK, ZHA_ERR_ARG, ZHA_ERR_CAPACITY, ZHA_ERR_CUDA, ZHA_ERR_STATE, ZHA_ERR_DEVICE = range(6)
_STATUS = {0: "ZHA_OK", 1: "ZHA_ERR_ARG", 2: "ZHA_ERR_CAPACITY", 3: "ZHA_ERR_CUDA",
           4: "ZHA_ERR_STATE", 5: "ZHA_ERR_DEVICE"}

# Every function declared in include/zha.h.
EXPORTS = ["zha_last_error", "zha_tree_create", "zha_tree_destroy", "zha_tree_info", "zha_build_tree",
           "zha_append", "zha_tree_export", "zha_decoder_create", "zha_decoder_destroy", "zha_route",
           "zha_sparse_attn", "zha_sparse_attn_static", "zha_dense_attn", "zha_decode", "zha_decoder_set_kernels",
           "zha_decoder_set_sync", "zha_decoder_export_kept", "zha_decoder_words",
           "zha_decoder_stats", "zha_profile_enable", "zha_profile_read", "zha_profile_reset",
           "zha_shard_decoder_create", "zha_shard_begin", "zha_shard_score", "zha_shard_hist", "zha_shard_cut",
           "zha_shard_finish", "zha_shard_attend", "zha_shard_combine"]


class ZhaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__("%s: %s" % (_STATUS.get(status, status), msg))
        self.status = status


ZHA_SUMMARY_F16X2, ZHA_SUMMARY_BF16, ZHA_SUMMARY_FP4 = 0, 1, 2


class Geometry(ctypes.Structure):
    _fields_ = [("C", ctypes.c_int32), ("L", ctypes.c_int32), ("R", ctypes.c_int32),
                ("d", ctypes.c_int32), ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("capacity", ctypes.c_int64), ("format", ctypes.c_int32)]


class ShardExchange(ctypes.Structure):
    """zha_shard_exchange: device pointers of the buffers the ranks exchange."""
    _fields_ = [("lane_max", ctypes.c_void_p), ("lane_cnt", ctypes.c_void_p), ("hist", ctypes.c_void_p),
                ("keys", ctypes.c_void_p), ("nkeys", ctypes.c_void_p), ("keys_all", ctypes.c_void_p),
                ("nkeys_all", ctypes.c_void_p), ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p),
                ("out_all", ctypes.c_void_p), ("lse_all", ctypes.c_void_p)]


SHARD_BINS = 2048
SHARD_KEYS = 2048


class DecodeStats(ctypes.Structure):
    _fields_ = [("union_nodes", ctypes.c_int64 * MAX_LEVELS), ("lane_nodes", ctypes.c_int64 * MAX_LEVELS),
                ("union_tokens", ctypes.c_int64), ("lane_tokens", ctypes.c_int64),
                ("node_bytes", ctypes.c_int64), ("status", ctypes.c_int32)]


_lib = None
_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64


def lib() -> ctypes.CDLL:
    """Load libzha.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libzha.so not found at %s; build it with "
                               "hierarchical_tree_indexed_build_b200.build_ext.build()" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        L.zha_last_error.restype = ctypes.c_char_p
        L.zha_tree_create.argtypes = [ctypes.POINTER(Geometry), ctypes.POINTER(_vp)]
        L.zha_tree_destroy.argtypes = [_vp]
        L.zha_tree_info.argtypes = [_vp, ctypes.POINTER(Geometry), ctypes.POINTER(_i64), ctypes.POINTER(_i64),
                                    ctypes.POINTER(_i64)]
        L.zha_build_tree.argtypes = [_vp, _vp, _i64, _vp, _vp]
        L.zha_append.argtypes = [_vp, _vp, _i64, _i64, _vp]
        L.zha_tree_export.argtypes = [_vp, _i32, _vp, _vp, _vp, _vp]
        L.zha_decoder_create.argtypes = [ctypes.POINTER(_vp), _i32, _i32, ctypes.POINTER(_vp)]
        L.zha_decoder_destroy.argtypes = [_vp]
        L.zha_route.argtypes = [_vp, _vp, _i32, ctypes.c_float, _vp]
        L.zha_sparse_attn.argtypes = [_vp, ctypes.POINTER(_vp), ctypes.POINTER(_vp), _vp, _i32, _vp, _vp]
        L.zha_sparse_attn_static.argtypes = [_vp, _vp, _i64, _i64, _i32, _i32, _i32, _i32, _i32, _vp, _i32,
                                             _vp, _i64, _vp, _vp]
        L.zha_dense_attn.argtypes = [_vp, ctypes.POINTER(_vp), ctypes.POINTER(_vp), _vp, _i32, _vp, _vp]
        L.zha_decode.argtypes = [_vp, ctypes.POINTER(_vp), ctypes.POINTER(_vp), _vp, _i32, ctypes.c_float,
                                 _vp, _vp]
        L.zha_decoder_set_kernels.argtypes = [_vp, _i32, _i32]
        L.zha_decoder_set_sync.argtypes = [_vp, _i32]
        L.zha_decoder_export_kept.argtypes = [_vp, _i32, _vp, _vp, _vp]
        L.zha_decoder_words.argtypes = [_vp, _i32]
        L.zha_decoder_words.restype = _i64
        L.zha_decoder_stats.argtypes = [_vp, ctypes.POINTER(DecodeStats), _vp]
        L.zha_profile_enable.argtypes = [_i32]
        L.zha_profile_read.argtypes = [ctypes.c_char_p, _i32, ctypes.POINTER(_i64),
                                       ctypes.POINTER(ctypes.c_double), _i32]
        L.zha_profile_read.restype = _i32
        L.zha_profile_reset.argtypes = []
        L.zha_shard_decoder_create.argtypes = [_vp, _i32, _i32, _i32, _i64, ctypes.POINTER(_vp)]
        L.zha_shard_begin.argtypes = [_vp, _vp, _i32, ctypes.c_float, _vp]
        for nm in ("zha_shard_score", "zha_shard_hist", "zha_shard_cut", "zha_shard_finish"):
            getattr(L, nm).argtypes = [_vp, _i32, ctypes.POINTER(ShardExchange), _vp]
        L.zha_shard_attend.argtypes = [_vp, _vp, _vp, ctypes.POINTER(ShardExchange), _vp]
        L.zha_shard_combine.argtypes = [_vp, ctypes.POINTER(ShardExchange), _vp, _vp]
        for name in EXPORTS:
            if name not in ("zha_last_error", "zha_decoder_words", "zha_profile_read"):
                getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(status: int):
    if status != ZHA_OK:
        raise ZhaError(status, lib().zha_last_error().decode())


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _ptr_array(ts: Sequence[torch.Tensor]):
    arr = (_vp * len(ts))()
    for i, t in enumerate(ts):
        arr[i] = t.data_ptr()
    return arr


# ----------------------------------------------------------------------------- C names

def zha_tree_create(geom: Geometry) -> int:
    h = _vp()
    _check(lib().zha_tree_create(ctypes.byref(geom), ctypes.byref(h)))
    return h.value


def zha_tree_destroy(tree: int):
    _check(lib().zha_tree_destroy(tree))


def zha_tree_info(tree: int):
    g = Geometry()
    n = _i64()
    lv = (_i64 * MAX_LEVELS)()
    nb = _i64()
    _check(lib().zha_tree_info(tree, ctypes.byref(g), ctypes.byref(n), lv, ctypes.byref(nb)))
    return g, n.value, list(lv)[:g.L], nb.value


def zha_build_tree(tree: int, K: int, n_tokens: int, q_ref: int, stream: int):
    _check(lib().zha_build_tree(tree, K, n_tokens, q_ref, stream))


def zha_append(tree: int, K: int, n_old: int, n_new: int, stream: int):
    _check(lib().zha_append(tree, K, n_old, n_new, stream))


def zha_tree_export(tree: int, level: int, m: Optional[int], lse: Optional[int], b: Optional[int], stream: int):
    _check(lib().zha_tree_export(tree, level, m, lse, b, stream))


def zha_decoder_create(trees: Sequence[int], max_queries: int) -> int:
    arr = (_vp * len(trees))(*trees)
    h = _vp()
    _check(lib().zha_decoder_create(arr, len(trees), max_queries, ctypes.byref(h)))
    return h.value


def zha_decoder_destroy(dec: int):
    _check(lib().zha_decoder_destroy(dec))


def zha_route(dec: int, Q: int, n_q: int, p: float, stream: int):
    _check(lib().zha_route(dec, Q, n_q, p, stream))


def zha_sparse_attn(dec: int, K, V, Q: int, n_q: int, out: int, stream: int):
    _check(lib().zha_sparse_attn(dec, K, V, Q, n_q, out, stream))


def zha_sparse_attn_static(K: int, V: int, ld: int, n_tokens: int, C: int, L: int, Hq: int, Hkv: int, d: int,
                           Q: int, n_q: int, kept1: int, words: int, out: int, stream: int):
    _check(lib().zha_sparse_attn_static(K, V, ld, n_tokens, C, L, Hq, Hkv, d, Q, n_q, kept1, words, out, stream))


def zha_dense_attn(dec: int, K, V, Q: int, n_q: int, out: int, stream: int):
    _check(lib().zha_dense_attn(dec, K, V, Q, n_q, out, stream))


def zha_decode(dec: int, K, V, Q: int, n_q: int, p: float, out: int, stream: int):
    _check(lib().zha_decode(dec, K, V, Q, n_q, p, out, stream))


ZHA_KERNELS_AUTO, ZHA_KERNELS_SIMT, ZHA_KERNELS_TENSOR = 0, 1, 2


def zha_decoder_set_kernels(dec: int, score: int, attn: int):
    _check(lib().zha_decoder_set_kernels(dec, score, attn))


def zha_decoder_set_sync(dec: int, on: bool):
    _check(lib().zha_decoder_set_sync(dec, 1 if on else 0))


def zha_decoder_export_kept(dec: int, level: int, bits: int, counts: Optional[int], stream: int):
    _check(lib().zha_decoder_export_kept(dec, level, bits, counts, stream))


def zha_decoder_words(dec: int, level: int) -> int:
    return lib().zha_decoder_words(dec, level)


def zha_decoder_stats(dec: int, stream: int) -> DecodeStats:
    st = DecodeStats()
    _check(lib().zha_decoder_stats(dec, ctypes.byref(st), stream))
    return st


def zha_profile_enable(on: bool):
    _check(lib().zha_profile_enable(1 if on else 0))


def zha_profile_reset():
    _check(lib().zha_profile_reset())


def zha_profile_read(max_kernels: int = 32, name_len: int = 64):
    """{kernel name: (launches, total device ms)} of the recorded launches."""
    names = ctypes.create_string_buffer(max_kernels * name_len)
    launches = (_i64 * max_kernels)()
    total = (ctypes.c_double * max_kernels)()
    n = lib().zha_profile_read(names, name_len, launches, total, max_kernels)
    out = {}
    for k in range(min(n, max_kernels)):
        nm = names.raw[k * name_len:(k + 1) * name_len].split(b"\0", 1)[0].decode()
        out[nm] = (int(launches[k]), float(total[k]))
    return out


def zha_shard_decoder_create(tree: int, max_queries: int, rank: int, world: int, token_offset: int) -> int:
    h = _vp()
    _check(lib().zha_shard_decoder_create(tree, max_queries, rank, world, token_offset, ctypes.byref(h)))
    return h.value


def zha_shard_begin(dec: int, Q: int, n_q: int, p: float, stream: int):
    _check(lib().zha_shard_begin(dec, Q, n_q, p, stream))


def zha_shard_score(dec: int, level: int, ex: ShardExchange, stream: int):
    _check(lib().zha_shard_score(dec, level, ctypes.byref(ex), stream))


def zha_shard_hist(dec: int, level: int, ex: ShardExchange, stream: int):
    _check(lib().zha_shard_hist(dec, level, ctypes.byref(ex), stream))


def zha_shard_cut(dec: int, level: int, ex: ShardExchange, stream: int):
    _check(lib().zha_shard_cut(dec, level, ctypes.byref(ex), stream))


def zha_shard_finish(dec: int, level: int, ex: ShardExchange, stream: int):
    _check(lib().zha_shard_finish(dec, level, ctypes.byref(ex), stream))


def zha_shard_attend(dec: int, K: int, V: int, ex: ShardExchange, stream: int):
    _check(lib().zha_shard_attend(dec, K, V, ctypes.byref(ex), stream))


def zha_shard_combine(dec: int, ex: ShardExchange, out: int, stream: int):
    _check(lib().zha_shard_combine(dec, ctypes.byref(ex), out, stream))


# ----------------------------------------------------------------------------- tensors

def _need(t: torch.Tensor, dtype, what: str):
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise ValueError("%s must be a contiguous CUDA %s tensor" % (what, dtype))


class Tree:
    """A summary tree over one sequence's KV cache (device memory owned by libzha)."""

    def __init__(self, C: int, L: int, R: int, d: int, n_q_heads: int, n_kv_heads: int, capacity: int,
                 format: int = ZHA_SUMMARY_F16X2):
        self.geom = Geometry(C, L, R, d, n_q_heads, n_kv_heads, capacity, format)
        self.handle = zha_tree_create(self.geom)

    def close(self):
        if self.handle:
            zha_tree_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def n_tokens(self) -> int:
        return zha_tree_info(self.handle)[1]

    def level_nodes(self) -> List[int]:
        return zha_tree_info(self.handle)[2]

    def build(self, K: torch.Tensor, n_tokens: int, q_ref: torch.Tensor, stream=None):
        _need(K, torch.bfloat16, "K")
        _need(q_ref, torch.bfloat16, "q_ref")
        zha_build_tree(self.handle, K.data_ptr(), n_tokens, q_ref.data_ptr(), _stream(stream))

    def append(self, K: torch.Tensor, n_old: int, n_new: int, stream=None):
        _need(K, torch.bfloat16, "K")
        zha_append(self.handle, K.data_ptr(), n_old, n_new, _stream(stream))

    def export(self, level: int, stream=None):
        g = self.geom
        nl = self.level_nodes()[level - 1]
        dev = torch.device("cuda", torch.cuda.current_device())
        m = torch.empty((g.n_kv_heads, nl, g.R, g.d), dtype=torch.float32, device=dev)
        lse = torch.empty((g.n_kv_heads, nl, g.R), dtype=torch.float32, device=dev)
        b = torch.empty((g.n_kv_heads, nl, g.R), dtype=torch.float32, device=dev)
        zha_tree_export(self.handle, level, m.data_ptr(), lse.data_ptr(), b.data_ptr(), _stream(stream))
        return m, lse, b


class Decoder:
    """Routing + attention workspace for a batch of trees."""

    def __init__(self, trees: Sequence[Tree], max_queries: int):
        self.trees = list(trees)
        self.handle = zha_decoder_create([t.handle for t in self.trees], max_queries)
        g = self.trees[0].geom
        self.Hq, self.Hkv, self.d = g.n_q_heads, g.n_kv_heads, g.d
        self.n_q = None

    def close(self):
        if self.handle:
            zha_decoder_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def route(self, Q: torch.Tensor, p: float, stream=None):
        _need(Q, torch.bfloat16, "Q")
        n_q = Q.shape[1]
        zha_route(self.handle, Q.data_ptr(), n_q, p, _stream(stream))
        self.n_q = n_q

    def sparse_attn(self, Ks, Vs, Q: torch.Tensor, out: torch.Tensor, stream=None):
        _need(out, torch.float32, "out")
        zha_sparse_attn(self.handle, _ptr_array(Ks), _ptr_array(Vs), Q.data_ptr(), Q.shape[1], out.data_ptr(),
                        _stream(stream))

    def dense_attn(self, Ks, Vs, Q: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None):
        """Dense exact attention of every query lane over its whole sequence (no routing)."""
        _need(Q, torch.bfloat16, "Q")
        if out is None:
            out = torch.empty(Q.shape, dtype=torch.float32, device=Q.device)
        _need(out, torch.float32, "out")
        zha_dense_attn(self.handle, _ptr_array(Ks), _ptr_array(Vs), Q.data_ptr(), Q.shape[1], out.data_ptr(),
                       _stream(stream))
        return out

    def decode(self, Ks, Vs, Q: torch.Tensor, p: float, out: Optional[torch.Tensor] = None, stream=None):
        _need(Q, torch.bfloat16, "Q")
        if out is None:
            out = torch.empty(Q.shape, dtype=torch.float32, device=Q.device)
        _need(out, torch.float32, "out")
        zha_decode(self.handle, _ptr_array(Ks), _ptr_array(Vs), Q.data_ptr(), Q.shape[1], p, out.data_ptr(),
                   _stream(stream))
        self.n_q = Q.shape[1]
        return out

    def set_kernels(self, score: int = ZHA_KERNELS_AUTO, attn: int = ZHA_KERNELS_AUTO):
        zha_decoder_set_kernels(self.handle, score, attn)

    def set_sync(self, on: bool = True):
        """Synchronous calls: each waits for its work and raises ZhaError(ZHA_ERR_DEVICE)
        when a kernel set the device status word."""
        zha_decoder_set_sync(self.handle, on)

    def words(self, level: int) -> int:
        return zha_decoder_words(self.handle, level)

    def export_kept(self, level: int, stream=None):
        """Kept bitmaps (int32 view of uint32 words) [n_lanes][words] and counts [n_lanes]."""
        n_lanes = len(self.trees) * self.n_q * self.Hq
        W = self.words(level)
        dev = torch.device("cuda", torch.cuda.current_device())
        bits = torch.empty((n_lanes, W), dtype=torch.int32, device=dev)
        counts = torch.empty((n_lanes,), dtype=torch.int32, device=dev)
        zha_decoder_export_kept(self.handle, level, bits.data_ptr(), counts.data_ptr(), _stream(stream))
        return bits, counts

    def stats(self, stream=None) -> DecodeStats:
        return zha_decoder_stats(self.handle, _stream(stream))


# ----------------------------------------------------------------------------- sharded sequence

def shard_ranges(n_tokens: int, C: int, L: int, world: int):
    """Token ranges [(offset, count)] of a sequence split over `world` ranks: every range
    starts at a multiple of C^L, ranks 0 .. world-2 hold equal multiples of C^L (as many whole
    top nodes as an even split allows) and the last rank holds the rest, tail included."""
    if world < 1:
        raise ValueError("world must be >= 1")
    top = C ** L
    per = (n_tokens // top) // world * top
    out, off = [], 0
    for r in range(world):
        cnt = per if r < world - 1 else n_tokens - off
        out.append((off, cnt))
        off += cnt
    return out


def check_shard_ranges(ranges, C: int, L: int):
    """Raises ValueError unless the ranks' (offset, count) pairs tile [0, N) in rank order with
    offsets on multiples of C^L, every rank but the last holding whole top nodes, and at most
    2^24 level-1 nodes in the sequence (the conditions zha.h states for a sharded sequence)."""
    top = C ** L
    end = 0
    for r, (off, cnt) in enumerate(ranges):
        if off != end:
            raise ValueError("rank %d starts at token %d, expected %d" % (r, off, end))
        if off % top:
            raise ValueError("rank %d starts at token %d, not a multiple of C^L = %d" % (r, off, top))
        if cnt < 0 or (r < len(ranges) - 1 and cnt % top):
            raise ValueError("rank %d holds %d tokens; every rank but the last holds whole top nodes" % (r, cnt))
        end = off + cnt
    if end // C > (1 << 24):
        raise ValueError("a sharded sequence holds at most 2^24 level-1 nodes")
    return end


class ShardedDecoder:
    """This rank's part of a sequence split over ranks (zha_shard_*): its own tree over its
    tokens, the exchange buffers the protocol's collectives act on, and the calls of one
    protocol step each.  ``shard_steps`` runs the protocol; ``decode_sharded`` runs it with
    torch.distributed collectives, ``decode_local_shards`` with several shards of one process."""

    def __init__(self, tree: Tree, max_queries: int, rank: int, world: int, token_offset: int):
        self.tree = tree
        self.rank, self.world, self.token_offset = rank, world, token_offset
        self.handle = zha_shard_decoder_create(tree.handle, max_queries, rank, world, token_offset)
        g = tree.geom
        self.Hq, self.d, self.L = g.n_q_heads, g.d, g.L
        self.max_queries = max_queries
        dev = torch.device("cuda", torch.cuda.current_device())
        lanes = max_queries * self.Hq
        z = lambda *shape, dt: torch.zeros(shape, dtype=dt, device=dev)
        self.bufs = {
            "lane_max": z(lanes, dt=torch.int32), "lane_cnt": z(lanes, dt=torch.int32),
            "hist": z(lanes, SHARD_BINS, dt=torch.int64), "keys": z(lanes, SHARD_KEYS, dt=torch.int64),
            "nkeys": z(lanes, dt=torch.int32), "keys_all": z(world, lanes, SHARD_KEYS, dt=torch.int64),
            "nkeys_all": z(world, lanes, dt=torch.int32), "out": z(lanes, self.d, dt=torch.float32),
            "lse": z(lanes, dt=torch.float32), "out_all": z(world, lanes, self.d, dt=torch.float32),
            "lse_all": z(world, lanes, dt=torch.float32),
        }
        self.n_q = None
        self._ex = None

    def close(self):
        if self.handle:
            zha_decoder_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _exchange(self) -> ShardExchange:
        # the _all buffers are rank-major over the call's lanes: [world][lanes][...] packed
        lanes = self.n_q * self.Hq
        b = self.bufs
        self._packed = {k: b[k].view(-1)[: self.world * lanes * (b[k][0, 0].numel())].view(
            self.world, lanes, *b[k].shape[2:]) for k in ("keys_all", "nkeys_all", "out_all", "lse_all")}
        ex = ShardExchange()
        for k in ("lane_max", "lane_cnt", "hist", "keys", "nkeys", "out", "lse"):
            setattr(ex, k, b[k].data_ptr())
        for k, t in self._packed.items():
            setattr(ex, k, t.data_ptr())
        return ex

    def gathered(self, name: str) -> torch.Tensor:
        """A gathered buffer as [world][lanes][...] (packed for the current call)."""
        return self._packed[name]

    def local(self, name: str) -> torch.Tensor:
        lanes = self.n_q * self.Hq
        return self.bufs[name][:lanes]

    def begin(self, Q: torch.Tensor, p: float, stream=None):
        _need(Q, torch.bfloat16, "Q")
        if Q.dim() == 4:
            Q = Q[0]
        self.Q = Q
        self.n_q = Q.shape[0]
        self._ex = self._exchange()
        zha_shard_begin(self.handle, Q.data_ptr(), self.n_q, p, _stream(stream))

    def score(self, level: int, stream=None):
        zha_shard_score(self.handle, level, self._ex, _stream(stream))

    def hist(self, level: int, stream=None):
        zha_shard_hist(self.handle, level, self._ex, _stream(stream))

    def cut(self, level: int, stream=None):
        zha_shard_cut(self.handle, level, self._ex, _stream(stream))

    def finish(self, level: int, stream=None):
        zha_shard_finish(self.handle, level, self._ex, _stream(stream))

    def attend(self, K: torch.Tensor, V: torch.Tensor, stream=None):
        _need(K, torch.bfloat16, "K")
        _need(V, torch.bfloat16, "V")
        zha_shard_attend(self.handle, K.data_ptr(), V.data_ptr(), self._ex, _stream(stream))

    def combine(self, out: torch.Tensor, stream=None):
        _need(out, torch.float32, "out")
        zha_shard_combine(self.handle, self._ex, out.data_ptr(), _stream(stream))

    def set_sync(self, on: bool = True):
        zha_decoder_set_sync(self.handle, on)

    def set_kernels(self, score: int = ZHA_KERNELS_AUTO, attn: int = ZHA_KERNELS_AUTO):
        zha_decoder_set_kernels(self.handle, score, attn)

    def words(self, level: int) -> int:
        return zha_decoder_words(self.handle, level)

    def export_kept(self, level: int, stream=None):
        """This shard's kept bitmaps [n_q x n_q_heads][words] (local node indices) and counts."""
        lanes = self.n_q * self.Hq
        W = self.words(level)
        dev = torch.device("cuda", torch.cuda.current_device())
        bits = torch.empty((lanes, W), dtype=torch.int32, device=dev)
        counts = torch.empty((lanes,), dtype=torch.int32, device=dev)
        zha_decoder_export_kept(self.handle, level, bits.data_ptr(), counts.data_ptr(), _stream(stream))
        return bits, counts

    def stats(self, stream=None) -> DecodeStats:
        return zha_decoder_stats(self.handle, _stream(stream))


def shard_steps(engine, K, V, Q, p: float, out):
    """The sharded decode protocol of one rank (zha.h, "sharded sequence"), as a generator:
    it makes the engine's calls and yields each collective as ("max" | "sum", name) or
    ("gather", name_all, name), for the caller to run over the ranks before resuming."""
    engine.begin(Q, p)
    for level in range(engine.L, 0, -1):
        engine.score(level)
        yield ("max", "lane_max")
        yield ("sum", "lane_cnt")
        engine.hist(level)
        yield ("sum", "hist")
        engine.cut(level)
        yield ("gather", "keys_all", "keys")
        yield ("gather", "nkeys_all", "nkeys")
        engine.finish(level)
    engine.attend(K, V)
    yield ("gather", "out_all", "out")
    yield ("gather", "lse_all", "lse")
    engine.combine(out)


class TorchCollectives:
    """The protocol's collectives over a torch.distributed process group (NCCL on GPUs)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group

    def run(self, engine, op):
        dist = self.dist
        if op[0] == "max":
            dist.all_reduce(engine.local(op[1]), op=dist.ReduceOp.MAX, group=self.group)
        elif op[0] == "sum":
            dist.all_reduce(engine.local(op[1]), op=dist.ReduceOp.SUM, group=self.group)
        else:
            dst, src = engine.gathered(op[1]), engine.local(op[2])
            if dist.get_backend(self.group) == "nccl":
                dist.all_gather_into_tensor(dst, src, group=self.group)
            else:
                parts = [torch.empty_like(src) for _ in range(dst.shape[0])]
                dist.all_gather(parts, src, group=self.group)
                dst.copy_(torch.stack(parts))


def decode_sharded(engine, K, V, Q, p: float, out, coll=None):
    """One rank's sharded decode: the protocol with its collectives run by `coll`
    (TorchCollectives over the default process group if None)."""
    coll = coll or TorchCollectives()
    for op in shard_steps(engine, K, V, Q, p, out):
        coll.run(engine, op)
    return out


def reduce_local(engines, op):
    """A protocol collective over shards that live in this one process (same device): the
    reduction or gather of the engines' buffers, written back into each."""
    if op[0] in ("max", "sum"):
        xs = torch.stack([e.local(op[1]) for e in engines])
        r = xs.max(0).values if op[0] == "max" else xs.sum(0)
        for e in engines:
            e.local(op[1]).copy_(r)
    else:
        g = torch.stack([e.local(op[2]) for e in engines])
        for e in engines:
            e.gathered(op[1]).copy_(g)


def decode_local_shards(engines, Ks, Vs, Q, p: float, outs):
    """The sharded decode of several shards held by one process, in lockstep: every shard's
    protocol advances to its next collective, the collective is taken over all of them, and
    so on.  No kernel waits on another shard's kernel."""
    gens = [shard_steps(e, K, V, Q, p, o) for e, K, V, o in zip(engines, Ks, Vs, outs)]
    while True:
        ops = []
        for g in gens:
            ops.append(next(g, None))
        if all(o is None for o in ops):
            return outs
        if any(o is None for o in ops) or any(o != ops[0] for o in ops):
            raise RuntimeError("shards left the protocol out of step: %s" % (ops,))
        reduce_local(engines, ops[0])
