"""ctypes wrapper of the float64 ZHA oracle (zha_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
CPU-baseline leg of the benchmark.  The CUDA path never imports it.  All arrays are
numpy float64 (keys, values and queries upcast exactly from their bf16 values).
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import List, Optional, Sequence

import numpy as np

from . import build as _build

_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.POINTER(ctypes.c_int64)
_I32 = ctypes.POINTER(ctypes.c_int32)
_U8 = ctypes.POINTER(ctypes.c_uint8)


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(_build.build())
        L.zo_num_threads.restype = ctypes.c_int
        L.zo_summaries.argtypes = [_D, ctypes.c_int, _D, ctypes.c_int, ctypes.c_int64, _I64,
                                   ctypes.c_int64, _D, _D, _D]
        L.zo_plane_estimate.argtypes = [_D, _D, ctypes.c_int, ctypes.c_int, _D]
        L.zo_plane_estimate.restype = ctypes.c_double
        L.zo_true_log_mass.argtypes = [_D, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, _D]
        L.zo_true_log_mass.restype = ctypes.c_double
        L.zo_topp.argtypes = [_D, _I64, ctypes.c_int64, ctypes.c_double, _U8, _D]
        L.zo_topp.restype = ctypes.c_int64
        L.zo_route.argtypes = [_D, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                               _D, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                               _D, _I32, ctypes.c_int, ctypes.c_double,
                               _U8, _U8, _D, _I64, _I64, _D]
        L.zo_attended_set.argtypes = [_U8, ctypes.c_int64, ctypes.c_int, ctypes.c_int, _I64]
        L.zo_attended_set.restype = ctypes.c_int64
        L.zo_attend.argtypes = [_D, _D, ctypes.c_int, _D, _I64, ctypes.c_int64, _D]
        L.zo_attend_batch.argtypes = [_D, _D, ctypes.c_int64, ctypes.c_int, _D, _I32, ctypes.c_int,
                                      _I64, _I64, _D]
        _lib = L
    return _lib


def num_threads() -> int:
    return lib().zo_num_threads()


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a, ptype):
    return a.ctypes.data_as(ptype)


def summaries(K: np.ndarray, qref: np.ndarray, span: int, nodes: Optional[Sequence[int]] = None):
    """Definition-level summaries of nodes of one KV head.

    K [N][d], qref [R][d]; node i covers tokens [i*span, (i+1)*span).  ``nodes`` defaults
    to every complete node.  Returns (m [n][R][d], lse [n][R], b [n][R])."""
    K = _c(K, np.float64)
    qref = _c(qref, np.float64)
    N, d = K.shape
    R = qref.shape[0]
    if nodes is None:
        nodes = np.arange(N // span, dtype=np.int64)
    nodes = _c(nodes, np.int64)
    assert nodes.size == 0 or (nodes.min() >= 0 and (nodes.max() + 1) * span <= N)
    n = nodes.size
    m = np.empty((n, R, d))
    lse = np.empty((n, R))
    b = np.empty((n, R))
    lib().zo_summaries(_p(K, _D), d, _p(qref, _D), R, span, _p(nodes, _I64), n,
                       _p(m, _D), _p(lse, _D), _p(b, _D))
    return m, lse, b


def plane_estimate(m: np.ndarray, b: np.ndarray, q: np.ndarray) -> float:
    m = _c(m, np.float64); b = _c(b, np.float64); q = _c(q, np.float64)
    R, d = m.shape
    return lib().zo_plane_estimate(_p(m, _D), _p(b, _D), R, d, _p(q, _D))


def true_log_mass(K: np.ndarray, t0: int, t1: int, q: np.ndarray) -> float:
    K = _c(K, np.float64); q = _c(q, np.float64)
    return lib().zo_true_log_mass(_p(K, _D), t0, t1, K.shape[1], _p(q, _D))


def topp(e: np.ndarray, idx: np.ndarray, p: float):
    """Top-p cut.  Returns (keep bool [n], k*, info[4])."""
    e = _c(e, np.float64); idx = _c(idx, np.int64)
    n = e.size
    keep = np.zeros(max(n, 1), dtype=np.uint8)
    info = np.empty(4)
    k = lib().zo_topp(_p(e, _D), _p(idx, _I64), n, float(p), _p(keep, _U8), _p(info, _D))
    return keep[:n].astype(bool), int(k), info


@dataclass
class Route:
    kept: List[np.ndarray]      # index l-1: bool [n_lanes][n_l]
    info: np.ndarray            # [L][n_lanes][4] decision margins (see zo_topp)
    kstar: np.ndarray           # [L][n_lanes]
    nfront: np.ndarray          # [L][n_lanes]
    scores: Optional[List[np.ndarray]] = None   # index l-1: [n_lanes][n_l] frontier estimates


def level_sizes(N: int, C: int, L: int) -> List[int]:
    return [N // C ** l for l in range(1, L + 1)]


def route(K: np.ndarray, qref: np.ndarray, C: int, L: int, N: int, q: np.ndarray,
          lane_g: np.ndarray, p: float, forced: Optional[List[np.ndarray]] = None,
          return_scores: bool = False) -> Route:
    """Top-down top-p routing of lanes through one sequence's tree.

    K [Hkv][ld][d]; qref [Hkv][R][d]; q [n_lanes][d]; lane_g [n_lanes].  ``forced`` (replay
    mode) is a per-level list of bool [n_lanes][n_l] kept sets that define the next
    frontier instead of the oracle's own."""
    K = _c(K, np.float64); qref = _c(qref, np.float64); q = _c(q, np.float64)
    lane_g = _c(lane_g, np.int32)
    Hkv, ld, d = K.shape
    R = qref.shape[1]
    n_lanes = q.shape[0]
    n1 = max(N // C, 1)
    sizes = level_sizes(N, C, L)
    kept = np.zeros((L, n_lanes, n1), dtype=np.uint8)
    fbuf = None
    if forced is not None:
        fbuf = np.zeros((L, n_lanes, n1), dtype=np.uint8)
        for v in range(L):
            fbuf[v, :, :sizes[v]] = np.asarray(forced[v], dtype=np.uint8)[:, :sizes[v]]
    info = np.empty((L, n_lanes, 4))
    kstar = np.empty((L, n_lanes), dtype=np.int64)
    nfront = np.empty((L, n_lanes), dtype=np.int64)
    sc = np.full((L, n_lanes, n1), np.nan) if return_scores else None
    lib().zo_route(_p(K, _D), ld, N, Hkv, d, _p(qref, _D), R, C, L, _p(q, _D), _p(lane_g, _I32),
                   n_lanes, float(p), _p(kept, _U8),
                   _p(fbuf, _U8) if fbuf is not None else ctypes.cast(None, _U8),
                   _p(info, _D), _p(kstar, _I64), _p(nfront, _I64),
                   _p(sc, _D) if sc is not None else ctypes.cast(None, _D))
    return Route([kept[v, :, :sizes[v]].astype(bool) for v in range(L)], info, kstar, nfront,
                  [sc[v, :, :sizes[v]] for v in range(L)] if sc is not None else None)


def attended_set(kept1: np.ndarray, N: int, C: int, L: int) -> np.ndarray:
    n1 = N // C
    k = np.zeros(max(n1, 1), dtype=np.uint8)
    k[:n1] = np.asarray(kept1, dtype=np.uint8)[:n1]
    tok = np.empty(max(N, 1), dtype=np.int64)
    n = lib().zo_attended_set(_p(k, _U8), N, C, L, _p(tok, _I64))
    return tok[:n].copy()


def attend(K: np.ndarray, V: np.ndarray, q: np.ndarray, tokens: np.ndarray) -> np.ndarray:
    """Exact softmax attention of q over the listed rows of K, V ([*][d], one head)."""
    K = _c(K, np.float64); V = _c(V, np.float64); q = _c(q, np.float64)
    tokens = _c(tokens, np.int64)
    out = np.empty(K.shape[1])
    lib().zo_attend(_p(K, _D), _p(V, _D), K.shape[1], _p(q, _D), _p(tokens, _I64), tokens.size,
                    _p(out, _D))
    return out


def attend_batch(K: np.ndarray, V: np.ndarray, q: np.ndarray, lane_g: np.ndarray,
                 token_lists: List[np.ndarray]) -> np.ndarray:
    """attend() for many lanes at once (OpenMP); K, V [Hkv][ld][d]."""
    K = _c(K, np.float64); V = _c(V, np.float64); q = _c(q, np.float64)
    lane_g = _c(lane_g, np.int32)
    Hkv, ld, d = K.shape
    offs = np.zeros(len(token_lists) + 1, dtype=np.int64)
    offs[1:] = np.cumsum([t.size for t in token_lists])
    tok = _c(np.concatenate(token_lists) if token_lists else np.zeros(1), np.int64)
    out = np.empty((len(token_lists), d))
    lib().zo_attend_batch(_p(K, _D), _p(V, _D), ld, d, _p(q, _D), _p(lane_g, _I32),
                          len(token_lists), _p(tok, _I64), _p(offs, _I64), _p(out, _D))
    return out


def decode(K: np.ndarray, V: np.ndarray, qref: np.ndarray, C: int, L: int, N: int,
           q: np.ndarray, lane_g: np.ndarray, p: float,
           forced: Optional[List[np.ndarray]] = None):
    """Route + attend, end to end.  Returns (Route, out [n_lanes][d], token lists)."""
    r = route(K, qref, C, L, N, q, lane_g, p, forced)
    kept1 = (forced[0] if forced is not None else r.kept[0]) if L >= 1 else None
    toks = [attended_set(kept1[x], N, C, L) for x in range(q.shape[0])]
    out = attend_batch(K, V, q, lane_g, toks)
    return r, out, toks


# MXFP4 (OCP Microscaling Formats (MX) Specification v1.0: the E2M1 element type, the E8M0
# shared scale and the conversion of a block of 32 values): the reduced-precision slope
# records of an FP4 router.  E2M1 magnitudes, indexed by the 3 low bits of a code
# (2 exponent bits, 1 mantissa bit, exponent bias 1):
E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def mxfp4(x: np.ndarray, block: int = 32):
    """Rounds x [..., n] (n a multiple of `block`) to MXFP4, block by block along the last axis.

    Per block: shared scale X = 2^(floor(log2 max|x|) - 2), the largest power of two not above
    the block maximum divided by 2^2 (2 being E2M1's largest exponent), as the E8M0 byte
    floor(log2 max|x|) - 2 + 127 clamped to [0, 254] (0 for an all-zero block); every element
    becomes the E2M1 value nearest to x / X, ties to the value with an even mantissa bit,
    magnitudes beyond 6 saturated to 6, keeping the sign.
    Returns (decoded values float64 [..., n], codes uint8 [..., n] (sign in bit 3; none for 0),
    scale bytes uint8 [..., n / block])."""
    x = np.asarray(x, dtype=np.float64)
    shp = x.shape
    xb = x.reshape(shp[:-1] + (shp[-1] // block, block))
    amax = np.abs(xb).max(axis=-1)
    _, ex = np.frexp(amax)                         # amax = f 2^ex, f in [0.5, 1): floor(log2) = ex - 1
    E = np.where(amax > 0, np.clip(ex - 1 - 2 + 127, 0, 254), 0).astype(np.int64)
    X = np.ldexp(1.0, E - 127)[..., None]
    y = xb / X
    a = np.abs(y)
    # nearest E2M1 magnitude: the midpoints between neighbours, a tie going to the even code
    mids = (E2M1_VALUES[:-1] + E2M1_VALUES[1:]) / 2       # 0.25 0.75 1.25 1.75 2.5 3.5 5
    idx = np.zeros(a.shape, dtype=np.int64)
    for k, mid in enumerate(mids):
        up_is_even = (k + 1) % 2 == 0
        idx += (a >= mid) if up_is_even else (a > mid)
    val = np.sign(y) * E2M1_VALUES[idx] * X
    codes = (idx | np.where((y < 0) & (idx > 0), 8, 0)).astype(np.uint8)
    return val.reshape(shp), codes.reshape(shp), E.astype(np.uint8)
