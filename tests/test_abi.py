"""Host-side checks of the C ABI that need no GPU: the library builds for sm_100a,
loads, exports every function include/zha.h declares, and rejects bad arguments with
status codes before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

from hierarchical_tree_indexed_build_b200 import build_ext, zha

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "zha.h")


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(zha_[a-z_]+)\s*\(", txt)))


@pytest.fixture(scope="module")
def libzha():
    build_ext.build()
    return zha.lib()


def test_header_declarations_match_binding():
    assert _declared() == sorted(zha.EXPORTS)


def test_library_exports_every_declared_symbol(libzha):
    out = subprocess.run(["nm", "-D", "--defined-only", zha.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r" T (zha_\w+)", out))
    for name in _declared():
        assert name in exported, name
        assert hasattr(libzha, name)


def test_build_targets_sm100a_only():
    assert build_ext.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]
    assert "-lineinfo" in build_ext.FLAGS


@pytest.mark.parametrize("field,value", [("C", 1), ("C", 2048), ("L", 0), ("L", 17), ("R", 3), ("R", 64),
                                         ("d", 96), ("n_kv_heads", 0), ("n_q_heads", 3), ("capacity", 0),
                                         ("capacity", 1 << 31), ("format", 3), ("format", -1)])
def test_tree_create_rejects_bad_geometry(libzha, field, value):
    g = zha.Geometry(4, 6, 16, 128, 16, 2, 65536)
    setattr(g, field, value)
    h = ctypes.c_void_p()
    st = libzha.zha_tree_create(ctypes.byref(g), ctypes.byref(h))
    assert st == zha.ZHA_ERR_ARG
    assert libzha.zha_last_error().decode() != ""
    assert h.value is None


def test_null_handles_are_rejected(libzha):
    assert libzha.zha_tree_destroy(None) == zha.ZHA_OK
    assert libzha.zha_decoder_destroy(None) == zha.ZHA_OK
    assert libzha.zha_build_tree(None, None, 0, None, None) == zha.ZHA_ERR_ARG
    assert libzha.zha_append(None, None, 0, 0, None) == zha.ZHA_ERR_ARG
    assert libzha.zha_tree_export(None, 1, None, None, None, None) == zha.ZHA_ERR_ARG
    h = ctypes.c_void_p()
    assert libzha.zha_decoder_create(None, 0, 1, ctypes.byref(h)) == zha.ZHA_ERR_ARG
    assert libzha.zha_route(None, None, 1, 0.9, None) == zha.ZHA_ERR_ARG
    assert libzha.zha_sparse_attn(None, None, None, None, 1, None, None) == zha.ZHA_ERR_ARG
    assert libzha.zha_dense_attn(None, None, None, None, 1, None, None) == zha.ZHA_ERR_ARG
    assert libzha.zha_shard_decoder_create(None, 1, 0, 1, 0, ctypes.byref(h)) == zha.ZHA_ERR_ARG
    assert libzha.zha_shard_begin(None, None, 1, 0.9, None) == zha.ZHA_ERR_ARG
    ex = zha.ShardExchange()
    for fn in (libzha.zha_shard_score, libzha.zha_shard_hist, libzha.zha_shard_cut, libzha.zha_shard_finish):
        assert fn(None, 1, ctypes.byref(ex), None) == zha.ZHA_ERR_ARG
    assert libzha.zha_shard_attend(None, None, None, ctypes.byref(ex), None) == zha.ZHA_ERR_ARG
    assert libzha.zha_shard_combine(None, ctypes.byref(ex), None, None) == zha.ZHA_ERR_ARG
    assert libzha.zha_decoder_export_kept(None, 1, None, None, None) == zha.ZHA_ERR_ARG
    assert libzha.zha_decoder_words(None, 1) == 0
    assert libzha.zha_decoder_stats(None, None, None) == zha.ZHA_ERR_ARG
    assert libzha.zha_tree_info(None, None, None, None, None) == zha.ZHA_ERR_ARG


def test_binding_raises_on_error_status(libzha):
    with pytest.raises(zha.ZhaError) as ei:
        zha.zha_tree_create(zha.Geometry(1, 1, 1, 64, 1, 1, 16))
    assert ei.value.status == zha.ZHA_ERR_ARG


def test_shard_exchange_layout_matches_the_header():
    # eleven pointers, in the order zha.h declares them
    assert ctypes.sizeof(zha.ShardExchange) == 11 * ctypes.sizeof(ctypes.c_void_p)
    names = [f[0] for f in zha.ShardExchange._fields_]
    hdr = open(os.path.join(ROOT, "include", "zha.h")).read()
    body = hdr[hdr.index("typedef struct zha_shard_exchange"):hdr.index("} zha_shard_exchange;")]
    flat = body.replace(" ", "")
    pos = [flat.index("*" + n + ";") for n in names]
    assert pos == sorted(pos)
    assert "#define ZHA_SHARD_BINS %d" % zha.SHARD_BINS in hdr
    assert "#define ZHA_SHARD_KEYS %d" % zha.SHARD_KEYS in hdr
