"""The C-ABI library loads and exports every symbol include/tfpaged.h
declares; host-side argument checks answer without touching a GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

import paged_kv_cache_segment_b200 as tf
from paged_kv_cache_segment_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"TF_API\s+[\w\s\*]+?\b(tf_\w+)\s*\(", src)
    return names


def test_header_declares_the_calls():
    names = declared_symbols()
    for n in ("tf_paged_attn_decode", "tf_attn_merge", "tf_paged_attn_prompt", "tf_ring_attn", "tf_argmax_rows"):
        assert n in names
    assert set(binding.EXPORTS) == set(names)


def test_library_exports_every_declared_symbol():
    lib = tf.load()
    for n in declared_symbols():
        assert hasattr(lib, n), n
    assert tf.tf_abi_version() == 1
    assert tf.tf_status_str(0) == "ok"


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: every case below fails a host check first


def call_decode(**kw):
    lib = tf.load()
    a = dict(q=FAKE, rows=4, hq=8, k=FAKE, v=FAKE, n_pages=16, psz=16, hkv=2, d=64, pt=FAKE, pt_len=8, segs=FAKE,
             n_segs=2, segs_host=None, pt_host=None, scale=0.125, split=0, nsm=2, po=FAKE, pm=FAKE, pl=FAKE, pf=FAKE,
             st=FAKE, stream=None)
    a.update(kw)
    return lib.tf_paged_attn_decode(*a.values())


def test_host_checks_of_decode():
    assert call_decode(d=96) == 4  # unsupported head dim
    assert call_decode(psz=24) == 4  # page size not a power of two
    assert call_decode(hq=7) == 4  # Hq not a multiple of Hkv
    assert call_decode(nsm=0) == 1
    assert call_decode(q=ctypes.c_void_p(0x10008)) == 6  # misaligned
    assert call_decode(scale=float("nan")) == 1
    assert call_decode(n_segs=0) == 0  # nothing to do, nothing launched
    segs = np.array([[0, 1, 37, 0, 3], [1, 1, 70, 3, 5]], np.int32)
    assert call_decode(segs_host=segs.ctypes.data_as(ctypes.c_void_p), n_segs=2, pt_len=8,
                       nsm=1, split=16) == 1  # needs more than one partial
    bad = segs.copy()
    bad[0, 2] = 49  # 3 pages of 16 hold 48 keys
    assert call_decode(segs_host=bad.ctypes.data_as(ctypes.c_void_p)) == 2
    pt = np.arange(8, dtype=np.int32)
    pt[4] = 16
    assert call_decode(segs_host=segs.ctypes.data_as(ctypes.c_void_p), pt_host=pt.ctypes.data_as(ctypes.c_void_p)) == 3
    zero_rows = segs.copy()
    zero_rows[:, 1] = 0
    assert call_decode(segs_host=zero_rows.ctypes.data_as(ctypes.c_void_p)) == 0


def test_host_checks_of_other_calls():
    lib = tf.load()
    assert lib.tf_attn_merge(FAKE, FAKE, FAKE, FAKE, 4, 8, 100, 2, FAKE, FAKE, None) == 4
    assert lib.tf_argmax_rows(FAKE, 4, 0, 10, FAKE, FAKE, None) == 1
    assert lib.tf_argmax_rows(FAKE, 4, 20, 10, FAKE, FAKE, None) == 1
    assert lib.tf_argmax_rows(FAKE, 0, 20, 20, FAKE, FAKE, None) == 0
    assert lib.tf_ring_workspace_bytes(17, 16, 256, 17) >= 17 * 16 * 17 * (256 + 2) * 4
    rs = np.zeros(1, binding.RING_SEG_DTYPE)
    rs[0] = (0, 0, 100, 5, 101)  # more valid slots than the ring holds
    ws = lib.tf_ring_workspace_bytes(1, 8, 64, 4)
    assert lib.tf_ring_attn(FAKE, 1, 8, FAKE, FAKE, 100, 2, 64, FAKE, 1, rs.ctypes.data_as(ctypes.c_void_p), 0.1, 64,
                            4, FAKE, ws, FAKE, FAKE, FAKE, None) == 1
    assert lib.tf_ring_attn(FAKE, 1, 8, FAKE, FAKE, 100, 2, 64, FAKE, 1, None, 0.1, 64, 4, FAKE, ws - 1, FAKE, FAKE,
                            FAKE, None) == 7
    seg = np.array([[0, 4, 3, 0, 1]], np.int32)  # more rows than keys
    assert lib.tf_paged_attn_prompt(FAKE, 4, 8, FAKE, FAKE, 4, 16, 2, 64, FAKE, 1, seg.ctypes.data_as(ctypes.c_void_p),
                                    0.1, FAKE, 1, None, FAKE, None) == 1


def test_host_checks_of_block_and_append():
    lib = tf.load()
    segs = np.array([[0, 4, 2, 0, 1]], np.int32)  # a block of 4 rows over 2 keys
    a = dict(q=FAKE, rows=4, hq=8, k=FAKE, v=FAKE, n_pages=16, psz=16, hkv=2, d=64, pt=FAKE, pt_len=8, segs=FAKE,
             n_segs=1, segs_host=segs.ctypes.data_as(ctypes.c_void_p), pt_host=None, scale=0.125, split=16, nsm=2,
             po=FAKE, pm=FAKE, pl=FAKE, pf=FAKE, st=FAKE, stream=None)
    assert call_decode(**a) == 1  # the causal count needs a key per row
    b = dict(a, d=96)
    assert lib.tf_paged_attn_block(*b.values()) == 4  # unsupported head dim
    none = segs.copy()
    none[0, 2] = 0  # rows but no key at all
    b = dict(a, segs_host=none.ctypes.data_as(ctypes.c_void_p))
    assert lib.tf_paged_attn_block(*b.values()) == 1

    def append(**kw):
        c = dict(kr=FAKE, vr=FAKE, rows=4, kp=FAKE, vp=FAKE, n_pages=16, psz=16, hkv=2, d=64, pt=FAKE, pt_len=8,
                 segs=FAKE, n_segs=1, segs_host=None, pt_host=None, st=FAKE, stream=None)
        c.update(kw)
        return lib.tf_kv_append(*c.values())

    assert append(d=96) == 4
    assert append(psz=24) == 4
    assert append(kr=ctypes.c_void_p(0x10008)) == 6  # misaligned
    assert append(n_segs=0) == 0
    rows_past = np.array([[0, 2, 17, 0, 1]], np.int32)  # key 16 lies past the one page of 16
    assert append(segs_host=rows_past.ctypes.data_as(ctypes.c_void_p)) == 2
    few_keys = np.array([[0, 3, 2, 0, 1]], np.int32)  # more new rows than keys
    assert append(segs_host=few_keys.ctypes.data_as(ctypes.c_void_p)) == 1
    pt = np.array([16], np.int32)  # a page id outside the pool
    ok = np.array([[0, 2, 5, 0, 1]], np.int32)
    assert append(segs_host=ok.ctypes.data_as(ctypes.c_void_p), pt_host=pt.ctypes.data_as(ctypes.c_void_p),
                  pt_len=1) == 3


def call_tree(**kw):
    lib = tf.load()
    a = dict(q=FAKE, rows=8, hq=8, k=FAKE, v=FAKE, slots=100, hkv=2, d=64, ts=FAKE, n_segs=1, ts_host=None,
             par=FAKE, n_par=8, par_host=None, scale=0.125, split=64, nsm=3, ws=FAKE, ws_bytes=1 << 30, out=FAKE,
             flags=FAKE, st=FAKE, stream=None)
    a.update(kw)
    return lib.tf_ring_tree_attn(*a.values())


def test_host_checks_of_the_tree_call():
    ts = np.zeros(1, binding.TREE_SEG_DTYPE)
    ts[0] = (0, 0, 50, 7, 20, 8, 0)
    par = np.array([-1, 0, 1, 1, 0, -1, 5, 2], np.int32)
    host = dict(ts_host=ts.ctypes.data_as(ctypes.c_void_p), par_host=par.ctypes.data_as(ctypes.c_void_p))
    assert call_tree(d=96) == 4  # head dim
    assert call_tree(hq=6) == 4  # 6 q-heads over 2 kv-heads: a group of 3 does not divide 128
    assert call_tree(split=32) == 4  # splits of fewer than 64 slots
    assert call_tree(nsm=0) == 1
    assert call_tree(n_segs=0) == 0
    assert call_tree(q=ctypes.c_void_p(0x10008)) == 6
    assert call_tree(ws_bytes=1000) == 7  # workspace too small
    assert tf.tf_ring_tree_workspace_bytes(8, 8, 64, 3) == -(-(8 * 8 * 3 * (64 * 4 + 9)) // 256) * 256
    # host tables: a parent at or past its node, a window plus nodes past the ring, too few partials
    for bad_par in ([-1, 1, 1, 1, 0, -1, 5, 2], [-1, 0, 1, 1, 0, -1, 7, 2], [-2, 0, 1, 1, 0, -1, 5, 2]):
        p2 = np.array(bad_par, np.int32)
        assert call_tree(ts_host=ts.ctypes.data_as(ctypes.c_void_p), par_host=p2.ctypes.data_as(ctypes.c_void_p)) == 1
    t2 = ts.copy()
    t2[0]["n_valid"] = 43
    assert call_tree(ts_host=t2.ctypes.data_as(ctypes.c_void_p), par_host=host["par_host"]) == 1
    assert call_tree(nsm=1, **host) == 1  # 28 keys that wrap need 2 partials
