"""float64 CPU oracle: ctypes binding of ``oracle.c``.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The library under
``paged_kv_cache_segment_b200`` never imports it, and this package imports
nothing from that library's compute path (it reads inputs produced by the
separate ``workloads`` generator module only through plain numpy arrays).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

RING_SEG_DTYPE = np.dtype(
    [("base", "<i8"), ("q_row", "<i4"), ("size", "<i4"), ("head", "<i4"), ("n_valid", "<i4")]
)

TREE_SEG_DTYPE = np.dtype(
    [("base", "<i8"), ("q_row", "<i4"), ("size", "<i4"), ("head", "<i4"), ("n_valid", "<i4"), ("n_nodes", "<i4"),
     ("parent_base", "<i4")]
)

ERRORS = {0: "ok", 1: "bad argument", 2: "keys past the stream's pages", 3: "page id outside the pool", 4: "out of memory"}


def build(src: str = _SRC, out: str = _LIB, extra: list[str] | None = None) -> str:
    """Compile the oracle with gcc (IEEE float64, OpenMP over independent units)."""
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c11", "-Wall", "-Wno-unknown-pragmas",
           src, "-o", out, "-lm"] + (extra or [])
    subprocess.run(cmd, check=True)
    return out


def _needs_build() -> bool:
    return (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)


class Oracle:
    """One loaded copy of the oracle library (a planted-control build loads its own)."""

    def __init__(self, path: str | None = None):
        if path is None:
            if _needs_build():
                build()
            path = _LIB
        self.path = path
        self.lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        L = self.lib
        L.orc_num_threads.restype = ctypes.c_int
        L.orc_gather_paged.argtypes = [P, P, i32, i32, i32, i32, P, i32, i32, i32, P, P]
        L.orc_gather_paged.restype = ctypes.c_int
        L.orc_paged_attn.argtypes = [P, i32, i32, P, P, i32, i32, i32, i32, P, i32, P, i32, f64, i32, P, P, P]
        L.orc_put_rows.argtypes = [P, P, i32, i32, i32, P, P, i32, i32, P, i32, P, i32]
        L.orc_paged_attn.restype = ctypes.c_int
        L.orc_partial.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, f64, P, P, P, P]
        L.orc_partial.restype = None
        L.orc_merge.argtypes = [P, P, P, P, i32, i32, P, P]
        L.orc_merge.restype = None
        L.orc_paged_partials.argtypes = [P, i32, i32, P, P, i32, i32, i32, i32, P, i32, P, i32, f64, i32, i32,
                                         P, P, P, P]
        L.orc_paged_partials.restype = ctypes.c_int
        L.orc_ring_attn.argtypes = [P, i32, i32, P, P, i64, i32, i32, P, i32, f64, P, P]
        L.orc_ring_attn.restype = ctypes.c_int
        L.orc_ring_tree_attn.argtypes = [P, i32, i32, P, P, i64, i32, i32, P, i32, P, i32, f64, P, P]
        L.orc_ring_tree_attn.restype = ctypes.c_int
        L.orc_argmax_rows.argtypes = [P, i32, i32, i64, P, P]
        L.orc_argmax_rows.restype = None

    # ------------------------------------------------------------------ utils
    @staticmethod
    def _p(a: np.ndarray):
        return a.ctypes.data_as(ctypes.c_void_p)

    @staticmethod
    def _check(rc: int, what: str):
        if rc != 0:
            raise ValueError(f"oracle {what}: {ERRORS.get(rc, rc)}")

    def num_threads(self) -> int:
        return int(self.lib.orc_num_threads())

    # --------------------------------------------------------------- gather
    def gather_paged(self, k_pool, v_pool, page_table, pt_base, n_stream_pages, n_keys):
        k_pool = np.ascontiguousarray(k_pool, np.uint16)
        v_pool = np.ascontiguousarray(v_pool, np.uint16)
        pt = np.ascontiguousarray(page_table, np.int32)
        n_pages, hkv, psz, d = k_pool.shape
        kd = np.zeros((n_keys, hkv, d), np.float64)
        vd = np.zeros((n_keys, hkv, d), np.float64)
        rc = self.lib.orc_gather_paged(self._p(k_pool), self._p(v_pool), n_pages, psz, hkv, d, self._p(pt),
                                       pt_base, n_stream_pages, n_keys, self._p(kd), self._p(vd))
        self._check(rc, "gather")
        return kd, vd

    # ------------------------------------------------------- rows into pages
    def put_rows(self, k_rows, v_rows, k_pool, v_pool, page_table, segs):
        """Copies of the pools with each stream's new rows written into its pages
        (orc_put_rows); k_rows, v_rows bf16 bits [rows][Hkv][D]."""
        k_rows = np.ascontiguousarray(k_rows, np.uint16)
        v_rows = np.ascontiguousarray(v_rows, np.uint16)
        kp = np.array(k_pool, np.uint16, copy=True, order="C")
        vp = np.array(v_pool, np.uint16, copy=True, order="C")
        pt = np.ascontiguousarray(page_table, np.int32)
        segs = np.ascontiguousarray(segs, np.int32).reshape(-1, 5)
        rows, hkv, d = k_rows.shape
        n_pages, hkv2, psz, d2 = kp.shape
        assert (hkv, d) == (hkv2, d2) and v_rows.shape == k_rows.shape
        rc = self.lib.orc_put_rows(self._p(k_rows), self._p(v_rows), rows, hkv, d, self._p(kp), self._p(vp), n_pages,
                                   psz, self._p(pt), len(pt), self._p(segs), len(segs))
        self._check(rc, "put_rows")
        return kp, vp

    # ------------------------------------------------------- paged attention
    def paged_attn(self, q, k_pool, v_pool, page_table, segs, scale, full=False, sel=None):
        """float64 out [rows][Hq][D] and uint8 flags [rows][Hq]; unselected entries stay 0."""
        q = np.ascontiguousarray(q, np.uint16)
        k_pool = np.ascontiguousarray(k_pool, np.uint16)
        v_pool = np.ascontiguousarray(v_pool, np.uint16)
        pt = np.ascontiguousarray(page_table, np.int32)
        segs = np.ascontiguousarray(segs, np.int32).reshape(-1, 5)
        rows, hq, d = q.shape
        n_pages, hkv, psz, d2 = k_pool.shape
        assert d == d2
        out = np.zeros((rows, hq, d), np.float64)
        flags = np.zeros((rows, hq), np.uint8)
        selp = None
        if sel is not None:
            sel = np.ascontiguousarray(sel, np.uint8).reshape(rows, hq)
            selp = self._p(sel)
        rc = self.lib.orc_paged_attn(self._p(q), rows, hq, self._p(k_pool), self._p(v_pool), n_pages, psz, hkv, d,
                                     self._p(pt), len(pt), self._p(segs), len(segs), float(scale), int(bool(full)),
                                     selp, self._p(out), self._p(flags))
        self._check(rc, "paged_attn")
        return out, flags

    def paged_partials(self, q, k_pool, v_pool, page_table, segs, scale, split_keys, n_splits_max):
        q = np.ascontiguousarray(q, np.uint16)
        k_pool = np.ascontiguousarray(k_pool, np.uint16)
        v_pool = np.ascontiguousarray(v_pool, np.uint16)
        pt = np.ascontiguousarray(page_table, np.int32)
        segs = np.ascontiguousarray(segs, np.int32).reshape(-1, 5)
        rows, hq, d = q.shape
        n_pages, hkv, psz, _ = k_pool.shape
        c = n_splits_max
        po = np.zeros((rows, hq, c, d), np.float64)
        pm = np.full((rows, hq, c), -np.inf, np.float64)
        pl = np.zeros((rows, hq, c), np.float64)
        pf = np.zeros((rows, hq, c), np.uint8)
        rc = self.lib.orc_paged_partials(self._p(q), rows, hq, self._p(k_pool), self._p(v_pool), n_pages, psz, hkv,
                                         d, self._p(pt), len(pt), self._p(segs), len(segs), float(scale),
                                         int(split_keys), int(n_splits_max), self._p(po), self._p(pm), self._p(pl),
                                         self._p(pf))
        self._check(rc, "paged_partials")
        return po, pm, pl, pf

    def partial(self, qv, kd, vd, g, a, b, n_vis, scale):
        qv = np.ascontiguousarray(qv, np.float64)
        kd = np.ascontiguousarray(kd, np.float64)
        vd = np.ascontiguousarray(vd, np.float64)
        n, hkv, d = kd.shape
        o = np.zeros(d, np.float64)
        m = np.zeros(1, np.float64)
        l = np.zeros(1, np.float64)
        f = np.zeros(1, np.uint8)
        self.lib.orc_partial(self._p(qv), self._p(kd), self._p(vd), hkv, d, g, a, b, n_vis, float(scale),
                             self._p(o), self._p(m), self._p(l), self._p(f))
        return o, float(m[0]), float(l[0]), int(f[0])

    def merge(self, o, m, l, flag):
        o = np.ascontiguousarray(o, np.float64)
        m = np.ascontiguousarray(m, np.float64)
        l = np.ascontiguousarray(l, np.float64)
        flag = np.ascontiguousarray(flag, np.uint8)
        c, d = o.shape
        out = np.zeros(d, np.float64)
        of = np.zeros(1, np.uint8)
        self.lib.orc_merge(self._p(o), self._p(m), self._p(l), self._p(flag), c, d, self._p(out), self._p(of))
        return out, int(of[0])

    def merge_all(self, po, pm, pl, pf):
        """Merge partials [rows][Hq][C](*D) into out [rows][Hq][D], flags [rows][Hq]."""
        rows, hq, c, d = po.shape
        out = np.zeros((rows, hq, d), np.float64)
        flags = np.zeros((rows, hq), np.uint8)
        for r in range(rows):
            for h in range(hq):
                out[r, h], flags[r, h] = self.merge(po[r, h], pm[r, h], pl[r, h], pf[r, h])
        return out, flags

    # --------------------------------------------------------------- ring
    def ring_attn(self, q, ring_k, ring_v, rsegs, scale):
        q = np.ascontiguousarray(q, np.uint16)
        ring_k = np.ascontiguousarray(ring_k, np.uint16)
        ring_v = np.ascontiguousarray(ring_v, np.uint16)
        rs = np.ascontiguousarray(np.asarray(rsegs).astype(RING_SEG_DTYPE))
        rows, hq, d = q.shape
        slots, hkv, d2 = ring_k.shape
        assert d == d2
        out = np.zeros((rows, hq, d), np.float64)
        flags = np.zeros((rows, hq), np.uint8)
        rc = self.lib.orc_ring_attn(self._p(q), rows, hq, self._p(ring_k), self._p(ring_v), slots, hkv, d,
                                    self._p(rs), len(rs), float(scale), self._p(out), self._p(flags))
        self._check(rc, "ring_attn")
        return out, flags

    def ring_tree_attn(self, q, ring_k, ring_v, tsegs, parents, scale):
        """Draft trees over rings (orc_ring_tree_attn): float64 out [rows][Hq][D]
        and uint8 flags [rows][Hq]; rows no tree names stay 0."""
        q = np.ascontiguousarray(q, np.uint16)
        ring_k = np.ascontiguousarray(ring_k, np.uint16)
        ring_v = np.ascontiguousarray(ring_v, np.uint16)
        ts = np.ascontiguousarray(np.asarray(tsegs).astype(TREE_SEG_DTYPE))
        par = np.ascontiguousarray(np.asarray(parents, np.int32).reshape(-1))
        rows, hq, d = q.shape
        slots, hkv, d2 = ring_k.shape
        assert d == d2
        out = np.zeros((rows, hq, d), np.float64)
        flags = np.zeros((rows, hq), np.uint8)
        rc = self.lib.orc_ring_tree_attn(self._p(q), rows, hq, self._p(ring_k), self._p(ring_v), slots, hkv, d,
                                         self._p(ts), len(ts), self._p(par), len(par), float(scale), self._p(out),
                                         self._p(flags))
        self._check(rc, "ring_tree_attn")
        return out, flags

    # --------------------------------------------------------------- argmax
    def argmax_rows(self, logits, n_cols=None):
        logits = np.ascontiguousarray(logits, np.uint16)
        rows, ld = logits.shape
        n_cols = ld if n_cols is None else n_cols
        ids = np.zeros(rows, np.int32)
        flags = np.zeros(rows, np.uint8)
        self.lib.orc_argmax_rows(self._p(logits), rows, n_cols, ld, self._p(ids), self._p(flags))
        return ids, flags


_default: Oracle | None = None


def get() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default
