"""Thin ctypes binding of libtfpaged.so (include/tfpaged.h).

Each function has the C name and does argument marshalling only: it checks
that tensors live on a CUDA device with the documented dtype and layout,
passes their data pointers and the current CUDA stream, and raises
``TfError`` when the library returns a status other than TF_OK.  All
computation happens in the library's kernels.  There is no fallback: if the
shared library cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtfpaged.so")

TF_OK = 0
STATUS_NAMES = {0: "TF_OK", 1: "TF_ERR_ARG", 2: "TF_ERR_PAST_PAGES", 3: "TF_ERR_BAD_PAGE", 4: "TF_ERR_UNSUPPORTED",
                5: "TF_ERR_CUDA", 6: "TF_ERR_ALIGN", 7: "TF_ERR_WORKSPACE"}
TF_DEV_BAD_SEG, TF_DEV_PAST_PAGES, TF_DEV_BAD_PAGE, TF_DEV_SPLITS, TF_DEV_TIMEOUT = 1, 2, 4, 8, 16
TF_OUT_F32, TF_OUT_BF16 = 0, 1

EXPORTS = ("tf_paged_attn_decode", "tf_paged_attn_block", "tf_kv_append", "tf_verify_round", "tf_attn_merge",
           "tf_paged_attn_prompt", "tf_ring_attn", "tf_ring_workspace_bytes", "tf_ring_tree_attn",
           "tf_ring_tree_workspace_bytes", "tf_ring_attn_noalloc", "tf_argmax_rows", "tf_choose_split_keys",
           "tf_status_str", "tf_abi_version", "tf_wait_limit_test")
# bytes of the scratch array tf_ring_attn_noalloc keeps in the library's device image
TF_RING_NOALLOC_SCRATCH_BYTES = 8 << 20

SEG_DTYPE = np.dtype([("q_row", "<i4"), ("n_rows", "<i4"), ("n_keys", "<i4"), ("pt_base", "<i4"), ("n_pages", "<i4")])
RING_SEG_DTYPE = np.dtype(
    [("base", "<i8"), ("q_row", "<i4"), ("size", "<i4"), ("head", "<i4"), ("n_valid", "<i4")]
)
TREE_SEG_DTYPE = np.dtype(
    [("base", "<i8"), ("q_row", "<i4"), ("size", "<i4"), ("head", "<i4"), ("n_valid", "<i4"), ("n_nodes", "<i4"),
     ("parent_base", "<i4")]
)


class TfError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn}: {STATUS_NAMES.get(code, code)}")


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library once and declare the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m paged_kv_cache_segment_b200.build`")
    lib = ctypes.CDLL(path)
    P, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    lib.tf_paged_attn_decode.argtypes = [P, i32, i32, P, P, i32, i32, i32, i32, P, i32, P, i32, P, P, f32, i32, i32,
                                         P, P, P, P, P, P]
    lib.tf_paged_attn_block.argtypes = lib.tf_paged_attn_decode.argtypes
    lib.tf_kv_append.argtypes = [P, P, i32, P, P, i32, i32, i32, i32, P, i32, P, i32, P, P, P, P]
    lib.tf_verify_round.argtypes = [P, i32, i32, P, P, i32, i32, i32, i32, P, i32, P, i32, P, P, f32, i32, i32, i32,
                                    P, P, P, P, P, P, P, i32, i32, i64, P, P, P, P]
    lib.tf_attn_merge.argtypes = [P, P, P, P, i32, i32, i32, i32, P, P, P]
    lib.tf_paged_attn_prompt.argtypes = [P, i32, i32, P, P, i32, i32, i32, i32, P, i32, P, f32, P, i32, P, P, P]
    lib.tf_ring_attn.argtypes = [P, i32, i32, P, P, i64, i32, i32, P, i32, P, f32, i32, i32, P, sz, P, P, P, P]
    lib.tf_ring_attn_noalloc.argtypes = [P, i32, i32, P, P, i64, i32, i32, P, i32, P, f32, i32, i32, P, P, P, P]
    lib.tf_ring_tree_attn.argtypes = [P, i32, i32, P, P, i64, i32, i32, P, i32, P, P, i32, P, f32, i32, i32, P, sz,
                                      P, P, P, P]
    lib.tf_ring_tree_workspace_bytes.argtypes = [i32, i32, i32, i32]
    lib.tf_ring_tree_workspace_bytes.restype = sz
    lib.tf_ring_workspace_bytes.argtypes = [i32, i32, i32, i32]
    lib.tf_ring_workspace_bytes.restype = sz
    lib.tf_argmax_rows.argtypes = [P, i32, i32, i64, P, P, P]
    lib.tf_choose_split_keys.argtypes = [P, i32, i32, i32, i32, i32, P, P]
    lib.tf_status_str.argtypes = [ctypes.c_int]
    lib.tf_status_str.restype = ctypes.c_char_p
    lib.tf_abi_version.restype = ctypes.c_int32
    lib.tf_wait_limit_test.argtypes = [ctypes.c_int32]
    lib.tf_wait_limit_test.restype = ctypes.c_int
    for name in ("tf_paged_attn_decode", "tf_paged_attn_block", "tf_kv_append", "tf_verify_round", "tf_attn_merge", "tf_paged_attn_prompt", "tf_ring_attn",
                 "tf_ring_attn_noalloc", "tf_ring_tree_attn", "tf_argmax_rows", "tf_choose_split_keys"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


# ---------------------------------------------------------------- helpers

def _dev(t: torch.Tensor, name: str, dtypes, min_dim=None) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


BF16 = (torch.bfloat16, torch.int16, torch.uint16)


def _stream(stream) -> int:
    """The raw cudaStream_t: the given stream, or the current one."""
    if stream is None:
        return torch._C._cuda_getCurrentRawStream(torch.cuda.current_device())
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _check(fn: str, rc: int):
    if rc != TF_OK:
        raise TfError(fn, rc)


def _host_ptr(a):
    if a is None:
        return None
    return a.ctypes.data


def as_segs_np(segs) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(segs, dtype=np.int32).reshape(-1, 5))
    return a


def as_rsegs_np(rsegs) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(rsegs).astype(RING_SEG_DTYPE))


def as_tsegs_np(tsegs) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(tsegs).astype(TREE_SEG_DTYPE))


def tsegs_to_device(tsegs, device) -> torch.Tensor:
    """A tree table as a device byte tensor (32 bytes an entry)."""
    return torch.from_numpy(as_tsegs_np(tsegs).view(np.uint8).copy()).to(device)


def rsegs_to_device(rsegs, device) -> torch.Tensor:
    """A ring table as a device byte tensor (24 bytes an entry)."""
    a = as_rsegs_np(rsegs)
    return torch.from_numpy(a.view(np.uint8).copy()).to(device)


# ---------------------------------------------------------------- the calls

def tf_paged_attn_decode(q, k_pool, v_pool, page_table, segs, *, scale, split_keys, n_splits_max, part_o, part_m,
                         part_l, part_flag, status, segs_host=None, page_table_host=None, stream=None):
    """Split-KV partials of paged attention (tf_paged_attn_decode)."""
    lib = load()
    rows, hq, d = q.shape
    n_pages, hkv, psz, d2 = k_pool.shape
    if d2 != d or tuple(v_pool.shape) != tuple(k_pool.shape):
        raise ValueError("q / pool head dims disagree")
    sh = as_segs_np(segs_host) if segs_host is not None else None
    pth = np.ascontiguousarray(np.asarray(page_table_host, np.int32)) if page_table_host is not None else None
    rc = lib.tf_paged_attn_decode(
        _dev(q, "q", BF16), rows, hq, _dev(k_pool, "k_pool", BF16), _dev(v_pool, "v_pool", BF16), n_pages, psz, hkv, d,
        _dev(page_table, "page_table", (torch.int32,)), page_table.numel(), _dev(segs, "segs", (torch.int32,)),
        segs.numel() // 5, _host_ptr(sh), _host_ptr(pth), float(scale), int(split_keys), int(n_splits_max),
        _dev(part_o, "part_o", (torch.float32,)), _dev(part_m, "part_m", (torch.float32,)),
        _dev(part_l, "part_l", (torch.float32,)), _dev(part_flag, "part_flag", (torch.uint8,)),
        _dev(status, "status", (torch.int32, torch.uint32)), _stream(stream))
    _check("tf_paged_attn_decode", rc)


def tf_paged_attn_block(q, k_pool, v_pool, page_table, segs, *, scale, split_keys, n_splits_max, part_o, part_m,
                        part_l, part_flag, status, segs_host=None, page_table_host=None, stream=None):
    """Split-KV partials where every row sees all of its stream's keys (tf_paged_attn_block)."""
    lib = load()
    rows, hq, d = q.shape
    n_pages, hkv, psz, d2 = k_pool.shape
    if d2 != d or tuple(v_pool.shape) != tuple(k_pool.shape):
        raise ValueError("q / pool head dims disagree")
    sh = as_segs_np(segs_host) if segs_host is not None else None
    pth = np.ascontiguousarray(np.asarray(page_table_host, np.int32)) if page_table_host is not None else None
    rc = lib.tf_paged_attn_block(
        _dev(q, "q", BF16), rows, hq, _dev(k_pool, "k_pool", BF16), _dev(v_pool, "v_pool", BF16), n_pages, psz, hkv, d,
        _dev(page_table, "page_table", (torch.int32,)), page_table.numel(), _dev(segs, "segs", (torch.int32,)),
        segs.numel() // 5, _host_ptr(sh), _host_ptr(pth), float(scale), int(split_keys), int(n_splits_max),
        _dev(part_o, "part_o", (torch.float32,)), _dev(part_m, "part_m", (torch.float32,)),
        _dev(part_l, "part_l", (torch.float32,)), _dev(part_flag, "part_flag", (torch.uint8,)),
        _dev(status, "status", (torch.int32, torch.uint32)), _stream(stream))
    _check("tf_paged_attn_block", rc)


def tf_kv_append(k_rows, v_rows, k_pool, v_pool, page_table, segs, *, status, segs_host=None, page_table_host=None,
                 stream=None):
    """Each stream's new rows [rows][Hkv][D] into their pages (tf_kv_append)."""
    lib = load()
    rows, hkv, d = k_rows.shape
    n_pages, hkv2, psz, d2 = k_pool.shape
    if (hkv2, d2) != (hkv, d) or tuple(v_pool.shape) != tuple(k_pool.shape) or tuple(v_rows.shape) != tuple(k_rows.shape):
        raise ValueError("rows / pool shapes disagree")
    sh = as_segs_np(segs_host) if segs_host is not None else None
    pth = np.ascontiguousarray(np.asarray(page_table_host, np.int32)) if page_table_host is not None else None
    rc = lib.tf_kv_append(
        _dev(k_rows, "k_rows", BF16), _dev(v_rows, "v_rows", BF16), rows, _dev(k_pool, "k_pool", BF16),
        _dev(v_pool, "v_pool", BF16), n_pages, psz, hkv, d, _dev(page_table, "page_table", (torch.int32,)),
        page_table.numel(), _dev(segs, "segs", (torch.int32,)), segs.numel() // 5, _host_ptr(sh), _host_ptr(pth),
        _dev(status, "status", (torch.int32, torch.uint32)), _stream(stream))
    _check("tf_kv_append", rc)


def tf_verify_round(q, k_pool, v_pool, page_table, segs, *, scale, split_keys, n_splits_max, part_o, part_m, part_l,
                    part_flag, out, flags, status, logits=None, ids=None, id_flags=None, n_cols=None, full=False,
                    segs_host=None, page_table_host=None, stream=None):
    """Partials, merge and (when logits are given) the row argmax of one round in one call (tf_verify_round)."""
    lib = load()
    rows, hq, d = q.shape
    n_pages, hkv, psz, d2 = k_pool.shape
    if d2 != d or tuple(v_pool.shape) != tuple(k_pool.shape):
        raise ValueError("q / pool head dims disagree")
    sh = as_segs_np(segs_host) if segs_host is not None else None
    pth = np.ascontiguousarray(np.asarray(page_table_host, np.int32)) if page_table_host is not None else None
    if logits is not None:
        if logits.dim() != 2 or logits.stride(1) != 1:
            raise ValueError("logits must be 2-D with unit column stride")
        n_lr, ld = logits.shape[0], logits.stride(0)
        nc = logits.shape[1] if n_cols is None else int(n_cols)
        lp, ip, fp = _dev(logits, "logits", BF16), _dev(ids, "ids", (torch.int32,)), _dev(id_flags, "id_flags",
                                                                                         (torch.uint8,))
    else:
        n_lr, ld, nc, lp, ip, fp = 0, 0, 0, None, None, None
    rc = lib.tf_verify_round(
        _dev(q, "q", BF16), rows, hq, _dev(k_pool, "k_pool", BF16), _dev(v_pool, "v_pool", BF16), n_pages, psz, hkv, d,
        _dev(page_table, "page_table", (torch.int32,)), page_table.numel(), _dev(segs, "segs", (torch.int32,)),
        segs.numel() // 5, _host_ptr(sh), _host_ptr(pth), float(scale), int(split_keys), int(n_splits_max),
        int(bool(full)), _dev(part_o, "part_o", (torch.float32,)), _dev(part_m, "part_m", (torch.float32,)),
        _dev(part_l, "part_l", (torch.float32,)), _dev(part_flag, "part_flag", (torch.uint8,)),
        _dev(out, "out", (torch.float32,)), _dev(flags, "flags", (torch.uint8,)), lp, n_lr, nc, ld, ip, fp,
        _dev(status, "status", (torch.int32, torch.uint32)), _stream(stream))
    _check("tf_verify_round", rc)


def tf_attn_merge(part_o, part_m, part_l, part_flag, out, flags, *, stream=None):
    """Fold partials [rows][Hq][C](*D) into out [rows][Hq][D] and flags (tf_attn_merge)."""
    lib = load()
    rows, hq, c, d = part_o.shape
    rc = lib.tf_attn_merge(_dev(part_o, "part_o", (torch.float32,)), _dev(part_m, "part_m", (torch.float32,)),
                           _dev(part_l, "part_l", (torch.float32,)), _dev(part_flag, "part_flag", (torch.uint8,)),
                           rows, hq, d, c, _dev(out, "out", (torch.float32,)), _dev(flags, "flags", (torch.uint8,)),
                           _stream(stream))
    _check("tf_attn_merge", rc)


def tf_paged_attn_prompt(q, k_pool, v_pool, page_table, seg_host, *, scale, out, flags=None, status, stream=None):
    """Causal prompt chunk through one stream's page-table row (tf_paged_attn_prompt).
    out dtype picks the output type: torch.bfloat16 or torch.float32."""
    lib = load()
    rows, hq, d = q.shape
    n_pages, hkv, psz, _ = k_pool.shape
    sh = as_segs_np(seg_host)
    if len(sh) != 1:
        raise ValueError("the prompt call takes one segment")
    out_dtype = TF_OUT_BF16 if out.dtype == torch.bfloat16 else TF_OUT_F32
    rc = lib.tf_paged_attn_prompt(
        _dev(q, "q", BF16), rows, hq, _dev(k_pool, "k_pool", BF16), _dev(v_pool, "v_pool", BF16), n_pages, psz, hkv, d,
        _dev(page_table, "page_table", (torch.int32,)), page_table.numel(), _host_ptr(sh), float(scale),
        _dev(out, "out", (torch.bfloat16, torch.float32)), out_dtype,
        None if flags is None else _dev(flags, "flags", (torch.uint8,)),
        _dev(status, "status", (torch.int32, torch.uint32)), _stream(stream))
    _check("tf_paged_attn_prompt", rc)


def tf_choose_split_keys(segs_host, *, n_q_heads: int, n_kv_heads: int, head_dim: int,
                         n_sms: int | None = None) -> tuple[int, int]:
    """(split_keys, n_splits_max) for a head-dim-256 batch the tcgen05
    partial kernel serves (tf_choose_split_keys).  n_sms defaults to the
    current device's."""
    lib = load()
    sh = as_segs_np(segs_host)
    if n_sms is None:
        n_sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    split, n_sp = ctypes.c_int32(0), ctypes.c_int32(0)
    _check("tf_choose_split_keys", lib.tf_choose_split_keys(_host_ptr(sh), len(sh), n_q_heads, n_kv_heads, head_dim, n_sms,
                                                            ctypes.byref(split), ctypes.byref(n_sp)))
    return int(split.value), int(n_sp.value)


def tf_ring_workspace_bytes(n_segs: int, n_q_heads: int, head_dim: int, n_splits_max: int) -> int:
    return int(load().tf_ring_workspace_bytes(n_segs, n_q_heads, head_dim, n_splits_max))


def tf_ring_attn(q, ring_k, ring_v, rsegs, *, scale, split_slots, n_splits_max, workspace, out, flags, status,
                 rsegs_host=None, stream=None):
    """Ring-of-slots attention for many rows in one launch (tf_ring_attn).
    rsegs is a device uint8 tensor holding the table (see rsegs_to_device)."""
    lib = load()
    rows, hq, d = q.shape
    slots, hkv, d2 = ring_k.shape
    n_segs = rsegs.numel() // RING_SEG_DTYPE.itemsize
    rh = as_rsegs_np(rsegs_host) if rsegs_host is not None else None
    rc = lib.tf_ring_attn(_dev(q, "q", BF16), rows, hq, _dev(ring_k, "ring_k", BF16), _dev(ring_v, "ring_v", BF16),
                          slots, hkv, d, _dev(rsegs, "rsegs", (torch.uint8, torch.int8)), n_segs, _host_ptr(rh),
                          float(scale), int(split_slots), int(n_splits_max),
                          _dev(workspace, "workspace", (torch.uint8,)), workspace.numel(),
                          _dev(out, "out", (torch.float32,)), _dev(flags, "flags", (torch.uint8,)),
                          _dev(status, "status", (torch.int32, torch.uint32)), _stream(stream))
    _check("tf_ring_attn", rc)


def tf_ring_tree_workspace_bytes(n_rows_total: int, n_q_heads: int, head_dim: int, n_splits_max: int) -> int:
    return int(load().tf_ring_tree_workspace_bytes(n_rows_total, n_q_heads, head_dim, n_splits_max))


def tf_ring_tree_attn(q, ring_k, ring_v, tsegs, parents, *, scale, split_slots, n_splits_max, workspace, out, flags,
                      status, tsegs_host=None, parents_host=None, stream=None):
    """Draft trees over rings, every tree in one launch (tf_ring_tree_attn).
    tsegs is a device uint8 tensor holding the table (see tsegs_to_device),
    parents a device int32 tensor."""
    lib = load()
    rows, hq, d = q.shape
    slots, hkv, d2 = ring_k.shape
    if d2 != d or tuple(ring_v.shape) != tuple(ring_k.shape):
        raise ValueError("q / ring head dims disagree")
    n_segs = tsegs.numel() // TREE_SEG_DTYPE.itemsize
    th = as_tsegs_np(tsegs_host) if tsegs_host is not None else None
    ph = np.ascontiguousarray(np.asarray(parents_host, np.int32)) if parents_host is not None else None
    rc = lib.tf_ring_tree_attn(_dev(q, "q", BF16), rows, hq, _dev(ring_k, "ring_k", BF16),
                               _dev(ring_v, "ring_v", BF16), slots, hkv, d,
                               _dev(tsegs, "tsegs", (torch.uint8, torch.int8)), n_segs, _host_ptr(th),
                               _dev(parents, "parents", (torch.int32,)), parents.numel(), _host_ptr(ph),
                               float(scale), int(split_slots), int(n_splits_max),
                               _dev(workspace, "workspace", (torch.uint8,)), workspace.numel(),
                               _dev(out, "out", (torch.float32,)), _dev(flags, "flags", (torch.uint8,)),
                               _dev(status, "status", (torch.int32, torch.uint32)), _stream(stream))
    _check("tf_ring_tree_attn", rc)


def tf_ring_attn_noalloc(q, ring_k, ring_v, rsegs, *, scale, split_slots, n_splits_max, out, flags, status,
                         rsegs_host=None, stream=None):
    """tf_ring_attn without a workspace, for callers that cannot allocate
    device memory: the partials go to a scratch array built into the
    library (TF_RING_NOALLOC_SCRATCH_BYTES bytes a GPU, held until exit).
    All calls on a device share it, so calls must not overlap on the GPU;
    the first call on a device should come before any stream capture."""
    lib = load()
    rows, hq, d = q.shape
    slots, hkv, d2 = ring_k.shape
    n_segs = rsegs.numel() // RING_SEG_DTYPE.itemsize
    rh = as_rsegs_np(rsegs_host) if rsegs_host is not None else None
    rc = lib.tf_ring_attn_noalloc(_dev(q, "q", BF16), rows, hq, _dev(ring_k, "ring_k", BF16),
                                  _dev(ring_v, "ring_v", BF16), slots, hkv, d,
                                  _dev(rsegs, "rsegs", (torch.uint8, torch.int8)), n_segs, _host_ptr(rh),
                                  float(scale), int(split_slots), int(n_splits_max),
                                  _dev(out, "out", (torch.float32,)), _dev(flags, "flags", (torch.uint8,)),
                                  _dev(status, "status", (torch.int32, torch.uint32)), _stream(stream))
    _check("tf_ring_attn_noalloc", rc)


def tf_argmax_rows(logits, ids, flags, *, n_cols=None, stream=None):
    """Greedy row argmax of bf16 logits [rows][ld] over the first n_cols columns."""
    lib = load()
    rows, ld = logits.shape
    n_cols = ld if n_cols is None else int(n_cols)
    rc = lib.tf_argmax_rows(_dev(logits, "logits", BF16), rows, n_cols, ld, _dev(ids, "ids", (torch.int32,)),
                            _dev(flags, "flags", (torch.uint8,)), _stream(stream))
    _check("tf_argmax_rows", rc)


def tf_status_str(code: int) -> str:
    return load().tf_status_str(int(code)).decode()


def tf_abi_version() -> int:
    return int(load().tf_abi_version())


def tf_wait_limit_test(on: bool) -> None:
    """Test hook: while on, kernels launched from this host thread issue no
    loads and their bounded waits run out after 5 ms (TF_DEV_TIMEOUT)."""
    _check("tf_wait_limit_test", load().tf_wait_limit_test(1 if on else 0))
