"""Helpers for the GPU parity tests: move seeded inputs to the device, run the
CUDA path through the C ABI, and compare with the float64 oracle."""
from __future__ import annotations

import numpy as np
import torch

import paged_kv_cache_segment_b200 as tf
from paged_kv_cache_segment_b200 import binding
from paged_kv_cache_segment_b200 import workloads as wl

# the stated tolerance for fp32 attention outputs from bf16 inputs
MAX_ABS = 2e-3
REL_L2 = 1e-3

DEV = "cuda"


def dev(a: np.ndarray) -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(DEV)
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def status_word() -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def run_decode(b: wl.PagedBatch, *, split_keys=None, n_splits_max=None, host_tables=True, merge=True, segs=None,
               page_table=None, block=False):
    """Partials + merge for a paged batch (block: every row over all of its
    stream's keys).  Returns dict of numpy results."""
    split_keys = b.split_keys if split_keys is None else split_keys
    n_splits_max = b.n_splits_max if n_splits_max is None else n_splits_max
    segs = b.segs if segs is None else segs
    page_table = b.page_table if page_table is None else page_table
    rows, hq, d = b.q.shape
    q, kp, vp = dev(b.q), dev(b.k_pool), dev(b.v_pool)
    pt, sg = dev(page_table), dev(np.ascontiguousarray(segs, np.int32))
    po = torch.full((rows, hq, n_splits_max, d), float("nan"), device=DEV)
    pm = torch.full((rows, hq, n_splits_max), float("nan"), device=DEV)
    pl = torch.full((rows, hq, n_splits_max), float("nan"), device=DEV)
    pf = torch.full((rows, hq, n_splits_max), 7, dtype=torch.uint8, device=DEV)
    st = status_word()
    (tf.tf_paged_attn_block if block else tf.tf_paged_attn_decode)(q, kp, vp, pt, sg, scale=b.scale, split_keys=split_keys, n_splits_max=n_splits_max,
                            part_o=po, part_m=pm, part_l=pl, part_flag=pf, status=st,
                            segs_host=segs if host_tables else None,
                            page_table_host=page_table if host_tables else None)
    res = {"status": int(st.item())}
    if merge:
        out = torch.full((rows, hq, d), float("nan"), device=DEV)
        fl = torch.full((rows, hq), 9, dtype=torch.uint8, device=DEV)
        tf.tf_attn_merge(po, pm, pl, pf, out, fl)
        res["out"] = out.cpu().numpy()
        res["flags"] = fl.cpu().numpy()
    torch.cuda.synchronize()
    res.update(po=po.cpu().numpy(), pm=pm.cpu().numpy(), pl=pl.cpu().numpy(), pf=pf.cpu().numpy())
    return res


def run_ring(b: wl.RingBatch, *, split_slots=None, n_splits_max=None):
    split_slots = b.split_slots if split_slots is None else split_slots
    n_splits_max = b.n_splits_max if n_splits_max is None else n_splits_max
    rows, hq, d = b.q.shape
    n = len(b.rsegs)
    ws = torch.zeros(tf.tf_ring_workspace_bytes(n, hq, d, n_splits_max), dtype=torch.uint8, device=DEV)
    out = torch.full((rows, hq, d), float("nan"), device=DEV)
    fl = torch.full((rows, hq), 9, dtype=torch.uint8, device=DEV)
    st = status_word()
    tf.tf_ring_attn(dev(b.q), dev(b.ring_k), dev(b.ring_v), binding.rsegs_to_device(b.rsegs, DEV), scale=b.scale,
                    split_slots=split_slots, n_splits_max=n_splits_max, workspace=ws, out=out, flags=fl, status=st,
                    rsegs_host=b.rsegs)
    torch.cuda.synchronize()
    return {"out": out.cpu().numpy(), "flags": fl.cpu().numpy(), "status": int(st.item())}


def run_prompt_chunks(b: wl.PagedBatch, spans, out_dtype=torch.bfloat16):
    rows, hq, d = b.q.shape
    q, kp, vp, pt = dev(b.q), dev(b.k_pool), dev(b.v_pool), dev(b.page_table)
    out = torch.full((rows, hq, d), float("nan"), dtype=out_dtype, device=DEV)
    fl = torch.full((rows, hq), 9, dtype=torch.uint8, device=DEV)
    st = status_word()
    for r0, r1 in spans:
        seg = wl.prompt_chunk_seg(b, r0, r1)
        tf.tf_paged_attn_prompt(q, kp, vp, pt, seg, scale=b.scale, out=out, flags=fl, status=st)
    torch.cuda.synchronize()
    return {"out": out.float().cpu().numpy(), "flags": fl.cpu().numpy(), "status": int(st.item())}


def run_argmax(logits: np.ndarray, n_cols=None):
    rows = logits.shape[0]
    ids = torch.full((rows,), -7, dtype=torch.int32, device=DEV)
    fl = torch.full((rows,), 9, dtype=torch.uint8, device=DEV)
    tf.tf_argmax_rows(dev(logits), ids, fl, n_cols=n_cols)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), fl.cpu().numpy()


def compare_attn(gpu_out, gpu_flags, orc_out, orc_flags, sel=None, max_abs=MAX_ABS, rel_l2=REL_L2, what=""):
    """Flags bit-exact; a flagged head is NaN on both sides; the rest within
    max-abs and relative-L2 of the oracle.  sel (bool [rows][Hq]) limits the
    check to computed pairs."""
    gpu_flags = np.asarray(gpu_flags)
    orc_flags = np.asarray(orc_flags)
    if sel is None:
        sel = np.ones(orc_flags.shape, bool)
    np.testing.assert_array_equal(gpu_flags[sel], orc_flags[sel], err_msg=f"{what}: flags differ")
    fl = orc_flags.astype(bool) & sel
    ok = (~orc_flags.astype(bool)) & sel
    if fl.any():
        assert np.isnan(gpu_out[fl]).all(), f"{what}: flagged heads must hold NaN"
    if ok.any():
        g = gpu_out[ok].astype(np.float64)
        o = orc_out[ok]
        assert np.isfinite(g).all(), f"{what}: unflagged output not finite"
        err = np.abs(g - o)
        mae = float(err.max())
        rl2 = float(np.linalg.norm(g - o) / max(np.linalg.norm(o), 1e-30))
        assert mae <= max_abs, f"{what}: max-abs error {mae:.3e} > {max_abs}"
        assert rl2 <= rel_l2, f"{what}: rel-L2 error {rl2:.3e} > {rel_l2}"
        return mae, rl2
    return 0.0, 0.0


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    return np.exp2(np.floor(np.log2(ax)) - 7)


# bf16-output prompt tolerance, derived from the arithmetic: the softmax
# weights enter the P.V product as bf16 (relative error <= 2^-9 each), so the
# fp32 sum is off by at most 2^-9 * max_j |V_jd|; rounding the output to bf16
# adds at most 2^-9 * |out|.  A factor 2 covers fp32 accumulation.  The
# relative L2 bound (3e-3) is about twice the rms the two roundings give.
PROMPT_BF16_REL_L2 = 3e-3


def prompt_bf16_bound(b, ref):
    """Per-element bound [rows][Hq][D] for a one-stream prompt batch."""
    n = int(b.segs[0][2])
    p = b.page_size
    pages = b.page_table[b.segs[0][3]: b.segs[0][3] + -(-n // p)]
    v = wl.bf16_bits_to_f32(b.v_pool[pages]).astype(np.float64)  # [pages][Hkv][P][D]
    v = v.transpose(1, 0, 2, 3).reshape(b.n_kv_heads, -1, b.head_dim)[:, :n]  # [Hkv][n][D]
    vmax = np.nanmax(np.abs(v), axis=1)  # [Hkv][D]
    g = np.arange(b.n_q_heads) // (b.n_q_heads // b.n_kv_heads)
    return 2.0 ** -8 * (vmax[g][None, :, :] + np.abs(ref))


def check_prompt_bf16(gpu, gflags, ref, rflags, bound, sel=None, what="prompt bf16"):
    if sel is None:
        sel = np.ones(rflags.shape, bool)
    np.testing.assert_array_equal(gflags[sel], rflags[sel], err_msg=f"{what}: flags differ")
    ok = sel & ~rflags.astype(bool)
    if (sel & rflags.astype(bool)).any():
        assert np.isnan(gpu[sel & rflags.astype(bool)]).all()
    err = np.abs(gpu[ok].astype(np.float64) - ref[ok])
    assert (err <= bound[ok]).all(), f"{what}: beyond the derived bound by {np.max(err - bound[ok]):.3e}"
    rl2 = np.linalg.norm(gpu[ok] - ref[ok]) / np.linalg.norm(ref[ok])
    assert rl2 <= PROMPT_BF16_REL_L2, f"{what}: rel-L2 {rl2:.3e}"
