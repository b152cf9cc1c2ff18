"""Draft trees over rings (tf_ring_tree_attn) against the float64 oracle,
through the C ABI: fp32 outputs within max-abs 2e-3 and relative L2 1e-3,
flags bit-exact, and a chain equal to the ring call over the slots it
extends."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_segment_b200 as tf
from paged_kv_cache_segment_b200 import binding
from paged_kv_cache_segment_b200 import workloads as wl

from _gpu import DEV, compare_attn, dev, status_word

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


def run_tree(b, *, split_slots=None, n_splits_max=None, host_tables=True, tsegs=None, parents=None):
    split_slots = b.split_slots if split_slots is None else split_slots
    n_splits_max = b.n_splits_max if n_splits_max is None else n_splits_max
    tsegs = b.tsegs if tsegs is None else tsegs
    parents = b.parents if parents is None else parents
    rows, hq, d = b.q.shape
    ws = torch.zeros(tf.tf_ring_tree_workspace_bytes(rows, hq, d, n_splits_max), dtype=torch.uint8, device=DEV)
    out = torch.full((rows, hq, d), float("nan"), device=DEV)
    fl = torch.full((rows, hq), 9, dtype=torch.uint8, device=DEV)
    st = status_word()
    tf.tf_ring_tree_attn(dev(b.q), dev(b.ring_k), dev(b.ring_v), binding.tsegs_to_device(tsegs, DEV),
                         dev(np.asarray(parents, np.int32)), scale=b.scale, split_slots=split_slots,
                         n_splits_max=n_splits_max, workspace=ws, out=out, flags=fl, status=st,
                         tsegs_host=tsegs if host_tables else None, parents_host=parents if host_tables else None)
    torch.cuda.synchronize()
    return {"out": out.cpu().numpy(), "flags": fl.cpu().numpy(), "status": int(st.item())}


def oracle_tree(orc, b, tsegs=None, parents=None):
    return orc.ring_tree_attn(b.q, b.ring_k, b.ring_v, b.tsegs if tsegs is None else tsegs,
                              b.parents if parents is None else parents, b.scale)


def test_drafter_trees_full(orc):
    """The 17-tree drafter workload: 4,200-slot rings, windows of 1,000-4,184
    slots, chain / star / binary / random trees of 4-16 nodes, slots outside
    every window and tree NaN."""
    b = wl.drafter_trees(6)
    r = run_tree(b)
    assert r["status"] == 0
    ref, rf = oracle_tree(orc, b)
    assert not rf.any()
    compare_attn(r["out"], r["flags"], ref, rf, what="drafter trees")


@pytest.mark.parametrize("hq,hkv,d,nodes,split", [(16, 2, 256, (4, 16), 128), (8, 8, 64, (1, 9), 64),
                                                  (8, 2, 128, (10, 64), 256), (32, 2, 128, (1, 8), 192),
                                                  (4, 1, 64, (30, 64), 64), (16, 1, 256, (2, 20), 512)])
def test_tree_shapes(orc, hq, hkv, d, nodes, split):
    """Head dims, groups of 1 to 16 (trees of up to 64 nodes take several
    128-query tiles), windows and trees that wrap, split sizes."""
    b = wl.make_tree_batch(hq * 100 + d + split, n_streams=9, ring_size=600, valid_lo=0, valid_hi=520,
                           nodes_lo=nodes[0], nodes_hi=nodes[1], n_q_heads=hq, n_kv_heads=hkv, head_dim=d,
                           split_slots=split)
    r = run_tree(b)
    assert r["status"] == 0
    ref, rf = oracle_tree(orc, b)
    compare_attn(r["out"], r["flags"], ref, rf, what=f"trees {hq}/{hkv} D{d}")


def test_tree_without_host_tables(orc):
    b = wl.make_tree_batch(41, n_streams=5, ring_size=300, valid_lo=10, valid_hi=250, nodes_lo=3, nodes_hi=12,
                           n_q_heads=16, n_kv_heads=2, head_dim=256, split_slots=64)
    r = run_tree(b, host_tables=False)
    assert r["status"] == 0
    ref, rf = oracle_tree(orc, b)
    compare_attn(r["out"], r["flags"], ref, rf, what="trees, device tables only")


def test_chain_equals_ring_rows():
    """A tree that is one chain, node by node, against tf_ring_attn over the
    ring whose window runs on through the chain's slots up to that node."""
    t = 12
    b = wl.make_tree_batch(5, n_streams=3, ring_size=900, valid_lo=100, valid_hi=880, nodes_lo=t, nodes_hi=t,
                           n_q_heads=16, n_kv_heads=2, head_dim=256, kinds=["chain"] * 3, split_slots=256)
    r = run_tree(b)
    assert r["status"] == 0
    rs = np.zeros(3 * t, wl.RING_SEG_DTYPE)
    for s, e in enumerate(b.tsegs):
        for i in range(t):
            rs[s * t + i] = (e["base"], e["q_row"] + i, e["size"], (e["head"] + i + 1) % e["size"],
                             e["n_valid"] + i + 1)
    rows, hq, d = b.q.shape
    n_sp = max(-(-int(x) // 256) for x in rs["n_valid"])
    ws = torch.zeros(tf.tf_ring_workspace_bytes(len(rs), hq, d, n_sp), dtype=torch.uint8, device=DEV)
    out = torch.full((rows, hq, d), float("nan"), device=DEV)
    fl = torch.full((rows, hq), 9, dtype=torch.uint8, device=DEV)
    st = status_word()
    tf.tf_ring_attn(dev(b.q), dev(b.ring_k), dev(b.ring_v), binding.rsegs_to_device(rs, DEV), scale=b.scale,
                    split_slots=256, n_splits_max=n_sp, workspace=ws, out=out, flags=fl, status=st, rsegs_host=rs)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    np.testing.assert_array_equal(r["flags"], fl.cpu().numpy())
    a, o = r["out"].astype(np.float64), out.cpu().numpy().astype(np.float64)
    assert np.abs(a - o).max() <= 2e-3
    assert np.linalg.norm(a - o) / np.linalg.norm(o) <= 1e-3


def test_tree_flags_follow_the_paths(orc):
    """A NaN in one node's value flags that node and its subtree only; an
    infinity in q flags one (row, head); an infinity in a window key flags
    every node of the tree on that kv-head."""
    b = wl.make_tree_batch(17, n_streams=4, ring_size=400, valid_lo=50, valid_hi=300, nodes_lo=8, nodes_hi=14,
                           n_q_heads=16, n_kv_heads=2, head_dim=256, split_slots=128,
                           kinds=["binary", "random", "chain", "star"])
    e0, e1 = b.tsegs[0], b.tsegs[1]
    b.ring_v[e0["base"] + (e0["head"] + 2) % e0["size"], 1, 77] = wl.BF16_NAN
    b.q[e1["q_row"] + 3, 5, 0] = wl.BF16_POS_INF
    e3 = b.tsegs[3]
    b.ring_k[e3["base"] + (e3["head"] - 1) % e3["size"], 0, 9] = wl.BF16_NEG_INF
    r = run_tree(b)
    ref, rf = oracle_tree(orc, b)
    assert rf.sum() > 10 and not rf.all()
    compare_attn(r["out"], r["flags"], ref, rf, what="tree flags")


def test_device_refuses_bad_parents(orc):
    """Without host tables, a parent at or past its node is found on the
    device: TF_DEV_BAD_SEG, that tree's bad rows flagged NaN, the other
    trees exact."""
    b = wl.make_tree_batch(23, n_streams=3, ring_size=300, valid_lo=20, valid_hi=200, nodes_lo=6, nodes_hi=6,
                           n_q_heads=8, n_kv_heads=2, head_dim=128, split_slots=64, kinds=["chain"] * 3)
    par = b.parents.copy()
    par[b.tsegs[1]["parent_base"] + 4] = 4  # node 4 of tree 1 names itself
    r = run_tree(b, host_tables=False, parents=par)
    assert r["status"] & binding.TF_DEV_BAD_SEG
    rows1 = slice(int(b.tsegs[1]["q_row"]), int(b.tsegs[1]["q_row"]) + 6)
    assert r["flags"][rows1][4].all() and np.isnan(r["out"][rows1][4]).all()
    ref, rf = oracle_tree(orc, b)  # the oracle on the good parents
    keep = np.ones(rf.shape, bool)
    keep[rows1] = False
    compare_attn(r["out"], r["flags"], ref, rf, sel=keep, what="trees beside a bad one")


def test_host_table_refusals():
    b = wl.make_tree_batch(3, n_streams=2, ring_size=200, valid_lo=20, valid_hi=150, nodes_lo=4, nodes_hi=4,
                           n_q_heads=8, n_kv_heads=2, head_dim=64, split_slots=64)
    par = b.parents.copy()
    par[1] = 1
    with pytest.raises(tf.TfError, match="ARG"):
        run_tree(b, parents=par)
    with pytest.raises(tf.TfError, match="ARG"):
        run_tree(b, n_splits_max=1)
