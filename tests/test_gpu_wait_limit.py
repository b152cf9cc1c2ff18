"""Failure detection without a fault: under the test hook (tf_wait_limit_test)
the warp-specialized and tensor-core kernels issue none of their loads, so
the bounded waits of their other warps run out (after 5 ms).  Each such
launch must report TF_DEV_TIMEOUT in its status word and leave the device
usable: the same call right after, hook off, gives the oracle's result.
No copy or MMA is in flight when a CTA gives up here, so nothing can land
after it has left."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_segment_b200 as tf
from paged_kv_cache_segment_b200 import binding
from paged_kv_cache_segment_b200 import workloads as wl

from _gpu import compare_attn, run_decode, run_prompt_chunks, run_ring
from test_gpu_tree import oracle_tree, run_tree

pytestmark = pytest.mark.gpu
TIMEOUT = binding.TF_DEV_TIMEOUT


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


def with_hook(fn):
    tf.tf_wait_limit_test(True)
    try:
        return fn()
    finally:
        tf.tf_wait_limit_test(False)


def oracle_paged(orc, b):
    return orc.paged_attn(b.q, b.k_pool, b.v_pool, b.page_table, b.segs, b.scale)


@pytest.mark.parametrize("kind", ["decode", "verify"])
def test_partials_wait_runs_out_then_recover(orc, kind):
    """Decode-shaped partials (the warp-specialized kernel, 4 queries a
    kv-head) and verify-shaped ones (the tensor-core kernel, up to 112)."""
    if kind == "decode":
        b = wl.make_paged_batch(31, [1, 1, 1], [700, 1500, 64], 32, 8, 128, 32, unused="nan", split_keys=256,
                                n_splits_max=6)
    else:
        b = wl.make_paged_batch(32, [5, 14], [900, 2100], 16, 2, 256, 32, unused="nan", split_keys=256,
                                n_splits_max=9)
    r = with_hook(lambda: run_decode(b))
    assert r["status"] & TIMEOUT
    r = run_decode(b)
    assert r["status"] == 0
    ref, rf = oracle_paged(orc, b)
    compare_attn(r["out"], r["flags"], ref, rf, what=f"{kind} after a run-out")


def test_ring_wait_runs_out_then_recovers(orc):
    b = wl.make_ring_batch(33, n_streams=3, ring_size=600, valid_lo=100, valid_hi=600, n_q_heads=16, n_kv_heads=2,
                           head_dim=256, split_slots=128)
    r = with_hook(lambda: run_ring(b))
    assert r["status"] & TIMEOUT
    r = run_ring(b)
    assert r["status"] == 0
    ref, rf = orc.ring_attn(b.q, b.ring_k, b.ring_v, b.rsegs, b.scale)
    compare_attn(r["out"], r["flags"], ref, rf, what="ring after a run-out")


def test_tree_wait_runs_out_then_recovers(orc):
    b = wl.make_tree_batch(34, n_streams=4, ring_size=900, valid_lo=100, valid_hi=700, nodes_lo=3, nodes_hi=12,
                           n_q_heads=16, n_kv_heads=2, head_dim=256, split_slots=256)
    r = with_hook(lambda: run_tree(b))
    assert r["status"] & TIMEOUT
    r = run_tree(b)
    assert r["status"] == 0
    ref, rf = oracle_tree(orc, b)
    compare_attn(r["out"], r["flags"], ref, rf, what="trees after a run-out")


def test_prompt_wait_runs_out_flags_every_row_then_recovers(orc):
    """A prompt chunk whose waits ran out writes every row as flagged NaN."""
    b, spans = wl.long_prompt(4, n_tokens=300, chunk=128)
    r = with_hook(lambda: run_prompt_chunks(b, spans, out_dtype=torch.float32))
    assert r["status"] & TIMEOUT
    assert (r["flags"] == 1).all() and np.isnan(r["out"]).all()
    r = run_prompt_chunks(b, spans, out_dtype=torch.float32)
    assert r["status"] == 0
    ref, rf = oracle_paged(orc, b)
    compare_attn(r["out"], r["flags"], ref, rf, what="prompt after a run-out")
