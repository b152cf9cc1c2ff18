"""tf_ring_attn_noalloc against tf_ring_attn, through the C ABI.

tf_ring_attn_noalloc is for callers that cannot allocate device memory (an
engine that gave all of it to the KV pool, a plugin hook where cudaMalloc is
not allowed): it keeps the partials in a scratch array built into the
library instead of a caller's workspace.  Its results must match the
workspace call within the tolerance the parity tests use, on two calls in a
row with different inputs (the scratch keeps the first call's contents).

This file is named to be collected last, so a failure here stops a run that
stops at the first failure only after every other test has run.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_segment_b200 as tf
from paged_kv_cache_segment_b200 import binding
from paged_kv_cache_segment_b200 import workloads as wl

from _gpu import MAX_ABS, REL_L2, dev, status_word

pytestmark = pytest.mark.gpu


def run_both(b):
    rows, hq, d = b.q.shape
    q, rk, rv = dev(b.q), dev(b.ring_k), dev(b.ring_v)
    rs = binding.rsegs_to_device(b.rsegs, "cuda")
    ws = torch.empty(tf.tf_ring_workspace_bytes(len(b.rsegs), hq, d, b.n_splits_max), dtype=torch.uint8,
                     device="cuda")
    out_a = torch.full((rows, hq, d), float("nan"), device="cuda")
    fl_a = torch.full((rows, hq), 9, dtype=torch.uint8, device="cuda")
    out_b = torch.full((rows, hq, d), float("nan"), device="cuda")
    fl_b = torch.full((rows, hq), 9, dtype=torch.uint8, device="cuda")
    st_a, st_b = status_word(), status_word()
    tf.tf_ring_attn(q, rk, rv, rs, scale=b.scale, split_slots=b.split_slots, n_splits_max=b.n_splits_max,
                    workspace=ws, out=out_a, flags=fl_a, status=st_a, rsegs_host=b.rsegs)
    tf.tf_ring_attn_noalloc(q, rk, rv, rs, scale=b.scale, split_slots=b.split_slots, n_splits_max=b.n_splits_max,
                            out=out_b, flags=fl_b, status=st_b, rsegs_host=b.rsegs)
    torch.cuda.synchronize()
    assert int(st_a.item()) == 0 and int(st_b.item()) == 0
    return out_a.cpu().numpy(), fl_a.cpu().numpy(), out_b.cpu().numpy(), fl_b.cpu().numpy()


def check_same(out_a, fl_a, out_b, fl_b):
    np.testing.assert_array_equal(fl_a, fl_b)
    ok = ~fl_a.astype(bool)
    assert np.isnan(out_b[~ok]).all()
    a, b = out_a[ok].astype(np.float64), out_b[ok].astype(np.float64)
    assert np.isfinite(b).all()
    assert np.abs(a - b).max() <= MAX_ABS
    assert np.linalg.norm(a - b) / max(np.linalg.norm(a), 1e-30) <= REL_L2


def test_no_alloc_matches_workspace_call_twice():
    # first call: the 17-row drafter ring
    first = wl.drafter_ring(5)
    check_same(*run_both(first))
    # second call, right after, on other rings and sizes (fewer rows, other
    # heads, a planted NaN): the scratch still holds the first call's partials
    second = wl.make_ring_batch(6, n_streams=5, ring_size=900, valid_lo=10, valid_hi=900, n_q_heads=16, n_kv_heads=2,
                                head_dim=256, split_slots=128, unused="normal")
    e = second.rsegs[2]
    second.ring_v[int(e["base"]) + (int(e["head"]) - 1) % int(e["size"]), 0, 5] = wl.BF16_NAN
    out_a, fl_a, out_b, fl_b = run_both(second)
    assert fl_a[2, :8].all()
    check_same(out_a, fl_a, out_b, fl_b)


def test_no_alloc_refuses_sizes_past_its_scratch():
    limit = binding.TF_RING_NOALLOC_SCRATCH_BYTES
    n = 400  # 400 rows x 16 heads x 17 partials x 258 floats is far past the built-in scratch
    assert tf.tf_ring_workspace_bytes(n, 16, 256, 17) > limit
    b = wl.make_ring_batch(7, n_streams=n, ring_size=64, valid_lo=1, valid_hi=64, n_q_heads=16, n_kv_heads=2,
                           head_dim=256, split_slots=16)
    out = torch.empty((n, 16, 256), device="cuda")
    fl = torch.empty((n, 16), dtype=torch.uint8, device="cuda")
    with pytest.raises(tf.TfError, match="WORKSPACE"):
        tf.tf_ring_attn_noalloc(dev(b.q), dev(b.ring_k), dev(b.ring_v), binding.rsegs_to_device(b.rsegs, "cuda"),
                                scale=b.scale, split_slots=16, n_splits_max=17, out=out, flags=fl,
                                status=status_word(), rsegs_host=b.rsegs)
