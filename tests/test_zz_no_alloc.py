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


def test_no_alloc_at_the_top_of_its_scratch():
    """Sizes whose partials fill the scratch to its last byte (487 rows x 5
    heads x 13 partials of head dim 64 need exactly 8 MiB) match the
    workspace call; one row more is refused."""
    limit = binding.TF_RING_NOALLOC_SCRATCH_BYTES
    n, hq, d, c = 487, 5, 64, 13
    assert tf.tf_ring_workspace_bytes(n, hq, d, c) == limit
    assert tf.tf_ring_workspace_bytes(n + 1, hq, d, c) > limit
    valids = [int(v) for v in np.random.default_rng(8).integers(1, 209, size=n)]
    valids[n // 2] = 208  # 13 partials of 16 slots
    b = wl.make_ring_batch(8, n_streams=n, ring_size=208, valid_lo=1, valid_hi=208, n_q_heads=hq, n_kv_heads=1,
                           head_dim=d, split_slots=16, valids=valids)
    assert b.n_splits_max == c
    check_same(*run_both(b))
    b2 = wl.make_ring_batch(9, n_streams=n + 1, ring_size=208, valid_lo=1, valid_hi=208, n_q_heads=hq, n_kv_heads=1,
                            head_dim=d, split_slots=16, valids=valids + [208])
    out = torch.empty((n + 1, hq, d), device="cuda")
    fl = torch.empty((n + 1, hq), dtype=torch.uint8, device="cuda")
    with pytest.raises(tf.TfError, match="WORKSPACE"):
        tf.tf_ring_attn_noalloc(dev(b2.q), dev(b2.ring_k), dev(b2.ring_v), binding.rsegs_to_device(b2.rsegs, "cuda"),
                                scale=b2.scale, split_slots=16, n_splits_max=c, out=out, flags=fl,
                                status=status_word(), rsegs_host=b2.rsegs)


def test_no_alloc_gives_the_workspace_calls_verdict_on_bad_arguments():
    """Arguments that are both wrong and too large for the scratch get the
    verdict tf_ring_attn gives them, not TF_ERR_WORKSPACE."""
    import ctypes

    lib = tf.load()
    big = 488  # with 5 heads, head dim 64 and 13 partials: past the scratch
    q = torch.zeros((big, 5, 64), dtype=torch.bfloat16, device="cuda")
    ring = torch.zeros((208, 1, 64), dtype=torch.bfloat16, device="cuda")
    rs = torch.zeros(big * 24, dtype=torch.uint8, device="cuda")
    out = torch.empty((big, 5, 64), device="cuda")
    fl = torch.empty((big, 5), dtype=torch.uint8, device="cuda")
    st = status_word()
    ws = torch.empty(tf.tf_ring_workspace_bytes(big, 5, 64, 13), dtype=torch.uint8, device="cuda")

    def both(split_slots, n_kv_heads, qp, rsp):
        a = lib.tf_ring_attn(qp, big, 5, ring.data_ptr(), ring.data_ptr(), 208, n_kv_heads, 64, rsp, big, None,
                             ctypes.c_float(0.125), split_slots, 13, ws.data_ptr(), ws.numel(), out.data_ptr(),
                             fl.data_ptr(), st.data_ptr(), None)
        b = lib.tf_ring_attn_noalloc(qp, big, 5, ring.data_ptr(), ring.data_ptr(), 208, n_kv_heads, 64, rsp, big,
                                     None, ctypes.c_float(0.125), split_slots, 13, out.data_ptr(), fl.data_ptr(),
                                     st.data_ptr(), None)
        return a, b

    assert both(8, 1, q.data_ptr(), rs.data_ptr()) == (4, 4)  # split_slots < 16: TF_ERR_UNSUPPORTED
    assert both(16, 2, q.data_ptr(), rs.data_ptr()) == (4, 4)  # 5 q-heads over 2 kv-heads
    assert both(16, 1, None, rs.data_ptr()) == (1, 1)  # no q: TF_ERR_ARG
    assert both(16, 1, q.data_ptr() + 2, rs.data_ptr()) == (6, 6)  # q misaligned: TF_ERR_ALIGN
    torch.cuda.synchronize()
    assert int(st.item()) == 0


_LAZY_CHILD = r"""
import sys
sys.path[:0] = [{root!r}, {tests!r}]
import numpy as np
import torch
import paged_kv_cache_segment_b200 as tf
from paged_kv_cache_segment_b200 import binding
from paged_kv_cache_segment_b200 import workloads as wl
from test_zz_no_alloc import check_same
from _gpu import dev, status_word

torch.cuda.init()
torch.zeros(1, device="cuda")
b = wl.make_ring_batch(10, n_streams=6, ring_size=700, valid_lo=20, valid_hi=700, n_q_heads=16, n_kv_heads=2,
                       head_dim=256, split_slots=128)
rows, hq, d = b.q.shape
q, rk, rv = dev(b.q), dev(b.ring_k), dev(b.ring_v)
rs = binding.rsegs_to_device(b.rsegs, "cuda")
out_a = torch.full((rows, hq, d), float("nan"), device="cuda")
fl_a = torch.full((rows, hq), 9, dtype=torch.uint8, device="cuda")
out_b = torch.full((rows, hq, d), float("nan"), device="cuda")
fl_b = torch.full((rows, hq), 9, dtype=torch.uint8, device="cuda")
st = status_word()
ws = torch.empty(tf.tf_ring_workspace_bytes(len(b.rsegs), hq, d, b.n_splits_max), dtype=torch.uint8, device="cuda")
# the workspace call first: it loads the ring kernels' device code
tf.tf_ring_attn(q, rk, rv, rs, scale=b.scale, split_slots=b.split_slots, n_splits_max=b.n_splits_max, workspace=ws,
                out=out_a, flags=fl_a, status=st, rsegs_host=b.rsegs)
torch.cuda.synchronize()
# a call with no rows places the scratch array
empty = torch.empty(0, dtype=torch.uint8, device="cuda")
free0 = torch.cuda.mem_get_info()[0]
tf.tf_ring_attn_noalloc(q, rk, rv, empty, scale=b.scale, split_slots=b.split_slots, n_splits_max=b.n_splits_max,
                        out=out_b, flags=fl_b, status=st)
torch.cuda.synchronize()
free1 = torch.cuda.mem_get_info()[0]
assert free0 - free1 >= binding.TF_RING_NOALLOC_SCRATCH_BYTES, (free0, free1)
# then the caller takes all but 512 MiB of the device for itself
hog = torch.empty(torch.cuda.mem_get_info()[0] - (512 << 20), dtype=torch.uint8, device="cuda")
for _ in range(2):
    tf.tf_ring_attn_noalloc(q, rk, rv, rs, scale=b.scale, split_slots=b.split_slots, n_splits_max=b.n_splits_max,
                            out=out_b, flags=fl_b, status=st, rsegs_host=b.rsegs)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    check_same(out_a.cpu().numpy(), fl_a.cpu().numpy(), out_b.cpu().numpy(), fl_b.cpu().numpy())
del hog
print("lazy ok")
"""


def test_no_alloc_first_call_places_the_scratch_under_lazy_loading():
    """In a fresh process with lazy module loading: a call with no rows
    places the scratch array (device memory drops by its size), after which
    the caller may take nearly all of the device's memory and the call still
    runs and matches the workspace call."""
    import os
    import subprocess
    import sys

    here = os.path.dirname(os.path.abspath(__file__))
    code = _LAZY_CHILD.format(root=os.path.dirname(here), tests=here)
    env = dict(os.environ, CUDA_MODULE_LOADING="LAZY")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "lazy ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
