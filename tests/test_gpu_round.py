"""GPU parity of the one-call verify round (tf_verify_round): partials, merge
and row argmax, each a programmatic dependent of the launch before it."""
import numpy as np
import pytest
import torch

import paged_kv_cache_segment_b200 as tf
from paged_kv_cache_segment_b200 import binding
from paged_kv_cache_segment_b200 import workloads as wl
from _gpu import DEV, compare_attn, dev, run_argmax, run_decode, status_word

pytestmark = pytest.mark.gpu


def _round(b, logits, full=False, host=True):
    rows, hq, d = b.q.shape
    c = b.n_splits_max
    po = torch.full((rows, hq, c, d), float("nan"), device=DEV)
    pm = torch.full((rows, hq, c), float("nan"), device=DEV)
    pl = torch.full((rows, hq, c), float("nan"), device=DEV)
    pf = torch.full((rows, hq, c), 7, dtype=torch.uint8, device=DEV)
    out = torch.full((rows, hq, d), float("nan"), device=DEV)
    fl = torch.full((rows, hq), 9, dtype=torch.uint8, device=DEV)
    ids = torch.full((logits.shape[0],), -7, dtype=torch.int32, device=DEV)
    afl = torch.full((logits.shape[0],), 9, dtype=torch.uint8, device=DEV)
    st = status_word()
    tf.tf_verify_round(dev(b.q), dev(b.k_pool), dev(b.v_pool), dev(b.page_table),
                       dev(np.ascontiguousarray(b.segs, np.int32)), scale=b.scale, split_keys=b.split_keys,
                       n_splits_max=c, part_o=po, part_m=pm, part_l=pl, part_flag=pf, out=out, flags=fl, status=st,
                       logits=dev(logits), ids=ids, id_flags=afl, full=full, segs_host=b.segs if host else None,
                       page_table_host=b.page_table if host else None)
    torch.cuda.synchronize()
    return (out.cpu().numpy(), fl.cpu().numpy(), ids.cpu().numpy(), afl.cpu().numpy(), int(st.item()))


@pytest.mark.parametrize("full", [False, True])
def test_round_equals_the_three_calls(orc, full):
    """The shared-verify batch and its logits: the one-call round gives the
    same bits as the partial, merge and argmax calls made one by one, and both
    match the oracle."""
    b = wl.shared_verify(3)
    logits = wl.verify_logits(3, int(b.segs[:, 1].sum()), n_cols=32000)
    out, fl, ids, afl, st = _round(b, logits, full=full)
    assert st == 0
    r = run_decode(b, block=full)
    np.testing.assert_array_equal(out.view(np.uint32), r["out"].view(np.uint32))
    np.testing.assert_array_equal(fl, r["flags"])
    ids2, afl2 = run_argmax(logits)
    np.testing.assert_array_equal(ids, ids2)
    np.testing.assert_array_equal(afl, afl2)
    ref, rf = orc.paged_attn(b.q, b.k_pool, b.v_pool, b.page_table, b.segs, b.scale, full=full)
    compare_attn(out, fl, ref, rf, what="round")
    eids, eflags = orc.argmax_rows(logits)
    np.testing.assert_array_equal(ids, eids)
    np.testing.assert_array_equal(afl, eflags)


def test_round_without_logits_and_refusals():
    b = wl.shared_verify(3)
    logits = wl.verify_logits(3, 4, n_cols=1000)
    # a bad argmax argument is refused before anything launches
    with pytest.raises(binding.TfError):
        tf.tf_verify_round(dev(b.q), dev(b.k_pool), dev(b.v_pool), dev(b.page_table), dev(b.segs), scale=b.scale,
                           split_keys=b.split_keys, n_splits_max=b.n_splits_max,
                           part_o=torch.empty(1, device=DEV), part_m=torch.empty(1, device=DEV),
                           part_l=torch.empty(1, device=DEV), part_flag=torch.empty(1, dtype=torch.uint8, device=DEV),
                           out=torch.empty(1, device=DEV), flags=torch.empty(1, dtype=torch.uint8, device=DEV),
                           status=status_word(), logits=dev(logits), ids=torch.empty(4, dtype=torch.int32, device=DEV),
                           id_flags=torch.empty(4, dtype=torch.uint8, device=DEV), n_cols=2000)


def test_round_at_the_chosen_split(orc):
    """The split tf_choose_split_keys picks for the shared-verify batch on
    this device (1,280 keys on 148 SMs: 20 tiles, not a power of two); the
    round still matches the oracle and flags exactly the planted heads."""
    b0 = wl.shared_verify(3)
    split, n_sp = tf.tf_choose_split_keys(b0.segs, n_q_heads=16, n_kv_heads=2, head_dim=256)
    b = wl.shared_verify(3, split_keys=split)
    assert b.n_splits_max == n_sp
    logits = wl.verify_logits(3, int(b.segs[:, 1].sum()), n_cols=32000)
    out, fl, ids, afl, st = _round(b, logits)
    assert st == 0
    ref, rf = orc.paged_attn(b.q, b.k_pool, b.v_pool, b.page_table, b.segs, b.scale)
    compare_attn(out, fl, ref, rf, what=f"round at {split}-key splits")
    eids, eflags = orc.argmax_rows(logits)
    np.testing.assert_array_equal(ids, eids)
    np.testing.assert_array_equal(afl, eflags)
