"""GPU parity of the FULL block attention (tf_paged_attn_block) and of the KV
append (tf_kv_append) against the float64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import paged_kv_cache_segment_b200 as tf
from paged_kv_cache_segment_b200 import binding
from paged_kv_cache_segment_b200 import workloads as wl
from _gpu import compare_attn, dev, run_decode, status_word

pytestmark = pytest.mark.gpu


# (rows, keys, hq, hkv, d, p, split): the first two take the warp-specialized
# kernel (at most 8 queries a kv-head), the next two the tcgen05 partials, the
# last the general kernel (a split that is no multiple of 64 keys).  Several
# blocks hold more rows than keys, as a drafter block at the start of a context.
BLOCK_SHAPES = [
    ([1, 2, 1], [70, 9, 1], 8, 4, 128, 32, 512),
    ([4, 1], [3000, 2], 16, 8, 64, 16, 256),
    ([9, 5, 3], [3, 700, 2048], 16, 4, 128, 16, 512),
    ([9, 2], [1, 1500], 8, 1, 256, 32, 1024),
    ([9, 4], [5, 300], 8, 2, 64, 16, 48),
]


@pytest.mark.parametrize("rows,keys,hq,hkv,d,p,split", BLOCK_SHAPES)
def test_block_matches_oracle(orc, rows, keys, hq, hkv, d, p, split):
    b = wl.make_paged_batch(31 + d + len(rows), rows, keys, hq, hkv, d, p, unused="nan", split_keys=split)
    r = run_decode(b, block=True)
    assert r["status"] == 0
    ref, rf = orc.paged_attn(b.q, b.k_pool, b.v_pool, b.page_table, b.segs, b.scale, full=True)
    assert not rf.any()
    compare_attn(r["out"], r["flags"], ref, rf, what="block")


def test_block_last_row_equals_causal_last_row():
    """A stream's last row sees every key under both rules: same kernel, same
    arithmetic, so the two calls agree bit for bit there (and only there)."""
    b = wl.make_paged_batch(7, [5, 3], [900, 77], 16, 2, 256, 32, unused="nan", split_keys=1024)
    rb = run_decode(b, block=True)
    rc = run_decode(b)
    for r0, r, _, _, _ in b.segs:
        last = r0 + r - 1
        np.testing.assert_array_equal(rb["out"][last], rc["out"][last])
        assert not np.array_equal(rb["out"][r0], rc["out"][r0])


def test_block_refuses_on_host_only_what_full_allows():
    b = wl.make_paged_batch(8, [4], [2], 8, 2, 64, 16, unused="nan", split_keys=64)
    run_decode(b, block=True)  # more rows than keys: fine for a block
    with pytest.raises(binding.TfError):
        run_decode(b)  # the causal count needs a key per row


# ----------------------------------------------------------------------------- KV append

def _rows(seed, n, hkv, d):
    rng = np.random.default_rng(seed)
    return wl.normal_bf16(rng, (n, hkv, d)), wl.normal_bf16(rng, (n, hkv, d))


def _append(kr, vr, kp, vp, pt, segs, host=True, segs_dev=None):
    st = status_word()
    tf.tf_kv_append(dev(kr), dev(vr), kp, vp, dev(pt), dev(segs if segs_dev is None else segs_dev), status=st,
                    segs_host=segs if host else None, page_table_host=pt if host else None)
    torch.cuda.synchronize()
    return int(st.item())


def _bits(t):
    return t.cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("rows,keys,hkv,d,p", [([3, 1, 5], [37, 8, 40], 2, 64, 8), ([16], [2048], 4, 256, 32),
                                               ([1] * 16, [1024 + 37 * i for i in range(16)], 8, 128, 32),
                                               ([2, 7], [33, 64], 3, 128, 256), ([128], [128], 1, 256, 16)])
def test_kv_append_matches_oracle(orc, rows, keys, hkv, d, p):
    """Byte for byte the pools the oracle's writer gives: the new rows in their
    slots, every other byte of both pools unchanged (poisoned pages included)."""
    b = wl.make_paged_batch(41 + d, rows, keys, hkv, hkv, d, p, unused="nan", extra_pages=3)
    kr, vr = _rows(42 + d, sum(rows), hkv, d)
    ekp, evp = orc.put_rows(kr, vr, b.k_pool, b.v_pool, b.page_table, b.segs)
    kp, vp = dev(b.k_pool), dev(b.v_pool)
    assert _append(kr, vr, kp, vp, b.page_table, b.segs) == 0
    np.testing.assert_array_equal(_bits(kp), ekp)
    np.testing.assert_array_equal(_bits(vp), evp)


def test_kv_append_refusals():
    b = wl.make_paged_batch(5, [2, 3], [10, 20], 2, 2, 64, 8, unused="nan")
    kr, vr = _rows(6, 5, 2, 64)
    past = b.segs.copy()
    past[1, 2] = past[1, 4] * 8 + 1  # a key past stream 1's pages
    # host tables: refused before any launch
    kp, vp = dev(b.k_pool), dev(b.v_pool)
    with pytest.raises(binding.TfError, match="PAST_PAGES"):
        _append(kr, vr, kp, vp, b.page_table, past)
    # device table only: the stream is skipped and reported, the other written
    st = _append(kr, vr, kp, vp, b.page_table, past, host=False)
    assert st & binding.TF_DEV_PAST_PAGES
    got = _bits(kp)
    assert not np.array_equal(got, b.k_pool)  # stream 0 written
    pages1 = b.page_table[b.segs[1, 3]:b.segs[1, 3] + b.segs[1, 4]]
    np.testing.assert_array_equal(got[pages1], b.k_pool[pages1])  # stream 1 untouched
    # a page id outside the pool: that row is skipped and reported
    bad = b.page_table.copy()
    bad[b.segs[0, 3] + 1] = b.k_pool.shape[0] + 5  # keys 8..9 of stream 0
    kp, vp = dev(b.k_pool), dev(b.v_pool)
    st = _append(kr, vr, kp, vp, bad, b.segs, host=False)
    assert st & binding.TF_DEV_BAD_PAGE


def test_append_then_prompt_equals_oracle(orc):
    """A prompt chunk whose own keys arrive by tf_kv_append (their slots NaN
    before) gives the oracle's result over the complete pools."""
    b, spans = wl.long_prompt(4, n_tokens=700, chunk=256)
    seg = b.segs[0]
    n = int(seg[2])
    kd, vd = orc.gather_paged(b.k_pool, b.v_pool, b.page_table, int(seg[3]), int(seg[4]), n)
    k_rows = wl.f32_to_bf16_bits(kd.astype(np.float32))  # exact: the values are bf16
    v_rows = wl.f32_to_bf16_bits(vd.astype(np.float32))
    nan_rows = np.full_like(k_rows, wl.BF16_NAN)
    one = np.array([[0, n, n, seg[3], seg[4]]], np.int32)
    kp0, vp0 = orc.put_rows(nan_rows, nan_rows, b.k_pool, b.v_pool, b.page_table, one)  # keys not yet written
    ref, rf = orc.paged_attn(b.q, b.k_pool, b.v_pool, b.page_table, b.segs, b.scale)
    kp, vp = dev(kp0), dev(vp0)
    pt = dev(b.page_table)
    q = dev(b.q)
    out = torch.full(tuple(b.q.shape), float("nan"), dtype=torch.float32, device="cuda")
    fl = torch.full(tuple(b.q.shape[:2]), 9, dtype=torch.uint8, device="cuda")
    st = status_word()
    for r0, r1 in spans:
        tf.tf_kv_append(dev(k_rows[r0:r1]).contiguous(), dev(v_rows[r0:r1]).contiguous(), kp, vp, pt,
                        dev(np.array([[0, r1 - r0, r1, seg[3], seg[4]]], np.int32)), status=st,
                        segs_host=np.array([[0, r1 - r0, r1, seg[3], seg[4]]], np.int32))
        tf.tf_paged_attn_prompt(q, kp, vp, pt, wl.prompt_chunk_seg(b, r0, r1), scale=b.scale, out=out, flags=fl,
                                status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    compare_attn(out.cpu().numpy(), fl.cpu().numpy(), ref, rf, what="append + prompt")
