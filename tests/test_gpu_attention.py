"""Parity of the CUDA attention path (through the C ABI) with the float64 oracle.

Tolerances: fp32 outputs within max-abs 2e-3 and relative L2 1e-3 of the
oracle; nonfinite flags, page/slot indexing (poison and layout pins) and
empty-partial markers bit-exact.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_segment_b200 as tf
from paged_kv_cache_segment_b200 import workloads as wl

from _gpu import (compare_attn, dev, run_decode, run_prompt_chunks, run_ring, status_word, bf16_ulp,
                  prompt_bf16_bound, check_prompt_bf16)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


def oracle_paged(orc, b, sel=None, full=False):
    return orc.paged_attn(b.q, b.k_pool, b.v_pool, b.page_table, b.segs, b.scale, full=full, sel=sel)


# ----------------------------------------------------------------------------
# the tiny decode (two streams, 37 and 70 keys, two partials each)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("unused", ["normal", "nan"])
def test_tiny_decode(orc, unused):
    b = wl.tiny_decode(1, unused=unused)
    r = run_decode(b)
    assert r["status"] == 0
    ref, rf = oracle_paged(orc, b)
    assert not rf.any()
    compare_attn(r["out"], r["flags"], ref, rf, what="tiny decode")


def test_tiny_decode_partials_match_oracle_partials(orc):
    b = wl.tiny_decode(1)
    r = run_decode(b)
    po, pm, pl, pf = orc.paged_partials(b.q, b.k_pool, b.v_pool, b.page_table, b.segs, b.scale, 0, 2)
    # same split rule: the same partials are empty on both sides
    np.testing.assert_array_equal(r["pl"] > 0, pl > 0)
    live = pl > 0
    # normalised partial and log-sum-exp agree within tolerance
    g = r["po"][live] / r["pl"][live][:, None]
    o = po[live] / pl[live][:, None]
    assert np.abs(g - o).max() < 2e-3
    np.testing.assert_allclose(r["pm"][live] + np.log(r["pl"][live]), pm[live] + np.log(pl[live]), atol=1e-4)
    np.testing.assert_array_equal(r["pf"], pf)


# ----------------------------------------------------------------------------
# multi-stream decode at its full size (16 streams, 8,192-page pool)
# ----------------------------------------------------------------------------

def test_multi_stream_decode_full(orc):
    b = wl.multi_stream_decode(2)
    r = run_decode(b)
    assert r["status"] == 0
    ref, rf = oracle_paged(orc, b)
    assert not rf.any(), "NaN-poisoned slots outside the streams' keys must never be read"
    compare_attn(r["out"], r["flags"], ref, rf, what="multi-stream decode")


@pytest.mark.parametrize("hq,hkv,d,p,split", [(8, 8, 64, 16, 64), (32, 8, 128, 32, 512), (16, 2, 256, 32, 128),
                                              (4, 1, 128, 8, 0), (12, 4, 64, 64, 96)])
def test_decode_shapes(orc, hq, hkv, d, p, split):
    rng = np.random.default_rng(d + hq)
    keys = [1, 2, 17, 63, 64, 65, 300, 1000]
    b = wl.make_paged_batch(d + p, rows=[1] * len(keys), keys=keys, n_q_heads=hq, n_kv_heads=hkv, head_dim=d,
                            page_size=p, unused="nan", split_keys=split, n_splits_max=3, extra_pages=5)
    r = run_decode(b)
    assert r["status"] == 0
    ref, rf = oracle_paged(orc, b)
    compare_attn(r["out"], r["flags"], ref, rf, what=f"decode {hq}/{hkv} D{d} P{p}")


# ----------------------------------------------------------------------------
# shared verify round: multi-row causal streams, planted nonfinite heads
# ----------------------------------------------------------------------------

def test_shared_verify_full(orc):
    b = wl.shared_verify(3)
    r = run_decode(b)
    assert r["status"] == 0
    ref, rf = oracle_paged(orc, b)
    assert rf.sum() == 2, "exactly the two planted heads are flagged by the oracle"
    compare_attn(r["out"], r["flags"], ref, rf, what="shared verify")


def test_verify_causal_flag_depends_on_mask(orc):
    """An Inf in K (or in V) at a key only a stream's later rows see flags
    exactly those rows' heads of that kv-head."""
    b = wl.make_paged_batch(31, rows=[5, 3], keys=[200, 70], n_q_heads=16, n_kv_heads=2, head_dim=256,
                            page_size=32, unused="nan", split_keys=64, n_splits_max=4)
    s0 = b.segs[0]
    key_k = s0[2] - 2  # seen by rows 3 and 4 of stream 0
    key_v = s0[2] - 1  # seen by row 4 only
    pk = b.page_table[s0[3] + key_k // 32]
    pv = b.page_table[s0[3] + key_v // 32]
    b.k_pool[pk, 1, key_k % 32, 9] = wl.BF16_POS_INF
    b.v_pool[pv, 0, key_v % 32, 3] = wl.BF16_NEG_INF
    r = run_decode(b)
    ref, rf = oracle_paged(orc, b)
    assert rf.sum() == 2 * 8 + 8
    compare_attn(r["out"], r["flags"], ref, rf, what="causal flags")


@pytest.mark.parametrize("rows", [[16, 16, 1], [9, 2, 13], [16]])
def test_verify_many_rows(orc, rows):
    keys = [max(r, k) for r, k in zip(rows, [2000, 33, 700])]
    b = wl.make_paged_batch(40 + len(rows), rows=rows, keys=keys, n_q_heads=16, n_kv_heads=2, head_dim=256,
                            page_size=32, unused="nan", split_keys=256, n_splits_max=8)
    r = run_decode(b)
    ref, rf = oracle_paged(orc, b)
    compare_attn(r["out"], r["flags"], ref, rf, what="verify rows")


def test_rows_equal_keys(orc):
    """n_keys == n_rows: row 0 sees one key, the last row sees all."""
    b = wl.make_paged_batch(50, rows=[7], keys=[7], n_q_heads=4, n_kv_heads=2, head_dim=64, page_size=8,
                            unused="nan", split_keys=0, n_splits_max=2)
    r = run_decode(b)
    ref, rf = oracle_paged(orc, b)
    compare_attn(r["out"], r["flags"], ref, rf, what="rows == keys")


# ----------------------------------------------------------------------------
# merge on its own, from synthetic partials
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("d", [64, 128, 256])
def test_merge_against_oracle_merge(orc, d):
    rng = np.random.default_rng(d)
    rows, hq, c = 5, 3, 7
    po = rng.standard_normal((rows, hq, c, d)).astype(np.float32) * 10
    pm = (rng.standard_normal((rows, hq, c)) * 4).astype(np.float32)
    pl = rng.uniform(0.5, 50, (rows, hq, c)).astype(np.float32)
    pf = np.zeros((rows, hq, c), np.uint8)
    pm[0, 0, 3:] = -np.inf
    pl[0, 0, 3:] = 0
    po[0, 0, 3:] = np.nan  # an empty partial's o is never read
    pf[1, 2, 4] = 1
    pl[2, 1, :] = 0
    pm[2, 1, :] = -np.inf  # no partial holds a key: flagged
    po[3, 0, 2, 5] = np.inf  # a nonfinite o: flagged
    # one in the last columns too: at D 256 the second of a head's two warps
    # finds it and the whole head (both halves) must come out flagged NaN
    po[4, 1, 1, d - 3] = -np.inf
    out = torch.empty((rows, hq, d), device="cuda")
    fl = torch.empty((rows, hq), dtype=torch.uint8, device="cuda")
    tf.tf_attn_merge(dev(po), dev(pm), dev(pl), dev(pf), out, fl)
    ref, rf = orc.merge_all(po.astype(np.float64), pm.astype(np.float64), pl.astype(np.float64), pf)
    assert rf.tolist() == (fl.cpu().numpy()).tolist()
    assert rf[1, 2] and rf[2, 1] and rf[3, 0] and rf[4, 1] and not rf[0, 0]
    o = out.cpu().numpy()
    assert np.isnan(o[3, 0]).all() and np.isnan(o[4, 1]).all()
    compare_attn(o, fl.cpu().numpy(), ref, rf, max_abs=1e-4, rel_l2=1e-6, what="merge")


# ----------------------------------------------------------------------------
# pins on the GPU: single key, equal scores, accumulation, layout, poison
# ----------------------------------------------------------------------------

def test_single_key_exact():
    b = wl.make_paged_batch(60, rows=[1, 1], keys=[1, 1], n_q_heads=8, n_kv_heads=2, head_dim=128, page_size=16,
                            unused="nan", split_keys=0, n_splits_max=1)
    r = run_decode(b)
    for s in range(2):
        page = b.page_table[b.segs[s][3]]
        for h in range(8):
            want = wl.bf16_bits_to_f32(b.v_pool[page, h // 4, 0])
            np.testing.assert_array_equal(r["out"][s, h], want)


def test_equal_scores_mean_of_values(orc):
    b = wl.make_paged_batch(61, rows=[1], keys=[300], n_q_heads=4, n_kv_heads=2, head_dim=64, page_size=32,
                            unused="nan", split_keys=128, n_splits_max=3)
    b.q[:] = 0
    r = run_decode(b)
    ref, rf = oracle_paged(orc, b)
    compare_attn(r["out"], r["flags"], ref, rf, what="q = 0")


def test_accumulation_exact_4200():
    """V = 1, q = 0 over 4,200 keys gives exactly 1.0: fp32 sums are exact
    here, where a bf16 accumulator would be far off."""
    b = wl.make_paged_batch(62, rows=[1], keys=[4200], n_q_heads=16, n_kv_heads=2, head_dim=256, page_size=32,
                            unused="nan", split_keys=0, n_splits_max=1)
    b.q[:] = 0
    for p_ in b.page_table:
        b.v_pool[p_] = np.where(np.isnan(wl.bf16_bits_to_f32(b.v_pool[p_])), b.v_pool[p_], np.uint16(0x3F80))
    r = run_decode(b)
    assert not r["flags"].any()
    np.testing.assert_array_equal(r["out"], np.ones_like(r["out"]))


def test_page_shuffle_is_byte_equal():
    """Moving every page to another pool slot and rewriting the table leaves
    the outputs byte-identical (linear vs paged layout equivalence)."""
    b = wl.make_paged_batch(63, rows=[1, 4, 2], keys=[500, 900, 77], n_q_heads=16, n_kv_heads=2, head_dim=256,
                            page_size=32, unused="nan", split_keys=256, n_splits_max=4, extra_pages=10)
    r1 = run_decode(b)
    rng = np.random.default_rng(5)
    perm = rng.permutation(b.n_pages)
    b2 = wl.PagedBatch(**{**b.__dict__})
    b2.k_pool = np.empty_like(b.k_pool)
    b2.v_pool = np.empty_like(b.v_pool)
    b2.k_pool[perm] = b.k_pool
    b2.v_pool[perm] = b.v_pool
    b2.page_table = perm[b.page_table].astype(np.int32)
    r2 = run_decode(b2)
    assert r1["out"].tobytes() == r2["out"].tobytes()
    assert r1["flags"].tobytes() == r2["flags"].tobytes()


def test_stale_page_control_goes_red(orc):
    """The pages' stale-page control: a first page id pointing at another
    stream's page must break parity (the check is not vacuous)."""
    b = wl.make_paged_batch(64, rows=[1, 1], keys=[100, 100], n_q_heads=8, n_kv_heads=2, head_dim=128,
                            page_size=32, unused="normal", split_keys=0, n_splits_max=2)
    ref, rf = oracle_paged(orc, b)
    bad = b.page_table.copy()
    bad[b.segs[0][3]] = b.page_table[b.segs[1][3] + 1]
    r = run_decode(b, page_table=bad)
    with pytest.raises(AssertionError):
        compare_attn(r["out"], r["flags"], ref, rf, what="stale page")


def test_repeat_determinism():
    b = wl.shared_verify(3, n_streams=3, key_hi=4000)
    outs = [run_decode(b) for _ in range(5)]
    for r in outs[1:]:
        assert r["out"].tobytes() == outs[0]["out"].tobytes()
        assert r["po"].tobytes() == outs[0]["po"].tobytes()


# ----------------------------------------------------------------------------
# device-side table errors: status bits, no trap
# ----------------------------------------------------------------------------

def test_device_reports_bad_page_and_past_pages():
    b = wl.make_paged_batch(70, rows=[1, 1, 1], keys=[40, 40, 40], n_q_heads=4, n_kv_heads=2, head_dim=64,
                            page_size=16, unused="nan", split_keys=0, n_splits_max=2, extra_pages=2)
    pt = b.page_table.copy()
    pt[b.segs[1][3] + 1] = b.n_pages + 5  # outside the pool
    segs = b.segs.copy()
    segs[2][2] = 49  # 3 pages of 16 hold 48 keys
    r = run_decode(b, segs=segs, page_table=pt, host_tables=False)
    assert r["status"] & tf.binding.TF_DEV_BAD_PAGE
    assert r["status"] & tf.binding.TF_DEV_PAST_PAGES
    assert r["flags"][1].all(), "a stream that hit a bad page is flagged"


def test_host_tables_refuse_before_launch():
    b = wl.tiny_decode(1)
    segs = b.segs.copy()
    segs[0][2] = 49  # stream 0 owns 3 pages of 16
    with pytest.raises(tf.TfError, match="PAST_PAGES"):
        run_decode(b, segs=segs)
    pt = b.page_table.copy()
    pt[0] = 99
    with pytest.raises(tf.TfError, match="BAD_PAGE"):
        run_decode(b, page_table=pt)


def test_too_many_splits_flagged_on_device():
    b = wl.make_paged_batch(71, rows=[1], keys=[1000], n_q_heads=4, n_kv_heads=2, head_dim=64, page_size=16,
                            unused="nan", split_keys=64, n_splits_max=4)
    r = run_decode(b, n_splits_max=4, host_tables=False)
    assert r["status"] & tf.binding.TF_DEV_SPLITS


def test_empty_calls_are_no_ops():
    b = wl.tiny_decode(1)
    r = run_decode(b, segs=np.zeros((0, 5), np.int32), merge=False)
    assert r["status"] == 0
    segs = b.segs.copy()
    segs[:, 1] = 0  # no rows this call
    r = run_decode(b, segs=segs, merge=False)
    assert r["status"] == 0 and np.isnan(r["pl"]).all()  # nothing written


# ----------------------------------------------------------------------------
# ring of slots
# ----------------------------------------------------------------------------

def test_drafter_ring_full(orc):
    b = wl.drafter_ring(5)
    r = run_ring(b)
    assert r["status"] == 0
    ref, rf = orc.ring_attn(b.q, b.ring_k, b.ring_v, b.rsegs, b.scale)
    assert not rf.any(), "NaN outside every ring's window must never be read"
    compare_attn(r["out"], r["flags"], ref, rf, what="drafter ring")


@pytest.mark.parametrize("size,head,n", [(100, 0, 100), (100, 0, 37), (100, 10, 100), (100, 10, 11), (100, 99, 1),
                                         (4200, 7, 4200), (4200, 4199, 3000), (64, 63, 64), (17, 5, 16)])
def test_ring_wrap_cases(orc, size, head, n):
    b = wl.make_ring_batch(size + head + n, n_streams=3, ring_size=size, valid_lo=n, valid_hi=n, n_q_heads=16,
                           n_kv_heads=2, head_dim=256, split_slots=64, heads=[head, (head + 1) % size, 0],
                           valids=[n, n, n])
    r = run_ring(b)
    ref, rf = orc.ring_attn(b.q, b.ring_k, b.ring_v, b.rsegs, b.scale)
    assert not rf.any()
    compare_attn(r["out"], r["flags"], ref, rf, what=f"ring {size}/{head}/{n}")


def test_ring_equals_unrolled_paged_byte_for_byte():
    """A ring read oldest-first equals the same keys laid out contiguously
    and read by the paged kernel, bit for bit, when the wrap falls on a tile
    boundary (same tiles, same fold order)."""
    # ring 0 does not wrap; ring 1 wraps at key 128, on a 64-key tile boundary
    b = wl.make_ring_batch(80, n_streams=2, ring_size=700, valid_lo=640, valid_hi=640, n_q_heads=16, n_kv_heads=2,
                           head_dim=256, split_slots=128, heads=[640, 512], valids=[640, 640])
    r = run_ring(b)
    for s in range(2):
        e = b.rsegs[s]
        n, size, head, base = int(e["n_valid"]), int(e["size"]), int(e["head"]), int(e["base"])
        slots = [(head - n + j) % size for j in range(n)]
        keys = b.ring_k[base + np.array(slots)]  # [n][Hkv][D]
        vals = b.ring_v[base + np.array(slots)]
        psz = 32
        npg = -(-n // psz)
        kp = np.full((npg, 2, psz, 256), wl.BF16_NAN, np.uint16)
        vp = np.full_like(kp, wl.BF16_NAN)
        for j in range(n):
            kp[j // psz, :, j % psz] = keys[j]
            vp[j // psz, :, j % psz] = vals[j]
        pb = wl.PagedBatch(q=b.q[s:s + 1].copy(), k_pool=kp, v_pool=vp, page_table=np.arange(npg, dtype=np.int32),
                           segs=np.array([[0, 1, n, 0, npg]], np.int32), n_q_heads=16, n_kv_heads=2, head_dim=256,
                           page_size=psz, scale=b.scale, split_keys=128, n_splits_max=b.n_splits_max)
        rp = run_decode(pb)
        assert rp["out"][0].tobytes() == r["out"][s].tobytes()


def test_ring_planted_nonfinite(orc):
    b = wl.make_ring_batch(81, n_streams=4, ring_size=300, valid_lo=100, valid_hi=300, n_q_heads=16, n_kv_heads=2,
                           head_dim=256, split_slots=64, unused="normal")
    e = b.rsegs[1]
    slot = (int(e["head"]) - 1) % int(e["size"])  # newest slot of ring 1
    b.ring_v[int(e["base"]) + slot, 1, 17] = wl.BF16_NAN
    e = b.rsegs[2]
    slot = (int(e["head"]) - int(e["n_valid"]) - 1) % int(e["size"])  # just outside ring 2's window
    b.ring_k[int(e["base"]) + slot, 0, 3] = wl.BF16_POS_INF
    r = run_ring(b)
    ref, rf = orc.ring_attn(b.q, b.ring_k, b.ring_v, b.rsegs, b.scale)
    assert rf[1, 8:].all() and not rf[1, :8].any() and not rf[2].any()
    compare_attn(r["out"], r["flags"], ref, rf, what="ring flags")


# ----------------------------------------------------------------------------
# causal prompt chunks through the page table
# ----------------------------------------------------------------------------

def _prompt_sel(rows, hq, chunk, rng, per_chunk=12):
    sel = np.zeros((rows, hq), bool)
    for a in range(0, rows, chunk):
        b_ = min(rows, a + chunk)
        picks = {a, a + 1, b_ - 1, b_ - 2} | set(rng.integers(a, b_, size=per_chunk).tolist())
        for p in picks:
            sel[p, :] = True
    return sel


def test_prompt_small_all_rows(orc):
    """f32 output: the fp32 tolerance (P fed as bf16 hi + lo).  bf16 output:
    the bound derived from bf16 weights and bf16 rounding."""
    b, spans = wl.long_prompt(4, n_tokens=700, chunk=256)
    ref, rf = orc.paged_attn(b.q, b.k_pool, b.v_pool, b.page_table, b.segs, b.scale)
    r = run_prompt_chunks(b, spans, out_dtype=torch.float32)
    assert r["status"] == 0
    compare_attn(r["out"], r["flags"], ref, rf, what="prompt f32")
    r = run_prompt_chunks(b, spans, out_dtype=torch.bfloat16)
    assert r["status"] == 0
    check_prompt_bf16(r["out"], r["flags"], ref, rf, prompt_bf16_bound(b, ref))


def test_long_prompt_sampled_rows(orc):
    """The 15,000-token prompt in 2,048-row chunks, every chunk's first and
    last rows and random rows checked against the oracle."""
    b, spans = wl.long_prompt(4)
    r = run_prompt_chunks(b, spans, out_dtype=torch.bfloat16)
    assert r["status"] == 0
    sel = _prompt_sel(b.n_rows_total, b.n_q_heads, 2048, np.random.default_rng(1))
    ref, rf = orc.paged_attn(b.q, b.k_pool, b.v_pool, b.page_table, b.segs, b.scale, sel=sel.astype(np.uint8))
    np.testing.assert_array_equal(r["flags"], np.zeros_like(r["flags"]))
    check_prompt_bf16(r["out"], r["flags"], ref, rf, prompt_bf16_bound(b, ref), sel=sel, what="long prompt")


def test_long_prompt_chunk6_and_last_chunk_every_row(orc):
    """The 15,000-token prompt run as the benchmark runs it (all eight
    2,048-row chunks back to back, each a programmatic dependent of the one
    before), then every row and head of chunk 6 (rows 12,288-14,335, the
    longest full chunk: 12,289-14,336 keys a row, all 64 query tiles of each
    kv-head) and of the last, ragged chunk (rows 14,336-14,999) against the
    oracle: the f32 output within max-abs 2e-3 / rel-L2 1e-3, the bf16
    output within the derived per-element bound and rel-L2 3e-3."""
    b, spans = wl.long_prompt(4)
    assert spans[6] == (12288, 14336) and spans[-1] == (14336, 15000)
    sel = np.zeros((b.n_rows_total, b.n_q_heads), np.uint8)
    sel[12288:15000, :] = 1
    ref, rf = orc.paged_attn(b.q, b.k_pool, b.v_pool, b.page_table, b.segs, b.scale, sel=sel)
    assert not rf[12288:].any()
    s = sel.astype(bool)
    r = run_prompt_chunks(b, spans, out_dtype=torch.float32)
    assert r["status"] == 0
    compare_attn(r["out"], r["flags"], ref, rf, sel=s, what="long prompt f32, chunk 6 + last")
    r = run_prompt_chunks(b, spans, out_dtype=torch.bfloat16)
    assert r["status"] == 0
    check_prompt_bf16(r["out"], r["flags"], ref, rf, prompt_bf16_bound(b, ref), sel=s,
                      what="long prompt bf16, chunk 6 + last")


@pytest.mark.parametrize("hq,hkv,d,p,n,chunk", [(16, 4, 256, 32, 700, 256), (8, 8, 64, 16, 300, 100),
                                                (8, 2, 128, 64, 513, 200), (4, 1, 128, 256, 1000, 384),
                                                (6, 2, 64, 16, 200, 64), (32, 4, 128, 32, 260, 260),
                                                (16, 2, 256, 8, 150, 150)])
def test_prompt_shapes(orc, hq, hkv, d, p, n, chunk):
    """Prompt chunks at several head counts, head dims and page sizes (G = 3
    takes the mma.sync path, every other shape the tensor-memory one)."""
    b = wl.make_paged_batch(n + d + p, rows=[n], keys=[n], n_q_heads=hq, n_kv_heads=hkv, head_dim=d, page_size=p,
                            unused="nan", split_keys=0, n_splits_max=1)
    spans = [(a, min(a + chunk, n)) for a in range(0, n, chunk)]
    r = run_prompt_chunks(b, spans, out_dtype=torch.float32)
    assert r["status"] == 0
    ref, rf = orc.paged_attn(b.q, b.k_pool, b.v_pool, b.page_table, b.segs, b.scale)
    compare_attn(r["out"], r["flags"], ref, rf, what=f"prompt {hq}/{hkv} D{d} P{p}")
    r = run_prompt_chunks(b, spans, out_dtype=torch.bfloat16)
    check_prompt_bf16(r["out"], r["flags"], ref, rf, prompt_bf16_bound(b, ref), what=f"prompt bf16 {hq}/{hkv} D{d}")


def test_prompt_nonfinite_flags(orc):
    """Inf in an early key (seen by rows 3 on), NaN in a value only the chunk's
    last rows see, -Inf in one q element: flags equal the oracle's."""
    n = 400
    b = wl.make_paged_batch(77, rows=[n], keys=[n], n_q_heads=16, n_kv_heads=4, head_dim=256, page_size=32,
                            unused="nan", split_keys=0, n_splits_max=1)
    pt = b.page_table
    b.k_pool[pt[3 // 32], 1, 3 % 32, 7] = wl.BF16_POS_INF
    b.v_pool[pt[395 // 32], 2, 395 % 32, 100] = wl.BF16_NAN
    b.q[250, 13, 0] = wl.BF16_NEG_INF
    spans = [(0, 200), (200, 400)]
    r = run_prompt_chunks(b, spans, out_dtype=torch.float32)
    ref, rf = orc.paged_attn(b.q, b.k_pool, b.v_pool, b.page_table, b.segs, b.scale)
    assert rf[3:, 4:8].all() and not rf[:3, 4:8].any()  # key 3 is seen by rows 3..
    assert rf[395:, 8:12].all() and not rf[:395, 8:12].any() and rf[250, 13]
    compare_attn(r["out"], r["flags"], ref, rf, what="prompt flags")
    r = run_prompt_chunks(b, spans, out_dtype=torch.bfloat16)
    check_prompt_bf16(r["out"], r["flags"], ref, rf, prompt_bf16_bound(b, ref), what="prompt flags bf16")
