"""Pins of the float64 oracle to things other than itself (no GPU).

Each test checks the oracle against a library routine on a special case
(torch's scaled_dot_product_attention in float64, numpy's argmax), a closed
form, an invariant the mathematics fixes, or a writer-side construction of
the same data.  The planted-control tests at the end edit the oracle's
source the way the pages' own contract controls edit theirs, rebuild it, and
require a pin to go red.
"""
import math
import os
import shutil
import subprocess
import tempfile

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from paged_kv_cache_segment_b200 import workloads as wl

TOL = 1e-11


# ----------------------------------------------------------------------------
# helpers that build inputs from the writer's side
# ----------------------------------------------------------------------------

def bfbits(x):
    return int(wl.f32_to_bf16_bits(np.array([x], np.float32))[0])


def bf16_round(x):
    return wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(np.asarray(x, np.float32))).astype(np.float64)


def scatter_into_pages(k_dense_bits, v_dense_bits, page_size, n_pool, rng, poison=True, reserve=None):
    """Write each stream's keys into pages drawn from a shuffled pool:
    key j goes to page table entry j // P, slot j % P.  `reserve` (per stream)
    takes at least that many pages for a stream.  Returns pool, table, segs."""
    hkv, d = k_dense_bits[0].shape[1:]
    shape = (n_pool, hkv, page_size, d)
    fill = wl.BF16_NAN if poison else np.uint16(0)
    kp = np.full(shape, fill, np.uint16)
    vp = np.full(shape, fill, np.uint16)
    perm = rng.permutation(n_pool).astype(np.int32)
    table = []
    nxt = 0
    bases = []
    for si, (kd, vd) in enumerate(zip(k_dense_bits, v_dense_bits)):
        n = kd.shape[0]
        npg = max(-(-n // page_size), reserve[si] if reserve is not None else 0)
        bases.append((len(table), npg))
        pages = perm[nxt:nxt + npg]
        nxt += npg
        table.extend(pages.tolist())
        for j in range(n):
            kp[pages[j // page_size], :, j % page_size, :] = kd[j]
            vp[pages[j // page_size], :, j % page_size, :] = vd[j]
    return kp, vp, np.array(table, np.int32), bases


def sdpa_reference(qf, kf, vf, scale, n_rows, n_keys, full=False):
    """torch SDPA in float64 with the bottom-right causal mask and GQA by
    repeating kv-heads.  qf [R][Hq][D], kf/vf [N][Hkv][D] (float64)."""
    hq, hkv = qf.shape[1], kf.shape[1]
    q = torch.from_numpy(qf).permute(1, 0, 2)  # [Hq][R][D]
    k = torch.from_numpy(kf).permute(1, 0, 2).repeat_interleave(hq // hkv, dim=0)
    v = torch.from_numpy(vf).permute(1, 0, 2).repeat_interleave(hq // hkv, dim=0)
    if full:
        mask = None
    else:
        mask = torch.ones(n_rows, n_keys, dtype=torch.bool).tril(diagonal=n_keys - n_rows)
    out = F.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=scale)
    return out.permute(1, 0, 2).numpy()


def make_streams(seed, rows, keys, hq, hkv, d, page_size, extra=3, poison=True):
    rng = np.random.default_rng(seed)
    ks = [wl.normal_bf16(rng, (n, hkv, d)) for n in keys]
    vs = [wl.normal_bf16(rng, (n, hkv, d)) for n in keys]
    n_pool = sum(-(-n // page_size) for n in keys) + extra
    kp, vp, table, bases = scatter_into_pages(ks, vs, page_size, n_pool, rng, poison)
    q = wl.normal_bf16(rng, (sum(rows), hq, d))
    segs = []
    r0 = 0
    for (b, npg), r, n in zip(bases, rows, keys):
        segs.append((r0, r, n, b, npg))
        r0 += r
    return q, ks, vs, kp, vp, table, np.array(segs, np.int32)


# ----------------------------------------------------------------------------
# attention against torch's float64 SDPA
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("hq,hkv,d,p", [(8, 2, 64, 16), (4, 4, 32, 8), (16, 2, 64, 32), (6, 3, 16, 4)])
def test_paged_attention_matches_sdpa(orc, hq, hkv, d, p):
    rows = [1, 3, 7, 1]
    keys = [5, 37, 70, 1]
    q, ks, vs, kp, vp, table, segs = make_streams(11 + d, rows, keys, hq, hkv, d, p)
    scale = 1.0 / math.sqrt(d)
    out, flags = orc.paged_attn(q, kp, vp, table, segs, scale)
    assert not flags.any(), "poisoned slots must never be read"
    for (r0, r, n, _, _), kd, vd in zip(segs, ks, vs):
        ref = sdpa_reference(wl.bf16_bits_to_f32(q[r0:r0 + r]).astype(np.float64),
                             wl.bf16_bits_to_f32(kd).astype(np.float64), wl.bf16_bits_to_f32(vd).astype(np.float64),
                             scale, r, n)
        np.testing.assert_allclose(out[r0:r0 + r], ref, rtol=0, atol=TOL)


def test_full_flag_matches_sdpa_without_mask(orc):
    rows, keys = [4, 2], [9, 20]
    q, ks, vs, kp, vp, table, segs = make_streams(5, rows, keys, 4, 2, 32, 8)
    out, flags = orc.paged_attn(q, kp, vp, table, segs, 0.3, full=True)
    assert not flags.any()
    for (r0, r, n, _, _), kd, vd in zip(segs, ks, vs):
        ref = sdpa_reference(wl.bf16_bits_to_f32(q[r0:r0 + r]).astype(np.float64),
                             wl.bf16_bits_to_f32(kd).astype(np.float64), wl.bf16_bits_to_f32(vd).astype(np.float64),
                             0.3, r, n, full=True)
        np.testing.assert_allclose(out[r0:r0 + r], ref, rtol=0, atol=TOL)


def test_full_block_may_be_longer_than_its_keys(orc):
    """[FULL]: a drafter block of up to nine rows over the keys [0, len + 1)
    may hold more rows than keys; every row sees them all."""
    rows, keys = [9, 3], [3, 1]
    q, ks, vs, kp, vp, table, segs = make_streams(6, rows, keys, 4, 2, 32, 8)
    out, flags = orc.paged_attn(q, kp, vp, table, segs, 0.25, full=True)
    assert not flags.any()
    for (r0, r, n, _, _), kd, vd in zip(segs, ks, vs):
        ref = sdpa_reference(wl.bf16_bits_to_f32(q[r0:r0 + r]).astype(np.float64),
                             wl.bf16_bits_to_f32(kd).astype(np.float64), wl.bf16_bits_to_f32(vd).astype(np.float64),
                             0.25, r, n, full=True)
        np.testing.assert_allclose(out[r0:r0 + r], ref, rtol=0, atol=TOL)
    with pytest.raises(ValueError):  # the causal count needs a key per row
        orc.paged_attn(q, kp, vp, table, segs, 0.25)


def append_case(seed, rows, keys, hkv, d, p, extra=3):
    """Streams of N keys whose last R keys arrive as new rows: the pools before
    (first N - R keys written, the rest NaN), the pools a writer gives with all N
    keys in place, the rows [sum R][Hkv][D] and the segment table."""
    rng = np.random.default_rng(seed)
    ks = [wl.normal_bf16(rng, (n, hkv, d)) for n in keys]
    vs = [wl.normal_bf16(rng, (n, hkv, d)) for n in keys]
    n_pool = sum(-(-n // p) for n in keys) + extra
    reserve = [-(-n // p) for n in keys]
    kp_all, vp_all, table, bases = scatter_into_pages(ks, vs, p, n_pool, np.random.default_rng(seed + 1),
                                                      reserve=reserve)
    kp_old, vp_old, table2, _ = scatter_into_pages([k[:n - r] for k, n, r in zip(ks, keys, rows)],
                                                   [v[:n - r] for v, n, r in zip(vs, keys, rows)], p, n_pool,
                                                   np.random.default_rng(seed + 1), reserve=reserve)
    assert np.array_equal(table, table2)
    k_rows = np.concatenate([k[n - r:] for k, n, r in zip(ks, keys, rows)])
    v_rows = np.concatenate([v[n - r:] for v, n, r in zip(vs, keys, rows)])
    segs, r0 = [], 0
    for (b, npg), r, n in zip(bases, rows, keys):
        segs.append((r0, r, n, b, npg))
        r0 += r
    return kp_old, vp_old, kp_all, vp_all, k_rows, v_rows, table, np.array(segs, np.int32)


@pytest.mark.parametrize("rows,keys,hkv,d,p", [([3, 1, 5], [37, 8, 40], 2, 16, 8), ([16], [16], 1, 8, 4),
                                               ([2, 7], [33, 64], 3, 32, 32)])
def test_put_rows_matches_the_writer(orc, rows, keys, hkv, d, p):
    """[WR]: putting the new rows gives byte for byte the pools a writer that
    placed every key from the start gives, and nothing else changes."""
    kp_old, vp_old, kp_all, vp_all, kr, vr, table, segs = append_case(21 + d, rows, keys, hkv, d, p)
    kp, vp = orc.put_rows(kr, vr, kp_old, vp_old, table, segs)
    assert np.array_equal(kp, kp_all) and np.array_equal(vp, vp_all)
    changed = int((kp != kp_old).sum() + (vp != vp_old).sum())
    assert changed == 2 * sum(rows) * hkv * d  # every named slot, nothing more


def test_gather_after_put_returns_the_rows(orc):
    rows, keys, hkv, d, p = [4, 1], [21, 9], 2, 16, 8
    kp_old, vp_old, _, _, kr, vr, table, segs = append_case(3, rows, keys, hkv, d, p)
    kp, vp = orc.put_rows(kr, vr, kp_old, vp_old, table, segs)
    for (r0, r, n, b, npg) in segs:
        kd, vd = orc.gather_paged(kp, vp, table, b, npg, n)
        k0, v0 = orc.gather_paged(kp_old, vp_old, table, b, npg, n)
        np.testing.assert_array_equal(kd[n - r:], wl.bf16_bits_to_f32(kr[r0:r0 + r]).astype(np.float64))
        np.testing.assert_array_equal(vd[n - r:], wl.bf16_bits_to_f32(vr[r0:r0 + r]).astype(np.float64))
        np.testing.assert_array_equal(kd[:n - r], k0[:n - r])  # earlier keys untouched


def test_put_rows_refusals(orc):
    kp_old, vp_old, _, _, kr, vr, table, segs = append_case(4, [2], [10], 1, 8, 4)
    past = segs.copy()
    past[0, 2] = past[0, 4] * 4 + 1  # a key past the stream's pages
    with pytest.raises(ValueError, match="past"):
        orc.put_rows(kr, vr, kp_old, vp_old, table, past)
    bad_table = table.copy()
    bad_table[segs[0, 3] + 2] = kp_old.shape[0]  # the page of keys 8..9 outside the pool
    with pytest.raises(ValueError, match="page id"):
        orc.put_rows(kr, vr, kp_old, vp_old, bad_table, segs)
    short = segs.copy()
    short[0, 2] = 1  # fewer keys than new rows
    with pytest.raises(ValueError):
        orc.put_rows(kr, vr, kp_old, vp_old, table, short)


def test_gather_is_the_writer_inverse(orc):
    q, ks, vs, kp, vp, table, segs = make_streams(3, [1, 1], [37, 70], 8, 2, 64, 16)
    for (r0, r, n, base, npg), kd, vd in zip(segs, ks, vs):
        gk, gv = orc.gather_paged(kp, vp, table, base, npg, n)
        np.testing.assert_array_equal(gk, wl.bf16_bits_to_f32(kd))
        np.testing.assert_array_equal(gv, wl.bf16_bits_to_f32(vd))


def test_gather_refuses_past_pages_and_bad_page(orc):
    q, ks, vs, kp, vp, table, segs = make_streams(3, [1], [37], 2, 1, 16, 16)
    with pytest.raises(ValueError, match="past"):
        orc.gather_paged(kp, vp, table, 0, 2, 37)  # 2 pages hold 32 keys
    bad = table.copy()
    bad[1] = kp.shape[0]
    with pytest.raises(ValueError, match="outside"):
        orc.gather_paged(kp, vp, bad, 0, 3, 37)


# ----------------------------------------------------------------------------
# closed forms and special cases
# ----------------------------------------------------------------------------

def test_single_key_returns_its_value_exactly(orc):
    q, ks, vs, kp, vp, table, segs = make_streams(8, [1, 1], [1, 1], 8, 2, 64, 16)
    out, flags = orc.paged_attn(q, kp, vp, table, segs, 0.125)
    assert not flags.any()
    for s, vd in enumerate(vs):
        for h in range(8):
            np.testing.assert_array_equal(out[s, h], wl.bf16_bits_to_f32(vd[0, h // 4]))


def test_zero_query_gives_mean_of_values(orc):
    q, ks, vs, kp, vp, table, segs = make_streams(9, [1], [50], 4, 2, 32, 8)
    q[:] = 0
    out, flags = orc.paged_attn(q, kp, vp, table, segs, 0.17)
    v = wl.bf16_bits_to_f32(vs[0]).astype(np.float64)
    for h in range(4):
        np.testing.assert_allclose(out[0, h], v[:, h // 2].mean(axis=0), rtol=0, atol=1e-14)


def test_two_key_softmax_by_hand(orc):
    """q = e0, K0 = 2 e0, K1 = 0, scale 1: weights e^2/(e^2+1) and 1/(e^2+1)."""
    d = 8
    ks = [np.zeros((2, 1, d), np.uint16)]
    ks[0][0, 0, 0] = bfbits(2.0)
    vs = [np.zeros((2, 1, d), np.uint16)]
    vs[0][0, 0, :] = bfbits(1.0)
    vs[0][1, 0, :] = bfbits(-3.0)
    rng = np.random.default_rng(0)
    kp, vp, table, bases = scatter_into_pages(ks, vs, 4, 3, rng)
    q = np.zeros((1, 1, d), np.uint16)
    q[0, 0, 0] = bfbits(1.0)
    segs = np.array([[0, 1, 2, bases[0][0], bases[0][1]]], np.int32)
    out, flags = orc.paged_attn(q, kp, vp, table, segs, 1.0)
    w0 = math.exp(2) / (math.exp(2) + 1)
    np.testing.assert_allclose(out[0, 0], np.full(d, w0 * 1.0 + (1 - w0) * -3.0), rtol=0, atol=1e-15)


def test_mha_when_heads_equal(orc):
    """Hq == Hkv: q-head h reads kv-head h (checked against per-head SDPA)."""
    q, ks, vs, kp, vp, table, segs = make_streams(13, [2], [19], 3, 3, 16, 4)
    out, _ = orc.paged_attn(q, kp, vp, table, segs, 0.25)
    ref = sdpa_reference(wl.bf16_bits_to_f32(q).astype(np.float64), wl.bf16_bits_to_f32(ks[0]).astype(np.float64),
                         wl.bf16_bits_to_f32(vs[0]).astype(np.float64), 0.25, 2, 19)
    np.testing.assert_allclose(out, ref, rtol=0, atol=TOL)


def test_accumulation_exact_over_4200_keys(orc):
    """V = 1 everywhere, q = 0: the output is 1 (a long sum that a 16-bit
    accumulator would get badly wrong); float64 rounding of 1/4200 only."""
    n, d = 4200, 16
    ks = [np.zeros((n, 1, d), np.uint16)]
    vs = [np.full((n, 1, d), bfbits(1.0), np.uint16)]
    kp, vp, table, bases = scatter_into_pages(ks, vs, 32, -(-n // 32) + 2, np.random.default_rng(1))
    q = np.zeros((1, 2, d), np.uint16)
    segs = np.array([[0, 1, n, 0, bases[0][1]]], np.int32)
    out, flags = orc.paged_attn(q, kp, vp, table, segs, 0.25)
    assert not flags.any()
    np.testing.assert_allclose(out, np.ones_like(out), rtol=0, atol=1e-12)


def test_causal_row_equals_one_row_call(orc):
    q, ks, vs, kp, vp, table, segs = make_streams(21, [6], [40], 4, 2, 32, 8)
    out, _ = orc.paged_attn(q, kp, vp, table, segs, 0.2)
    r0, r, n, base, npg = segs[0]
    for i in range(r):
        one = np.array([[0, 1, n - r + i + 1, base, npg]], np.int32)
        o1, _ = orc.paged_attn(q[i:i + 1], kp, vp, table, one, 0.2)
        np.testing.assert_array_equal(out[i], o1[0])


# ----------------------------------------------------------------------------
# split / merge
# ----------------------------------------------------------------------------

def test_merge_by_hand():
    """Two partials (m=0, l=1, o=1) and (m=ln 3, l=1, o=2): the merged value
    is (1*1 + 3*2) / (1*1 + 3*1) = 7/4; an empty third partial is ignored."""
    o = np.array([[1.0], [2.0], [123.0]])
    m = np.array([0.0, math.log(3.0), -np.inf])
    l = np.array([1.0, 1.0, 0.0])
    out, f = oracle.get().merge(o, m, l, np.zeros(3, np.uint8))
    assert f == 0
    assert abs(out[0] - 7 / 4) < 1e-15


def test_merge_flags_by_hand(orc):
    """The merged head is flagged (and NaN) when a partial carries a flag,
    when no partial holds a key, or when a live partial's o is nonfinite; an
    empty partial (l = 0) is never read, so NaN there changes nothing."""
    o = np.array([[1.0, -2.0], [2.0, 4.0]])
    m = np.array([0.0, math.log(3.0)])
    l = np.array([1.0, 1.0])
    out, f = orc.merge(o, m, l, np.array([0, 1], np.uint8))  # a flagged partial
    assert f == 1 and np.isnan(out).all()
    out, f = orc.merge(o, np.full(2, -np.inf), np.zeros(2), np.zeros(2, np.uint8))  # no key anywhere
    assert f == 1 and np.isnan(out).all()
    bad = o.copy()
    bad[1, 1] = np.inf  # nonfinite o in a live partial
    out, f = orc.merge(bad, m, l, np.zeros(2, np.uint8))
    assert f == 1 and np.isnan(out).all()
    empty = np.array([[1.0, -2.0], [np.nan, np.nan]])  # the second partial holds no key
    out, f = orc.merge(empty, np.array([0.0, -np.inf]), np.array([1.0, 0.0]), np.zeros(2, np.uint8))
    assert f == 0 and out.tolist() == [1.0, -2.0]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_merged_partials_equal_unsplit(orc, seed):
    rng = np.random.default_rng(seed)
    q, ks, vs, kp, vp, table, segs = make_streams(30 + seed, [3], [61], 4, 2, 32, 8)
    kd, vd = orc.gather_paged(kp, vp, table, 0, segs[0][4], 61)
    ref, _ = orc.paged_attn(q, kp, vp, table, segs, 0.18)
    for i in range(3):
        n_vis = 61 - 3 + i + 1
        cuts = np.sort(rng.choice(np.arange(1, 61), size=4, replace=False))
        bounds = [0] + cuts.tolist() + [61, 61]  # the last range is empty
        for h in range(4):
            qv = wl.bf16_bits_to_f32(q[i, h]).astype(np.float64)
            parts = [orc.partial(qv, kd, vd, h // 2, a, b, n_vis, 0.18) for a, b in zip(bounds[:-1], bounds[1:])]
            o = np.stack([p[0] for p in parts])
            out, f = orc.merge(o, np.array([p[1] for p in parts]), np.array([p[2] for p in parts]),
                               np.array([p[3] for p in parts], np.uint8))
            assert f == 0
            np.testing.assert_allclose(out, ref[i, h], rtol=0, atol=1e-13)


def test_paged_partials_follow_the_split_rule(orc):
    """split_keys = 0: two partials a stream of ceil(ceil(N/2)/P)*P keys; the
    merge of the oracle's partials equals the unsplit result."""
    b = wl.tiny_decode(1)
    po, pm, pl, pf = orc.paged_partials(b.q, b.k_pool, b.v_pool, b.page_table, b.segs, b.scale, 0, 2)
    out, fl = orc.merge_all(po, pm, pl, pf)
    ref, rf = orc.paged_attn(b.q, b.k_pool, b.v_pool, b.page_table, b.segs, b.scale)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-13)
    np.testing.assert_array_equal(fl, rf)
    # stream 0 (37 keys): [0,32) + [32,37) -> l of split 1 sums 5 terms, each <= 1
    assert np.all(pl[0, :, 1] <= 5.0 + 1e-12) and np.all(pl[0, :, 1] > 0)


# ----------------------------------------------------------------------------
# nonfinite flags: input-level brute force
# ----------------------------------------------------------------------------

def test_flags_match_input_level_definition(orc):
    rows, keys = [4, 1], [30, 12]
    hq, hkv, d = 4, 2, 16
    q, ks, vs, kp, vp, table, segs = make_streams(41, rows, keys, hq, hkv, d, 8)
    # plant: q Inf at (row 1, head 3); K NaN at stream-0 key 28 head 0 (seen only by rows 2, 3);
    # V +Inf at stream-0 key 29 head 1 (seen only by row 3); V NaN at stream-1 key 0 head 0
    q[1, 3, 5] = wl.BF16_POS_INF
    b0 = segs[0][3]
    kp[table[b0 + 28 // 8], 0, 28 % 8, 2] = wl.BF16_NAN
    vp[table[b0 + 29 // 8], 1, 29 % 8, 7] = wl.BF16_POS_INF
    b1 = segs[1][3]
    vp[table[b1], 0, 0, 0] = wl.BF16_NAN
    # K -Inf at stream-1 key 5 head 1 against q[4, 2, 3] = +1: that score is
    # -Inf, its weight 0 and the output finite, so only the score check can
    # flag the head (q[4, 3, 3] = -1 makes the other head's score +Inf)
    kp[table[b1], 1, 5, 3] = wl.BF16_NEG_INF
    q[4, 2, 3] = 0x3F80  # +1.0
    q[4, 3, 3] = 0xBF80  # -1.0
    out, flags = orc.paged_attn(q, kp, vp, table, segs, 0.25)
    expect = np.zeros_like(flags)
    for (r0, r, n, base, npg) in segs:
        gk, gv = orc.gather_paged(kp, vp, table, base, npg, n)
        for i in range(r):
            for h in range(hq):
                g = h // (hq // hkv)
                n_vis = n - r + i + 1
                qf = wl.bf16_bits_to_f32(q[r0 + i, h])
                bad = (not np.isfinite(qf).all()) or (not np.isfinite(gk[:n_vis, g]).all()) \
                    or (not np.isfinite(gv[:n_vis, g]).all())
                expect[r0 + i, h] = bad
    np.testing.assert_array_equal(flags, expect)
    assert expect.sum() >= 4
    assert np.isnan(out[flags.astype(bool)]).all()
    assert np.isfinite(out[~flags.astype(bool)]).all()


# ----------------------------------------------------------------------------
# ring of slots
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("size,written,n_valid", [(10, 7, 7), (10, 10, 10), (10, 13, 6), (10, 25, 10), (10, 30, 4),
                                                  (16, 16, 3)])
def test_ring_matches_a_writer(orc, size, written, n_valid):
    """A writer puts key t into slot t mod size; after `written` keys the head
    is written mod size, and the last n_valid keys, oldest first, are the ones
    the row attends to."""
    hq, hkv, d = 4, 2, 16
    rng = np.random.default_rng(size * 100 + written)
    stream_k = wl.normal_bf16(rng, (written, hkv, d))
    stream_v = wl.normal_bf16(rng, (written, hkv, d))
    other = 5  # a second ring before this one, so base != 0
    ring_k = np.full(((other + size), hkv, d), wl.BF16_NAN, np.uint16)
    ring_v = np.full_like(ring_k, wl.BF16_NAN)
    for t in range(written):
        ring_k[other + t % size] = stream_k[t]
        ring_v[other + t % size] = stream_v[t]
    # poison every slot outside the readable window
    live = {(written - 1 - j) % size for j in range(n_valid)}
    for s in range(size):
        if s not in live:
            ring_k[other + s] = wl.BF16_NAN
            ring_v[other + s] = wl.BF16_NAN
    q = wl.normal_bf16(rng, (2, hq, d))
    rs = np.zeros(1, oracle.RING_SEG_DTYPE)
    rs[0] = (other, 1, size, written % size, n_valid)
    out, flags = orc.ring_attn(q, ring_k, ring_v, rs, 0.3)
    assert not flags[1].any()
    ref = sdpa_reference(wl.bf16_bits_to_f32(q[1:2]).astype(np.float64),
                         wl.bf16_bits_to_f32(stream_k[written - n_valid:]).astype(np.float64),
                         wl.bf16_bits_to_f32(stream_v[written - n_valid:]).astype(np.float64), 0.3, 1, n_valid,
                         full=True)
    np.testing.assert_allclose(out[1], ref[0], rtol=0, atol=TOL)


# ----------------------------------------------------------------------------
# draft trees over a ring
# ----------------------------------------------------------------------------

def write_tree_ring(rng, size, head, window_k, window_v, node_k, node_v, hkv, d, other=3):
    """A writer's ring: the window's keys (oldest first) in the slots before
    `head`, node a in slot head + a (mod size); every other slot NaN; a second
    ring of `other` slots first, so base != 0."""
    ring_k = np.full((other + size, hkv, d), wl.BF16_NAN, np.uint16)
    ring_v = np.full_like(ring_k, wl.BF16_NAN)
    n = window_k.shape[0]
    for j in range(n):
        ring_k[other + (head - n + j) % size] = window_k[j]
        ring_v[other + (head - n + j) % size] = window_v[j]
    for a in range(node_k.shape[0]):
        ring_k[other + (head + a) % size] = node_k[a]
        ring_v[other + (head + a) % size] = node_v[a]
    return ring_k, ring_v, other


def ancestor_closure(parents):
    """[T][T] bool: a is node i itself or one of its ancestors, by boolean
    matrix squaring of (identity | parent edges) until nothing changes."""
    t = len(parents)
    m = np.eye(t, dtype=bool)
    for i, p_ in enumerate(parents):
        if p_ >= 0:
            m[i, p_] = True
    while True:
        m2 = m | ((m.astype(np.int64) @ m.astype(np.int64)) > 0)
        if (m2 == m).all():
            return m
        m = m2


def tree_case(seed, size, head, n_valid, parents, hq=4, hkv=2, d=16):
    rng = np.random.default_rng(seed)
    t = len(parents)
    wk, wv = wl.normal_bf16(rng, (n_valid, hkv, d)), wl.normal_bf16(rng, (n_valid, hkv, d))
    nk, nv = wl.normal_bf16(rng, (t, hkv, d)), wl.normal_bf16(rng, (t, hkv, d))
    ring_k, ring_v, base = write_tree_ring(rng, size, head, wk, wv, nk, nv, hkv, d)
    q = wl.normal_bf16(rng, (t + 2, hq, d))
    ts = np.zeros(1, oracle.TREE_SEG_DTYPE)
    ts[0] = (base, 1, size, head, n_valid, t, 2)
    par = np.array([7, 7] + list(parents), np.int32)  # two unrelated entries first
    return q, ring_k, ring_v, ts, par, (wk, wv, nk, nv)


TREE_SHAPES = [
    (13, 5, 6, [-1, 0, 1, 2]),                 # a chain, window wraps
    (16, 0, 9, [-1, -1, -1, -1, -1]),           # a star at head 0: the window wraps from the ring's end
    (20, 17, 8, [-1, 0, 0, 1, 1, 2, 2]),        # a binary tree whose nodes wrap
    (12, 4, 0, [-1, 0, -1, 2, 1, 3]),           # no window at all
    (30, 11, 12, [-1, 0, 1, 0, 3, 3, 5, -1, 7, 2]),
]


@pytest.mark.parametrize("size,head,n_valid,parents", TREE_SHAPES)
def test_tree_matches_sdpa_with_ancestor_mask(orc, size, head, n_valid, parents):
    """Node i against float64 SDPA over [window ++ all nodes] with a mask
    that opens the window and node i's ancestors-or-self (a transitive
    closure of the parent edges, computed apart from the oracle's walk)."""
    q, ring_k, ring_v, ts, par, (wk, wv, nk, nv) = tree_case(size * 7 + head, size, head, n_valid, parents)
    out, flags = orc.ring_tree_attn(q, ring_k, ring_v, ts, par, 0.3)
    t = len(parents)
    assert not flags[1:1 + t].any()
    kf = wl.bf16_bits_to_f32(np.concatenate([wk, nk])).astype(np.float64)
    vf = wl.bf16_bits_to_f32(np.concatenate([wv, nv])).astype(np.float64)
    qf = wl.bf16_bits_to_f32(q[1:1 + t]).astype(np.float64)
    hq, hkv = qf.shape[1], kf.shape[1]
    mask = np.concatenate([np.ones((t, n_valid), bool), ancestor_closure(parents)], axis=1)
    qt = torch.from_numpy(qf).permute(1, 0, 2)
    kt = torch.from_numpy(kf).permute(1, 0, 2).repeat_interleave(hq // hkv, dim=0)
    vt = torch.from_numpy(vf).permute(1, 0, 2).repeat_interleave(hq // hkv, dim=0)
    ref = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.from_numpy(mask), scale=0.3)
    np.testing.assert_allclose(out[1:1 + t], ref.permute(1, 0, 2).numpy(), rtol=0, atol=TOL)
    assert not out[0].any() and not out[1 + t:].any()  # rows no tree names are untouched


def test_tree_chain_equals_ring_rows(orc):
    """A tree that is one chain equals, node by node, the ring call whose
    window runs on through the chain's slots up to that node: the same keys
    in the same order, so bit for bit."""
    parents = [-1, 0, 1, 2, 3, 4]
    q, ring_k, ring_v, ts, par, _ = tree_case(5, 17, 14, 9, parents)
    out, flags = orc.ring_tree_attn(q, ring_k, ring_v, ts, par, 0.3)
    e = ts[0]
    for i in range(len(parents)):
        rs = np.zeros(1, oracle.RING_SEG_DTYPE)
        rs[0] = (e["base"], 1 + i, e["size"], (e["head"] + i + 1) % e["size"], e["n_valid"] + i + 1)
        o2, f2 = orc.ring_attn(q, ring_k, ring_v, rs, 0.3)
        assert np.array_equal(out[1 + i], o2[1 + i]) and flags[1 + i].tolist() == f2[1 + i].tolist()


def test_tree_star_node_equals_window_plus_itself(orc):
    """A node with no parent sees the window and itself: the ring call over a
    fresh ring the writer fills with the window and then that node."""
    parents = [-1, -1, -1, -1]
    q, ring_k, ring_v, ts, par, (wk, wv, nk, nv) = tree_case(6, 11, 3, 6, parents)
    out, _ = orc.ring_tree_attn(q, ring_k, ring_v, ts, par, 0.3)
    rng = np.random.default_rng(0)
    for i in range(4):
        rk, rv, base = write_tree_ring(rng, 7, 0, np.concatenate([wk, nk[i:i + 1]]), np.concatenate([wv, nv[i:i + 1]]),
                                       nk[:0], nv[:0], 2, 16)
        rs = np.zeros(1, oracle.RING_SEG_DTYPE)
        rs[0] = (base, 1 + i, 7, 0, 7)
        o2, _ = orc.ring_attn(q, rk, rv, rs, 0.3)
        assert np.array_equal(out[1 + i], o2[1 + i])


def test_tree_flags_follow_the_paths(orc):
    """A NaN in node 2's value flags node 2 and the nodes under it, nothing
    else; an infinity in a window key flags every node."""
    parents = [-1, 0, 1, 0, 2, 3]  # node 2's subtree: 2, 4
    q, ring_k, ring_v, ts, par, _ = tree_case(9, 20, 6, 7, parents)
    e = ts[0]
    ring_v[e["base"] + (e["head"] + 2) % e["size"], 1, 3] = wl.BF16_NAN
    _, flags = orc.ring_tree_attn(q, ring_k, ring_v, ts, par, 0.3)
    want = np.zeros((len(parents), 4), np.uint8)
    want[[2, 4], 2:4] = 1  # kv-head 1 serves q-heads 2 and 3
    np.testing.assert_array_equal(flags[1:1 + len(parents)], want)
    ring_k[e["base"] + (e["head"] - 3) % e["size"], 0, 0] = wl.BF16_POS_INF
    _, flags = orc.ring_tree_attn(q, ring_k, ring_v, ts, par, 0.3)
    assert flags[1:1 + len(parents), 0:2].all()


def test_tree_refusals(orc):
    parents = [-1, 0, 1]
    q, ring_k, ring_v, ts, par, _ = tree_case(3, 10, 2, 4, parents)
    for bad_par in ([-1, 1, 1], [-1, 0, 3], [0, 0, 1], [-1, -2, 0]):
        p2 = par.copy()
        p2[2:] = bad_par
        with pytest.raises(ValueError):
            orc.ring_tree_attn(q, ring_k, ring_v, ts, p2, 0.3)
    ts2 = ts.copy()
    ts2[0]["n_valid"] = 8  # window + nodes past the ring
    with pytest.raises(ValueError):
        orc.ring_tree_attn(q, ring_k, ring_v, ts2, par, 0.3)


# ----------------------------------------------------------------------------
# argmax
# ----------------------------------------------------------------------------

def test_argmax_matches_numpy_first_occurrence(orc):
    logits = wl.make_logits(7, 32, 3001, sigma=3.0, tie_rows=list(range(0, 32, 3)))
    ids, flags = orc.argmax_rows(logits)
    vals = wl.bf16_bits_to_f32(logits).astype(np.float64)
    assert not flags.any()
    np.testing.assert_array_equal(ids, np.argmax(vals, axis=1))


def test_argmax_tie_rules(orc):
    logits = wl.make_logits(8, 6, 500, tie_rows=[0, 1, 2])
    logits2 = wl.make_logits(8, 6, 500, tie_rows=[0, 1, 2], tie_before=True)
    for lg in (logits, logits2):
        ids, flags = orc.argmax_rows(lg)
        vals = wl.bf16_bits_to_f32(lg)
        for r in range(3):
            mx = vals[r].max()
            where = np.flatnonzero(vals[r] == mx)
            assert len(where) >= 2
            assert ids[r] == where[0]


def test_argmax_signed_zero_and_all_equal(orc):
    lg = np.zeros((3, 8), np.uint16)
    lg[0, :] = 0xBF80  # -1.0
    lg[0, 3] = 0x8000  # -0.0 ...
    lg[0, 5] = 0x0000  # ... ties with +0.0: lower id wins
    lg[1, :] = 0x3F80  # all 1.0
    lg[2, :] = 0xFF7F  # most negative finite bf16
    lg[2, 6] = 0x8000
    lg[2, 2] = 0x0000
    ids, flags = orc.argmax_rows(lg)
    assert ids.tolist() == [3, 0, 2]
    assert not flags.any()


def test_argmax_nonfinite_rows_flagged(orc):
    lg = wl.make_logits(9, 5, 100, nan_rows=[1], posinf_rows=[2], neginf_rows=[3])
    ids, flags = orc.argmax_rows(lg)
    assert flags.tolist() == [0, 1, 1, 1, 0]
    assert ids[1] == ids[2] == ids[3] == -1


def test_argmax_respects_row_stride(orc):
    lg = wl.make_logits(10, 3, 100, ld=136)
    ids, flags = orc.argmax_rows(lg, n_cols=100)
    assert not flags.any()  # the NaN padding past column 100 is not read
    np.testing.assert_array_equal(ids, np.argmax(wl.bf16_bits_to_f32(lg[:, :100]), axis=1))


def test_golden_argmax_rules(orc):
    """Hand-derived rows in tests/golden/argmax_rules.txt."""
    path = os.path.join(os.path.dirname(__file__), "golden", "argmax_rules.txt")
    for line in open(path):
        line = line.split("#")[0].strip()
        if not line:
            continue
        vals, expect = line.split("->")
        row = np.array([float(x) for x in vals.split()], np.float32)
        bits = wl.f32_to_bf16_bits(row)[None, :]
        bits[0][np.signbit(row) & (row == 0)] = 0x8000
        ids, flags = orc.argmax_rows(bits)
        want_id, want_flag = (int(x) for x in expect.split())
        assert (ids[0], flags[0]) == (want_id, want_flag), line


def test_golden_attention_by_hand(orc):
    """Hand-computed cases in tests/golden/attention_by_hand.txt."""
    path = os.path.join(os.path.dirname(__file__), "golden", "attention_by_hand.txt")
    cases = [l.split("#")[0].strip() for l in open(path)]
    for line in [c for c in cases if c]:
        qs, ks_, vs_, sc, want = (part.strip() for part in line.split("|"))
        qv = [float(x) for x in qs.split()]
        keys = [[float(x) for x in k.split()] for k in ks_.split(";")]
        vals = [[float(x) for x in v.split()] for v in vs_.split(";")]
        d = len(qv)
        kb = [wl.f32_to_bf16_bits(np.array(keys, np.float32)).reshape(len(keys), 1, d)]
        vb = [wl.f32_to_bf16_bits(np.array(vals, np.float32)).reshape(len(vals), 1, d)]
        kp, vp, table, bases = scatter_into_pages(kb, vb, 2, bases_pages(len(keys)), np.random.default_rng(0))
        q = wl.f32_to_bf16_bits(np.array(qv, np.float32)).reshape(1, 1, d)
        segs = np.array([[0, 1, len(keys), 0, bases[0][1]]], np.int32)
        out, flags = orc.paged_attn(q, kp, vp, table, segs, float(sc))
        np.testing.assert_allclose(out[0, 0], [float(x) for x in want.split()], rtol=0, atol=1e-9)


def bases_pages(n):
    return -(-n // 2) + 1


# ----------------------------------------------------------------------------
# planted controls: edit the oracle's source, rebuild, and a pin must go red
# ----------------------------------------------------------------------------

CONTROLS = {
    "tie_to_highest_id": ("if (best < 0 || v > best_v) {", "if (best < 0 || v >= best_v) {"),
    "nan_not_flagged": ("                bad = 1;\n                continue;", "                continue;"),
    "stale_first_page": ("int32_t page = page_table[pt_base + j / page_size];",
                         "int32_t page = page_table[pt_base + (j / page_size == 0 ? 1 : j / page_size)];"),
    "scale_dropped": ("s[j] = scale * dot;", "s[j] = dot;"),
    "gqa_modulo": ("h / group, n_vis, scale, sc,", "h % group, n_vis, scale, sc,"),
    "merge_weight_dropped": ("if (l[c] > 0.0) denom += exp(m[c] - mx) * l[c];", "if (l[c] > 0.0) denom += l[c];"),
    "ring_no_lag": ("int32_t slot = ((e.head - n + j) % e.size + e.size) % e.size;",
                    "int32_t slot = ((e.head + j) % e.size + e.size) % e.size;"),
    "put_rows_reversed": ("const int32_t j = n_keys - n_rows + i;\n            const int64_t page",
                          "const int32_t j = n_keys - 1 - i;\n            const int64_t page"),
    "causal_count_short": ("const int32_t n_vis = full ? n_keys : n_keys - n_rows + i + 1;",
                           "const int32_t n_vis = full ? n_keys : n_keys - n_rows + i;"),
    "full_ignored": ("const int32_t n_vis = full ? n_keys : n_keys - n_rows + i + 1;",
                     "const int32_t n_vis = n_keys - n_rows + i + 1;"),
    "partial_causal_short": ("h / group, a, b, n_keys - n_rows + i + 1, scale,",
                             "h / group, a, b, n_keys - n_rows + i, scale,"),
    "slot_shifted": ("int32_t slot = j % page_size;", "int32_t slot = (j + 1) % page_size;"),
    "merge_flag_dropped": ("        if (flag[c]) bad = 1;\n", "        (void)flag[c];\n"),
    "score_check_dropped": ("        if (!isfinite(s[j])) bad = 1;\n", "        (void)s[j];\n"),
    "output_check_dropped": ("        if (!isfinite(out[d])) bad = 1;\n    if (n_vis <= 0) bad = 1;",
                             "        (void)out[d];\n    if (n_vis <= 0) bad = 1;"),
    "flagged_output_kept": ("        for (int32_t d = 0; d < head_dim; ++d) out[d] = NAN;\n    *flag = (uint8_t)bad;",
                            "        (void)out;\n    *flag = (uint8_t)bad;"),
    "merge_reads_empty": ("        if (!(l[c] > 0.0)) continue;\n        double w", "        double w"),
    "tree_node_slot_shifted": ("slot = (e.head + path[depth - 1 - (j - e.n_valid)]) % e.size;",
                               "slot = (e.head + 1 + path[depth - 1 - (j - e.n_valid)]) % e.size;"),
    "tree_path_without_self": ("for (int32_t a = i; a >= 0; a = parents[e.parent_base + a]) path[depth++] = a;",
                               "for (int32_t a = parents[e.parent_base + i]; a >= 0; a = parents[e.parent_base + a]) "
                               "path[depth++] = a;"),
    "tree_as_chain": ("for (int32_t a = i; a >= 0; a = parents[e.parent_base + a]) path[depth++] = a;",
                      "for (int32_t a = i; a >= 0; a = a - 1) path[depth++] = a;"),
    "tree_window_shifted": ("slot = ((e.head - e.n_valid + j) % e.size + e.size) % e.size;\n                    else",
                            "slot = ((e.head - e.n_valid + 1 + j) % e.size + e.size) % e.size;\n                    else"),
    "zeros_by_sign": ("if (best < 0 || v > best_v) {",
                      "if (best < 0 || v > best_v || (v == best_v && signbit(best_v) && !signbit(v))) {"),
}


def build_control(name):
    old, new = CONTROLS[name]
    src = open(oracle._SRC).read()
    assert src.count(old) == 1, f"control {name} no longer matches the source"
    tmp = tempfile.mkdtemp(prefix="orc_ctl_")
    path = os.path.join(tmp, "oracle.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = oracle.build(path, os.path.join(tmp, "liboracle_ctl.so"))
    return oracle.Oracle(lib), tmp


def run_pin(o, pin):
    try:
        pin(o)
    except (AssertionError, ValueError):
        return False
    return True


PIN_FOR = {
    "tie_to_highest_id": lambda o: test_argmax_tie_rules(o),
    "nan_not_flagged": lambda o: test_argmax_nonfinite_rows_flagged(o),
    "stale_first_page": lambda o: test_paged_attention_matches_sdpa(o, 8, 2, 64, 16),
    "scale_dropped": lambda o: test_paged_attention_matches_sdpa(o, 8, 2, 64, 16),
    "gqa_modulo": lambda o: test_paged_attention_matches_sdpa(o, 8, 2, 64, 16),
    "merge_weight_dropped": lambda o: test_merged_partials_equal_unsplit(o, 0),
    "ring_no_lag": lambda o: test_ring_matches_a_writer(o, 10, 13, 6),
    "put_rows_reversed": lambda o: test_put_rows_matches_the_writer(o, [3, 1, 5], [37, 8, 40], 2, 16, 8),
    "causal_count_short": lambda o: test_paged_attention_matches_sdpa(o, 8, 2, 64, 16),
    "full_ignored": lambda o: test_full_flag_matches_sdpa_without_mask(o),
    "partial_causal_short": lambda o: test_paged_partials_follow_the_split_rule(o),
    "slot_shifted": lambda o: test_paged_attention_matches_sdpa(o, 8, 2, 64, 16),
    "merge_flag_dropped": lambda o: test_merge_flags_by_hand(o),
    "output_check_dropped": lambda o: test_flags_match_input_level_definition(o),
    "score_check_dropped": lambda o: test_flags_match_input_level_definition(o),
    "flagged_output_kept": lambda o: test_flags_match_input_level_definition(o),
    "merge_reads_empty": lambda o: test_merge_flags_by_hand(o),
    "zeros_by_sign": lambda o: test_argmax_signed_zero_and_all_equal(o),
    "tree_node_slot_shifted": lambda o: test_tree_matches_sdpa_with_ancestor_mask(o, *TREE_SHAPES[2]),
    "tree_path_without_self": lambda o: test_tree_matches_sdpa_with_ancestor_mask(o, *TREE_SHAPES[4]),
    "tree_as_chain": lambda o: test_tree_matches_sdpa_with_ancestor_mask(o, *TREE_SHAPES[4]),
    "tree_window_shifted": lambda o: test_tree_matches_sdpa_with_ancestor_mask(o, *TREE_SHAPES[0]),
}


@pytest.mark.parametrize("name", sorted(CONTROLS))
def test_planted_control_goes_red(orc, name):
    assert run_pin(orc, PIN_FOR[name]), "the pin must pass on the real oracle"
    ctl, tmp = build_control(name)
    try:
        assert not run_pin(ctl, PIN_FOR[name]), f"control {name} was not caught"
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
