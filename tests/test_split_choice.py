"""tf_choose_split_keys: the host-side choice of a split size for the tcgen05
partial kernel at head dim 256 (one CTA per stream, kv-head, split and
128-query tile, one CTA an SM).  It list-schedules the kernel's CTAs in
launch order over the SMs, each costing its 64-key tiles plus eight, and
keeps the split whose last SM finishes first (#1394, "lfm2: a cheaper DSpark
hold", commit list: a hold's attention partials take all of its query rows
in one wave)."""
import ctypes
import heapq

import numpy as np
import pytest

import paged_kv_cache_segment_b200 as tf
from paged_kv_cache_segment_b200 import binding
from paged_kv_cache_segment_b200 import workloads as wl

OVERHEAD = 8  # tiles a CTA, as the header states


def candidates(max_keys):
    s = 256
    while True:
        yield s
        if s >= max_keys:
            return
        s = s + 128 if s < 4096 else (s + 1024 if s < 16384 else s * 2)


def makespan(segs, hq, hkv, split, n_sms):
    """The schedule the header describes, written out with a heap."""
    rt = 128 // (hq // hkv)
    live = [s for s in segs if s[1] > 0]
    n_qt = -(-max(s[1] for s in live) // rt)
    n_sp_max = max(-(-s[2] // split) for s in live)
    free = [0.0] * n_sms
    for s in segs:
        t_rows, n = int(s[1]), int(s[2])
        n_sp = -(-n // split) if t_rows > 0 else 0
        for _ in range(hkv):
            for c in range(n_sp_max):
                for t in range(n_qt):
                    qt = n_qt - 1 - t
                    if c >= n_sp or qt * rt >= t_rows:
                        continue
                    keys = split if c + 1 < n_sp else n - c * split
                    heapq.heappush(free, heapq.heappop(free) + OVERHEAD + -(-keys // 64))
    return max(free)


def choose(segs, hq, hkv, n_sms):
    return tf.tf_choose_split_keys(np.asarray(segs, np.int32).reshape(-1, 5), n_q_heads=hq, n_kv_heads=hkv,
                                   head_dim=256, n_sms=n_sms)


def test_one_wave_when_it_fits():
    """8 one-row streams of 9,600 keys, 2 kv-heads, 148 SMs: the smallest
    split that puts all CTAs in one wave is 1,152 (9 splits, 144 CTAs; 1,024
    needs 160).  Every larger split only lengthens the longest CTA, and any
    two-wave split costs at least twice the overhead plus its tiles."""
    segs = [[i, 1, 9600, 0, 0] for i in range(8)]
    assert choose(segs, 16, 2, 148) == (1152, 9)


def test_one_sm_takes_one_split_a_stream():
    """On one SM the finish time is the sum of all costs: the fewest CTAs
    win, one split a stream (the first candidate at or past 5,000 keys)."""
    assert choose([[0, 3, 5000, 0, 0], [3, 2, 700, 0, 0]], 8, 2, 1) == (5120, 1)


def test_many_sms_take_the_smallest_split():
    """With an SM for every CTA the longest CTA sets the time: 256 keys."""
    assert choose([[0, 1, 20000, 0, 0]], 8, 8, 100000) == (256, 79)


def test_batches_too_large_to_simulate_take_one_split_a_stream():
    """65,535 one-row streams x 8 kv-heads is 524,280 CTAs even at one split a
    stream, past the 2^18 the call simulates: it returns the first candidate
    holding the longest stream (1,000 keys -> 1,024) without simulating."""
    segs = np.zeros((65535, 5), np.int32)
    segs[:, 0] = np.arange(65535)
    segs[:, 1] = 1
    segs[:, 2] = 1000
    segs[7, 2] = 900
    assert choose(segs, 8, 8, 148) == (1024, 1)


def test_an_sm_count_past_the_grid_costs_nothing():
    """More SMs than CTAs: each CTA has its own SM whatever the count, so
    2^31 - 1 SMs answer like 100,000 (and allocate nothing of that size)."""
    segs = [[0, 1, 20000, 0, 0], [1, 4, 3000, 0, 0]]
    assert choose(segs, 8, 8, 2**31 - 1) == choose(segs, 8, 8, 100000)


def test_short_and_empty_batches():
    assert choose([[0, 1, 100, 0, 0]], 8, 2, 148) == (256, 1)
    assert choose(np.zeros((0, 5)), 8, 2, 148) == (256, 1)
    assert choose([[0, 0, 5000, 0, 0]], 8, 2, 148) == (256, 1)  # a stream with no rows is ignored
    # a stream with no rows does not count toward the longest stream
    assert choose([[0, 0, 90000, 0, 0], [0, 1, 300, 0, 0]], 8, 2, 1)[1] == 1


@pytest.mark.parametrize("seed,hq,hkv,n_sms", [(0, 16, 2, 148), (1, 32, 8, 148), (2, 8, 1, 20), (3, 64, 4, 148),
                                               (4, 16, 16, 7)])
def test_the_choice_is_the_earliest_finish(seed, hq, hkv, n_sms):
    """Random batches: the returned split finishes no later than any other
    candidate under the stated schedule, is the largest such, and its
    n_splits_max covers the longest stream."""
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 12))
    segs = [[0, int(rng.integers(0, 20)), int(rng.integers(1, 20000)), 0, 0] for _ in range(n)]
    segs[0][1] = max(segs[0][1], 1)
    split, n_sp = choose(segs, hq, hkv, n_sms)
    max_keys = max(s[2] for s in segs if s[1] > 0)
    times = {s: makespan(segs, hq, hkv, s, n_sms) for s in candidates(max_keys)}
    best = min(times.values())
    assert times[split] == best
    assert split == max(s for s, t in times.items() if t == best)
    assert n_sp == -(-max_keys // split)


def test_verify_batch_goes_to_one_wave():
    """The shared-verify batch (8 streams x 1-16 rows, 16/2 heads, contexts
    2,048-16,384) on 148 SMs: every CTA in one wave."""
    b = wl.shared_verify(3)
    split, n_sp = choose(b.segs, 16, 2, 148)
    rt = 128 // 8
    ctas = sum(2 * -(-int(s[1]) // rt) * -(-int(s[2]) // split) for s in b.segs)
    assert ctas <= 148
    assert split % 128 == 0 and n_sp == -(-int(b.segs[:, 2].max()) // split)


def test_refusals():
    lib = tf.load()
    segs = np.array([[0, 1, 100, 0, 0]], np.int32)
    sp, ns = ctypes.c_int32(0), ctypes.c_int32(0)
    ptr = segs.ctypes.data_as(ctypes.c_void_p)

    def call(s=ptr, n=1, hq=8, hkv=2, d=256, sms=148, a=ctypes.byref(sp), b=ctypes.byref(ns)):
        return lib.tf_choose_split_keys(s, n, hq, hkv, d, sms, a, b)

    assert call() == 0
    assert call(s=None) == 1
    assert call(n=-1) == 1
    assert call(sms=0) == 1
    assert call(hq=0) == 1
    assert call(a=None) == 1
    assert call(b=None) == 1
    assert call(hq=9) == 4  # not a multiple of the kv-heads
    assert call(hq=24, hkv=1) == 4  # a group of 24 does not divide 128
    assert call(d=128) == 4  # two CTAs an SM: not the modelled schedule
    assert call(d=64) == 4
    bad = np.array([[0, -1, 100, 0, 0]], np.int32)
    sp.value, ns.value = -5, -6
    assert call(s=bad.ctypes.data_as(ctypes.c_void_p)) == 1
    assert (sp.value, ns.value) == (-5, -6)  # outputs are written only on success
    with pytest.raises(binding.TfError):
        choose(segs, 8, 3, 148)
