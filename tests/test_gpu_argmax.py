"""Parity of the CUDA row argmax (through the C ABI) with the oracle: ids and
flags bit-exact."""
import numpy as np
import pytest

import oracle
from paged_kv_cache_segment_b200 import workloads as wl

from _gpu import run_argmax

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


@pytest.mark.parametrize("tie_before", [False, True])
def test_tiny_argmax(orc, tie_before):
    lg = wl.tiny_argmax(1, tie_before=tie_before)
    ids, fl = run_argmax(lg)
    rid, rfl = orc.argmax_rows(lg)
    np.testing.assert_array_equal(ids, rid)
    np.testing.assert_array_equal(fl, rfl)
    assert fl.tolist() == [0, 0, 1, 0]


def test_verify_logits_full_width(orc):
    """Every verify row's 128,000 logits ~N(0, 3) with ties in about a quarter of the rows."""
    lg = wl.verify_logits(3, 68)
    ids, fl = run_argmax(lg)
    rid, rfl = orc.argmax_rows(lg)
    np.testing.assert_array_equal(ids, rid)
    np.testing.assert_array_equal(fl, rfl)


def test_planted_ties_and_nonfinite(orc):
    lg = wl.make_logits(5, 40, 128000, 3.0, tie_rows=list(range(0, 40, 2)), nan_rows=[3], posinf_rows=[5],
                        neginf_rows=[7])
    # a tie across CTA boundaries: the max copied into the first and last columns
    j = int(np.argmax(wl.bf16_bits_to_f32(lg[9])))
    lg[9, 0] = lg[9, j]
    lg[9, -1] = lg[9, j]
    ids, fl = run_argmax(lg)
    rid, rfl = orc.argmax_rows(lg)
    np.testing.assert_array_equal(ids, rid)
    np.testing.assert_array_equal(fl, rfl)
    assert ids[9] == 0 and fl[3] and fl[5] and fl[7] and ids[3] == -1


def test_signed_zero_and_constant_rows(orc):
    lg = np.full((4, 128000), 0xBF80, np.uint16)  # -1.0
    lg[0, 70000] = 0x8000  # -0.0 first
    lg[0, 90000] = 0x0000  # +0.0 ties: lower id
    lg[1, :] = 0x3F80  # all equal
    lg[2, 5] = 0x0000
    lg[2, 3] = 0x8000
    lg[3, 127999] = 0x4000  # max in the last column
    ids, fl = run_argmax(lg)
    rid, rfl = orc.argmax_rows(lg)
    np.testing.assert_array_equal(ids, rid)
    assert ids.tolist() == [70000, 0, 3, 127999]


@pytest.mark.parametrize("n_cols,ld", [(1, 1), (7, 8), (1000, 1000), (1001, 1001), (1001, 1024), (127999, 128000),
                                       (128000, 128003), (64, 64), (65, 72)])
def test_ragged_widths_and_strides(orc, n_cols, ld):
    lg = wl.make_logits(n_cols, 9, n_cols, 2.0, ld=ld, tie_rows=[1, 4])
    ids, fl = run_argmax(lg, n_cols=n_cols)
    rid, rfl = orc.argmax_rows(lg, n_cols=n_cols)
    np.testing.assert_array_equal(ids, rid)
    np.testing.assert_array_equal(fl, rfl)


def test_many_rows(orc):
    lg = wl.make_logits(11, 3000, 257, 1.0, tie_rows=list(range(0, 3000, 7)), nan_rows=[100, 2999])
    ids, fl = run_argmax(lg)
    rid, rfl = orc.argmax_rows(lg)
    np.testing.assert_array_equal(ids, rid)
    np.testing.assert_array_equal(fl, rfl)
