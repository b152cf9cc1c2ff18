"""GPU parity at the edges of the supported shapes: large pages with splits
that start inside a page, more queries a kv-head than one 128-query tile,
more streams than the warp-specialized kernel's table holds, and prompt tiles
of few rows (large GQA groups)."""
import numpy as np
import pytest
import torch

from paged_kv_cache_segment_b200 import workloads as wl
from _gpu import check_prompt_bf16, compare_attn, prompt_bf16_bound, run_decode, run_prompt_chunks

pytestmark = pytest.mark.gpu


def oracle_paged(orc, b, full=False):
    return orc.paged_attn(b.q, b.k_pool, b.v_pool, b.page_table, b.segs, b.scale, full=full)


@pytest.mark.parametrize("rows,hq,hkv,d,p,split", [
    ([1, 1, 1], 8, 2, 128, 256, 512),     # warp-specialized kernel, pages of 256
    ([12, 3], 16, 2, 256, 1024, 512),     # tcgen05 partials: splits start in the middle of a 1,024-key page
    ([5, 9], 16, 4, 64, 512, 192),        # tcgen05 partials, 192-key splits (3 tiles) across pages of 512
    ([2, 9], 8, 2, 128, 1024, 96),        # general kernel (split not a multiple of 64)
])
def test_large_pages(orc, rows, hq, hkv, d, p, split):
    keys = [max(r, k) for r, k in zip(rows, [2500, 1100, 700])]
    b = wl.make_paged_batch(60 + p + d, rows=rows, keys=keys, n_q_heads=hq, n_kv_heads=hkv, head_dim=d,
                            page_size=p, unused="nan", split_keys=split, extra_pages=2)
    r = run_decode(b)
    assert r["status"] == 0
    ref, rf = oracle_paged(orc, b)
    assert not rf.any()
    compare_attn(r["out"], r["flags"], ref, rf, what=f"P{p} split {split}")


@pytest.mark.parametrize("rows,hq,hkv", [([20, 7], 16, 2), ([9], 32, 2)])
def test_more_queries_than_a_tile(orc, rows, hq, hkv):
    """20 rows x 8 q-heads = 160 and 9 x 16 = 144 queries a kv-head: two
    128-query tiles of the tcgen05 partial kernel per (stream, kv-head, split)."""
    keys = [1500, 900][:len(rows)]
    b = wl.make_paged_batch(71 + hq, rows=rows, keys=keys, n_q_heads=hq, n_kv_heads=hkv, head_dim=128, page_size=32,
                            unused="nan", split_keys=256)
    r = run_decode(b)
    assert r["status"] == 0
    ref, rf = oracle_paged(orc, b)
    compare_attn(r["out"], r["flags"], ref, rf, what="two query tiles")
    r = run_decode(b, block=True)
    ref, rf = oracle_paged(orc, b, full=True)
    compare_attn(r["out"], r["flags"], ref, rf, what="two query tiles, FULL")


def test_many_streams(orc):
    """300 one-row streams: past the warp-specialized kernel's table (256
    streams at head dim 128), so the general kernel takes them."""
    rng = np.random.default_rng(5)
    keys = [int(x) for x in rng.integers(1, 400, 300)]
    b = wl.make_paged_batch(81, rows=[1] * 300, keys=keys, n_q_heads=8, n_kv_heads=2, head_dim=128, page_size=16,
                            unused="nan", split_keys=128)
    r = run_decode(b)
    assert r["status"] == 0
    ref, rf = oracle_paged(orc, b)
    compare_attn(r["out"], r["flags"], ref, rf, what="300 streams")


@pytest.mark.parametrize("hq,hkv,d,p,n,chunk", [(16, 1, 64, 16, 300, 100), (128, 1, 64, 8, 40, 40)])
def test_prompt_large_groups(orc, hq, hkv, d, p, n, chunk):
    """Groups of 16 and 128 q-heads: 8 rows and 1 row a 128-query tile."""
    spans = [(a, min(a + chunk, n)) for a in range(0, n, chunk)]
    b = wl.make_paged_batch(90 + hq, rows=[n], keys=[n], n_q_heads=hq, n_kv_heads=hkv, head_dim=d, page_size=p,
                            unused="nan")
    ref, rf = oracle_paged(orc, b)
    r = run_prompt_chunks(b, spans, out_dtype=torch.float32)
    assert r["status"] == 0
    compare_attn(r["out"], r["flags"], ref, rf, what=f"prompt G{hq // hkv} f32")
    r = run_prompt_chunks(b, spans, out_dtype=torch.bfloat16)
    assert r["status"] == 0
    check_prompt_bf16(r["out"], r["flags"], ref, rf, prompt_bf16_bound(b, ref), what=f"prompt G{hq // hkv} bf16")
