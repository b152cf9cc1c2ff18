"""Seeded synthetic inputs for paged KV-cache segment attention.

This module only draws random numbers and lays them out: bf16 query rows, a
shuffled pool of K/V pages, page tables, segment tables, rings of slots and
logit rows.  It holds none of the attention arithmetic, so both the CUDA path
and the float64 oracle can consume the same bits.

Randomness is numpy's PCG64 (``numpy.random.default_rng(seed)``).  Integer
ranges ``U{a..b}`` are inclusive at both ends.

Layouts (all C-contiguous):

* ``q``          uint16 (bf16 bits)  [rows][Hq][D]
* ``k_pool``     uint16 (bf16 bits)  [pages][Hkv][P][D]   (``v_pool`` alike)
* ``page_table`` int32  [sum of the streams' page counts]
* ``segs``       int32  [S][5] = (q_row, n_rows, n_keys, pt_base, n_pages)
* ``ring_k``     uint16 (bf16 bits)  [total slots][Hkv][D] (``ring_v`` alike)
* ``rsegs``      structured array of RING_SEG_DTYPE
* ``tsegs``      structured array of TREE_SEG_DTYPE, ``parents`` int32
* ``logits``     uint16 (bf16 bits)  [rows][ld]

The workload shapes follow the pages: many streams' rows in one launch from a
segment table (TensorFold #1503 "lfm2_moe CUDA: attention pages from the
shared KV pool", commit list, the segments commit), pages of 32 positions at
head dim 256 with a shuffled pool (TensorFold #1653 "spark25 CUDA: the full
layers' caches in pages of the core pool", PR body, Checks), a 4,200-slot ring
(TensorFold #1562 "Qwen3.6 MTP drafter on CUDA", PR body, Numbers) and
128,000-wide logit rows (TensorFold #1503, commit list, lfm2_argmax).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

SEG_FIELDS = ("q_row", "n_rows", "n_keys", "pt_base", "n_pages")

# Field order chosen so the C struct has no padding: int64 first.
RING_SEG_DTYPE = np.dtype(
    [("base", "<i8"), ("q_row", "<i4"), ("size", "<i4"), ("head", "<i4"), ("n_valid", "<i4")]
)

# A draft tree over a ring (32 bytes, no padding): node i of the tree is query
# row q_row + i, its K/V sit at slot (head + i) mod size, its parent is
# parents[parent_base + i] (-1 for a root).
TREE_SEG_DTYPE = np.dtype(
    [("base", "<i8"), ("q_row", "<i4"), ("size", "<i4"), ("head", "<i4"), ("n_valid", "<i4"), ("n_nodes", "<i4"),
     ("parent_base", "<i4")]
)

BF16_NAN = np.uint16(0x7FC0)
BF16_POS_INF = np.uint16(0x7F80)
BF16_NEG_INF = np.uint16(0xFF80)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); NaN stays NaN."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    rounded = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        rounded = np.where(nan, BF16_NAN, rounded)
    return rounded


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(rng: np.random.Generator, shape, sigma: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if sigma != 1.0:
        x *= np.float32(sigma)
    return f32_to_bf16_bits(x)


@dataclass
class PagedBatch:
    """Inputs of one paged decode / verify / prompt call."""

    q: np.ndarray
    k_pool: np.ndarray
    v_pool: np.ndarray
    page_table: np.ndarray
    segs: np.ndarray
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    page_size: int
    scale: float
    split_keys: int = 0
    n_splits_max: int = 1
    notes: dict = field(default_factory=dict)

    @property
    def n_rows_total(self) -> int:
        return int(self.q.shape[0])

    @property
    def n_pages(self) -> int:
        return int(self.k_pool.shape[0])

    def kv_bytes(self) -> int:
        """Algorithmic K+V bytes one pass reads: every visible key once per kv-head."""
        n_keys = int(self.segs[:, 2].sum()) if len(self.segs) else 0
        return n_keys * self.n_kv_heads * self.head_dim * 2 * 2


@dataclass
class RingBatch:
    """Inputs of one ring attention call."""

    q: np.ndarray
    ring_k: np.ndarray
    ring_v: np.ndarray
    rsegs: np.ndarray
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    scale: float
    split_slots: int = 512
    n_splits_max: int = 1

    @property
    def n_rows_total(self) -> int:
        return int(self.q.shape[0])

    def kv_bytes(self) -> int:
        return int(self.rsegs["n_valid"].sum()) * self.n_kv_heads * self.head_dim * 2 * 2


@dataclass
class TreeBatch:
    """Inputs of one ring tree attention call: every stream's draft tree over
    its ring (the window is the n_valid slots before the head, the nodes
    follow the head)."""

    q: np.ndarray
    ring_k: np.ndarray
    ring_v: np.ndarray
    tsegs: np.ndarray
    parents: np.ndarray
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    scale: float
    split_slots: int = 512
    n_splits_max: int = 1

    @property
    def n_rows_total(self) -> int:
        return int(self.q.shape[0])

    def kv_bytes(self) -> int:
        """Algorithmic K+V bytes: the window and every node once per kv-head."""
        keys = int(self.tsegs["n_valid"].sum() + self.tsegs["n_nodes"].sum())
        return keys * self.n_kv_heads * self.head_dim * 2 * 2


def tree_parents(kind: str, n: int, rng: np.random.Generator) -> list[int]:
    """Parent indices of an n-node tree in topological order (parent < node,
    -1 for a root): a chain, several roots (a star), a binary heap, or each
    node under a uniformly drawn earlier node or the window."""
    if kind == "chain":
        return [i - 1 for i in range(n)]
    if kind == "star":
        return [-1] * n
    if kind == "binary":
        return [(i - 1) // 2 if i > 0 else -1 for i in range(n)]
    if kind == "random":
        return [int(rng.integers(-1, i)) for i in range(n)]
    raise ValueError(kind)


TREE_KINDS = ("chain", "star", "binary", "random")


def n_splits_for(n_keys: int, split_keys: int, n_splits_max: int, page_size: int) -> int:
    """How many partials a stream of n_keys keys produces (bookkeeping only)."""
    if n_keys <= 0:
        return 0
    if split_keys > 0:
        return -(-n_keys // split_keys)
    per = -(-n_keys // n_splits_max)
    per = -(-per // page_size) * page_size
    return -(-n_keys // per)


def make_paged_batch(
    seed: int,
    rows: list[int],
    keys: list[int],
    n_q_heads: int,
    n_kv_heads: int,
    head_dim: int,
    page_size: int,
    n_pool_pages: int | None = None,
    unused: str = "normal",
    split_keys: int = 0,
    n_splits_max: int = 2,
    extra_pages: int = 0,
) -> PagedBatch:
    """Streams with ``rows[s]`` query rows over ``keys[s]`` keys each.

    Pages are drawn from a random permutation of the pool, so neighbouring keys
    of a stream sit in unrelated pages.  ``unused`` fills pages no stream owns,
    and the slots past a stream's last key, with ``"normal"`` data, ``"nan"``
    (poison: any read of them sets a nonfinite flag) or ``"zero"``.
    """
    assert len(rows) == len(keys)
    rng = np.random.default_rng(seed)
    pages_per = [-(-k // page_size) for k in keys]
    need = sum(pages_per)
    if n_pool_pages is None:
        n_pool_pages = need + extra_pages
    assert n_pool_pages >= need, "pool too small"
    perm = rng.permutation(n_pool_pages).astype(np.int32)
    page_table = perm[:need].copy()
    segs = np.zeros((len(rows), 5), dtype=np.int32)
    q_row = 0
    pt = 0
    for s, (r, k) in enumerate(zip(rows, keys)):
        segs[s] = (q_row, r, k, pt, pages_per[s])
        q_row += r
        pt += pages_per[s]
    shape = (n_pool_pages, n_kv_heads, page_size, head_dim)
    if unused == "normal":
        k_pool = normal_bf16(rng, shape)
        v_pool = normal_bf16(rng, shape)
    else:
        fill = BF16_NAN if unused == "nan" else np.uint16(0)
        k_pool = np.full(shape, fill, dtype=np.uint16)
        v_pool = np.full(shape, fill, dtype=np.uint16)
        for s in range(len(rows)):
            _, _, n_keys, base, n_pg = segs[s]
            for p in range(n_pg):
                page = page_table[base + p]
                n_live = min(page_size, n_keys - p * page_size)
                k_pool[page, :, :n_live, :] = normal_bf16(rng, (n_kv_heads, n_live, head_dim))
                v_pool[page, :, :n_live, :] = normal_bf16(rng, (n_kv_heads, n_live, head_dim))
    q = normal_bf16(rng, (q_row, n_q_heads, head_dim))
    if split_keys == 0:
        n_splits_max = max(1, n_splits_max)
    else:
        n_splits_max = max([n_splits_for(k, split_keys, n_splits_max, page_size) for k in keys] + [1])
    return PagedBatch(
        q=q,
        k_pool=k_pool,
        v_pool=v_pool,
        page_table=page_table,
        segs=segs,
        n_q_heads=n_q_heads,
        n_kv_heads=n_kv_heads,
        head_dim=head_dim,
        page_size=page_size,
        scale=1.0 / math.sqrt(head_dim),
        split_keys=split_keys,
        n_splits_max=n_splits_max,
    )


def make_ring_batch(
    seed: int,
    n_streams: int,
    ring_size: int,
    valid_lo: int,
    valid_hi: int,
    n_q_heads: int,
    n_kv_heads: int,
    head_dim: int,
    unused: str = "nan",
    split_slots: int = 512,
    heads: list[int] | None = None,
    valids: list[int] | None = None,
) -> RingBatch:
    """``n_streams`` one-row streams, each with its own ring of ``ring_size`` slots.

    A ring's write head is the slot the next key goes to; its ``n_valid``
    readable slots are the ones written just before the head, oldest first, so
    a head below ``n_valid`` makes the read wrap.  Slots outside the readable
    window hold ``unused`` data (NaN poison by default).
    """
    rng = np.random.default_rng(seed)
    if heads is None:
        heads = [int(h) for h in rng.integers(0, ring_size, size=n_streams)]
    if valids is None:
        valids = [int(v) for v in rng.integers(valid_lo, valid_hi + 1, size=n_streams)]
    total = n_streams * ring_size
    shape = (total, n_kv_heads, head_dim)
    if unused == "normal":
        ring_k = normal_bf16(rng, shape)
        ring_v = normal_bf16(rng, shape)
    else:
        fill = BF16_NAN if unused == "nan" else np.uint16(0)
        ring_k = np.full(shape, fill, dtype=np.uint16)
        ring_v = np.full(shape, fill, dtype=np.uint16)
    rsegs = np.zeros(n_streams, dtype=RING_SEG_DTYPE)
    for s in range(n_streams):
        base = s * ring_size
        head, n = heads[s], valids[s]
        rsegs[s] = (base, s, ring_size, head, n)
        if unused != "normal":
            # the readable window: the n slots just before the head, wrapping
            start = head - n
            if start >= 0:
                spans = [(start, head)]
            else:
                spans = [(ring_size + start, ring_size), (0, head)]
            for a, b in spans:
                if b > a:
                    ring_k[base + a : base + b] = normal_bf16(rng, (b - a, n_kv_heads, head_dim))
                    ring_v[base + a : base + b] = normal_bf16(rng, (b - a, n_kv_heads, head_dim))
    q = normal_bf16(rng, (n_streams, n_q_heads, head_dim))
    n_splits_max = max(-(-v // split_slots) for v in valids)
    return RingBatch(
        q=q,
        ring_k=ring_k,
        ring_v=ring_v,
        rsegs=rsegs,
        n_q_heads=n_q_heads,
        n_kv_heads=n_kv_heads,
        head_dim=head_dim,
        scale=1.0 / math.sqrt(head_dim),
        split_slots=split_slots,
        n_splits_max=n_splits_max,
    )


def make_tree_batch(
    seed: int,
    n_streams: int,
    ring_size: int,
    valid_lo: int,
    valid_hi: int,
    nodes_lo: int,
    nodes_hi: int,
    n_q_heads: int,
    n_kv_heads: int,
    head_dim: int,
    unused: str = "nan",
    split_slots: int = 512,
    kinds: list[str] | None = None,
    heads: list[int] | None = None,
    valids: list[int] | None = None,
    nodes: list[int] | None = None,
) -> TreeBatch:
    """``n_streams`` draft trees, each over its own ring of ``ring_size`` slots.

    A ring's write head is drawn at random; its window is the ``n_valid`` slots
    before the head (U{valid_lo..valid_hi}), and the tree's ``n_nodes``
    (U{nodes_lo..nodes_hi}) nodes are written at the head and the slots after
    it, so the window and the nodes wrap whenever they pass the ring's end.
    Tree shapes cycle through chain, star, binary and random unless ``kinds``
    is given.  Slots outside the window and the nodes hold ``unused`` data.
    """
    rng = np.random.default_rng(seed)
    if heads is None:
        heads = [int(h) for h in rng.integers(0, ring_size, size=n_streams)]
    if nodes is None:
        nodes = [int(n) for n in rng.integers(nodes_lo, nodes_hi + 1, size=n_streams)]
    if valids is None:
        valids = [int(v) for v in rng.integers(valid_lo, valid_hi + 1, size=n_streams)]
    valids = [min(v, ring_size - n) for v, n in zip(valids, nodes)]
    if kinds is None:
        kinds = [TREE_KINDS[s % len(TREE_KINDS)] for s in range(n_streams)]
    total = n_streams * ring_size
    shape = (total, n_kv_heads, head_dim)
    if unused == "normal":
        ring_k = normal_bf16(rng, shape)
        ring_v = normal_bf16(rng, shape)
    else:
        fill = BF16_NAN if unused == "nan" else np.uint16(0)
        ring_k = np.full(shape, fill, dtype=np.uint16)
        ring_v = np.full(shape, fill, dtype=np.uint16)
    tsegs = np.zeros(n_streams, dtype=TREE_SEG_DTYPE)
    parents: list[int] = []
    q_row = 0
    for s in range(n_streams):
        base = s * ring_size
        head, n, t = heads[s], valids[s], nodes[s]
        tsegs[s] = (base, q_row, ring_size, head, n, t, len(parents))
        parents += tree_parents(kinds[s], t, rng)
        q_row += t
        if unused != "normal":
            # the window before the head and the nodes from the head on
            for j in range(-n, t):
                slot = (head + j) % ring_size
                ring_k[base + slot] = normal_bf16(rng, (n_kv_heads, head_dim))
                ring_v[base + slot] = normal_bf16(rng, (n_kv_heads, head_dim))
    q = normal_bf16(rng, (q_row, n_q_heads, head_dim))
    keys = [v + t for v, t in zip(valids, nodes)]
    # a split never crosses the ring's end, so a wrapping range takes one more
    n_splits_max = max(-(-k // split_slots) + 1 for k in keys)
    return TreeBatch(
        q=q,
        ring_k=ring_k,
        ring_v=ring_v,
        tsegs=tsegs,
        parents=np.asarray(parents, np.int32),
        n_q_heads=n_q_heads,
        n_kv_heads=n_kv_heads,
        head_dim=head_dim,
        scale=1.0 / math.sqrt(head_dim),
        split_slots=split_slots,
        n_splits_max=n_splits_max,
    )


def make_logits(
    seed: int,
    n_rows: int,
    n_cols: int,
    sigma: float = 1.0,
    ld: int | None = None,
    tie_rows: list[int] | None = None,
    nan_rows: list[int] | None = None,
    posinf_rows: list[int] | None = None,
    neginf_rows: list[int] | None = None,
    tie_before: bool = False,
) -> np.ndarray:
    """bf16 logit rows ~N(0, sigma), with planted ties and nonfinite values.

    A tie row copies its largest value to a second column: a later column by
    default, an earlier one with ``tie_before`` (then the copy is the first
    occurrence, and the answer moves to it).
    """
    rng = np.random.default_rng(seed)
    ld = n_cols if ld is None else ld
    out = np.zeros((n_rows, ld), dtype=np.uint16)
    out[:, :n_cols] = normal_bf16(rng, (n_rows, n_cols), sigma)
    vals = bf16_bits_to_f32(out[:, :n_cols])
    for r in tie_rows or []:
        j = int(np.argmax(vals[r]))
        if tie_before:
            k = int(rng.integers(0, j)) if j > 0 else None
        else:
            k = int(rng.integers(j + 1, n_cols)) if j + 1 < n_cols else None
        if k is not None:
            out[r, k] = out[r, j]
    for rows_, bits in ((nan_rows, BF16_NAN), (posinf_rows, BF16_POS_INF), (neginf_rows, BF16_NEG_INF)):
        for r in rows_ or []:
            out[r, int(rng.integers(0, n_cols))] = bits
    if ld > n_cols:
        out[:, n_cols:] = BF16_NAN  # padding past the row is never read
    return out


# --------------------------------------------------------------------------
# The five workloads.  Sizes are the ones the pages' problem statement fixes;
# each is generated from its own seed.
# --------------------------------------------------------------------------


def tiny_decode(seed: int = 1, unused: str = "normal") -> PagedBatch:
    """2 one-row streams over 37 and 70 keys; 8/2 heads, D 64, pages of 16,
    a 16-page shuffled pool; two partials a stream, then a merge."""
    return make_paged_batch(
        seed, rows=[1, 1], keys=[37, 70], n_q_heads=8, n_kv_heads=2, head_dim=64,
        page_size=16, n_pool_pages=16, unused=unused, split_keys=0, n_splits_max=2,
    )


def tiny_argmax(seed: int = 1, tie_before: bool = False) -> np.ndarray:
    """4 rows x 1,000 bf16 ~N(0,1): row 1 with a planted tie, row 2 with a NaN."""
    return make_logits(seed, 4, 1000, 1.0, tie_rows=[1], nan_rows=[2], tie_before=tie_before)


def multi_stream_decode(seed: int = 2, n_streams: int = 16, unused: str = "nan") -> PagedBatch:
    """16 one-row streams, contexts U{1,024..8,192}; 32/8 heads, D 128, pages
    of 32 in a shuffled pool of 8,192 pages; 512-key partials + merge."""
    rng = np.random.default_rng(seed + 1000)
    keys = [int(k) for k in rng.integers(1024, 8192 + 1, size=n_streams)]
    return make_paged_batch(
        seed, rows=[1] * n_streams, keys=keys, n_q_heads=32, n_kv_heads=8, head_dim=128,
        page_size=32, n_pool_pages=8192, unused=unused, split_keys=512,
    )


def shared_verify(seed: int = 3, n_streams: int = 8, unused: str = "nan", plant: bool = True,
                  key_lo: int = 2048, key_hi: int = 16384, split_keys: int = 1024) -> PagedBatch:
    """8 streams with U{1..16} rows each, causal within their new rows;
    contexts U{2,048..16,384}; 16/2 heads, D 256, pages of 32, shuffled pool.

    Two (row, q-head) pairs get a +Inf planted in one element of q, so their
    scores go nonfinite and exactly those two heads must be flagged.
    """
    rng = np.random.default_rng(seed + 1000)
    rows = [int(r) for r in rng.integers(1, 16 + 1, size=n_streams)]
    keys = [int(k) for k in rng.integers(key_lo, key_hi + 1, size=n_streams)]
    keys = [max(k, r) for k, r in zip(keys, rows)]
    b = make_paged_batch(
        seed, rows=rows, keys=keys, n_q_heads=16, n_kv_heads=2, head_dim=256,
        page_size=32, unused=unused, split_keys=split_keys, extra_pages=64,
    )
    if plant:
        total = b.n_rows_total * b.n_q_heads
        picks = rng.choice(total, size=2, replace=False)
        planted = []
        for p in picks:
            row, h = divmod(int(p), b.n_q_heads)
            d = int(rng.integers(0, b.head_dim))
            b.q[row, h, d] = BF16_POS_INF
            planted.append((row, h))
        b.notes["planted"] = planted
    return b


def verify_logits(seed: int, n_rows: int, n_cols: int = 128000) -> np.ndarray:
    """Every verify row's logits ~N(0, sigma 3), ties planted in about a quarter of the rows."""
    rng = np.random.default_rng(seed + 2000)
    tie_rows = [r for r in range(n_rows) if rng.random() < 0.25]
    return make_logits(seed + 3000, n_rows, n_cols, 3.0, tie_rows=tie_rows)


def long_prompt(seed: int = 4, n_tokens: int = 15000, chunk: int = 2048) -> tuple[PagedBatch, list[tuple[int, int]]]:
    """One stream's 15,000-token prompt, every key already in 469 shuffled pages
    of 32; 16/4 heads, D 256.  Returns the batch (segment = whole prompt) and
    the chunk spans [(row0, row1), ...] of 2,048 rows each."""
    b = make_paged_batch(
        seed, rows=[n_tokens], keys=[n_tokens], n_q_heads=16, n_kv_heads=4, head_dim=256,
        page_size=32, unused="nan", split_keys=0, n_splits_max=1,
    )
    spans = [(a, min(a + chunk, n_tokens)) for a in range(0, n_tokens, chunk)]
    return b, spans


def prompt_chunk_seg(b: PagedBatch, row0: int, row1: int) -> np.ndarray:
    """Segment of the chunk of rows [row0, row1) of a one-stream prompt: the
    chunk ends at key row1, and its rows are q/out rows row0.. (bookkeeping)."""
    s = b.segs[0]
    return np.array([row0, row1 - row0, row1, s[3], -(-row1 // b.page_size)], dtype=np.int32)


def drafter_trees(seed: int = 6, n_streams: int = 17, unused: str = "nan", split_slots: int = 768) -> TreeBatch:
    """17 streams, each a draft tree of U{4..16} nodes (chain, star, binary
    and random shapes in turn) after a window of U{1,000..4,184} slots of its
    own 4,200-slot ring; 16/2 heads, D 256."""
    return make_tree_batch(
        seed, n_streams=n_streams, ring_size=4200, valid_lo=1000, valid_hi=4184, nodes_lo=4, nodes_hi=16,
        n_q_heads=16, n_kv_heads=2, head_dim=256, unused=unused, split_slots=split_slots,
    )


def drafter_ring(seed: int = 5, n_streams: int = 17, unused: str = "nan", split_slots: int = 320) -> RingBatch:
    """17 one-row streams, each over its own ring of 4,200 slots with a random
    write head; valid counts U{1,000..4,200}; 16/2 heads, D 256."""
    return make_ring_batch(
        seed, n_streams=n_streams, ring_size=4200, valid_lo=1000, valid_hi=4200,
        n_q_heads=16, n_kv_heads=2, head_dim=256, unused=unused, split_slots=split_slots,
    )
