/*
 * tfpaged.h - C ABI of a B200 (sm_100a) library for multi-stream attention
 * over a paged bf16 KV cache.
 *
 * Sources of the operations (TensorFold pull requests, by title and section):
 *  - #1503 "lfm2_moe CUDA: attention pages from the shared KV pool, and the
 *    prompt cache", commit list: one launch a layer over every stream's rows
 *    from a table of cache addresses, row offsets and key counts (the
 *    segment table); split-KV chunk and merge bodies over paged caches
 *    (tf_paged_attn_chunk_segs_*, tf_paged_attn_merge_segs_*); lfm2_argmax
 *    (first largest logit, ties to the lower id, nonfinite rows flagged);
 *    forward refuses rows past a slot's pages.
 *  - #1653 "spark25 CUDA: the full layers' caches in pages of the core pool",
 *    PR body: decode reads K/V through the whole page table, prompt rows
 *    through the slot's row (tf_wrows_prompt_256_p32_pg); pages of 32 and 256
 *    positions; review thread: the paged merge's nonfinite-head handling and
 *    the per-chunk page lookup hoisted out of the key loop.
 *  - #1562 "Qwen3.6 MTP drafter on CUDA: draft a shared round's streams
 *    together", PR body: many streams' rows in one launch, each over its own
 *    ring of slots (tf_q36m_attn_rows); slots stepped with a wrap, the next
 *    group of slots in flight while the current one folds.
 *
 * Conventions shared by every call:
 *  - All pointers except those named *_host are DEVICE pointers.  The caller
 *    owns every buffer; the library allocates nothing, keeps no mutable
 *    global state and never synchronizes: work is enqueued on `stream`
 *    (NULL = the legacy default stream) and the call returns.
 *  - bf16 data is passed as raw 16-bit patterns (`const void*`).
 *  - The return value reports host-checkable errors only (bad sizes, null
 *    pointers, unsupported shapes, misaligned buffers and, when a host copy
 *    of a table is given, table errors).  Nothing is launched when it is not
 *    TF_OK.
 *  - Errors the device finds in a table (bad segment, keys past a stream's
 *    pages, a page id outside the pool, too many splits) are OR-ed as
 *    TF_DEV_* bits into the caller's uint32 `status` word (device memory;
 *    the caller zeroes it); the affected work is skipped and, where it has
 *    outputs, flagged.  No kernel ever traps, asserts or spins unbounded.
 *  - Nonfinite data is not an error: the affected (row, head) is reported in
 *    the flags output and its output holds NaN.
 *
 * Data layout (a reading: the pages give no layout):
 *  - q:      bf16 [n_rows_total][Hq][D]
 *  - K pool: bf16 [n_pages][Hkv][page_size][D], V pool alike, separate arrays
 *  - page table: int32; stream s owns entries [pt_base, pt_base + n_pages)
 *  - q-head h reads kv-head h / (Hq / Hkv)
 *  - row i of a stream with n_rows new rows and n_keys keys sees keys
 *    [0, n_keys - n_rows + i + 1) (causal within the new rows)
 *  - partials: o f32 [n_rows_total][Hq][n_splits_max][D] (unnormalised
 *    sum e^(s - m) v), m f32 and l f32 [n_rows_total][Hq][n_splits_max]
 *    (m = max score in natural-log units, l = sum e^(s - m)), flag u8 alike.
 */
#ifndef TFPAGED_H
#define TFPAGED_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TF_API __attribute__((visibility("default")))
#else
#define TF_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t / CUstream). */
typedef struct CUstream_st *tf_stream_t;

typedef enum {
    TF_OK = 0,
    TF_ERR_ARG = 1,         /* a null pointer, a negative or inconsistent size */
    TF_ERR_PAST_PAGES = 2,  /* a host table asks for keys past a stream's pages */
    TF_ERR_BAD_PAGE = 3,    /* a host table names a page outside the pool */
    TF_ERR_UNSUPPORTED = 4, /* head dim, page size or head counts outside what is built */
    TF_ERR_CUDA = 5,        /* a launch failed (cudaGetLastError after the launch) */
    TF_ERR_ALIGN = 6,       /* a buffer is not aligned as documented */
    TF_ERR_WORKSPACE = 7    /* the workspace is smaller than the size query returns */
} tf_status;

/* Bits OR-ed into the device status word. */
#define TF_DEV_BAD_SEG 0x1u    /* a segment's rows or page range fall outside the buffers */
#define TF_DEV_PAST_PAGES 0x2u /* n_keys > n_pages * page_size (the pages' PastPages refusal) */
#define TF_DEV_BAD_PAGE 0x4u   /* a page id outside [0, n_pages of the pool) */
#define TF_DEV_SPLITS 0x8u     /* a stream needs more partials than n_splits_max */
#define TF_DEV_TIMEOUT 0x10u   /* a bounded wait inside a kernel gave up; that CTA's outputs are flagged */

/* One stream's entry in the segment table (device array, int32 fields). */
typedef struct {
    int32_t q_row;   /* first row of the stream in q / partials / out */
    int32_t n_rows;  /* its query rows this call (0 = nothing to do) */
    int32_t n_keys;  /* keys visible to its last row, its new rows included */
    int32_t pt_base; /* first entry of its pages in the page table */
    int32_t n_pages; /* how many page-table entries it owns */
} tf_seg;

/* One row's entry in a ring table (device array).  Slots [base, base+size)
 * of the ring arrays form the ring; `head` is the slot the next key will be
 * written to, and the row attends to the n_valid slots written just before
 * it, oldest first: slot_j = (head - n_valid + j) mod size. */
typedef struct {
    int64_t base;
    int32_t q_row;
    int32_t size;
    int32_t head;
    int32_t n_valid;
} tf_ring_seg;

/* One draft tree's entry in a tree table (device array, 32 bytes).  The tree
 * lives in a ring of slots [base, base + size): its window is the n_valid
 * slots before `head` (oldest first), node i (0 <= i < n_nodes) is query row
 * q_row + i and its key and value sit at slot (head + i) mod size, right
 * after the window; its parent is parents[parent_base + i], -1 for a root
 * (a child of the window's last slot), else a node index below i. */
typedef struct {
    int64_t base;
    int32_t q_row;
    int32_t size;
    int32_t head;
    int32_t n_valid;
    int32_t n_nodes;
    int32_t parent_base;
} tf_tree_seg;

enum { TF_OUT_F32 = 0, TF_OUT_BF16 = 1 };

/*
 * Split-KV partials of paged attention for every row of every stream in one
 * launch (the segment kernels of #1503, commit list; decode and verify reads
 * through the whole page table, #1653 PR body).
 *
 * Partial c of stream s covers keys [c*K, min((c+1)*K, n_keys)) where K =
 * split_keys when split_keys > 0, else K = ceil(ceil(n_keys/n_splits_max)/P)*P.
 * For each row i and q-head h it writes m, l, o over the keys of that range
 * that the row sees, and flag = a visible score, or a visible value row, or
 * o is nonfinite.  A partial holding no visible key has m = -inf, l = 0 and
 * o = 0; a slot c at or past the stream's partial count gets m = -inf, l = 0,
 * flag = 0 and its o is left unwritten.
 *
 *  q          bf16 [n_rows_total][n_q_heads][head_dim]
 *  k_pool, v_pool  bf16 [n_pages][n_kv_heads][page_size][head_dim], 16-byte aligned
 *  page_table int32 [page_table_len]
 *  segs       tf_seg [n_segs] (device);  segs_host: optional host copy of
 *             the same table; when given it is validated first (and page ids
 *             too, when page_table_host is given)
 *  scale      score scale (1/sqrt(head_dim) for plain attention)
 *  part_*     outputs as laid out above
 *  status     uint32 device word for TF_DEV_* bits (not cleared by the call)
 *
 * Supported: head_dim in {64, 128, 256}; page_size a power of two in
 * [8, 1024]; n_q_heads a multiple of n_kv_heads; q, pools 16-byte aligned.
 */
TF_API tf_status tf_paged_attn_decode(const void *q, int32_t n_rows_total, int32_t n_q_heads, const void *k_pool,
                               const void *v_pool, int32_t n_pages, int32_t page_size, int32_t n_kv_heads,
                               int32_t head_dim, const int32_t *page_table, int32_t page_table_len,
                               const tf_seg *segs, int32_t n_segs, const tf_seg *segs_host,
                               const int32_t *page_table_host, float scale, int32_t split_keys,
                               int32_t n_splits_max, float *part_o, float *part_m, float *part_l,
                               uint8_t *part_flag, uint32_t *status, tf_stream_t stream);

/*
 * tf_paged_attn_decode with the FULL rule of #1394 ("lfm2: a cheaper DSpark
 * hold", commit list: the block attention and merge kernels with a FULL
 * template flag): every row of a stream sees all of its stream's keys
 * [0, n_keys) instead of the causal count, as a drafter block (the pending
 * token and its mask tokens) attends over the context keys [0, len + 1).
 * Arguments, layouts, outputs and errors are those of tf_paged_attn_decode,
 * except that a stream may have more rows than keys (at least one key when it
 * has rows).  The partials merge with tf_attn_merge.
 */
TF_API tf_status tf_paged_attn_block(const void *q, int32_t n_rows_total, int32_t n_q_heads, const void *k_pool,
                              const void *v_pool, int32_t n_pages, int32_t page_size, int32_t n_kv_heads,
                              int32_t head_dim, const int32_t *page_table, int32_t page_table_len,
                              const tf_seg *segs, int32_t n_segs, const tf_seg *segs_host,
                              const int32_t *page_table_host, float scale, int32_t split_keys,
                              int32_t n_splits_max, float *part_o, float *part_m, float *part_l,
                              uint8_t *part_flag, uint32_t *status, tf_stream_t stream);

/*
 * One verify round's device work in one call: split-KV partials of every
 * stream (the causal count, or with `full` != 0 the FULL rule of
 * tf_paged_attn_block), their merge into out/flags, then the greedy argmax of
 * n_logit_rows logit rows into ids/id_flags.  The merge and the argmax are
 * launched as programmatic dependents of the launch before each, so their
 * launches overlap the previous kernel's tail; each still reads its inputs
 * only after the previous grid has finished.  Sources: #1394 ("lfm2: a
 * cheaper DSpark hold", commit list: a hold's attention partials take all of
 * its query rows in one wave, then merge in one, with a barrier only where a
 * step reads an earlier step's writes) and #1503 (commit list: the verify
 * rows' argmax on the GPU instead of a host scan).
 *
 * Arguments: those of tf_paged_attn_decode, tf_attn_merge (out, flags) and
 * tf_argmax_rows (logits bf16 [n_logit_rows][ld], n_cols, ids, id_flags);
 * n_logit_rows = 0 skips the argmax.  The logits are the caller's (the rows'
 * head outputs); nothing in the attention feeds them.  Every argument is
 * checked before the first launch; the result equals the three calls made
 * one after another.
 */
TF_API tf_status tf_verify_round(const void *q, int32_t n_rows_total, int32_t n_q_heads, const void *k_pool,
                                 const void *v_pool, int32_t n_pages, int32_t page_size, int32_t n_kv_heads,
                                 int32_t head_dim, const int32_t *page_table, int32_t page_table_len,
                                 const tf_seg *segs, int32_t n_segs, const tf_seg *segs_host,
                                 const int32_t *page_table_host, float scale, int32_t split_keys,
                                 int32_t n_splits_max, int32_t full, float *part_o, float *part_m, float *part_l,
                                 uint8_t *part_flag, float *out, uint8_t *flags, const void *logits,
                                 int32_t n_logit_rows, int32_t n_cols, int64_t ld, int32_t *ids, uint8_t *id_flags,
                                 uint32_t *status, tf_stream_t stream);

/*
 * A split size for tf_paged_attn_decode, tf_paged_attn_block and
 * tf_verify_round on batches of more than 8 queries a kv-head at head dim
 * 256, which the tcgen05 partial kernel serves with one CTA an SM (one CTA
 * per stream, kv-head, split and 128-query tile).  Host only: reads the
 * table, launches nothing.  Source: #1394 ("lfm2: a cheaper DSpark hold",
 * commit list: a hold's attention partials take all of its query rows in one
 * wave).
 *
 * For each candidate size S (256 to 4,096 keys by 128, then by 1,024 to
 * 16,384, then doubling, up to the first S that holds the longest stream in
 * one split) the call lists the kernel's CTAs in launch order, gives each a
 * cost of its 64-key tiles plus a fixed start-up and epilogue cost of eight
 * tiles (a CTA with no keys costs nothing), hands them in that order to
 * whichever of n_sms SMs frees first, and keeps the S whose last SM finishes
 * first (the larger S on a tie).  Grids of more than 2^18 CTAs are not
 * simulated; when no candidate's grid is that small, the call returns the
 * first S that holds the longest stream in one split (the fewest CTAs).
 * The costs model the kernel on a B200 (on a verify batch of 8 streams x
 * 1-16 rows and 2,048-16,384 keys it chose 1,280 keys, the fastest of the
 * sizes measured from 1,024 to 1,536, and one wave: 61 us against 78 us at
 * 1,024); the result is a performance choice only: every split gives the
 * same attention up to rounding.  Head dims 64 and 128 run two CTAs an SM,
 * whose overlap this schedule does not describe (on a drafter-block batch it
 * chose 2,432 keys, 13 % slower than 512), so they are refused.
 *
 *  segs_host     host segment table, n_segs entries (n_rows and n_keys are
 *                read; streams with no rows are ignored)
 *  n_q_heads, n_kv_heads, head_dim  as for tf_paged_attn_decode
 *  n_sms         the device's SM count (148 on a B200)
 *  split_keys    out: the chosen S, a multiple of 128 (256 for a batch with
 *                no rows or keys)
 *  n_splits_max  out: ceil(n_keys / S) of the longest stream with rows, >= 1
 *
 * Returns TF_OK, or TF_ERR_ARG for a null pointer, n_segs < 0, n_sms <= 0,
 * heads <= 0 or a segment with negative rows or keys, or TF_ERR_UNSUPPORTED
 * when head_dim is not 256, n_q_heads is not a multiple of n_kv_heads or 128
 * is not a multiple of the group; the outputs are written only on TF_OK.
 */
TF_API tf_status tf_choose_split_keys(const tf_seg *segs_host, int32_t n_segs, int32_t n_q_heads,
                                      int32_t n_kv_heads, int32_t head_dim, int32_t n_sms, int32_t *split_keys,
                                      int32_t *n_splits_max);

/*
 * Append each stream's new rows' keys and values into its pages: the
 * counterpart of tf_wrows_put in #1653 ("spark25 CUDA: the full layers'
 * caches in pages of the core pool", PR body: the rows kernel writes kr/vr
 * and tf_wrows_put copies them into the pages; forward refuses rows past a
 * slot's pages, PastPages).
 *
 * Row i (0 <= i < n_rows) of stream s is key j = n_keys - n_rows + i of that
 * stream (a stream's new rows are its last keys, the convention of every
 * attention call here).  For every kv-head g:
 *   k_pool[page][g][j % page_size][:] = k_rows[q_row + i][g][:], same for v,
 *   page = page_table[pt_base + j / page_size].
 * Nothing else in the pools changes.
 *
 *  k_rows, v_rows  bf16 [n_rows_total][n_kv_heads][head_dim], 16-byte aligned
 *  k_pool, v_pool  bf16 [n_pages][n_kv_heads][page_size][head_dim] (written)
 *  page_table, segs, segs_host, page_table_host, status: as for
 *             tf_paged_attn_decode; a row whose key lies past the stream's
 *             pages (TF_ERR_PAST_PAGES from the host check, TF_DEV_PAST_PAGES
 *             on the device) or whose page id is out of range
 *             (TF_ERR_BAD_PAGE / TF_DEV_BAD_PAGE) is not written.
 * Streams must not share pages for the rows they write (two writes to one
 * slot race).  Supported head dims and page sizes: as tf_paged_attn_decode.
 */
TF_API tf_status tf_kv_append(const void *k_rows, const void *v_rows, int32_t n_rows_total, void *k_pool,
                              void *v_pool, int32_t n_pages, int32_t page_size, int32_t n_kv_heads,
                              int32_t head_dim, const int32_t *page_table, int32_t page_table_len,
                              const tf_seg *segs, int32_t n_segs, const tf_seg *segs_host,
                              const int32_t *page_table_host, uint32_t *status, tf_stream_t stream);

/*
 * Fold partials into the final output (the merge bodies of #1503, commit
 * list; the nonfinite-head handling of #1653, review thread).  Per (row, head):
 * M = max m_c over partials with l_c > 0, L = sum e^(m_c - M) l_c,
 * out = sum e^(m_c - M) o_c / L; flag = OR of the partials' flags, or out
 * nonfinite, or no partial holds a key; a flagged head's out is NaN.
 * o_c is read only for partials with l_c > 0.
 *
 *  out   f32 [n_rows_total][n_q_heads][head_dim];  flags u8 [n_rows_total][n_q_heads]
 */
TF_API tf_status tf_attn_merge(const float *part_o, const float *part_m, const float *part_l, const uint8_t *part_flag,
                        int32_t n_rows_total, int32_t n_q_heads, int32_t head_dim, int32_t n_splits_max, float *out,
                        uint8_t *flags, tf_stream_t stream);

/*
 * Causal prompt chunk through one stream's page-table row (the _pg prompt
 * kernel of #1653, commit list and PR body): rows i = 0..n_rows-1 of the
 * chunk (q/out rows seg.q_row + i) attend to keys [0, n_keys - n_rows + i + 1),
 * every key already in the pool.  Scores and sums in fp32 on the tensor
 * cores; out is bf16 (out_dtype TF_OUT_BF16) or f32 [rows][Hq][D].
 * flags (nullable) u8 [rows][Hq] as for the merge; a flagged head's out is NaN.
 *
 *  seg_host  the stream's segment, in HOST memory (the chunk's size sets the grid)
 *
 * Ordering: the chunk may begin while the call before it on the stream is
 * still finishing, when that call is one of this library's attention or
 * merge calls (consecutive chunks overlap, the next filling the SMs the last
 * one's final wave leaves idle).  It reads only q, the pools and the page
 * table, which those calls never write; two such calls must not write the
 * same out rows.  After any other work on the stream (a kernel of the
 * caller's, tf_kv_append, a copy) it starts when that work has finished.
 *
 * Supported: head_dim in {64, 128, 256}; page sizes as for decode.
 */
TF_API tf_status tf_paged_attn_prompt(const void *q, int32_t n_rows_total, int32_t n_q_heads, const void *k_pool,
                               const void *v_pool, int32_t n_pages, int32_t page_size, int32_t n_kv_heads,
                               int32_t head_dim, const int32_t *page_table, int32_t page_table_len,
                               const tf_seg *seg_host, float scale, void *out, int32_t out_dtype, uint8_t *flags,
                               uint32_t *status, tf_stream_t stream);

/*
 * Attention of many rows, each over its own ring of slots, in one launch
 * (tf_q36m_attn_rows of #1562, PR body), split over the ring's valid slots
 * into partials of split_slots slots and merged into out.
 *
 *  q          bf16 [n_rows_total][n_q_heads][head_dim]
 *  ring_k, ring_v  bf16 [ring_slots_total][n_kv_heads][head_dim], 16-byte aligned
 *  rsegs      tf_ring_seg [n_segs] (device); rsegs_host: optional host copy, validated
 *  workspace  device scratch of at least tf_ring_workspace_bytes(...) bytes;
 *             it holds the partials between the partial and merge kernels,
 *             laid out per table entry, and needs no initialisation
 *  out        f32 [n_rows_total][n_q_heads][head_dim];  flags u8 [n_rows_total][n_q_heads]
 *             Only the rows the table names are written.
 *
 * Supported: head_dim in {64, 128, 256}; n_q_heads a multiple of n_kv_heads;
 * split_slots >= 16; n_splits_max >= ceil(n_valid / split_slots) for every
 * entry (else TF_DEV_SPLITS and the entry is skipped).
 */
TF_API tf_status tf_ring_attn(const void *q, int32_t n_rows_total, int32_t n_q_heads, const void *ring_k,
                              const void *ring_v, int64_t ring_slots_total, int32_t n_kv_heads, int32_t head_dim,
                              const tf_ring_seg *rsegs, int32_t n_segs, const tf_ring_seg *rsegs_host, float scale,
                              int32_t split_slots, int32_t n_splits_max, void *workspace, size_t workspace_bytes,
                              float *out, uint8_t *flags, uint32_t *status, tf_stream_t stream);

/* Workspace bytes tf_ring_attn needs for these sizes (0 on bad sizes). */
TF_API size_t tf_ring_workspace_bytes(int32_t n_segs, int32_t n_q_heads, int32_t head_dim, int32_t n_splits_max);

/*
 * Draft-tree attention over rings, many trees in one launch: the tree kernel
 * of #1562 ("Qwen3.6 MTP drafter on CUDA: draft a shared round's streams
 * together", PR body: tf_q36m_attn_tree folds ring slots in the same groups
 * and order as the two other ring kernels, and a tree checked against its
 * chains gives their results).
 * The page names the kernel only; the layout here is a reading of it.
 *
 * Node i of a tree attends, with every q-head of its row, to the tree's
 * window and then to the nodes on its path from the root down to itself;
 * no other node.  A tree that is one chain (parent of i = i - 1) gives
 * node i the ring attention of tf_ring_attn over the n_valid + i + 1 slots
 * before slot head + i + 1: the causal rule over rows written after the
 * window.
 *
 * The window and the nodes, keys [0, n_valid + n_nodes) from slot
 * (head - n_valid) mod size on, are split into partials of split_slots keys
 * that never cross the ring's end: the run before the wrap and the run after
 * it are cut apart, so a range that wraps takes one partial more than
 * ceil((n_valid + n_nodes) / split_slots).  The partials merge into out.
 *
 *  q          bf16 [n_rows_total][n_q_heads][head_dim]
 *  ring_k, ring_v  bf16 [ring_slots_total][n_kv_heads][head_dim], 16-byte
 *             aligned, ring_slots_total <= 2^31 - 65
 *  tsegs      tf_tree_seg [n_segs] (device); tsegs_host: optional host copy,
 *             validated (with parents_host, the parents too); the trees' rows
 *             must not overlap
 *  parents    int32 [n_parents] (device)
 *  workspace  device scratch of at least tf_ring_tree_workspace_bytes(...)
 *             bytes for the partials (by query row); needs no initialisation
 *  out        f32 [n_rows_total][n_q_heads][head_dim]; flags u8 [rows][Hq]
 *             (a nonfinite visible score, value or output; the head's out is
 *             NaN).  Only the trees' rows are written.
 *
 * Supported: head_dim in {64, 128, 256}; n_q_heads a multiple of n_kv_heads
 * whose group G divides 128; 1 <= n_nodes <= 64 a tree; split_slots >= 64.
 * Device-found errors: a bad entry or a parent outside [-1, node) sets
 * TF_DEV_BAD_SEG, too few partial slots TF_DEV_SPLITS; the tree's rows are
 * then flagged NaN.
 */
TF_API tf_status tf_ring_tree_attn(const void *q, int32_t n_rows_total, int32_t n_q_heads, const void *ring_k,
                                   const void *ring_v, int64_t ring_slots_total, int32_t n_kv_heads,
                                   int32_t head_dim, const tf_tree_seg *tsegs, int32_t n_segs,
                                   const tf_tree_seg *tsegs_host, const int32_t *parents, int32_t n_parents,
                                   const int32_t *parents_host, float scale, int32_t split_slots,
                                   int32_t n_splits_max, void *workspace, size_t workspace_bytes, float *out,
                                   uint8_t *flags, uint32_t *status, tf_stream_t stream);

/* Workspace bytes tf_ring_tree_attn needs (0 on bad sizes). */
TF_API size_t tf_ring_tree_workspace_bytes(int32_t n_rows_total, int32_t n_q_heads, int32_t head_dim,
                                           int32_t n_splits_max);

/*
 * tf_ring_attn for callers that cannot allocate device memory.  The pages
 * have no counterpart of this call; it exists for this library's users.
 *
 * Some callers have no workspace to give: a serving engine that hands all
 * device memory to its KV pool at start-up and keeps no allocator on the
 * decode path, or a host framework that calls this library from a plugin
 * hook where cudaMalloc, and the device-wide synchronization it can imply,
 * is not allowed.  This call keeps the partials in a scratch array that is
 * part of the library's own device image: TF_RING_NOALLOC_SCRATCH_BYTES
 * bytes that every GPU which loads the library holds until the process
 * exits.  Arguments and results are tf_ring_attn's, less the workspace.
 *
 *  - Arguments are checked as tf_ring_attn checks them, with the same
 *    verdicts; sound arguments whose tf_ring_workspace_bytes(n_segs,
 *    n_q_heads, head_dim, n_splits_max) exceeds TF_RING_NOALLOC_SCRATCH_BYTES
 *    are refused with TF_ERR_WORKSPACE.  Nothing is launched on a refusal.
 *  - Every call looks up the scratch array's address on the current device
 *    (cudaGetSymbolAddress); TF_ERR_CUDA if that fails.  The library never
 *    calls cudaMalloc, but the CUDA runtime places the array (and each
 *    kernel's code) in device memory when it loads this library's device
 *    code, which under lazy module loading (the CUDA 12 default,
 *    CUDA_MODULE_LOADING=LAZY) happens on first use.  So make one call on
 *    each device (n_segs = 0 is enough to place the array; a small real call
 *    also loads the kernels) before handing the device's memory to a pool,
 *    and before any stream capture.
 *  - Every call on a device shares the one scratch array and leaves its
 *    partials there.  Nothing in it needs to start at zero (every partial
 *    the merge reads is written first by the same call), but two calls whose
 *    kernels overlap on the GPU (different streams, no ordering between them)
 *    race on it: order them, or use tf_ring_attn with separate workspaces.
 */
#define TF_RING_NOALLOC_SCRATCH_BYTES (8u << 20)
TF_API tf_status tf_ring_attn_noalloc(const void *q, int32_t n_rows_total, int32_t n_q_heads, const void *ring_k,
                                      const void *ring_v, int64_t ring_slots_total, int32_t n_kv_heads,
                                      int32_t head_dim, const tf_ring_seg *rsegs, int32_t n_segs,
                                      const tf_ring_seg *rsegs_host, float scale, int32_t split_slots,
                                      int32_t n_splits_max, float *out, uint8_t *flags, uint32_t *status,
                                      tf_stream_t stream);

/*
 * Greedy row argmax (lfm2_argmax of #1503, commit list): for each of n_rows
 * rows of n_cols bf16 logits (row stride ld elements), ids[r] = the lowest
 * column holding the row's largest value, values compared as real numbers
 * (-0 equals +0); flags[r] = 1 and ids[r] = -1 when the row holds a NaN or
 * an infinity.  One launch; each row is split over a cluster of CTAs that
 * reduce through distributed shared memory, so no workspace is needed.
 */
TF_API tf_status tf_argmax_rows(const void *logits, int32_t n_rows, int32_t n_cols, int64_t ld, int32_t *ids,
                         uint8_t *flags, tf_stream_t stream);

/* Text of a status code (static storage). */
TF_API const char *tf_status_str(tf_status s);

/* ABI version of this header: bumped when a signature changes. */
TF_API int32_t tf_abi_version(void);

/*
 * Test hook for the bounded waits, so failure detection can be tested
 * without a fault: while on != 0, the warp-specialized and tensor-core
 * kernels launched from the calling host thread (decode, block and verify
 * partials, ring, tree and prompt calls) issue none of their loads, so the
 * waits of their other warps run out after 5 ms.  Each such launch reports
 * TF_DEV_TIMEOUT in its status word, leaves the outputs it did not reach
 * unwritten or flagged (a prompt chunk's rows come out as flagged NaN), and
 * leaves the device usable: no copy or MMA is in flight when its CTAs exit.
 * on = 0 restores normal launches.  Needed only by tests; TF_OK always.
 */
TF_API tf_status tf_wait_limit_test(int32_t on);

#ifdef __cplusplus
}
#endif

#endif /* TFPAGED_H */
