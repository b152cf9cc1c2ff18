/*
 * oracle.c - plain float64 CPU oracle for multi-stream attention over a paged
 * bf16 KV cache, its split/merge form, the ring-of-slots variant and the
 * greedy row argmax.
 *
 * TEST INFRASTRUCTURE.  This library defines what the CUDA path must compute;
 * it is not part of that path.  Only the tests, the package's smoke check and
 * the benchmark's CPU-baseline leg may load it.  It shares no code, header,
 * table or helper with the CUDA library.
 *
 * Every function is the textbook definition written out in float64: bf16
 * inputs are widened exactly, scores are full dot products, the softmax is
 * exp(s - max) / sum, and nothing is blocked, fused or reordered.  OpenMP only
 * spreads independent (row, head) units over host cores.
 *
 * Sources (TensorFold pull requests; page title, then section):
 *  [SEG]  #1503 "lfm2_moe CUDA: attention pages from the shared KV pool, and
 *         the prompt cache", commit list: one launch a layer over every row
 *         from a table of the streams' cache addresses, row offsets and key
 *         counts, checked against float64 attention.
 *  [CHUNK] #1503, commit list: the shared-window chunk and merge bodies
 *         (tf_paged_attn_chunk_segs_*, tf_paged_attn_merge_segs_*).
 *  [POOL] #1503, commit list: keys and values read through a slot's page
 *         table; forward refuses rows past a slot's pages.
 *  [PG]   #1653 "spark25 CUDA: the full layers' caches in pages of the core
 *         pool", PR body: decode reads through the whole table, prompt rows
 *         through the slot's row; pages of 256 and of 32 positions.
 *  [FULL] #1394 "lfm2: a cheaper DSpark hold", commit list: the FULL flag
 *         gives every block row the keys [0, len + 1); the target's own
 *         kernels keep their causal count.
 *  [NF]   #1653, review thread: the paged merge's handling of a nonfinite
 *         head (the sentence is cut off on the page).
 *  [RING] #1562 "Qwen3.6 MTP drafter on CUDA: draft a shared round's streams
 *         together", PR body: each row reads its own stream's ring, slots and
 *         segment from a table; slots are stepped with a wrap.
 *  [ARG]  #1503, commit list: lfm2_argmax picks each row's first largest
 *         logit, ties to the lower id, and flags a row with a nonfinite logit.
 *  [WR]   #1653, PR body: the rows kernel writes a stream's new K/V rows and
 *         tf_wrows_put copies them into the stream's pages; forward refuses
 *         rows past a slot's pages (PastPages).
 *  [TREE] #1562, PR body: tf_q36m_attn_tree folds ring slots like the other
 *         two ring kernels, and a tree checked against the chains it is
 *         made of gives their results.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - pool layout [page][kv_head][slot][D], K and V in separate arrays;
 *  - row i of a stream with R new rows and N keys sees keys [0, N - R + i + 1);
 *  - q-head h reads kv-head h / (Hq / Hkv);
 *  - a ring's head is the next slot to be written; its n readable slots are
 *    the n before the head, oldest first: slot_j = (head - n + j) mod size;
 *  - a (row, head) is flagged when a score or the output is nonfinite; its
 *    output is then NaN;
 *  - an argmax row holding a NaN or an infinity is flagged and gets id -1;
 *  - a draft tree's nodes sit in the ring right after its head, node i at
 *    slot head + i; node i sees the window, then its ancestors from the root
 *    down, then itself (a chain is then the causal rule over rows written
 *    after the window).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_OK = 0, ORC_ERR_ARG = 1, ORC_ERR_PAST_PAGES = 2, ORC_ERR_BAD_PAGE = 3, ORC_ERR_NOMEM = 4 };

/* A ring entry: slots [base, base + size) of the ring arrays belong to it.
 * Same field order as the library's struct (int64 first, no padding), since
 * both must read one table. */
typedef struct {
    int64_t base;
    int32_t q_row, size, head, n_valid;
} orc_ring_seg;

/* A tree entry over a ring: the ring is slots [base, base + size); the
 * window is the n_valid slots before `head`; node i (0 <= i < n_nodes) is
 * query row q_row + i, its key and value sit at slot (head + i) mod size, and
 * its parent is parents[parent_base + i] (-1 for a root, else a smaller node
 * index).  Same field order as the library's struct (32 bytes, no padding). */
typedef struct {
    int64_t base;
    int32_t q_row, size, head, n_valid, n_nodes, parent_base;
} orc_tree_seg;

/* Exact widening of a bf16 bit pattern. */
static double bf(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Gather keys [0, n_keys) of one stream into dense arrays kd, vd of shape
 * [n_keys][Hkv][D]: key j lives in page page_table[pt_base + j / P] at slot
 * j % P ([POOL], [PG]).  Returns ORC_ERR_PAST_PAGES when the stream's pages
 * cannot hold n_keys keys and ORC_ERR_BAD_PAGE for a page id outside the pool.
 */
int orc_gather_paged(const uint16_t *k_pool, const uint16_t *v_pool, int32_t n_pages, int32_t page_size,
                     int32_t n_kv_heads, int32_t head_dim, const int32_t *page_table, int32_t pt_base,
                     int32_t n_stream_pages, int32_t n_keys, double *kd, double *vd)
{
    if (n_keys < 0 || page_size <= 0) return ORC_ERR_ARG;
    if ((int64_t)n_keys > (int64_t)n_stream_pages * page_size) return ORC_ERR_PAST_PAGES;
    for (int32_t j = 0; j < n_keys; ++j) {
        int32_t page = page_table[pt_base + j / page_size];
        int32_t slot = j % page_size;
        if (page < 0 || page >= n_pages) return ORC_ERR_BAD_PAGE;
        for (int32_t g = 0; g < n_kv_heads; ++g) {
            int64_t src = (((int64_t)page * n_kv_heads + g) * page_size + slot) * head_dim;
            int64_t dst = ((int64_t)j * n_kv_heads + g) * head_dim;
            for (int32_t d = 0; d < head_dim; ++d) {
                kd[dst + d] = bf(k_pool[src + d]);
                vd[dst + d] = bf(v_pool[src + d]);
            }
        }
    }
    return ORC_OK;
}

/*
 * Softmax attention of one query vector over keys [0, n_vis) of kv-head g of
 * dense K/V [n][Hkv][D]: s_j = scale * <q, K_j>, out = sum_j e^(s_j - max) V_j
 * / sum_j e^(s_j - max).  flag = some s_j or some out_d is nonfinite; a
 * flagged output is NaN.
 */
static void attend(const double *qv, const double *kd, const double *vd, int32_t n_kv_heads, int32_t head_dim,
                   int32_t g, int32_t n_vis, double scale, double *s, double *out, uint8_t *flag)
{
    int bad = 0;
    for (int32_t j = 0; j < n_vis; ++j) {
        const double *kj = kd + ((int64_t)j * n_kv_heads + g) * head_dim;
        double dot = 0.0;
        for (int32_t d = 0; d < head_dim; ++d) dot += qv[d] * kj[d];
        s[j] = scale * dot;
        if (!isfinite(s[j])) bad = 1;
    }
    double mx = -INFINITY;
    for (int32_t j = 0; j < n_vis; ++j)
        if (s[j] > mx) mx = s[j];
    double denom = 0.0;
    for (int32_t j = 0; j < n_vis; ++j) denom += exp(s[j] - mx);
    for (int32_t d = 0; d < head_dim; ++d) out[d] = 0.0;
    for (int32_t j = 0; j < n_vis; ++j) {
        double p = exp(s[j] - mx) / denom;
        const double *vj = vd + ((int64_t)j * n_kv_heads + g) * head_dim;
        for (int32_t d = 0; d < head_dim; ++d) out[d] += p * vj[d];
    }
    for (int32_t d = 0; d < head_dim; ++d)
        if (!isfinite(out[d])) bad = 1;
    if (n_vis <= 0) bad = 1;
    if (bad)
        for (int32_t d = 0; d < head_dim; ++d) out[d] = NAN;
    *flag = (uint8_t)bad;
}

/*
 * Paged attention for every row of every segment ([SEG], [POOL], [PG]).
 * segs is int32 [n_segs][5] = (q_row, n_rows, n_keys, pt_base, n_pages).
 * Row i of a segment sees keys [0, n_keys - n_rows + i + 1) (the causal
 * count; with full != 0 every row sees all n_keys keys, as [FULL]).
 * q-head h reads kv-head h / (Hq / Hkv).
 * sel (nullable) is uint8 [n_rows_total][Hq]: only marked (row, head) pairs
 * are computed; out is float64 [n_rows_total][Hq][D], flags uint8 [rows][Hq].
 */
int orc_paged_attn(const uint16_t *q, int32_t n_rows_total, int32_t n_q_heads, const uint16_t *k_pool,
                   const uint16_t *v_pool, int32_t n_pages, int32_t page_size, int32_t n_kv_heads, int32_t head_dim,
                   const int32_t *page_table, int32_t pt_len, const int32_t *segs, int32_t n_segs, double scale,
                   int32_t full, const uint8_t *sel, double *out, uint8_t *flags)
{
    if (n_kv_heads <= 0 || n_q_heads % n_kv_heads != 0) return ORC_ERR_ARG;
    const int32_t group = n_q_heads / n_kv_heads;
    for (int32_t s = 0; s < n_segs; ++s) {
        const int32_t q_row = segs[5 * s + 0], n_rows = segs[5 * s + 1], n_keys = segs[5 * s + 2];
        const int32_t pt_base = segs[5 * s + 3], n_pg = segs[5 * s + 4];
        /* the causal count needs a key per row; a FULL block row needs one key */
        const int32_t keys_needed = full ? (n_rows > 0 ? 1 : 0) : n_rows;
        if (q_row < 0 || n_rows < 0 || q_row + n_rows > n_rows_total || n_keys < keys_needed || pt_base < 0 ||
            n_pg < 0 || pt_base + n_pg > pt_len)
            return ORC_ERR_ARG;
        if (n_rows == 0) continue;
        double *kd = (double *)malloc(sizeof(double) * ((size_t)n_keys * n_kv_heads * head_dim + 1));
        double *vd = (double *)malloc(sizeof(double) * ((size_t)n_keys * n_kv_heads * head_dim + 1));
        if (!kd || !vd) {
            free(kd);
            free(vd);
            return ORC_ERR_NOMEM;
        }
        int rc = orc_gather_paged(k_pool, v_pool, n_pages, page_size, n_kv_heads, head_dim, page_table, pt_base,
                                  n_pg, n_keys, kd, vd);
        if (rc != ORC_OK) {
            free(kd);
            free(vd);
            return rc;
        }
        const int64_t units = (int64_t)n_rows * n_q_heads;
#pragma omp parallel
        {
            double *qv = (double *)malloc(sizeof(double) * head_dim);
            double *sc = (double *)malloc(sizeof(double) * ((size_t)n_keys + 1));
#pragma omp for schedule(dynamic, 1)
            for (int64_t u = 0; u < units; ++u) {
                const int32_t i = (int32_t)(u / n_q_heads), h = (int32_t)(u % n_q_heads);
                const int64_t row = (int64_t)q_row + i;
                if (sel && !sel[row * n_q_heads + h]) continue;
                const uint16_t *qs = q + (row * n_q_heads + h) * head_dim;
                for (int32_t d = 0; d < head_dim; ++d) qv[d] = bf(qs[d]);
                const int32_t n_vis = full ? n_keys : n_keys - n_rows + i + 1;
                attend(qv, kd, vd, n_kv_heads, head_dim, h / group, n_vis, scale, sc,
                       out + (row * n_q_heads + h) * head_dim, flags + row * n_q_heads + h);
            }
            free(qv);
            free(sc);
        }
        free(kd);
        free(vd);
    }
    return ORC_OK;
}

/*
 * A stream's new rows into its pages ([WR]).  Row i of segment s is the
 * stream's key j = n_keys - n_rows + i (its new rows are its last keys); for
 * every kv-head g its K row and V row are copied to slot j % page_size of page
 * page_table[pt_base + j / page_size]:
 *     k_pool[page][g][slot][:] = k_rows[q_row + i][g][:]   (same for v).
 * Every entry is checked before anything is copied: a bad entry gives
 * ORC_ERR_ARG, a key past the stream's pages ORC_ERR_PAST_PAGES, a page id
 * out of range ORC_ERR_BAD_PAGE, and the pools are then left as they were.
 */
int orc_put_rows(const uint16_t *k_rows, const uint16_t *v_rows, int32_t n_rows_total, int32_t n_kv_heads,
                 int32_t head_dim, uint16_t *k_pool, uint16_t *v_pool, int32_t n_pages, int32_t page_size,
                 const int32_t *page_table, int32_t pt_len, const int32_t *segs, int32_t n_segs)
{
    if (n_kv_heads <= 0 || head_dim <= 0 || page_size <= 0) return ORC_ERR_ARG;
    for (int32_t s = 0; s < n_segs; ++s) {
        const int32_t q_row = segs[5 * s + 0], n_rows = segs[5 * s + 1], n_keys = segs[5 * s + 2];
        const int32_t pt_base = segs[5 * s + 3], n_pg = segs[5 * s + 4];
        if (q_row < 0 || n_rows < 0 || q_row + n_rows > n_rows_total || n_keys < n_rows || pt_base < 0 ||
            n_pg < 0 || pt_base + n_pg > pt_len)
            return ORC_ERR_ARG;
        if ((int64_t)n_keys > (int64_t)n_pg * page_size) return ORC_ERR_PAST_PAGES;
        for (int32_t i = 0; i < n_rows; ++i) {
            const int32_t j = n_keys - n_rows + i;
            const int32_t pid = page_table[pt_base + j / page_size];
            if (pid < 0 || pid >= n_pages) return ORC_ERR_BAD_PAGE;
        }
    }
    for (int32_t s = 0; s < n_segs; ++s) {
        const int32_t q_row = segs[5 * s + 0], n_rows = segs[5 * s + 1], n_keys = segs[5 * s + 2];
        const int32_t pt_base = segs[5 * s + 3];
        for (int32_t i = 0; i < n_rows; ++i) {
            const int32_t j = n_keys - n_rows + i;
            const int64_t page = page_table[pt_base + j / page_size];
            const int64_t slot = j % page_size;
            for (int32_t g = 0; g < n_kv_heads; ++g) {
                const int64_t src = ((int64_t)(q_row + i) * n_kv_heads + g) * head_dim;
                const int64_t dst = ((page * n_kv_heads + g) * page_size + slot) * head_dim;
                for (int32_t d = 0; d < head_dim; ++d) {
                    k_pool[dst + d] = k_rows[src + d];
                    v_pool[dst + d] = v_rows[src + d];
                }
            }
        }
    }
    return ORC_OK;
}

/*
 * One online-softmax partial ([CHUNK]): for one query over the keys
 * [a, b) of a stream that the query sees (j < n_vis), m = max s_j,
 * l = sum e^(s_j - m), o = sum e^(s_j - m) V_j.  An empty range gives
 * m = -inf, l = 0, o = 0.  flag = some visible score or o is nonfinite.
 * qv is float64 [D]; kd/vd dense [n][Hkv][D].
 */
void orc_partial(const double *qv, const double *kd, const double *vd, int32_t n_kv_heads, int32_t head_dim,
                 int32_t g, int32_t a, int32_t b, int32_t n_vis, double scale, double *o, double *m, double *l,
                 uint8_t *flag)
{
    int bad = 0;
    int32_t hi = b < n_vis ? b : n_vis;
    double mx = -INFINITY;
    int32_t n = hi > a ? hi - a : 0;
    double *s = (double *)malloc(sizeof(double) * ((size_t)n + 1));
    for (int32_t j = a; j < hi; ++j) {
        const double *kj = kd + ((int64_t)j * n_kv_heads + g) * head_dim;
        double dot = 0.0;
        for (int32_t d = 0; d < head_dim; ++d) dot += qv[d] * kj[d];
        s[j - a] = scale * dot;
        if (!isfinite(s[j - a])) bad = 1;
        if (s[j - a] > mx) mx = s[j - a];
    }
    double sum = 0.0;
    for (int32_t d = 0; d < head_dim; ++d) o[d] = 0.0;
    for (int32_t j = a; j < hi; ++j) {
        double p = exp(s[j - a] - mx);
        sum += p;
        const double *vj = vd + ((int64_t)j * n_kv_heads + g) * head_dim;
        for (int32_t d = 0; d < head_dim; ++d) o[d] += p * vj[d];
    }
    for (int32_t d = 0; d < head_dim; ++d)
        if (!isfinite(o[d])) bad = 1;
    free(s);
    *m = mx;
    *l = sum;
    *flag = (uint8_t)bad;
}

/*
 * Merge of C partials of one (row, head) ([CHUNK], [NF]):
 * M = max m_c over partials with l_c > 0, L = sum e^(m_c - M) l_c,
 * out = sum e^(m_c - M) o_c / L.  flag = OR of the partials' flags, or out
 * nonfinite, or no partial holds a key; a flagged output is NaN.
 * o is float64 [C][D]; m, l float64 [C]; flag uint8 [C].
 */
void orc_merge(const double *o, const double *m, const double *l, const uint8_t *flag, int32_t n_parts,
               int32_t head_dim, double *out, uint8_t *out_flag)
{
    int bad = 0, any = 0;
    double mx = -INFINITY;
    for (int32_t c = 0; c < n_parts; ++c) {
        if (flag[c]) bad = 1;
        if (l[c] > 0.0) {
            any = 1;
            if (m[c] > mx) mx = m[c];
        }
    }
    double denom = 0.0;
    for (int32_t c = 0; c < n_parts; ++c)
        if (l[c] > 0.0) denom += exp(m[c] - mx) * l[c];
    for (int32_t d = 0; d < head_dim; ++d) out[d] = 0.0;
    for (int32_t c = 0; c < n_parts; ++c) {
        if (!(l[c] > 0.0)) continue;
        double w = exp(m[c] - mx) / denom;
        for (int32_t d = 0; d < head_dim; ++d) out[d] += w * o[(int64_t)c * head_dim + d];
    }
    for (int32_t d = 0; d < head_dim; ++d)
        if (!isfinite(out[d])) bad = 1;
    if (!any) bad = 1;
    if (bad)
        for (int32_t d = 0; d < head_dim; ++d) out[d] = NAN;
    *out_flag = (uint8_t)bad;
}

/*
 * Partials of every (row, head) of a paged call, split the way the decode
 * call splits ([CHUNK]): split c of a stream covers keys [c K, (c+1) K) with
 * K = split_keys, or, when split_keys == 0, K = ceil(ceil(N / n_splits_max)
 * / P) * P.  Slots c at or past the stream's split count are empty partials
 * (m = -inf, l = 0, o = 0).  Outputs: o [rows][Hq][C][D], m, l [rows][Hq][C],
 * flag [rows][Hq][C] with C = n_splits_max.
 */
int orc_paged_partials(const uint16_t *q, int32_t n_rows_total, int32_t n_q_heads, const uint16_t *k_pool,
                       const uint16_t *v_pool, int32_t n_pages, int32_t page_size, int32_t n_kv_heads,
                       int32_t head_dim, const int32_t *page_table, int32_t pt_len, const int32_t *segs,
                       int32_t n_segs, double scale, int32_t split_keys, int32_t n_splits_max, double *po,
                       double *pm, double *pl, uint8_t *pf)
{
    if (n_kv_heads <= 0 || n_q_heads % n_kv_heads != 0 || n_splits_max <= 0) return ORC_ERR_ARG;
    const int32_t group = n_q_heads / n_kv_heads;
    for (int32_t s = 0; s < n_segs; ++s) {
        const int32_t q_row = segs[5 * s + 0], n_rows = segs[5 * s + 1], n_keys = segs[5 * s + 2];
        const int32_t pt_base = segs[5 * s + 3], n_pg = segs[5 * s + 4];
        if (q_row < 0 || n_rows < 0 || q_row + n_rows > n_rows_total || n_keys < n_rows || pt_base < 0 ||
            n_pg < 0 || pt_base + n_pg > pt_len)
            return ORC_ERR_ARG;
        if (n_rows == 0) continue;
        int32_t per = split_keys;
        if (per <= 0) {
            per = (n_keys + n_splits_max - 1) / n_splits_max;
            per = (per + page_size - 1) / page_size * page_size;
        }
        const int32_t n_sp = (n_keys + per - 1) / per;
        if (n_sp > n_splits_max) return ORC_ERR_ARG;
        double *kd = (double *)malloc(sizeof(double) * ((size_t)n_keys * n_kv_heads * head_dim + 1));
        double *vd = (double *)malloc(sizeof(double) * ((size_t)n_keys * n_kv_heads * head_dim + 1));
        if (!kd || !vd) {
            free(kd);
            free(vd);
            return ORC_ERR_NOMEM;
        }
        int rc = orc_gather_paged(k_pool, v_pool, n_pages, page_size, n_kv_heads, head_dim, page_table, pt_base,
                                  n_pg, n_keys, kd, vd);
        if (rc != ORC_OK) {
            free(kd);
            free(vd);
            return rc;
        }
        const int64_t units = (int64_t)n_rows * n_q_heads * n_splits_max;
#pragma omp parallel
        {
            double *qv = (double *)malloc(sizeof(double) * head_dim);
#pragma omp for schedule(dynamic, 4)
            for (int64_t u = 0; u < units; ++u) {
                const int32_t c = (int32_t)(u % n_splits_max);
                const int32_t h = (int32_t)((u / n_splits_max) % n_q_heads);
                const int32_t i = (int32_t)(u / ((int64_t)n_splits_max * n_q_heads));
                const int64_t row = (int64_t)q_row + i;
                const int64_t at = (row * n_q_heads + h) * n_splits_max + c;
                const uint16_t *qs = q + (row * n_q_heads + h) * head_dim;
                for (int32_t d = 0; d < head_dim; ++d) qv[d] = bf(qs[d]);
                int32_t a = c * per, b = (c + 1) * per;
                if (b > n_keys) b = n_keys;
                if (c >= n_sp) a = b = 0;
                orc_partial(qv, kd, vd, n_kv_heads, head_dim, h / group, a, b, n_keys - n_rows + i + 1, scale,
                            po + at * head_dim, pm + at, pl + at, pf + at);
            }
            free(qv);
        }
        free(kd);
        free(vd);
    }
    return ORC_OK;
}

/*
 * Ring attention ([RING]): each table entry is one query row attending, with
 * all its q-heads, to the n_valid slots written just before the ring's head,
 * oldest first: slot_j = (head - n_valid + j) mod size, read from
 * ring arrays [slots_total][Hkv][D] at base + slot_j.  No causal mask.
 * out float64 [n_rows_total][Hq][D]; flags uint8 [rows][Hq].
 */
int orc_ring_attn(const uint16_t *q, int32_t n_rows_total, int32_t n_q_heads, const uint16_t *ring_k,
                  const uint16_t *ring_v, int64_t slots_total, int32_t n_kv_heads, int32_t head_dim,
                  const orc_ring_seg *rs, int32_t n_segs, double scale, double *out, uint8_t *flags)
{
    if (n_kv_heads <= 0 || n_q_heads % n_kv_heads != 0) return ORC_ERR_ARG;
    const int32_t group = n_q_heads / n_kv_heads;
    for (int32_t s = 0; s < n_segs; ++s) {
        const orc_ring_seg e = rs[s];
        if (e.q_row < 0 || e.q_row >= n_rows_total || e.size <= 0 || e.n_valid < 1 || e.n_valid > e.size ||
            e.head < 0 || e.head >= e.size || e.base < 0 || e.base + e.size > slots_total)
            return ORC_ERR_ARG;
        const int32_t n = e.n_valid;
        double *kd = (double *)malloc(sizeof(double) * (size_t)n * n_kv_heads * head_dim);
        double *vd = (double *)malloc(sizeof(double) * (size_t)n * n_kv_heads * head_dim);
        if (!kd || !vd) {
            free(kd);
            free(vd);
            return ORC_ERR_NOMEM;
        }
        for (int32_t j = 0; j < n; ++j) {
            int32_t slot = ((e.head - n + j) % e.size + e.size) % e.size;
            for (int32_t g = 0; g < n_kv_heads; ++g)
                for (int32_t d = 0; d < head_dim; ++d) {
                    int64_t src = ((e.base + slot) * n_kv_heads + g) * head_dim + d;
                    int64_t dst = ((int64_t)j * n_kv_heads + g) * head_dim + d;
                    kd[dst] = bf(ring_k[src]);
                    vd[dst] = bf(ring_v[src]);
                }
        }
#pragma omp parallel
        {
            double *qv = (double *)malloc(sizeof(double) * head_dim);
            double *sc = (double *)malloc(sizeof(double) * (size_t)n);
#pragma omp for schedule(dynamic, 1)
            for (int32_t h = 0; h < n_q_heads; ++h) {
                const uint16_t *qs = q + ((int64_t)e.q_row * n_q_heads + h) * head_dim;
                for (int32_t d = 0; d < head_dim; ++d) qv[d] = bf(qs[d]);
                attend(qv, kd, vd, n_kv_heads, head_dim, h / group, n, scale, sc,
                       out + ((int64_t)e.q_row * n_q_heads + h) * head_dim, flags + (int64_t)e.q_row * n_q_heads + h);
            }
            free(qv);
            free(sc);
        }
        free(kd);
        free(vd);
    }
    return ORC_OK;
}

/*
 * Tree attention over a ring ([RING], [TREE]): node i of entry e sees, in this
 * order, the window slots slot_j = (head - n_valid + j) mod size for
 * j = 0..n_valid-1 (oldest first), then the nodes on its path from the root
 * down to itself, node a at slot (head + a) mod size.  The keys of that list
 * are gathered densely and attended with every q-head of row q_row + i, no
 * mask.  An entry must have n_nodes >= 1, n_valid >= 0, n_valid + n_nodes <=
 * size, and -1 <= parent < node for every node; else ORC_ERR_ARG.
 */
int orc_ring_tree_attn(const uint16_t *q, int32_t n_rows_total, int32_t n_q_heads, const uint16_t *ring_k,
                       const uint16_t *ring_v, int64_t slots_total, int32_t n_kv_heads, int32_t head_dim,
                       const orc_tree_seg *ts, int32_t n_segs, const int32_t *parents, int32_t n_parents,
                       double scale, double *out, uint8_t *flags)
{
    if (n_kv_heads <= 0 || n_q_heads % n_kv_heads != 0) return ORC_ERR_ARG;
    const int32_t group = n_q_heads / n_kv_heads;
    for (int32_t s = 0; s < n_segs; ++s) {
        const orc_tree_seg e = ts[s];
        if (e.n_nodes < 1 || e.n_valid < 0 || e.size <= 0 || (int64_t)e.n_valid + e.n_nodes > e.size ||
            e.head < 0 || e.head >= e.size || e.base < 0 || e.base + e.size > slots_total || e.q_row < 0 ||
            (int64_t)e.q_row + e.n_nodes > n_rows_total || e.parent_base < 0 ||
            (int64_t)e.parent_base + e.n_nodes > n_parents)
            return ORC_ERR_ARG;
        for (int32_t i = 0; i < e.n_nodes; ++i) {
            const int32_t par = parents[e.parent_base + i];
            if (par < -1 || par >= i) return ORC_ERR_ARG;
        }
    }
    for (int32_t s = 0; s < n_segs; ++s) {
        const orc_tree_seg e = ts[s];
        const int64_t per_key = (int64_t)n_kv_heads * head_dim;
        const int32_t cap = e.n_valid + e.n_nodes;
        const int64_t units = (int64_t)e.n_nodes * n_q_heads;
        int bad_alloc = 0;
#pragma omp parallel
        {
            double *kd = (double *)malloc(sizeof(double) * (size_t)(cap * per_key));
            double *vd = (double *)malloc(sizeof(double) * (size_t)(cap * per_key));
            double *qv = (double *)malloc(sizeof(double) * head_dim);
            double *sc = (double *)malloc(sizeof(double) * (size_t)cap);
            int32_t *path = (int32_t *)malloc(sizeof(int32_t) * (size_t)e.n_nodes);
            if (!kd || !vd || !qv || !sc || !path) {
#pragma omp atomic write
                bad_alloc = 1;
            }
#pragma omp for schedule(dynamic, 1)
            for (int64_t u = 0; u < units; ++u) {
                if (bad_alloc) continue;
                const int32_t i = (int32_t)(u / n_q_heads), h = (int32_t)(u % n_q_heads);
                /* the node's path, root first */
                int32_t depth = 0;
                for (int32_t a = i; a >= 0; a = parents[e.parent_base + a]) path[depth++] = a;
                int32_t n_keys = 0;
                for (int32_t j = 0; j < e.n_valid + depth; ++j) {
                    int32_t slot;
                    if (j < e.n_valid)
                        slot = ((e.head - e.n_valid + j) % e.size + e.size) % e.size;
                    else
                        slot = (e.head + path[depth - 1 - (j - e.n_valid)]) % e.size;
                    for (int32_t g = 0; g < n_kv_heads; ++g)
                        for (int32_t d = 0; d < head_dim; ++d) {
                            const int64_t src = ((e.base + slot) * n_kv_heads + g) * head_dim + d;
                            const int64_t dst = ((int64_t)n_keys * n_kv_heads + g) * head_dim + d;
                            kd[dst] = bf(ring_k[src]);
                            vd[dst] = bf(ring_v[src]);
                        }
                    ++n_keys;
                }
                const int64_t row = (int64_t)e.q_row + i;
                const uint16_t *qs = q + (row * n_q_heads + h) * head_dim;
                for (int32_t d = 0; d < head_dim; ++d) qv[d] = bf(qs[d]);
                attend(qv, kd, vd, n_kv_heads, head_dim, h / group, n_keys, scale, sc,
                       out + (row * n_q_heads + h) * head_dim, flags + row * n_q_heads + h);
            }
            free(kd);
            free(vd);
            free(qv);
            free(sc);
            free(path);
        }
        if (bad_alloc) return ORC_ERR_NOMEM;
    }
    return ORC_OK;
}

/*
 * Greedy row argmax ([ARG]): for each row of n_cols bf16 logits (row stride
 * ld elements), id = the lowest column holding the row's largest value,
 * comparing values as real numbers (so -0 equals +0); a row holding a NaN or
 * an infinity is flagged and gets id -1.
 */
void orc_argmax_rows(const uint16_t *logits, int32_t n_rows, int32_t n_cols, int64_t ld, int32_t *ids,
                     uint8_t *flags)
{
#pragma omp parallel for schedule(static)
    for (int32_t r = 0; r < n_rows; ++r) {
        const uint16_t *row = logits + (int64_t)r * ld;
        int bad = 0;
        int32_t best = -1;
        double best_v = 0.0;
        for (int32_t j = 0; j < n_cols; ++j) {
            double v = bf(row[j]);
            if (!isfinite(v)) {
                bad = 1;
                continue;
            }
            if (best < 0 || v > best_v) {
                best = j;
                best_v = v;
            }
        }
        ids[r] = bad ? -1 : best;
        flags[r] = (uint8_t)bad;
    }
}
