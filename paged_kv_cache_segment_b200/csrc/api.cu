// api.cu - the extern "C" entry points declared in include/tfpaged.h: argument
// checks on the host, then stream-ordered kernel launches.  Nothing here
// allocates device memory, synchronizes or keeps state between calls.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <functional>
#include <vector>
#include <cuda_runtime.h>

#include "tf_internal.h"

using namespace tfp;

// The timeout test hook: per host thread, so a test that turns it on touches
// no other thread's launches.
namespace tfp {
namespace {
thread_local uint64_t g_wait_runout_ns = 0;
}
uint64_t test_wait_runout_ns() { return g_wait_runout_ns; }
}  // namespace tfp

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int log2_exact(int x) {
    if (x <= 0 || (x & (x - 1))) return -1;
    int r = 0;
    while ((1 << r) < x) ++r;
    return r;
}

bool head_dim_ok(int d) { return d == 64 || d == 128 || d == 256; }

tf_status cuda_status(cudaError_t e) { return e == cudaSuccess ? TF_OK : TF_ERR_CUDA; }

int split_len(int n_keys, int split_keys, int n_splits_max, int page_size) {
    if (split_keys > 0) return split_keys;
    int per = (n_keys + n_splits_max - 1) / n_splits_max;
    return (per + page_size - 1) / page_size * page_size;
}

// Checks of a host copy of a segment table; see tf_paged_attn_decode.
tf_status check_segs_host(const tf_seg *sh, int n_segs, int n_rows_total, int page_table_len, int page_size,
                          int n_pages, const int32_t *pt_host, int split_keys, int n_splits_max, int *max_rows,
                          bool full = false) {
    int mr = 0;
    for (int s = 0; s < n_segs; ++s) {
        const tf_seg e = sh[s];
        if (e.q_row < 0 || e.n_rows < 0 || (int64_t)e.q_row + e.n_rows > n_rows_total ||
            e.n_keys < (full ? (e.n_rows > 0 ? 1 : 0) : e.n_rows) ||
            e.pt_base < 0 || e.n_pages < 0 || (int64_t)e.pt_base + e.n_pages > page_table_len)
            return TF_ERR_ARG;
        if ((int64_t)e.n_keys > (int64_t)e.n_pages * page_size) return TF_ERR_PAST_PAGES;
        if (e.n_rows > 0 && n_splits_max > 0) {
            const int per = split_len(e.n_keys, split_keys, n_splits_max, page_size);
            if ((e.n_keys + per - 1) / per > n_splits_max) return TF_ERR_ARG;
        }
        if (pt_host) {
            const int used = (e.n_keys + page_size - 1) / page_size;
            for (int k = 0; k < used; ++k) {
                const int pid = pt_host[e.pt_base + k];
                if (pid < 0 || pid >= n_pages) return TF_ERR_BAD_PAGE;
            }
        }
        if (e.n_rows > mr) mr = e.n_rows;
    }
    *max_rows = mr;
    return TF_OK;
}

tf_status ring_merge(const float *po, const float *pm, const float *pl, const uint8_t *pf, int n_segs, int n_q_heads,
                     int head_dim, int n_splits_max, int n_rows_total, const tf_ring_seg *rsegs, int split_slots,
                     int64_t ring_slots_total, float *out, uint8_t *flags, cudaStream_t st) {
    MergeParams mp{};
    mp.part_o = po;
    mp.part_m = pm;
    mp.part_l = pl;
    mp.part_flag = pf;
    mp.n_units = (int64_t)n_segs * n_q_heads;
    mp.n_parts = n_splits_max;
    mp.hq = n_q_heads;
    mp.n_rows_total = n_rows_total;
    mp.rsegs = rsegs;
    mp.split_slots = split_slots;
    mp.ring_slots_total = ring_slots_total;
    mp.out = out;
    mp.flags = flags;
    return cuda_status(launch_merge(mp, head_dim, kMergeRing, st));
}

// Cost of one CTA of the tcgen05 partial kernel at head dim 256, in 64-key tiles: its
// start-up and epilogue (tensor memory, barriers, Q, the first loads' latency,
// writing o, m, l) count as this many tiles.  Set from a sweep of split sizes
// on a verify batch (8 streams x 1-16 rows, contexts 2,048-16,384, D 256):
// values from 3 to 11 all choose the split that measured fastest there.
constexpr double kSplitCtaOverheadTiles = 8.0;
// Grids larger than this are not simulated (a batch that big fills the SMs
// many times over whatever the split), which bounds the call's host time.
constexpr int64_t kSplitMaxSimulatedCtas = (int64_t)1 << 18;

// Finish time, in tiles, of the partial kernel's grid for split size S: the
// CTAs (x = split * n_qt + query tile fastest, then kv-head, then stream) go
// in launch order to whichever SM frees first.  CTAs with no work cost 0.
double partial_makespan(const tf_seg *sh, int n_segs, int n_kv_heads, int rt, int n_qt, int S, int n_sp_max,
                        int n_sms, std::vector<double> &heap) {
    heap.assign((size_t)n_sms, 0.0);  // a min-heap of SM free times
    auto take = [&](double cost) {
        std::pop_heap(heap.begin(), heap.end(), std::greater<double>());
        heap.back() += cost;
        std::push_heap(heap.begin(), heap.end(), std::greater<double>());
    };
    for (int z = 0; z < n_segs; ++z) {
        const int T = sh[z].n_rows, N = sh[z].n_keys;
        const int n_sp = T > 0 ? (N + S - 1) / S : 0;
        for (int y = 0; y < n_kv_heads; ++y)
            for (int c = 0; c < n_sp_max; ++c)
                for (int t = 0; t < n_qt; ++t) {
                    const int qt = n_qt - 1 - t;
                    if (c >= n_sp || qt * rt >= T) continue;  // exits at once
                    const int keys = (c + 1 < n_sp ? S : N - c * S);
                    take(kSplitCtaOverheadTiles + (keys + 63) / 64);
                }
    }
    return *std::max_element(heap.begin(), heap.end());
}

}  // namespace

// Split-KV partials of every row of every stream (the causal count, or with
// `full` every row over all of its stream's keys).
static tf_status paged_partials(bool full, const void *q, int32_t n_rows_total, int32_t n_q_heads, const void *k_pool,
                               const void *v_pool, int32_t n_pages, int32_t page_size, int32_t n_kv_heads,
                               int32_t head_dim, const int32_t *page_table, int32_t page_table_len,
                               const tf_seg *segs, int32_t n_segs, const tf_seg *segs_host,
                               const int32_t *page_table_host, float scale, int32_t split_keys,
                               int32_t n_splits_max, float *part_o, float *part_m, float *part_l,
                               uint8_t *part_flag, uint32_t *status, tf_stream_t stream) {
    if (n_rows_total < 0 || n_q_heads <= 0 || n_kv_heads <= 0 || n_pages < 0 || page_table_len < 0 || n_segs < 0 ||
        split_keys < 0 || n_splits_max <= 0 || !std::isfinite(scale))
        return TF_ERR_ARG;
    if (n_q_heads % n_kv_heads != 0) return TF_ERR_UNSUPPORTED;
    if (!head_dim_ok(head_dim)) return TF_ERR_UNSUPPORTED;
    const int lp = log2_exact(page_size);
    if (lp < 3 || lp > 10) return TF_ERR_UNSUPPORTED;
    if (split_keys > 0 && split_keys < 16) return TF_ERR_UNSUPPORTED;
    if (n_segs > 65535) return TF_ERR_UNSUPPORTED;
    if (n_segs == 0 || n_rows_total == 0) return TF_OK;
    if (!q || !k_pool || !v_pool || !page_table || !segs || !part_o || !part_m || !part_l || !part_flag || !status)
        return TF_ERR_ARG;
    if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(part_o)) return TF_ERR_ALIGN;
    const int group = n_q_heads / n_kv_heads;
    int max_rows = n_rows_total;
    if (segs_host) {
        const tf_status st = check_segs_host(segs_host, n_segs, n_rows_total, page_table_len, page_size, n_pages,
                                             page_table_host, split_keys, n_splits_max, &max_rows, full);
        if (st != TF_OK) return st;
        if (max_rows == 0) return TF_OK;
    }
    const int64_t n_qgroups = ((int64_t)max_rows * group + 63) / 64;
    if (n_qgroups * n_kv_heads > 65535 || n_splits_max > (1 << 30)) return TF_ERR_UNSUPPORTED;

    // decode-shaped calls (a host table, at most 8 queries per stream and
    // kv-head, splits aligned to the page boxes) take the warp-specialized kernel
    const int tile_keys = 64;  // the warp-specialized kernel's tile
    const int box_rows = page_size < tile_keys ? page_size : tile_keys;
    if (segs_host && (int64_t)max_rows * group <= 8 && decode_ws_supported(head_dim, n_segs) &&
        (split_keys == 0 || split_keys % box_rows == 0)) {
        int64_t items = 0;
        for (int s = 0; s < n_segs; ++s) {
            const tf_seg e = segs_host[s];
            if (e.n_rows == 0) continue;
            const int per = split_len(e.n_keys, split_keys, n_splits_max, page_size);
            items += (int64_t)((e.n_keys + per - 1) / per) * n_kv_heads;
        }
        WsParams w{};
        w.q = static_cast<const uint16_t *>(q);
        w.n_rows_total = n_rows_total;
        w.hq = n_q_heads;
        w.hkv = n_kv_heads;
        w.group = group;
        w.n_segs = n_segs;
        w.segs = segs;
        w.page_table = page_table;
        w.n_pages = n_pages;
        w.log2_page = lp;
        w.pt_len = page_table_len;
        w.scale_log2 = scale * 1.4426950408889634f;
        w.split_keys = split_keys;
        w.n_splits_max = n_splits_max;
        w.full = full ? 1 : 0;
        w.part_o = part_o;
        w.part_m = part_m;
        w.part_l = part_l;
        w.part_flag = part_flag;
        w.status = status;
        return cuda_status(
            launch_decode_ws(w, head_dim, false, k_pool, v_pool, items, reinterpret_cast<cudaStream_t>(stream)));
    }

    // more queries per kv-head (a verify round): the tcgen05 kernel, one CTA
    // per (stream, kv-head, split, 128-query tile)
    if (partial_tc_supported(head_dim, group, page_size, split_keys)) {
        const int rt = 128 / group;
        const int64_t n_qt = ((int64_t)max_rows + rt - 1) / rt;
        if (n_qt * n_splits_max <= 0x7fffffff) {
            PromptTcParams t{};
            t.q = static_cast<const uint16_t *>(q);
            t.page_table = page_table;
            t.n_pages = n_pages;
            t.log2_page = lp;
            t.hq = n_q_heads;
            t.hkv = n_kv_heads;
            t.group = group;
            t.n_rows_total = n_rows_total;
            t.scale_log2 = scale * 1.4426950408889634f;
            t.segs = segs;
            t.pt_len = page_table_len;
            t.split_keys = split_keys;
            t.n_splits_max = n_splits_max;
            t.n_qt = (int)n_qt;
            t.full = full ? 1 : 0;
            t.part_o = part_o;
            t.part_m = part_m;
            t.part_l = part_l;
            t.part_flag = part_flag;
            t.status = status;
            return cuda_status(
                launch_partial_tc(t, head_dim, k_pool, v_pool, n_segs, reinterpret_cast<cudaStream_t>(stream)));
        }
    }

    AttnParams p{};
    p.q = static_cast<const uint16_t *>(q);
    p.n_rows_total = n_rows_total;
    p.hq = n_q_heads;
    p.hkv = n_kv_heads;
    p.group = group;
    p.k = static_cast<const uint16_t *>(k_pool);
    p.v = static_cast<const uint16_t *>(v_pool);
    p.n_pages = n_pages;
    p.log2_page = lp;
    p.pt_len = page_table_len;
    p.page_table = page_table;
    p.segs = segs;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.split_keys = split_keys;
    p.n_splits_max = n_splits_max;
    p.n_qgroups = (int)n_qgroups;
    p.full = full ? 1 : 0;
    p.part_o = part_o;
    p.part_m = part_m;
    p.part_l = part_l;
    p.part_flag = part_flag;
    p.status = status;
    const dim3 grid((unsigned)n_splits_max, (unsigned)(n_qgroups * n_kv_heads), (unsigned)n_segs);
    return cuda_status(launch_attn_partial(p, head_dim, false, false, grid, reinterpret_cast<cudaStream_t>(stream)));
}

// The row argmax; `early`: the argmax of a verify round, launched right after
// this library's merge, which may read the logits before the merge finishes
// (no kernel of the round writes them).
static tf_status argmax_call(const void *logits, int32_t n_rows, int32_t n_cols, int64_t ld, int32_t *ids,
                             uint8_t *flags, bool early, tf_stream_t stream) {
    if (n_rows < 0 || n_cols <= 0 || ld < n_cols) return TF_ERR_ARG;
    if (n_rows == 0) return TF_OK;
    if (!logits || !ids || !flags) return TF_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(logits) & 1u) != 0) return TF_ERR_ALIGN;
    ArgmaxParams p{};
    p.logits = static_cast<const uint16_t *>(logits);
    p.n_rows = n_rows;
    p.n_cols = n_cols;
    p.ld = ld;
    p.ids = ids;
    p.flags = flags;
    const bool vec = aligned16(logits) && (ld % 8) == 0;
    return cuda_status(launch_argmax(p, vec, early, reinterpret_cast<cudaStream_t>(stream)));
}

extern "C" {

tf_status tf_paged_attn_decode(const void *q, int32_t n_rows_total, int32_t n_q_heads, const void *k_pool,
                               const void *v_pool, int32_t n_pages, int32_t page_size, int32_t n_kv_heads,
                               int32_t head_dim, const int32_t *page_table, int32_t page_table_len,
                               const tf_seg *segs, int32_t n_segs, const tf_seg *segs_host,
                               const int32_t *page_table_host, float scale, int32_t split_keys,
                               int32_t n_splits_max, float *part_o, float *part_m, float *part_l,
                               uint8_t *part_flag, uint32_t *status, tf_stream_t stream) {
    return paged_partials(false, q, n_rows_total, n_q_heads, k_pool, v_pool, n_pages, page_size, n_kv_heads,
                          head_dim, page_table, page_table_len, segs, n_segs, segs_host, page_table_host, scale,
                          split_keys, n_splits_max, part_o, part_m, part_l, part_flag, status, stream);
}

tf_status tf_paged_attn_block(const void *q, int32_t n_rows_total, int32_t n_q_heads, const void *k_pool,
                              const void *v_pool, int32_t n_pages, int32_t page_size, int32_t n_kv_heads,
                              int32_t head_dim, const int32_t *page_table, int32_t page_table_len,
                              const tf_seg *segs, int32_t n_segs, const tf_seg *segs_host,
                              const int32_t *page_table_host, float scale, int32_t split_keys,
                              int32_t n_splits_max, float *part_o, float *part_m, float *part_l,
                              uint8_t *part_flag, uint32_t *status, tf_stream_t stream) {
    return paged_partials(true, q, n_rows_total, n_q_heads, k_pool, v_pool, n_pages, page_size, n_kv_heads,
                          head_dim, page_table, page_table_len, segs, n_segs, segs_host, page_table_host, scale,
                          split_keys, n_splits_max, part_o, part_m, part_l, part_flag, status, stream);
}

tf_status tf_kv_append(const void *k_rows, const void *v_rows, int32_t n_rows_total, void *k_pool, void *v_pool,
                       int32_t n_pages, int32_t page_size, int32_t n_kv_heads, int32_t head_dim,
                       const int32_t *page_table, int32_t page_table_len, const tf_seg *segs, int32_t n_segs,
                       const tf_seg *segs_host, const int32_t *page_table_host, uint32_t *status,
                       tf_stream_t stream) {
    if (n_rows_total < 0 || n_kv_heads <= 0 || n_pages < 0 || page_table_len < 0 || n_segs < 0) return TF_ERR_ARG;
    if (!head_dim_ok(head_dim)) return TF_ERR_UNSUPPORTED;
    const int lp = log2_exact(page_size);
    if (lp < 3 || lp > 10) return TF_ERR_UNSUPPORTED;
    if (n_segs > 65535) return TF_ERR_UNSUPPORTED;
    if (n_segs == 0 || n_rows_total == 0) return TF_OK;
    if (!k_rows || !v_rows || !k_pool || !v_pool || !page_table || !segs || !status) return TF_ERR_ARG;
    if (!aligned16(k_rows) || !aligned16(v_rows) || !aligned16(k_pool) || !aligned16(v_pool)) return TF_ERR_ALIGN;
    int max_rows = n_rows_total;
    if (segs_host) {
        const tf_status st = check_segs_host(segs_host, n_segs, n_rows_total, page_table_len, page_size, n_pages,
                                             page_table_host, 0, 0, &max_rows);
        if (st != TF_OK) return st;
        if (max_rows == 0) return TF_OK;
    }
    if ((int64_t)max_rows * n_kv_heads > ((int64_t)1 << 34)) return TF_ERR_UNSUPPORTED;
    AppendParams p{};
    p.k_rows = static_cast<const uint16_t *>(k_rows);
    p.v_rows = static_cast<const uint16_t *>(v_rows);
    p.k_pool = static_cast<uint16_t *>(k_pool);
    p.v_pool = static_cast<uint16_t *>(v_pool);
    p.n_rows_total = n_rows_total;
    p.hkv = n_kv_heads;
    p.n_pages = n_pages;
    p.log2_page = lp;
    p.pt_len = page_table_len;
    p.page_table = page_table;
    p.segs = segs;
    p.status = status;
    return cuda_status(launch_kv_append(p, head_dim, n_segs, max_rows, reinterpret_cast<cudaStream_t>(stream)));
}

tf_status tf_verify_round(const void *q, int32_t n_rows_total, int32_t n_q_heads, const void *k_pool,
                          const void *v_pool, int32_t n_pages, int32_t page_size, int32_t n_kv_heads,
                          int32_t head_dim, const int32_t *page_table, int32_t page_table_len, const tf_seg *segs,
                          int32_t n_segs, const tf_seg *segs_host, const int32_t *page_table_host, float scale,
                          int32_t split_keys, int32_t n_splits_max, int32_t full, float *part_o, float *part_m,
                          float *part_l, uint8_t *part_flag, float *out, uint8_t *flags, const void *logits,
                          int32_t n_logit_rows, int32_t n_cols, int64_t ld, int32_t *ids, uint8_t *id_flags,
                          uint32_t *status, tf_stream_t stream) {
    // the argmax's arguments first, so a refusal launches nothing
    if (n_logit_rows < 0) return TF_ERR_ARG;
    if (n_logit_rows > 0) {
        if (n_cols <= 0 || ld < n_cols || !logits || !ids || !id_flags) return TF_ERR_ARG;
        if ((reinterpret_cast<uintptr_t>(logits) & 1u) != 0) return TF_ERR_ALIGN;
    }
    if (n_rows_total > 0 && n_q_heads > 0 && (!out || !flags)) return TF_ERR_ARG;
    if (n_rows_total > 0 && out && !aligned16(out)) return TF_ERR_ALIGN;
    tf_status st = paged_partials(full != 0, q, n_rows_total, n_q_heads, k_pool, v_pool, n_pages, page_size,
                                  n_kv_heads, head_dim, page_table, page_table_len, segs, n_segs, segs_host,
                                  page_table_host, scale, split_keys, n_splits_max, part_o, part_m, part_l,
                                  part_flag, status, stream);
    if (st != TF_OK) return st;
    if (n_segs > 0 && n_rows_total > 0) {
        st = tf_attn_merge(part_o, part_m, part_l, part_flag, n_rows_total, n_q_heads, head_dim, n_splits_max, out,
                           flags, stream);
        if (st != TF_OK) return st;
    }
    if (n_logit_rows == 0) return TF_OK;
    // the merge just launched is this library's: the argmax may read the
    // logits while it drains
    const bool after_merge = n_segs > 0 && n_rows_total > 0;
    return argmax_call(logits, n_logit_rows, n_cols, ld, ids, id_flags, after_merge, stream);
}

tf_status tf_choose_split_keys(const tf_seg *segs_host, int32_t n_segs, int32_t n_q_heads, int32_t n_kv_heads,
                               int32_t head_dim, int32_t n_sms, int32_t *split_keys, int32_t *n_splits_max) {
    if (n_segs < 0 || n_q_heads <= 0 || n_kv_heads <= 0 || n_sms <= 0 || !split_keys || !n_splits_max ||
        (n_segs > 0 && !segs_host))
        return TF_ERR_ARG;
    // the schedule below is that of one CTA an SM (head dim 256); the two
    // CTAs an SM of head dims 64 and 128 overlap in a way it does not model
    if (head_dim != 256) return TF_ERR_UNSUPPORTED;
    if (n_q_heads % n_kv_heads != 0 || 128 % (n_q_heads / n_kv_heads) != 0) return TF_ERR_UNSUPPORTED;
    const int rt = 128 / (n_q_heads / n_kv_heads);  // rows a 128-query tile
    int max_rows = 0, max_keys = 0;
    for (int s = 0; s < n_segs; ++s) {
        if (segs_host[s].n_rows < 0 || segs_host[s].n_keys < 0) return TF_ERR_ARG;
        if (segs_host[s].n_rows == 0) continue;
        max_rows = std::max(max_rows, segs_host[s].n_rows);
        max_keys = std::max(max_keys, segs_host[s].n_keys);
    }
    int best_s = 256;
    if (max_rows > 0 && max_keys > 0) {
        const int n_qt = (max_rows + rt - 1) / rt;
        std::vector<double> heap;
        double best_t = -1.0;
        // candidates: 256 .. 4,096 by 128, then by 1,024 to 16,384, then doubling
        for (int64_t S = 256; S <= (int64_t)1 << 30;) {
            const int n_sp_max = (int)((max_keys + S - 1) / S);
            const int64_t ctas = (int64_t)n_segs * n_kv_heads * n_sp_max * n_qt;
            if (ctas <= kSplitMaxSimulatedCtas) {
                // SMs past the grid's CTA count stay idle: the heap needs no more
                const int slots = (int)std::min<int64_t>(n_sms, std::max<int64_t>(ctas, 1));
                const double t = partial_makespan(segs_host, n_segs, n_kv_heads, rt, n_qt, (int)S, n_sp_max, slots,
                                                  heap);
                if (best_t < 0.0 || t <= best_t) {  // the larger split on a tie
                    best_t = t;
                    best_s = (int)S;
                }
            }
            if (S >= max_keys || S >= ((int64_t)1 << 30)) {  // one split a stream: larger sizes change nothing
                if (best_t < 0.0) best_s = (int)S;  // nothing simulated: the fewest CTAs
                break;
            }
            S = S < 4096 ? S + 128 : (S < 16384 ? S + 1024 : S * 2);
        }
    }
    *split_keys = best_s;
    *n_splits_max = max_keys > 0 ? (int32_t)((max_keys + best_s - 1) / best_s) : 1;
    return TF_OK;
}

tf_status tf_attn_merge(const float *part_o, const float *part_m, const float *part_l, const uint8_t *part_flag,
                        int32_t n_rows_total, int32_t n_q_heads, int32_t head_dim, int32_t n_splits_max, float *out,
                        uint8_t *flags, tf_stream_t stream) {
    if (n_rows_total < 0 || n_q_heads <= 0 || n_splits_max <= 0) return TF_ERR_ARG;
    if (!head_dim_ok(head_dim)) return TF_ERR_UNSUPPORTED;
    if (n_rows_total == 0) return TF_OK;
    if (!part_o || !part_m || !part_l || !part_flag || !out || !flags) return TF_ERR_ARG;
    if (!aligned16(part_o) || !aligned16(out)) return TF_ERR_ALIGN;
    MergeParams p{};
    p.part_o = part_o;
    p.part_m = part_m;
    p.part_l = part_l;
    p.part_flag = part_flag;
    p.n_units = (int64_t)n_rows_total * n_q_heads;
    p.n_parts = n_splits_max;
    p.hq = n_q_heads;
    p.n_rows_total = n_rows_total;
    p.out = out;
    p.flags = flags;
    return cuda_status(launch_merge(p, head_dim, kMergeRows, reinterpret_cast<cudaStream_t>(stream)));
}

tf_status tf_paged_attn_prompt(const void *q, int32_t n_rows_total, int32_t n_q_heads, const void *k_pool,
                               const void *v_pool, int32_t n_pages, int32_t page_size, int32_t n_kv_heads,
                               int32_t head_dim, const int32_t *page_table, int32_t page_table_len,
                               const tf_seg *seg_host, float scale, void *out, int32_t out_dtype, uint8_t *flags,
                               uint32_t *status, tf_stream_t stream) {
    if (!seg_host || n_rows_total < 0 || n_q_heads <= 0 || n_kv_heads <= 0 || n_pages < 0 || page_table_len < 0 ||
        !std::isfinite(scale))
        return TF_ERR_ARG;
    if (out_dtype != TF_OUT_F32 && out_dtype != TF_OUT_BF16) return TF_ERR_ARG;
    if (n_q_heads % n_kv_heads != 0 || !head_dim_ok(head_dim)) return TF_ERR_UNSUPPORTED;
    const int lp = log2_exact(page_size);
    if (lp < 3 || lp > 10) return TF_ERR_UNSUPPORTED;
    int max_rows = 0;
    const tf_status st =
        check_segs_host(seg_host, 1, n_rows_total, page_table_len, page_size, n_pages, nullptr, 0, 1, &max_rows);
    if (st != TF_OK) return st;
    if (max_rows == 0) return TF_OK;
    if (!q || !k_pool || !v_pool || !page_table || !out || !status) return TF_ERR_ARG;
    if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(out)) return TF_ERR_ALIGN;
    const int group = n_q_heads / n_kv_heads;
    const int64_t n_qgroups = ((int64_t)max_rows * group + 63) / 64;
    if (n_qgroups * n_kv_heads > 65535) return TF_ERR_UNSUPPORTED;

    if (prompt_tc_supported(head_dim, group, page_size)) {
        PromptTcParams t{};
        t.q = static_cast<const uint16_t *>(q);
        t.q_row = seg_host->q_row;
        t.n_rows = seg_host->n_rows;
        t.n_keys = seg_host->n_keys;
        t.pt_base = seg_host->pt_base;
        t.n_pg = seg_host->n_pages;
        t.page_table = page_table;
        t.n_pages = n_pages;
        t.log2_page = lp;
        t.hq = n_q_heads;
        t.hkv = n_kv_heads;
        t.group = group;
        t.n_rows_total = n_rows_total;
        t.scale_log2 = scale * 1.4426950408889634f;
        t.out = out;
        t.out_bf16 = out_dtype == TF_OUT_BF16;
        t.out_flags = flags;
        t.status = status;
        return cuda_status(launch_prompt_tc(t, head_dim, k_pool, v_pool, reinterpret_cast<cudaStream_t>(stream)));
    }
    AttnParams p{};
    p.q = static_cast<const uint16_t *>(q);
    p.n_rows_total = n_rows_total;
    p.hq = n_q_heads;
    p.hkv = n_kv_heads;
    p.group = group;
    p.k = static_cast<const uint16_t *>(k_pool);
    p.v = static_cast<const uint16_t *>(v_pool);
    p.n_pages = n_pages;
    p.log2_page = lp;
    p.pt_len = page_table_len;
    p.page_table = page_table;
    p.seg0 = *seg_host;
    p.seg_inline = 1;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.split_keys = 0;
    p.n_splits_max = 1;
    p.n_qgroups = (int)n_qgroups;
    p.out = out;
    p.out_bf16 = out_dtype == TF_OUT_BF16;
    p.out_flags = flags;
    p.status = status;
    const dim3 grid(1u, (unsigned)(n_qgroups * n_kv_heads), 1u);
    return cuda_status(launch_attn_partial(p, head_dim, false, true, grid, reinterpret_cast<cudaStream_t>(stream)));
}

size_t tf_ring_workspace_bytes(int32_t n_segs, int32_t n_q_heads, int32_t head_dim, int32_t n_splits_max) {
    if (n_segs < 0 || n_q_heads <= 0 || head_dim <= 0 || n_splits_max <= 0) return 0;
    const size_t parts = (size_t)n_segs * n_q_heads * n_splits_max;
    const size_t o = parts * head_dim * sizeof(float);
    const size_t ml = 2 * parts * sizeof(float);
    return ((o + ml + parts + 255) / 256) * 256;
}

tf_status tf_ring_attn(const void *q, int32_t n_rows_total, int32_t n_q_heads, const void *ring_k, const void *ring_v,
                       int64_t ring_slots_total, int32_t n_kv_heads, int32_t head_dim, const tf_ring_seg *rsegs,
                       int32_t n_segs, const tf_ring_seg *rsegs_host, float scale, int32_t split_slots,
                       int32_t n_splits_max, void *workspace, size_t workspace_bytes, float *out, uint8_t *flags,
                       uint32_t *status, tf_stream_t stream) {
    if (n_rows_total < 0 || n_q_heads <= 0 || n_kv_heads <= 0 || ring_slots_total < 0 || n_segs < 0 ||
        n_splits_max <= 0 || !std::isfinite(scale))
        return TF_ERR_ARG;
    if (n_q_heads % n_kv_heads != 0 || !head_dim_ok(head_dim) || split_slots < 16) return TF_ERR_UNSUPPORTED;
    if (n_segs > 65535) return TF_ERR_UNSUPPORTED;
    if (n_segs == 0) return TF_OK;
    if (!q || !ring_k || !ring_v || !rsegs || !workspace || !out || !flags || !status) return TF_ERR_ARG;
    if (!aligned16(q) || !aligned16(ring_k) || !aligned16(ring_v) || !aligned16(out) || !aligned16(workspace))
        return TF_ERR_ALIGN;
    if (workspace_bytes < tf_ring_workspace_bytes(n_segs, n_q_heads, head_dim, n_splits_max)) return TF_ERR_WORKSPACE;
    if (rsegs_host) {
        for (int s = 0; s < n_segs; ++s) {
            const tf_ring_seg e = rsegs_host[s];
            if (e.q_row < 0 || e.q_row >= n_rows_total || e.size <= 0 || e.n_valid < 1 || e.n_valid > e.size ||
                e.head < 0 || e.head >= e.size || e.base < 0 || e.base + e.size > ring_slots_total)
                return TF_ERR_ARG;
            if ((e.n_valid + split_slots - 1) / split_slots > n_splits_max) return TF_ERR_ARG;
        }
    }
    const int group = n_q_heads / n_kv_heads;
    const int n_qgroups = (group + 63) / 64;
    if ((int64_t)n_qgroups * n_kv_heads > 65535) return TF_ERR_UNSUPPORTED;
    const size_t parts = (size_t)n_segs * n_q_heads * n_splits_max;
    float *po = static_cast<float *>(workspace);
    float *pm = po + parts * head_dim;
    float *pl = pm + parts;
    uint8_t *pf = reinterpret_cast<uint8_t *>(pl + parts);
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

    cudaError_t e = cudaSuccess;
    if (group <= 8 && decode_ws_supported(head_dim, n_segs) && ring_slots_total <= 0x7fffffff) {
        WsParams w{};
        w.q = static_cast<const uint16_t *>(q);
        w.n_rows_total = n_rows_total;
        w.hq = n_q_heads;
        w.hkv = n_kv_heads;
        w.group = group;
        w.n_segs = n_segs;
        w.rsegs = rsegs;
        w.ring_slots_total = ring_slots_total;
        w.scale_log2 = scale * 1.4426950408889634f;
        w.split_keys = split_slots;
        w.n_splits_max = n_splits_max;
        w.part_o = po;
        w.part_m = pm;
        w.part_l = pl;
        w.part_flag = pf;
        w.status = status;
        e = launch_decode_ws(w, head_dim, true, ring_k, ring_v, (int64_t)n_segs * n_kv_heads * n_splits_max, st);
        if (e != cudaSuccess) return TF_ERR_CUDA;
        return ring_merge(po, pm, pl, pf, n_segs, n_q_heads, head_dim, n_splits_max, n_rows_total, rsegs, split_slots,
                          ring_slots_total, out, flags, st);
    }

    AttnParams p{};
    p.q = static_cast<const uint16_t *>(q);
    p.n_rows_total = n_rows_total;
    p.hq = n_q_heads;
    p.hkv = n_kv_heads;
    p.group = group;
    p.k = static_cast<const uint16_t *>(ring_k);
    p.v = static_cast<const uint16_t *>(ring_v);
    p.rsegs = rsegs;
    p.ring_slots_total = ring_slots_total;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.split_keys = split_slots;
    p.n_splits_max = n_splits_max;
    p.n_qgroups = n_qgroups;
    p.part_o = po;
    p.part_m = pm;
    p.part_l = pl;
    p.part_flag = pf;
    p.status = status;
    const dim3 grid((unsigned)n_splits_max, (unsigned)(n_qgroups * n_kv_heads), (unsigned)n_segs);
    e = launch_attn_partial(p, head_dim, true, false, grid, st);
    if (e != cudaSuccess) return TF_ERR_CUDA;
    return ring_merge(po, pm, pl, pf, n_segs, n_q_heads, head_dim, n_splits_max, n_rows_total, rsegs, split_slots,
                      ring_slots_total, out, flags, st);
}

size_t tf_ring_tree_workspace_bytes(int32_t n_rows_total, int32_t n_q_heads, int32_t head_dim, int32_t n_splits_max) {
    if (n_rows_total < 0 || n_q_heads <= 0 || head_dim <= 0 || n_splits_max <= 0) return 0;
    const size_t parts = (size_t)n_rows_total * n_q_heads * n_splits_max;
    const size_t o = parts * head_dim * sizeof(float);
    const size_t ml = 2 * parts * sizeof(float);
    return ((o + ml + parts + 255) / 256) * 256;
}

tf_status tf_ring_tree_attn(const void *q, int32_t n_rows_total, int32_t n_q_heads, const void *ring_k,
                            const void *ring_v, int64_t ring_slots_total, int32_t n_kv_heads, int32_t head_dim,
                            const tf_tree_seg *tsegs, int32_t n_segs, const tf_tree_seg *tsegs_host,
                            const int32_t *parents, int32_t n_parents, const int32_t *parents_host, float scale,
                            int32_t split_slots, int32_t n_splits_max, void *workspace, size_t workspace_bytes,
                            float *out, uint8_t *flags, uint32_t *status, tf_stream_t stream) {
    if (n_rows_total < 0 || n_q_heads <= 0 || n_kv_heads <= 0 || ring_slots_total < 0 || n_segs < 0 ||
        n_parents < 0 || n_splits_max <= 0 || !std::isfinite(scale))
        return TF_ERR_ARG;
    if (n_q_heads % n_kv_heads != 0 || !head_dim_ok(head_dim) || split_slots < 64) return TF_ERR_UNSUPPORTED;
    const int group = n_q_heads / n_kv_heads;
    if (!tree_tc_supported(head_dim, group)) return TF_ERR_UNSUPPORTED;
    // a 64-slot box may start at the last slot: its rows stay below 2^31
    if (n_segs > 65535 || ring_slots_total > 0x7fffffff - 64) return TF_ERR_UNSUPPORTED;
    if (n_segs == 0 || n_rows_total == 0) return TF_OK;
    if (!q || !ring_k || !ring_v || !tsegs || !parents || !workspace || !out || !flags || !status) return TF_ERR_ARG;
    if (!aligned16(q) || !aligned16(ring_k) || !aligned16(ring_v) || !aligned16(out) || !aligned16(workspace))
        return TF_ERR_ALIGN;
    if (workspace_bytes < tf_ring_tree_workspace_bytes(n_rows_total, n_q_heads, head_dim, n_splits_max))
        return TF_ERR_WORKSPACE;
    int max_nodes = kTreeMaxNodes;
    if (tsegs_host) {
        max_nodes = 1;
        for (int s = 0; s < n_segs; ++s) {
            const tf_tree_seg e = tsegs_host[s];
            if (!tree_seg_ok(e, n_rows_total, n_parents, ring_slots_total)) return TF_ERR_ARG;
            if (tree_splits(e, split_slots).n_sp > n_splits_max) return TF_ERR_ARG;
            if (parents_host)
                for (int i = 0; i < e.n_nodes; ++i) {
                    const int pa = parents_host[e.parent_base + i];
                    if (pa < -1 || pa >= i) return TF_ERR_ARG;
                }
            max_nodes = std::max(max_nodes, (int)e.n_nodes);
        }
    }
    const int rt = 128 / group;  // rows a 128-query tile
    const int n_qt = (max_nodes + rt - 1) / rt;
    if ((int64_t)n_qt * n_splits_max > 0x7fffffff) return TF_ERR_UNSUPPORTED;
    const size_t parts = (size_t)n_rows_total * n_q_heads * n_splits_max;
    float *po = static_cast<float *>(workspace);
    float *pm = po + parts * head_dim;
    float *pl = pm + parts;
    uint8_t *pf = reinterpret_cast<uint8_t *>(pl + parts);
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

    PromptTcParams t{};
    t.q = static_cast<const uint16_t *>(q);
    t.hq = n_q_heads;
    t.hkv = n_kv_heads;
    t.group = group;
    t.n_rows_total = n_rows_total;
    t.scale_log2 = scale * 1.4426950408889634f;
    t.split_keys = split_slots;
    t.n_splits_max = n_splits_max;
    t.n_qt = n_qt;
    t.part_o = po;
    t.part_m = pm;
    t.part_l = pl;
    t.part_flag = pf;
    t.status = status;
    t.tsegs = tsegs;
    t.parents = parents;
    t.n_parents = n_parents;
    t.ring_slots_total = ring_slots_total;
    if (launch_tree_tc(t, head_dim, ring_k, ring_v, n_segs, st) != cudaSuccess) return TF_ERR_CUDA;

    MergeParams mp{};
    mp.part_o = po;
    mp.part_m = pm;
    mp.part_l = pl;
    mp.part_flag = pf;
    mp.n_units = (int64_t)n_segs * max_nodes * n_q_heads;
    mp.n_parts = n_splits_max;
    mp.hq = n_q_heads;
    mp.n_rows_total = n_rows_total;
    mp.split_slots = split_slots;
    mp.ring_slots_total = ring_slots_total;
    mp.tsegs = tsegs;
    mp.tree_nodes = max_nodes;
    mp.n_parents = n_parents;
    mp.out = out;
    mp.flags = flags;
    return cuda_status(launch_merge(mp, head_dim, kMergeTree, st));
}

tf_status tf_argmax_rows(const void *logits, int32_t n_rows, int32_t n_cols, int64_t ld, int32_t *ids,
                         uint8_t *flags, tf_stream_t stream) {
    return argmax_call(logits, n_rows, n_cols, ld, ids, flags, false, stream);
}

const char *tf_status_str(tf_status s) {
    switch (s) {
        case TF_OK: return "ok";
        case TF_ERR_ARG: return "bad argument";
        case TF_ERR_PAST_PAGES: return "keys past a stream's pages";
        case TF_ERR_BAD_PAGE: return "page id outside the pool";
        case TF_ERR_UNSUPPORTED: return "unsupported shape";
        case TF_ERR_CUDA: return "CUDA launch error";
        case TF_ERR_ALIGN: return "misaligned buffer";
        case TF_ERR_WORKSPACE: return "workspace too small";
    }
    return "unknown status";
}

int32_t tf_abi_version(void) { return 1; }

tf_status tf_wait_limit_test(int32_t on) {
    tfp::g_wait_runout_ns = on ? 5000000ull : 0ull;  // 5 ms
    return TF_OK;
}

}  // extern "C"
