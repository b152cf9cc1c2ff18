// tf_internal.h - parameter blocks and launchers shared between the C-ABI
// entry points (api.cu) and the kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/tfpaged.h"

namespace tfp {

// Parameters of the split-KV attention kernel (paged or ring source).
struct AttnParams {
    const uint16_t *q;
    int n_rows_total, hq, hkv, group;
    const uint16_t *k, *v;  // pool [pages][Hkv][P][D] or ring [slots][Hkv][D]
    // paged source
    int n_pages, log2_page, pt_len;
    const int32_t *page_table;
    const tf_seg *segs;
    tf_seg seg0;     // used instead of segs[0] when seg_inline != 0 (one-stream prompt calls)
    int seg_inline;
    // ring source
    const tf_ring_seg *rsegs;
    int64_t ring_slots_total;
    float scale_log2;  // scale * log2(e)
    int split_keys, n_splits_max, n_qgroups;
    int full;  // every row sees all of its stream's keys (no causal count)
    // partial outputs [unit][n_splits_max](*D)
    float *part_o, *part_m, *part_l;
    uint8_t *part_flag;
    // direct outputs [row][Hq](*D)
    void *out;
    int out_bf16;
    uint8_t *out_flags;
    uint32_t *status;
};

struct MergeParams {
    const float *part_o, *part_m, *part_l;
    const uint8_t *part_flag;
    int64_t n_units;  // units of partials (rows x heads, or ring entries x heads)
    int n_parts, hq, n_rows_total;
    const tf_ring_seg *rsegs;  // ring merge: unit s * Hq + h writes row rsegs[s].q_row
    int split_slots;           // ring merge: partials of entry s are ceil(n_valid / split_slots)
    int64_t ring_slots_total;
    // tree merge: unit (s * tree_nodes + i) * Hq + h writes row tsegs[s].q_row + i
    const tf_tree_seg *tsegs;
    int tree_nodes;
    int n_parents;
    float *out;
    uint8_t *flags;
};

// Parameters of the tensor-core prompt kernel (one stream's chunk).
struct PromptTcParams {
    const uint16_t *q;                         // bf16 [n_rows_total][hq][D]
    int q_row, n_rows, n_keys, pt_base, n_pg;  // the prompt chunk's segment
    const int32_t *page_table;
    int n_pages, log2_page, hq, hkv, group, n_rows_total;
    float scale_log2;
    // prompt: final rows
    void *out;
    int out_bf16;
    uint8_t *out_flags;
    // split-KV partials: segment table, splits, q-tiles of the grid, outputs
    const tf_seg *segs;
    int pt_len, split_keys, n_splits_max, n_qt;
    int full;  // every row sees all of its stream's keys (no causal count)
    float *part_o, *part_m, *part_l;
    uint8_t *part_flag;
    uint32_t *status;
    // draft trees over rings: one table entry per tree; partials are laid
    // out by query row like the paged partials
    const tf_tree_seg *tsegs;
    const int32_t *parents;
    int n_parents;
    int64_t ring_slots_total;
    // the timeout test hook (tf_wait_limit_test): the TMA warp issues nothing
    // and every bounded wait gives up after wait_ns (0: the 2 s default)
    int test_idle;
    uint64_t wait_ns;
};

// Parameters of the KV append (rows into their pages).
struct AppendParams {
    const uint16_t *k_rows, *v_rows;  // bf16 [n_rows_total][hkv][D]
    uint16_t *k_pool, *v_pool;        // bf16 [n_pages][hkv][P][D]
    int n_rows_total, hkv, n_pages, log2_page, pt_len;
    const int32_t *page_table;
    const tf_seg *segs;
    uint32_t *status;
};

// Parameters of the warp-specialized decode kernel (paged or ring source).
struct WsParams {
    const uint16_t *q;
    int n_rows_total, hq, hkv, group;
    int n_segs;
    // paged
    const tf_seg *segs;
    const int32_t *page_table;
    int n_pages, log2_page, pt_len;
    // ring
    const tf_ring_seg *rsegs;
    int64_t ring_slots_total;
    float scale_log2;
    int split_keys, n_splits_max;
    int full;  // every row sees all of its stream's keys (no causal count)
    float *part_o, *part_m, *part_l;
    uint8_t *part_flag;
    uint32_t *status;
    // the timeout test hook (tf_wait_limit_test): the producer issues nothing
    // and every bounded wait gives up after wait_ns (0: the 2 s default)
    int test_idle;
    uint64_t wait_ns;
};

struct ArgmaxParams {
    const uint16_t *logits;
    int n_rows, n_cols;
    int64_t ld;
    int32_t *ids;
    uint8_t *flags;
};

// The timeout test hook: while set (tf_wait_limit_test), the warp-specialized
// and tensor-core kernels launched on this host thread issue no loads and
// give up their bounded waits after this many nanoseconds (0: hook off).
uint64_t test_wait_runout_ns();

cudaError_t launch_attn_partial(const AttnParams &p, int head_dim, bool ring, bool direct, dim3 grid,
                                cudaStream_t st);
enum MergeMode { kMergeRows = 0, kMergeRing = 1, kMergeTree = 2 };
cudaError_t launch_merge(const MergeParams &p, int head_dim, int mode, cudaStream_t st);
cudaError_t launch_argmax(const ArgmaxParams &p, bool vec, bool early, cudaStream_t st);
bool prompt_tc_supported(int head_dim, int group, int page_size);
bool decode_ws_supported(int head_dim, int n_segs);
cudaError_t launch_decode_ws(const WsParams &p, int head_dim, bool ring, const void *k, const void *v,
                             int64_t n_items_bound, cudaStream_t st);
cudaError_t launch_kv_append(const AppendParams &p, int head_dim, int n_segs, int max_rows, cudaStream_t st);
cudaError_t launch_prompt_tc(const PromptTcParams &p, int head_dim, const void *k, const void *v, cudaStream_t st);
bool partial_tc_supported(int head_dim, int group, int page_size, int split_keys);
cudaError_t launch_partial_tc(const PromptTcParams &p, int head_dim, const void *k, const void *v, int n_segs,
                              cudaStream_t st);

constexpr int kArgmaxCluster = 2;

// The most nodes a draft tree may have (a node's ancestors are a 64-bit mask).
constexpr int kTreeMaxNodes = 64;

// Splits of a draft tree's keys: the keys [0, n_valid + n_nodes) run from
// slot start = (head - n_valid) mod size; those at or past wrap_at = size -
// start sit at slot key - wrap_at.  Splits never cross the wrap: the first
// run [0, na) and the second [na, N) are cut into split_slots-key pieces.
struct TreeSplits {
    int start, wrap_at, n_keys, na, sa, n_sp;
};
__host__ __device__ inline TreeSplits tree_splits(const tf_tree_seg &e, int split_slots) {
    TreeSplits t;
    t.start = e.head - e.n_valid;
    if (t.start < 0) t.start += e.size;
    t.wrap_at = e.size - t.start;
    t.n_keys = e.n_valid + e.n_nodes;
    t.na = t.n_keys < t.wrap_at ? t.n_keys : t.wrap_at;
    t.sa = (t.na + split_slots - 1) / split_slots;
    t.n_sp = t.sa + (t.n_keys - t.na + split_slots - 1) / split_slots;
    return t;
}
// An entry the tree kernels can read: sizes and ranges only (the parents are
// checked as each node's path is walked).
__host__ __device__ inline bool tree_seg_ok(const tf_tree_seg &e, int n_rows_total, int n_parents,
                                            int64_t ring_slots_total) {
    return e.n_nodes >= 1 && e.n_nodes <= kTreeMaxNodes && e.n_valid >= 0 && e.size > 0 &&
           (int64_t)e.n_valid + e.n_nodes <= e.size && e.head >= 0 && e.head < e.size && e.base >= 0 &&
           e.base + e.size <= ring_slots_total && e.q_row >= 0 && (int64_t)e.q_row + e.n_nodes <= n_rows_total &&
           e.parent_base >= 0 && (int64_t)e.parent_base + e.n_nodes <= n_parents;
}
bool tree_tc_supported(int head_dim, int group);
cudaError_t launch_tree_tc(const PromptTcParams &p, int head_dim, const void *k, const void *v, int n_segs,
                           cudaStream_t st);

}  // namespace tfp
