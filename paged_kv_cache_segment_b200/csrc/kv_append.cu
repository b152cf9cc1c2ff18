// kv_append.cu - a stream's new rows' keys and values into its pages.
//
// Source: TensorFold #1653 "spark25 CUDA: the full layers' caches in pages of
// the core pool", PR body: the rows kernel writes kr / vr and tf_wrows_put
// copies them into the pages; forward refuses rows past a slot's pages
// (PastPages).
//
// Row i of a stream with n_rows rows and n_keys keys is the stream's key
// j = n_keys - n_rows + i: page page_table[pt_base + j / P], slot j % P.  One
// warp moves one (row, kv-head): the row's D bf16 of K and then of V as
// 16-byte chunks, one chunk a lane (two at head dim 256), so every copy is a
// contiguous, aligned run on both sides.  Invalid table entries set status
// bits and are skipped; nothing outside the named slots is written.
#include <cstdint>

#include "tf_common.cuh"
#include "tf_internal.h"

namespace tfp {

constexpr int kAppendWarps = 8;

template <int D>
__global__ void __launch_bounds__(kAppendWarps * 32) kv_append_kernel(const AppendParams p) {
    const tf_seg e = p.segs[blockIdx.y];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool bad = e.q_row < 0 || e.n_rows < 0 || (int64_t)e.q_row + e.n_rows > p.n_rows_total ||
                     e.n_keys < e.n_rows || e.pt_base < 0 || e.n_pages < 0 ||
                     (int64_t)e.pt_base + e.n_pages > p.pt_len;
    if (bad) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(p.status, TF_DEV_BAD_SEG);
        return;
    }
    if ((int64_t)e.n_keys > ((int64_t)e.n_pages << p.log2_page)) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(p.status, TF_DEV_PAST_PAGES);
        return;
    }
    const int64_t w = (int64_t)blockIdx.x * kAppendWarps + warp;  // (row, kv-head) of this warp
    const int i = (int)(w / p.hkv), g = (int)(w - (int64_t)i * p.hkv);
    if (i >= e.n_rows) return;
    const int j = e.n_keys - e.n_rows + i;
    const int page = p.page_table[e.pt_base + (j >> p.log2_page)];
    if (page < 0 || page >= p.n_pages) {
        if (lane == 0) atomicOr(p.status, TF_DEV_BAD_PAGE);
        return;
    }
    const int slot = j & ((1 << p.log2_page) - 1);
    const int64_t src = ((int64_t)(e.q_row + i) * p.hkv + g) * D;
    const int64_t dst = (((int64_t)page * p.hkv + g) << p.log2_page | slot) * D;
    constexpr int kChunks = D / 8;  // 16-byte chunks of one row of K (or V)
#pragma unroll
    for (int c = lane; c < 2 * kChunks; c += 32) {
        const bool is_v = c >= kChunks;
        const int cc = is_v ? c - kChunks : c;
        const uint4 x = __ldg(reinterpret_cast<const uint4 *>((is_v ? p.v_rows : p.k_rows) + src) + cc);
        reinterpret_cast<uint4 *>((is_v ? p.v_pool : p.k_pool) + dst)[cc] = x;
    }
}

cudaError_t launch_kv_append(const AppendParams &p, int head_dim, int n_segs, int max_rows, cudaStream_t st) {
    if (n_segs == 0 || max_rows == 0) return cudaSuccess;
    const int64_t warps = (int64_t)max_rows * p.hkv;
    const dim3 grid((unsigned)((warps + kAppendWarps - 1) / kAppendWarps), (unsigned)n_segs);
    switch (head_dim) {
        case 64: kv_append_kernel<64><<<grid, kAppendWarps * 32, 0, st>>>(p); break;
        case 128: kv_append_kernel<128><<<grid, kAppendWarps * 32, 0, st>>>(p); break;
        case 256: kv_append_kernel<256><<<grid, kAppendWarps * 32, 0, st>>>(p); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace tfp
