// decode_ws.cu - split-KV partials for decode-shaped work (at most 8 queries
// per (stream, kv-head)): a persistent, warp-specialized kernel.
//
// Sources (TensorFold pull requests, by title and section):
//  - #1503 "lfm2_moe CUDA: attention pages from the shared KV pool, and the
//    prompt cache", commit list: every stream's rows in one launch from a
//    segment table; paged split-KV chunk bodies.
//  - #1653 "spark25 CUDA: the full layers' caches in pages of the core pool",
//    review thread and commit list: page lookups hoisted out of the key loop,
//    the next page's id fetched ahead of its use.
//  - #1562 "Qwen3.6 MTP drafter on CUDA", PR body: each row over its own ring
//    of slots, stepped with a wrap; the next group in flight while the
//    current one folds.
//
// Shape of the kernel:
//  - One CTA per SM walks a list of work items (stream or ring row, kv-head,
//    split); the list is the exact set of non-empty items, enumerated from a
//    per-CTA prefix sum over the segment table.
//  - Warp 4 is the producer: one lane issues TMA boxes (one box per page and
//    64-column slab, 128-byte swizzle) for each 64-key tile into a ring of
//    stages guarded by full/empty mbarriers, and a bulk copy of the item's
//    queries into a small ring of query buffers.  It runs ahead across item
//    boundaries, so an item's epilogue overlaps the next item's loads.
//  - Warps 0-3 consume: each takes 16 keys of a tile.  With the keys as the
//    MMA's M side and the (up to 8) queries as N, S^T = K Q^T and
//    O^T += V^T P^T each take one m16n8k16 per 16 columns of D; P^T is
//    formed in registers with movmatrix (bf16 hi + bf16 lo, about 16 bits).
//  - At an item's end the four warps' online-softmax states meet in shared
//    memory (a two-level tree) and one partial per (row, q-head) is written.
#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "tf_common.cuh"
#include "tf_internal.h"
#include "tf_sm100.cuh"
#include "tma_host.h"

namespace tfp {

constexpr int kWsQ = 8;  // queries per item (the MMA's N)

// Per head dim: NC consumer warps, each folding 16 keys of a 16*NC-key tile,
// and a ring of kStages tiles.  Head dims up to 128 are sized so that two
// CTAs share an SM: while one CTA combines its warps at the end of an item,
// the other keeps streaming.  Head dim 256 needs one SM per CTA for three
// stages.  kPrefixMax bounds the streams a call may have on this kernel.
template <int D>
struct WsCfg {
    static constexpr int NC = 4;
    static constexpr int kThreads = (NC + 1) * 32;  // + one producer warp
    static constexpr int TK = 16 * NC;              // keys per tile
    static constexpr int kSlab = TK * 128;          // TK rows x 128 bytes (64 bf16 columns)
    static constexpr int kSlabs = D / 64;
    static constexpr int kTileBytes = kSlabs * kSlab;
    static constexpr int kStageBytes = 2 * kTileBytes;  // K then V
    static constexpr int kStages = D == 256 ? 3 : (D == 128 ? 3 : 6);
    static constexpr int kNQ = 2;
    static constexpr int kPrefixMax = D == 256 ? 512 : 256;
    static constexpr int kMinBlocks = D == 256 ? 1 : 2;
    static constexpr int kQBytes = kWsQ * D * 2;
    static constexpr int kCombStride = D + 4;  // floats a query row of the combine buffer (no bank conflicts)
    static constexpr int kCombBytes = (NC / 2) * kWsQ * kCombStride * 4;
    static constexpr int kOffQ = kStages * kStageBytes;
    static constexpr int kOffComb = kOffQ + kNQ * kQBytes;
    static constexpr int kOffPrefix = kOffComb + kCombBytes;
    // the stream prefix of items, the prefix of full-split items, the tail order
    static constexpr int kSmem = kOffPrefix + 3 * (kPrefixMax + 1) * 4 + 1024;
};

struct WsItem {
    int s, g, c;
    int q_row, n_rows, n_keys;
    int key_lo, key_hi, full_hi, causal0;
    int pt_base, n_pg;             // paged
    int64_t base;                  // ring
    int size, start, wrap_at;      // ring: keys j >= wrap_at sit at slots j - wrap_at
};

// Stream s's entry and the number of its non-empty partials (0 if the entry is
// invalid or has no rows).  `bits` collects TF_DEV_* codes.
template <bool RING>
__device__ __forceinline__ int ws_stream_splits(const WsParams &p, int s, uint32_t &bits) {
    if constexpr (RING) {
        const tf_ring_seg e = p.rsegs[s];
        const bool bad = e.q_row < 0 || e.q_row >= p.n_rows_total || e.size <= 0 || e.n_valid < 1 ||
                         e.n_valid > e.size || e.head < 0 || e.head >= e.size || e.base < 0 ||
                         e.base + e.size > p.ring_slots_total;
        if (bad) {
            bits |= TF_DEV_BAD_SEG;
            return 0;
        }
        const int n = (e.n_valid + p.split_keys - 1) / p.split_keys;
        if (n > p.n_splits_max) {
            bits |= TF_DEV_SPLITS;
            return 0;
        }
        return n;
    } else {
        const tf_seg e = p.segs[s];
        const bool bad = e.q_row < 0 || e.n_rows < 0 || (int64_t)e.q_row + e.n_rows > p.n_rows_total ||
                         e.n_keys < (p.full ? (e.n_rows > 0 ? 1 : 0) : e.n_rows) || e.pt_base < 0 || e.n_pages < 0 ||
                         (int64_t)e.pt_base + e.n_pages > p.pt_len;
        if (bad) {
            bits |= TF_DEV_BAD_SEG;
            return 0;
        }
        if ((int64_t)e.n_keys > ((int64_t)e.n_pages << p.log2_page)) {
            bits |= TF_DEV_PAST_PAGES;
            return 0;
        }
        if (e.n_rows == 0 || e.n_rows * p.group > kWsQ) return 0;
        int per = p.split_keys;
        if (per <= 0) {
            per = (e.n_keys + p.n_splits_max - 1) / p.n_splits_max;
            per = ((per + (1 << p.log2_page) - 1) >> p.log2_page) << p.log2_page;
        }
        const int n = (e.n_keys + per - 1) / per;
        if (n > p.n_splits_max) {
            bits |= TF_DEV_SPLITS;
            return 0;
        }
        return n;
    }
}

// Work order.  Items are dealt to the CTAs in a snake (round r goes left to
// right when r is even, right to left when odd) over a balanced order: every
// stream's full-length splits first, then the streams' last (shorter) splits
// by decreasing length.  The heavy items spread evenly and the light ones fill
// the gaps, so the last CTA to finish carries about the average load.
__device__ __forceinline__ int ws_snake(int k, int bid, int grid) {
    return k * grid + ((k & 1) ? grid - 1 - bid : bid);
}

// Keys of stream s's split length, and the number of TK-key tiles its last
// split takes (0 if the stream has no splits).
template <bool RING>
__device__ __forceinline__ int ws_split_len(const WsParams &p, int s) {
    if constexpr (RING) {
        return p.split_keys;
    } else {
        int per = p.split_keys;
        if (per <= 0) {
            const tf_seg e = p.segs[s];
            per = (e.n_keys + p.n_splits_max - 1) / p.n_splits_max;
            per = ((per + (1 << p.log2_page) - 1) >> p.log2_page) << p.log2_page;
        }
        return per;
    }
}

template <bool RING>
__device__ __forceinline__ WsItem ws_resolve(const WsParams &p, const int *prefix, const int *prefix_full,
                                             const int *tail_order, int n_full, int idx) {
    int lo, g, c;
    if (idx < n_full) {
        // a full-length split: the stream is the last prefix_full entry <= idx
        lo = 0;
        int hi = p.n_segs;  // prefix_full[lo] <= idx < prefix_full[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (prefix_full[mid] <= idx)
                lo = mid;
            else
                hi = mid;
        }
        const int n_f = (prefix[lo + 1] - prefix[lo]) / p.hkv - 1;  // full splits per kv-head
        const int r = idx - prefix_full[lo];
        g = r / n_f;
        c = r - g * n_f;
    } else {
        // a last split, in the tail order
        const int t = idx - n_full;
        lo = tail_order[t / p.hkv];
        g = t % p.hkv;
        c = (prefix[lo + 1] - prefix[lo]) / p.hkv - 1;
    }
    WsItem it;
    it.s = lo;
    it.g = g;
    it.c = c;
    if constexpr (RING) {
        const tf_ring_seg e = p.rsegs[lo];
        it.q_row = e.q_row;
        it.n_rows = 1;
        it.n_keys = e.n_valid;
        it.base = e.base;
        it.size = e.size;
        it.start = e.head - e.n_valid;
        if (it.start < 0) it.start += e.size;
        it.wrap_at = e.size - it.start;  // keys at or past this index wrapped to slot 0
        it.key_lo = it.c * p.split_keys;
        it.key_hi = min(it.n_keys, it.key_lo + p.split_keys);
        it.pt_base = 0;
        it.n_pg = 0;
    } else {
        const tf_seg e = p.segs[lo];
        it.q_row = e.q_row;
        it.n_rows = e.n_rows;
        it.n_keys = e.n_keys;
        it.pt_base = e.pt_base;
        it.n_pg = e.n_pages;
        int per = p.split_keys;
        if (per <= 0) {
            per = (e.n_keys + p.n_splits_max - 1) / p.n_splits_max;
            per = ((per + (1 << p.log2_page) - 1) >> p.log2_page) << p.log2_page;
        }
        it.key_lo = it.c * per;
        it.key_hi = min(it.n_keys, it.key_lo + per);
        it.base = 0;
        it.size = it.start = 0;
        it.wrap_at = 0x7fffffff;
    }
    // keys every row sees: [0, causal0); row i sees [0, causal0 + i) (with
    // the full flag every row sees all n_keys)
    it.causal0 = p.full ? it.n_keys : it.n_keys - it.n_rows + 1;
    it.full_hi = min(it.key_hi, it.causal0);
    return it;
}

// Next tile [j0, j0 + rows) of an item: TK keys, cut at the ring's wrap point.
template <int TK>
__device__ __forceinline__ int ws_tile_rows(const WsItem &it, int j0) {
    int j1 = min(j0 + TK, it.key_hi);
    if (j0 < it.wrap_at && j1 > it.wrap_at) j1 = it.wrap_at;
    return j1 - j0;
}

template <int D, bool RING>
__global__ void __launch_bounds__(WsCfg<D>::kThreads, WsCfg<D>::kMinBlocks)
    decode_ws_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const WsParams p) {
    using C = WsCfg<D>;
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[C::kStages], empty_bar[C::kStages];
    __shared__ __align__(8) uint64_t qfull_bar[C::kNQ], qempty_bar[C::kNQ];
    __shared__ uint32_t s_meta[C::kStages];
    __shared__ WsItem s_item[C::kNQ];  // the item of each query buffer, resolved by the producer
    __shared__ float comb_m[C::NC / 2][kWsQ], comb_l[C::NC / 2][kWsQ];
    __shared__ uint32_t comb_f[C::NC / 2][kWsQ];
    __shared__ int s_total, s_full;
    __shared__ uint32_t s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint64_t lim = p.wait_ns ? p.wait_ns : 2000000000ull;  // every bounded wait's limit
    const uint32_t sraw = smem_u32(smem_raw);
    const uint32_t sbase = (sraw + 1023u) & ~1023u;
    unsigned char *base_ptr = smem_raw + (sbase - sraw);
    int *prefix = reinterpret_cast<int *>(base_ptr + C::kOffPrefix);
    int *prefix_full = prefix + (C::kPrefixMax + 1);
    int *tail_order = prefix_full + (C::kPrefixMax + 1);
    constexpr int kBuckets = 64;  // tail lengths, in tiles (longer tails share the top bucket)
    __shared__ int s_bucket[kBuckets];
    float *comb_o = reinterpret_cast<float *>(base_ptr + C::kOffComb);

    // ---- prologue: barriers, the item prefix, empty-partial markers
    if (tid == 0) {
        for (int i = 0; i < C::kStages; ++i) {
            mbar_init(smem_u32(&full_bar[i]), 1);
            mbar_init(smem_u32(&empty_bar[i]), C::NC);
        }
        for (int i = 0; i < C::kNQ; ++i) {
            mbar_init(smem_u32(&qfull_bar[i]), 1);
            mbar_init(smem_u32(&qempty_bar[i]), C::NC);
        }
        fence_barrier_init();
        s_abort = 0;
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    if (!RING && warp == 1) {
        // the page table's first 16 KB into L2 while warp 0 works out the
        // items, so the producer's first page-id reads do not go to DRAM
        const int n = min(p.pt_len, 4096);
        for (int i = lane * 32; i < n; i += 32 * 32) prefetch_l2(p.page_table + i);
    }
    if (warp == 0) {
        // per stream: its items (splits x Hkv), its full-length ones, and the
        // tile count of its last split, bucketed for the tail order
        uint32_t bits = 0;
        int running = 0, running_full = 0;
        s_bucket[lane] = 0;
        s_bucket[lane + 32] = 0;
        __syncwarp();
        for (int b0 = 0; b0 < p.n_segs; b0 += 32) {
            const int s = b0 + lane;
            const int n_sp = s < p.n_segs ? ws_stream_splits<RING>(p, s, bits) : 0;
            const int units = n_sp * p.hkv, full = n_sp > 0 ? (n_sp - 1) * p.hkv : 0;
            if (n_sp > 0) {
                const int n_keys = RING ? p.rsegs[s].n_valid : p.segs[s].n_keys;
                const int tail = n_keys - (n_sp - 1) * ws_split_len<RING>(p, s);
                atomicAdd(&s_bucket[min(kBuckets, (tail + C::TK - 1) / C::TK) - 1], 1);
            }
            int incl = units, incl_f = full;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o), vf = __shfl_up_sync(0xffffffffu, incl_f, o);
                if (lane >= o) {
                    incl += v;
                    incl_f += vf;
                }
            }
            if (s < p.n_segs) {
                prefix[s] = running + incl - units;
                prefix_full[s] = running_full + incl_f - full;
            }
            running += __shfl_sync(0xffffffffu, incl, 31);
            running_full += __shfl_sync(0xffffffffu, incl_f, 31);
        }
        __syncwarp();
        if (lane == 0) {
            prefix[p.n_segs] = running;
            prefix_full[p.n_segs] = running_full;
            s_total = running;
            s_full = running_full;
        }
        {
            // bucket starts in the tail order, longest tails first: lane l
            // holds buckets 63 - 2l and 62 - 2l, and an exclusive scan over
            // the lanes gives each bucket the count of the longer ones
            const int hi = kBuckets - 1 - 2 * lane, lo = hi - 1;
            const int n_hi = s_bucket[hi], n_lo = s_bucket[lo];
            int incl = n_hi + n_lo;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            const int before = incl - n_hi - n_lo;
            __syncwarp();
            s_bucket[hi] = before;
            s_bucket[lo] = before + n_hi;
        }
        __syncwarp();
        // each stream with splits takes the next place of its bucket, streams
        // in index order within a bucket
        for (int b0 = 0; b0 < p.n_segs; b0 += 32) {
            const int s = b0 + lane;
            int bk = -1;
            if (s < p.n_segs) {
                const int units = prefix[s + 1] - prefix[s];
                if (units > 0) {
                    const int n_sp = units / p.hkv;
                    const int n_keys = RING ? p.rsegs[s].n_valid : p.segs[s].n_keys;
                    const int tail = n_keys - (n_sp - 1) * ws_split_len<RING>(p, s);
                    bk = min(kBuckets, (tail + C::TK - 1) / C::TK) - 1;
                }
            }
            const uint32_t same = __match_any_sync(0xffffffffu, bk);
            const int rank = __popc(same & ((1u << lane) - 1u));
            if (bk >= 0) tail_order[s_bucket[bk] + rank] = s;
            __syncwarp();
            if (bk >= 0 && rank == 0) s_bucket[bk] += __popc(same);
            __syncwarp();
        }
        bits |= __reduce_or_sync(0xffffffffu, bits);
        if (lane == 0 && bits && blockIdx.x == 0) atomicOr(p.status, bits);
    }
    __syncthreads();
    const int total = s_total, n_full = s_full;
    const int bid = (int)blockIdx.x, grid = (int)gridDim.x;

    if (warp == C::NC) {
        // ---- producer warp
        if constexpr (!RING) {
            // lanes 1..31: empty markers for partial slots past each stream's count
            if (lane > 0) {
                for (int s = blockIdx.x; s < p.n_segs; s += gridDim.x) {
                    const int n_sp = (prefix[s + 1] - prefix[s]) / p.hkv;
                    const tf_seg e = p.segs[s];
                    if (n_sp == 0) continue;  // invalid or empty streams are left as they are
                    const int extra = p.n_splits_max - n_sp;
                    const int cnt = e.n_rows * p.hq * extra;
                    for (int k = lane - 1; k < cnt; k += 31) {
                        const int c = n_sp + k % extra, uh = k / extra;
                        const int64_t at = ((int64_t)e.q_row * p.hq + uh) * p.n_splits_max + c;
                        p.part_m[at] = -INFINITY;
                        p.part_l[at] = 0.f;
                        p.part_flag[at] = 0;
                    }
                }
            }
        }
        // The whole warp walks the items; lane 0 issues the copies.  Page ids
        // come a window of 32 at a time (one coalesced load by the warp), and
        // the next item's window is requested before the current item's tiles
        // are issued, so no tile waits on a page-table read.  (Under the
        // timeout test hook it issues nothing: the consumers' waits run out.)
        if (!p.test_idle) {
            const int P = 1 << p.log2_page, BR = P < C::TK ? P : C::TK, n_box = C::TK / BR;
            auto load_window = [&](const WsItem &w, int w0) -> int {
                if constexpr (RING) {
                    return 0;
                } else {
                    const int idx = w0 + lane;
                    return idx < w.n_pg ? p.page_table[w.pt_base + idx] : -2;
                }
            };
            uint32_t tc = 0, qc = 0;
            bool ok = true;
            // an item goes to the consumers with its queries (a bulk copy into
            // the next of the kNQ query buffers); item k + 1 is published as
            // soon as item k's first tile has gone out, so its queries land
            // while item k's tiles stream
            auto publish = [&](const WsItem &w) -> bool {
                const uint32_t qs = qc % C::kNQ;
                if (qc >= (uint32_t)C::kNQ && !mbar_wait(smem_u32(&qempty_bar[qs]), ((qc / C::kNQ) - 1) & 1, lim))
                    return false;
                if (lane == 0) {
                    s_item[qs] = w;  // published with the queries (the arrive below releases it)
                    const uint32_t qdst = sbase + C::kOffQ + qs * C::kQBytes;
                    const uint32_t qbytes = (uint32_t)(p.group * D * 2);
                    mbar_arrive_expect_tx(smem_u32(&qfull_bar[qs]), qbytes * w.n_rows);
                    for (int i = 0; i < w.n_rows; ++i)
                        bulk_load(qdst + i * qbytes, p.q + ((int64_t)(w.q_row + i) * p.hq + w.g * p.group) * D,
                                  qbytes, smem_u32(&qfull_bar[qs]));
                }
                ++qc;
                return true;
            };
            int k = 0, L = ws_snake(0, bid, grid);
            WsItem it{};
            int win = 0, w0 = 0;
            if (L < total) {
                it = ws_resolve<RING>(p, prefix, prefix_full, tail_order, n_full, L);
                w0 = it.key_lo >> p.log2_page;
                win = load_window(it, w0);
                ok = publish(it);
            }
            while (L < total && ok) {
                // the next item is resolved, its page ids requested and its
                // queries published once this item's first tile has gone out
                // (so a CTA's first copy waits on nothing but its own page ids)
                const int L_next = ws_snake(k + 1, bid, grid);
                WsItem nx{};
                int win_next = 0, w0_next = 0;
                bool sent_next = false;
                auto prep_next = [&]() -> bool {
                    sent_next = true;
                    if (L_next >= total) return true;
                    nx = ws_resolve<RING>(p, prefix, prefix_full, tail_order, n_full, L_next);
                    w0_next = nx.key_lo >> p.log2_page;
                    win_next = load_window(nx, w0_next);
                    return publish(nx);
                };
                for (int j0 = it.key_lo; j0 < it.key_hi;) {
                    const int rows = ws_tile_rows<C::TK>(it, j0);
                    const uint32_t st = tc % C::kStages;
                    if (tc >= (uint32_t)C::kStages &&
                        !mbar_wait(smem_u32(&empty_bar[st]), ((tc / C::kStages) - 1) & 1, lim)) {
                        ok = false;
                        break;
                    }
                    const uint32_t dK = sbase + st * C::kStageBytes, dV = dK + C::kTileBytes;
                    const uint32_t fb = smem_u32(&full_bar[st]);
                    if constexpr (RING) {
                        if (lane == 0) {
                            int slot = it.start + j0;
                            if (slot >= it.size) slot -= it.size;
                            s_meta[st] = 0;
                            mbar_arrive_expect_tx(fb, 2u * C::kTileBytes);
                            const int row = (int)(it.base + slot);
#pragma unroll
                            for (int s = 0; s < C::kSlabs; ++s) {
                                tma_load_3d(dK + s * C::kSlab, &tmK, fb, 64 * s, it.g, row);
                                tma_load_3d(dV + s * C::kSlab, &tmV, fb, 64 * s, it.g, row);
                            }
                        }
                    } else {
                        if (((j0 + rows - 1) >> p.log2_page) - w0 >= 32) {  // past the window: slide it
                            w0 = j0 >> p.log2_page;
                            win = load_window(it, w0);
                        }
                        int pid[C::TK / 8];
                        uint32_t bad = 0, bytes = 0;
                        for (int b = 0; b < n_box; ++b) {
                            const int key0 = j0 + b * BR;
                            const int r = (key0 >> p.log2_page) - w0;
                            const int id = __shfl_sync(0xffffffffu, win, r & 31);
                            pid[b] = -1;
                            if (key0 < j0 + rows) {
                                if (id < 0 || id >= p.n_pages)
                                    bad = 1;
                                else {
                                    pid[b] = id;
                                    bytes += 2u * BR * 128 * C::kSlabs;
                                }
                            }
                        }
                        if (lane == 0) {
                            s_meta[st] = bad;
                            mbar_arrive_expect_tx(fb, bytes);
                            for (int b = 0; b < n_box; ++b) {
                                if (pid[b] < 0) continue;
                                const int key0 = j0 + b * BR;
#pragma unroll
                                for (int s = 0; s < C::kSlabs; ++s) {
                                    tma_load_4d(dK + s * C::kSlab + b * BR * 128, &tmK, fb, 64 * s, key0 & (P - 1),
                                                it.g, pid[b]);
                                    tma_load_4d(dV + s * C::kSlab + b * BR * 128, &tmV, fb, 64 * s, key0 & (P - 1),
                                                it.g, pid[b]);
                                }
                            }
                            if (bad) atomicOr(p.status, TF_DEV_BAD_PAGE);
                        }
                    }
                    ++tc;
                    j0 += rows;
                    if (!sent_next && !prep_next()) {
                        ok = false;
                        break;
                    }
                }
                if (ok && !sent_next && !prep_next()) ok = false;
                L = L_next;
                ++k;
                it = nx;
                win = win_next;
                w0 = w0_next;
            }
            if (!ok && lane == 0) {
                atomicOr(p.status, TF_DEV_TIMEOUT);
                s_abort = 1;
            }
        }
        asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    } else {
        // ---- consumer warps
        const int gq = lane >> 2, t4 = lane & 3;
        const float scale_log2 = p.scale_log2;
        uint32_t tc = 0, qc = 0;
        for (int k = 0, L = ws_snake(0, bid, grid); L < total; L = ws_snake(++k, bid, grid)) {
            // the item (resolved by the producer) and its queries -> B fragments
            // (Q^T), kept in registers
            const uint32_t qs = qc % C::kNQ;
            // (no barrier here: a warp that finishes an item's combine late joins
            // the next item late; a wait that gives up skips the item's tiles and
            // the loop-end barrier takes every warp out)
            const bool q_ok = mbar_wait(smem_u32(&qfull_bar[qs]), (qc / C::kNQ) & 1, lim);
            WsItem it = s_item[qs];
            if (!q_ok) it.key_lo = it.key_hi = 0;
            const int q_item = it.n_rows * p.group;
            uint32_t qb[D / 16][2];
            {
                const uint32_t qsrc = sbase + C::kOffQ + qs * C::kQBytes;
    #pragma unroll
                for (int ks = 0; ks < D / 16; ks += 2) {
                    const uint32_t a = qsrc + (lane & 7) * (D * 2) + (2 * ks + (lane >> 3)) * 16;
                    ldsm_x4(a, qb[ks][0], qb[ks][1], qb[ks + 1][0], qb[ks + 1][1]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&qempty_bar[qs]));
            ++qc;

            // per-thread state: queries 2*t4 and 2*t4+1; O^T rows d = 16*mt + gq (+8)
            const int qa = 2 * t4, qb_ = qa + 1;
            const int lim_a = qa < q_item ? min(it.key_hi, it.causal0 + qa / p.group) : it.key_hi;
            const int lim_b = qb_ < q_item ? min(it.key_hi, it.causal0 + qb_ / p.group) : it.key_hi;
            float o[D / 16][4];
    #pragma unroll
            for (int mt = 0; mt < D / 16; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
            float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
            uint32_t e0 = 0, e1 = 0, tb0 = 0, tb1 = 0, badp = 0;
            const int kb = warp * 16;
            bool aborted = !q_ok;

            for (int j0 = it.key_lo; j0 < it.key_hi;) {
                const int rows = ws_tile_rows<C::TK>(it, j0);
                const uint32_t st = tc % C::kStages;
                if (!mbar_wait(smem_u32(&full_bar[st]), (tc / C::kStages) & 1, lim)) {
                    aborted = true;
                    break;
                }
                badp |= s_meta[st];
                const uint32_t sK = sbase + st * C::kStageBytes, sV = sK + C::kTileBytes;
                bool wrote = false;
                if (kb < rows) {
                    // clean this warp's V rows: past the tile's keys -> 0; seen by only
                    // some rows and nonfinite -> 0 and flag the rows that see it
                    if (kb + 16 > rows || j0 + kb + 16 > it.full_hi) {
                        unsigned char *vrows = base_ptr + st * C::kStageBytes + C::kTileBytes;
                        // rows past the tile's keys hold other keys' values: zero them
                        for (int idx = lane; idx < 16 * C::kSlabs * 8; idx += 32) {
                            const int r = kb + idx / (C::kSlabs * 8);
                            const int rest = idx % (C::kSlabs * 8), sl = rest / 8, ch = rest % 8;
                            if (r >= rows) {
                                *reinterpret_cast<uint4 *>(vrows + sl * C::kSlab + r * 128 + ch * 16) =
                                    make_uint4(0, 0, 0, 0);
                                wrote = true;
                            }
                        }
                        // rows only some of the item's rows see: one lane scans one row;
                        // a nonfinite row is zeroed and flags the queries that see it
                        uint32_t nf = 0;
                        if (lane < 16) {
                            const int r = kb + lane;
                            if (r < rows && j0 + r >= it.full_hi) {
                                for (int sl = 0; sl < C::kSlabs; ++sl) {
                                    const uint4 *rp = reinterpret_cast<const uint4 *>(vrows + sl * C::kSlab + r * 128);
    #pragma unroll
                                    for (int ch = 0; ch < 8; ++ch) {
                                        const uint4 v = rp[ch];
                                        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
    #pragma unroll
                                        for (int e = 0; e < 4; ++e)
                                            nf |= (((w4[e] & 0x7f80u) == 0x7f80u) ||
                                                   ((w4[e] & 0x7f800000u) == 0x7f800000u))
                                                      ? 1u
                                                      : 0u;
                                    }
                                }
                                if (nf) {
                                    for (int sl = 0; sl < C::kSlabs; ++sl) {
                                        uint4 *wp = reinterpret_cast<uint4 *>(vrows + sl * C::kSlab + r * 128);
    #pragma unroll
                                        for (int ch = 0; ch < 8; ++ch) wp[ch] = make_uint4(0, 0, 0, 0);
                                    }
                                    wrote = true;
                                }
                            }
                        }
                        const uint32_t badrows = __ballot_sync(0xffffffffu, nf != 0) & 0xffffu;
                        for (int r = 0; r < 16; ++r)
                            if ((badrows >> r) & 1u) {
                                const int key = j0 + kb + r;
                                if (key < lim_a) tb0 = 1;
                                if (key < lim_b) tb1 = 1;
                            }
                        __syncwarp();
                    }

                    // ---- S^T = K Q^T for this warp's 16 keys
                    // two accumulators (even / odd k-steps) halve the MMA dependency chain
                    float s4[4] = {0.f, 0.f, 0.f, 0.f}, s5[4] = {0.f, 0.f, 0.f, 0.f};
    #pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const int r = kb + (lane & 7) + (((lane >> 3) & 1) << 3);
                        const int ch = 2 * ks + (lane >> 4);
                        const uint32_t a = sK + (ch >> 3) * C::kSlab + r * 128 + (((ch & 7) ^ (r & 7)) << 4);
                        uint32_t a0, a1, a2, a3;
                        ldsm_x4(a, a0, a1, a2, a3);
                        if (ks & 1)
                            mma_bf16(s5, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
                        else
                            mma_bf16(s4, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
                    }
                    s4[0] += s5[0];
                    s4[1] += s5[1];
                    s4[2] += s5[2];
                    s4[3] += s5[3];
                    // mask, check, online softmax (queries qa, qb_ ; keys rows kb+gq, kb+gq+8)
                    const int ra = kb + gq, rb = ra + 8;
                    const int ka = j0 + ra, kbk = j0 + rb;
                    const bool va0 = ra < rows && ka < lim_a, va1 = ra < rows && ka < lim_b;
                    const bool vb0 = rb < rows && kbk < lim_a, vb1 = rb < rows && kbk < lim_b;
                    float x0 = s4[0] * scale_log2, x1 = s4[1] * scale_log2, x2 = s4[2] * scale_log2,
                          x3 = s4[3] * scale_log2;
                    e0 = max(e0, max(va0 ? exp_bits(x0) : 0u, vb0 ? exp_bits(x2) : 0u));
                    e1 = max(e1, max(va1 ? exp_bits(x1) : 0u, vb1 ? exp_bits(x3) : 0u));
                    x0 = va0 ? x0 : -INFINITY;
                    x1 = va1 ? x1 : -INFINITY;
                    x2 = vb0 ? x2 : -INFINITY;
                    x3 = vb1 ? x3 : -INFINITY;
                    float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
    #pragma unroll
                    for (int o_ = 4; o_ < 32; o_ <<= 1) {
                        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o_));
                        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o_));
                    }
                    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
                    const float mu0 = (mn0 == -INFINITY) ? 0.f : mn0, mu1 = (mn1 == -INFINITY) ? 0.f : mn1;
                    const float al0 = ex2(m0 - mu0), al1 = ex2(m1 - mu1);
                    m0 = mn0;
                    m1 = mn1;
                    const float p0 = ex2(x0 - mu0), p1 = ex2(x1 - mu1), p2 = ex2(x2 - mu0), p3 = ex2(x3 - mu1);
                    l0 = l0 * al0 + p0 + p2;
                    l1 = l1 * al1 + p1 + p3;
                    if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
    #pragma unroll
                        for (int mt = 0; mt < D / 16; ++mt) {
                            o[mt][0] *= al0;
                            o[mt][1] *= al1;
                            o[mt][2] *= al0;
                            o[mt][3] *= al1;
                        }
                    }
                    // P^T fragments: (keys 2t4.., query gq) from (key gq.., queries 2t4..)
                    const uint32_t h01 = pack_bf16x2(p0, p1), h23 = pack_bf16x2(p2, p3);
                    const uint32_t r01 = pack_bf16x2(p0 - bf16_lo_to_f32(h01), p1 - bf16_hi_to_f32(h01));
                    const uint32_t r23 = pack_bf16x2(p2 - bf16_lo_to_f32(h23), p3 - bf16_hi_to_f32(h23));
                    const uint32_t bh0 = movmatrix_t(h01), bh1 = movmatrix_t(h23);
                    const uint32_t bl0 = movmatrix_t(r01), bl1 = movmatrix_t(r23);
                    // ---- O^T += V^T P^T
    #pragma unroll
                    for (int mt = 0; mt < D / 16; ++mt) {
                        const int r = kb + (lane & 7) + ((lane >> 4) << 3);
                        const int ch = 2 * mt + ((lane >> 3) & 1);
                        const uint32_t a = sV + (ch >> 3) * C::kSlab + r * 128 + (((ch & 7) ^ (r & 7)) << 4);
                        uint32_t a0, a1, a2, a3;
                        ldsm_x4_t(a, a0, a1, a2, a3);
                        mma_bf16(o[mt], a0, a1, a2, a3, bh0, bh1);
                        mma_bf16(o[mt], a0, a1, a2, a3, bl0, bl1);
                    }
                }
                __syncwarp();
                if (wrote) fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&empty_bar[st]));
                ++tc;
                j0 += rows;
            }
            if (named_bar_red_or(1, C::NC * 32, aborted)) {  // every consumer warp leaves together
                if (tid == 0) {
                    atomicOr(p.status, TF_DEV_TIMEOUT);
                    s_abort = 1;
                }
                break;
            }

            // ---- combine the four warps (tree through shared memory) and write
    #pragma unroll
            for (int o_ = 4; o_ < 32; o_ <<= 1) {
                l0 += __shfl_xor_sync(0xffffffffu, l0, o_);
                l1 += __shfl_xor_sync(0xffffffffu, l1, o_);
                e0 = max(e0, __shfl_xor_sync(0xffffffffu, e0, o_));
                e1 = max(e1, __shfl_xor_sync(0xffffffffu, e1, o_));
                tb0 |= __shfl_xor_sync(0xffffffffu, tb0, o_);
                tb1 |= __shfl_xor_sync(0xffffffffu, tb1, o_);
            }
            uint32_t f0 = (e0 == 0x7f800000u) | tb0 | badp, f1 = (e1 == 0x7f800000u) | tb1 | badp;
            auto put = [&](int slot) {
                float *dst = comb_o + slot * kWsQ * C::kCombStride;
    #pragma unroll
                for (int mt = 0; mt < D / 16; ++mt) {
                    dst[qa * C::kCombStride + 16 * mt + gq] = o[mt][0];
                    dst[qb_ * C::kCombStride + 16 * mt + gq] = o[mt][1];
                    dst[qa * C::kCombStride + 16 * mt + gq + 8] = o[mt][2];
                    dst[qb_ * C::kCombStride + 16 * mt + gq + 8] = o[mt][3];
                }
                if (gq == 0) {
                    comb_m[slot][qa] = m0;
                    comb_m[slot][qb_] = m1;
                    comb_l[slot][qa] = l0;
                    comb_l[slot][qb_] = l1;
                    comb_f[slot][qa] = f0;
                    comb_f[slot][qb_] = f1;
                }
            };
            auto take = [&](int slot) {
                const float *src = comb_o + slot * kWsQ * C::kCombStride;
                const float ma = comb_m[slot][qa], mb = comb_m[slot][qb_];
                const float la = comb_l[slot][qa], lb = comb_l[slot][qb_];
                f0 |= comb_f[slot][qa];
                f1 |= comb_f[slot][qb_];
                const float M0 = fmaxf(m0, ma), M1 = fmaxf(m1, mb);
                const float u0 = (M0 == -INFINITY) ? 0.f : M0, u1 = (M1 == -INFINITY) ? 0.f : M1;
                const float w0 = ex2(m0 - u0), w1 = ex2(m1 - u1), wa = ex2(ma - u0), wb = ex2(mb - u1);
                l0 = l0 * w0 + la * wa;
                l1 = l1 * w1 + lb * wb;
                m0 = M0;
                m1 = M1;
    #pragma unroll
                for (int mt = 0; mt < D / 16; ++mt) {
                    o[mt][0] = o[mt][0] * w0 + src[qa * C::kCombStride + 16 * mt + gq] * wa;
                    o[mt][1] = o[mt][1] * w1 + src[qb_ * C::kCombStride + 16 * mt + gq] * wb;
                    o[mt][2] = o[mt][2] * w0 + src[qa * C::kCombStride + 16 * mt + gq + 8] * wa;
                    o[mt][3] = o[mt][3] * w1 + src[qb_ * C::kCombStride + 16 * mt + gq + 8] * wb;
                }
            };
            // Warps 2 and 3 hand their states to warps 0 and 1 and go on to the
            // next item; warp 1 then hands its state to warp 0, which writes the
            // item's partials from its registers.  The slots are free again before
            // the next item's combine: every warp passes the loop-end barrier first.
            if (warp >= 2) put(warp - 2);
            named_bar_sync(1, C::NC * 32);
            if (warp < 2) {
                take(warp);
                named_bar_sync(2, 64);  // warp 0 has read slot 0: warp 1 may refill it
                if (warp == 1) put(0);
                named_bar_sync(2, 64);
            }
            if (warp == 0) {
                take(0);
                bool nf0 = !isfinite(l0), nf1 = !isfinite(l1);
    #pragma unroll
                for (int mt = 0; mt < D / 16; ++mt) {
                    nf0 |= !isfinite(o[mt][0]) || !isfinite(o[mt][2]);
                    nf1 |= !isfinite(o[mt][1]) || !isfinite(o[mt][3]);
                }
    #pragma unroll
                for (int o_ = 4; o_ < 32; o_ <<= 1) {
                    nf0 |= __shfl_xor_sync(0xffffffffu, nf0, o_);
                    nf1 |= __shfl_xor_sync(0xffffffffu, nf1, o_);
                }
                f0 |= nf0;
                f1 |= nf1;
                // this lane's queries qa, qb_ and dims 16 mt + gq (+ 8): eight
                // consecutive floats of a row per four lanes
                auto slot_of = [&](int qq) {
                    const int i = qq / p.group, hl = qq - i * p.group;
                    const int64_t u = RING ? (int64_t)it.s * p.hq + it.g * p.group + hl
                                           : (int64_t)(it.q_row + i) * p.hq + it.g * p.group + hl;
                    return u * p.n_splits_max + it.c;
                };
                if (qa < q_item) {
                    const int64_t at = slot_of(qa);
                    float *dst = p.part_o + at * D;
    #pragma unroll
                    for (int mt = 0; mt < D / 16; ++mt) {
                        dst[16 * mt + gq] = o[mt][0];
                        dst[16 * mt + gq + 8] = o[mt][2];
                    }
                    if (gq == 0) {
                        p.part_m[at] = (m0 == -INFINITY) ? -INFINITY : m0 * kLn2;
                        p.part_l[at] = l0;
                        p.part_flag[at] = (uint8_t)(f0 ? 1 : 0);
                    }
                }
                if (qb_ < q_item) {
                    const int64_t at = slot_of(qb_);
                    float *dst = p.part_o + at * D;
    #pragma unroll
                    for (int mt = 0; mt < D / 16; ++mt) {
                        dst[16 * mt + gq] = o[mt][1];
                        dst[16 * mt + gq + 8] = o[mt][3];
                    }
                    if (gq == 0) {
                        p.part_m[at] = (m1 == -INFINITY) ? -INFINITY : m1 * kLn2;
                        p.part_l[at] = l1;
                        p.part_flag[at] = (uint8_t)(f1 ? 1 : 0);
                    }
                }
            }
        }
    }

    // ---- a CTA that gave up (a bounded wait ran out) must not leave while
    // copies it issued are still landing in its shared memory: each stage's
    // and query buffer's barrier gets a bounded wait for the phase it is in
    // (a TMA box or bulk copy in flight completes it; an idle one times out
    // after 20 ms), then the CTA exits
    __syncthreads();
    if (s_abort && tid == 0) {
        for (int i = 0; i < C::kStages; ++i) {
            mbar_wait(smem_u32(&full_bar[i]), 0u, 20000000ull);
            mbar_wait(smem_u32(&full_bar[i]), 1u, 20000000ull);
        }
        for (int i = 0; i < C::kNQ; ++i) {
            mbar_wait(smem_u32(&qfull_bar[i]), 0u, 20000000ull);
            mbar_wait(smem_u32(&qfull_bar[i]), 1u, 20000000ull);
        }
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

// CTAs of a persistent launch on the current device: its SM count times the
// CTAs of the kernel an SM holds.  Both are facts of the device and the
// kernel, so each instance looks them up once per device and keeps them.
template <int D, bool RING>
static int ws_grid_cap() {
    constexpr int kMaxDevices = 64;
    static std::atomic<int> cap[kMaxDevices];  // 0: not looked up yet
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    const int known = cap[dev].load(std::memory_order_relaxed);
    if (known > 0) return known;
    int n = 148, per_sm = 1;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 148;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_ws_kernel<D, RING>, WsCfg<D>::kThreads,
                                                      WsCfg<D>::kSmem) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    cap[dev].store(n * per_sm, std::memory_order_relaxed);
    return n * per_sm;
}

template <int D, bool RING>
static cudaError_t launch_ws_t(const WsParams &p, const void *k, const void *v, int64_t n_items_bound,
                               cudaStream_t st) {
    CUtensorMap mk, mv;
    if (RING) {
        const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)p.hkv, (cuuint64_t)p.ring_slots_total};
        const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)p.hkv * D * 2};
        const cuuint32_t box[3] = {64, 1, (cuuint32_t)WsCfg<D>::TK};
        if (!make_tensor_map_bf16(&mk, k, 3, dims, strides, box)) return cudaErrorInvalidValue;
        if (!make_tensor_map_bf16(&mv, v, 3, dims, strides, box)) return cudaErrorInvalidValue;
    } else {
        const int P = 1 << p.log2_page, BR = P < WsCfg<D>::TK ? P : WsCfg<D>::TK;
        const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)P, (cuuint64_t)p.hkv, (cuuint64_t)p.n_pages};
        const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)P * D * 2, (cuuint64_t)p.hkv * P * D * 2};
        const cuuint32_t box[4] = {64, (cuuint32_t)BR, 1, 1};
        if (!make_tensor_map_bf16(&mk, k, 4, dims, strides, box)) return cudaErrorInvalidValue;
        if (!make_tensor_map_bf16(&mv, v, 4, dims, strides, box)) return cudaErrorInvalidValue;
    }
    auto kern = decode_ws_kernel<D, RING>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, WsCfg<D>::kSmem);
    if (e != cudaSuccess) return e;
    int64_t grid = ws_grid_cap<D, RING>();
    if (n_items_bound < grid) grid = n_items_bound < 1 ? 1 : n_items_bound;
    WsParams q = p;
    if (const uint64_t runout = test_wait_runout_ns()) {
        q.test_idle = 1;
        q.wait_ns = runout;
    }
    kern<<<(unsigned)grid, WsCfg<D>::kThreads, WsCfg<D>::kSmem, st>>>(mk, mv, q);
    return cudaGetLastError();
}

bool decode_ws_supported(int head_dim, int n_segs) {
    switch (head_dim) {
        case 64: return n_segs >= 1 && n_segs <= WsCfg<64>::kPrefixMax;
        case 128: return n_segs >= 1 && n_segs <= WsCfg<128>::kPrefixMax;
        case 256: return n_segs >= 1 && n_segs <= WsCfg<256>::kPrefixMax;
        default: return false;
    }
}

cudaError_t launch_decode_ws(const WsParams &p, int head_dim, bool ring, const void *k, const void *v,
                             int64_t n_items_bound, cudaStream_t st) {
    switch (head_dim) {
        case 64: return ring ? launch_ws_t<64, true>(p, k, v, n_items_bound, st)
                             : launch_ws_t<64, false>(p, k, v, n_items_bound, st);
        case 128: return ring ? launch_ws_t<128, true>(p, k, v, n_items_bound, st)
                              : launch_ws_t<128, false>(p, k, v, n_items_bound, st);
        case 256: return ring ? launch_ws_t<256, true>(p, k, v, n_items_bound, st)
                              : launch_ws_t<256, false>(p, k, v, n_items_bound, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace tfp
