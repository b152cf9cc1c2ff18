// prompt_tc.cu - causal prompt chunk through the page table on the 5th-generation
// tensor cores (tcgen05 + tensor memory), tiles fed by TMA.
//
// Source: TensorFold #1653 "spark25 CUDA: the full layers' caches in pages of
// the core pool", commit list and PR body: prompt rows read the chunk's keys
// through the slot's page-table row (the _pg prompt kernel, head dim 256,
// pages of 32); review thread: the per-chunk page lookup is hoisted out of the
// key loop.
//
// One CTA computes 128 queries: 128/G consecutive rows x the G q-heads that
// share kv-head g, so one K/V tile serves all of them.  Ten warps split the
// work by role: a TMA warp, an MMA warp and eight softmax warps.  Per 64-key
// tile:
//   1. the TMA warp brings K (and V) in 128-byte-swizzled 64-column slabs, one
//      box per page (or per 64-key span of a larger page) and slab, every lane
//      issuing one box; the CTA's page ids were copied to shared memory once,
//      so no page-table read sits in the key loop;
//   2. the MMA warp issues S = Q K^T (M 128, N 64, K = D) into tensor memory,
//      one tile ahead of the softmax (two S buffers).  Q itself sits in tensor
//      memory (the softmax warps put it there once), so the MMAs read only K
//      from shared memory: shared-memory bandwidth, not the tensor pipe, is
//      what an M = 128 tile runs out of first;
//   3. two softmax threads share a query row, 32 key columns each: they load
//      their S columns from tensor memory, mask them causally, swap their
//      maxima through shared memory and fold the tile into a running max / sum
//      with a lazy rescale (the reference max moves only when it rises by 2^8);
//   4. the weights go back to tensor memory (into the S columns they came
//      from) and the MMA warp issues O += P V (A from tensor memory, B = V in
//      shared memory, MN-major).  For f32 output P is fed as bf16 hi + bf16 lo
//      (two MMAs, about 16 bits a weight, so the fp32 tolerance holds); for
//      bf16 output P is one bf16, whose rounding is below the output's own;
//   5. O stays in tensor memory until the epilogue divides by the sum.
// K and V each have three buffers; a buffer is refilled as soon as the MMA
// that read it has completed.
// Nonfinite handling matches the other attention kernels: visible scores are
// checked through their exponent bits, value rows that only some rows see
// are scanned and zeroed, and the final O and sum are checked.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "tf_common.cuh"
#include "tf_internal.h"
#include "tf_sm100.cuh"
#include "tma_host.h"

namespace tfp {

// Eight softmax warps: warps q and q + 4 share the tensor-memory lane quadrant
// q (query rows 32q .. 32q + 31) and take 32 of a tile's 64 key columns each,
// so every SM sub-partition has two softmax warps to interleave.
constexpr int kPTSoftmax = 256;
constexpr int kPTThreads = kPTSoftmax + 64;   // + an MMA warp and a TMA warp
constexpr int kPTMmaWarp = kPTSoftmax / 32, kPTTmaWarp = kPTMmaWarp + 1;
// named barriers: 1 the softmax warps, 2-5 a softmax warp pair, kTmemBar the
// tensor-memory hand-out to the softmax and MMA warps
constexpr int kTmemBar = 6;
constexpr int kQM = 128;                      // queries a CTA (the MMA's M)
constexpr int kBN = 64;                       // keys a tile
constexpr int kKVSlab = kBN * 128;            // 64 key rows x 128 bytes
constexpr int kKVStages = 3;                  // K and V buffers in flight
// tensor-memory columns: two S tiles, Q (D/2 columns of bf16 pairs), O
constexpr uint32_t kColS0 = 0, kColS1 = 64, kColQ = 128, kColO = 256;

// Split-KV partials at head dim <= 128 run two CTAs to an SM: both fit in
// registers and shared memory, and while one holds the tensor memory the other
// starts (barriers, page ids, its first K/V stages, Q into registers) and
// waits in the allocation.  A prompt chunk's CTA has the SM to itself.
template <int D, bool PARTIAL>
__host__ __device__ constexpr bool pt_paired() { return PARTIAL && D <= 128; }

template <int D, bool PAIRED>
struct PTCfg {
    static constexpr int kSlabs = D / 64;
    static constexpr int kKVBytes = kSlabs * kKVSlab;
    // kKVStages K buffers, then kKVStages V buffers, then the page ids
    static constexpr int kOffK = 0;
    static constexpr int kOffV = kKVStages * kKVBytes;
    // page ids held in shared memory (16 KB; 4 KB, 8,192 keys at pages of 8 or
    // more, for a split when two CTAs share the SM)
    static constexpr int kPidCap = PAIRED ? 1024 : 4096;
    static constexpr int kOffPid = 2 * kKVStages * kKVBytes;
    static constexpr int kSmemBytes = kOffPid + kPidCap * 4 + 1024;
    static constexpr uint32_t kTmemCols = 512;
};

// Bounded wait that gives up at once after any thread of the CTA gave up, so
// every role keeps its barrier sequence without waiting twice the timeout.
__device__ __forceinline__ bool pt_wait(uint32_t bar, uint32_t phase, volatile uint32_t *abort_flag, uint64_t lim) {
    if (*abort_flag) return false;
    if (mbar_wait(bar, phase, lim)) return true;
    *abort_flag = 1;
    return false;
}

// barrier slots
constexpr int kBarQ = 0;                            // Q in tensor memory (softmax warps arrive)
constexpr int kBarKFull = 1;                        // [kKVStages] K tile landed
constexpr int kBarVFull = kBarKFull + kKVStages;    // [kKVStages] V tile landed
constexpr int kBarKFree = kBarVFull + kKVStages;    // [kKVStages] QK that read the K buffer done
constexpr int kBarVFree = kBarKFree + kKVStages;    // [kKVStages] P V that read the V buffer done
constexpr int kBarS = kBarVFree + kKVStages;        // [2] QK done: S tile ready
constexpr int kBarPr = kBarS + 2;                   // [2] P written, V cleaned (softmax warps arrive)
constexpr int kBarO = kBarPr + 2;                   // [2] P V done
constexpr int kNumBars = kBarO + 2;

template <int D, bool HILO, bool PARTIAL, bool TREE = false>
__global__ void __launch_bounds__(kPTThreads, pt_paired<D, PARTIAL>() ? 2 : 1)
    prompt_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const PromptTcParams p) {
    using C = PTCfg<D, pt_paired<D, PARTIAL>()>;
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t bars[kNumBars];
    __shared__ uint32_t s_tmem;
    __shared__ uint32_t s_vbad[4];
    __shared__ uint32_t s_err, s_abort;
    __shared__ float s_xmax[2][2][kQM];     // [tile parity][column half][row]: the halves' tile maxima
    __shared__ float s_xl[2][kQM];          // [column half][row]: final partial sums
    __shared__ uint32_t s_xbad[2][2][kQM];  // [exchange][column half][row]: nonfinite findings
    __shared__ int s_par[TREE ? kTreeMaxNodes : 1];  // a draft tree's parents

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint64_t lim = p.wait_ns ? p.wait_ns : 2000000000ull;  // every bounded wait's limit
    // the merge that follows may launch now; it waits for this grid to finish
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    unsigned char *sbase_ptr = smem_raw + (sbase - smem_u32(smem_raw));
    auto sK = [&](int s) { return sbase + C::kOffK + s * C::kKVBytes; };
    auto sV = [&](int s) { return sbase + C::kOffV + s * C::kKVBytes; };
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    volatile uint32_t *abort_flag = &s_abort;
    bool sent_row = false;  // this thread sent a staged row with a bulk copy

    const int G = p.group, RT = kQM / p.group;  // rows a tile
    // partials: kv-head blockIdx.y; a prompt chunk: the launch order (block
    // x fastest, then y) walks the query tiles from the most keys down, every
    // kv-head's tile in turn, so the longest tiles of all heads start first
    const int lin = (int)(blockIdx.y * gridDim.x + blockIdx.x);
    const int g = PARTIAL ? (int)blockIdx.y : lin % (int)gridDim.y;
    const int P = 1 << p.log2_page, BR = P < kBN ? P : kBN, n_box = kBN / BR;

    // ---- the work item: a segment (the prompt's one, or entry blockIdx.z of
    // the table), a tile of 128/G rows and, for partials, a split of the keys
    int q_row = p.q_row, T = p.n_rows, N = p.n_keys, pt_base = p.pt_base, n_pg = p.n_pg;
    int qt, split = 0, key_lo = 0, key_hi_split;
    // a draft tree (entry blockIdx.z of the tree table): the ring row of the
    // split's first key, the window's length, the tree's parents' base
    int64_t t_row0 = 0;
    int t_valid = 0, t_pbase = 0;
    if constexpr (PARTIAL) {
        split = (int)blockIdx.x / p.n_qt;
        qt = p.n_qt - 1 - (int)blockIdx.x % p.n_qt;  // the most keys first
        int n_sp;
        if constexpr (TREE) {
            const tf_tree_seg e = p.tsegs[blockIdx.z];
            if (!tree_seg_ok(e, p.n_rows_total, p.n_parents, p.ring_slots_total)) {
                if (tid == 0) atomicOr(p.status, TF_DEV_BAD_SEG);
                return;
            }
            const TreeSplits ts = tree_splits(e, p.split_keys);
            if (ts.n_sp > p.n_splits_max) {
                if (tid == 0) atomicOr(p.status, TF_DEV_SPLITS);
                return;
            }
            q_row = e.q_row;
            T = e.n_nodes;
            N = ts.n_keys;
            t_valid = e.n_valid;
            t_pbase = e.parent_base;
            n_sp = ts.n_sp;
            // splits never cross the ring's end: the run before it, then the run after
            if (split < ts.sa) {
                key_lo = split * p.split_keys;
                key_hi_split = min(ts.na, key_lo + p.split_keys);
            } else {
                key_lo = ts.na + (split - ts.sa) * p.split_keys;
                key_hi_split = min(N, key_lo + p.split_keys);
            }
            t_row0 = e.base + (key_lo < ts.wrap_at ? ts.start + key_lo : key_lo - ts.wrap_at);
        } else {
            const tf_seg sg = p.segs[blockIdx.z];
            q_row = sg.q_row;
            T = sg.n_rows;
            N = sg.n_keys;
            pt_base = sg.pt_base;
            n_pg = sg.n_pages;
            const int keys_needed = p.full ? (T > 0 ? 1 : 0) : T;  // the causal count needs a key per row
            const bool bad = q_row < 0 || T < 0 || (int64_t)q_row + T > p.n_rows_total || N < keys_needed ||
                             pt_base < 0 || n_pg < 0 || (int64_t)pt_base + n_pg > p.pt_len;
            if (bad) {
                if (tid == 0) atomicOr(p.status, TF_DEV_BAD_SEG);
                return;
            }
            if ((int64_t)N > ((int64_t)n_pg << p.log2_page)) {
                if (tid == 0) atomicOr(p.status, TF_DEV_PAST_PAGES);
                return;
            }
            n_sp = (N + p.split_keys - 1) / p.split_keys;
            if (n_sp > p.n_splits_max) {
                if (tid == 0) atomicOr(p.status, TF_DEV_SPLITS);
                return;
            }
            key_lo = split * p.split_keys;
            key_hi_split = min(N, key_lo + p.split_keys);
        }
        if (qt * RT >= T) return;
        if (split >= n_sp) {
            // a partial slot past the stream's count: an empty partial, o untouched
            for (int r = tid; r < min(RT, T - qt * RT) * G; r += kPTThreads) {
                const int64_t at = ((int64_t)(q_row + qt * RT + r / G) * p.hq + g * G + r % G) * p.n_splits_max + split;
                p.part_m[at] = -INFINITY;
                p.part_l[at] = 0.f;
                p.part_flag[at] = 0;
            }
            return;
        }
    } else {
        qt = (int)gridDim.x - 1 - lin / (int)gridDim.y;  // the most keys first
        key_hi_split = N;
    }
    const int row0 = qt * RT;  // segment-relative first row
    const int rows_here = min(RT, T - row0);
    // row i of the segment sees keys [0, causal0 + i) (all N with the full
    // flag); a tree's node sees the window [0, n_valid) and its path's nodes
    const int causal0 = (PARTIAL && p.full) ? N : N - T + 1;
    // keys the last valid row sees, and keys every row of the tile sees
    const int key_hi_eff = TREE ? key_hi_split : min(key_hi_split, causal0 + row0 + rows_here - 1);
    const int full_hi = TREE ? min(key_hi_eff, t_valid) : min(key_hi_eff, causal0 + row0);
    const int n_tiles = key_hi_eff > key_lo ? (key_hi_eff - key_lo + kBN - 1) / kBN : 0;
    if (PARTIAL && n_tiles == 0) {
        // no row of the tile sees a key of this split: m = -inf, l = 0, o = 0
        for (int r = tid; r < rows_here * G; r += kPTThreads) {
            const int64_t at = ((int64_t)(q_row + row0 + r / G) * p.hq + g * G + r % G) * p.n_splits_max + split;
            p.part_m[at] = -INFINITY;
            p.part_l[at] = 0.f;
            p.part_flag[at] = 0;
            for (int d = 0; d < D; d += 4)
                *reinterpret_cast<float4 *>(p.part_o + at * D + d) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        return;
    }

    // The CTA's page ids (pages pg_lo .. of its key range), read once here by
    // every thread (coalesced), so the TMA warp never waits on a page-table
    // read inside the key loop.
    int *pids = reinterpret_cast<int *>(sbase_ptr + C::kOffPid);
    const int pg_lo = key_lo >> p.log2_page;
    if constexpr (TREE) {
        // a tree has no pages; its parents go to shared memory instead
        for (int i = tid; i < T; i += kPTThreads) s_par[i] = p.parents[t_pbase + i];
    } else {
        const int n_pid = min((key_hi_eff + P - 1) >> p.log2_page, n_pg) - pg_lo;
        for (int i = tid; i < n_pid && i < C::kPidCap; i += kPTThreads) {
            const int id = p.page_table[pt_base + pg_lo + i];
            pids[i] = (id < 0 || id >= p.n_pages) ? -1 : id;
        }
    }
    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i)
            mbar_init(bar(i), (i == kBarQ || i == kBarPr || i == kBarPr + 1) ? kPTSoftmax / 32u : 1u);
        fence_barrier_init();
        s_err = 0;
        s_abort = 0;
        s_vbad[0] = s_vbad[1] = s_vbad[2] = s_vbad[3] = 0;
    }
    __syncthreads();
    // Tensor memory comes later (take_tmem): the TMA warp needs none and
    // starts on the K/V stages at once, the softmax warps first fetch Q.
    uint32_t tmem = 0;
    auto take_tmem = [&]() {
        if (warp == 0) {
            tmem_alloc(smem_u32(&s_tmem), C::kTmemCols);  // waits while another CTA of the SM holds it
            tmem_relinquish();
        }
        tc_fence_before();
        named_bar_sync(kTmemBar, kPTThreads - 32);  // the softmax warps and the MMA warp
        tc_fence_after();
        tmem = s_tmem;
    };

    // every lane of a helper warp waits; the answer is the warp's, so all lanes branch alike
    auto wwait = [&](uint32_t b, uint32_t phase) { return __all_sync(0xffffffffu, pt_wait(b, phase, abort_flag, lim)); };
    if (warp == kPTTmaWarp) {
        // ================= TMA warp: the K/V boxes of a tile go out one per lane,
        // so one warp instruction issues all of them; a buffer is refilled as
        // soon as the MMA that read it is done
        if (lane == 0) {
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
        }
        const int n_copies = n_box * C::kSlabs;  // boxes of one K (or V) tile, <= 32
        // K or V tile t into stage t % kKVStages: one box per page (or per
        // 64-key span of a larger page) and 64-column slab; page ids come from
        // shared memory
        auto issue_kv = [&](int t, bool is_v) {
            const int kt = key_lo + t * kBN, s = t % kKVStages;
            const uint32_t dst0 = is_v ? sV(s) : sK(s);
            const uint32_t full = bar((is_v ? kBarVFull : kBarKFull) + s);
            const CUtensorMap *map = is_v ? &tmV : &tmK;
            if constexpr (TREE) {
                // a split's slots are contiguous: one 64-slot box per slab
                // (rows past the split read neighbouring slots, or zeros past
                // the arrays, and are masked)
                if (lane == 0) mbar_arrive_expect_tx(full, (uint32_t)C::kKVBytes);
                __syncwarp();
                if (lane < C::kSlabs)
                    tma_load_3d(dst0 + lane * kKVSlab, map, full, 64 * lane, g, (int)(t_row0 + (kt - key_lo)));
                return;
            }
            // lane i < n_copies owns box x = i / slabs, slab sl = i % slabs
            const int x = lane / C::kSlabs, sl = lane % C::kSlabs;
            const int key0 = kt + x * BR;
            int id = -1;
            if (lane < n_copies && key0 < key_hi_eff) {
                const int idx = key0 >> p.log2_page;
                if (idx >= n_pg)
                    id = -2;
                else if (idx - pg_lo < C::kPidCap)
                    id = pids[idx - pg_lo];
                else  // past the shared-memory copy (very long prompts with small pages)
                    id = p.page_table[pt_base + idx];
                if (id < 0 || id >= p.n_pages) {
                    id = -1;
                    s_err = 1;
                    atomicOr(p.status, TF_DEV_BAD_PAGE);
                }
            }
            const uint32_t live = __ballot_sync(0xffffffffu, id >= 0);
            if (lane == 0) mbar_arrive_expect_tx(full, (uint32_t)__popc(live) * (uint32_t)(BR * 128));
            __syncwarp();
            if (id >= 0) tma_load_4d(dst0 + sl * kKVSlab + x * BR * 128, map, full, 64 * sl, key0 & (P - 1), g, id);
        };
        // (under the timeout test hook it issues nothing: the other warps' waits run out)
        for (int t = 0; t < n_tiles && !p.test_idle; ++t) {
            const int s = t % kKVStages;
            const uint32_t fph = (uint32_t)((t / kKVStages - 1) & 1);  // completion of tile t - kKVStages
            // K(t) once QK(t - stages) has read the buffer, V(t) once P V(t - stages) has
            if (t >= kKVStages && !wwait(bar(kBarKFree + s), fph)) break;
            issue_kv(t, false);
            if (t >= kKVStages && !wwait(bar(kBarVFree + s), fph)) break;
            issue_kv(t, true);
        }
    } else if (warp == kPTMmaWarp) {
        // ================= MMA warp: lane 0 issues every tcgen05.mma
        take_tmem();
        const uint32_t idesc_qk = umma_idesc_bf16(kQM, kBN, false, false);
        const uint32_t idesc_pv = umma_idesc_bf16(kQM, D, false, true);
        // S(t) = Q K(t)^T with Q (the A operand) in tensor memory
        auto issue_qk = [&](int t) {
            if (lane == 0) {
                const int b = t & 1, s = t % kKVStages;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const int sl = k >> 2, kk = k & 3;
                    const uint64_t bd = umma_desc_sw128(sK(s) + sl * kKVSlab + kk * 32, 16, 1024);
                    umma_ts(tmem + (b ? kColS1 : kColS0), tmem + kColQ + k * 8, bd, idesc_qk, k > 0 ? 1u : 0u);
                }
                umma_commit(bar(kBarS + b));
                umma_commit(bar(kBarKFree + s));
            }
            __syncwarp();
        };
        if (n_tiles > 0 && wwait(bar(kBarQ), 0) && wwait(bar(kBarKFull), 0)) issue_qk(0);
        // every lane tests, the warp acts on the answer all lanes agree on
        auto ready = [&](uint32_t bb, uint32_t phase) { return __all_sync(0xffffffffu, mbar_test_wait(bb, phase)); };
        // O += P(j) V(j)
        auto issue_pv = [&](int j) {
            const int b = j & 1, s = j % kKVStages;
            if (lane == 0) {
                tc_fence_after();
                const uint32_t sb = tmem + (b ? kColS1 : kColS0);
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk) {
                    const uint64_t bd = umma_desc_sw128(sV(s) + kk * 16 * 128, kKVSlab, 1024);
                    umma_ts(tmem + kColO, sb + kk * 8, bd, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
                    if (HILO) umma_ts(tmem + kColO, sb + 32 + kk * 8, bd, idesc_pv, 1u);
                }
                umma_commit(bar(kBarO + b));
                umma_commit(bar(kBarVFree + s));
            }
            __syncwarp();
        };
        for (int j = 0; j < n_tiles && !*abort_flag; ++j) {
            const int b = j & 1, s = j % kKVStages, j1 = j + 1;
            // Two independent groups: the next tile's scores QK(j+1) (its S
            // buffer held P(j-1), whose P V went out before, in order) and
            // P V(j) (P written, V landed and cleaned).  They touch different
            // S buffers, so whichever is ready goes out first.  The poll is
            // bounded like every wait; P V(j+1) and QK(j+2) come only after both.
            bool need_qk = j1 < n_tiles, need_pv = true;
            const uint64_t t_poll = global_ns();
            while (need_qk || need_pv) {
                bool moved = false;
                if (need_qk && ready(bar(kBarKFull + j1 % kKVStages), (uint32_t)((j1 / kKVStages) & 1))) {
                    issue_qk(j1);
                    need_qk = false;
                    moved = true;
                }
                if (need_pv && ready(bar(kBarPr + b), (uint32_t)((j >> 1) & 1)) &&
                    ready(bar(kBarVFull + s), (uint32_t)((j / kKVStages) & 1))) {
                    issue_pv(j);
                    need_pv = false;
                    moved = true;
                }
                if (!moved) {
                    const bool give_up = __any_sync(0xffffffffu, *abort_flag != 0 ||
                                                                   global_ns() - t_poll > lim);
                    if (give_up) {
                        *abort_flag = 1;
                        break;
                    }
                    __nanosleep(32);
                }
            }
        }
    } else {
        // ================= softmax warps: row qi of the tile, key columns 32h .. 32h + 31
        const int quad = warp & 3, h = warp >> 2;
        const int qi = quad * 32 + lane;
        const int row_i = row0 + qi / G;  // chunk-relative
        const bool valid_row = row_i < T;
        const int lim = valid_row ? min(key_hi_eff, causal0 + row_i) : key_hi_eff;
        // a tree node's path: bit a set for each node a on it (itself
        // included), walked up the parents in shared memory; a parent outside
        // [-1, node) makes the row bad.  Rows past the tree see everything.
        uint64_t anc = ~0ull;
        uint32_t path_bad = 0;
        if constexpr (TREE) {
            if (valid_row) {
                anc = 0;
                for (int a = row_i, steps = 0; a >= 0 && steps < kTreeMaxNodes; ++steps) {
                    anc |= 1ull << a;
                    const int pa = s_par[a];
                    if (pa < -1 || pa >= a) {
                        path_bad = 1;
                        break;
                    }
                    a = pa;
                }
            }
            if (__any_sync(0xffffffffu, path_bad != 0) && lane == 0) atomicOr(p.status, TF_DEV_BAD_SEG);
        }
        // key k is seen by this thread's row: the causal count, or a tree
        // node's window and path
        auto visible = [&](int k) -> bool {
            if constexpr (TREE)
                return k < key_hi_eff && (k < t_valid || ((anc >> (unsigned)(k - t_valid)) & 1ull) != 0);
            else
                return k < lim;
        };
        const float scale_log2 = p.scale_log2;
        float m_ref = -INFINITY, l_run = 0.f;
        uint32_t emax = 0, tail_bad = path_bad;
        const uint32_t pair_bar = 2 + quad;  // warps quad and quad + 4
        uint32_t lane_base = 0;

        // Q into tensor memory, the A operand of every QK: this thread's half
        // of its row straight from global memory (bf16 pairs are the operand's
        // 32-bit columns as they are); rows past the chunk are zero
        {
            constexpr int kWH = D / 4;  // 32-bit words a half row
            const uint4 *src = reinterpret_cast<const uint4 *>(
                p.q + ((int64_t)(q_row + (valid_row ? row_i : 0)) * p.hq + g * G + qi % G) * D + h * (D / 2));
            uint32_t w[kWH / 16][16];
#pragma unroll
            for (int v = 0; v < kWH / 4; ++v) {
                const uint4 x = valid_row ? __ldg(src + v) : make_uint4(0u, 0u, 0u, 0u);
                w[v >> 2][4 * (v & 3)] = x.x;
                w[v >> 2][4 * (v & 3) + 1] = x.y;
                w[v >> 2][4 * (v & 3) + 2] = x.z;
                w[v >> 2][4 * (v & 3) + 3] = x.w;
            }
            take_tmem();
            lane_base = tmem + ((uint32_t)(quad * 32) << 16);
#pragma unroll
            for (int c = 0; c < kWH / 16; ++c) tmem_st16(lane_base + kColQ + h * kWH + c * 16, w[c]);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kBarQ));
        }

        for (int j = 0; j < n_tiles; ++j) {
            const int b = j & 1, kt = key_lo + j * kBN;
            const uint32_t ph = (uint32_t)((j >> 1) & 1);
            const uint32_t colS = b ? kColS1 : kColS0;
            const int kh = kt + 32 * h;  // this half's first key
            pt_wait(bar(kBarS + b), ph, abort_flag, lim);
            tc_fence_after();
            float sv[32];
            {
                uint32_t r[32];
                tmem_ld32(lane_base + colS + 32 * h, r);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) sv[c] = __uint_as_float(r[c]);
            }
            // the half's largest score (four independent chains); nonfinite
            // visible scores: NaN and +inf reach the row sum (checked at the
            // end), -inf is caught by the min
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            if (kt + kBN > full_hi) {
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const bool vis = visible(kh + c);
                    emax = max(emax, vis ? exp_bits(sv[c]) : 0u);
                    sv[c] = vis ? sv[c] : -INFINITY;
                    m4[c & 3] = fmaxf(m4[c & 3], sv[c]);
                }
            } else {
                float n4[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    m4[c & 3] = fmaxf(m4[c & 3], sv[c]);
                    n4[c & 3] = fminf(n4[c & 3], sv[c]);
                }
                if (fminf(fminf(n4[0], n4[1]), fminf(n4[2], n4[3])) == -INFINITY) emax = 0x7f800000u;
            }
            const float mine = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            // the row's tile maximum: swap halves with the partner warp
            s_xmax[b][h][qi] = mine;
            named_bar_sync(pair_bar, 64);
            float mx = fmaxf(mine, s_xmax[b][h ^ 1][qi]);
            mx *= scale_log2;  // scale > 0: the max commutes with it
            // lazy rescale: the reference max moves only when it rises by 2^8;
            // both halves see the same maximum, so they move together
            float alpha = 1.f;
            if (mx > m_ref + 8.f || (m_ref == -INFINITY && mx != -INFINITY)) {
                alpha = (m_ref == -INFINITY) ? 0.f : ex2(m_ref - mx);
                m_ref = mx;
            }
            const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
            // the weights replace the scores in tensor memory (the partner has
            // loaded its half: it passed the pair barrier): keys 32h .. 32h + 31
            // as bf16 pairs in columns 16h .. 16h + 15, the low parts 32 further
            {
                uint32_t hi[16];
                float ls0 = 0.f, ls1 = 0.f;
                if constexpr (HILO) {
                    uint32_t lo[16];
#pragma unroll
                    for (int w = 0; w < 16; ++w) {
                        const float p0 = ex2(fmaf(sv[2 * w], scale_log2, -mu));
                        const float p1 = ex2(fmaf(sv[2 * w + 1], scale_log2, -mu));
                        ls0 += p0;
                        ls1 += p1;
                        hi[w] = pack_bf16x2(p0, p1);
                        lo[w] = pack_bf16x2(p0 - bf16_lo_to_f32(hi[w]), p1 - bf16_hi_to_f32(hi[w]));
                    }
                    tmem_st16(lane_base + colS + 32 + 16 * h, lo);
                } else {
#pragma unroll
                    for (int w = 0; w < 16; ++w) {
                        const float p0 = ex2(fmaf(sv[2 * w], scale_log2, -mu));
                        const float p1 = ex2(fmaf(sv[2 * w + 1], scale_log2, -mu));
                        ls0 += p0;
                        ls1 += p1;
                        hi[w] = pack_bf16x2(p0, p1);
                    }
                }
                l_run = l_run * alpha + (ls0 + ls1);
                tmem_st16(lane_base + colS + 16 * h, hi);
            }
            // O holds the tiles before this one: rescale it once P V(j-1) is
            // done; this half rescales O columns h * D/2 .. (h + 1) * D/2 - 1
            if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                pt_wait(bar(kBarO + ((j - 1) & 1)), (uint32_t)(((j - 1) >> 1) & 1), abort_flag, lim);
                tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < D / 64; ++c) {
                    uint32_t r[32];
                    const uint32_t col = kColO + h * (D / 2) + c * 32;
                    tmem_ld32(lane_base + col, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int w = 0; w < 32; ++w) r[w] = __float_as_uint(__uint_as_float(r[w]) * alpha);
                    tmem_st32(lane_base + col, r);
                }
            }
            tmem_wait_st();
            // V rows this tile must not feed into P V: past every row's keys ->
            // zero; seen by only some rows and nonfinite -> zero and flag
            if (kt + kBN > full_hi) {
                pt_wait(bar(kBarVFull + j % kKVStages), (uint32_t)((j / kKVStages) & 1), abort_flag, lim);
                named_bar_sync(1, kPTSoftmax);
                if (tid == 0) s_vbad[0] = s_vbad[1] = 0;
                named_bar_sync(1, kPTSoftmax);
                unsigned char *vb = sbase_ptr + C::kOffV + (j % kKVStages) * C::kKVBytes;
                for (int idx = tid; idx < kBN * C::kSlabs; idx += kPTSoftmax) {
                    const int r = idx % kBN, sl = idx / kBN;
                    uint4 *rowp = reinterpret_cast<uint4 *>(vb + sl * kKVSlab + r * 128);
                    const int key = kt + r;
                    if (key >= key_hi_eff) {
#pragma unroll
                        for (int k = 0; k < 8; ++k) rowp[k] = make_uint4(0, 0, 0, 0);
                    } else if (key >= full_hi) {
                        bool nf = false;
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const uint4 v = rowp[k];
                            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                nf |= ((w4[e] & 0x7f80u) == 0x7f80u) || ((w4[e] & 0x7f800000u) == 0x7f800000u);
                        }
                        if (nf) atomicOr(&s_vbad[r >> 5], 1u << (r & 31));
                    }
                }
                named_bar_sync(1, kPTSoftmax);
                const uint32_t vb0 = s_vbad[0], vb1 = s_vbad[1];
                if (vb0 | vb1) {
                    for (int idx = tid; idx < kBN * C::kSlabs; idx += kPTSoftmax) {
                        const int r = idx % kBN, sl = idx / kBN;
                        if ((((r < 32) ? vb0 : vb1) >> (r & 31)) & 1u) {
                            uint4 *rowp = reinterpret_cast<uint4 *>(vb + sl * kKVSlab + r * 128);
#pragma unroll
                            for (int k = 0; k < 8; ++k) rowp[k] = make_uint4(0, 0, 0, 0);
                        }
                    }
                    for (int r = 0; r < kBN; ++r)
                        if (((((r < 32) ? vb0 : vb1) >> (r & 31)) & 1u) && visible(kt + r)) tail_bad = 1;
                }
                fence_proxy_async_smem();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kBarPr + b));
        }

        // ---- epilogue: the halves' sums and findings meet, then each half
        // stores its D/2 columns of O (divided by the sum, or raw for a partial)
        if (n_tiles > 0) pt_wait(bar(kBarO + ((n_tiles - 1) & 1)), (uint32_t)(((n_tiles - 1) >> 1) & 1), abort_flag, lim);
        tc_fence_after();
        const bool aborted = *abort_flag != 0;
        s_xl[h][qi] = l_run;
        s_xbad[0][h][qi] = (emax == 0x7f800000u ? 1u : 0u) | tail_bad;
        named_bar_sync(pair_bar, 64);
        const float l_sum = s_xl[0][qi] + s_xl[1][qi];
        uint32_t bad = s_xbad[0][0][qi] | s_xbad[0][1][qi] | s_err | (aborted ? 1u : 0u);
        // a finished row always sees a key; a partial row may see none here
        if (!isfinite(l_sum) || (!PARTIAL && !(l_sum > 0.f))) bad = 1;
        const int64_t u = (int64_t)(q_row + row_i) * p.hq + g * G + (qi % G);
        const int64_t at = u * (PARTIAL ? p.n_splits_max : 1) + split;  // partial slot
        // O goes out through shared memory when the tile has many rows: each
        // thread stages its half row in the K/V buffers (free once the last
        // P V is done; rows padded by 16 bytes, so a warp's 16-byte stores hit
        // distinct banks) and sends it with one bulk copy, where direct stores
        // would have each warp instruction touch 32 rows.  A tile of few rows
        // (under 64 queries) stores directly: its fixed cost is lower.
        const int d0 = h * (D / 2);
        const bool out16 = !PARTIAL && p.out_bf16;
        const bool staged = rows_here * G >= 64;
        constexpr int kRowW = D + 4;  // 32-bit words a staged row (f32; a bf16 row uses half)
        const uint32_t row_w = out16 ? (uint32_t)(D / 2 + 4) : (uint32_t)kRowW;
        uint32_t *stage = reinterpret_cast<uint32_t *>(sbase_ptr + C::kOffK) + qi * row_w + (out16 ? d0 / 2 : d0);
        uint32_t *gout = PARTIAL ? reinterpret_cast<uint32_t *>(p.part_o + at * D + d0)
                                 : (out16 ? reinterpret_cast<uint32_t *>(reinterpret_cast<uint16_t *>(p.out) + u * D + d0)
                                          : reinterpret_cast<uint32_t *>(reinterpret_cast<float *>(p.out) + u * D + d0));
        const bool direct = !staged && valid_row && !aborted;
        uint32_t obad = 0;
#pragma unroll 1
        for (int cc = 0; cc < D / 64; ++cc) {
            uint32_t r[32];
            tmem_ld32(lane_base + kColO + d0 + cc * 32, r);
            tmem_wait_ld();
            float o[32];
#pragma unroll
            for (int w = 0; w < 32; ++w) {
                o[w] = PARTIAL ? __uint_as_float(r[w]) : __uint_as_float(r[w]) / l_sum;
                obad |= !isfinite(o[w]);
            }
            if (staged || direct) {
                uint32_t *dst = staged ? stage : gout;
                if (out16) {
                    uint4 *d4 = reinterpret_cast<uint4 *>(dst + cc * 16);
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        d4[w] = make_uint4(pack_bf16x2(o[8 * w], o[8 * w + 1]), pack_bf16x2(o[8 * w + 2], o[8 * w + 3]),
                                           pack_bf16x2(o[8 * w + 4], o[8 * w + 5]),
                                           pack_bf16x2(o[8 * w + 6], o[8 * w + 7]));
                } else {
                    float4 *d4 = reinterpret_cast<float4 *>(dst + cc * 32);
#pragma unroll
                    for (int w = 0; w < 8; ++w) d4[w] = make_float4(o[4 * w], o[4 * w + 1], o[4 * w + 2], o[4 * w + 3]);
                }
            }
        }
        // a nonfinite output in either half flags the whole row
        s_xbad[1][h][qi] = obad;
        named_bar_sync(pair_bar, 64);
        bad |= s_xbad[1][0][qi] | s_xbad[1][1][qi];
        // a flagged prompt row goes out as canonical NaN (partials keep o:
        // the flag marks them); a CTA that gave up writes it directly, since
        // copies may still be landing in its buffers
        if (!PARTIAL && bad && valid_row) {
            const uint32_t nanw = out16 ? 0x7fc07fc0u : 0x7fc00000u;
            uint32_t *dst = (staged && !aborted) ? stage : gout;
            const int words = out16 ? D / 4 : D / 2;
            for (int w = 0; w < words; w += 4)
                *reinterpret_cast<uint4 *>(dst + w) = make_uint4(nanw, nanw, nanw, nanw);
        }
        if (staged && valid_row && !aborted) {
            fence_proxy_async_smem();
            bulk_store(gout, smem_u32(stage), out16 ? (uint32_t)(D / 2) * 2u : (uint32_t)(D / 2) * 4u);
            bulk_commit();
            sent_row = true;
        }
        if (valid_row) {
            if (PARTIAL) {
                // natural-log reference max, sum, flag: the merge weighs partial
                // c by e^(m_c - M); a flagged partial flags the merged head
                if (h == 0) {
                    p.part_m[at] = (m_ref == -INFINITY) ? -INFINITY : m_ref * kLn2;
                    p.part_l[at] = l_sum;
                    p.part_flag[at] = (uint8_t)(bad ? 1 : 0);
                }
            } else {
                if (p.out_flags && h == 0) p.out_flags[u] = (uint8_t)(bad ? 1 : 0);
            }
        }
        // (a bulk copy is waited for at the very end, after the tensor
        // memory is released, so a CTA waiting for its SM starts sooner)
    }
    // everyone: report a timeout, give in-flight work a bounded chance to land,
    // release tensor memory
    __syncthreads();
    if (s_abort) {
        if (tid == 0) atomicOr(p.status, TF_DEV_TIMEOUT);
        if (tid == 0)
            for (int i = 0; i < kNumBars; ++i) {
                mbar_wait(bar(i), 0u, 20000000ull);
                mbar_wait(bar(i), 1u, 20000000ull);
            }
        __syncthreads();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
    // a thread that sent a staged row stays until the copy has read it from
    // shared memory; the grid's completion makes its writes visible
    if (sent_row) bulk_wait_read();
}

// ---------------------------------------------------------------------------
// host side: tensor maps and launch
// ---------------------------------------------------------------------------

bool prompt_tc_supported(int head_dim, int group, int page_size) {
    return (head_dim == 64 || head_dim == 128 || head_dim == 256) && group >= 1 && group <= 128 &&
           (128 % group) == 0 && page_size >= 8;
}

template <int D, bool PARTIAL>
static cudaError_t launch_tc_t(const PromptTcParams &p, const void *k, const void *v, int n_segs, cudaStream_t st) {
    CUtensorMap mk, mv;
    const int RT = kQM / p.group, P = 1 << p.log2_page, BR = P < kBN ? P : kBN;
    {
        const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)P, (cuuint64_t)p.hkv, (cuuint64_t)p.n_pages};
        const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)P * D * 2, (cuuint64_t)p.hkv * P * D * 2};
        const cuuint32_t box[4] = {64, (cuuint32_t)BR, 1, 1};
        if (!make_tensor_map_bf16(&mk, k, 4, dims, strides, box)) return cudaErrorInvalidValue;
        if (!make_tensor_map_bf16(&mv, v, 4, dims, strides, box)) return cudaErrorInvalidValue;
    }
    // partials are fp32: P goes in as bf16 hi + lo
    auto kern = PARTIAL ? prompt_tc_kernel<D, true, true>
                        : (p.out_bf16 ? prompt_tc_kernel<D, false, false> : prompt_tc_kernel<D, true, false>);
    using C = PTCfg<D, pt_paired<D, PARTIAL>()>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    if (pt_paired<D, PARTIAL>()) {  // all of the unified memory as shared memory, so two CTAs fit
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (e != cudaSuccess) return e;
    }
    const dim3 grid = PARTIAL ? dim3((unsigned)(p.n_qt * p.n_splits_max), (unsigned)p.hkv, (unsigned)n_segs)
                              : dim3((unsigned)((p.n_rows + RT - 1) / RT), (unsigned)p.hkv);
    PromptTcParams q = p;
    if (const uint64_t runout = test_wait_runout_ns()) {
        q.test_idle = 1;
        q.wait_ns = runout;
    }
    if (PARTIAL) {
        kern<<<grid, kPTThreads, C::kSmemBytes, st>>>(mk, mv, q);
        return cudaGetLastError();
    }
    // A prompt chunk may start while the call before it on the stream (this
    // library's previous chunk, or another of its attention calls) finishes:
    // it reads q, the pools and the page table, which none of them writes, so
    // the next chunk's tiles fill the SMs the previous chunk's last wave
    // leaves idle.
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kPTThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, mk, mv, q);
}

cudaError_t launch_prompt_tc(const PromptTcParams &p, int head_dim, const void *k, const void *v, cudaStream_t st) {
    switch (head_dim) {
        case 64: return launch_tc_t<64, false>(p, k, v, 1, st);
        case 128: return launch_tc_t<128, false>(p, k, v, 1, st);
        case 256: return launch_tc_t<256, false>(p, k, v, 1, st);
        default: return cudaErrorInvalidValue;
    }
}

bool partial_tc_supported(int head_dim, int group, int page_size, int split_keys) {
    return prompt_tc_supported(head_dim, group, page_size) && split_keys > 0 && split_keys % kBN == 0;
}

cudaError_t launch_partial_tc(const PromptTcParams &p, int head_dim, const void *k, const void *v, int n_segs,
                              cudaStream_t st) {
    if (n_segs == 0) return cudaSuccess;
    switch (head_dim) {
        case 64: return launch_tc_t<64, true>(p, k, v, n_segs, st);
        case 128: return launch_tc_t<128, true>(p, k, v, n_segs, st);
        case 256: return launch_tc_t<256, true>(p, k, v, n_segs, st);
        default: return cudaErrorInvalidValue;
    }
}

bool tree_tc_supported(int head_dim, int group) {
    return (head_dim == 64 || head_dim == 128 || head_dim == 256) && group >= 1 && group <= 128 &&
           (128 % group) == 0;
}

// Draft trees: the partial kernel with ring addressing (a 3-D tensor map over
// [slots][Hkv][D], boxes of 64 slots) and the ancestor mask on the nodes.
template <int D>
static cudaError_t launch_tree_t(const PromptTcParams &p, const void *k, const void *v, int n_segs,
                                 cudaStream_t st) {
    CUtensorMap mk, mv;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)p.hkv, (cuuint64_t)p.ring_slots_total};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)p.hkv * D * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)kBN};
    if (!make_tensor_map_bf16(&mk, k, 3, dims, strides, box)) return cudaErrorInvalidValue;
    if (!make_tensor_map_bf16(&mv, v, 3, dims, strides, box)) return cudaErrorInvalidValue;
    auto kern = prompt_tc_kernel<D, true, true, true>;
    using C = PTCfg<D, pt_paired<D, true>()>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    if (pt_paired<D, true>()) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (e != cudaSuccess) return e;
    }
    const dim3 grid((unsigned)(p.n_qt * p.n_splits_max), (unsigned)p.hkv, (unsigned)n_segs);
    PromptTcParams q = p;
    if (const uint64_t runout = test_wait_runout_ns()) {
        q.test_idle = 1;
        q.wait_ns = runout;
    }
    kern<<<grid, kPTThreads, C::kSmemBytes, st>>>(mk, mv, q);
    return cudaGetLastError();
}

cudaError_t launch_tree_tc(const PromptTcParams &p, int head_dim, const void *k, const void *v, int n_segs,
                           cudaStream_t st) {
    if (n_segs == 0) return cudaSuccess;
    switch (head_dim) {
        case 64: return launch_tree_t<64>(p, k, v, n_segs, st);
        case 128: return launch_tree_t<128>(p, k, v, n_segs, st);
        case 256: return launch_tree_t<256>(p, k, v, n_segs, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace tfp
