// attn_partial.cu - split-KV attention over many streams in one launch.
//
// One CTA is one work item: (stream or ring row s, kv-head g, key split c,
// query group qg).  It streams the split's keys and values through shared
// memory in tiles of 64 keys with a multi-stage cp.async pipeline, folds them
// into an online-softmax state on the tensor cores (bf16 m16n8k16, fp32
// accumulation) and writes one partial (m, l, o, flag) per (row, q-head), or,
// in direct mode, the normalised output.  The merge kernel at the end of this
// file folds partials.
//
// Sources (TensorFold pull requests, by title and section):
//  - #1503 "lfm2_moe CUDA: attention pages from the shared KV pool, and the
//    prompt cache", commit list: every stream's rows in one launch from a
//    segment table; paged split-KV chunk and merge bodies.
//  - #1653 "spark25 CUDA: the full layers' caches in pages of the core pool",
//    review thread and commit list: the per-chunk page lookup hoisted out of
//    the key loop, the next page's id loaded a tile early; a nonfinite head
//    kept off the merge's fast path.
//  - #1562 "Qwen3.6 MTP drafter on CUDA: draft a shared round's streams
//    together", PR body: each row over its own ring of slots, slots stepped
//    with a wrap rather than a 64-bit modulo, the next group in flight while
//    the current one folds.
//
// Design points specific to this implementation:
//  - Queries of one work item are the rows x q-heads of the stream that share
//    kv-head g, numbered qi = i * G + h_local; a CTA takes up to 64 of them
//    (four 16-row MMA tiles).  With fewer query tiles than warps, the warps
//    split each key tile instead and combine through shared memory.
//  - K/V tiles live in shared memory with 16-byte chunks XOR-swizzled by row,
//    so ldmatrix reads are free of bank conflicts.
//  - P is fed to the P.V product as bf16 hi + bf16 lo (two MMAs), which keeps
//    about 16 significant bits of each softmax weight; a single bf16 P would
//    leave a relative error near 1e-3 in the output.
//  - Nonfinite detection: the exponent bits of every visible score are
//    max-reduced (a nonfinite score has them all set); values are caught
//    through o going nonfinite, except for keys that only some rows of a
//    stream see, whose value rows are scanned and zeroed in shared memory so
//    rows that do not see them are not poisoned through a 0 * inf product.
#include <cstdint>
#include <cuda_runtime.h>

#include "tf_common.cuh"
#include "tf_internal.h"

namespace tfp {

constexpr int kThreads = 128;  // four warps
constexpr int kTK = 64;        // keys per tile
constexpr int kMaxQ = 64;      // queries per CTA
constexpr int kMaxPg = 9;      // page ids one tile can span (64 keys, pages >= 8, unaligned start)

template <int D>
struct Cfg {
    static constexpr int kRowBytes = D * 2;
    static constexpr int kCpr = D / 8;  // 16-byte chunks per row
    static constexpr int kTileBytes = kTK * kRowBytes;
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kStages = (D == 256) ? 3 : 4;
    static constexpr int kQBytes = kMaxQ * kRowBytes;
    static constexpr int kRowsPerPass = kThreads / kCpr;  // tile rows one pass of the CTA covers
    static constexpr int kPasses = kTK / kRowsPerPass;
    static constexpr int kPipeBytes = kStages * kStageBytes;
    // combine buffers (reuse the pipeline's space): o [4 warps][16][D] f32
    static constexpr int kCombBytes = 4 * 16 * D * 4;
    static constexpr int kQOffset = kPipeBytes > kCombBytes ? kPipeBytes : kCombBytes;
    static constexpr int kSmemBytes = kQOffset + kQBytes;
};

enum class Src { kPaged, kRing };

struct WorkState {
    int s, g, c, q0, nq;
    int q_row, n_rows, n_keys;  // stream
    int key_lo, key_hi, key_hi_eff;
    int n_tiles;
    // paged
    int pt_base, n_pg;
    // ring
    int64_t ring_base;
    int ring_size, ring_start;
};

// Output unit (row, q-head) of query qi of the item.
__device__ __forceinline__ int64_t unit_of(const AttnParams &p, const WorkState &w, int qi, Src src) {
    const int i = qi / p.group, hl = qi - (qi / p.group) * p.group;
    const int h = w.g * p.group + hl;
    if (src == Src::kRing) return (int64_t)w.s * p.hq + h;
    return (int64_t)(w.q_row + i) * p.hq + h;
}

template <int D, int KPW>
__device__ __forceinline__ void fold_tile(uint32_t sQ, uint32_t sK, uint32_t sV, int kbase, int jt, bool need_mask,
                                          int lim_lo, int lim_hi, float scale_log2, float (&o)[D / 8][4],
                                          float (&m)[2], float (&l)[2], uint32_t (&emax)[2], int lane) {
    constexpr int NT = KPW / 8;
    constexpr int RB = D * 2;
    float s[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;

    // S = Q K^T over the warp's KPW keys
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(sQ + swz(lane & 15, 2 * ks + (lane >> 4), RB), a0, a1, a2, a3);
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4(sK + swz(kbase + 16 * np + (lane & 7) + ((lane >> 4) << 3), 2 * ks + ((lane >> 3) & 1), RB), b0,
                    b1, b2, b3);
            mma_bf16(s[2 * np], a0, a1, a2, a3, b0, b1);
            mma_bf16(s[2 * np + 1], a0, a1, a2, a3, b2, b3);
        }
    }

    // scale into the log2 domain, mask, check
    const int t = lane & 3;
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float x = s[nt][e] * scale_log2;
            const int key = jt + kbase + 8 * nt + 2 * t + (e & 1);
            const bool vis = !need_mask || key < ((e < 2) ? lim_lo : lim_hi);
            const uint32_t eb = vis ? exp_bits(x) : 0u;
            if (e < 2)
                emax[0] = max(emax[0], eb);
            else
                emax[1] = max(emax[1], eb);
            x = vis ? x : -INFINITY;
            s[nt][e] = x;
            if (e < 2)
                mx0 = fmaxf(mx0, x);
            else
                mx1 = fmaxf(mx1, x);
        }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m[0], mx0), mn1 = fmaxf(m[1], mx1);
    const float mu0 = (mn0 == -INFINITY) ? 0.f : mn0, mu1 = (mn1 == -INFINITY) ? 0.f : mn1;
    const float al0 = ex2(m[0] - mu0), al1 = ex2(m[1] - mu1);
    m[0] = mn0;
    m[1] = mn1;
    float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        s[nt][0] = ex2(s[nt][0] - mu0);
        s[nt][1] = ex2(s[nt][1] - mu0);
        s[nt][2] = ex2(s[nt][2] - mu1);
        s[nt][3] = ex2(s[nt][3] - mu1);
        ls0 += s[nt][0] + s[nt][1];
        ls1 += s[nt][2] + s[nt][3];
    }
    l[0] = l[0] * al0 + ls0;
    l[1] = l[1] * al1 + ls1;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
        o[nt][0] *= al0;
        o[nt][1] *= al0;
        o[nt][2] *= al1;
        o[nt][3] *= al1;
    }

    // O += P V with P = hi + lo (both bf16)
#pragma unroll
    for (int kk = 0; kk < KPW / 16; ++kk) {
        const uint32_t h0 = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
        const uint32_t h1 = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
        const uint32_t h2 = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        const uint32_t h3 = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
        const uint32_t r0 = pack_bf16x2(s[2 * kk][0] - bf16_lo_to_f32(h0), s[2 * kk][1] - bf16_hi_to_f32(h0));
        const uint32_t r1 = pack_bf16x2(s[2 * kk][2] - bf16_lo_to_f32(h1), s[2 * kk][3] - bf16_hi_to_f32(h1));
        const uint32_t r2 =
            pack_bf16x2(s[2 * kk + 1][0] - bf16_lo_to_f32(h2), s[2 * kk + 1][1] - bf16_hi_to_f32(h2));
        const uint32_t r3 =
            pack_bf16x2(s[2 * kk + 1][2] - bf16_lo_to_f32(h3), s[2 * kk + 1][3] - bf16_hi_to_f32(h3));
#pragma unroll
        for (int dp = 0; dp < D / 16; ++dp) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(sV + swz(kbase + 16 * kk + (lane & 7) + (((lane >> 3) & 1) << 3), 2 * dp + (lane >> 4), RB),
                      b0, b1, b2, b3);
            mma_bf16(o[2 * dp], h0, h1, h2, h3, b0, b1);
            mma_bf16(o[2 * dp], r0, r1, r2, r3, b0, b1);
            mma_bf16(o[2 * dp + 1], h0, h1, h2, h3, b2, b3);
            mma_bf16(o[2 * dp + 1], r0, r1, r2, r3, b2, b3);
        }
    }
}

template <int D, Src SRC, bool DIRECT>
__global__ void __launch_bounds__(kThreads, (D == 256) ? 1 : 2) attn_partial_kernel(const AttnParams p) {
    using C = Cfg<D>;
    extern __shared__ __align__(1024) unsigned char smem[];
    __shared__ int s_pid[C::kStages + 1][kMaxPg];
    __shared__ uint32_t s_vbad[2];
    __shared__ int s_flag;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    WorkState w;
    w.s = blockIdx.z;
    w.c = blockIdx.x;
    w.g = blockIdx.y / p.n_qgroups;
    // the last query group (the most keys under a causal mask) is scheduled first
    const int qg = p.n_qgroups - 1 - (int)(blockIdx.y - w.g * p.n_qgroups);

    // ---- resolve the work item from the table --------------------------------
    int per;
    if constexpr (SRC == Src::kPaged) {
        const tf_seg sg = p.seg_inline ? p.seg0 : p.segs[w.s];
        w.q_row = sg.q_row;
        w.n_rows = sg.n_rows;
        w.n_keys = sg.n_keys;
        w.pt_base = sg.pt_base;
        w.n_pg = sg.n_pages;
        const bool bad = w.q_row < 0 || w.n_rows < 0 || (int64_t)w.q_row + w.n_rows > p.n_rows_total ||
                         w.n_keys < (p.full ? (w.n_rows > 0 ? 1 : 0) : w.n_rows) || w.pt_base < 0 || w.n_pg < 0 ||
                         (int64_t)w.pt_base + w.n_pg > p.pt_len;
        if (bad) {
            if (tid == 0) atomicOr(p.status, TF_DEV_BAD_SEG);
            return;
        }
        if ((int64_t)w.n_keys > ((int64_t)w.n_pg << p.log2_page)) {
            if (tid == 0) atomicOr(p.status, TF_DEV_PAST_PAGES);
            return;
        }
        if (p.split_keys > 0) {
            per = p.split_keys;
        } else {
            per = (w.n_keys + p.n_splits_max - 1) / p.n_splits_max;
            per = ((per + (1 << p.log2_page) - 1) >> p.log2_page) << p.log2_page;
        }
    } else {
        const tf_ring_seg rs = p.rsegs[w.s];
        w.q_row = rs.q_row;
        w.n_rows = 1;
        w.n_keys = rs.n_valid;
        w.ring_base = rs.base;
        w.ring_size = rs.size;
        const bool bad = rs.q_row < 0 || rs.q_row >= p.n_rows_total || rs.size <= 0 || rs.n_valid < 1 ||
                         rs.n_valid > rs.size || rs.head < 0 || rs.head >= rs.size || rs.base < 0 ||
                         rs.base + rs.size > p.ring_slots_total;
        if (bad) {
            if (tid == 0) atomicOr(p.status, TF_DEV_BAD_SEG);
            return;
        }
        w.ring_start = rs.head - rs.n_valid;
        if (w.ring_start < 0) w.ring_start += rs.size;
        per = p.split_keys;
    }
    if (w.n_rows == 0) return;
    const int n_sp = (w.n_keys + per - 1) / per;
    if (n_sp > p.n_splits_max) {
        if (tid == 0) atomicOr(p.status, TF_DEV_SPLITS);
        return;
    }
    const int q_item = w.n_rows * p.group;
    w.q0 = qg * kMaxQ;
    if (w.q0 >= q_item) return;
    w.nq = min(kMaxQ, q_item - w.q0);

    if (w.c >= n_sp) {
        // a partial slot past the stream's count: an empty partial, o untouched
        if constexpr (!DIRECT) {
            for (int r = tid; r < w.nq; r += kThreads) {
                const int64_t at = unit_of(p, w, w.q0 + r, SRC) * p.n_splits_max + w.c;
                p.part_m[at] = -INFINITY;
                p.part_l[at] = 0.f;
                p.part_flag[at] = 0;
            }
        }
        return;
    }
    w.key_lo = w.c * per;
    w.key_hi = min(w.n_keys, w.key_lo + per);
    const int i_min = w.q0 / p.group, i_max = (w.q0 + w.nq - 1) / p.group;
    // keys every row sees: [0, causal0) (with the full flag: all of them)
    const int causal0 = p.full ? w.n_keys : w.n_keys - w.n_rows + 1;
    w.key_hi_eff = min(w.key_hi, causal0 + i_max);
    w.n_tiles = w.key_hi_eff > w.key_lo ? (w.key_hi_eff - w.key_lo + kTK - 1) / kTK : 0;
    const int full_hi = min(w.key_hi, causal0 + i_min);  // below this key no masking is needed

    const int nqt = (w.nq + 15) >> 4;
    const int kw_ways = nqt == 1 ? 4 : (nqt == 2 ? 2 : 1);
    const int my_qt = warp % (4 / kw_ways) < nqt ? warp % (4 / kw_ways) : -1;  // -1: idle warp (nqt == 3)
    const int my_kw = warp / (4 / kw_ways);

    const uint32_t sbase = smem_u32(smem);
    const uint32_t sQ = sbase + C::kQOffset;
    const uint16_t *__restrict__ kg = p.k;
    const uint16_t *__restrict__ vg = p.v;
    const int log2p = p.log2_page;
    const int pmask = (1 << log2p) - 1;

    // page ids of tile t into s_pid[slot] (paged source only)
    auto load_ids = [&](int t) {
        if constexpr (SRC == Src::kPaged) {
            if (tid < kMaxPg) {
                const int kt = w.key_lo + t * kTK;
                const int idx = (kt >> log2p) + tid;
                int pid = -2;
                if (idx < w.n_pg && ((int64_t)idx << log2p) < w.key_hi_eff) {
                    pid = p.page_table[w.pt_base + idx];
                    if (pid < 0 || pid >= p.n_pages) pid = -1;
                }
                s_pid[t % (C::kStages + 1)][tid] = pid;
            }
        }
    };
    // cp.async the K and V rows of tile t into pipeline stage t % stages
    bool bad_page = false;
    auto issue_tile = [&](int t) {
        const int kt = w.key_lo + t * kTK;
        const uint32_t stK = sbase + (t % C::kStages) * C::kStageBytes;
        const uint32_t stV = stK + C::kTileBytes;
        const int col = tid % C::kCpr;
        int slot0 = 0;
        if constexpr (SRC == Src::kRing) {
            slot0 = w.ring_start + kt;
            while (slot0 >= w.ring_size) slot0 -= w.ring_size;  // at most twice: start < size, kt < size
        }
#pragma unroll
        for (int ps = 0; ps < C::kPasses; ++ps) {
            const int row = tid / C::kCpr + ps * C::kRowsPerPass;
            const int j = kt + row;
            bool ok = j < w.key_hi_eff;
            int64_t off = 0;
            if constexpr (SRC == Src::kPaged) {
                const int pid = s_pid[t % (C::kStages + 1)][(j >> log2p) - (kt >> log2p)];
                if (ok && pid < 0) {
                    bad_page = true;
                    ok = false;
                }
                off = ((((int64_t)(ok ? pid : 0) * p.hkv + w.g) << log2p) + (j & pmask)) * D + col * 8;
            } else {
                int sl = slot0 + row;
                if (sl >= w.ring_size) sl -= w.ring_size;
                off = ((w.ring_base + sl) * p.hkv + w.g) * D + col * 8;
            }
            const uint32_t so = swz(row, col, C::kRowBytes);
            cp_async_16(stK + so, ok ? (const void *)(kg + off) : (const void *)kg, ok ? 16u : 0u);
            cp_async_16(stV + so, ok ? (const void *)(vg + off) : (const void *)vg, ok ? 16u : 0u);
        }
    };

    // ---- prologue: page ids, Q, first stages --------------------------------
    for (int t = 0; t < C::kStages && t < w.n_tiles; ++t) load_ids(t);
    if (tid == 0) {
        s_flag = 0;
        s_vbad[0] = s_vbad[1] = 0;
    }
    __syncthreads();
    {
        const int col = tid % C::kCpr;
        for (int r = tid / C::kCpr; r < kMaxQ; r += C::kRowsPerPass) {
            const int qi = w.q0 + r;
            const bool ok = r < w.nq;
            int64_t off = 0;
            if (ok) {
                const int i = qi / p.group, hl = qi - i * p.group;
                off = ((int64_t)(w.q_row + i) * p.hq + w.g * p.group + hl) * D + col * 8;
            }
            cp_async_16(sQ + swz(r, col, C::kRowBytes), ok ? (const void *)(p.q + off) : (const void *)p.q,
                        ok ? 16u : 0u);
        }
    }
#pragma unroll
    for (int t = 0; t < C::kStages - 1; ++t) {
        if (t < w.n_tiles) issue_tile(t);
        cp_async_commit();
    }

    // ---- per-thread softmax state --------------------------------------------
    float o[D / 8][4];
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    uint32_t emax[2] = {0u, 0u};
    bool tail_bad[2] = {false, false};
    const int gq = lane >> 2;
    int lim_lo = w.key_hi, lim_hi = w.key_hi;
    if (my_qt >= 0) {
        const int qa = w.q0 + my_qt * 16 + gq, qb = qa + 8;
        if (qa < q_item) lim_lo = min(w.key_hi, causal0 + qa / p.group);
        if (qb < q_item) lim_hi = min(w.key_hi, causal0 + qb / p.group);
    }
    const float scale_log2 = p.scale_log2;

    // ---- main loop ------------------------------------------------------------
    for (int t = 0; t < w.n_tiles; ++t) {
        cp_async_wait<C::kStages - 2>();
        __syncthreads();
        if (t + C::kStages < w.n_tiles) load_ids(t + C::kStages);
        if (t + C::kStages - 1 < w.n_tiles) issue_tile(t + C::kStages - 1);
        cp_async_commit();

        const int kt = w.key_lo + t * kTK;
        const uint32_t stK = sbase + (t % C::kStages) * C::kStageBytes;
        const uint32_t stV = stK + C::kTileBytes;
        const bool need_mask = kt + kTK > full_hi;

        // value rows that only some rows see: scan, zero the nonfinite ones
        if (w.n_rows > 1 && kt + kTK > causal0) {
            const int r_lo = max(0, causal0 - kt), r_hi = min(kTK, w.key_hi_eff - kt);
            unsigned char *vt = smem + (t % C::kStages) * C::kStageBytes + C::kTileBytes;
            for (int idx = tid; idx < (r_hi - r_lo) * C::kCpr; idx += kThreads) {
                const int r = r_lo + idx / C::kCpr, cc = idx % C::kCpr;
                const uint4 v4 = *reinterpret_cast<const uint4 *>(vt + swz(r, cc, C::kRowBytes));
                const uint32_t wds[4] = {v4.x, v4.y, v4.z, v4.w};
                bool nf = false;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    nf |= ((wds[k] & 0x7f80u) == 0x7f80u) || ((wds[k] & 0x7f800000u) == 0x7f800000u);
                if (nf) atomicOr(&s_vbad[r >> 5], 1u << (r & 31));
            }
            __syncthreads();
            const uint32_t vb0 = s_vbad[0], vb1 = s_vbad[1];
            if (vb0 | vb1) {
                for (int idx = tid; idx < kTK * C::kCpr; idx += kThreads) {
                    const int r = idx / C::kCpr, cc = idx % C::kCpr;
                    if (((r < 32 ? vb0 : vb1) >> (r & 31)) & 1u)
                        *reinterpret_cast<uint4 *>(vt + swz(r, cc, C::kRowBytes)) = make_uint4(0, 0, 0, 0);
                }
                // a row that sees a zeroed key is flagged
#pragma unroll
                for (int r = 0; r < kTK; ++r) {
                    if (((r < 32 ? vb0 : vb1) >> (r & 31)) & 1u) {
                        if (kt + r < lim_lo) tail_bad[0] = true;
                        if (kt + r < lim_hi) tail_bad[1] = true;
                    }
                }
                __syncthreads();
                if (tid == 0) s_vbad[0] = s_vbad[1] = 0;
            }
        }

        if (my_qt >= 0) {
            const uint32_t sQw = sQ + my_qt * 16 * C::kRowBytes;
            if (kw_ways == 4)
                fold_tile<D, 16>(sQw, stK, stV, my_kw * 16, kt, need_mask, lim_lo, lim_hi, scale_log2, o, m, l, emax,
                                 lane);
            else if (kw_ways == 2)
                fold_tile<D, 32>(sQw, stK, stV, my_kw * 32, kt, need_mask, lim_lo, lim_hi, scale_log2, o, m, l, emax,
                                 lane);
            else
                fold_tile<D, 64>(sQw, stK, stV, 0, kt, need_mask, lim_lo, lim_hi, scale_log2, o, m, l, emax, lane);
        }
    }
    cp_async_wait<0>();
    if (bad_page) s_flag = 1;
    __syncthreads();
    if (s_flag && tid == 0) atomicOr(p.status, TF_DEV_BAD_PAGE);

    // ---- combine the warps' states through shared memory ----------------------
    // o of warp (qt, kw) for row r of its tile sits at comb row kw * nqt * 16 + qt * 16 + r
    float *comb_o = reinterpret_cast<float *>(smem);
    __shared__ float comb_m[4][kMaxQ], comb_l[4][kMaxQ];
    __shared__ uint8_t comb_f[4][kMaxQ];
    if (my_qt >= 0) {
        l[0] += __shfl_xor_sync(0xffffffffu, l[0], 1);
        l[0] += __shfl_xor_sync(0xffffffffu, l[0], 2);
        l[1] += __shfl_xor_sync(0xffffffffu, l[1], 1);
        l[1] += __shfl_xor_sync(0xffffffffu, l[1], 2);
        uint32_t f0 = (emax[0] == 0x7f800000u) | tail_bad[0], f1 = (emax[1] == 0x7f800000u) | tail_bad[1];
        f0 |= __shfl_xor_sync(0xffffffffu, f0, 1);
        f0 |= __shfl_xor_sync(0xffffffffu, f0, 2);
        f1 |= __shfl_xor_sync(0xffffffffu, f1, 1);
        f1 |= __shfl_xor_sync(0xffffffffu, f1, 2);
        const int ra = my_qt * 16 + gq, rb = ra + 8;
        if ((lane & 3) == 0) {
            comb_m[my_kw][ra] = m[0];
            comb_m[my_kw][rb] = m[1];
            comb_l[my_kw][ra] = l[0];
            comb_l[my_kw][rb] = l[1];
            comb_f[my_kw][ra] = (uint8_t)f0;
            comb_f[my_kw][rb] = (uint8_t)f1;
        }
        float *oa = comb_o + ((size_t)my_kw * nqt * 16 + ra) * D;
        float *ob = comb_o + ((size_t)my_kw * nqt * 16 + rb) * D;
        const int t2 = 2 * (lane & 3);
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt) {
            *reinterpret_cast<float2 *>(oa + nt * 8 + t2) = make_float2(o[nt][0], o[nt][1]);
            *reinterpret_cast<float2 *>(ob + nt * 8 + t2) = make_float2(o[nt][2], o[nt][3]);
        }
    }
    __syncthreads();

    // ---- epilogue: one warp per query row -------------------------------------
    for (int r = warp; r < w.nq; r += 4) {
        float mk[4], lk[4];
        float M = -INFINITY;
        uint32_t f = s_flag;
        for (int k = 0; k < kw_ways; ++k) {
            mk[k] = comb_m[k][r];
            lk[k] = comb_l[k][r];
            f |= comb_f[k][r];
            M = fmaxf(M, mk[k]);
        }
        const float Mu = (M == -INFINITY) ? 0.f : M;
        float wk[4], L = 0.f;
        for (int k = 0; k < kw_ways; ++k) {
            wk[k] = ex2(mk[k] - Mu);
            L += wk[k] * lk[k];
        }
        const int64_t u = unit_of(p, w, w.q0 + r, SRC);
        bool nf = !isfinite(L);
        for (int d0 = lane * 4; d0 < D; d0 += 128) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int k = 0; k < kw_ways; ++k) {
                const float4 v = *reinterpret_cast<const float4 *>(comb_o + ((size_t)k * nqt * 16 + r) * D + d0);
                acc.x += wk[k] * v.x;
                acc.y += wk[k] * v.y;
                acc.z += wk[k] * v.z;
                acc.w += wk[k] * v.w;
            }
            nf |= !isfinite(acc.x) || !isfinite(acc.y) || !isfinite(acc.z) || !isfinite(acc.w);
            if constexpr (!DIRECT) {
                const int64_t at = u * p.n_splits_max + w.c;
                *reinterpret_cast<float4 *>(p.part_o + at * D + d0) = acc;
            } else {
                // stash the unnormalised sum back for the second pass below
                *reinterpret_cast<float4 *>(comb_o + (size_t)r * D + d0) = acc;
            }
        }
        f |= __any_sync(0xffffffffu, nf) ? 1u : 0u;
        if constexpr (!DIRECT) {
            if (lane == 0) {
                const int64_t at = u * p.n_splits_max + w.c;
                p.part_m[at] = (M == -INFINITY) ? -INFINITY : M * kLn2;
                p.part_l[at] = L;
                p.part_flag[at] = (uint8_t)(f ? 1 : 0);
            }
        } else {
            if (!(L > 0.f)) f = 1;
            __syncwarp();
            for (int d0 = lane * 4; d0 < D; d0 += 128) {
                float4 acc = *reinterpret_cast<const float4 *>(comb_o + (size_t)r * D + d0);
                if (f) {
                    acc = make_float4(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000),
                                      __int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
                } else {
                    acc.x /= L;
                    acc.y /= L;
                    acc.z /= L;
                    acc.w /= L;
                }
                if (p.out_bf16) {
                    uint2 pk;
                    pk.x = pack_bf16x2(acc.x, acc.y);
                    pk.y = pack_bf16x2(acc.z, acc.w);
                    *reinterpret_cast<uint2 *>(reinterpret_cast<uint16_t *>(p.out) + u * D + d0) = pk;
                } else {
                    *reinterpret_cast<float4 *>(reinterpret_cast<float *>(p.out) + u * D + d0) = acc;
                }
            }
            if (lane == 0 && p.out_flags) p.out_flags[u] = (uint8_t)(f ? 1 : 0);
        }
    }
}

// ---------------------------------------------------------------------------
// merge: one warp per (row, q-head) unit
// ---------------------------------------------------------------------------
// Lane c holds partial c's weight e^(m_c - M) (0 for an empty partial); the o
// rows are then read with independent, predicated loads four partials at a
// time.  The kernel may be launched as a programmatic dependent of the
// partial kernel: it waits for that grid before it reads a partial or writes
// anything.  A ring or tree merge reads its table entry before that wait:
// the partial kernel before it never writes the table, and that kernel
// started only after all earlier work on the stream had finished.
template <int D, int MODE>
__global__ void __launch_bounds__(128) merge_kernel(const MergeParams p) {
    // a dependent launch (a verify round's argmax) may start; it waits for
    // this grid's completion before it reads anything
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // A (row, head) takes SL adjacent warps of the block, each a 128-column
    // slice of o (two at D 256, so a warp holds one round of 16 partials in
    // registers; one below).  Every output element sees the same arithmetic
    // in the same order whichever warp holds it.
    constexpr int SL = D > 128 ? D / 128 : 1;
    constexpr int DW = D / SL;  // columns a warp
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sl = warp % SL, dbase = sl * DW;
    const int64_t u = (int64_t)blockIdx.x * (4 / SL) + warp / SL;
    if (u >= p.n_units) return;  // all warps of a unit leave together
    int64_t out_u = u, pu = u;  // the output row's unit, the partials' unit
    int C = p.n_parts;
    const float qnan = __int_as_float(0x7fc00000);
    if constexpr (MODE == kMergeRows) asm volatile("griddepcontrol.wait;" ::: "memory");
    if constexpr (MODE == kMergeRing) {
        // only rows the table names are written; a bad entry (the partial
        // kernel skipped it) gives a flagged NaN row
        const int64_t s = u / p.hq, h = u - s * p.hq;
        const tf_ring_seg e = p.rsegs[s];
        if (e.q_row < 0 || e.q_row >= p.n_rows_total) return;
        out_u = (int64_t)e.q_row * p.hq + h;
        const bool bad = e.size <= 0 || e.n_valid < 1 || e.n_valid > e.size || e.head < 0 || e.head >= e.size ||
                         e.base < 0 || e.base + e.size > p.ring_slots_total ||
                         (e.n_valid + p.split_slots - 1) / p.split_slots > p.n_parts;
        asm volatile("griddepcontrol.wait;" ::: "memory");
        if (bad) {
            for (int d0 = dbase + lane * 4; d0 < dbase + DW; d0 += 128)
                *reinterpret_cast<float4 *>(p.out + out_u * D + d0) = make_float4(qnan, qnan, qnan, qnan);
            if (lane == 0 && sl == 0) p.flags[out_u] = 1;
            return;
        }
        C = (e.n_valid + p.split_slots - 1) / p.split_slots;
    } else if constexpr (MODE == kMergeTree) {
        // unit (s * tree_nodes + i) * Hq + h: node i of tree s; its partials
        // sit at its query row.  Only the trees' rows are written; an entry
        // the partial kernel skipped gives flagged NaN rows.
        const int64_t per = (int64_t)p.tree_nodes * p.hq;
        const int64_t s = u / per, rem = u - s * per;
        const int i = (int)(rem / p.hq), h = (int)(rem - (int64_t)i * p.hq);
        const tf_tree_seg e = p.tsegs[s];
        if (i >= e.n_nodes || e.q_row < 0 || (int64_t)e.q_row + i >= p.n_rows_total) return;
        out_u = pu = (int64_t)(e.q_row + i) * p.hq + h;
        const bool ok = tree_seg_ok(e, p.n_rows_total, p.n_parents, p.ring_slots_total) &&
                        tree_splits(e, p.split_slots).n_sp <= p.n_parts;
        asm volatile("griddepcontrol.wait;" ::: "memory");
        if (!ok) {
            for (int d0 = dbase + lane * 4; d0 < dbase + DW; d0 += 128)
                *reinterpret_cast<float4 *>(p.out + out_u * D + d0) = make_float4(qnan, qnan, qnan, qnan);
            if (lane == 0 && sl == 0) p.flags[out_u] = 1;
            return;
        }
        C = tree_splits(e, p.split_slots).n_sp;
    }
    const float *pm = p.part_m + pu * p.n_parts;
    const float *pl = p.part_l + pu * p.n_parts;
    const uint8_t *pf = p.part_flag + pu * p.n_parts;
    const float *po = p.part_o + pu * p.n_parts * D;

    // Everything a chunk of up to 16 partials needs is loaded in one round:
    // lane c's (m, l, flag) and every lane's slice of each o row.  An empty
    // partial's o is never multiplied in (its weight selects 0), so its
    // unwritten contents cannot leak into the sum.
    constexpr int NV = (DW + 127) / 128;
    constexpr int CH = 16;
    float4 acc[NV];
#pragma unroll
    for (int k = 0; k < NV; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    float M = -INFINITY, L = 0.f;
    uint32_t f = 0, any = 0;
    for (int c0 = 0; c0 < C; c0 += CH) {
        const int n = min(CH, C - c0);
        float4 v[CH][NV];
#pragma unroll
        for (int j = 0; j < CH; ++j)
#pragma unroll
            for (int k = 0; k < NV; ++k) {
                const int d0 = dbase + k * 128 + lane * 4;
                v[j][k] = (j < n && d0 < dbase + DW)
                              ? *reinterpret_cast<const float4 *>(po + (int64_t)(c0 + j) * D + d0)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        float mc = -INFINITY, lc = 0.f;
        if (lane < n) {
            mc = pm[c0 + lane];
            lc = pl[c0 + lane];
            f |= pf[c0 + lane];
        }
        const bool live = lc > 0.f;
        if (live) any = 1;
        // chunk max, merged into the running max (rescaling what came before)
        float mx = live ? mc : -INFINITY;
#pragma unroll
        for (int x = 16; x; x >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, x));
        const float Mn = fmaxf(M, mx);
        if (Mn != -INFINITY) {
            const float r = (M == -INFINITY) ? 0.f : ex2((M - Mn) * kLog2e);
            L *= r;
#pragma unroll
            for (int k = 0; k < NV; ++k) {
                acc[k].x *= r;
                acc[k].y *= r;
                acc[k].z *= r;
                acc[k].w *= r;
            }
            M = Mn;
        }
        const float w = live ? ex2((mc - M) * kLog2e) : 0.f;
        L += w * lc;  // lane-partial, reduced below
#pragma unroll
        for (int j = 0; j < CH; ++j) {
            const float wj = __shfl_sync(0xffffffffu, w, j);
            if (j < n && wj != 0.f) {
#pragma unroll
                for (int k = 0; k < NV; ++k) {
                    acc[k].x += wj * v[j][k].x;
                    acc[k].y += wj * v[j][k].y;
                    acc[k].z += wj * v[j][k].z;
                    acc[k].w += wj * v[j][k].w;
                }
            }
        }
    }
#pragma unroll
    for (int x = 16; x; x >>= 1) {
        f |= __shfl_xor_sync(0xffffffffu, f, x);
        any |= __shfl_xor_sync(0xffffffffu, any, x);
    }
#pragma unroll
    for (int x = 16; x; x >>= 1) L += __shfl_xor_sync(0xffffffffu, L, x);
    bool nf = !isfinite(L) || !any;
#pragma unroll
    for (int k = 0; k < NV; ++k) {
        const int d0 = dbase + k * 128 + lane * 4;
        if (d0 < dbase + DW) {
            acc[k].x /= L;
            acc[k].y /= L;
            acc[k].z /= L;
            acc[k].w /= L;
            nf |= !isfinite(acc[k].x) || !isfinite(acc[k].y) || !isfinite(acc[k].z) || !isfinite(acc[k].w);
        }
    }
    uint32_t nfw = __any_sync(0xffffffffu, nf) ? 1u : 0u;
    if constexpr (SL > 1) {
        // a nonfinite output in any slice flags the whole head: the unit's
        // warps swap their findings (a barrier of just those warps)
        __shared__ uint32_t s_nf[4];
        if (lane == 0) s_nf[warp] = nfw;
        asm volatile("bar.sync %0, %1;" ::"r"(1 + warp / SL), "r"(32 * SL) : "memory");
#pragma unroll
        for (int i = 0; i < SL; ++i) nfw |= s_nf[(warp / SL) * SL + i];
    }
    f |= nfw;
#pragma unroll
    for (int k = 0; k < NV; ++k) {
        const int d0 = dbase + k * 128 + lane * 4;
        if (d0 < dbase + DW) {
            const float4 v = f ? make_float4(qnan, qnan, qnan, qnan) : acc[k];
            *reinterpret_cast<float4 *>(p.out + out_u * D + d0) = v;
        }
    }
    if (lane == 0 && sl == 0) p.flags[out_u] = (uint8_t)(f ? 1 : 0);
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
template <int D, Src SRC, bool DIRECT>
static cudaError_t launch_partial_t(const AttnParams &p, dim3 grid, cudaStream_t st) {
    using C = Cfg<D>;
    auto kern = attn_partial_kernel<D, SRC, DIRECT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, C::kSmemBytes, st>>>(p);
    return cudaGetLastError();
}

template <Src SRC, bool DIRECT>
static cudaError_t launch_partial_d(const AttnParams &p, int head_dim, dim3 grid, cudaStream_t st) {
    switch (head_dim) {
        case 64: return launch_partial_t<64, SRC, DIRECT>(p, grid, st);
        case 128: return launch_partial_t<128, SRC, DIRECT>(p, grid, st);
        case 256: return launch_partial_t<256, SRC, DIRECT>(p, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_attn_partial(const AttnParams &p, int head_dim, bool ring, bool direct, dim3 grid,
                                cudaStream_t st) {
    if (ring) return launch_partial_d<Src::kRing, false>(p, head_dim, grid, st);
    if (direct) return launch_partial_d<Src::kPaged, true>(p, head_dim, grid, st);
    return launch_partial_d<Src::kPaged, false>(p, head_dim, grid, st);
}

template <int D, int MODE>
static cudaError_t launch_merge_t(const MergeParams &p, cudaStream_t st) {
    cudaLaunchConfig_t cfg{};
    constexpr int units = D > 128 ? 4 / (D / 128) : 4;  // (row, head) units a 128-thread block
    cfg.gridDim = dim3((unsigned)((p.n_units + units - 1) / units));
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, merge_kernel<D, MODE>, p);
}

template <int D>
static cudaError_t launch_merge_m(const MergeParams &p, int mode, cudaStream_t st) {
    switch (mode) {
        case kMergeRows: return launch_merge_t<D, kMergeRows>(p, st);
        case kMergeRing: return launch_merge_t<D, kMergeRing>(p, st);
        case kMergeTree: return launch_merge_t<D, kMergeTree>(p, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_merge(const MergeParams &p, int head_dim, int mode, cudaStream_t st) {
    if (p.n_units == 0) return cudaSuccess;
    cudaError_t e;
    switch (head_dim) {
        case 64: e = launch_merge_m<64>(p, mode, st); break;
        case 128: e = launch_merge_m<128>(p, mode, st); break;
        case 256: e = launch_merge_m<256>(p, mode, st); break;
        default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace tfp
