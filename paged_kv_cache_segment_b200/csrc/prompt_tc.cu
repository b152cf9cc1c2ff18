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
//      one tile ahead of the softmax (two S buffers);
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
// K and V each have two buffers; a buffer is refilled as soon as the MMA that
// read it has completed.
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
constexpr int kQM = 128;                      // queries a CTA (the MMA's M)
constexpr int kBN = 64;                       // keys a tile
constexpr int kQSlab = kQM * 128;             // 128 query rows x 128 bytes
constexpr int kKVSlab = kBN * 128;            // 64 key rows x 128 bytes
constexpr uint32_t kColS0 = 0, kColS1 = 64, kColO = 256;  // tensor-memory columns

template <int D>
struct PTCfg {
    static constexpr int kSlabs = D / 64;
    static constexpr int kQBytes = kSlabs * kQSlab;
    static constexpr int kKVBytes = kSlabs * kKVSlab;
    // Q, two K buffers, two V buffers
    static constexpr int kOffK = kQBytes;
    static constexpr int kOffV = kQBytes + 2 * kKVBytes;
    static constexpr int kPidCap = 4096;  // page ids held in shared memory (16 KB)
    static constexpr int kOffPid = kQBytes + 4 * kKVBytes;
    static constexpr int kSmemBytes = kOffPid + kPidCap * 4 + 1024;
    static constexpr uint32_t kTmemCols = 512;
};

// Bounded wait that gives up at once after any thread of the CTA gave up, so
// every role keeps its barrier sequence without waiting twice the timeout.
__device__ __forceinline__ bool pt_wait(uint32_t bar, uint32_t phase, volatile uint32_t *abort_flag) {
    if (*abort_flag) return false;
    if (mbar_wait(bar, phase)) return true;
    *abort_flag = 1;
    return false;
}

template <int D, bool HILO>
__global__ void __launch_bounds__(kPTThreads, 1)
    prompt_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const PromptTcParams p) {
    using C = PTCfg<D>;
    extern __shared__ unsigned char smem_raw[];
    // barriers: q; k[2]; v[2]; s[2] (QK done); pr[2] (P written, V cleaned); o[2] (PV done)
    __shared__ __align__(8) uint64_t bars[11];
    __shared__ uint32_t s_tmem;
    __shared__ uint32_t s_vbad[4];
    __shared__ uint32_t s_err, s_abort;
    __shared__ float s_xmax[2][2][kQM];     // [tile parity][column half][row]: the halves' tile maxima
    __shared__ float s_xl[2][kQM];          // [column half][row]: final partial sums
    __shared__ uint32_t s_xbad[2][2][kQM];  // [exchange][column half][row]: nonfinite findings

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    unsigned char *sbase_ptr = smem_raw + (sbase - smem_u32(smem_raw));
    const uint32_t sQ = sbase;
    auto sK = [&](int b) { return sbase + C::kOffK + b * C::kKVBytes; };
    auto sV = [&](int b) { return sbase + C::kOffV + b * C::kKVBytes; };
    const uint32_t bq = smem_u32(&bars[0]);
    auto bk = [&](int b) { return smem_u32(&bars[1 + b]); };
    auto bv = [&](int b) { return smem_u32(&bars[3 + b]); };
    auto bsq = [&](int b) { return smem_u32(&bars[5 + b]); };
    auto bpr = [&](int b) { return smem_u32(&bars[7 + b]); };
    auto bo = [&](int b) { return smem_u32(&bars[9 + b]); };
    volatile uint32_t *abort_flag = &s_abort;

    const int G = p.group, RT = kQM / p.group;  // rows a tile
    const int g = blockIdx.y;
    const int qt = (int)gridDim.x - 1 - (int)blockIdx.x;  // the most keys first
    const int row0 = qt * RT;                              // chunk-relative first row
    const int T = p.n_rows, N = p.n_keys;
    const int rows_here = min(RT, T - row0);
    const int key_hi_eff = N - T + row0 + rows_here;  // keys the last valid row sees
    const int full_hi = N - T + row0 + 1;             // keys every row of the tile sees
    const int n_tiles = (key_hi_eff + kBN - 1) / kBN;
    const int P = 1 << p.log2_page, BR = P < kBN ? P : kBN, n_box = kBN / BR;

    // The CTA's page ids, read once here by every thread (coalesced), so the
    // issuer never waits on a page-table read inside the key loop.
    int *pids = reinterpret_cast<int *>(sbase_ptr + C::kOffPid);
    const int n_pid = min((key_hi_eff + P - 1) >> p.log2_page, p.n_pg);
    for (int i = tid; i < n_pid && i < C::kPidCap; i += kPTThreads) {
        const int id = p.page_table[p.pt_base + i];
        pids[i] = (id < 0 || id >= p.n_pages) ? -1 : id;
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(&s_tmem), C::kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 11; ++i) mbar_init(smem_u32(&bars[i]), (i >= 7 && i <= 8) ? kPTSoftmax / 32u : 1u);
        fence_barrier_init();
        s_err = 0;
        s_abort = 0;
        s_vbad[0] = s_vbad[1] = s_vbad[2] = s_vbad[3] = 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    // every lane of a helper warp waits; the answer is the warp's, so all lanes branch alike
    auto wwait = [&](uint32_t bar, uint32_t phase) { return __all_sync(0xffffffffu, pt_wait(bar, phase, abort_flag)); };
    if (warp == kPTTmaWarp) {
        // ================= TMA warp: the K/V boxes of a tile go out one per lane,
        // so one warp instruction issues all of them; a buffer is refilled as
        // soon as the MMA that read it is done
        if (lane == 0) {
            prefetch_tensormap(&tmQ);
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
        }
        const int n_copies = n_box * C::kSlabs;  // boxes of one K (or V) tile, <= 32
        // K or V tile t into buffer t & 1: one box per page (or per 64-key span
        // of a larger page) and 64-column slab; page ids come from shared memory
        auto issue_kv = [&](int t, bool is_v) {
            const int kt = t * kBN, b = t & 1;
            const uint32_t dst0 = is_v ? sV(b) : sK(b);
            const uint32_t bar = is_v ? bv(b) : bk(b);
            const CUtensorMap *map = is_v ? &tmV : &tmK;
            // lane i < n_copies owns box x = i / slabs, slab sl = i % slabs
            const int x = lane / C::kSlabs, sl = lane % C::kSlabs;
            const int key0 = kt + x * BR;
            int id = -1;
            if (lane < n_copies && key0 < key_hi_eff) {
                const int idx = key0 >> p.log2_page;
                if (idx >= p.n_pg)
                    id = -2;
                else if (idx < C::kPidCap)
                    id = pids[idx];
                else  // past the shared-memory copy (very long prompts with small pages)
                    id = p.page_table[p.pt_base + idx];
                if (id < 0 || id >= p.n_pages) {
                    id = -1;
                    s_err = 1;
                    atomicOr(p.status, TF_DEV_BAD_PAGE);
                }
            }
            const uint32_t live = __ballot_sync(0xffffffffu, id >= 0);
            if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)__popc(live) * (uint32_t)(BR * 128));
            __syncwarp();
            if (id >= 0) tma_load_4d(dst0 + sl * kKVSlab + x * BR * 128, map, bar, 64 * sl, key0 & (P - 1), g, id);
        };
        if (lane == 0) mbar_arrive_expect_tx(bq, (uint32_t)C::kQBytes);
        __syncwarp();
        if (lane < C::kSlabs) tma_load_3d(sQ + lane * kQSlab, &tmQ, bq, 64 * lane, g * G, p.q_row + row0);
        for (int t = 0; t < n_tiles; ++t) {
            const int pb = (t - 2) & 1;
            const uint32_t pph = (uint32_t)(((t - 2) >> 1) & 1);
            // K(t) once QK(t-2) has read the buffer, V(t) once P V(t-2) has
            if (t >= 2 && !wwait(bsq(pb), pph)) break;
            issue_kv(t, false);
            if (t >= 2 && !wwait(bo(pb), pph)) break;
            issue_kv(t, true);
        }
    } else if (warp == kPTMmaWarp) {
        // ================= MMA warp: lane 0 issues every tcgen05.mma
        const uint32_t idesc_qk = umma_idesc_bf16(kQM, kBN, false, false);
        const uint32_t idesc_pv = umma_idesc_bf16(kQM, D, false, true);
        auto issue_qk = [&](int t) {
            if (lane == 0) {
                const int b = t & 1;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const int sl = k >> 2, kk = k & 3;
                    const uint64_t ad = umma_desc_sw128(sQ + sl * kQSlab + kk * 32, 16, 1024);
                    const uint64_t bd = umma_desc_sw128(sK(b) + sl * kKVSlab + kk * 32, 16, 1024);
                    umma_ss(tmem + (b ? kColS1 : kColS0), ad, bd, idesc_qk, k > 0 ? 1u : 0u);
                }
                umma_commit(bsq(b));
            }
            __syncwarp();
        };
        if (n_tiles > 0 && wwait(bq, 0) && wwait(bk(0), 0)) issue_qk(0);
        for (int j = 0; j < n_tiles; ++j) {
            const int b = j & 1;
            const uint32_t ph = (uint32_t)((j >> 1) & 1);
            // the next tile's scores while the softmax warps work on this one;
            // its S buffer held P(j-1), whose P V was issued before (in order)
            if (j + 1 < n_tiles && wwait(bk((j + 1) & 1), (uint32_t)(((j + 1) >> 1) & 1))) issue_qk(j + 1);
            // P(j) written (and V(j) cleaned) and V(j) landed: O += P V
            const bool ok = wwait(bpr(b), ph) && wwait(bv(b), ph);
            if (ok && lane == 0) {
                tc_fence_after();
                const uint32_t sb = tmem + (b ? kColS1 : kColS0);
#pragma unroll
                for (int kk = 0; kk < kBN / 16; ++kk) {
                    const uint64_t bd = umma_desc_sw128(sV(b) + kk * 16 * 128, kKVSlab, 1024);
                    umma_ts(tmem + kColO, sb + kk * 8, bd, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
                    if (HILO) umma_ts(tmem + kColO, sb + 32 + kk * 8, bd, idesc_pv, 1u);
                }
                umma_commit(bo(b));
            }
            __syncwarp();
        }
    } else {
        // ================= softmax warps: row qi of the tile, key columns 32h .. 32h + 31
        const int quad = warp & 3, h = warp >> 2;
        const int qi = quad * 32 + lane;
        const int row_i = row0 + qi / G;  // chunk-relative
        const bool valid_row = row_i < T;
        const int lim = valid_row ? (N - T + row_i + 1) : key_hi_eff;
        const float scale_log2 = p.scale_log2;
        float m_ref = -INFINITY, l_run = 0.f;
        uint32_t emax = 0, tail_bad = 0;
        const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
        const uint32_t pair_bar = 2 + quad;  // warps quad and quad + 4

        for (int j = 0; j < n_tiles; ++j) {
            const int b = j & 1, kt = j * kBN;
            const uint32_t ph = (uint32_t)((j >> 1) & 1);
            const uint32_t colS = b ? kColS1 : kColS0;
            const int kh = kt + 32 * h;  // this half's first key
            pt_wait(bsq(b), ph, abort_flag);
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
                    const bool vis = kh + c < lim;
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
                pt_wait(bo((j - 1) & 1), (uint32_t)(((j - 1) >> 1) & 1), abort_flag);
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
                pt_wait(bv(b), ph, abort_flag);
                named_bar_sync(1, kPTSoftmax);
                if (tid == 0) s_vbad[0] = s_vbad[1] = 0;
                named_bar_sync(1, kPTSoftmax);
                unsigned char *vb = sbase_ptr + C::kOffV + b * C::kKVBytes;
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
                        if (((((r < 32) ? vb0 : vb1) >> (r & 31)) & 1u) && kt + r < lim) tail_bad = 1;
                }
                fence_proxy_async_smem();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bpr(b));
        }

        // ---- epilogue: the halves' sums and findings meet, then each half
        // divides and stores its D/2 columns of O
        if (n_tiles > 0) pt_wait(bo((n_tiles - 1) & 1), (uint32_t)(((n_tiles - 1) >> 1) & 1), abort_flag);
        tc_fence_after();
        const bool aborted = *abort_flag != 0;
        s_xl[h][qi] = l_run;
        s_xbad[0][h][qi] = (emax == 0x7f800000u ? 1u : 0u) | tail_bad;
        named_bar_sync(pair_bar, 64);
        const float l_sum = s_xl[0][qi] + s_xl[1][qi];
        uint32_t bad = s_xbad[0][0][qi] | s_xbad[0][1][qi] | s_err | (aborted ? 1u : 0u);
        if (!(l_sum > 0.f) || !isfinite(l_sum)) bad = 1;
        const int64_t u = (int64_t)(p.q_row + row_i) * p.hq + g * G + (qi % G);
        const int d0 = h * (D / 2);
        uint32_t obad = 0;
#pragma unroll 1
        for (int c = 0; c < D / 64; ++c) {
            uint32_t r[32];
            tmem_ld32(lane_base + kColO + d0 + c * 32, r);
            tmem_wait_ld();
            float o[32];
#pragma unroll
            for (int w = 0; w < 32; ++w) {
                o[w] = __uint_as_float(r[w]) / l_sum;
                obad |= !isfinite(o[w]);
            }
            if (valid_row && !aborted) {
                if (p.out_bf16) {
                    uint4 *dst =
                        reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(p.out) + u * D + d0 + c * 32);
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        dst[w] = make_uint4(pack_bf16x2(o[8 * w], o[8 * w + 1]), pack_bf16x2(o[8 * w + 2], o[8 * w + 3]),
                                            pack_bf16x2(o[8 * w + 4], o[8 * w + 5]),
                                            pack_bf16x2(o[8 * w + 6], o[8 * w + 7]));
                } else {
                    float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(p.out) + u * D + d0 + c * 32);
#pragma unroll
                    for (int w = 0; w < 8; ++w) dst[w] = make_float4(o[4 * w], o[4 * w + 1], o[4 * w + 2], o[4 * w + 3]);
                }
            }
        }
        // a nonfinite output in either half flags the whole row
        s_xbad[1][h][qi] = obad;
        named_bar_sync(pair_bar, 64);
        bad |= s_xbad[1][0][qi] | s_xbad[1][1][qi];
        if (valid_row) {
            if (bad) {
                const float qnan = __int_as_float(0x7fc00000);
                for (int d = d0; d < d0 + D / 2; d += 8) {
                    if (p.out_bf16)
                        *reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(p.out) + u * D + d) =
                            make_uint4(0x7fc07fc0u, 0x7fc07fc0u, 0x7fc07fc0u, 0x7fc07fc0u);
                    else {
                        float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(p.out) + u * D + d);
                        dst[0] = make_float4(qnan, qnan, qnan, qnan);
                        dst[1] = make_float4(qnan, qnan, qnan, qnan);
                    }
                }
            }
            if (p.out_flags && h == 0) p.out_flags[u] = (uint8_t)(bad ? 1 : 0);
        }
    }
    // everyone: report a timeout, give in-flight work a bounded chance to land,
    // release tensor memory
    __syncthreads();
    if (s_abort) {
        if (tid == 0) atomicOr(p.status, TF_DEV_TIMEOUT);
        if (tid == 0)
            for (int i = 0; i < 11; ++i) {
                mbar_wait(smem_u32(&bars[i]), 0u, 20000000ull);
                mbar_wait(smem_u32(&bars[i]), 1u, 20000000ull);
            }
        __syncthreads();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// host side: tensor maps and launch
// ---------------------------------------------------------------------------

bool prompt_tc_supported(int head_dim, int group, int page_size) {
    return (head_dim == 64 || head_dim == 128 || head_dim == 256) && group >= 1 && group <= 128 &&
           (128 % group) == 0 && page_size >= 8;
}

template <int D>
static cudaError_t launch_prompt_tc_t(const PromptTcParams &p, const void *q, const void *k, const void *v,
                                      cudaStream_t st) {
    CUtensorMap mq, mk, mv;
    const int G = p.group, RT = kQM / G, P = 1 << p.log2_page, BR = P < kBN ? P : kBN;
    {
        const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)p.hq, (cuuint64_t)p.n_rows_total};
        const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)p.hq * D * 2};
        const cuuint32_t box[3] = {64, (cuuint32_t)G, (cuuint32_t)RT};
        if (!make_tensor_map_bf16(&mq, q, 3, dims, strides, box)) return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)P, (cuuint64_t)p.hkv, (cuuint64_t)p.n_pages};
        const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)P * D * 2, (cuuint64_t)p.hkv * P * D * 2};
        const cuuint32_t box[4] = {64, (cuuint32_t)BR, 1, 1};
        if (!make_tensor_map_bf16(&mk, k, 4, dims, strides, box)) return cudaErrorInvalidValue;
        if (!make_tensor_map_bf16(&mv, v, 4, dims, strides, box)) return cudaErrorInvalidValue;
    }
    auto kern = p.out_bf16 ? prompt_tc_kernel<D, false> : prompt_tc_kernel<D, true>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PTCfg<D>::kSmemBytes);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((p.n_rows + RT - 1) / RT), (unsigned)p.hkv);
    kern<<<grid, kPTThreads, PTCfg<D>::kSmemBytes, st>>>(mq, mk, mv, p);
    return cudaGetLastError();
}

cudaError_t launch_prompt_tc(const PromptTcParams &p, int head_dim, const void *q, const void *k, const void *v,
                             cudaStream_t st) {
    switch (head_dim) {
        case 64: return launch_prompt_tc_t<64>(p, q, k, v, st);
        case 128: return launch_prompt_tc_t<128>(p, q, k, v, st);
        case 256: return launch_prompt_tc_t<256>(p, q, k, v, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace tfp
