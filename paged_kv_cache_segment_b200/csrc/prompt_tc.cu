// prompt_tc.cu - causal prompt chunk through the page table on the 5th-generation
// tensor cores (tcgen05 + tensor memory), tiles fed by TMA.
//
// Source: TensorFold #1653 "spark25 CUDA: the full layers' caches in pages of
// the core pool", commit list and PR body: prompt rows read the chunk's keys
// through the slot's page-table row (the _pg prompt kernel, head dim 256,
// pages of 32); review thread: the per-chunk page lookup is hoisted out of the
// key loop.
//
// One CTA of four warps computes 128 queries: 128/G consecutive rows x the G
// q-heads that share kv-head g, so one K/V tile serves all of them.  Per
// 128-key tile:
//   1. TMA brings K (and V) in 128-byte-swizzled 64-column slabs; page ids are
//      resolved once per tile (a box per page), so no lookup sits in any
//      inner loop;
//   2. one thread issues S = Q K^T (M 128, N 128, K = D) into tensor memory;
//   3. every thread owns one query row: it loads its S row from tensor memory,
//      masks it causally, and folds it into a running max / sum with a lazy
//      rescale (the reference max moves only when it rises by more than 2^8);
//   4. the weights go back to tensor memory as bf16 hi + bf16 lo and one
//      thread issues O += P_hi V + P_lo V (A from tensor memory, B = V in
//      shared memory, MN-major), so each weight keeps about 16 bits;
//   5. O stays in tensor memory until the epilogue divides by the sum.
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

constexpr int kPTThreads = 128;
constexpr int kBN = 128;                // keys per tile
constexpr int kSlabBytes = 128 * 128;   // 128 rows x 128 bytes (64 bf16 columns)
constexpr uint32_t kColS = 0, kColPhi = 128, kColPlo = 192, kColO = 256;

template <int D>
struct PTCfg {
    static constexpr int kSlabs = D / 64;
    static constexpr int kTileBytes = kSlabs * kSlabBytes;  // 128 rows x D bf16
    static constexpr int kSmemBytes = 3 * kTileBytes + 1024; // Q, K, V + alignment slack
    static constexpr uint32_t kTmemCols = (256 + D) <= 512 ? 512 : 0;
};

__device__ __forceinline__ void report_timeout(uint32_t *status) { atomicOr(status, TF_DEV_TIMEOUT); }

template <int D>
__global__ void __launch_bounds__(kPTThreads, 1)
    prompt_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const PromptTcParams p) {
    using C = PTCfg<D>;
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t bars[5];  // q, k, v, s, o
    __shared__ uint32_t s_tmem;
    __shared__ uint32_t s_vbad[4];
    __shared__ int s_err;

    const int tid = threadIdx.x, warp = tid >> 5;
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    unsigned char *sbase_ptr = smem_raw + (sbase - smem_u32(smem_raw));
    const uint32_t sQ = sbase, sK = sbase + C::kTileBytes, sV = sbase + 2 * C::kTileBytes;
    const uint32_t bq = smem_u32(&bars[0]), bk = smem_u32(&bars[1]), bv = smem_u32(&bars[2]),
                   bs = smem_u32(&bars[3]), bo = smem_u32(&bars[4]);

    const int G = p.group, RT = kBN / p.group;  // rows per tile
    const int g = blockIdx.y;
    const int qt = (int)gridDim.x - 1 - (int)blockIdx.x;  // the most keys first
    const int row0 = qt * RT;                              // chunk-relative first row
    const int T = p.n_rows, N = p.n_keys;
    const int rows_here = min(RT, T - row0);
    const int key_hi_eff = N - T + row0 + rows_here;  // keys the last valid row sees
    const int full_hi = N - T + row0 + 1;             // keys every row of the tile sees
    const int n_tiles = (key_hi_eff + kBN - 1) / kBN;
    const int P = 1 << p.log2_page, BR = P < kBN ? P : kBN, n_box = kBN / BR;

    if (warp == 0) {
        tmem_alloc(smem_u32(&s_tmem), C::kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 5; ++i) mbar_init(smem_u32(&bars[i]), 1);
        fence_barrier_init();
        s_err = 0;
        s_vbad[0] = s_vbad[1] = s_vbad[2] = s_vbad[3] = 0;
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    // K or V tile t into its buffer: one box per page (or per 128-key span of a
    // larger page); page ids are read once here, the tile's only lookup.
    auto issue_kv = [&](int t, bool is_v) {
        const int kt = t * kBN;
        const uint32_t dst0 = is_v ? sV : sK;
        const uint32_t bar = is_v ? bv : bk;
        const CUtensorMap *map = is_v ? &tmV : &tmK;
        int pid[16];
        uint32_t bytes = 0;
        for (int b = 0; b < n_box; ++b) {
            const int key0 = kt + b * BR;
            int id = -1;
            if (key0 < key_hi_eff) {
                const int idx = key0 >> p.log2_page;
                id = (idx < p.n_pg) ? p.page_table[p.pt_base + idx] : -2;
                if (id < 0 || id >= p.n_pages) {
                    id = -1;
                    s_err = 1;
                    atomicOr(p.status, TF_DEV_BAD_PAGE);
                } else {
                    bytes += (uint32_t)(BR * 128 * C::kSlabs);
                }
            }
            pid[b] = id;
        }
        mbar_arrive_expect_tx(bar, bytes);
        for (int b = 0; b < n_box; ++b) {
            if (pid[b] < 0) continue;
            const int key0 = kt + b * BR;
            for (int s = 0; s < C::kSlabs; ++s)
                tma_load_4d(dst0 + s * kSlabBytes + b * BR * 128, map, bar, 64 * s, key0 & (P - 1), g, pid[b]);
        }
    };

    if (tid == 0) {
        mbar_arrive_expect_tx(bq, (uint32_t)C::kTileBytes);
        for (int s = 0; s < C::kSlabs; ++s) tma_load_3d(sQ + s * kSlabBytes, &tmQ, bq, 64 * s, g * G, p.q_row + row0);
        if (n_tiles > 0) {
            issue_kv(0, false);
            issue_kv(0, true);
        }
    }

    // this thread's query
    const int qi = tid;
    const int row_i = row0 + qi / G;  // chunk-relative
    const bool valid_row = row_i < T;
    const int lim = valid_row ? (N - T + row_i + 1) : key_hi_eff;
    const float scale_log2 = p.scale_log2;
    float m_ref = -INFINITY, l_run = 0.f;
    uint32_t emax = 0, tail_bad = 0, timed_out = 0;

    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const uint32_t idesc_qk = umma_idesc_bf16(128, kBN, false, false);
    const uint32_t idesc_pv = umma_idesc_bf16(128, D, false, true);

    for (int t = 0; t < n_tiles; ++t) {
        const int kt = t * kBN;
        const uint32_t ph = (uint32_t)(t & 1);
        // ---- S = Q K^T
        if (!mbar_wait(bk, ph)) timed_out = 1;
        if (t == 0 && !mbar_wait(bq, 0)) timed_out = 1;
        if (__syncthreads_or(timed_out)) break;
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const int s = k >> 2, kk = k & 3;
                const uint64_t ad = umma_desc_sw128(sQ + s * kSlabBytes + kk * 32, 16, 1024);
                const uint64_t bd = umma_desc_sw128(sK + s * kSlabBytes + kk * 32, 16, 1024);
                umma_ss(tmem + kColS, ad, bd, idesc_qk, k > 0 ? 1u : 0u);
            }
            umma_commit(bs);
        }
        if (!mbar_wait(bs, ph)) timed_out = 1;
        if (__syncthreads_or(timed_out)) break;
        tc_fence_after();
        if (tid == 0 && t + 1 < n_tiles) issue_kv(t + 1, false);  // the K buffer is free again

        // ---- softmax over this thread's row
        float sv[kBN];
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(lane_base + kColS + c * 32, r);
#pragma unroll
            for (int j = 0; j < 32; ++j) sv[c * 32 + j] = __uint_as_float(r[j]);
        }
        tmem_wait_ld();
        const bool need_mask = kt + kBN > full_hi;
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < kBN; ++c) {
            float x = sv[c] * scale_log2;
            const bool vis = !need_mask || (kt + c < lim);
            emax = max(emax, vis ? exp_bits(x) : 0u);
            x = vis ? x : -INFINITY;
            sv[c] = x;
            mx = fmaxf(mx, x);
        }
        float alpha = 1.f;
        if (mx > m_ref + 8.f || (m_ref == -INFINITY && mx != -INFINITY)) {
            alpha = (m_ref == -INFINITY) ? 0.f : ex2(m_ref - mx);
            m_ref = mx;
        }
        const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
        float ls = 0.f;
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) {
            uint32_t hi[16], lo[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float p0 = ex2(sv[c * 32 + 2 * j] - mu), p1 = ex2(sv[c * 32 + 2 * j + 1] - mu);
                ls += p0 + p1;
                hi[j] = pack_bf16x2(p0, p1);
                lo[j] = pack_bf16x2(p0 - bf16_lo_to_f32(hi[j]), p1 - bf16_hi_to_f32(hi[j]));
            }
            tmem_st16(lane_base + kColPhi + c * 16, hi);
            tmem_st16(lane_base + kColPlo + c * 16, lo);
        }
        l_run = l_run * alpha + ls;
        // rescale O when this row's reference max moved (O holds the previous tiles)
        if (t > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(lane_base + kColO + c * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * alpha);
                tmem_st32(lane_base + kColO + c * 32, r);
            }
        }
        tmem_wait_st();

        // ---- V: wait, then clean the rows this tile must not feed into P V
        if (!mbar_wait(bv, ph)) timed_out = 1;
        if (__syncthreads_or(timed_out)) break;
        if (kt + kBN > full_hi) {
            // rows past every valid row's keys: zero; rows only some rows see: zero if nonfinite
            for (int idx = tid; idx < kBN * C::kSlabs; idx += kPTThreads) {
                const int r = idx % kBN, s = idx / kBN;
                const int key = kt + r;
                uint4 *rowp = reinterpret_cast<uint4 *>(sbase_ptr + 2 * C::kTileBytes + s * kSlabBytes + r * 128);
                if (key >= key_hi_eff) {
#pragma unroll
                    for (int k = 0; k < 8; ++k) rowp[k] = make_uint4(0, 0, 0, 0);
                } else if (key >= full_hi) {
                    bool nf = false;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint4 v = rowp[k];
                        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            nf |= ((w[e] & 0x7f80u) == 0x7f80u) || ((w[e] & 0x7f800000u) == 0x7f800000u);
                    }
                    if (nf) atomicOr(&s_vbad[r >> 5], 1u << (r & 31));
                }
            }
            __syncthreads();
            const uint32_t vb[4] = {s_vbad[0], s_vbad[1], s_vbad[2], s_vbad[3]};
            if (vb[0] | vb[1] | vb[2] | vb[3]) {
                for (int idx = tid; idx < kBN * C::kSlabs; idx += kPTThreads) {
                    const int r = idx % kBN, s = idx / kBN;
                    if ((vb[r >> 5] >> (r & 31)) & 1u) {
                        uint4 *rowp =
                            reinterpret_cast<uint4 *>(sbase_ptr + 2 * C::kTileBytes + s * kSlabBytes + r * 128);
#pragma unroll
                        for (int k = 0; k < 8; ++k) rowp[k] = make_uint4(0, 0, 0, 0);
                    }
                }
                for (int r = 0; r < kBN; ++r)
                    if (((vb[r >> 5] >> (r & 31)) & 1u) && kt + r < lim) tail_bad = 1;
            }
            fence_proxy_async_smem();
            __syncthreads();
            if (tid == 0) s_vbad[0] = s_vbad[1] = s_vbad[2] = s_vbad[3] = 0;
        }
        tc_fence_before();
        __syncthreads();

        // ---- O += P V (A = P from tensor memory, B = V MN-major)
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < kBN / 16; ++kk) {
                const uint64_t bd = umma_desc_sw128(sV + kk * 16 * 128, kSlabBytes, 1024);
                umma_ts(tmem + kColO, tmem + kColPhi + kk * 8, bd, idesc_pv, (t > 0 || kk > 0) ? 1u : 0u);
                umma_ts(tmem + kColO, tmem + kColPlo + kk * 8, bd, idesc_pv, 1u);
            }
            umma_commit(bo);
        }
        if (!mbar_wait(bo, ph)) timed_out = 1;
        if (__syncthreads_or(timed_out)) break;
        tc_fence_after();
        if (tid == 0 && t + 1 < n_tiles) issue_kv(t + 1, true);  // the V buffer is free again
    }

    // ---- epilogue: O / l, nonfinite check, store
    timed_out = __syncthreads_or(timed_out) ? 1u : 0u;  // uniform over the CTA
    if (timed_out) {
        // give in-flight copies and MMAs a bounded chance to land before the
        // tensor memory is released
        if (tid == 0) report_timeout(p.status);
        for (int i = 0; i < 2; ++i) {
            mbar_wait(bk, (uint32_t)i, 20000000ull);
            mbar_wait(bv, (uint32_t)i, 20000000ull);
            mbar_wait(bs, (uint32_t)i, 20000000ull);
            mbar_wait(bo, (uint32_t)i, 20000000ull);
        }
    }
    uint32_t bad = (emax == 0x7f800000u) | tail_bad | (uint32_t)s_err | timed_out;
    if (!(l_run > 0.f) || !isfinite(l_run)) bad = 1;
    const int64_t u = (int64_t)(p.q_row + row_i) * p.hq + g * G + (qi % G);
    if (!timed_out) {
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(lane_base + kColO + c * 32, r);
            tmem_wait_ld();
            float o[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                o[j] = __uint_as_float(r[j]) / l_run;
                bad |= !isfinite(o[j]);
            }
            if (valid_row) {
                if (p.out_bf16) {
                    uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(p.out) + u * D + c * 32);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        dst[j] = make_uint4(pack_bf16x2(o[8 * j], o[8 * j + 1]), pack_bf16x2(o[8 * j + 2], o[8 * j + 3]),
                                            pack_bf16x2(o[8 * j + 4], o[8 * j + 5]),
                                            pack_bf16x2(o[8 * j + 6], o[8 * j + 7]));
                } else {
                    float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(p.out) + u * D + c * 32);
#pragma unroll
                    for (int j = 0; j < 8; ++j) dst[j] = make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
                }
            }
        }
    }
    if (valid_row) {
        if (bad) {
            const float qnan = __int_as_float(0x7fc00000);
            for (int d = 0; d < D; d += 8) {
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
        if (p.out_flags) p.out_flags[u] = (uint8_t)(bad ? 1 : 0);
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
    const int G = p.group, RT = 128 / G, P = 1 << p.log2_page, BR = P < 128 ? P : 128;
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
    auto kern = prompt_tc_kernel<D>;
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
