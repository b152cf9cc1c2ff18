// argmax.cu - greedy row argmax over bf16 logit rows.
//
// Rule (TensorFold #1503 "lfm2_moe CUDA: attention pages from the shared KV
// pool, and the prompt cache", commit list, lfm2_argmax): each row's first
// largest logit, ties to the lower id, a row holding a nonfinite logit
// flagged.  Readings: values compare as real numbers (-0 == +0), a flagged
// row reports id -1.
//
// Each row is split over a cluster of two CTAs of 1,024 threads (a 128,000-
// wide row is then one batch of eight 16-byte loads a thread, all in flight,
// with the fewest CTAs to launch and barriers to cross).  Every thread works
// on the 32-bit words it holds in registers, two bf16 values each:
// max.bf16x2 keeps the largest value of each half and max.u16x2 over the
// magnitude bits the largest exponent pattern (reaching 0x7f80 means a NaN or
// an infinity).  Values compare through key, an order-preserving 16-bit
// image with -0 mapped to +0's key.  The CTA's largest key comes from the
// warps' maxima (one barrier); then only the threads whose own largest value
// it is look for it again among their words with an IEEE compare (so -0
// equals +0), and the smallest column any of them finds is the CTA's first
// column holding it (a warp with none of those threads skips the search).
// The row's answer is the largest key and, among equal keys, the smallest
// column: each CTA stores its pair into rank 0's shared memory (distributed
// shared memory), one cluster barrier, and rank 0 writes the id and flag.
//
// A first split cluster barrier (arrive at entry, wait before the first
// remote store) makes sure every CTA of the cluster has started before any of
// them writes into another's shared memory.  Rank 0's slots alternate between
// two buffers by row parity, so a CTA that runs ahead on its next row never
// overwrites a pair rank 0 has not read yet.
//
// EARLY (the argmax of a verify round, launched right after this library's
// merge as a programmatic dependent): the logits are the caller's and no
// kernel of the round writes them, so the loads and reductions run while the
// merge drains; the writing thread waits for the merge's grid before it
// stores, so the argmax grid never completes before the merge's.

#include <cooperative_groups.h>

#include <climits>
#include <cstdint>

#include "tf_common.cuh"
#include "tf_internal.h"

namespace cg = cooperative_groups;

namespace tfp {

constexpr int kArgThreads = 1024;
constexpr int kArgBatch = 8;  // 16-byte vectors in flight per thread
constexpr int kArgWarps = kArgThreads / 32;

__device__ __forceinline__ uint32_t max_bf16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
// Per half: 0xffff where the two bf16 values are equal (so -0 equals +0).
__device__ __forceinline__ uint32_t eq_bf16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("set.eq.u32.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
// Order-preserving 16-bit key of one bf16 value, -0 taken as +0, and back
// (the inverse gives +0 for the zero key).
__device__ __forceinline__ uint32_t key16(uint32_t b) {
    b = (b == 0x8000u) ? 0u : b;
    return (b & 0x8000u) ? (b ^ 0xffffu) : (b | 0x8000u);
}
__device__ __forceinline__ uint32_t unkey16(uint32_t k) { return (k & 0x8000u) ? (k ^ 0x8000u) : (k ^ 0xffffu); }

// The pair with the largest key and, among equal keys, the smallest column,
// over the 32 lanes of a warp; every lane gets the answer.
__device__ __forceinline__ void warp_best(uint32_t &key, int &col) {
    const uint32_t k = __reduce_max_sync(0xffffffffu, key);
    col = __reduce_min_sync(0xffffffffu, key == k ? col : INT_MAX);
    key = k;
}

template <bool VEC, bool EARLY>
__global__ void __cluster_dims__(kArgmaxCluster, 1, 1) __launch_bounds__(kArgThreads)
    argmax_kernel(const ArgmaxParams p) {
    // a stand-alone call may run as a programmatic dependent of the launch
    // before it: nothing is read before that grid has finished
    if constexpr (!EARLY) asm volatile("griddepcontrol.wait;" ::: "memory");
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ uint32_t w_key[kArgWarps], w_bad[kArgWarps];
    __shared__ int s_col;  // the CTA's first column holding its largest value
    // rank 0's slots, filled by every CTA of the cluster, two buffers by row parity
    __shared__ uint32_t x_key[2][kArgmaxCluster], x_bad[2][kArgmaxCluster];
    __shared__ int x_col[2][kArgmaxCluster];

    // columns per CTA, a multiple of 8 so vectors never straddle two CTAs
    const int per = ((p.n_cols + kArgmaxCluster * 8 - 1) / (kArgmaxCluster * 8)) * 8;
    const int c0 = min(p.n_cols, rank * per), c1 = min(p.n_cols, c0 + per);
    const uint32_t kNegInf2 = 0xff80ff80u, kPad2 = 0xff7fff7fu;
    // A CTA may touch another CTA's shared memory only once every CTA of the
    // cluster is running: arrive here, wait before the first remote store
    // (the loads overlap the wait).
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
    bool joined = false, waited = !EARLY;

    for (int row = blockIdx.y, it = 0; row < p.n_rows; row += gridDim.y, ++it) {
        const uint16_t *rp = p.logits + (int64_t)row * p.ld;
        // ---- the thread's largest value and largest magnitude pattern
        uint32_t words[kArgBatch * 4];
        uint32_t vmax = kNegInf2, mag = 0u;
        const uint4 *vp = reinterpret_cast<const uint4 *>(rp);
        const int v0 = c0 >> 3, v1 = VEC ? (c1 >> 3) : v0;
        if constexpr (VEC) {
            // a thread's vectors are v0 + tid + k * kArgThreads
#pragma unroll
            for (int k = 0; k < kArgBatch; ++k) {
                const int v = v0 + tid + k * kArgThreads;
                // padding: the most negative finite bf16 (leaves the max and the
                // magnitude test alone; the column search skips it by index)
                const uint4 x = v < v1 ? __ldg(vp + v) : make_uint4(kPad2, kPad2, kPad2, kPad2);
                words[4 * k] = x.x;
                words[4 * k + 1] = x.y;
                words[4 * k + 2] = x.z;
                words[4 * k + 3] = x.w;
            }
#pragma unroll
            for (int k = 0; k < kArgBatch * 4; ++k) {
                vmax = max_bf16x2(vmax, words[k]);
                mag = max_u16x2(mag, words[k] & 0x7fff7fffu);
            }
            // vectors past the ones held (rows wider than 8 x 1,024 x 8 columns a CTA)
            for (int v = v0 + tid + kArgBatch * kArgThreads; v < v1; v += kArgThreads) {
                const uint4 x = __ldg(vp + v);
                const uint32_t wd[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    vmax = max_bf16x2(vmax, wd[e]);
                    mag = max_u16x2(mag, wd[e] & 0x7fff7fffu);
                }
            }
        }
        // scalar columns: the row's ragged tail, or everything without 16-byte access
        for (int c = (VEC ? (v1 << 3) : c0) + tid; c < c1; c += kArgThreads) {
            const uint32_t b = rp[c];
            vmax = max_bf16x2(vmax, b | 0xff800000u);
            mag = max_u16x2(mag, b & 0x7fffu);
        }
        // nonfinite: some half's magnitude pattern reached the all-ones exponent
        const uint32_t bad = ((mag & 0xffffu) >= 0x7f80u || (mag >> 16) >= 0x7f80u) ? 1u : 0u;
        const uint32_t key = max(key16(vmax & 0xffffu), key16(vmax >> 16));
        // ---- the CTA's largest key: each warp's maximum, then every warp
        // reduces the 32 warps' (one barrier)
        const uint32_t wbad = __reduce_or_sync(0xffffffffu, bad);
        {
            const uint32_t wkey = __reduce_max_sync(0xffffffffu, key);
            if (lane == 0) {
                w_key[warp] = wkey;
                w_bad[warp] = wbad;
            }
        }
        if (it == 0 && tid == 0) s_col = INT_MAX;
        __syncthreads();
        const uint32_t ckey = __reduce_max_sync(0xffffffffu, w_key[lane]);  // kArgWarps == 32: a lane a warp
        // ---- the first column holding the CTA's largest value, looked for
        // again only by the threads whose own largest value it is (a warp with
        // none of them skips the search)
        auto first_col = [&](uint32_t M) -> int {
            const uint32_t M2 = M | (M << 16);
            int col = INT_MAX;
            if constexpr (VEC) {
#pragma unroll
                for (int j = 0; j < kArgBatch * 4; ++j) {
                    const uint32_t e = eq_bf16x2(words[j], M2);
                    const int v = v0 + tid + (j >> 2) * kArgThreads;
                    if (col == INT_MAX && e && v < v1) col = v * 8 + (j & 3) * 2 + ((e & 0xffffu) ? 0 : 1);
                }
                for (int v = v0 + tid + kArgBatch * kArgThreads; v < v1 && col == INT_MAX; v += kArgThreads) {
                    const uint4 x = __ldg(vp + v);
                    const uint32_t wd[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t e = eq_bf16x2(wd[q], M2);
                        if (col == INT_MAX && e) col = v * 8 + 2 * q + ((e & 0xffffu) ? 0 : 1);
                    }
                }
            }
            for (int c = (VEC ? (v1 << 3) : c0) + tid; c < c1 && col == INT_MAX; c += kArgThreads)
                if (eq_bf16x2(rp[c], M) & 0xffffu) col = c;
            return col;
        };
        if (__any_sync(0xffffffffu, key == ckey)) {
            const int col = __reduce_min_sync(0xffffffffu, key == ckey ? first_col(unkey16(ckey)) : INT_MAX);
            if (lane == 0) atomicMin(&s_col, col);
        }
        // ---- the CTA's pair, then the cluster's on rank 0
        if (!joined) {
            asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
            joined = true;
        }
        __syncthreads();
        const int buf = it & 1;
        if (warp == 0) {
            const uint32_t b = __reduce_or_sync(0xffffffffu, w_bad[lane]);
            if (lane == 0) {
                *cluster.map_shared_rank(&x_key[buf][rank], 0) = ckey;
                *cluster.map_shared_rank(&x_col[buf][rank], 0) = s_col;
                *cluster.map_shared_rank(&x_bad[buf][rank], 0) = b;
                s_col = INT_MAX;  // for the next row (read here, set again after its first barrier)
            }
        }
        cluster.sync();
        if (rank == 0 && tid == 0) {
            uint32_t K = 0, B = 0;
            int C = INT_MAX;
#pragma unroll
            for (int i = 0; i < kArgmaxCluster; ++i) {
                const uint32_t k = x_key[buf][i];
                const int c = x_col[buf][i];
                if (k > K || (k == K && c < C)) {
                    K = k;
                    C = c;
                }
                B |= x_bad[buf][i];
            }
            if (!waited) {
                asm volatile("griddepcontrol.wait;" ::: "memory");
                waited = true;
            }
            p.ids[row] = B ? -1 : C;
            p.flags[row] = (uint8_t)(B ? 1 : 0);
        }
    }
}

cudaError_t launch_argmax(const ArgmaxParams &p, bool vec, bool early, cudaStream_t st) {
    if (p.n_rows == 0) return cudaSuccess;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(kArgmaxCluster, (unsigned)(p.n_rows < 65535 ? p.n_rows : 65535));
    cfg.blockDim = dim3(kArgThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (early)
        return vec ? cudaLaunchKernelEx(&cfg, argmax_kernel<true, true>, p)
                   : cudaLaunchKernelEx(&cfg, argmax_kernel<false, true>, p);
    return vec ? cudaLaunchKernelEx(&cfg, argmax_kernel<true, false>, p)
               : cudaLaunchKernelEx(&cfg, argmax_kernel<false, false>, p);
}

}  // namespace tfp
