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
// on 32-bit words, two bf16
// values each: max.bf16x2 keeps the largest value of each half and
// max.u16x2 over the magnitude bits keeps the largest exponent pattern
// (reaching 0x7f80 means a NaN or an infinity).  The cluster agrees on the
// row's largest value (each CTA stores its block maximum, as an
// order-preserving 16-bit key, into every CTA's shared memory; one cluster
// barrier; local reads), then each thread finds the first column equal to it
// among the words it still holds in registers (an IEEE compare, so -0 equals
// +0), and the CTAs' first columns meet on rank 0 the same way.  No
// workspace and no inter-CTA counters: the cluster barriers order the
// exchanges, and a first split barrier (arrive at entry, wait before the
// first remote store) makes sure every CTA of the cluster has started before
// any of them writes into another's shared memory.

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
// Order-preserving 16-bit key of one bf16 value, and back.
__device__ __forceinline__ uint32_t key16(uint32_t b) { return (b & 0x8000u) ? (b ^ 0xffffu) : (b | 0x8000u); }
__device__ __forceinline__ uint32_t unkey16(uint32_t k) { return (k & 0x8000u) ? (k ^ 0x8000u) : (k ^ 0xffffu); }

template <bool VEC>
__global__ void __cluster_dims__(kArgmaxCluster, 1, 1) __launch_bounds__(kArgThreads)
    argmax_kernel(const ArgmaxParams p) {
    // may run as a programmatic dependent of the launch before it (a verify
    // round's merge): nothing is read before that grid has finished
    asm volatile("griddepcontrol.wait;" ::: "memory");
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ uint32_t w_red[kArgWarps];
    __shared__ uint32_t x_max[kArgmaxCluster];  // filled by every CTA of the cluster
    __shared__ int x_idx[kArgmaxCluster];       // filled on rank 0

    // columns per CTA, a multiple of 8 so vectors never straddle two CTAs
    const int per = ((p.n_cols + kArgmaxCluster * 8 - 1) / (kArgmaxCluster * 8)) * 8;
    const int c0 = min(p.n_cols, rank * per), c1 = min(p.n_cols, c0 + per);
    const uint32_t kNegInf2 = 0xff80ff80u, kPad2 = 0xff7fff7fu;
    // A CTA may touch another CTA's shared memory only once every CTA of the
    // cluster is running: arrive here, wait before the first remote store
    // (the loads of pass 1 overlap the wait).
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
    bool joined = false;

    for (int row = blockIdx.y; row < p.n_rows; row += gridDim.y) {
        const uint16_t *rp = p.logits + (int64_t)row * p.ld;
        // ---- pass 1: the largest value and the largest magnitude pattern
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
                // magnitude test alone; pass 2 skips it by its vector index)
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
            // vectors past the ones held (rows wider than 8 x 256 x 8 columns a CTA)
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
        uint32_t k = max(key16(vmax & 0xffffu), key16(vmax >> 16));
        // ---- the cluster's largest value (as a key) and any nonfinite value
        k = __reduce_max_sync(0xffffffffu, k);
        const uint32_t wbad = __reduce_or_sync(0xffffffffu, bad);
        if (lane == 0) w_red[warp] = k | (wbad << 31);
        if (!joined) {
            asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
            joined = true;
        }
        __syncthreads();
        if (tid < kArgmaxCluster) {
            uint32_t m = 0;
#pragma unroll
            for (int i = 0; i < kArgWarps; ++i) m = max(m, w_red[i]);  // the flag bit rides on top
            *cluster.map_shared_rank(&x_max[rank], tid) = m;         // every CTA tells every CTA
        }
        cluster.sync();
        uint32_t K = 0, B = 0;
#pragma unroll
        for (int i = 0; i < kArgmaxCluster; ++i) {
            K = max(K, x_max[i] & 0xffffu);
            B |= x_max[i] >> 31;
        }
        const uint32_t M = unkey16(K);
        const uint32_t M2 = M | (M << 16);
        // ---- pass 2: the first column holding the largest value
        int best = INT_MAX;
        if constexpr (VEC) {
#pragma unroll
            for (int j = 0; j < kArgBatch * 4; ++j) {
                const uint32_t e = eq_bf16x2(words[j], M2);
                const int v = v0 + tid + (j >> 2) * kArgThreads;
                if (best == INT_MAX && e && v < v1) best = v * 8 + (j & 3) * 2 + ((e & 0xffffu) ? 0 : 1);
            }
            for (int v = v0 + tid + kArgBatch * kArgThreads; v < v1 && best == INT_MAX; v += kArgThreads) {
                const uint4 x = __ldg(vp + v);
                const uint32_t wd[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t e = eq_bf16x2(wd[q], M2);
                    if (best == INT_MAX && e) best = v * 8 + 2 * q + ((e & 0xffffu) ? 0 : 1);
                }
            }
        }
        for (int c = (VEC ? (v1 << 3) : c0) + tid; c < c1 && best == INT_MAX; c += kArgThreads)
            if (eq_bf16x2(rp[c], M) & 0xffffu) best = c;
        best = __reduce_min_sync(0xffffffffu, best);
        if (lane == 0) w_red[warp] = (uint32_t)best;
        __syncthreads();
        if (tid == 0) {
            int b = INT_MAX;
#pragma unroll
            for (int i = 0; i < kArgWarps; ++i) b = min(b, (int)w_red[i]);
            *cluster.map_shared_rank(&x_idx[rank], 0) = b;
        }
        cluster.sync();
        if (rank == 0 && tid == 0) {
            int b = INT_MAX;
#pragma unroll
            for (int i = 0; i < kArgmaxCluster; ++i) b = min(b, x_idx[i]);
            p.ids[row] = B ? -1 : b;
            p.flags[row] = (uint8_t)(B ? 1 : 0);
        }
    }
}

cudaError_t launch_argmax(const ArgmaxParams &p, bool vec, cudaStream_t st) {
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
    return vec ? cudaLaunchKernelEx(&cfg, argmax_kernel<true>, p) : cudaLaunchKernelEx(&cfg, argmax_kernel<false>, p);
}

}  // namespace tfp
