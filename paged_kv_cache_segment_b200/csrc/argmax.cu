// argmax.cu - greedy row argmax over bf16 logit rows.
//
// Rule (TensorFold #1503 "lfm2_moe CUDA: attention pages from the shared KV
// pool, and the prompt cache", commit list, lfm2_argmax): each row's first
// largest logit, ties to the lower id, a row holding a nonfinite logit
// flagged.  Readings: values compare as real numbers (-0 == +0), a flagged
// row reports id -1.
//
// Each row is split over a cluster of 8 CTAs.  Every CTA streams its share of
// the row with 16-byte loads, keeps per thread the first column holding its
// largest value, reduces over its warps, and the cluster's rank-0 CTA folds
// the 8 CTA results through distributed shared memory.  No workspace and no
// inter-CTA counters: the cluster barrier orders the exchange.
//
// Comparing bf16 values as reals uses an order-preserving 16-bit key: for a
// non-negative value the bits with the sign bit set, for a negative value all
// bits inverted, and -0 mapped to +0 first.
#include <cooperative_groups.h>

#include <climits>
#include <cstdint>

#include "tf_common.cuh"
#include "tf_internal.h"

namespace cg = cooperative_groups;

namespace tfp {

constexpr int kArgThreads = 256;
constexpr int kArgBatch = 8;  // 16-byte vectors in flight per thread

__device__ __forceinline__ uint32_t order_key(uint32_t b) {
    b = (b == 0x8000u) ? 0u : b;
    return (b & 0x8000u) ? (b ^ 0xffffu) : (b | 0x8000u);
}

__device__ __forceinline__ void take(uint32_t b, int col, uint32_t &best, int &best_col, uint32_t &bad) {
    bad |= ((b & 0x7f80u) == 0x7f80u);
    const uint32_t k = order_key(b);
    if (k > best) {
        best = k;
        best_col = col;
    }
}

// (key, col) pairs: the larger key wins, then the lower column.
__device__ __forceinline__ void better_of(uint32_t &k, int &c, uint32_t k2, int c2) {
    if (k2 > k || (k2 == k && c2 < c)) {
        k = k2;
        c = c2;
    }
}

template <bool VEC>
__global__ void __cluster_dims__(kArgmaxCluster, 1, 1) __launch_bounds__(kArgThreads) argmax_kernel(const ArgmaxParams p) {
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ uint32_t w_key[kArgThreads / 32], w_bad[kArgThreads / 32];
    __shared__ int w_col[kArgThreads / 32];
    __shared__ uint32_t c_key, c_bad;
    __shared__ int c_col;

    // columns per CTA, a multiple of 8 so vectors never straddle two CTAs
    const int per = ((p.n_cols + kArgmaxCluster * 8 - 1) / (kArgmaxCluster * 8)) * 8;
    const int c0 = min(p.n_cols, rank * per), c1 = min(p.n_cols, c0 + per);

    for (int row = blockIdx.y; row < p.n_rows; row += gridDim.y) {
        const uint16_t *rp = p.logits + (int64_t)row * p.ld;
        uint32_t best = 0u, bad = 0u;
        int best_col = INT_MAX;
        if constexpr (VEC) {
            const uint4 *vp = reinterpret_cast<const uint4 *>(rp);
            const int v0 = c0 >> 3, v1 = c1 >> 3;  // whole vectors [v0, v1)
            for (int vb = v0 + tid; vb < v1; vb += kArgThreads * kArgBatch) {
                uint4 buf[kArgBatch];
#pragma unroll
                for (int k = 0; k < kArgBatch; ++k) {
                    const int v = vb + k * kArgThreads;
                    buf[k] = v < v1 ? __ldg(vp + v) : make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u);
                }
#pragma unroll
                for (int k = 0; k < kArgBatch; ++k) {
                    const int v = vb + k * kArgThreads;
                    if (v < v1) {
                        const uint32_t wd[4] = {buf[k].x, buf[k].y, buf[k].z, buf[k].w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            take(wd[e] & 0xffffu, v * 8 + 2 * e, best, best_col, bad);
                            take(wd[e] >> 16, v * 8 + 2 * e + 1, best, best_col, bad);
                        }
                    }
                }
            }
            // ragged tail of the row (last CTA only)
            for (int c = (v1 << 3) + tid; c < c1; c += kArgThreads) take(rp[c], c, best, best_col, bad);
        } else {
            for (int c = c0 + tid; c < c1; c += kArgThreads) take(rp[c], c, best, best_col, bad);
        }
        // warp, then CTA
#pragma unroll
        for (int x = 16; x; x >>= 1) {
            const uint32_t k2 = __shfl_xor_sync(0xffffffffu, best, x);
            const int c2 = __shfl_xor_sync(0xffffffffu, best_col, x);
            better_of(best, best_col, k2, c2);
            bad |= __shfl_xor_sync(0xffffffffu, bad, x);
        }
        if (lane == 0) {
            w_key[warp] = best;
            w_col[warp] = best_col;
            w_bad[warp] = bad;
        }
        __syncthreads();
        if (tid == 0) {
            uint32_t k = w_key[0], b = w_bad[0];
            int c = w_col[0];
            for (int i = 1; i < kArgThreads / 32; ++i) {
                better_of(k, c, w_key[i], w_col[i]);
                b |= w_bad[i];
            }
            c_key = k;
            c_col = c;
            c_bad = b;
        }
        cluster.sync();
        if (rank == 0 && tid == 0) {
            uint32_t k = c_key, b = c_bad;
            int c = c_col;
            for (int r = 1; r < kArgmaxCluster; ++r) {
                const uint32_t *rk = cluster.map_shared_rank(&c_key, r);
                const int *rc = cluster.map_shared_rank(&c_col, r);
                const uint32_t *rb = cluster.map_shared_rank(&c_bad, r);
                better_of(k, c, *rk, *rc);
                b |= *rb;
            }
            p.ids[row] = b ? -1 : c;
            p.flags[row] = (uint8_t)(b ? 1 : 0);
        }
        cluster.sync();  // rank 0 has read every CTA's result before anyone reuses it
    }
}

cudaError_t launch_argmax(const ArgmaxParams &p, bool vec, cudaStream_t st) {
    if (p.n_rows == 0) return cudaSuccess;
    const dim3 grid(kArgmaxCluster, (unsigned)(p.n_rows < 65535 ? p.n_rows : 65535));
    if (vec)
        argmax_kernel<true><<<grid, kArgThreads, 0, st>>>(p);
    else
        argmax_kernel<false><<<grid, kArgThreads, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace tfp
