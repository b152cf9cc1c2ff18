// ring_noalloc.cu - tf_ring_attn for callers that cannot allocate device memory.
//
// tf_ring_attn needs a caller-provided workspace for the partials that pass
// between its two kernels.  Some callers have no way to provide one: a serving
// engine that hands all device memory to its KV pool at start-up and keeps no
// allocator on the decode path, or a host framework that calls this library
// from a plugin hook where cudaMalloc (and the device-wide synchronization it
// can imply) is not allowed.  tf_ring_attn_noalloc serves them with a scratch
// array that is part of this library's own device image: a file-scope
// __device__ array, sized once at compile time, that every GPU which loads the
// library holds until the process exits.
//
// The kernels and their arithmetic are exactly tf_ring_attn's; only where the
// partials live differs.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "tf_internal.h"

namespace {

constexpr size_t kScratchBytes = (size_t)TF_RING_NOALLOC_SCRATCH_BYTES;

// The partials of every tf_ring_attn_noalloc call on a device.
__device__ __align__(256) unsigned char g_ring_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices];  // device address of g_ring_scratch, per device, once resolved

// The device address of the scratch array on the current device.  In host
// code `g_ring_scratch` names a host-side stand-in, not device memory, so the
// address is asked from the runtime once per device and cached.
cudaError_t scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_ring_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" {

tf_status tf_ring_attn_noalloc(const void *q, int32_t n_rows_total, int32_t n_q_heads, const void *ring_k,
                               const void *ring_v, int64_t ring_slots_total, int32_t n_kv_heads, int32_t head_dim,
                               const tf_ring_seg *rsegs, int32_t n_segs, const tf_ring_seg *rsegs_host, float scale,
                               int32_t split_slots, int32_t n_splits_max, float *out, uint8_t *flags,
                               uint32_t *status, tf_stream_t stream) {
    const size_t need = tf_ring_workspace_bytes(n_segs, n_q_heads, head_dim, n_splits_max);
    if (need > kScratchBytes) return TF_ERR_WORKSPACE;
    if (n_segs <= 0) {
        // let tf_ring_attn give its verdict on the other arguments without a workspace
        return tf_ring_attn(q, n_rows_total, n_q_heads, ring_k, ring_v, ring_slots_total, n_kv_heads, head_dim, rsegs,
                            n_segs, rsegs_host, scale, split_slots, n_splits_max, nullptr, 0, out, flags, status,
                            stream);
    }
    void *ws = nullptr;
    if (scratch_address(&ws) != cudaSuccess) return TF_ERR_CUDA;
    return tf_ring_attn(q, n_rows_total, n_q_heads, ring_k, ring_v, ring_slots_total, n_kv_heads, head_dim, rsegs,
                        n_segs, rsegs_host, scale, split_slots, n_splits_max, ws, kScratchBytes, out, flags, status,
                        stream);
}

}  // extern "C"
