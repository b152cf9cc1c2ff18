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

#include <cuda_runtime.h>

#include "tf_internal.h"

namespace {

constexpr size_t kScratchBytes = (size_t)TF_RING_NOALLOC_SCRATCH_BYTES;

// The partials of every tf_ring_attn_noalloc call on a device.
__device__ __align__(256) unsigned char g_ring_scratch[kScratchBytes];

}  // namespace

extern "C" {

// In host code `g_ring_scratch` names a host-side stand-in, not device
// memory, so every call asks the runtime for the array's address on the
// current device (cheap once this file's device code is loaded).  Asking on
// every call, instead of caching, keeps the address right across a device
// reset or a different context on the same device.  Under lazy module
// loading (the CUDA 12 default) the first ask is what places the array in
// device memory.  The arguments are then judged by tf_ring_attn itself, with
// the scratch as its workspace: bad arguments get its verdict, and only a
// call whose arguments are sound but whose partials need more than the
// scratch holds gets TF_ERR_WORKSPACE.
tf_status tf_ring_attn_noalloc(const void *q, int32_t n_rows_total, int32_t n_q_heads, const void *ring_k,
                               const void *ring_v, int64_t ring_slots_total, int32_t n_kv_heads, int32_t head_dim,
                               const tf_ring_seg *rsegs, int32_t n_segs, const tf_ring_seg *rsegs_host, float scale,
                               int32_t split_slots, int32_t n_splits_max, float *out, uint8_t *flags,
                               uint32_t *status, tf_stream_t stream) {
    void *ws = nullptr;
    if (cudaGetSymbolAddress(&ws, g_ring_scratch) != cudaSuccess || ws == nullptr) return TF_ERR_CUDA;
    return tf_ring_attn(q, n_rows_total, n_q_heads, ring_k, ring_v, ring_slots_total, n_kv_heads, head_dim, rsegs,
                        n_segs, rsegs_host, scale, split_slots, n_splits_max, ws, kScratchBytes, out, flags, status,
                        stream);
}

}  // extern "C"
