// tma_host.h - building TMA tensor maps on the host without linking libcuda:
// the driver's encoder is fetched once through the runtime's entry-point query.
#pragma once

#include <cuda.h>

namespace tfp {

// A tiled bf16 tensor map with 128-byte swizzle, L2 promotion of 256 bytes and
// zero fill out of bounds.  dims[0] is the contiguous dimension; strides are
// the byte strides of dims[1..rank-1].  Returns false if the encoder is
// unavailable or rejects the arguments.
bool make_tensor_map_bf16(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims,
                          const cuuint64_t *strides, const cuuint32_t *box);

}  // namespace tfp
