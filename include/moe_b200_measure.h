/*
 * moe_b200_measure.h -- measurement aids exported by libmoe_b200.so.
 *
 * No counterpart on the pages: these calls are not steps of the layer.  The
 * benchmark uses them to measure, on the GPU it runs on, the ceilings that the
 * layer's kernels are compared against.
 */
#ifndef MOE_B200_MEASURE_H
#define MOE_B200_MEASURE_H

#include "moe_b200.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Streaming read of `bytes` bytes of device memory at `buf` (16-byte aligned,
 * bytes a multiple of 16), as the weight-streaming GEMMs read their panels:
 * 16-byte non-caching loads, eight in flight per thread, one grid of 4 CTAs of
 * 512 threads per SM, no writes except one word of `sink` (a device uint32,
 * written only if the data xor-folds to all ones, so the loads cannot be
 * elided).  Time it with events on `stream`: bytes / time is the read
 * ceiling of this GPU's HBM, which a read-only kernel is held to (a copy moves
 * the same bytes twice and peaks lower).
 * INVALID_ARG for a null or misaligned pointer or a size not a multiple of 16. */
MOE_API moe_status_t moe_measure_hbm_read(const void* buf, size_t bytes, uint32_t* sink, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_MEASURE_H */
