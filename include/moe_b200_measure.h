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

/* The weight-panel stream of the grouped GEMMs, without the GEMM: one CTA per SM
 * copies panels of `buf` into a ring of shared-memory stages with TMA and
 * discards them, so that the rate the copy engine and the memory system give
 * this access pattern can be measured on its own.
 *
 * buf is viewed as a row-major bf16 matrix [rows, 7168] (the layer's hidden
 * size; rows = bytes / 14336, at least 128) cut into panels of 128 rows.  Each
 * CTA walks panels in 64-column steps: a step copies `boxes` boxes (1..3) of
 * 128 x 64 elements (16 KB each), box b from its own panel (as the up kernels
 * read a gate and an up panel side by side), with the 128-byte swizzle of the
 * MMA operands; with `contiguous` != 0 each box is instead one 16-byte-aligned
 * bulk copy of 16 KB of consecutive bytes of the panel (the panel stored box by
 * box).  `stages` steps (2..16, boxes * stages * 16 KB <= 192 KB) are in flight;
 * `warps` threads per CTA (1..4, each the first lane of its own warp; stages a
 * multiple of warps) take the steps in turn, each waiting for its own oldest
 * step and then issuing its next one into the same slot; `steps` steps per CTA.
 * A buffer of a few tens of MB stays in L2; GBs stream from HBM.
 *
 * *bytes_moved (host, nullable) receives the bytes one call copies (CTAs x
 * steps x boxes x 16 KB); time the call with events on `stream`.  err
 * (device int32, nullable) gets MOE_ERR_TIMEOUT if a copy did not land within
 * the bounded wait (the kernel then waits, bounded, for its other copies and
 * returns).  INVALID_ARG for a null or misaligned buffer, a buffer under one
 * panel, or boxes / stages / warps / steps outside the ranges above. */
MOE_API moe_status_t moe_measure_tma_stream(const void* buf, size_t bytes, int boxes, int stages, int contiguous,
                                            int warps, int steps, int32_t* err, size_t* bytes_moved,
                                            moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_MEASURE_H */
