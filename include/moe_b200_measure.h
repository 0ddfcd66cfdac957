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

/* The copy mix of one stage of the NVFP4 GEMMs, without the GEMM: one CTA per
 * SM, two issuing warps, copies into a ring of `stages` (2..4) shared-memory
 * slots that are discarded, so that the rate of a stage's copies can be
 * measured against their mix.
 *
 * buf (16-byte aligned, at least 256 MB) is split in two.  Its first 7/8 is a
 * byte matrix [rows, 3584] (e2m1 codes of weight rows of 7168 elements) cut
 * into panels of 128 rows; its first 8192 rows (28 MB, which stay in L2) also
 * serve as token rows.  Its last 1/8 holds 2 KB scale chunks.  A step is one
 * k-step of 256 elements: the first warp copies two code boxes of 128 rows x
 * 128 bytes (32 KB, 128-byte swizzle) from two panels; what else a step holds
 * is `mix`:
 *   0  nothing (the code boxes alone);
 *   1  a box of 64 token rows x 128 bytes (8 KB), copied by the second warp;
 *   2  the token box and three 2 KB scale chunks, all four copied by the
 *      second warp (the copies of a stage of the NVFP4 kernels);
 *   3  the same bytes, one scale chunk copied by the first warp;
 *   4  the token box, and on every fourth step three 8 KB chunks (the scales
 *      of four k-steps in one copy each), copied by the second warp.
 * `steps` (>= 8) steps per CTA.  *bytes_moved (host, nullable) receives the
 * bytes one call copies; time the call with events on `stream`.  err (device
 * int32, nullable) gets MOE_ERR_TIMEOUT if a copy did not land within the
 * bounded wait.  INVALID_ARG for a null or misaligned buffer, a buffer under
 * 256 MB, or mix / stages / steps outside the ranges above. */
MOE_API moe_status_t moe_measure_tma_mix(const void* buf, size_t bytes, int mix, int stages, int steps, int32_t* err,
                                         size_t* bytes_moved, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_MEASURE_H */
