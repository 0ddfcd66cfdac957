// Expert-major block plan ("[flashinfer] ... AlphaMoE NVFP4 커널 최적화",
// flashinfer PR #6511 analysis, §5 "moe_align_block_size_kernel 동기화 개선").
//
// The page describes a per-expert histogram, a prefix scan copied into a
// shared prefix[] array, and a binary search over prefix[] that gives each
// padded block its expert; the bug it fixes is a missing barrier between the
// prefix[] write and the searches.  This kernel keeps that structure on one
// CTA of 1024 threads and makes the slot order inside each expert stable
// (ascending slot id), so the plan is a deterministic function of topk_ids:
//
//  A. each warp owns one contiguous segment of the M*K slots and counts it
//     into its own row of a [32][E] shared histogram (warp match_any gives
//     the lanes holding the same expert; the group leader adds the group
//     size, so no atomics are needed);
//  B. thread e sums its column -> expert_counts[e]; a block-wide exclusive
//     scan of the padded counts -> prefix[]; barrier (the page's fix); then
//     each column is turned into per-warp write cursors;
//  C. each warp walks its segment again in order and scatters slot f to
//     cursor + (rank among equal experts in the 32-slot group);
//  D. padding rows get the sentinel M*K; block b gets the expert found by a
//     binary search for the last prefix[e] <= b*B.
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

__global__ void __launch_bounds__(kThreads) align_kernel(const int32_t* __restrict__ topk_ids, int n, int E, int B,
                                                         int32_t* __restrict__ sorted_ids,
                                                         int32_t* __restrict__ block_expert,
                                                         int32_t* __restrict__ counts_out,
                                                         int32_t* __restrict__ offsets_out,
                                                         int32_t* __restrict__ ntpp_out, int32_t* err) {
  extern __shared__ int smem[];
  int* hist = smem;                  // [kWarps][E]: counts, then write cursors
  int* prefix = hist + kWarps * E;   // [E + 1]
  __shared__ int warp_sums[kWarps];
  __shared__ int bad;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const unsigned lt_mask = (1u << lane) - 1u;

  for (int i = tid; i < kWarps * E; i += kThreads) hist[i] = 0;
  if (tid == 0) bad = 0;
  __syncthreads();

  const int seg = (n + kWarps - 1) / kWarps;
  const int f_begin = min(n, warp * seg), f_end = min(n, f_begin + seg);

  // A: per-warp histogram of the segment
  for (int base = f_begin; base < f_end; base += 32) {
    const int f = base + lane;
    const bool act = f < f_end;
    const int e = act ? topk_ids[f] : -1;
    const bool ok = act && e >= 0 && e < E;
    if (act && !ok) bad = 1;
    const unsigned okmask = __ballot_sync(0xffffffffu, ok);
    const unsigned peers = __match_any_sync(0xffffffffu, ok ? e : -1) & okmask;
    if (ok && (__ffs(peers) - 1) == lane) hist[warp * E + e] += __popc(peers);
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) set_error(err, kErrInvalidInput);
    return;
  }

  // B: counts, padded exclusive prefix, per-warp cursors
  int count = 0;
  if (tid < E)
    for (int w = 0; w < kWarps; ++w) count += hist[w * E + tid];
  const int padded = (tid < E) ? (count + B - 1) / B * B : 0;
  int incl = padded;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int ws = warp_sums[lane];
    int wincl = ws;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, wincl, off);
      if (lane >= off) wincl += v;
    }
    warp_sums[lane] = wincl - ws;  // exclusive prefix over warps
  }
  __syncthreads();
  const int excl = warp_sums[warp] + incl - padded;
  if (tid < E) prefix[tid] = excl;
  if (tid == E - 1) prefix[E] = excl + padded;
  __syncthreads();  // every prefix[] entry is written before any thread reads it

  const int total = prefix[E];
  if (tid < E) {
    counts_out[tid] = count;
    offsets_out[tid] = prefix[tid];
    int run = prefix[tid];
    for (int w = 0; w < kWarps; ++w) {
      const int c = hist[w * E + tid];
      hist[w * E + tid] = run;
      run += c;
    }
  }
  if (tid == 0) {
    offsets_out[E] = total;
    *ntpp_out = total;
  }
  __syncthreads();

  // C: stable scatter
  for (int base = f_begin; base < f_end; base += 32) {
    const int f = base + lane;
    const bool act = f < f_end;
    const int e = act ? topk_ids[f] : -1;
    const unsigned actmask = __ballot_sync(0xffffffffu, act);
    const unsigned peers = __match_any_sync(0xffffffffu, e) & actmask;
    int pos = 0;
    if (act) pos = hist[warp * E + e] + __popc(peers & lt_mask);
    __syncwarp();
    if (act) {
      sorted_ids[pos] = f;
      if ((__ffs(peers) - 1) == lane) hist[warp * E + e] += __popc(peers);
    }
    __syncwarp();
  }
  __syncthreads();

  // D: padding and block -> expert
  for (int e = warp; e < E; e += kWarps) {
    const int start = hist[(kWarps - 1) * E + e];  // = prefix[e] + count[e]
    for (int pos = start + lane; pos < prefix[e + 1]; pos += 32) sorted_ids[pos] = n;
  }
  for (int b = tid; b * B < total; b += kThreads) {
    const int row = b * B;
    int lo = 0, hi = E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (prefix[mid] <= row) lo = mid; else hi = mid - 1;
    }
    block_expert[b] = lo;
  }
}

}  // namespace

cudaError_t launch_align(const int32_t* topk_ids, int M, int K, int E, int B, int32_t* sorted_ids,
                         int32_t* block_expert, int32_t* expert_counts, int32_t* expert_offsets, int32_t* ntpp,
                         int32_t* err, cudaStream_t stream) {
  const size_t smem = sizeof(int) * (static_cast<size_t>(kWarps) * E + E + 1);
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t st = cudaFuncSetAttribute(align_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          static_cast<int>(sizeof(int) * (kWarps * 1024 + 1025)));
    if (st != cudaSuccess) return st;
    attr_set = true;
  }
  align_kernel<<<1, kThreads, smem, stream>>>(topk_ids, M * K, E, B, sorted_ids, block_expert, expert_counts,
                                             expert_offsets, ntpp, err);
  return cudaGetLastError();
}

}  // namespace moe
