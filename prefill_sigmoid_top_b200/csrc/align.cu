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
//     into its own row of a [32][E] shared histogram;
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

// Dynamic shared memory budget: the 227 KB per-block limit minus room for the
// kernel's static shared variables.
constexpr size_t kSmemLimit = 227 * 1024 - 1024;

template <int kWarps>
__global__ void __launch_bounds__(kWarps * 32) align_kernel(const int32_t* __restrict__ topk_ids, int n, int E, int B,
                                                         int32_t* __restrict__ sorted_ids,
                                                         int32_t* __restrict__ block_expert,
                                                         int32_t* __restrict__ counts_out,
                                                         int32_t* __restrict__ offsets_out,
                                                         int32_t* __restrict__ ntpp_out, int32_t* err,
                                                         int stage_ids) {
  constexpr int kThreads = kWarps * 32;
  extern __shared__ int smem[];
  int* hist = smem;                  // [kWarps][E]: counts, then write cursors
  int* prefix = hist + kWarps * E;   // [E + 1]
  int* staged = prefix + E + 1;      // [n] when stage_ids (they fit in shared memory)
  __shared__ int warp_sums[kWarps];
  __shared__ int bad;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const unsigned lt_mask = (1u << lane) - 1u;

  for (int i = tid; i < kWarps * E; i += kThreads) hist[i] = 0;
  if (tid == 0) bad = 0;
  // Stage the ids once with all threads (many loads in flight), so the two
  // in-order passes below read shared memory instead of waiting on global loads.
  const bool use_staged = stage_ids != 0;
  if (use_staged)
    for (int i = tid; i < n; i += kThreads) staged[i] = topk_ids[i];
  const int32_t* ids = use_staged ? staged : topk_ids;
  __syncthreads();

  const int seg = (n + kWarps - 1) / kWarps;
  const int f_begin = min(n, warp * seg), f_end = min(n, f_begin + seg);

  // A: per-warp histogram of the segment (shared-memory atomics: only the
  // counts matter here, not the order)
  for (int base = f_begin; base < f_end; base += 32) {
    const int f = base + lane;
    if (f < f_end) {
      const int e = ids[f];
      if (e >= 0 && e < E)
        atomicAdd(&hist[warp * E + e], 1);
      else
        bad = 1;
    }
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
    const int ws = lane < kWarps ? warp_sums[lane] : 0;
    int wincl = ws;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, wincl, off);
      if (lane >= off) wincl += v;
    }
    if (lane < kWarps) warp_sums[lane] = wincl - ws;  // exclusive prefix over warps
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
    const int e = act ? ids[f] : -1;
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


template <int kWarps>
cudaError_t launch_align_variant(const int32_t* topk_ids, int n, int E, int B, int32_t* sorted_ids,
                                 int32_t* block_expert, int32_t* expert_counts, int32_t* expert_offsets,
                                 int32_t* ntpp, int32_t* err, cudaStream_t stream) {
  const size_t base = sizeof(int) * (static_cast<size_t>(kWarps) * E + E + 1);
  const bool stage = base + sizeof(int) * static_cast<size_t>(n) <= kSmemLimit;
  const size_t smem = base + (stage ? sizeof(int) * static_cast<size_t>(n) : 0);
  if (smem > kSmemLimit) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t st = cudaGetDevice(&dev);
  if (st != cudaSuccess) return st;
  static bool attr_set[64] = {};
  if (dev < 64 && !attr_set[dev]) {
    st = cudaFuncSetAttribute(align_kernel<kWarps>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kSmemLimit));
    if (st != cudaSuccess) return st;
    attr_set[dev] = true;
  }
  align_kernel<kWarps><<<1, kWarps * 32, smem, stream>>>(topk_ids, n, E, B, sorted_ids, block_expert, expert_counts,
                                                       expert_offsets, ntpp, err, stage ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace

// One CTA; its thread count must cover the experts (one thread per expert in
// the prefix step).  Few slots: 8 warps, so that the per-expert loops over
// the warps' histogram rows are short; otherwise 32 warps.
cudaError_t launch_align(const int32_t* topk_ids, int M, int K, int E, int B, int32_t* sorted_ids,
                         int32_t* block_expert, int32_t* expert_counts, int32_t* expert_offsets, int32_t* ntpp,
                         int32_t* err, cudaStream_t stream) {
  const int n = M * K;
  if (n <= 4096 && E <= 256)
    return launch_align_variant<8>(topk_ids, n, E, B, sorted_ids, block_expert, expert_counts, expert_offsets, ntpp,
                                   err, stream);
  return launch_align_variant<32>(topk_ids, n, E, B, sorted_ids, block_expert, expert_counts, expert_offsets, ntpp,
                                  err, stream);
}

}  // namespace moe
