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
#include <cstdlib>
#include <cstring>

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


// Many slots: C CTAs, CTA c placing the slots of its own contiguous segment
// [c*seg, (c+1)*seg).  Every CTA reads all the ids (they sit in L2) and counts,
// per expert, all of them and those before its segment, so each one knows the
// padded prefix and where its segment's slots of expert e start inside e's
// rows without exchanging anything with the other CTAs.  Inside the segment
// the placement is the one-CTA kernel's (per-warp counts, then a stable
// in-order scatter), so the plan is the same, bit for bit.  CTA c also writes
// the padding of experts e = c, c + C, ... and the block -> expert entries of
// blocks b = c, c + C, ...
template <int kWarps>
__global__ void __launch_bounds__(kWarps * 32) align_multi_kernel(const int32_t* __restrict__ topk_ids, int n, int E,
                                                               int B, int seg, int32_t* __restrict__ sorted_ids,
                                                               int32_t* __restrict__ block_expert,
                                                               int32_t* __restrict__ counts_out,
                                                               int32_t* __restrict__ offsets_out,
                                                               int32_t* __restrict__ ntpp_out, int32_t* err) {
  constexpr int kThreads = kWarps * 32;
  extern __shared__ int smem[];
  int* all = smem;                   // [E] every slot
  int* before = all + E;             // [E] slots before this CTA's segment
  int* prefix = before + E;          // [E + 1]
  int* hist = prefix + E + 1;        // [kWarps][E]: this segment's counts per warp, then write cursors
  __shared__ int warp_sums[kWarps];
  __shared__ int bad;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const unsigned lt_mask = (1u << lane) - 1u;
  const int c = blockIdx.x, C = gridDim.x;
  const int s_begin = min(n, c * seg), s_end = min(n, s_begin + seg);

  for (int i = tid; i < 2 * E; i += kThreads) smem[i] = 0;
  for (int i = tid; i < kWarps * E; i += kThreads) hist[i] = 0;
  if (tid == 0) bad = 0;
  __syncthreads();

  // counts over all slots and over the slots before the segment
  for (int f = tid; f < n; f += kThreads) {
    const int e = __ldg(topk_ids + f);
    if (e >= 0 && e < E) {
      atomicAdd(&all[e], 1);
      if (f < s_begin) atomicAdd(&before[e], 1);
    } else {
      bad = 1;
    }
  }
  // this segment, split into one contiguous piece per warp
  const int wseg = (s_end - s_begin + kWarps - 1) / kWarps;
  const int f_begin = min(s_end, s_begin + warp * wseg), f_end = min(s_end, f_begin + wseg);
  for (int base = f_begin; base < f_end; base += 32) {
    const int f = base + lane;
    if (f < f_end) {
      const int e = __ldg(topk_ids + f);
      if (e >= 0 && e < E) atomicAdd(&hist[warp * E + e], 1);
    }
  }
  __syncthreads();
  if (bad) {
    if (tid == 0 && c == 0) set_error(err, kErrInvalidInput);
    return;
  }

  // padded exclusive prefix over the experts, one block scan per kThreads experts
  int carry = 0;
  for (int e0 = 0; e0 < E; e0 += kThreads) {
    const int e = e0 + tid;
    const int padded = e < E ? (all[e] + B - 1) / B * B : 0;
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
      if (lane < kWarps) warp_sums[lane] = wincl - ws;
    }
    __syncthreads();
    if (e < E) prefix[e] = carry + warp_sums[warp] + incl - padded;
    __syncthreads();
    const int last = min(E, e0 + kThreads) - 1;
    carry = prefix[last] + (all[last] + B - 1) / B * B;
    __syncthreads();
  }
  if (tid == 0) prefix[E] = carry;
  __syncthreads();  // every prefix[] entry is written before any thread reads it

  const int total = prefix[E];
  for (int e = tid; e < E; e += kThreads) {
    if (c == 0) {
      counts_out[e] = all[e];
      offsets_out[e] = prefix[e];
    }
    int run = prefix[e] + before[e];
    for (int w = 0; w < kWarps; ++w) {
      const int cnt = hist[w * E + e];
      hist[w * E + e] = run;
      run += cnt;
    }
  }
  if (tid == 0 && c == 0) {
    offsets_out[E] = total;
    *ntpp_out = total;
  }
  __syncthreads();

  // stable scatter of this segment
  for (int base = f_begin; base < f_end; base += 32) {
    const int f = base + lane;
    const bool act = f < f_end;
    const int e = act ? __ldg(topk_ids + f) : -1;
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

  // padding of this CTA's experts and block -> expert of its blocks
  for (int e = c + C * warp; e < E; e += C * kWarps)
    for (int pos = prefix[e] + all[e] + lane; pos < prefix[e + 1]; pos += 32) sorted_ids[pos] = n;
  for (int b = c + C * tid; b * B < total; b += C * kThreads) {
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
cudaError_t launch_align_multi(const int32_t* topk_ids, int n, int E, int B, int32_t* sorted_ids,
                               int32_t* block_expert, int32_t* expert_counts, int32_t* expert_offsets, int32_t* ntpp,
                               int32_t* err, cudaStream_t stream) {
  const size_t smem = sizeof(int) * (3 * static_cast<size_t>(E) + 1 + static_cast<size_t>(kWarps) * E);
  if (smem > kSmemLimit) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t st = cudaGetDevice(&dev);
  if (st != cudaSuccess) return st;
  static bool attr_set[64] = {};
  if (dev < 64 && !attr_set[dev]) {
    st = cudaFuncSetAttribute(align_multi_kernel<kWarps>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kSmemLimit));
    if (st != cudaSuccess) return st;
    attr_set[dev] = true;
  }
  const int seg = 512;
  const int ctas = (n + seg - 1) / seg;
  align_multi_kernel<kWarps><<<ctas, kWarps * 32, smem, stream>>>(topk_ids, n, E, B, seg, sorted_ids, block_expert,
                                                                expert_counts, expert_offsets, ntpp, err);
  return cudaGetLastError();
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

// MOE_ALIGN_MULTI=0 keeps the one-CTA kernel for every size (the tests compare both).
bool align_multi_enabled() {
  const char* env = std::getenv("MOE_ALIGN_MULTI");
  return env == nullptr || std::strcmp(env, "0") != 0;
}

}  // namespace

// Up to 4096 slots: one CTA, whose thread count must cover the experts (one
// thread per expert in the prefix step); 8 warps, so that the per-expert loops
// over the warps' histogram rows are short (else 32 warps).  More slots: the
// multi-CTA kernel, one CTA per 512 slots.
cudaError_t launch_align(const int32_t* topk_ids, int M, int K, int E, int B, int32_t* sorted_ids,
                         int32_t* block_expert, int32_t* expert_counts, int32_t* expert_offsets, int32_t* ntpp,
                         int32_t* err, cudaStream_t stream) {
  const int n = M * K;
  if (n > 4096 && align_multi_enabled())  // many slots: one CTA per 512 of them
    return launch_align_multi<16>(topk_ids, n, E, B, sorted_ids, block_expert, expert_counts, expert_offsets, ntpp,
                                  err, stream);
  if (n <= 4096 && E <= 256)
    return launch_align_variant<8>(topk_ids, n, E, B, sorted_ids, block_expert, expert_counts, expert_offsets, ntpp,
                                   err, stream);
  return launch_align_variant<32>(topk_ids, n, E, B, sorted_ids, block_expert, expert_counts, expert_offsets, ntpp,
                                  err, stream);
}

}  // namespace moe
