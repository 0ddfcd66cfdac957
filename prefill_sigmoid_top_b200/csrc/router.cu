// Sigmoid top-k router ("[sglang] [NPU] GLM-4.7-Flash 성능 최적화", sglang
// PR #29509 analysis, §2 "MoE TopK Scoring Function": scores are sigmoid,
// norm_type=1, rather than softmax).
//
// Two launches:
//  1. router_logits_staged_kernel: z[t,e] = x[t] . w_router[e] + bias[e] in
//     fp32, in the canonical order that makes the selection reproducible bit
//     for bit: partial l (l = 0..31) accumulates, one fma per element and in
//     increasing h, the elements h = 256*j + 8*l + i (i = 0..7, j = 0..H/256-1);
//     the 32 partials are then combined with an xor butterfly (offsets 16, 8,
//     4, 2, 1), which adds partial l and l+16 first, then the results 8
//     apart, and so on; the bias is added last.  Lane l of a warp owns
//     partial l of each of the warp's (token, expert) pairs; x and w_router
//     arrive through a shared-memory ring of 256-element slabs (cp.async).
//     Few tokens: 8 tokens x 1 expert per warp, 16 slabs in flight.  Many
//     tokens: 8 tokens x 8 experts per warp, 4 x 2 warps.  Every fma takes its bf16
//     operands directly (fma.rn.f32.bf16: exact product, one rounding), so no
//     bf16 -> fp32 conversion is issued.
//  2. router_topk_kernel: one warp per token selects the K largest logits
//     (descending; equal logits -> lower expert id) by K rounds of a warp
//     argmax, then w_k = s_k / sum s with s = 1 / (1 + exp(-z)).
//  2'. router_topk_ext_kernel: the routing variants of the same page (its
//     norm_type: 0 = softmax, 1 = sigmoid scores), optional renormalisation,
//     a routed scale, and a bias that only shifts the selection key.  The
//     selection is the same warp argmax on the key; the score of a selected
//     expert is taken from the logit without the selection-only bias.
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "router_dot.cuh"
#include "router_select.cuh"

namespace moe {
namespace {

// ---------------------------------------------------------------------------
// Logits.  x and w_router reach the warps through a ring of kStages slabs of
// 256 hidden elements (512 bytes per row), copied with 16-byte cp.async by
// all threads, so that kStages - 1 slabs of loads are in flight while one is
// being used.  Warp (wt, we) of the CTA owns kTt tokens x kTe experts; lane l
// of every warp keeps partial l of each of its pairs, i.e. the elements
// h = 256 j + 8 l + i, taken with one fma each in increasing h, and the 32
// partials are combined with the xor butterfly.  The result is the canonical
// value for any tile shape.
__device__ __forceinline__ void cp_async_16(void* smem_dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(smem_dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int kPending>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(kPending) : "memory");
}

template <int kTt, int kTe, int kWt, int kWe, int kStages>
struct StagedCfg {
  static constexpr int kThreads = kWt * kWe * 32;
  static constexpr int kRowsX = kWt * kTt;  // tokens per CTA
  static constexpr int kRowsW = kWe * kTe;  // experts per CTA
  static constexpr int kRows = kRowsX + kRowsW;
  static constexpr int kStageBytes = kRows * 512;
  static constexpr int kSmem = kStages * kStageBytes;
  static constexpr int kCopyIters = (kRows * 32 + kThreads - 1) / kThreads;
  static_assert(kTt * kTe <= 64, "pairs per warp");
};

template <int kTt, int kTe, int kWt, int kWe, int kStages>
__global__ void __launch_bounds__(kWt * kWe * 32) router_logits_staged_kernel(const uint16_t* __restrict__ x,
                                                                             const uint16_t* __restrict__ w_router,
                                                                             const float* __restrict__ bias, int M,
                                                                             int H, int E,
                                                                             float* __restrict__ logits) {
  using C = StagedCfg<kTt, kTe, kWt, kWe, kStages>;
  extern __shared__ __align__(128) uint8_t slabs[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wt = warp / kWe, we = warp % kWe;
  const int t_base = blockIdx.x * C::kRowsX, e_base = blockIdx.y * C::kRowsW;
  const int nj = H / 256;

  auto issue = [&](int j) {
    uint8_t* st = slabs + (j % kStages) * C::kStageBytes;
#pragma unroll
    for (int it = 0; it < C::kCopyIters; ++it) {
      const int idx = threadIdx.x + it * C::kThreads;
      if (idx >= C::kRows * 32) break;
      const int r = idx >> 5, c = idx & 31;
      const uint16_t* row;
      bool valid;
      if (r < C::kRowsX) {
        valid = t_base + r < M;
        row = x + static_cast<size_t>(valid ? t_base + r : 0) * H;
      } else {
        valid = e_base + r - C::kRowsX < E;
        row = w_router + static_cast<size_t>(valid ? e_base + r - C::kRowsX : 0) * H;
      }
      cp_async_16(st + r * 512 + c * 16, row + 256 * j + 8 * c, valid ? 16 : 0);  // 0 bytes -> zero fill
    }
  };

  float acc[kTt][kTe];
#pragma unroll
  for (int t = 0; t < kTt; ++t)
#pragma unroll
    for (int q = 0; q < kTe; ++q) acc[t][q] = 0.0f;

#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < nj) issue(s);
    cp_async_commit();
  }
#pragma unroll 1
  for (int j = 0; j < nj; ++j) {
    if (j + kStages - 1 < nj) issue(j + kStages - 1);  // into the stage released at the end of j - 1
    cp_async_commit();
    cp_async_wait<kStages - 1>();  // this thread's copies of slab j have landed
    __syncthreads();               // and everyone else's
    const uint8_t* st = slabs + (j % kStages) * C::kStageBytes;
    uint4 xv[kTt], wv[kTe];
#pragma unroll
    for (int t = 0; t < kTt; ++t) xv[t] = *reinterpret_cast<const uint4*>(st + (wt * kTt + t) * 512 + lane * 16);
#pragma unroll
    for (int q = 0; q < kTe; ++q)
      wv[q] = *reinterpret_cast<const uint4*>(st + (C::kRowsX + we * kTe + q) * 512 + lane * 16);
#pragma unroll
    for (int i = 0; i < 8; ++i)  // increasing h inside the chunk
#pragma unroll
      for (int t = 0; t < kTt; ++t)
#pragma unroll
        for (int q = 0; q < kTe; ++q)
          acc[t][q] = (i & 1) ? fma_bf16<true>(word(xv[t], i >> 1), word(wv[q], i >> 1), acc[t][q])
                              : fma_bf16<false>(word(xv[t], i >> 1), word(wv[q], i >> 1), acc[t][q]);
    __syncthreads();  // the stage may be refilled
  }
#pragma unroll
  for (int t = 0; t < kTt; ++t)
#pragma unroll
    for (int q = 0; q < kTe; ++q) {
      float v = acc[t][q];
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, off));
      const int tok = t_base + wt * kTt + t, e = e_base + we * kTe + q;
      if (lane == ((t * kTe + q) & 31) && tok < M && e < E) {
        const float b = bias != nullptr ? bias[e] : 0.0f;
        logits[static_cast<size_t>(tok) * E + e] = __fadd_rn(v, b);
      }
    }
}

template <int kTt, int kTe, int kWt, int kWe, int kStages>
cudaError_t launch_staged(const uint16_t* x, const uint16_t* w_router, const float* bias, int M, int H, int E,
                          float* logits, cudaStream_t stream) {
  using C = StagedCfg<kTt, kTe, kWt, kWe, kStages>;
  auto kern = router_logits_staged_kernel<kTt, kTe, kWt, kWe, kStages>;
  int dev = 0;
  cudaError_t st = cudaGetDevice(&dev);
  if (st != cudaSuccess) return st;
  static bool attr_set[64] = {};
  if (C::kSmem > 48 * 1024 && dev < 64 && !attr_set[dev]) {
    st = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (st != cudaSuccess) return st;
    attr_set[dev] = true;
  }
  dim3 grid((M + C::kRowsX - 1) / C::kRowsX, (E + C::kRowsW - 1) / C::kRowsW);
  kern<<<grid, C::kThreads, C::kSmem, stream>>>(x, w_router, bias, M, H, E, logits);
  return cudaGetLastError();
}

template <int kPerLane>
__global__ void __launch_bounds__(128) router_topk_kernel(const float* __restrict__ logits, int M, int E, int K,
                                                          int32_t* __restrict__ topk_ids,
                                                          float* __restrict__ topk_w) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (t >= M) return;
  const float* zt = logits + static_cast<size_t>(t) * E;
  topk_sigmoid_token<kPerLane>([&](int e) { return zt[e]; }, E, K, lane, topk_ids + static_cast<size_t>(t) * K,
                               topk_w + static_cast<size_t>(t) * K);
}

template <int kPerLane>
__global__ void __launch_bounds__(128) router_topk_ext_kernel(const float* __restrict__ logits,
                                                              const float* __restrict__ sel_bias, int M, int E,
                                                              int K, int scoring, int renormalize, float scale,
                                                              int32_t* __restrict__ topk_ids,
                                                              float* __restrict__ topk_w) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (t >= M) return;
  const float* zt = logits + static_cast<size_t>(t) * E;
  float z[kPerLane], v[kPerLane];
  bool live[kPerLane];
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    const int e = lane + 32 * i;
    live[i] = e < E;
    z[i] = live[i] ? selection_key(zt[e]) : -INFINITY;
    v[i] = (live[i] && sel_bias != nullptr) ? selection_key(__fadd_rn(z[i], sel_bias[e])) : z[i];
  }
  // softmax over all E experts: max, then the sum of exp(z - max)
  float zmax = -INFINITY, denom = 0.0f;
  if (scoring == MOE_SCORE_SOFTMAX) {
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) zmax = fmaxf(zmax, z[i]);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) zmax = fmaxf(zmax, __shfl_xor_sync(0xffffffffu, zmax, off));
#pragma unroll
    for (int i = 0; i < kPerLane; ++i)
      if (live[i]) denom += expf(z[i] - zmax);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) denom += __shfl_xor_sync(0xffffffffu, denom, off);
  }
  int sel_id = 0;
  for (int k = 0; k < K; ++k) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i)
      if (live[i] && better(v[i], lane + 32 * i, bv, bi)) {
        bv = v[i];
        bi = lane + 32 * i;
      }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (better(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
    }
#pragma unroll
    for (int i = 0; i < kPerLane; ++i)
      if (lane + 32 * i == bi) live[i] = false;
    if (lane == k) sel_id = bi;
  }
  float p = 0.0f;
  if (lane < K) {
    const float zs = selection_key(zt[sel_id]);
    if (scoring == MOE_SCORE_SOFTMAX)  // the common 1/denom cancels when renormalising
      p = renormalize ? expf(zs - zmax) : expf(zs - zmax) / denom;
    else
      p = 1.0f / (1.0f + expf(-zs));
  }
  float total = p;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) total += __shfl_xor_sync(0xffffffffu, total, off);
  if (lane < K) {
    topk_ids[static_cast<size_t>(t) * K + lane] = sel_id;
    topk_w[static_cast<size_t>(t) * K + lane] = (renormalize ? p / total : p) * scale;
  }
}

}  // namespace

cudaError_t launch_router_logits(const uint16_t* x, const uint16_t* w_router, const float* bias, int M, int H, int E,
                                 float* logits, cudaStream_t stream) {
  if (M <= 64)  // few tokens: one expert per warp, so that many warps share the reads of w_router; deep ring
    return launch_staged<8, 1, 1, 4, 16>(x, w_router, bias, M, H, E, logits, stream);
  // Many tokens: 8 tokens x 8 experts per warp, 4 x 2 warps per CTA (32 tokens x 16 experts), so that
  // each slab row brought into shared memory serves more pairs than with 2 x 2 warps (the rows are
  // re-read from L2 E/16 and M/32 times instead of E/16 and M/16).  Measured on a B200, moe_route at
  // M = 2048 / 1000 / 512 tokens: 247 / 146 / 82 us against 269 / 160 / 108 us with 2 x 2 warps.
  // MOE_ROUTER_TILE=0 keeps the 2 x 2 shape (the tests compare both).
  const char* env = std::getenv("MOE_ROUTER_TILE");
  if (env != nullptr && std::strcmp(env, "0") == 0)
    return launch_staged<8, 8, 2, 2, 4>(x, w_router, bias, M, H, E, logits, stream);
  return launch_staged<8, 8, 4, 2, 4>(x, w_router, bias, M, H, E, logits, stream);
}

cudaError_t launch_router_topk(const float* logits, int M, int E, int K, int32_t* topk_ids, float* topk_w,
                               cudaStream_t stream) {
  dim3 grid((M + 3) / 4);
  if (E <= 64)
    router_topk_kernel<2><<<grid, 128, 0, stream>>>(logits, M, E, K, topk_ids, topk_w);
  else if (E <= 256)
    router_topk_kernel<8><<<grid, 128, 0, stream>>>(logits, M, E, K, topk_ids, topk_w);
  else
    router_topk_kernel<32><<<grid, 128, 0, stream>>>(logits, M, E, K, topk_ids, topk_w);
  return cudaGetLastError();
}

cudaError_t launch_router_topk_ext(const float* logits, const float* sel_bias, int M, int E, int K, int scoring,
                                   int renormalize, float scale, int32_t* topk_ids, float* topk_w,
                                   cudaStream_t stream) {
  dim3 grid((M + 3) / 4);
  if (E <= 64)
    router_topk_ext_kernel<2><<<grid, 128, 0, stream>>>(logits, sel_bias, M, E, K, scoring, renormalize, scale,
                                                        topk_ids, topk_w);
  else if (E <= 256)
    router_topk_ext_kernel<8><<<grid, 128, 0, stream>>>(logits, sel_bias, M, E, K, scoring, renormalize, scale,
                                                        topk_ids, topk_w);
  else
    router_topk_ext_kernel<32><<<grid, 128, 0, stream>>>(logits, sel_bias, M, E, K, scoring, renormalize, scale,
                                                         topk_ids, topk_w);
  return cudaGetLastError();
}

}  // namespace moe

// ---------------------------------------------------------------------------
// moe_route_noalloc: moe_route for callers that cannot allocate device memory.
// The [M,E] logits live in this fixed array instead of a caller workspace.
// Device code could name the array directly; host code only has a host-side
// stand-in for it, so every call looks up the array's device address on the
// current device and passes it to the kernels as a plain pointer.  The lookup
// allocates nothing and is not cached: an address kept from an earlier call
// would dangle after a device reset or a new primary context.
namespace {

static __device__ __align__(256) float g_route_logits_scratch[MOE_ROUTE_NOALLOC_MAX_LOGITS];

// Device address of the array on the current device.
cudaError_t route_scratch_address(float** out) {
  void* ptr = nullptr;
  const cudaError_t st = cudaGetSymbolAddress(&ptr, g_route_logits_scratch);
  if (st != cudaSuccess) return st;
  *out = static_cast<float*>(ptr);
  return cudaSuccess;
}

}  // namespace

extern "C" moe_status_t moe_route_noalloc(const moe_bf16_t* x, const moe_bf16_t* w_router, const float* bias,
                                          moe_shape_t s, int32_t* topk_ids, float* topk_w, moe_stream_t stream) {
  const int v = moe::check_route_args(s, x, w_router, topk_ids, topk_w);
  if (v != MOE_OK) return static_cast<moe_status_t>(v);
  if (static_cast<long long>(s.M) * s.E > MOE_ROUTE_NOALLOC_MAX_LOGITS) return MOE_ERR_UNSUPPORTED;
  float* logits = nullptr;
  if (route_scratch_address(&logits) != cudaSuccess) return MOE_ERR_CUDA;
  auto cs = static_cast<cudaStream_t>(stream);
  if (moe::launch_router_logits(x, w_router, bias, s.M, s.H, s.E, logits, cs) != cudaSuccess) return MOE_ERR_CUDA;
  if (moe::launch_router_topk(logits, s.M, s.E, s.top_k, topk_ids, topk_w, cs) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}
