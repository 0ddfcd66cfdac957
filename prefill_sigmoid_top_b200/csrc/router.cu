// Sigmoid top-k router ("[sglang] [NPU] GLM-4.7-Flash 성능 최적화", sglang
// PR #29509 analysis, §2 "MoE TopK Scoring Function": scores are sigmoid,
// norm_type=1, rather than softmax).
//
// Two launches:
//  1. router_logits_kernel: z[t,e] = x[t] . w_router[e] + bias[e] in fp32, in
//     the canonical order that makes the selection reproducible bit for bit:
//     lane l of a warp accumulates, one fma per element and in increasing h,
//     the elements h = 256*j + 8*l + i (i = 0..7, j = 0..H/256-1), i.e. the
//     16-byte chunk the lane loads in a coalesced 512-byte warp load; the 32
//     lane partials are then combined with an xor butterfly (offsets 16, 8, 4,
//     2, 1), which adds partial l and l+16 first, then the results 8 apart,
//     and so on; the bias is added last.
//     Register tiling: each lane carries 8 tokens x 4 experts partials (1
//     expert for small batches), so a chunk of x and of w_router is loaded
//     once per 32 fmas; the next chunk is loaded while this one is used.
//  2. router_topk_kernel: one warp per token selects the K largest logits
//     (descending; equal logits -> lower expert id) by K rounds of a warp
//     argmax, then w_k = s_k / sum s with s = 1 / (1 + exp(-z)).
//  2'. router_topk_ext_kernel: the routing variants of the same page (its
//     norm_type: 0 = softmax, 1 = sigmoid scores), optional renormalisation,
//     a routed scale, and a bias that only shifts the selection key.  The
//     selection is the same warp argmax on the key; the score of a selected
//     expert is taken from the logit without the selection-only bias.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kTokPerWarp = 8;
constexpr int kWarps = 4;

__device__ __forceinline__ uint4 ld_nc_16(const uint16_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ float elem(const uint4& v, int i) {
  const uint32_t w = (i < 2) ? v.x : (i < 4) ? v.y : (i < 6) ? v.z : v.w;
  return (i & 1) ? bf16_hi(w) : bf16_lo(w);
}

// kExp experts x 8 tokens of partials per lane.  With kPipe the next chunk's
// loads are issued before the current chunk's fmas (software pipelining), so
// the L2 latency of one chunk hides behind the arithmetic of the previous one;
// it doubles the load registers, so it is used where there are few warps.
template <int kExp, bool kPipe>
__global__ void __launch_bounds__(kWarps * 32) router_logits_kernel(const uint16_t* __restrict__ x,
                                                                    const uint16_t* __restrict__ w_router,
                                                                    const float* __restrict__ bias, int M, int H,
                                                                    int E, float* __restrict__ logits) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kTokPerWarp;
  const int e0 = (blockIdx.y * kWarps + warp) * kExp;
  if (e0 >= E) return;

  float acc[kTokPerWarp][kExp];
#pragma unroll
  for (int t = 0; t < kTokPerWarp; ++t)
#pragma unroll
    for (int q = 0; q < kExp; ++q) acc[t][q] = 0.0f;

  const int nchunk = H / 256;
  uint4 wv[kExp], xv[kTokPerWarp];
  auto load = [&](int j, uint4 (&wd)[kExp], uint4 (&xd)[kTokPerWarp]) {
    const int h = 256 * j + 8 * lane;
#pragma unroll
    for (int q = 0; q < kExp; ++q)
      wd[q] = (e0 + q < E) ? ld_nc_16(w_router + static_cast<size_t>(e0 + q) * H + h) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int t = 0; t < kTokPerWarp; ++t)
      xd[t] = (t0 + t < M) ? ld_nc_16(x + static_cast<size_t>(t0 + t) * H + h) : make_uint4(0, 0, 0, 0);
  };
  if (kPipe) load(0, wv, xv);
#pragma unroll 1
  for (int j = 0; j < nchunk; ++j) {
    uint4 wn[kExp], xn[kTokPerWarp];
    if (kPipe) {
      if (j + 1 < nchunk) load(j + 1, wn, xn);
    } else {
      load(j, wv, xv);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)  // increasing h inside the chunk
#pragma unroll
      for (int t = 0; t < kTokPerWarp; ++t)
#pragma unroll
        for (int q = 0; q < kExp; ++q) acc[t][q] = __fmaf_rn(elem(xv[t], i), elem(wv[q], i), acc[t][q]);
    if (kPipe && j + 1 < nchunk) {
#pragma unroll
      for (int q = 0; q < kExp; ++q) wv[q] = wn[q];
#pragma unroll
      for (int t = 0; t < kTokPerWarp; ++t) xv[t] = xn[t];
    }
  }

#pragma unroll
  for (int t = 0; t < kTokPerWarp; ++t)
#pragma unroll
    for (int q = 0; q < kExp; ++q) {
      float v = acc[t][q];
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, off));
      acc[t][q] = v;
    }
  // lane l stores pair l = (t, q) = (l / kExp, l % kExp)
#pragma unroll
  for (int t = 0; t < kTokPerWarp; ++t)
#pragma unroll
    for (int q = 0; q < kExp; ++q)
      if (lane == t * kExp + q && t0 + t < M && e0 + q < E) {
        const float b = bias != nullptr ? bias[e0 + q] : 0.0f;
        logits[static_cast<size_t>(t0 + t) * E + e0 + q] = __fadd_rn(acc[t][q], b);
      }
}

// (value, id) ordering of the selection: larger value first, then lower id.
__device__ __forceinline__ bool better(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

template <int kPerLane>
__global__ void __launch_bounds__(128) router_topk_kernel(const float* __restrict__ logits, int M, int E, int K,
                                                          int32_t* __restrict__ topk_ids,
                                                          float* __restrict__ topk_w) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (t >= M) return;
  float v[kPerLane];
  bool live[kPerLane];
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    const int e = lane + 32 * i;
    live[i] = e < E;
    v[i] = live[i] ? logits[static_cast<size_t>(t) * E + e] : -INFINITY;
  }
  float sel_v = 0.0f;
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
    for (int i = 0; i < kPerLane; ++i)  // the owner retires the winner
      if (lane + 32 * i == bi) live[i] = false;
    if (lane == k) {
      sel_v = bv;
      sel_id = bi;
    }
  }
  const float s = (lane < K) ? 1.0f / (1.0f + expf(-sel_v)) : 0.0f;
  float total = s;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) total += __shfl_xor_sync(0xffffffffu, total, off);
  if (lane < K) {
    topk_ids[static_cast<size_t>(t) * K + lane] = sel_id;
    topk_w[static_cast<size_t>(t) * K + lane] = s / total;
  }
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
    z[i] = live[i] ? zt[e] : -INFINITY;
    v[i] = (live[i] && sel_bias != nullptr) ? __fadd_rn(z[i], sel_bias[e]) : z[i];
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
    const float zs = zt[sel_id];
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
  const int tok_blocks = (M + kTokPerWarp - 1) / kTokPerWarp;
  if (M <= 64) {  // few tokens: one expert per warp, so that enough warps stream W_r
    dim3 grid(tok_blocks, (E + kWarps - 1) / kWarps);
    router_logits_kernel<1, true><<<grid, kWarps * 32, 0, stream>>>(x, w_router, bias, M, H, E, logits);
  } else {
    dim3 grid(tok_blocks, (E + 4 * kWarps - 1) / (4 * kWarps));
    router_logits_kernel<4, false><<<grid, kWarps * 32, 0, stream>>>(x, w_router, bias, M, H, E, logits);
  }
  return cudaGetLastError();
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
// stand-in for it, so the device address is looked up once per device (with
// that device current) and passed to the kernels as a plain pointer.
namespace {

static __device__ __align__(256) float g_route_logits_scratch[MOE_ROUTE_NOALLOC_MAX_LOGITS];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
float* g_scratch_ptr[kMaxDevices] = {};

// Device address of the array on the current device (set-up on first use).
cudaError_t route_scratch_address(float** out) {
  int dev = 0;
  cudaError_t st = cudaGetDevice(&dev);
  if (st != cudaSuccess) return st;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    st = cudaGetSymbolAddress(&ptr, g_route_logits_scratch);
    if (st != cudaSuccess) return st;
    g_scratch_ptr[dev] = static_cast<float*>(ptr);
  }
  *out = g_scratch_ptr[dev];
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
