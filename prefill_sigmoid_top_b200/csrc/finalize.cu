// Top-k weighted sum + residual add + RMSNorm in one pass ("[flashinfer]
// Kimi K3를 위한 초고속 통신 최적화", flashinfer PR #5701 analysis: the MoE
// finalize fused with RMSNorm; §2 HT preset: one 128-thread consumer group per
// token, 7 vectors of bf16x8 per thread = 896 packs = one H=7168 row; §3:
// RMS_EPS = 1e-5 and WEIGHT_BIAS = 0, so gamma multiplies as is).
//
// Many tokens: one CTA of 256 threads per token.  Each thread owns up to 4 packs of 8
// hidden elements (p = tid + 256*i), keeps s = x + sum_k w_k * y_k for them
// in 32 fp32 registers, and only out (and optionally bf16(s)) is written:
// the expert sum never goes back to HBM before the norm.  The loop over the
// K expert rows is unrolled by 4, so 16 independent 16-byte loads per thread
// are in flight.
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxPacks = 4;  // H <= 4 * 8 * 256 = 8192

__device__ __forceinline__ uint4 ld_stream_16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
  f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
  f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
  f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

// At most 64 registers a thread, so that four CTAs (1024 threads) share an SM:
// the kernel waits on loads, and more resident warps keep more of them in
// flight (measured 99 -> 91 us at 2048 tokens, 56 -> 46 us at 1000).
__global__ void __launch_bounds__(kThreads, 4) finalize_kernel(const uint16_t* __restrict__ x,
                                                            const uint16_t* __restrict__ y,
                                                            const float* __restrict__ topk_w,
                                                            const uint16_t* __restrict__ gamma, float eps, int K,
                                                            int H, uint16_t* __restrict__ out,
                                                            uint16_t* __restrict__ residual_out) {
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  const int npk = H / 8;
  float acc[kMaxPacks][8];

#pragma unroll
  for (int i = 0; i < kMaxPacks; ++i) {
    const int p = tid + kThreads * i;
    if (p < npk) {
      unpack8(ld_stream_16(x + static_cast<size_t>(t) * H + p * 8), acc[i]);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
    }
  }
  const uint16_t* yt = y + static_cast<size_t>(t) * K * H;
#pragma unroll 4
  for (int k = 0; k < K; ++k) {
    const float wk = topk_w[static_cast<size_t>(t) * K + k];
    uint4 v[kMaxPacks];
#pragma unroll
    for (int i = 0; i < kMaxPacks; ++i) {
      const int p = tid + kThreads * i;
      v[i] = (p < npk) ? ld_stream_16(yt + static_cast<size_t>(k) * H + p * 8) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < kMaxPacks; ++i) {
      float f[8];
      unpack8(v[i], f);
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(wk, f[j], acc[i][j]);
    }
  }

  float ss = 0.0f;
#pragma unroll
  for (int i = 0; i < kMaxPacks; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) ss = fmaf(acc[i][j], acc[i][j], ss);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  __shared__ float part[kThreads / 32];
  if ((tid & 31) == 0) part[tid >> 5] = ss;
  __syncthreads();
  float total = 0.0f;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) total += part[w];
  const float inv = 1.0f / sqrtf(total / static_cast<float>(H) + eps);

#pragma unroll
  for (int i = 0; i < kMaxPacks; ++i) {
    const int p = tid + kThreads * i;
    if (p >= npk) continue;
    float g[8];
    unpack8(*reinterpret_cast<const uint4*>(gamma + p * 8), g);
    uint4 o, r;
    o.x = pack_bf16x2(acc[i][0] * inv * g[0], acc[i][1] * inv * g[1]);
    o.y = pack_bf16x2(acc[i][2] * inv * g[2], acc[i][3] * inv * g[3]);
    o.z = pack_bf16x2(acc[i][4] * inv * g[4], acc[i][5] * inv * g[5]);
    o.w = pack_bf16x2(acc[i][6] * inv * g[6], acc[i][7] * inv * g[7]);
    *reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * H + p * 8) = o;
    if (residual_out != nullptr) {
      r.x = pack_bf16x2(acc[i][0], acc[i][1]);
      r.y = pack_bf16x2(acc[i][2], acc[i][3]);
      r.z = pack_bf16x2(acc[i][4], acc[i][5]);
      r.w = pack_bf16x2(acc[i][6], acc[i][7]);
      *reinterpret_cast<uint4*>(residual_out + static_cast<size_t>(t) * H + p * 8) = r;
    }
  }
}

// Few tokens: one CTA per token leaves most SMs idle and each CTA waits on
// K rows of y in turn, so each token's row is split over a cluster of kSplit
// CTAs (128 threads, one 8-element pack per thread).  Each CTA reduces the
// sum of squares of its slice; the kSplit partials are exchanged through
// distributed shared memory and added in rank order, so every CTA of the
// cluster applies the same 1/rms.
constexpr int kSplit = 8;
constexpr int kSplitThreads = 128;

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_peer_f32(const float* local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_addr(local)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

__global__ void __launch_bounds__(kSplitThreads) finalize_split_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ y, const float* __restrict__ topk_w,
    const uint16_t* __restrict__ gamma, float eps, int K, int H, uint16_t* __restrict__ out,
    uint16_t* __restrict__ residual_out) {
  __shared__ float part[kSplitThreads / 32];
  __shared__ float cta_ss;
  const int t = blockIdx.y;
  const int tid = threadIdx.x;
  const uint32_t q = cluster_rank();
  const int npk = H / 8;
  const int per = (npk + kSplit - 1) / kSplit;
  const int p = static_cast<int>(q) * per + tid;
  const bool live = tid < per && p < npk;

  float acc[8];
  if (live) {
    unpack8(ld_stream_16(x + static_cast<size_t>(t) * H + p * 8), acc);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
  }
  const uint16_t* yt = y + static_cast<size_t>(t) * K * H;
#pragma unroll 8
  for (int k = 0; k < K; ++k) {
    const float wk = topk_w[static_cast<size_t>(t) * K + k];
    const uint4 v = live ? ld_stream_16(yt + static_cast<size_t>(k) * H + p * 8) : make_uint4(0, 0, 0, 0);
    float f[8];
    unpack8(v, f);
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = fmaf(wk, f[j], acc[j]);
  }
  float ss = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) ss = fmaf(acc[j], acc[j], ss);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if ((tid & 31) == 0) part[tid >> 5] = ss;
  __syncthreads();
  if (tid == 0) {
    float c = 0.0f;
#pragma unroll
    for (int w = 0; w < kSplitThreads / 32; ++w) c += part[w];
    cta_ss = c;
  }
  cluster_sync_all();  // every CTA's partial is written
  float total = 0.0f;
#pragma unroll
  for (int r = 0; r < kSplit; ++r) total += ld_peer_f32(&cta_ss, static_cast<uint32_t>(r));
  cluster_sync_all();  // no CTA leaves while a peer may still read its partial
  const float inv = 1.0f / sqrtf(total / static_cast<float>(H) + eps);
  if (!live) return;
  float g[8];
  unpack8(*reinterpret_cast<const uint4*>(gamma + p * 8), g);
  uint4 o;
  o.x = pack_bf16x2(acc[0] * inv * g[0], acc[1] * inv * g[1]);
  o.y = pack_bf16x2(acc[2] * inv * g[2], acc[3] * inv * g[3]);
  o.z = pack_bf16x2(acc[4] * inv * g[4], acc[5] * inv * g[5]);
  o.w = pack_bf16x2(acc[6] * inv * g[6], acc[7] * inv * g[7]);
  *reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * H + p * 8) = o;
  if (residual_out != nullptr) {
    uint4 r;
    r.x = pack_bf16x2(acc[0], acc[1]);
    r.y = pack_bf16x2(acc[2], acc[3]);
    r.z = pack_bf16x2(acc[4], acc[5]);
    r.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(residual_out + static_cast<size_t>(t) * H + p * 8) = r;
  }
}

// Self-test of the bounded waits every pipelined kernel uses: thread 0 waits
// on an mbarrier that nothing ever arrives at, gives up after limit_ns and
// records MOE_ERR_TIMEOUT, exactly as a kernel whose copies never landed would.
__global__ void wait_timeout_selftest_kernel(int32_t* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait_bounded(&bar, 0, nullptr, limit_ns)) set_error(err, kErrTimeout);
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(int32_t* err, uint64_t limit_ns, cudaStream_t stream) {
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(err, limit_ns);
  return cudaGetLastError();
}

cudaError_t launch_finalize(const uint16_t* x, const uint16_t* y, const float* topk_w, const uint16_t* gamma,
                            float eps, int M, int K, int H, uint16_t* out, uint16_t* residual_out,
                            cudaStream_t stream) {
  if (M <= 64 && H / 8 <= kSplit * kSplitThreads) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(kSplit, M);
    cfg.blockDim = dim3(kSplitThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kSplit;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, finalize_split_kernel, x, y, topk_w, gamma, eps, K, H, out, residual_out);
  }
  finalize_kernel<<<M, kThreads, 0, stream>>>(x, y, topk_w, gamma, eps, K, H, out, residual_out);
  return cudaGetLastError();
}

}  // namespace moe
