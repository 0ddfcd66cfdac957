// The tensor-parallel finalize: top-k weighted sum of this rank's partial
// expert rows, reduction across the G ranks over NVLink, residual add and
// RMSNorm in one kernel ("[flashinfer] Kimi K3를 위한 초고속 통신 최적화",
// flashinfer PR #5701 analysis: intro -- MoE finalize + all-reduce + RMSNorm
// fused; §2 -- the exchange protocol chosen by M: a one-round low-latency
// exchange for M <= 24, bulk transfers above; §3 -- RMS_EPS = 1e-5,
// WEIGHT_BIAS = 0).  The definitions, the buffer protocol and the error
// behaviour are stated in include/moe_b200_tp.h.
//
// Per token the arithmetic is that of the single-GPU finalize kernels, step
// for step: each thread owns the same 8-element packs, p_r = (rank 0: x) +
// sum_k w_k y_r[k] by fmaf in k order, s = p_0 + p_1 + ... in rank order, and
// the sum of squares is reduced in the same tree (M <= 64: 8 slices of 128
// threads, as the cluster kernel; else 256 threads x 4 packs).  With G = 1
// nothing is exchanged and the result is the finalize's, bit for bit.
//
// Exchange: the partial rows are stored straight into the peers' group
// buffers (16-byte stores through the peer mapping; no multicast), then one
// thread sets a flag per (source rank, token) with a system-scope release.
// The readers spin (bounded) on their own buffer's flags with system-scope
// acquires and read the rows through L2.  Every CTA stores all it sends
// before it waits for anything, and the launch is cooperative (all CTAs of a
// rank resident together), so every wait is for data already on its way.
#include <cudaTypedefs.h>

#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "moe_b200_tp.h"

namespace moe {
namespace {

constexpr uint64_t kTpWaitLimitNs = 2000ull * 1000ull * 1000ull;  // ranks may reach the finalize far apart

// Byte layout of one group buffer (the same on every rank).
struct TpLayout {
  size_t epoch, done, pflag, oflag, parts, outs, res, total;
  int rows;  // fp32 partial rows per (parity, source)
};

__host__ __device__ inline size_t tp_align(size_t v) { return (v + 255) / 256 * 256; }

__host__ __device__ inline TpLayout tp_layout(int G, int max_tokens, int H) {
  TpLayout L{};
  const int owned = (max_tokens + G - 1) / G;
  const int one = max_tokens < MOE_TP_ONESHOT_MAX_TOKENS ? max_tokens : MOE_TP_ONESHOT_MAX_TOKENS;
  L.rows = owned > one ? owned : one;
  L.epoch = 0;
  L.done = 4;
  L.pflag = 256;
  L.oflag = tp_align(L.pflag + static_cast<size_t>(G) * max_tokens * 4);
  L.parts = tp_align(L.oflag + static_cast<size_t>(max_tokens) * 4);
  L.outs = tp_align(L.parts + 2ull * G * L.rows * H * 4);
  L.res = tp_align(L.outs + 2ull * max_tokens * H * 2);
  L.total = tp_align(L.res + 2ull * max_tokens * H * 2);
  return L;
}

struct TpArgs {
  const uint16_t* x;
  const float* topk_w;
  const uint16_t* gamma;
  const uint16_t* y[MOE_TP_MAX_RANKS];   // per CTA row (emulated rank), or [0] alone
  uint16_t* out[MOE_TP_MAX_RANKS];
  uint16_t* res[MOE_TP_MAX_RANKS];       // nullable entries
  uint8_t* bufs[MOE_TP_MAX_RANKS];       // group buffers by rank
  int32_t* err;
  int rank0;                             // rank of CTA row 0
  int G, M, K, H, max_tokens;
  int twoshot;
  float eps;
};

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

__device__ __forceinline__ void st_release_sys(uint32_t* p, uint32_t v) {
  asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Waits until *flag has reached call number e (wrapping compare).  False on expiry.
__device__ bool wait_flag(const uint32_t* flag, uint32_t e) {
  if (static_cast<int32_t>(ld_acquire_sys(flag) - e) >= 0) return true;
  const uint64_t t0 = global_timer_ns();
  uint32_t ns = 32;
  while (true) {
    __nanosleep(ns);
    if (ns < 1024) ns *= 2;
    if (static_cast<int32_t>(ld_acquire_sys(flag) - e) >= 0) return true;
    if (global_timer_ns() - t0 > kTpWaitLimitNs) return false;
  }
}

// Thread -> pack mapping of the two single-GPU finalize kernels.
template <bool kFew>
struct Packs {
  static constexpr int kThreads = kFew ? 1024 : 256;
  static constexpr int kNP = kFew ? 1 : 4;
  // pack index of slot i of thread tid, or -1
  __device__ static int pack(int tid, int i, int npk) {
    if (kFew) {
      const int per = (npk + 7) / 8, q = tid >> 7, lt = tid & 127;
      const int p = q * per + lt;
      return (lt < per && p < npk) ? p : -1;
    }
    const int p = tid + 256 * i;
    return p < npk ? p : -1;
  }
};

template <bool kFew>
__global__ void __launch_bounds__(Packs<kFew>::kThreads) tp_finalize_kernel(TpArgs a) {
  using P = Packs<kFew>;
  constexpr int NP = P::kNP;
  __shared__ float part[P::kThreads / 32];
  __shared__ int abort_s;
  const int tid = threadIdx.x;
  const int row = blockIdx.y;                 // emulated rank index (0 for a real rank)
  const int rank = a.rank0 + row;
  const int G = a.G, M = a.M, K = a.K, H = a.H;
  const int npk = H / 8;
  const int nb = gridDim.x;
  const uint16_t* __restrict__ y = a.y[row];
  uint16_t* __restrict__ out = a.out[row];
  uint16_t* __restrict__ res = a.res[row];
  const TpLayout L = tp_layout(G, a.max_tokens, H);
  uint8_t* own = a.bufs[rank];
  if (tid == 0) abort_s = 0;

  // this call's number and data parity (the last CTA of the call advances the number)
  uint32_t e = 1;
  if (G > 1) e = *reinterpret_cast<volatile uint32_t*>(own + L.epoch) + 1;
  const int par = e & 1;
  __syncthreads();

  // weighted sum of this rank's partial rows (+ x on rank 0), the finalize's order
  auto local_partial = [&](int t, float (&acc)[NP][8]) {
#pragma unroll
    for (int i = 0; i < NP; ++i) {
      const int p = P::pack(tid, i, npk);
      if (p >= 0 && rank == 0) {
        unpack8(ld_stream_16(a.x + static_cast<size_t>(t) * H + p * 8), acc[i]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
      }
    }
    const uint16_t* yt = y + static_cast<size_t>(t) * K * H;
#pragma unroll 4
    for (int k = 0; k < K; ++k) {
      const float wk = a.topk_w[static_cast<size_t>(t) * K + k];
      uint4 v[NP];
#pragma unroll
      for (int i = 0; i < NP; ++i) {
        const int p = P::pack(tid, i, npk);
        v[i] = p >= 0 ? ld_stream_16(yt + static_cast<size_t>(k) * H + p * 8) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int i = 0; i < NP; ++i) {
        float f[8];
        unpack8(v[i], f);
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(wk, f[j], acc[i][j]);
      }
    }
  };

  // sum of squares, 1/rms, out and residual rows (local), in the finalize kernels' tree
  auto finish = [&](int t, float (&s)[NP][8], uint4 (&ob)[NP], uint4 (&rb)[NP]) {
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < NP; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) ss = fmaf(s[i][j], s[i][j], ss);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    __syncthreads();  // part[] is free (an earlier token may still be reading it)
    if ((tid & 31) == 0) part[tid >> 5] = ss;
    __syncthreads();
    float total = 0.0f;
    if (kFew) {  // 8 slices of 4 warps: each slice's sum, then the slices in order
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        float c = 0.0f;
#pragma unroll
        for (int w = 0; w < 4; ++w) c += part[q * 4 + w];
        total += c;
      }
    } else {
#pragma unroll
      for (int w = 0; w < P::kThreads / 32; ++w) total += part[w];
    }
    const float inv = 1.0f / sqrtf(total / static_cast<float>(H) + a.eps);
#pragma unroll
    for (int i = 0; i < NP; ++i) {
      const int p = P::pack(tid, i, npk);
      if (p < 0) continue;
      float g[8];
      unpack8(*reinterpret_cast<const uint4*>(a.gamma + p * 8), g);
      ob[i].x = pack_bf16x2(s[i][0] * inv * g[0], s[i][1] * inv * g[1]);
      ob[i].y = pack_bf16x2(s[i][2] * inv * g[2], s[i][3] * inv * g[3]);
      ob[i].z = pack_bf16x2(s[i][4] * inv * g[4], s[i][5] * inv * g[5]);
      ob[i].w = pack_bf16x2(s[i][6] * inv * g[6], s[i][7] * inv * g[7]);
      rb[i].x = pack_bf16x2(s[i][0], s[i][1]);
      rb[i].y = pack_bf16x2(s[i][2], s[i][3]);
      rb[i].z = pack_bf16x2(s[i][4], s[i][5]);
      rb[i].w = pack_bf16x2(s[i][6], s[i][7]);
      *reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * H + p * 8) = ob[i];
      if (res != nullptr) *reinterpret_cast<uint4*>(res + static_cast<size_t>(t) * H + p * 8) = rb[i];
    }
  };

  auto part_row = [&](uint8_t* buf, int src, int r) {
    return reinterpret_cast<float*>(buf + L.parts) + ((static_cast<size_t>(par) * G + src) * L.rows + r) * H;
  };
  auto pflag = [&](uint8_t* buf, int src, int t) {
    return reinterpret_cast<uint32_t*>(buf + L.pflag) + static_cast<size_t>(src) * a.max_tokens + t;
  };
  auto oflag = [&](uint8_t* buf, int t) { return reinterpret_cast<uint32_t*>(buf + L.oflag) + t; };
  auto out_row = [&](uint8_t* buf, size_t off, int t) {
    return reinterpret_cast<uint16_t*>(buf + off) + (static_cast<size_t>(par) * a.max_tokens + t) * H;
  };
  // thread 0 waits for a flag; the whole CTA learns whether it arrived (abort_s is written only by
  // thread 0 before the first barrier and read by all between the two)
  auto cta_wait = [&](const uint32_t* flag) -> bool {
    if (tid == 0 && abort_s == 0 && !wait_flag(flag, e)) {
      set_error(a.err, kErrTimeout);
      abort_s = 1;
    }
    __syncthreads();
    const bool ok = abort_s == 0;
    __syncthreads();
    return ok;
  };

  // ---- phase 1: local partials; G = 1 finishes here, otherwise they are sent (no waiting)
  for (int t = blockIdx.x; t < M; t += nb) {
    float acc[NP][8];
    local_partial(t, acc);
    if (G == 1) {
      uint4 ob[NP], rb[NP];
      finish(t, acc, ob, rb);
      continue;
    }
    const int owner = t % G;
    const int d0 = a.twoshot ? owner : 0, d1 = a.twoshot ? owner + 1 : G;
    const int r = a.twoshot ? t / G : t;
    for (int d = d0; d < d1; ++d) {
      float* dst = part_row(a.bufs[d], rank, r);
#pragma unroll
      for (int i = 0; i < NP; ++i) {
        const int p = P::pack(tid, i, npk);
        if (p < 0) continue;
        reinterpret_cast<float4*>(dst + p * 8)[0] = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
        reinterpret_cast<float4*>(dst + p * 8)[1] = make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
      }
    }
    __syncthreads();
    if (tid == 0) {
      __threadfence_system();
      for (int d = d0; d < d1; ++d) st_release_sys(pflag(a.bufs[d], rank, t), e);
    }
  }

  if (G > 1) {
    // ---- phase 2: reduce (every token: ONESHOT; owned tokens: TWOSHOT), normalise, send finished rows
    const int nred = a.twoshot ? (M - rank + G - 1) / G : M;
    for (int j = blockIdx.x; j < nred; j += nb) {
      const int t = a.twoshot ? rank + j * G : j;
      const int r = a.twoshot ? j : t;
      bool ok = true;
      for (int src = 0; src < G && ok; ++src) ok = cta_wait(pflag(own, src, t));
      if (!ok) break;
      float s[NP][8];
#pragma unroll
      for (int i = 0; i < NP; ++i) {
        const int p = P::pack(tid, i, npk);
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) s[i][jj] = 0.0f;
        if (p < 0) continue;
        for (int src = 0; src < G; ++src) {
          const float4* q = reinterpret_cast<const float4*>(part_row(own, src, r) + p * 8);
          const float4 lo = __ldcg(q), hi = __ldcg(q + 1);
          const float v[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) s[i][jj] = src == 0 ? v[jj] : __fadd_rn(s[i][jj], v[jj]);
        }
      }
      uint4 ob[NP], rb[NP];
      finish(t, s, ob, rb);
      if (a.twoshot) {
        for (int d = 0; d < G; ++d) {
          if (d == rank) continue;
#pragma unroll
          for (int i = 0; i < NP; ++i) {
            const int p = P::pack(tid, i, npk);
            if (p < 0) continue;
            *reinterpret_cast<uint4*>(out_row(a.bufs[d], L.outs, t) + p * 8) = ob[i];
            if (res != nullptr) *reinterpret_cast<uint4*>(out_row(a.bufs[d], L.res, t) + p * 8) = rb[i];
          }
        }
        __syncthreads();
        if (tid == 0) {
          __threadfence_system();
          for (int d = 0; d < G; ++d)
            if (d != rank) st_release_sys(oflag(a.bufs[d], t), e);
        }
      }
    }

    // ---- phase 3 (TWOSHOT): the rows other ranks finished, copied from this rank's buffer
    if (a.twoshot) {
      for (int t = blockIdx.x; t < M; t += nb) {
        if (t % G == rank) continue;
        if (!cta_wait(oflag(own, t))) break;
#pragma unroll
        for (int i = 0; i < NP; ++i) {
          const int p = P::pack(tid, i, npk);
          if (p < 0) continue;
          const uint4 o = __ldcg(reinterpret_cast<const uint4*>(out_row(own, L.outs, t) + p * 8));
          *reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * H + p * 8) = o;
          if (res != nullptr) {
            const uint4 q = __ldcg(reinterpret_cast<const uint4*>(out_row(own, L.res, t) + p * 8));
            *reinterpret_cast<uint4*>(res + static_cast<size_t>(t) * H + p * 8) = q;
          }
        }
      }
    }

    // ---- the last CTA of this rank advances the call number
    __syncthreads();
    if (tid == 0 && abort_s == 0) {
      __threadfence();
      unsigned* done = reinterpret_cast<unsigned*>(own + L.done);
      if (atomicAdd(done, 1u) == static_cast<unsigned>(nb) - 1) {
        *done = 0;
        __threadfence();
        *reinterpret_cast<volatile uint32_t*>(own + L.epoch) = e;
      }
    }
  }
}

template <bool kFew>
cudaError_t launch_tp(const TpArgs& a, int rows, cudaStream_t stream) {
  auto kern = tp_finalize_kernel<kFew>;
  constexpr int threads = Packs<kFew>::kThreads;
  int dev = 0, sms = 0, per_sm = 0;
  cudaError_t st = cudaGetDevice(&dev);
  if (st == cudaSuccess) st = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (st == cudaSuccess) st = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, 0);
  if (st != cudaSuccess) return st;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int cap = per_sm * sms / rows;  // CTAs per rank that are resident together
  if (cap < 1) return cudaErrorCooperativeLaunchTooLarge;
  const int nb = a.M < cap ? a.M : cap;
  TpArgs args = a;
  if (a.G == 1) {  // nothing is exchanged, no CTA waits for another: a plain launch
    kern<<<dim3(nb, rows), threads, 0, stream>>>(args);
    return cudaGetLastError();
  }
  void* params[] = {&args};
  return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kern), dim3(nb, rows), dim3(threads), params, 0,
                                     stream);
}

bool want_twoshot(int M, int G, int max_tokens) {
  if (G <= 1) return false;
  const TpLayout L = tp_layout(G, max_tokens, 256);
  if (const char* env = std::getenv("MOE_TP_PROTOCOL")) {
    if (std::strcmp(env, "oneshot") == 0 && M <= L.rows) return false;
    if (std::strcmp(env, "twoshot") == 0) return true;
  }
  return M > MOE_TP_ONESHOT_MAX_TOKENS;
}

}  // namespace

size_t tp_buffer_bytes(int G, int max_tokens, int H) { return tp_layout(G, max_tokens, H).total; }

int tp_protocol(int M, int G, int max_tokens) { return want_twoshot(M, G, max_tokens) ? 1 : 0; }

cudaError_t launch_tp_finalize(const uint16_t* x, const uint16_t* const* ys, const float* topk_w,
                               const uint16_t* gamma, float eps, int M, int K, int H, int G, int max_tokens,
                               int rank0, int rows, void* const* bufs, uint16_t* const* outs,
                               uint16_t* const* residual_outs, int32_t* err, cudaStream_t stream) {
  TpArgs a{};
  a.x = x;
  a.topk_w = topk_w;
  a.gamma = gamma;
  for (int r = 0; r < rows; ++r) {
    a.y[r] = ys[r];
    a.out[r] = outs[r];
    a.res[r] = residual_outs != nullptr ? residual_outs[r] : nullptr;
  }
  for (int r = 0; r < G; ++r) a.bufs[r] = bufs != nullptr ? static_cast<uint8_t*>(bufs[r]) : nullptr;
  a.err = err;
  a.rank0 = rank0;
  a.G = G;
  a.M = M;
  a.K = K;
  a.H = H;
  a.max_tokens = max_tokens;
  a.twoshot = want_twoshot(M, G, max_tokens) ? 1 : 0;
  a.eps = eps;
  // the thread shapes of the single-GPU finalize: 8 slices of 128 threads per token up to 64 tokens
  if (M <= 64 && H / 8 <= 8 * 128) return launch_tp<true>(a, rows, stream);
  return launch_tp<false>(a, rows, stream);
}

}  // namespace moe

// ---------------------------------------------------------------------------
// C ABI (include/moe_b200_tp.h): argument checks and the IPC plumbing.
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Start of the device allocation that contains p (driver entry point looked up at run time, so the
// library does not link the driver library itself).
bool allocation_base(const void* p, void** base) {
  static PFN_cuPointerGetAttribute_v4000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuPointerGetAttribute", &f, 4000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuPointerGetAttribute_v4000>(f);
  });
  if (fn == nullptr) return false;
  CUdeviceptr start = 0;
  if (fn(&start, CU_POINTER_ATTRIBUTE_RANGE_START_ADDR, reinterpret_cast<CUdeviceptr>(p)) != CUDA_SUCCESS)
    return false;
  *base = reinterpret_cast<void*>(start);
  return true;
}

moe_status_t check_sizes(int32_t world, int32_t max_tokens, int32_t hidden) {
  if (world < 1 || world > MOE_TP_MAX_RANKS || max_tokens < 1) return MOE_ERR_UNSUPPORTED;
  if (hidden < 256 || hidden % 256 != 0 || hidden > 8192) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

}  // namespace

extern "C" {

size_t moe_tp_buffer_bytes(int32_t world, int32_t max_tokens, int32_t hidden) {
  if (check_sizes(world, max_tokens, hidden) != MOE_OK) return 0;
  return moe::tp_buffer_bytes(world, max_tokens, hidden);
}

int moe_tp_protocol(int32_t M, int32_t world, int32_t max_tokens) {
  if (world < 1 || world > MOE_TP_MAX_RANKS || M < 1 || max_tokens < 1) return -1;
  return moe::tp_protocol(M, world, max_tokens);
}

}  // extern "C"

namespace {
moe_status_t check_finalize_args(const moe_bf16_t* x, const float* topk_w, const moe_bf16_t* gamma, float eps,
                                 const moe_shape_t& s, int32_t world, int32_t max_tokens) {
  if (s.M < 1 || s.top_k < 1 || s.top_k > 32 || s.H < 256 || s.H % 256 != 0 || s.H > 8192)
    return MOE_ERR_UNSUPPORTED;
  moe_status_t st = check_sizes(world, max_tokens, s.H);
  if (st != MOE_OK) return st;
  if (s.M > max_tokens) return MOE_ERR_UNSUPPORTED;
  if (!x || !topk_w || !gamma || !aligned16(x) || !aligned16(gamma)) return MOE_ERR_INVALID_ARG;
  if (!(eps >= 0.0f)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}
}  // namespace

extern "C" {

moe_status_t moe_tp_finalize_allreduce_rmsnorm(const moe_bf16_t* x, const moe_bf16_t* y_partial,
                                               const float* topk_w, const moe_bf16_t* gamma, float eps,
                                               moe_shape_t s, const moe_tp_group_t* g, moe_bf16_t* out,
                                               moe_bf16_t* residual_out, int32_t* err_flag, moe_stream_t stream) {
  if (g == nullptr) return MOE_ERR_INVALID_ARG;
  moe_status_t st = check_finalize_args(x, topk_w, gamma, eps, s, g->world, g->max_tokens);
  if (st != MOE_OK) return st;
  if (g->hidden != s.H) return MOE_ERR_UNSUPPORTED;
  if (g->rank < 0 || g->rank >= g->world) return MOE_ERR_INVALID_ARG;
  if (!y_partial || !out || !aligned16(y_partial) || !aligned16(out) || (residual_out && !aligned16(residual_out)))
    return MOE_ERR_INVALID_ARG;
  if (g->world > 1)
    for (int r = 0; r < g->world; ++r)
      if (g->bufs[r] == nullptr || (reinterpret_cast<uintptr_t>(g->bufs[r]) & 255u) != 0) return MOE_ERR_INVALID_ARG;
  const uint16_t* ys[1] = {y_partial};
  uint16_t* outs[1] = {out};
  uint16_t* rs[1] = {residual_out};
  const cudaError_t e = moe::launch_tp_finalize(x, ys, topk_w, gamma, eps, s.M, s.top_k, s.H, g->world,
                                                g->max_tokens, g->rank, 1, g->bufs, outs, rs, err_flag,
                                                static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_tp_finalize_emulated(const moe_bf16_t* x, const moe_bf16_t* const* y_partials, const float* topk_w,
                                      const moe_bf16_t* gamma, float eps, moe_shape_t s, int32_t world,
                                      int32_t max_tokens, void* const* bufs, moe_bf16_t* const* outs,
                                      moe_bf16_t* const* residual_outs, int32_t* err_flag, moe_stream_t stream) {
  moe_status_t st = check_finalize_args(x, topk_w, gamma, eps, s, world, max_tokens);
  if (st != MOE_OK) return st;
  if (!y_partials || !outs || (world > 1 && !bufs)) return MOE_ERR_INVALID_ARG;
  for (int r = 0; r < world; ++r) {
    if (!y_partials[r] || !outs[r] || !aligned16(y_partials[r]) || !aligned16(outs[r])) return MOE_ERR_INVALID_ARG;
    if (residual_outs && (!residual_outs[r] || !aligned16(residual_outs[r]))) return MOE_ERR_INVALID_ARG;
    if (world > 1 && (bufs[r] == nullptr || (reinterpret_cast<uintptr_t>(bufs[r]) & 255u) != 0))
      return MOE_ERR_INVALID_ARG;
  }
  const cudaError_t e = moe::launch_tp_finalize(x, y_partials, topk_w, gamma, eps, s.M, s.top_k, s.H, world,
                                                max_tokens, 0, world, bufs, outs, residual_outs, err_flag,
                                                static_cast<cudaStream_t>(stream));
  if (e == cudaErrorCooperativeLaunchTooLarge) {
    (void)cudaGetLastError();
    return MOE_ERR_UNSUPPORTED;
  }
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_tp_ipc_handle(const void* buf, void* handle_out) {
  if (!buf || !handle_out) return MOE_ERR_INVALID_ARG;
  static_assert(sizeof(cudaIpcMemHandle_t) + sizeof(uint64_t) == MOE_TP_IPC_HANDLE_BYTES, "IPC handle size");
  // the handle names the whole allocation; the buffer may sit at an offset inside it
  void* base = nullptr;
  if (!allocation_base(buf, &base)) return MOE_ERR_CUDA;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, const_cast<void*>(buf)) != cudaSuccess) return MOE_ERR_CUDA;
  const uint64_t off = static_cast<uint64_t>(static_cast<const uint8_t*>(buf) - static_cast<const uint8_t*>(base));
  std::memcpy(handle_out, &h, sizeof(h));
  std::memcpy(static_cast<uint8_t*>(handle_out) + sizeof(h), &off, sizeof(off));
  return MOE_OK;
}

moe_status_t moe_tp_ipc_open(const void* handle, void** buf_out) {
  if (!handle || !buf_out) return MOE_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  uint64_t off = 0;
  std::memcpy(&h, handle, sizeof(h));
  std::memcpy(&off, static_cast<const uint8_t*>(handle) + sizeof(h), sizeof(off));
  void* base = nullptr;
  if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) return MOE_ERR_CUDA;
  *buf_out = static_cast<uint8_t*>(base) + off;
  return MOE_OK;
}

moe_status_t moe_tp_ipc_close(void* buf) {
  if (!buf) return MOE_ERR_INVALID_ARG;
  void* base = nullptr;
  if (!allocation_base(buf, &base)) return MOE_ERR_CUDA;
  return cudaIpcCloseMemHandle(base) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"
