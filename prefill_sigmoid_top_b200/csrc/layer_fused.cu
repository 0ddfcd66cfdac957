// The whole routed MoE layer in one persistent launch, for decode shapes
// ("AWS Trainium2에서 GLM-5.3-Flash를 위한 NKI 레이어 메가커널: 디코드 스텝의
// 시간 사용처와 우리가 변경한 것": a layer per kernel, no hand-off between
// kernels inside the step; "[flashinfer] ... AlphaMoE NVFP4 커널 최적화",
// flashinfer PR #6511 analysis, §6: the route chain route -> align -> up ->
// down -> finalize, with the align launch folded away).
//
// The same arithmetic as the separate kernels, bit for bit (same fma order in
// the router, same MMA shapes and K order in the projections, the finalize's
// reduction order), on one cooperative grid of one CTA per SM:
//
//  1. router logits: a CTA takes 8 tokens x 6 experts at a time, their rows
//     staged whole in shared memory by bulk copies; lane l keeps partial l of
//     each pair in the canonical order.  z goes to the workspace; one bounded
//     grid barrier.
//  2. top-k and plan, redundantly in every CTA (at most 1024 routed slots):
//     warp-argmax top-k of every token, per-expert counts, the padded and the
//     compact prefix, and the slot ids of every expert in ascending slot
//     order (the expert-major plan without its padding).  CTA 0 writes the
//     routing outputs; the plan rows are written by the CTAs expert by expert.
//  3. projections: one global counter hands out work in a fixed order -- all
//     up tiles (expert, 128 rows of W_gate and W_up, <= 32 routed rows), then
//     all down tiles (expert, 256 rows of W_down, <= 32 rows), then one
//     finalize item per token.  A down tile of expert e waits (bounded) until
//     every up tile of e has published its h rows; a finalize item waits until
//     every down tile has published its y rows.  Work is claimed in list order
//     and a claimed tile never waits on a later one, so every wait ends.
//     The down tiles of the first experts start while the last up tiles are
//     still streaming, so no SM idles between the two projections.
//  4. finalize + residual + RMSNorm by the 4 epilogue warps, in the reduction
//     order of the finalize kernel the separate launches would use: up to 64
//     tokens, 8 slices per token on 8 CTAs whose partial sums of squares meet
//     in the workspace (added in slice order); more, one token per item.
//
// Warp roles in the 192-thread CTA (after phases 1-2, which all warps share):
//   warp 0      producer: claims work, queues it for the other roles, and
//               fills a ring of 6 slots of (two 128x64 weight boxes + up to 32
//               token rows x 64) -- up: the gate and the up rows of one k-step
//               with the token rows gathered by tile::gather4; down: rows
//               256w..256w+127 and 256w+128.. of W_down with h rows of the plan
//               (16-row boxes).  192 KB of weights in flight per SM, what the
//               weight stream needs at HBM speed.  After queueing a finalize
//               item it claims nothing more until that item is done, so the
//               finalize items spread over the CTAs.
//   warp 1      MMA issuer (one lane): per slot 2 x 4 tcgen05.mma (K = 16), one
//               per weight box, into one of two accumulator sets in tensor
//               memory.
//   warps 2-5   epilogue (tensor-memory lane quarter = warp % 4): SwiGLU into
//               h, or y scattered to its slot; then the finalize items.
// Every wait is bounded; a timeout sets the error word and unwinds.
#include "common.cuh"
#include "kernels.h"
#include "router_dot.cuh"

namespace moe {
namespace {

// Phase timeline of the launch, per CTA (timeline build only, -DMOE_LAYER_TRACE; see layer_trace.py):
// global-timer stamps (ns) of fixed points, the producer's total waits, and tile counts.
enum LayerTraceSlot {
  kLtStart = 0,         // kernel entry
  kLtBarrier = 1,       // the grid barrier after the router logits passed
  kLtPlan = 2,          // top-k and plan done, roles start
  kLtFirstDown = 3,     // the producer claimed its first down tile
  kLtLastUpPub = 4,     // this CTA published its last up tile
  kLtLastDownPub = 5,   // this CTA published its last down tile
  kLtFinStart = 6,      // first finalize item began (all y rows ready)
  kLtFinEnd = 7,        // last finalize item ended
  kLtWaitRows = 8,      // total ns the producer waited for an expert's h rows
  kLtWaitSlot = 9,      // total ns the producer waited for a free ring slot
  kLtUpTiles = 10,      // up tiles this CTA's epilogue finished
  kLtDownTiles = 11,    // down tiles
  kLtEnd = 12,          // kernel exit
  kLtSlots = 16
};
#ifdef MOE_LAYER_TRACE
constexpr int kLtCtas = 1024;
__device__ unsigned long long g_layer_trace[kLtCtas][kLtSlots];
#define MOE_LT(slot) g_layer_trace[blockIdx.x < kLtCtas ? blockIdx.x : kLtCtas - 1][(slot)]
#define MOE_LT_SET(slot, v) (MOE_LT(slot) = (v))
#define MOE_LT_FIRST(slot, v) (MOE_LT(slot) = MOE_LT(slot) ? MOE_LT(slot) : (v))
#define MOE_LT_ADD(slot, v) (MOE_LT(slot) += (v))
#define MOE_LT_NOW() global_timer_ns()
#else
#define MOE_LT_SET(slot, v) ((void)0)
#define MOE_LT_FIRST(slot, v) ((void)0)
#define MOE_LT_ADD(slot, v) ((void)0)
#define MOE_LT_NOW() 0ull
#endif

constexpr int kThreads = 192;
constexpr int kWarps = kThreads / 32;
constexpr int kBM = 128;                     // weight rows per tile (MMA M)
constexpr int kBK = 64;                      // contraction elements per slot
constexpr int kNmax = 32;                    // routed rows per token tile
constexpr int kATile = kBM * kBK * 2;            // 16 KB
constexpr int kBTile = kNmax * kBK * 2;          // 4 KB
constexpr int kSlotBytes = 2 * kATile + kBTile;  // 36 KB, a multiple of 1024
constexpr int kSlots = 6;
constexpr int kQueue = 4;
constexpr int kAccCols = 64;                 // two accumulators of kNmax columns: gate/up, or two W_down row blocks
constexpr int kTmemCols = 2 * kAccCols;
constexpr int kEpiWarp0 = 2;
constexpr int kEpiThreads = 128;
constexpr int kSplit = 8;                    // finalize: 8 accumulator sets of one 8-element pack
constexpr int kRtTok = 8;                    // router item: tokens (x experts, one per warp)
constexpr int kTopkPerLane = 8;              // E <= 256

enum : int { kKindUp = 0, kKindDown = 1, kKindFin = 2, kKindEnd = 3 };

// Shared memory (the dynamic base is 1024-byte aligned; the kernel checks).
// The ring takes almost all of it, so the plan is packed: int16 wherever the
// value fits (slot ids, compact offsets and token-tile prefixes stay below 2^15).
constexpr int kRingOff = 0;
constexpr int kNumBars = 2 * kSlots + 2 + 2 + 2 * kQueue + 3;
constexpr int kBarOff = kSlots * kSlotBytes;
constexpr int kWordOff = kBarOff + ((kNumBars * 8 + 15) / 16) * 16;  // tmem base, abort flag
constexpr int kQueueOff = kWordOff + 16;                             // int4 [kQueue], then the epilogue's item
constexpr int kPartOff = kQueueOff + 16 * (kQueue + 1);              // float [kSplit][4], then the weights [32]
constexpr int kIntOff = kPartOff + (4 * kSplit + 32) * 4;            // int32 offp, then int16 offc, tp, sl

__host__ __device__ constexpr int fused_smem_bytes(int E, int nslots) {
  return (kIntOff + 4 * (E + 1) + 2 * (2 * (E + 1) + nslots) + 15) / 16 * 16;
}
// One CTA per SM: at most 227 KB of dynamic shared memory.
constexpr int kSmemPerCta = 232448;
static_assert(fused_smem_bytes(256, 1024) <= kSmemPerCta, "the largest plan fits");
static_assert(kSlotBytes % 1024 == 0, "slot alignment");

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// Through L2 only: the data was written by other SMs during this launch.
__device__ __forceinline__ float ld_cg_f32(const float* p) {
  float v;
  asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p) : "memory");
  return v;
}

// Waits (acquire) until *p >= target.  Gives up after the wait limit or once
// *abort is set.
__device__ bool wait_count(const unsigned* p, unsigned target, const volatile int* abort) {
  if (ld_acquire(p) >= target) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 8; ++i) {
      __nanosleep(64);
      if (ld_acquire(p) >= target) return true;
    }
    if (abort != nullptr && *abort) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) return false;
  }
}

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
  f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
  f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
  f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

// (value, id) order of the selection: larger value first, then lower id.
__device__ __forceinline__ bool better(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// Expert of work index q inside a projection with W weight tiles per token
// tile: the largest e with tp[e] <= q / W (tp = prefix of token tiles).
__device__ __forceinline__ int4 decode_work(const int16_t* tp, int E, int W, int q, int kind) {
  const int u = q / W;
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tp[mid] <= u) lo = mid; else hi = mid - 1;
  }
  const int nt = tp[lo + 1] - tp[lo];
  const int rel = q - W * tp[lo];
  return make_int4(kind, lo, rel / nt, rel % nt);
}

__global__ void __launch_bounds__(kThreads, 1)
    layer_fused_kernel(const __grid_constant__ CUtensorMap tm_gate, const __grid_constant__ CUtensorMap tm_up,
                       const __grid_constant__ CUtensorMap tm_down, const __grid_constant__ CUtensorMap tm_x,
                       const __grid_constant__ CUtensorMap tm_h, const FusedLayerArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  uint8_t* ring = smem + kRingOff;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* empty = full + kSlots;
  uint64_t* accf = empty + kSlots;  // [2]
  uint64_t* acce = accf + 2;        // [2]
  uint64_t* tqf = acce + 2;         // [kQueue]
  uint64_t* tqe = tqf + kQueue;     // [kQueue]
  uint64_t* drain = tqe + kQueue;
  uint64_t* fin_bar = drain + 1;    // a finalize item of this CTA is done
  uint64_t* rt_bar = fin_bar + 1;   // the router rows of an item have landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kWordOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kWordOff + 4);
  volatile int* epi_go = reinterpret_cast<volatile int*>(smem + kWordOff + 8);  // epilogue group: outcome of a wait
  volatile float* fin_total = reinterpret_cast<volatile float*>(smem + kWordOff + 12);  // a token's sum of squares
  volatile int* epi_item = reinterpret_cast<volatile int*>(smem + kQueueOff + 16 * kQueue);  // int4
  int4* queue = reinterpret_cast<int4*>(smem + kQueueOff);
  float* part = reinterpret_cast<float*>(smem + kPartOff);
  float* fin_w = part + 4 * kSplit;  // [top_k] routing weights of the token being finalized
  const int E = args.E, M = args.M, K = args.top_k, H = args.H, I = args.I;
  const int nslots = M * K;
  int* offp = reinterpret_cast<int*>(smem + kIntOff);         // [E+1] padded prefix (plan rows)
  int16_t* offc = reinterpret_cast<int16_t*>(offp + E + 1);  // [E+1] compact prefix (into sl)
  int16_t* tp = offc + E + 1;                                // [E+1] prefix of token tiles
  int16_t* sl = tp + E + 1;                                  // [nslots] slot ids, expert-major, ascending
  // routed rows of expert e (its plan rows before the padding)
  auto cnt = [&](int e) -> int { return offc[e + 1] - offc[e]; };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) MOE_LT_SET(kLtStart, MOE_LT_NOW());
  unsigned* bar_word = args.sync;
  unsigned* next_work = args.sync + 1;
  unsigned* down_done = args.sync + 2;
  unsigned* up_done = args.sync + 3;  // [E]
  unsigned* fin_cnt = up_done + E;     // [M] slices of a token whose partial is written (M <= 64)
  float* fin_part = reinterpret_cast<float*>(fin_cnt + M);  // [M][8] per-slice sums of squares
  if ((smem_addr(smem_raw) & 1023u) != 0) {  // the 128-byte swizzle needs 1024-byte aligned tiles
    if (tid == 0) set_error(args.err, kErrUnsupported);
    return;
  }

  // ------------------------------------------------ 1. router logits
  // A CTA item = 8 tokens x ne experts.  Their rows are copied whole into the
  // ring with bulk copies on one mbarrier; warp w < ne then takes expert
  // e0 + w for the 8 tokens from shared memory, lane l keeping partial l
  // (chunks 32j + l, one fma per element in increasing h).
  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(rt_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  {
    const int row_bytes = H * 2;
    const int ne = min(kWarps, kSlots * kSlotBytes / row_bytes - kRtTok);  // >= 5 for H <= 8192
    const int tgroups = (M + kRtTok - 1) / kRtTok, egroups = (E + ne - 1) / ne;
    const int items = tgroups * egroups;
    const int nj = H / 256;
    int round = 0;
    for (int it = blockIdx.x; it < items; it += gridDim.x, ++round) {
      const int t0 = (it / egroups) * kRtTok, e0 = (it % egroups) * ne;
      const int nt = min(kRtTok, M - t0), nex = min(ne, E - e0);
      if (tid == 0) {
        mbar_arrive_expect_tx(rt_bar, static_cast<uint32_t>((nt + nex) * row_bytes));
        for (int r = 0; r < nt; ++r)
          bulk_load(ring + r * row_bytes, args.x + static_cast<size_t>(t0 + r) * H, row_bytes, rt_bar);
        for (int r = 0; r < nex; ++r)
          bulk_load(ring + (kRtTok + r) * row_bytes, args.w_router + static_cast<size_t>(e0 + r) * H, row_bytes,
                    rt_bar);
      }
      if (!mbar_wait_bounded(rt_bar, round & 1, nullptr)) {
        *abort_flag = 1;
        set_error(args.err, kErrTimeout);
      } else if (warp < nex) {
        const uint4* wrow = reinterpret_cast<const uint4*>(ring + (kRtTok + warp) * row_bytes) + lane;
        const uint4* xrow = reinterpret_cast<const uint4*>(ring) + lane;
        const int rv = row_bytes / 16;
        float acc[kRtTok];
#pragma unroll
        for (int t = 0; t < kRtTok; ++t) acc[t] = 0.0f;
#pragma unroll 2
        for (int j = 0; j < nj; ++j) {
          const uint4 wa = wrow[32 * j];
#pragma unroll
          for (int t = 0; t < kRtTok; ++t) {
            const uint4 xa = xrow[t * rv + 32 * j];
#pragma unroll
            for (int i = 0; i < 8; ++i)  // increasing h inside the 8-element chunk
              acc[t] = (i & 1) ? fma_bf16<true>(word(xa, i >> 1), word(wa, i >> 1), acc[t])
                               : fma_bf16<false>(word(xa, i >> 1), word(wa, i >> 1), acc[t]);
          }
        }
        const int e = e0 + warp;
        const float b = args.bias != nullptr ? args.bias[e] : 0.0f;
#pragma unroll
        for (int t = 0; t < kRtTok; ++t) {
          float v = acc[t];
#pragma unroll
          for (int off = 16; off >= 1; off >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, off));
          if (lane == 0 && t < nt) args.logits[static_cast<size_t>(t0 + t) * E + e] = __fadd_rn(v, b);
        }
      }
      __syncthreads();  // the rows may be replaced by the next item's copies
    }
  }
  // grid barrier: every logit is written (the counter was zeroed before the launch)
  if (tid == 0) {
    __threadfence();
    atomicAdd(bar_word, 1u);
    if (!wait_count(bar_word, gridDim.x, nullptr)) {
      *abort_flag = 1;
      set_error(args.err, kErrTimeout);
    }
    MOE_LT_SET(kLtBarrier, MOE_LT_NOW());
  }
  __syncthreads();
  if (*abort_flag) return;  // before any asynchronous work

  // ------------------------------------------------ 2. top-k and plan (every CTA)
  int* ids_s = reinterpret_cast<int*>(ring);  // [nslots] scratch in the ring
  int* run = ids_s + nslots;                  // [E] scratch
  int* cnt_s = run + E;                       // [E] scratch
  // Two tokens per warp at a time (t and t + kWarps), their selections
  // interleaved so that the two dependent chains overlap; each token takes
  // exactly the steps of the router's top-k kernel.
  for (int t = warp; t < M; t += 2 * kWarps) {
    const int tt[2] = {t, t + kWarps};
    float v[2][kTopkPerLane];
    bool live[2][kTopkPerLane];
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int i = 0; i < kTopkPerLane; ++i) {
        const int e = lane + 32 * i;
        live[u][i] = e < E && tt[u] < M;
        // plain L2 loads (not volatile), so that all of them are in flight at once
        const float z = live[u][i] ? __ldcg(args.logits + static_cast<size_t>(tt[u]) * E + e) : -INFINITY;
        v[u][i] = isnan(z) ? -INFINITY : z;  // a NaN logit ranks below every other (the router's rule)
      }
    float sel_v[2] = {0.0f, 0.0f};
    int sel_id[2] = {0, 0};
    for (int k = 0; k < K; ++k) {
      float bv[2] = {-INFINITY, -INFINITY};
      int bi[2] = {0x7fffffff, 0x7fffffff};
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int i = 0; i < kTopkPerLane; ++i)
          if (live[u][i] && better(v[u][i], lane + 32 * i, bv[u], bi[u])) {
            bv[u] = v[u][i];
            bi[u] = lane + 32 * i;
          }
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1)
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const float ov = __shfl_xor_sync(0xffffffffu, bv[u], off);
          const int oi = __shfl_xor_sync(0xffffffffu, bi[u], off);
          if (better(ov, oi, bv[u], bi[u])) {
            bv[u] = ov;
            bi[u] = oi;
          }
        }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
#pragma unroll
        for (int i = 0; i < kTopkPerLane; ++i)
          if (lane + 32 * i == bi[u]) live[u][i] = false;
        if (lane == k) {
          sel_v[u] = bv[u];
          sel_id[u] = bi[u];
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (tt[u] >= M) break;
      const float sv = (lane < K) ? 1.0f / (1.0f + expf(-sel_v[u])) : 0.0f;
      float total = sv;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) total += __shfl_xor_sync(0xffffffffu, total, off);
      if (lane < K) {
        ids_s[tt[u] * K + lane] = sel_id[u];
        if (blockIdx.x == 0) {
          args.topk_ids[static_cast<size_t>(tt[u]) * K + lane] = sel_id[u];
          args.topk_w[static_cast<size_t>(tt[u]) * K + lane] = sv / total;
        }
      }
    }
  }
  for (int e = tid; e < E; e += kThreads) cnt_s[e] = 0;
  __syncthreads();
  for (int f = tid; f < nslots; f += kThreads) atomicAdd(&cnt_s[ids_s[f]], 1);
  __syncthreads();
  const int B = args.block_size;
  if (warp == 0) {
    // padded prefix, compact prefix and token-tile prefix in one pass
    const int per = (E + 31) / 32;
    const int lo = min(E, lane * per), hi = min(E, lo + per);
    int sp = 0, sc = 0, st = 0;
    for (int e = lo; e < hi; ++e) {
      sp += (cnt_s[e] + B - 1) / B * B;
      sc += cnt_s[e];
      st += (cnt_s[e] + kNmax - 1) / kNmax;
    }
    int ip = sp, ic = sc, it = st;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, ip, off);
      const int b = __shfl_up_sync(0xffffffffu, ic, off);
      const int c = __shfl_up_sync(0xffffffffu, it, off);
      if (lane >= off) {
        ip += a;
        ic += b;
        it += c;
      }
    }
    int rp = ip - sp, rc = ic - sc, rt = it - st;
    for (int e = lo; e < hi; ++e) {
      offp[e] = rp;
      offc[e] = static_cast<int16_t>(rc);
      tp[e] = static_cast<int16_t>(rt);
      run[e] = rc;
      rp += (cnt_s[e] + B - 1) / B * B;
      rc += cnt_s[e];
      rt += (cnt_s[e] + kNmax - 1) / kNmax;
    }
    if (lane == 31) {
      offp[E] = ip;
      offc[E] = static_cast<int16_t>(ic);
      tp[E] = static_cast<int16_t>(it);
    }
    __syncwarp();
    // slot ids of every expert in ascending slot order (a stable counting sort)
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int base = 0; base < nslots; base += 32) {
      const int f = base + lane;
      const bool ok = f < nslots;
      const int e = ok ? ids_s[f] : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, e);
      const int r0 = ok ? run[e] : 0;
      __syncwarp();
      if (ok) {
        sl[r0 + __popc(peers & lt_mask)] = static_cast<int16_t>(f);
        if ((peers & lt_mask) == 0) run[e] = r0 + __popc(peers);
      }
      __syncwarp();
    }
  }
  if (tid == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], kEpiThreads / 32);
    }
    for (int q = 0; q < kQueue; ++q) {
      mbar_init(&tqf[q], 1);
      mbar_init(&tqe[q], 2);  // the MMA thread and the epilogue thread
    }
    mbar_init(drain, 1);
    mbar_init(fin_bar, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  fence_proxy_async_shared();  // the scratch writes above come before the ring's TMA writes
  tc_fence_before_sync();
  __syncthreads();  // the plan is complete; the ring scratch is free again
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  // the plan in the workspace: CTA 0 the header, every CTA the rows of its experts
  if (blockIdx.x == 0) {
    for (int e = tid; e <= E; e += kThreads) args.offsets[e] = offp[e];
    for (int e = tid; e < E; e += kThreads) {
      args.counts[e] = cnt(e);
      for (int b = offp[e] / B; b < offp[e + 1] / B; ++b) args.block_expert[b] = e;
    }
    if (tid == 0) *args.ntpp = offp[E];
  }
  for (int e = blockIdx.x; e < E; e += gridDim.x) {
    const int ce = cnt(e);
    const int pe = (ce + B - 1) / B * B;
    for (int r = tid; r < pe; r += kThreads)
      args.sorted_ids[offp[e] + r] = r < ce ? static_cast<int>(sl[offc[e] + r]) : nslots;
  }
  if (blockIdx.x == 0) {
    // the routing outputs are published with the finalize counter (one extra count)
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      red_release_add(down_done, 1u);
    }
  }

  const int Wu = I / kBM, Wd = H / (2 * kBM);
  const int ntiles = tp[E];
  const int n_up = Wu * ntiles, n_down = Wd * ntiles;
  // finalize items: 8 slices per token up to 64 tokens (as the few-token
  // finalize kernel's 8-CTA clusters), else one item per token
  const bool split_fin = M <= 64;
  const int n_fin = split_fin ? M * kSplit : M;
  const int n_work = n_up + n_down + n_fin;

  if (warp == 0) {
    // ------------------------------------------------ producer
    if (lane == 0) {
      MOE_LT_SET(kLtPlan, MOE_LT_NOW());
      prefetch_tensor_map(&tm_gate);
      prefetch_tensor_map(&tm_up);
      prefetch_tensor_map(&tm_down);
      prefetch_tensor_map(&tm_x);
      prefetch_tensor_map(&tm_h);
    }
    const uint64_t pol_first = l2_policy_evict_first(), pol_normal = l2_policy_evict_normal();
    int it = 0;  // ring slots issued
    int nfin = 0;  // finalize items queued by this CTA
    bool alive = true;
    for (int j = 0; alive; ++j) {
      if (nfin > 0) {
        // the previous finalize item must be done before another is claimed
        bool fd = true;
        if (lane == 0) {
          fd = mbar_wait_bounded(fin_bar, (nfin - 1) & 1, abort_flag);
          if (!fd) {
            *abort_flag = 1;
            set_error(args.err, kErrTimeout);
          }
        }
        if (!__shfl_sync(0xffffffffu, fd, 0)) break;
      }
      int q = 0;
      if (lane == 0) q = static_cast<int>(atomicAdd(next_work, 1u));
      q = __shfl_sync(0xffffffffu, q, 0);
      int4 w;
      if (q < n_up) w = decode_work(tp, E, Wu, q, kKindUp);
      else if (q < n_up + n_down) w = decode_work(tp, E, Wd, q - n_up, kKindDown);
      else if (q < n_work) {
        const int f = q - n_up - n_down;
        w = split_fin ? make_int4(kKindFin, f / kSplit, f % kSplit, 0) : make_int4(kKindFin, f, 0, 0);
      }
      else w = make_int4(kKindEnd, 0, 0, 0);
      bool ok = true;
      if (lane == 0) {
        ok = mbar_wait_bounded(&tqe[j % kQueue], ((j / kQueue) & 1) ^ 1, abort_flag);
        if (ok) {
          queue[j % kQueue] = w;
          mbar_arrive_one(&tqf[j % kQueue]);
        } else {
          *abort_flag = 1;
          set_error(args.err, kErrTimeout);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok || w.x == kKindEnd) break;
      if (w.x == kKindFin) {
        ++nfin;
        continue;
      }
      const bool up = w.x == kKindUp;
      const int e = w.y, wt = w.z, lt = w.w;
      if (!up && lane == 0) MOE_LT_FIRST(kLtFirstDown, MOE_LT_NOW());
      const int nrows = min(kNmax, cnt(e) - lt * kNmax);
      const int N = (nrows + 15) & ~15;
      const int row0 = offp[e] + lt * kNmax;
      const int c0 = offc[e] + lt * kNmax;
      const uint64_t pol = cnt(e) <= kNmax ? pol_first : pol_normal;
      // the slot's two weight boxes: gate and up rows 128w.. (up), or rows
      // 256w.. and 256w+128.. of W_down (down)
      const int a_row0 = up ? e * I + wt * kBM : e * H + wt * 2 * kBM;
      const int a_row1 = up ? a_row0 : a_row0 + kBM;
      const CUtensorMap* am0 = up ? &tm_gate : &tm_down;
      const CUtensorMap* am1 = up ? &tm_up : &tm_down;
      const int nsteps = up ? H / kBK : I / kBK;
      const uint32_t bytes = 2 * kATile + static_cast<uint32_t>(N) * kBK * 2;
      // gather4 rows of this lane (up): plan rows 4*lane .. 4*lane+3 of the tile
      int r[4] = {0, 0, 0, 0};
      if (up) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int n = 4 * lane + i;
          r[i] = n < nrows ? static_cast<int>(sl[c0 + n]) / K : 0;
        }
      }
      if (!up) {
        // the h rows of this expert come from its up tiles (other CTAs): wait
        // before the tile's first copy, so that a failed wait leaves no slot
        // half issued
        bool dep = true;
        if (lane == 0) {
          [[maybe_unused]] const unsigned long long t0 = MOE_LT_NOW();
          dep = wait_count(up_done + e, static_cast<unsigned>(Wu * (tp[e + 1] - tp[e])), abort_flag);
          MOE_LT_ADD(kLtWaitRows, MOE_LT_NOW() - t0);
          if (dep) {
            fence_proxy_async_global();
          } else {
            *abort_flag = 1;
            set_error(args.err, kErrTimeout);
          }
        }
        if (!__shfl_sync(0xffffffffu, dep, 0)) break;
      }
      for (int step = 0; step < nsteps; ++step, ++it) {
        const int s = it % kSlots;
        bool fs = true;
        if (lane == 0) {
          [[maybe_unused]] const unsigned long long t0 = MOE_LT_NOW();
          fs = mbar_wait_bounded(&empty[s], ((it / kSlots) & 1) ^ 1, abort_flag);
          MOE_LT_ADD(kLtWaitSlot, MOE_LT_NOW() - t0);
        }
        fs = __shfl_sync(0xffffffffu, fs, 0);
        if (!fs) {
          if (lane == 0) {
            *abort_flag = 1;
            set_error(args.err, kErrTimeout);
          }
          alive = false;
          break;
        }
        uint8_t* st = ring + s * kSlotBytes;
        uint8_t* bt = st + 2 * kATile;
        const int k = step;
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[s], bytes);
          tma_load_2d_hint(am0, &full[s], st, k * kBK, a_row0, pol);
          tma_load_2d_hint(am1, &full[s], st + kATile, k * kBK, a_row1, pol);
          if (!up)  // issued by the lane that acquired the h rows
            for (int b = 0; b < N / 16; ++b)
              tma_load_2d(&tm_h, &full[s], bt + b * 16 * (kBK * 2), k * kBK, row0 + 16 * b);
        }
        __syncwarp();
        if (up && 4 * lane < N)
          tma_gather4(&tm_x, &full[s], bt + lane * 4 * (kBK * 2), k * kBK, r[0], r[1], r[2], r[3]);
      }
    }
    // Do not leave while copies issued by this CTA may still land.
    if (lane == 0) {
      for (int k = max(0, it - kSlots); k < it; ++k) {
        const int s = k % kSlots;
        if (!mbar_wait_bounded(&full[s], (k / kSlots) & 1, nullptr, kWaitLimitNs / 8)) {
          set_error(args.err, kErrTimeout);
          break;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0, ti = 0;
      for (int j = 0;; ++j) {
        if (!mbar_wait_bounded(&tqf[j % kQueue], (j / kQueue) & 1, abort_flag)) {
          *abort_flag = 1;
          set_error(args.err, kErrTimeout);
          break;
        }
        const int4 w = queue[j % kQueue];
        mbar_arrive_one(&tqe[j % kQueue]);
        if (w.x == kKindEnd) break;
        if (w.x == kKindFin) continue;
        const bool up = w.x == kKindUp;
        const int e = w.y, lt = w.w;
        const int nrows = min(kNmax, cnt(e) - lt * kNmax);
        const int N = (nrows + 15) & ~15;
        const uint32_t idesc = umma_idesc_bf16(kBM, N);
        const int ab = ti & 1;
        if (!mbar_wait_bounded(&acce[ab], ((ti >> 1) & 1) ^ 1, abort_flag)) {
          *abort_flag = 1;
          set_error(args.err, kErrTimeout);
          break;
        }
        tc_fence_after_sync();
        const int nsteps = up ? H / kBK : I / kBK;
        bool ok = true;
        for (int step = 0; step < nsteps; ++step, ++it) {
          const int s = it % kSlots;
          if (!mbar_wait_bounded(&full[s], (it / kSlots) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          uint8_t* st = ring + s * kSlotBytes;
          const uint64_t da0 = umma_desc_sw128(st);
          const uint64_t da1 = umma_desc_sw128(st + kATile);
          const uint64_t db = umma_desc_sw128(st + 2 * kATile);
          const uint32_t d = tmem + ab * kAccCols;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint32_t acc = (step | kk) != 0 ? 1u : 0u;
            umma_bf16_ss(d, da0 + 2 * kk, db + 2 * kk, idesc, acc);
            umma_bf16_ss(d + kNmax, da1 + 2 * kk, db + 2 * kk, idesc, acc);
          }
          umma_commit(&empty[s]);
        }
        if (!ok) {
          *abort_flag = 1;
          set_error(args.err, kErrTimeout);
          break;
        }
        umma_commit(&accf[ab]);
        ++ti;
      }
      // every MMA of this CTA has completed before tensor memory is released
      umma_commit(drain);
      if (!mbar_wait_bounded(drain, 0, nullptr, kWaitLimitNs / 8)) set_error(args.err, kErrTimeout);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ epilogue + finalize
    const int et = tid - kEpiWarp0 * 32;  // 0..127
    const int quarter = warp & 3;         // tensor-memory lanes 32*quarter ..
    int ti = 0;
    for (int j = 0;; ++j) {
      // One thread takes every wait of the group and passes the outcome on
      // through shared memory, so that the four warps always leave together
      // (a named barrier has no time limit).
      if (et == 0) {
        int4 w = make_int4(kKindEnd, 0, 0, 0);
        if (mbar_wait_bounded(&tqf[j % kQueue], (j / kQueue) & 1, abort_flag)) {
          w = queue[j % kQueue];
          mbar_arrive_one(&tqe[j % kQueue]);
        } else {
          *abort_flag = 1;
          set_error(args.err, kErrTimeout);
        }
        epi_item[0] = w.x;
        epi_item[1] = w.y;
        epi_item[2] = w.z;
        epi_item[3] = w.w;
      }
      epi_sync();
      const int4 w = make_int4(epi_item[0], epi_item[1], epi_item[2], epi_item[3]);
      if (w.x == kKindEnd) break;
      if (w.x == kKindFin) {
        // ---- finalize: a slice of token t (up to 64 tokens) or all of it,
        // in the reduction order of the finalize kernel the separate launches
        // use for this many tokens
        const int t = w.y;
        if (et == 0) {
          const bool ready = wait_count(down_done, static_cast<unsigned>(n_down + 1), abort_flag);
          if (!ready) {
            *abort_flag = 1;
            set_error(args.err, kErrTimeout);
          }
          MOE_LT_FIRST(kLtFinStart, MOE_LT_NOW());
          *epi_go = ready ? 1 : 0;
        }
        epi_sync();
        if (!*epi_go) break;
        if (et < K) fin_w[et] = ld_cg_f32(args.topk_w + static_cast<size_t>(t) * K + et);
        epi_sync();
        const int npk = H / 8;
        const uint16_t* xt = args.x + static_cast<size_t>(t) * H;
        const uint16_t* yt = args.y + static_cast<size_t>(t) * K * H;
        if (split_fin) {
          // Slice w.z of 8: pack slice*per + et (the few-token kernel's CTA
          // `slice` of the token's cluster).  Its sum of squares goes to the
          // workspace; the 8 partials are added in slice order by every slice.
          const int slice = w.z;
          const int per = (npk + kSplit - 1) / kSplit;
          const int p = slice * per + et;
          const bool live = et < per && p < npk;
          float a[8];
          if (live) {
            unpack8(__ldg(reinterpret_cast<const uint4*>(xt + p * 8)), a);
          } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) a[j] = 0.0f;
          }
          for (int k0 = 0; k0 < K; k0 += 16) {
            uint4 v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              v[i] = (live && k0 + i < K)
                         ? __ldcg(reinterpret_cast<const uint4*>(yt + static_cast<size_t>(k0 + i) * H + p * 8))
                         : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              if (k0 + i >= K) break;
              const float wk = fin_w[k0 + i];
              float f[8];
              unpack8(v[i], f);
#pragma unroll
              for (int j = 0; j < 8; ++j) a[j] = fmaf(wk, f[j], a[j]);
            }
          }
          float ss = 0.0f;
#pragma unroll
          for (int j = 0; j < 8; ++j) ss = fmaf(a[j], a[j], ss);
#pragma unroll
          for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
          if (lane == 0) part[et >> 5] = ss;
          epi_sync();
          if (et == 0) {
            float c = 0.0f;
#pragma unroll
            for (int wq = 0; wq < 4; ++wq) c += part[wq];
            fin_part[t * kSplit + slice] = c;
            __threadfence();
            red_release_add(fin_cnt + t, 1u);
            const bool all = wait_count(fin_cnt + t, kSplit, abort_flag);
            float total = 0.0f;
            if (all) {
              float pr[kSplit];  // all 8 loads in flight, then added in slice order
#pragma unroll
              for (int r = 0; r < kSplit; ++r) pr[r] = __ldcg(fin_part + t * kSplit + r);
#pragma unroll
              for (int r = 0; r < kSplit; ++r) total += pr[r];
            } else {
              *abort_flag = 1;
              set_error(args.err, kErrTimeout);
            }
            *fin_total = total;
            *epi_go = all ? 1 : 0;
          }
          epi_sync();
          if (!*epi_go) break;
          const float inv = 1.0f / sqrtf(*fin_total / static_cast<float>(H) + args.eps);
          if (live) {
            float g[8];
            unpack8(__ldg(reinterpret_cast<const uint4*>(args.gamma + p * 8)), g);
            uint4 o;
            o.x = pack_bf16x2(a[0] * inv * g[0], a[1] * inv * g[1]);
            o.y = pack_bf16x2(a[2] * inv * g[2], a[3] * inv * g[3]);
            o.z = pack_bf16x2(a[4] * inv * g[4], a[5] * inv * g[5]);
            o.w = pack_bf16x2(a[6] * inv * g[6], a[7] * inv * g[7]);
            *reinterpret_cast<uint4*>(args.out + static_cast<size_t>(t) * H + p * 8) = o;
            if (args.residual_out != nullptr) {
              uint4 r;
              r.x = pack_bf16x2(a[0], a[1]);
              r.y = pack_bf16x2(a[2], a[3]);
              r.z = pack_bf16x2(a[4], a[5]);
              r.w = pack_bf16x2(a[6], a[7]);
              *reinterpret_cast<uint4*>(args.residual_out + static_cast<size_t>(t) * H + p * 8) = r;
            }
          }
          if (et == 0) {
            MOE_LT_SET(kLtFinEnd, MOE_LT_NOW());
            mbar_arrive_one(fin_bar);
          }
          continue;
        }
        // The whole token: the many-token kernel's 256-thread CTA, virtual
        // thread et + 128*(q/4) owning packs vt + 256*(q%4).
        float acc[kSplit][8];
        auto pack_of = [&](int q) -> int { return et + 128 * (q >> 2) + 256 * (q & 3); };
#pragma unroll
        for (int q = 0; q < kSplit; ++q) {
          const int p = pack_of(q);
          if (p < npk) {
            unpack8(__ldg(reinterpret_cast<const uint4*>(xt + p * 8)), acc[q]);
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[q][i] = 0.0f;
          }
        }
        // 4 expert rows x 8 packs = 32 loads in flight a thread; each element
        // still takes its K terms in increasing k
        for (int k0 = 0; k0 < K; k0 += 4) {
          uint4 v[4][kSplit];
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int q = 0; q < kSplit; ++q) {
              const int p = pack_of(q);
              v[i][q] = (k0 + i < K && p < npk)
                            ? __ldcg(reinterpret_cast<const uint4*>(yt + static_cast<size_t>(k0 + i) * H + p * 8))
                            : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (k0 + i >= K) break;
            const float wk = fin_w[k0 + i];
#pragma unroll
            for (int q = 0; q < kSplit; ++q) {
              float f[8];
              unpack8(v[i][q], f);
#pragma unroll
              for (int j = 0; j < 8; ++j) acc[q][j] = fmaf(wk, f[j], acc[q][j]);
            }
          }
        }
        // per virtual thread: its packs in order; butterfly per virtual warp;
        // the 8 virtual warps in order
#pragma unroll
        for (int hv = 0; hv < 2; ++hv) {
          float ss = 0.0f;
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) ss = fmaf(acc[4 * hv + i][j], acc[4 * hv + i][j], ss);
#pragma unroll
          for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
          if (lane == 0) part[4 * hv + (et >> 5)] = ss;
        }
        epi_sync();
        float total = 0.0f;
#pragma unroll
        for (int wq = 0; wq < 8; ++wq) total += part[wq];
        epi_sync();  // part[] may be reused by the next item
        const float inv = 1.0f / sqrtf(total / static_cast<float>(H) + args.eps);
#pragma unroll
        for (int q = 0; q < kSplit; ++q) {
          const int p = pack_of(q);
          if (p >= npk) continue;
          float g[8];
          unpack8(__ldg(reinterpret_cast<const uint4*>(args.gamma + p * 8)), g);
          uint4 o;
          o.x = pack_bf16x2(acc[q][0] * inv * g[0], acc[q][1] * inv * g[1]);
          o.y = pack_bf16x2(acc[q][2] * inv * g[2], acc[q][3] * inv * g[3]);
          o.z = pack_bf16x2(acc[q][4] * inv * g[4], acc[q][5] * inv * g[5]);
          o.w = pack_bf16x2(acc[q][6] * inv * g[6], acc[q][7] * inv * g[7]);
          *reinterpret_cast<uint4*>(args.out + static_cast<size_t>(t) * H + p * 8) = o;
          if (args.residual_out != nullptr) {
            uint4 r;
            r.x = pack_bf16x2(acc[q][0], acc[q][1]);
            r.y = pack_bf16x2(acc[q][2], acc[q][3]);
            r.z = pack_bf16x2(acc[q][4], acc[q][5]);
            r.w = pack_bf16x2(acc[q][6], acc[q][7]);
            *reinterpret_cast<uint4*>(args.residual_out + static_cast<size_t>(t) * H + p * 8) = r;
          }
        }
        if (et == 0) {
          MOE_LT_SET(kLtFinEnd, MOE_LT_NOW());
          mbar_arrive_one(fin_bar);  // fin_w and part[] are free again (last epi_sync above)
        }
        continue;
      }
      // ---- a projection tile
      const bool up = w.x == kKindUp;
      const int e = w.y, wt = w.z, lt = w.w;
      const int nrows = min(kNmax, cnt(e) - lt * kNmax);
      const int N = (nrows + 15) & ~15;
      const int ab = ti & 1;
      if (et == 0) {
        const bool got = mbar_wait_bounded(&accf[ab], (ti >> 1) & 1, abort_flag);
        if (!got) {
          *abort_flag = 1;
          set_error(args.err, kErrTimeout);
        }
        *epi_go = got ? 1 : 0;
      }
      epi_sync();
      if (!*epi_go) break;
      tc_fence_after_sync();
      const uint32_t lane_base = tmem + ab * kAccCols + (static_cast<uint32_t>(quarter * 32) << 16);
      if (up) {
        const int col = wt * kBM + quarter * 32 + lane;  // I index
        const int row0 = offp[e] + lt * kNmax;
        for (int c = 0; c < N; c += 16) {
          uint32_t d0[16], d1[16];
          tmem_load_16(lane_base + c, d0);
          tmem_load_16(lane_base + kNmax + c, d1);
          tmem_load_wait();
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const int n = c + q;
            if (n < nrows) {
              const float g = __uint_as_float(d0[q]);
              const float u = __uint_as_float(d1[q]);
              const float hv = g / (1.0f + expf(-g)) * u;
              reinterpret_cast<__nv_bfloat16*>(args.h)[static_cast<size_t>(row0 + n) * I + col] =
                  __float2bfloat16_rn(hv);
            }
          }
        }
      } else {
        const int col = wt * 2 * kBM + quarter * 32 + lane;  // H index of the first row block
        const int c0 = offc[e] + lt * kNmax;
        for (int c = 0; c < N; c += 16) {
          uint32_t d0[16], d1[16];
          tmem_load_16(lane_base + c, d0);
          tmem_load_16(lane_base + kNmax + c, d1);
          tmem_load_wait();
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const int n = c + q;
            if (n < nrows) {
              __nv_bfloat16* yr = reinterpret_cast<__nv_bfloat16*>(args.y) + static_cast<size_t>(sl[c0 + n]) * H;
              yr[col] = __float2bfloat16_rn(__uint_as_float(d0[q]));
              yr[col + kBM] = __float2bfloat16_rn(__uint_as_float(d1[q]));
            }
          }
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_one(&acce[ab]);
      // publish the tile: h is read by TMA (the async proxy) in other CTAs
      fence_proxy_async_global();
      epi_sync();
      if (et == 0) {
        __threadfence();
        red_release_add(up ? up_done + e : down_done, 1u);
        MOE_LT_SET(up ? kLtLastUpPub : kLtLastDownPub, MOE_LT_NOW());
        MOE_LT_ADD(up ? kLtUpTiles : kLtDownTiles, 1ull);
      }
      ++ti;
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
  if (tid == 0) MOE_LT_SET(kLtEnd, MOE_LT_NOW());
}

}  // namespace

int layer_fused_smem_bytes(int E, int nslots) { return fused_smem_bytes(E, nslots); }

cudaError_t launch_layer_fused(const CUtensorMap& w_gate, const CUtensorMap& w_up, const CUtensorMap& w_down,
                               const CUtensorMap& x_rows, const CUtensorMap& h_rows, const FusedLayerArgs& args,
                               int num_sms, cudaStream_t stream) {
  if (args.E > 32 * kTopkPerLane || args.top_k > 32 || args.M * args.top_k > kRouteMaxSlots || args.H % 256 != 0 ||
      args.H / 8 > kSplit * kEpiThreads || args.I % kBM != 0 || args.block_size % 16 != 0)
    return cudaErrorInvalidValue;
  const int smem = fused_smem_bytes(args.E, args.M * args.top_k);
  if ((args.M * args.top_k + 2 * args.E) * 4 > kSlots * kSlotBytes) return cudaErrorInvalidValue;  // plan scratch
  int dev = 0;
  cudaError_t st = cudaGetDevice(&dev);
  if (st != cudaSuccess) return st;
  static int attr_bytes[64] = {};
  if (dev < 64 && attr_bytes[dev] < smem) {
    st = cudaFuncSetAttribute(layer_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (st != cudaSuccess) return st;
    attr_bytes[dev] = smem;
  }
  int per_sm = 0;
  st = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, layer_fused_kernel, kThreads, smem);
  if (st != cudaSuccess) return st;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms));  // one CTA per SM
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // all CTAs resident: the grid barrier and the waits need it
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, layer_fused_kernel, w_gate, w_up, w_down, x_rows, h_rows, args);
}

}  // namespace moe

#ifdef MOE_LAYER_TRACE
// Host access to the phase timeline of the last single-launch layers (timeline build only).
extern "C" __attribute__((visibility("default"))) int moe_layer_trace_read(void* host, size_t bytes) {
  return cudaMemcpyFromSymbol(host, moe::g_layer_trace, bytes) == cudaSuccess ? 0 : 1;
}
extern "C" __attribute__((visibility("default"))) int moe_layer_trace_clear() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, moe::g_layer_trace) != cudaSuccess) return 1;
  return cudaMemset(p, 0, sizeof(moe::g_layer_trace)) == cudaSuccess ? 0 : 1;
}
#endif
