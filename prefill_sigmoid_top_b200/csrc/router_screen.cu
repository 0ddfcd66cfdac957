// Screened sigmoid top-k routing for many tokens ("[sglang] [NPU] GLM-4.7-Flash 성능 최적화", sglang PR
// #29509 analysis, §2 "MoE TopK Scoring Function": sigmoid scores of z = x . w_router + bias).
//
// Same ids and weights as the plain router (router.cu), bit for bit: the selection runs on the
// canonical fp32 logits, but those are computed only for the experts that can be selected.
//
//  1. screen_quantize_kernel: every row v of x [M,H] and of w_router [E,H] becomes integers
//     X_h = rint(v_h / s) with a power of two s = 2^(e - 13) (v's largest magnitude is f * 2^e,
//     f in [0.5, 1); bf16 has 8 significant bits, so |X| <= 8160), stored as two signed 8-bit digits
//     X = 128 hi + lo, lo in [-64, 63], hi in [-64, 64], with the row's bounds from exact integer sums:
//     eps = max |v - s X| (<= s/2), sum |v| <= s sum |X| + H eps, ||v||_2 <= s ||X||_2 + sqrt(H) eps,
//     and whether v is finite.
//  2. screen_gemm_kernel (tcgen05 kind::i8, int32 accumulators): for 128 tokens x 128 experts and a
//     slice of H, HH = sum hi hi, HL = sum (hi_x lo_w + lo_x hi_w), LL = sum lo lo, exactly; their
//     combination P = 16384 HH + 128 HL + LL = sum X_x X_w is an integer below 2^53, stored as fp64
//     per slice of H.
//  3. screen_route_kernel, one 4-warp CTA per token:
//     - P = sum over the slices (exact), za = s_x s_w P + b, and a bound d >= |z - za| on the canonical
//       fp32 logit z, from  |x.w - s_x s_w P| <= eps_x s_w sum|X_w| + eps_w sum|x|  and the error of the
//       canonical fp32 sum,  |z - (x.w + b)| <= g_n (||x|| ||w|| + |b|) + n 2^-149  (n = H/32 + 6 roundings
//       of a sum of products of bf16 values, the last term for underflow; sum |x_h w_h| <= ||x|| ||w||),
//       plus margins for the fp64 arithmetic of the bound itself (valid while ||x|| ||w|| + |b| < 2^120,
//       so that no fp32 sum of the canonical order overflows; otherwise the pair is a candidate);
//     - with A the K experts of largest za and L = min over A of (za - d), an expert whose za + d < L
//       has z < L <= z of each of the K experts of A, so it cannot be selected: the others (at least the
//       K of A) are the candidates; a row that is not finite makes all its pairs candidates;
//     - the canonical fp32 logit of every candidate, with the plain router's per-lane fma sequence, xor
//       butterfly and bias add (router_dot.cuh), the others -inf;
//     - the plain router's per-token top-k and weights on those logits (router_select.cuh): the K
//       largest are candidates with their canonical values, so ids and weights are the plain router's.
#include <cmath>
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "router_dot.cuh"
#include "router_select.cuh"

namespace moe {
namespace {

constexpr int kSBM = 128;                       // tokens per GEMM tile (MMA M)
constexpr int kSBN = 128;                       // experts per GEMM tile (MMA N)
constexpr int kSChunk = 128;                    // int8 elements of H per stage (one 128-byte row)
constexpr int kSStages = 3;
constexpr int kSXBox = kSBM * kSChunk;          // x digit box: 16 KB
constexpr int kSWBox = kSBN * kSChunk;          // w digit box: 16 KB
constexpr int kSStageBytes = 2 * kSXBox + 2 * kSWBox;
constexpr int kSSmem = 1024 + kSStages * kSStageBytes + 256;
constexpr int kSThreads = 192;                  // warps: 0 producer, 1 MMA issuer, 2-5 producers then epilogue
constexpr int kSTargetCtas = 148;               // one wave on the B200's 148 SMs
constexpr uint32_t kSTmemCols = 512;            // HH, HL, LL accumulators of 128 columns

struct RowStats {
  double s, eps, n1, n2, nhat1, finite, pad0, pad1;
};
static_assert(sizeof(RowStats) == 64, "row stats");

// ---------------------------------------------------------------------------- 1. digits and bounds
constexpr int kQThreads = 128;                  // one CTA per row
constexpr int kQPer = 8;                        // 16-byte chunks per thread (H <= 8192)

__global__ void __launch_bounds__(kQThreads) screen_quantize_kernel(const uint16_t* __restrict__ x,
                                                                    const uint16_t* __restrict__ w, int M, int E,
                                                                    int H, int8_t* __restrict__ hi,
                                                                    int8_t* __restrict__ lo,
                                                                    RowStats* __restrict__ stats) {
  __shared__ float red_f[kQThreads / 32];
  __shared__ int red_i[kQThreads / 32];
  __shared__ long long red_l[kQThreads / 32];
  const int row = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint16_t* src = row < M ? x + static_cast<size_t>(row) * H : w + static_cast<size_t>(row - M) * H;
  const int nc = H / 8;
  uint4 v[kQPer];  // chunks tid, tid + 128, ... of the row, read once
  float m = 0.0f;
  bool fin = true;
#pragma unroll
  for (int k = 0; k < kQPer; ++k) {
    const int c = tid + kQThreads * k;
    v[k] = c < nc ? *reinterpret_cast<const uint4*>(src + c * 8) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int k = 0; k < kQPer; ++k) {
    const uint32_t wd[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float a = bf16_lo(wd[i]), b = bf16_hi(wd[i]);
      fin = fin && isfinite(a) && isfinite(b);
      m = fmaxf(m, fmaxf(fabsf(a), fabsf(b)));
    }
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  const int wfin = __all_sync(0xffffffffu, fin) ? 1 : 0;
  if (lane == 0) {
    red_f[warp] = m;
    red_i[warp] = wfin;
  }
  __syncthreads();
  m = 0.0f;
  fin = true;
#pragma unroll
  for (int q = 0; q < kQThreads / 32; ++q) {
    m = fmaxf(m, red_f[q]);
    fin = fin && red_i[q] != 0;
  }
  __syncthreads();  // red_* are reused below
  int ex = 0;
  frexpf(m, &ex);  // m = f * 2^ex, f in [0.5, 1) (m = 0: ex = 0)
  // s = 2^(ex - 13) as a float needs ex - 13 >= -149 and 1/s needs 13 - ex <= 127; a row that misses
  // either (subnormals only) or is not finite gets no digits: eps = its largest magnitude
  const bool scaled = fin && ex - 13 >= -149 && 13 - ex <= 127;
  const float s = scaled ? ldexpf(1.0f, ex - 13) : 1.0f;
  const float inv_s = scaled ? ldexpf(1.0f, 13 - ex) : 0.0f;
  float eps = 0.0f;
  int nh = 0;
  long long nx2 = 0;
  int8_t* hrow = hi + static_cast<size_t>(row) * H;
  int8_t* lrow = lo + static_cast<size_t>(row) * H;
#pragma unroll
  for (int k = 0; k < kQPer; ++k) {
    const int c = tid + kQThreads * k;
    if (c >= nc) break;
    const uint32_t wd[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
    uint32_t hpk[2] = {0u, 0u}, lpk[2] = {0u, 0u};
    int sq = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float f = (i & 1) ? bf16_hi(wd[i >> 1]) : bf16_lo(wd[i >> 1]);
      float q = rintf(f * inv_s);              // exact scaling by a power of two
      if (!(fabsf(q) <= 8160.0f)) q = 0.0f;    // only rows that are not finite
      const int X = static_cast<int>(q);
      const int h = (X + 64) >> 7;             // floor((X + 64) / 128)
      const int l = X - 128 * h;               // [-64, 63]
      hpk[i >> 2] |= (static_cast<uint32_t>(h) & 0xFFu) << (8 * (i & 3));
      lpk[i >> 2] |= (static_cast<uint32_t>(l) & 0xFFu) << (8 * (i & 3));
      eps = fmaxf(eps, fabsf(f - s * q));      // exact: f and s q are within a factor 2 (or q = 0)
      nh += X < 0 ? -X : X;
      sq += X * X;                             // 8 squares of |X| <= 8160: below 2^31
    }
    nx2 += sq;
    *reinterpret_cast<uint2*>(hrow + c * 8) = make_uint2(hpk[0], hpk[1]);
    *reinterpret_cast<uint2*>(lrow + c * 8) = make_uint2(lpk[0], lpk[1]);
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    eps = fmaxf(eps, __shfl_xor_sync(0xffffffffu, eps, off));
    nh += __shfl_xor_sync(0xffffffffu, nh, off);
    nx2 += __shfl_xor_sync(0xffffffffu, nx2, off);
  }
  if (lane == 0) {
    red_f[warp] = eps;
    red_i[warp] = nh;
    red_l[warp] = nx2;
  }
  __syncthreads();
  if (tid == 0) {
    eps = 0.0f;
    nh = 0;
    nx2 = 0;
#pragma unroll
    for (int q = 0; q < kQThreads / 32; ++q) {
      eps = fmaxf(eps, red_f[q]);
      nh += red_i[q];
      nx2 += red_l[q];
    }
    RowStats st;
    const double sd = s, ed = eps;
    st.s = sd;
    st.eps = ed;
    st.nhat1 = sd * nh;                                                          // exact
    st.n1 = (sd * nh + static_cast<double>(H) * ed) * (1.0 + 1e-12);             // >= sum |v|
    st.n2 = (sd * sqrt(static_cast<double>(nx2)) + sqrt(static_cast<double>(H)) * ed) * (1.0 + 1e-12);
    st.finite = fin ? 1.0 : 0.0;
    st.pad0 = st.pad1 = 0.0;
    stats[row] = st;
  }
}

// ---------------------------------------------------------------------------- 2. integer partial logits
// Instruction descriptor of kind::i8 with signed 8-bit A and B, int32 accumulator, both K-major:
// D format (2 = s32) at bits [4,6), A format (1 = signed) at [7,10), B format at [10,13),
// N >> 3 at [17,23), M >> 4 at [24,29).
__host__ __device__ constexpr uint32_t umma_idesc_s8(uint32_t M, uint32_t N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

__device__ __forceinline__ void umma_s8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

struct ScreenGemmArgs {
  double* partial;  // [slices][M][E]
  int32_t* err;
  int M, E, chunks_per_slice;
};

// Byte offset of box b in a stage (0: x hi, 1: x lo, 2: w hi, 3: w lo); every box starts 1024-aligned.
__device__ __forceinline__ int box_offset(int b) { return b < 2 ? b * kSXBox : 2 * kSXBox + (b - 2) * kSWBox; }

__global__ void __launch_bounds__(kSThreads, 1)
    screen_gemm_kernel(const __grid_constant__ CUtensorMap tm_xh, const __grid_constant__ CUtensorMap tm_xl,
                       const __grid_constant__ CUtensorMap tm_wh, const __grid_constant__ CUtensorMap tm_wl,
                       const ScreenGemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + kSStages * kSStageBytes);
  uint64_t* empty = full + kSStages;
  uint64_t* acc_full = empty + kSStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kSBM, e0 = blockIdx.y * kSBN;
  const int c_begin = blockIdx.z * a.chunks_per_slice, nchunks = a.chunks_per_slice;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kSStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == 1) {
    tmem_alloc(tmem_slot, kSTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  // ---- producers: box b of every stage from its own warp (0, 2, 3, 4: a thread's copies are served one
  // after another, so four issuers keep four in flight); warp 0 posts the stage's bytes (a copy that
  // lands before the post leaves the phase open: the post's arrival is still pending)
  const int box = warp == 0 ? 0 : (warp >= 2 && warp <= 4 ? warp - 1 : -1);
  if (box >= 0 && lane == 0) {
    const CUtensorMap* map = box == 0 ? &tm_xh : box == 1 ? &tm_xl : box == 2 ? &tm_wh : &tm_wl;
    const int row = box < 2 ? t0 : e0;
    prefetch_tensor_map(map);
    int issued = 0;
    for (int i = 0; i < nchunks; ++i) {
      const int s = i % kSStages;
      if (!mbar_wait_bounded(&empty[s], ((i / kSStages) & 1) ^ 1, abort_flag)) {
        *abort_flag = 1;
        set_error(a.err, kErrTimeout);
        break;
      }
      if (box == 0) mbar_arrive_expect_tx(&full[s], kSStageBytes);
      tma_load_2d(map, &full[s], ring + s * kSStageBytes + box_offset(box), (c_begin + i) * kSChunk, row);
      issued = i + 1;
    }
    // Do not go on while copies issued here may still land (after an abort the MMA issuer stops
    // consuming): wait, bounded, for the last stages.
    for (int i = issued > kSStages ? issued - kSStages : 0; i < issued; ++i)
      if (!mbar_wait_bounded(&full[i % kSStages], (i / kSStages) & 1, nullptr, kWaitLimitNs / 8)) {
        set_error(a.err, kErrTimeout);
        break;
      }
  }
  __syncwarp();

  if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_s8(kSBM, kSBN);
      const uint32_t d_hh = tmem, d_hl = tmem + kSBN, d_ll = tmem + 2 * kSBN;
      for (int i = 0; i < nchunks; ++i) {
        const int s = i % kSStages;
        if (!mbar_wait_bounded(&full[s], (i / kSStages) & 1, abort_flag)) {
          *abort_flag = 1;
          set_error(a.err, kErrTimeout);
          break;
        }
        tc_fence_after_sync();
        const uint8_t* st = ring + s * kSStageBytes;
        const uint64_t dxh = umma_desc_sw128(st + box_offset(0)), dxl = umma_desc_sw128(st + box_offset(1));
        const uint64_t dwh = umma_desc_sw128(st + box_offset(2)), dwl = umma_desc_sw128(st + box_offset(3));
#pragma unroll
        for (int kk = 0; kk < kSChunk / 32; ++kk) {  // 32 int8 elements (32 bytes) per MMA
          const uint32_t acc = (i | kk) != 0 ? 1u : 0u;
          umma_s8_ss(d_hh, dxh + 2 * kk, dwh + 2 * kk, idesc, acc);
          umma_s8_ss(d_hl, dxh + 2 * kk, dwl + 2 * kk, idesc, acc);
          umma_s8_ss(d_hl, dxl + 2 * kk, dwh + 2 * kk, idesc, 1u);
          umma_s8_ss(d_ll, dxl + 2 * kk, dwl + 2 * kk, idesc, acc);
        }
        umma_commit(&empty[s]);
      }
      umma_commit(acc_full);  // also after an abort, so that the epilogue is not left waiting
    }
    __syncwarp();
  } else if (warp >= 2) {
    // epilogue: warp w reads tensor-memory lanes 32 (w % 4) .. + 31 = tokens of the tile
    const int q = warp & 3;
    bool ok = true;
    if (lane == 0) ok = mbar_wait_bounded(acc_full, 0, abort_flag);
    ok = __shfl_sync(0xffffffffu, ok, 0) && !*abort_flag;
    tc_fence_after_sync();
    if (!ok) {
      if (lane == 0) set_error(a.err, kErrTimeout);
    } else {
      // lane = token of this warp's 32; each 16-column block goes through shared memory (the ring is
      // idle once the accumulators are complete) so that the stores are 128-byte runs of one token's row
      const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
      double* stage = reinterpret_cast<double*>(ring) + (warp - 2) * 32 * 17;  // [32 tokens][16 + 1]
      const int half = lane >> 4, col = lane & 15;
#pragma unroll 1
      for (int cb = 0; cb < kSBN; cb += 16) {
        uint32_t hh[16], hl[16], ll[16];
        tmem_load_16(lane_base + cb, hh);
        tmem_load_16(lane_base + kSBN + cb, hl);
        tmem_load_16(lane_base + 2 * kSBN + cb, ll);
        tmem_load_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j)  // exact: an integer below 2^53
          stage[lane * 17 + j] = 16384.0 * static_cast<int32_t>(hh[j]) + 128.0 * static_cast<int32_t>(hl[j]) +
                                 static_cast<double>(static_cast<int32_t>(ll[j]));
        __syncwarp();
        const int e = e0 + cb + col;
#pragma unroll 4
        for (int r = half; r < 32; r += 2) {  // two tokens' 16 columns per store instruction
          const int t = t0 + q * 32 + r;
          if (t < a.M && e < a.E)
            a.partial[(static_cast<size_t>(blockIdx.z) * a.M + t) * a.E + e] = stage[r * 17 + col];
        }
        __syncwarp();
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kSTmemCols);
}

// ---------------------------------------------------------------------------- 3. one CTA per token
template <int kPer>
__global__ void __launch_bounds__(128) screen_route_kernel(const uint16_t* __restrict__ x,
                                                           const uint16_t* __restrict__ w_router,
                                                           const float* __restrict__ bias,
                                                           const double* __restrict__ partial, int slices,
                                                           const RowStats* __restrict__ stats, int M, int E, int K,
                                                           int H, int32_t* __restrict__ topk_ids,
                                                           float* __restrict__ topk_w) {
  constexpr int kWarps = 4;
  extern __shared__ __align__(16) uint8_t sm[];
  uint16_t* xs = reinterpret_cast<uint16_t*>(sm);                          // [H] the token's row
  float* zs = reinterpret_cast<float*>(sm + static_cast<size_t>(H) * 2);  // [E] canonical logits or -inf
  int* cs = reinterpret_cast<int*>(zs + E);                                // [E] candidates
  __shared__ int ncand_s;
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint16_t* xt = x + static_cast<size_t>(t) * H;
  for (int c = threadIdx.x; c < H / 8; c += 32 * kWarps)
    reinterpret_cast<uint4*>(xs)[c] = reinterpret_cast<const uint4*>(xt)[c];

  if (warp == 0) {
    // ---- bounds and candidates.  The bound is formed in fp64, then kept as fp32 rounded outward (the
    // lower end down, the upper end up), so that every comparison below stays on the safe side.
    const RowStats xst = stats[t];
    const double n = static_cast<double>(H / 32 + 6), u = 0x1p-24;
    const double gam = n * u / (1.0 - n * u);
    const double under = (n + 8.0) * 0x1p-149;  // absolute error of fp32 sums near underflow
    double p[kPer];  // exact sums of integers below 2^53, all loads of a slice in flight together
#pragma unroll
    for (int i = 0; i < kPer; ++i) p[i] = 0.0;
#pragma unroll 4
    for (int sl = 0; sl < slices; ++sl) {
      const double* ps = partial + (static_cast<size_t>(sl) * M + t) * E + lane;
#pragma unroll
      for (int i = 0; i < kPer; ++i)
        if (lane + 32 * i < E) p[i] += ps[32 * i];
    }
    float za[kPer], lo[kPer], hi[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = lane + 32 * i;
      za[i] = -INFINITY;
      lo[i] = -INFINITY;
      hi[i] = INFINITY;
      if (e >= E) continue;
      const RowStats ws = stats[M + e];
      const double b = bias != nullptr ? static_cast<double>(bias[e]) : 0.0;
      // the bound below holds while no fp32 sum of the canonical order can overflow: every partial sum is
      // at most sum |x_h w_h| + |b| <= ||x|| ||w|| + |b| (times 1 + g_n), far below 2^128 under 2^120
      if (xst.finite != 0.0 && ws.finite != 0.0 && isfinite(b) && xst.n2 * ws.n2 + fabs(b) < 0x1p120) {
        const double z = xst.s * ws.s * p[i] + b;
        double d = xst.eps * ws.nhat1 + ws.eps * xst.n1 + gam * (xst.n2 * ws.n2 + fabs(b)) + under;
        d = d * (1.0 + 1e-9) + fabs(z) * 0x1p-50;
        za[i] = __double2float_rn(z);
        lo[i] = __double2float_rd(z - d);
        hi[i] = __double2float_ru(z + d);
      }
    }
    // the K largest approximate logits and the least lower bound among them
    unsigned picked = 0u;  // bit i: expert lane + 32 i taken
    float L = INFINITY;
    for (int k = 0; k < K; ++k) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        if (e < E && !((picked >> i) & 1u) && (bi == 0x7fffffff || za[i] > bv)) {
          bv = za[i];
          bi = e;
        }
      }
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
        if (oi != 0x7fffffff && (bi == 0x7fffffff || ov > bv || (ov == bv && oi < bi))) {
          bv = ov;
          bi = oi;
        }
      }
#pragma unroll
      for (int i = 0; i < kPer; ++i)
        if (lane + 32 * i == bi) {
          picked |= 1u << i;
          L = fminf(L, lo[i]);
        }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) L = fminf(L, __shfl_xor_sync(0xffffffffu, L, off));
    int base = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      const int e = lane + 32 * i;
      const bool c = e < E && (((picked >> i) & 1u) || hi[i] >= L);
      const unsigned mask = __ballot_sync(0xffffffffu, c);
      if (c) cs[base + __popc(mask & ((1u << lane) - 1u))] = e;
      else if (e < E) zs[e] = -INFINITY;
      base += __popc(mask);
    }
    if (lane == 0) ncand_s = base;
  }
  __syncthreads();

  // ---- canonical logits of the candidates: lane l's partial over h = 256 j + 8 l + i, in increasing h,
  // one fma each; the xor butterfly; the bias.  A warp takes two candidates at a time (its loads of both
  // in flight together); with an odd count the second of the last pair repeats the first.
  const int nc = ncand_s;
  const int nj = H / 256;
  const uint16_t* xl = xs + 8 * lane;
  for (int c = 2 * warp; c < nc; c += 2 * kWarps) {
    const int ea = cs[c], eb = cs[c + 1 < nc ? c + 1 : c];
    const uint16_t* wa = w_router + static_cast<size_t>(ea) * H + 8 * lane;
    const uint16_t* wb = w_router + static_cast<size_t>(eb) * H + 8 * lane;
    float acca = 0.0f, accb = 0.0f;
    int j = 0;
    for (; j + 4 <= nj; j += 4) {  // four slabs of each row in flight
      uint4 va[4], vb[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        va[q] = *reinterpret_cast<const uint4*>(wa + 256 * (j + q));
        vb[q] = *reinterpret_cast<const uint4*>(wb + 256 * (j + q));
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 xv = *reinterpret_cast<const uint4*>(xl + 256 * (j + q));
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          acca = (i & 1) ? fma_bf16<true>(word(xv, i >> 1), word(va[q], i >> 1), acca)
                         : fma_bf16<false>(word(xv, i >> 1), word(va[q], i >> 1), acca);
          accb = (i & 1) ? fma_bf16<true>(word(xv, i >> 1), word(vb[q], i >> 1), accb)
                         : fma_bf16<false>(word(xv, i >> 1), word(vb[q], i >> 1), accb);
        }
      }
    }
    for (; j < nj; ++j) {
      const uint4 va = *reinterpret_cast<const uint4*>(wa + 256 * j);
      const uint4 vb = *reinterpret_cast<const uint4*>(wb + 256 * j);
      const uint4 xv = *reinterpret_cast<const uint4*>(xl + 256 * j);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        acca = (i & 1) ? fma_bf16<true>(word(xv, i >> 1), word(va, i >> 1), acca)
                       : fma_bf16<false>(word(xv, i >> 1), word(va, i >> 1), acca);
        accb = (i & 1) ? fma_bf16<true>(word(xv, i >> 1), word(vb, i >> 1), accb)
                       : fma_bf16<false>(word(xv, i >> 1), word(vb, i >> 1), accb);
      }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      acca = __fadd_rn(acca, __shfl_xor_sync(0xffffffffu, acca, off));
      accb = __fadd_rn(accb, __shfl_xor_sync(0xffffffffu, accb, off));
    }
    if (lane == 0) {
      zs[ea] = __fadd_rn(acca, bias != nullptr ? bias[ea] : 0.0f);
      zs[eb] = __fadd_rn(accb, bias != nullptr ? bias[eb] : 0.0f);
    }
  }
  __syncthreads();

  // ---- the plain router's selection and weights on these logits
  if (warp == 0)
    topk_sigmoid_token<kPer>([&](int e) { return zs[e]; }, E, K, lane, topk_ids + static_cast<size_t>(t) * K,
                             topk_w + static_cast<size_t>(t) * K);
}

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

int screen_tiles(int M, int E) { return ((M + kSBM - 1) / kSBM) * ((E + kSBN - 1) / kSBN); }

// Slices of H per tile: the largest divisor of the chunk count with tiles x slices within one wave.
int screen_slices(int M, int H, int E) {
  const int tiles = screen_tiles(M, E), chunks = H / kSChunk;
  int best = 1;
  for (int d = 1; d <= chunks; ++d)
    if (chunks % d == 0 && tiles * d <= kSTargetCtas) best = d;
  return best;
}

struct ScreenLayout {
  size_t hi, lo, stats, partial, total;
};

ScreenLayout screen_layout(int M, int H, int E) {
  ScreenLayout L{};
  const size_t R = static_cast<size_t>(M) + E;
  size_t off = 0;
  L.hi = off;
  off = align256(off + R * H);
  L.lo = off;
  off = align256(off + R * H);
  L.stats = off;
  off = align256(off + R * sizeof(RowStats));
  L.partial = off;
  off = align256(off + static_cast<size_t>(screen_slices(M, H, E)) * M * E * sizeof(double));
  L.total = off;
  return L;
}

template <int kPer>
cudaError_t launch_route_kernel(const uint16_t* x, const uint16_t* w_router, const float* bias,
                                const double* partial, int slices, const RowStats* stats, int M, int E, int K, int H,
                                int32_t* topk_ids, float* topk_w, cudaStream_t stream) {
  const int smem = H * 2 + E * 8;
  auto kern = screen_route_kernel<kPer>;
  if (smem > 48 * 1024) {
    const cudaError_t st = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (st != cudaSuccess) return st;
  }
  kern<<<M, 128, smem, stream>>>(x, w_router, bias, partial, slices, stats, M, E, K, H, topk_ids, topk_w);
  return cudaGetLastError();
}

}  // namespace

bool screen_shape_ok(int M, int H, int E, int K) {
  return M >= 128 && H % 256 == 0 && H <= 8192 && E <= 1024 && K <= 32 && K <= E;
}

bool screen_eligible(int M, int H, int E, int K) {
  if (!screen_shape_ok(M, H, E, K)) return false;
  const char* env = std::getenv("MOE_ROUTER_SCREEN");
  return !(env != nullptr && std::strcmp(env, "0") == 0);
}

size_t screen_scratch_bytes(int M, int H, int E) { return screen_layout(M, H, E).total; }

cudaError_t launch_route_screened(const uint16_t* x, const uint16_t* w_router, const float* bias, int M, int H, int E,
                                  int K, uint8_t* scratch, int32_t* topk_ids, float* topk_w, int32_t* err,
                                  cudaStream_t stream) {
  const ScreenLayout L = screen_layout(M, H, E);
  auto* hi = reinterpret_cast<int8_t*>(scratch + L.hi);
  auto* lo = reinterpret_cast<int8_t*>(scratch + L.lo);
  auto* stats = reinterpret_cast<RowStats*>(scratch + L.stats);
  auto* partial = reinterpret_cast<double*>(scratch + L.partial);
  const int R = M + E;

  screen_quantize_kernel<<<R, kQThreads, 0, stream>>>(x, w_router, M, E, H, hi, lo, stats);
  cudaError_t st = cudaGetLastError();
  if (st != cudaSuccess) return st;

  // digit planes as [rows, H] int8 tensors read in 128-byte-wide boxes with the 128-byte swizzle
  CUtensorMap mxh, mxl, mwh, mwl;
  if (!encode_map_u8(&mxh, hi, M, H, kSBM) || !encode_map_u8(&mxl, lo, M, H, kSBM) ||
      !encode_map_u8(&mwh, hi + static_cast<size_t>(M) * H, E, H, kSBN) ||
      !encode_map_u8(&mwl, lo + static_cast<size_t>(M) * H, E, H, kSBN))
    return cudaErrorInvalidValue;
  const int slices = screen_slices(M, H, E);
  int dev = 0;
  if ((st = cudaGetDevice(&dev)) != cudaSuccess) return st;
  static bool attr[64] = {};
  if (dev < 64 && !attr[dev]) {
    if ((st = cudaFuncSetAttribute(screen_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSSmem)) !=
        cudaSuccess)
      return st;
    attr[dev] = true;
  }
  ScreenGemmArgs ga{partial, err, M, E, H / kSChunk / slices};
  dim3 grid((M + kSBM - 1) / kSBM, (E + kSBN - 1) / kSBN, slices);
  screen_gemm_kernel<<<grid, kSThreads, kSSmem, stream>>>(mxh, mxl, mwh, mwl, ga);
  if ((st = cudaGetLastError()) != cudaSuccess) return st;

  if (E <= 64)
    return launch_route_kernel<2>(x, w_router, bias, partial, slices, stats, M, E, K, H, topk_ids, topk_w, stream);
  if (E <= 256)
    return launch_route_kernel<8>(x, w_router, bias, partial, slices, stats, M, E, K, H, topk_ids, topk_w, stream);
  return launch_route_kernel<32>(x, w_router, bias, partial, slices, stats, M, E, K, H, topk_ids, topk_w, stream);
}

}  // namespace moe
