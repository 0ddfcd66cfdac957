// NVFP4 expert weights and activations ("[flashinfer] ... AlphaMoE NVFP4 커널
// 최적화", flashinfer PR #6511 analysis, intro: e2m1 values with e4m3 block
// scales; §2: weights repacked offline by a separate preparation step; §4:
// activation scale factors produced for and read by the GEMM itself).
//
// Quantisation recipe (identical for weights and activations; all fp32, one
// rounding per operation, in this order):
//   gs = amax / (6*448), or 1 if amax == 0           (one per matrix)
//   sb = e4m3_rn_satfinite(blockamax / 6 / gs)      (one per 16 elements)
//   q  = e2m1_rn_satfinite(v / (sb * gs)), 0 if sb == 0
// so v ~ q * sb * gs.  The conversions are CUDA's __nv_cvt_float_to_fp8 /
// __nv_cvt_float_to_fp4 (round to nearest even, saturate to finite).
//
// Layouts:
//   codes   uint8 [rows, cols/2]: element 2i in the low nibble of byte i.
//   scales  uint8 e4m3 [rows, cols/16] (as quantised), or repacked into
//   atoms   512-byte blocks covering 128 rows x 64 columns, ordered
//           [rows/128][cols/64]: byte (r%32)*16 + ((r%128)/32)*4 + (c/16)%4,
//           the layout tcgen05.cp ... 32x128b.warpx4 moves into tensor memory
//           for the block-scaled MMA.
//   blob    codes followed by atoms (one blob per projection, all experts).
// Activations are quantised into a tile-aligned copy: token tile `ti` (128
// plan rows of one expert) occupies rows [128 ti, 128 ti + 128) of the codes
// and atoms ti of the scale factors, so a tile's scale factors are whole atoms.
//
// GEMM: persistent, one CTA per SM, like the bf16 persistent kernel, with the
// operands e2m1 (256 elements = 128 bytes per stage row) and the block-16
// scales brought to shared memory by bulk copies, moved into tensor memory by
// tcgen05.cp and applied by tcgen05.mma.kind::mxf4nvf4.block_scale.block16.
// The fp32 accumulators are multiplied by gs_weight[e] * gs_activation in the
// epilogue.  Roles: warp 0 weight producer, warp 2 activation producer, warp 3
// scale-factor copier, warp 1 MMA issuer, warps 4-11 epilogue.  The copies of
// a stage's scale factors into tensor memory are issued by warp 3, up to four
// stages ahead, and signalled to the MMA issuer through an mbarrier: an MMA
// issued by the same thread right after the copies it reads waits for them,
// and with few token rows per tile the MMAs are too short to hide that wait
// (measured: the up GEMM of the 1000-token workload 978 -> 830 us).
#include <cuda_fp16.h>
#include <cuda_fp4.h>

#include <algorithm>
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"
#include "tile_list.cuh"

namespace moe {
namespace {

__device__ __forceinline__ float nvfp4_global_scale(float amax) { return amax == 0.0f ? 1.0f : amax / 2688.0f; }

// One 16-element block -> two words of packed e2m1 codes and the e4m3 scale.
__device__ __forceinline__ uint8_t quantize_block16(const float (&v)[16], float gs, uint32_t (&packed)[2]) {
  float bamax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) bamax = fmaxf(bamax, fabsf(v[i]));
  float t = bamax / 6.0f;
  t = t / gs;
  const __nv_fp8_storage_t sc = __nv_cvt_float_to_fp8(t, __NV_SATFINITE, __NV_E4M3);
  packed[0] = 0u;
  packed[1] = 0u;
  if (sc != 0) {
    const float sbf = __half2float(__half(__nv_cvt_fp8_to_halfraw(sc, __NV_E4M3)));
    const float d = sbf * gs;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t q = static_cast<uint32_t>(__nv_cvt_float_to_fp4(v[i] / d, __NV_E2M1, cudaRoundNearest)) & 0xFu;
      packed[i >> 3] |= q << (4 * (i & 7));
    }
  }
  return static_cast<uint8_t>(sc);
}

__device__ __forceinline__ void load16_bf16(const uint16_t* p, float (&v)[16]) {
  const uint4 a = *reinterpret_cast<const uint4*>(p);
  const uint4 b = *reinterpret_cast<const uint4*>(p + 8);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = bf16_lo(w[i]);
    v[2 * i + 1] = bf16_hi(w[i]);
  }
}

__device__ __forceinline__ void block_max_to(unsigned* dst, float mx) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  __shared__ float part[32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) part[warp] = mx;
  __syncthreads();
  if (warp == 0) {
    mx = (lane < static_cast<int>(blockDim.x >> 5)) ? part[lane] : 0.0f;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if (lane == 0 && mx > 0.0f) atomicMax(dst, __float_as_uint(mx));  // non-negative floats order as their bits
  }
}

// amax_bits[m] = max |src[m, :]| over n_per_mat bf16 values (n_per_mat % 8 == 0).
__global__ void __launch_bounds__(256) amax_kernel(const uint16_t* __restrict__ src, int64_t n_per_mat,
                                                   unsigned* __restrict__ amax_bits) {
  const uint16_t* p = src + static_cast<int64_t>(blockIdx.y) * n_per_mat;
  float mx = 0.0f;
  for (int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 8; i < n_per_mat;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x * 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(p + i);
    mx = fmaxf(mx, fmaxf(fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x))), fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y)))));
    mx = fmaxf(mx, fmaxf(fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))), fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w)))));
  }
  block_max_to(&amax_bits[blockIdx.y], mx);
}

__global__ void global_scale_kernel(const unsigned* __restrict__ amax_bits, int n, float* __restrict__ gs) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) gs[i] = nvfp4_global_scale(__uint_as_float(amax_bits[i]));
}

// One thread per 16-element block of [rows_total, cols] (matrices of rows_per_mat rows).
__global__ void __launch_bounds__(256) quantize_kernel(const uint16_t* __restrict__ src, int64_t total_blocks,
                                                       int64_t blocks_per_row, int64_t rows_per_mat,
                                                       const unsigned* __restrict__ amax_bits,
                                                       uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < total_blocks;
       b += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = (b / blocks_per_row) / rows_per_mat;
    const float gs = nvfp4_global_scale(__uint_as_float(amax_bits[m]));
    float v[16];
    load16_bf16(src + b * 16, v);
    uint32_t packed[2];
    scales[b] = quantize_block16(v, gs, packed);
    *reinterpret_cast<uint2*>(codes + b * 8) = make_uint2(packed[0], packed[1]);
  }
}

// scales [rows, kb] (kb = cols/16) -> atoms [rows/128][kb/4][512].
__global__ void scales_to_atoms_kernel(const uint8_t* __restrict__ scales, int64_t rows, int kb,
                                       uint8_t* __restrict__ atoms) {
  const int64_t n = rows * kb;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / kb;
    const int j = static_cast<int>(i % kb);
    const int64_t atom = (r / 128) * (kb / 4) + j / 4;
    const int rr = static_cast<int>(r % 128);
    atoms[atom * 512 + (rr % 32) * 16 + (rr / 32) * 4 + (j % 4)] = scales[i];
  }
}

// ---------------------------------------------------------------- activations
// amax over the real plan rows of h ([cap, cols] in plan order).
__global__ void __launch_bounds__(256) plan_rows_amax_kernel(const uint16_t* __restrict__ h,
                                                             const int32_t* __restrict__ sorted_ids,
                                                             const int32_t* __restrict__ ntpp, int nslots, int cols,
                                                             int cap, unsigned* __restrict__ amax_bits) {
  float mx = 0.0f;
  const int rows_per_block = 8;
  for (int rr = 0; rr < rows_per_block; ++rr) {
    const int r = blockIdx.x * rows_per_block + rr;
    if (r >= cap || r >= *ntpp) break;
    const int id = sorted_ids[r];
    if (id < 0 || id >= nslots) continue;
    const uint16_t* p = h + static_cast<int64_t>(r) * cols;
    for (int c = threadIdx.x * 8; c < cols; c += blockDim.x * 8) {
      const uint4 v = *reinterpret_cast<const uint4*>(p + c);
      mx = fmaxf(mx, fmaxf(fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x))), fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y)))));
      mx = fmaxf(mx, fmaxf(fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))), fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w)))));
    }
  }
  block_max_to(amax_bits, mx);
}

// Which expert owns token tile ti (tiles numbered expert by expert,
// ceil(count/128) each): after the call s_info = {expert or -1, tile index
// inside the expert}.  Every thread calls it; s_cnt holds the counts.
__device__ void locate_tile(const int* s_cnt, int E, int ti, int* s_info) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) s_info[0] = -1;
  __syncthreads();
  if (warp == 0) {
    const int per = (E + 31) / 32;
    const int lo = min(E, lane * per), hi = min(E, lo + per);
    int sum = 0;
    for (int e = lo; e < hi; ++e) sum += (s_cnt[e] + 127) / 128;
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    int t = incl - sum;
    if (ti >= t && ti < incl) {
      for (int e = lo; e < hi; ++e) {
        const int n = (s_cnt[e] + 127) / 128;
        if (ti < t + n) {
          s_info[0] = e;
          s_info[1] = ti - t;
          break;
        }
        t += n;
      }
    }
  }
  __syncthreads();
}

// Token tile `blockIdx.x` -> rows [128 ti, 128 ti + nrows) of the tile-aligned
// NVFP4 copy of h (plan order, `cols` wide): codes and scale atoms.  Rows past
// the expert's count are not written: the GEMM computes their columns from
// whatever they hold and never stores them (a column of the product depends
// on its own row of this operand only).  Each thread takes 64 consecutive
// elements of one row (four 16-element blocks): eight 16-byte loads, two
// 16-byte code stores, and the four scales as one 32-bit word (four column
// blocks of one atom row are adjacent bytes); blockIdx.y splits the row's
// 64-element groups over a few CTAs per tile.
__global__ void __launch_bounds__(256) quantize_tiles_kernel(
    const uint16_t* __restrict__ src, const int32_t* __restrict__ counts, const int32_t* __restrict__ offsets, int E,
    int cols, const unsigned* __restrict__ amax_bits, uint8_t* __restrict__ codes, uint8_t* __restrict__ atoms) {
  __shared__ int s_cnt[1024];
  __shared__ int s_info[2];
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += blockDim.x) s_cnt[e] = counts[e];
  __syncthreads();
  const int ti = blockIdx.x;
  locate_tile(s_cnt, E, ti, s_info);
  const int e = s_info[0];
  if (e < 0) return;
  const int local = s_info[1];
  const int nrows = min(128, s_cnt[e] - local * 128);
  const int row0 = offsets[e] + local * 128;
  const float gs = nvfp4_global_scale(__uint_as_float(*amax_bits));
  const int ngrp = cols / 64;  // 64-element groups per row
  // this CTA's slice of the groups: [g0, g1)
  const int per = (ngrp + gridDim.y - 1) / gridDim.y;
  const int g0 = blockIdx.y * per, g1 = min(ngrp, g0 + per);
  const int width = g1 - g0;
  for (int idx = tid; idx < nrows * width; idx += blockDim.x) {
    const int r = idx / width;
    const int gi = g0 + (idx - r * width);
    const uint16_t* row = src + static_cast<int64_t>(row0 + r) * cols + gi * 64;
    uint32_t packed[4][2];
    uint32_t scw = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      float v[16];
      load16_bf16(row + b * 16, v);
      scw |= static_cast<uint32_t>(quantize_block16(v, gs, packed[b])) << (8 * b);
    }
    uint8_t* cdst = codes + (static_cast<int64_t>(ti) * 128 + r) * (cols / 2) + gi * 32;
    reinterpret_cast<uint4*>(cdst)[0] = make_uint4(packed[0][0], packed[0][1], packed[1][0], packed[1][1]);
    reinterpret_cast<uint4*>(cdst)[1] = make_uint4(packed[2][0], packed[2][1], packed[3][0], packed[3][1]);
    *reinterpret_cast<uint32_t*>(atoms + (static_cast<int64_t>(ti) * ngrp + gi) * 512 + (r % 32) * 16 +
                                 (r / 32) * 4) = scw;
  }
}

// x enters the up projection once per routed slot, i.e. up to top_k times per
// token, so it is quantised once per token (quantize_kernel) and this kernel
// copies each slot's codes and scales into the tile-aligned layout: token tile
// `blockIdx.x`, row r <- token sorted_ids[row0 + r] / top_k.  The tile's token
// ids are staged in shared memory first; then every thread copies independent
// 16-byte code chunks and 4-byte scale words (four column blocks of one scale
// atom row), so many loads are in flight; blockIdx.y splits the columns over
// 8 CTAs per tile, so that each thread has few copies to chain.  Rows past the expert's count are
// not written (as above).
__global__ void __launch_bounds__(256) gather_tiles_kernel(
    const uint8_t* __restrict__ tok_codes, const uint8_t* __restrict__ tok_scales,
    const int32_t* __restrict__ sorted_ids, const int32_t* __restrict__ counts, const int32_t* __restrict__ offsets,
    int E, int top_k, int nslots, int cols, uint8_t* __restrict__ codes, uint8_t* __restrict__ atoms) {
  __shared__ int s_cnt[1024];
  __shared__ int s_info[2];
  __shared__ int s_tok[128];
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += blockDim.x) s_cnt[e] = counts[e];
  __syncthreads();
  const int ti = blockIdx.x;
  locate_tile(s_cnt, E, ti, s_info);
  const int e = s_info[0];
  if (e < 0) return;
  const int local = s_info[1];
  const int nrows = min(128, s_cnt[e] - local * 128);
  const int row0 = offsets[e] + local * 128;
  for (int r = tid; r < nrows; r += blockDim.x) {
    const int id = sorted_ids[row0 + r];
    s_tok[r] = (id >= 0 && id < nslots) ? id / top_k : -1;
  }
  __syncthreads();
  const int cb16 = cols / 32;  // 16-byte code chunks per row
  const int nw = cols / 64;    // scale words per row
  // this CTA's slice of the chunks [c0, c0 + cw) and scale words [a0, a0 + aw)
  const int cper = (cb16 + gridDim.y - 1) / gridDim.y, aper = (nw + gridDim.y - 1) / gridDim.y;
  const int c0 = blockIdx.y * cper, cw = max(0, min(cb16, c0 + cper) - c0);
  const int a0 = blockIdx.y * aper, aw = max(0, min(nw, a0 + aper) - a0);
  const uint4* src = reinterpret_cast<const uint4*>(tok_codes);
  uint4* dst = reinterpret_cast<uint4*>(codes) + static_cast<int64_t>(ti) * 128 * cb16;
#pragma unroll 4
  for (int i = tid; i < nrows * cw; i += blockDim.x) {
    const int r = i / cw, c = c0 + (i - r * cw);
    const int t = s_tok[r];
    dst[static_cast<int64_t>(r) * cb16 + c] = t >= 0 ? src[static_cast<int64_t>(t) * cb16 + c] : make_uint4(0, 0, 0, 0);
  }
  const uint32_t* ssrc = reinterpret_cast<const uint32_t*>(tok_scales);
#pragma unroll 4
  for (int i = tid; i < nrows * aw; i += blockDim.x) {
    const int r = i / aw, a = a0 + (i - r * aw);
    const int t = s_tok[r];
    *reinterpret_cast<uint32_t*>(atoms + (static_cast<int64_t>(ti) * nw + a) * 512 + (r % 32) * 16 + (r / 32) * 4) =
        t >= 0 ? ssrc[static_cast<int64_t>(t) * nw + a] : 0u;
  }
}

// ---------------------------------------------------------------- GEMM
constexpr int kBM = 128;
constexpr int kNmax = 128;
constexpr int kElemsPerStage = 256;          // e2m1 elements of one 128-byte stage row
constexpr int kBoxBytes = kBM * 128;         // 128 rows x 128 bytes
constexpr int kSfChunk = 4 * 512;            // 4 atoms: 128 rows x 256 elements of scales
constexpr int kBRows = 32;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 128 + 32 * kEpiWarps;
constexpr int kStagesA = 4;
constexpr int kStagesB = 3;
constexpr int kAStage = 2 * kBoxBytes + 2 * kSfChunk;  // 36 KB
constexpr int kBStage = kNmax * 128 + kSfChunk;        // 18 KB
constexpr int kMisc = 10240;
constexpr int kSmem = 1024 + kStagesA * kAStage + kStagesB * kBStage + kMisc;
constexpr int kSfCols = 48;  // per slot: SFA0 [0,16), SFA1 [16,32), SFB [32,48)
constexpr int kSfSlots = 4;
static_assert(kSmem <= 227 * 1024, "shared memory");
static_assert(kSmem > 116 * 1024, "one CTA per SM");
static_assert(2 * kNmax + kSfSlots * kSfCols <= 512, "tensor memory");

template <bool kUp>
__global__ void __launch_bounds__(kThreads, 1)
    persistent_nvfp4_kernel(const __grid_constant__ CUtensorMap tm_a0, const __grid_constant__ CUtensorMap tm_a1,
                            const __grid_constant__ CUtensorMap tm_b, const Nvfp4GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_ring = smem;
  uint8_t* b_ring = a_ring + kStagesA * kAStage;
  uint8_t* misc = b_ring + kStagesB * kBStage;
  uint64_t* a_full = reinterpret_cast<uint64_t*>(misc);
  uint64_t* a_empty = a_full + kStagesA;
  uint64_t* b_full = a_empty + kStagesA;
  uint64_t* b_empty = b_full + kStagesB;
  uint64_t* acc_full = b_empty + kStagesB;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* sf_full = acc_empty + 1;       // [kSfSlots]
  uint64_t* sf_empty = sf_full + kSfSlots; // [kSfSlots]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sf_empty + kSfSlots);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* cnt = const_cast<int*>(abort_flag + 1);  // [E]
  int* prefix = cnt + 1024;                     // [E + 1]

  const GroupedGemmArgs& g = args.g;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = g.E;
  const int W = kUp ? g.rows_per_expert / kBM : g.rows_per_expert / (2 * kBM);

  for (int e = tid; e < E; e += kThreads) cnt[e] = g.expert_counts[e];
  if (tid == 0) *abort_flag = 0;
  __syncthreads();
  if (warp == 0) build_tile_prefix<kNmax>(cnt, prefix, E, W, lane);
  if (tid == 0) {
    for (int s = 0; s < kStagesA; ++s) {
      mbar_init(&a_full[s], 1);
      mbar_init(&a_empty[s], 1);
    }
    for (int s = 0; s < kStagesB; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kEpiWarps);
    for (int q = 0; q < kSfSlots; ++q) {
      mbar_init(&sf_full[q], 1);
      mbar_init(&sf_empty[q], 1);
    }
    fence_mbar_init();
  }
  __syncthreads();
  const int total = prefix[E];
  if (static_cast<int>(blockIdx.x) >= total) return;
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int nk = g.kdim / kElemsPerStage;
  const int kblk64 = g.kdim / 64;  // scale atoms per 128 rows
  const int nslots = g.M * g.top_k;

  if (warp == 0) {
    // ------------------------------------------------ weight producer (codes + scales)
    // lane 0 waits for the slot and posts the byte count; lanes 0-3 issue the
    // stage's two code boxes and two scale copies in parallel.
    int ka = 0;
    bool alive = true;
    for (int tile = blockIdx.x; tile < total && alive; tile += gridDim.x) {
      const TileCoord c = decode_tile<kNmax>(prefix, cnt, E, tile);
      const uint64_t pol = cnt[c.e] <= kNmax ? l2_policy_evict_first() : l2_policy_evict_normal();
      const int row_a0 = kUp ? c.e * g.rows_per_expert + c.w * kBM : c.e * g.rows_per_expert + c.w * 2 * kBM;
      const int row_a1 = kUp ? row_a0 : row_a0 + kBM;
      const uint8_t* sf0 = args.sfa0 + static_cast<int64_t>(row_a0 / kBM) * kblk64 * 512;
      const uint8_t* sf1 = args.sfa1 + static_cast<int64_t>(row_a1 / kBM) * kblk64 * 512;
      for (int k = 0; k < nk; ++k, ++ka) {
        const int s = ka % kStagesA;
        bool ok = true;
        if (lane == 0) {
          ok = mbar_wait_bounded(&a_empty[s], ((ka / kStagesA) & 1) ^ 1, abort_flag);
          if (ok) mbar_arrive_expect_tx(&a_full[s], kAStage);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          if (lane == 0) {
            *abort_flag = 1;
            set_error(g.err, kErrTimeout);
          }
          alive = false;
          break;
        }
        uint8_t* st = a_ring + s * kAStage;
        if (lane == 0)
          tma_load_2d_hint(&tm_a0, &a_full[s], st, k * 128, row_a0, pol);
        else if (lane == 1)
          tma_load_2d_hint(kUp ? &tm_a1 : &tm_a0, &a_full[s], st + kBoxBytes, k * 128, row_a1, pol);
        else if (lane == 2)
          bulk_load(st + 2 * kBoxBytes, sf0 + k * kSfChunk, kSfChunk, &a_full[s]);
        else if (lane == 3)
          bulk_load(st + 2 * kBoxBytes + kSfChunk, sf1 + k * kSfChunk, kSfChunk, &a_full[s]);
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------ activation producer (tile-aligned codes + scales)
    int kb = 0;
    bool alive = true;
    for (int tile = blockIdx.x; tile < total && alive; tile += gridDim.x) {
      const TileCoord c = decode_tile<kNmax>(prefix, cnt, E, tile);
      const int nrows = min(kNmax, cnt[c.e] - c.t * kNmax);
      const int ti = prefix[c.e] / W + c.t;  // global token-tile index
      const int nbox = (nrows + kBRows - 1) / kBRows;
      const uint8_t* sfb = args.sfb + static_cast<int64_t>(ti) * kblk64 * 512;
      for (int k = 0; k < nk; ++k, ++kb) {
        const int s = kb % kStagesB;
        bool ok = true;
        if (lane == 0) {
          ok = mbar_wait_bounded(&b_empty[s], ((kb / kStagesB) & 1) ^ 1, abort_flag);
          if (ok) mbar_arrive_expect_tx(&b_full[s], nbox * kBRows * 128 + kSfChunk);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          if (lane == 0) {
            *abort_flag = 1;
            set_error(g.err, kErrTimeout);
          }
          alive = false;
          break;
        }
        uint8_t* st = b_ring + s * kBStage;
        if (lane < nbox)
          tma_load_2d(&tm_b, &b_full[s], st + lane * kBRows * 128, k * 128, ti * kNmax + lane * kBRows);
        else if (lane == 31)
          bulk_load(st + kNmax * 128, sfb + k * kSfChunk, kSfChunk, &b_full[s]);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      int ka = 0, kb = 0, j = 0, step = 0;
      bool alive = true;
      for (int tile = blockIdx.x; tile < total && alive; tile += gridDim.x, ++j) {
        const TileCoord c = decode_tile<kNmax>(prefix, cnt, E, tile);
        const int nrows = min(kNmax, cnt[c.e] - c.t * kNmax);
        const int N = (nrows + 15) & ~15;
        const uint32_t idesc = umma_idesc_nvfp4(kBM, N);
        if (!mbar_wait_bounded(acc_empty, (j & 1) ^ 1, abort_flag)) {
          *abort_flag = 1;
          set_error(g.err, kErrTimeout);
          break;
        }
        tc_fence_after_sync();
        const uint32_t d0 = tmem, d1 = tmem + kNmax;
        for (int k = 0; k < nk; ++k, ++ka, ++kb, ++step) {
          const int sa = ka % kStagesA, sb = kb % kStagesB;
          if (!mbar_wait_bounded(&a_full[sa], (ka / kStagesA) & 1, abort_flag) ||
              !mbar_wait_bounded(&b_full[sb], (kb / kStagesB) & 1, abort_flag)) {
            *abort_flag = 1;
            set_error(g.err, kErrTimeout);
            alive = false;
            break;
          }
          const int slot = step % kSfSlots;
          if (!mbar_wait_bounded(&sf_full[slot], (step / kSfSlots) & 1, abort_flag)) {
            *abort_flag = 1;
            set_error(g.err, kErrTimeout);
            alive = false;
            break;
          }
          tc_fence_after_sync();
          const uint8_t* ast = a_ring + sa * kAStage;
          const uint8_t* bst = b_ring + sb * kBStage;
          const uint32_t sf = tmem + 2 * kNmax + slot * kSfCols;
          const uint64_t da0 = umma_desc_sw128(ast);
          const uint64_t da1 = umma_desc_sw128(ast + kBoxBytes);
          const uint64_t db = umma_desc_sw128(bst);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (k | kk) != 0 ? 1u : 0u;
            umma_nvfp4_ss(d0, da0 + 2 * kk, db + 2 * kk, idesc, sf + 4 * kk, sf + 32 + 4 * kk, acc);
            umma_nvfp4_ss(d1, da1 + 2 * kk, db + 2 * kk, idesc, sf + 16 + 4 * kk, sf + 32 + 4 * kk, acc);
          }
          umma_commit(&a_empty[sa]);
          umma_commit(&b_empty[sb]);
          umma_commit(&sf_empty[slot]);
        }
        umma_commit(acc_full);
      }
    }
    __syncwarp();
  } else if (warp == 3) {
    // ------------------------------------------------ scale-factor copier (runs ahead of the MMA issuer)
    if (lane == 0) {
      int st = 0;
      bool alive = true;
      for (int tile = blockIdx.x; tile < total && alive; tile += gridDim.x) {
        for (int k = 0; k < nk; ++k, ++st) {
          const int slot = st % kSfSlots, sa = st % kStagesA, sb = st % kStagesB;
          if (!mbar_wait_bounded(&sf_empty[slot], ((st / kSfSlots) & 1) ^ 1, abort_flag) ||
              !mbar_wait_bounded(&a_full[sa], (st / kStagesA) & 1, abort_flag) ||
              !mbar_wait_bounded(&b_full[sb], (st / kStagesB) & 1, abort_flag)) {
            *abort_flag = 1;
            set_error(g.err, kErrTimeout);
            alive = false;
            break;
          }
          tc_fence_after_sync();
          const uint8_t* ast = a_ring + sa * kAStage;
          const uint8_t* bst = b_ring + sb * kBStage;
          const uint32_t sf = tmem + 2 * kNmax + slot * kSfCols;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            tmem_copy_32x16B_x4(sf + 4 * kk, smem_desc_32x16B(ast + 2 * kBoxBytes + kk * 512));
            tmem_copy_32x16B_x4(sf + 16 + 4 * kk, smem_desc_32x16B(ast + 2 * kBoxBytes + kSfChunk + kk * 512));
            tmem_copy_32x16B_x4(sf + 32 + 4 * kk, smem_desc_32x16B(bst + kNmax * 128 + kk * 512));
          }
          umma_commit(&sf_full[slot]);
        }
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------ epilogue: drain tensor memory first, then compute
    const int q = warp & 3;
    const int half = (warp - 4) >> 2;
    const float act_gs = nvfp4_global_scale(__uint_as_float(*args.act_amax));
    float hmax = 0.0f;  // up: max |h| of the values this thread stores
    int j = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++j) {
      const TileCoord c = decode_tile<kNmax>(prefix, cnt, E, tile);
      const int nrows = min(kNmax, cnt[c.e] - c.t * kNmax);
      const int N = (nrows + 15) & ~15;
      const int row0 = g.expert_offsets[c.e] + c.t * kNmax;
      bool ok = true;
      if (lane == 0) ok = mbar_wait_bounded(acc_full, j & 1, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      tc_fence_after_sync();
      const bool go = __shfl_sync(0xffffffffu, ok && !*abort_flag, 0);
      if (!go) {
        if (lane == 0 && !ok) set_error(g.err, kErrTimeout);
        break;
      }
      const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
      uint32_t v0[4][16], v1[4][16];  // this warp's chunks: 16 * (2i + half)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int cb = 16 * (2 * i + half);
        if (cb < N) {
          tmem_load_16(lane_base + cb, v0[i]);
          tmem_load_16(lane_base + kNmax + cb, v1[i]);
        }
      }
      tmem_load_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_one(acc_empty);  // tensor memory is free for the next tile
      const float s0 = args.gs_a0[c.e] * act_gs;
      const float s1 = args.gs_a1[c.e] * act_gs;
      // lane l holds column col0 + l for the 16 tokens of each chunk: pack token pairs as bf16,
      // transpose 8 x 8 inside each group of 8 lanes, and lane (8 g + b) writes tokens 2b and 2b + 1
      // at columns col0 + 8 g .. + 7 with one 16-byte store each
      const int g8 = lane >> 3, b8 = lane & 7;
      const int col8 = (kUp ? c.w * kBM : c.w * 2 * kBM) + q * 32 + 8 * g8;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int cb = 16 * (2 * i + half);
        if (cb >= N) break;
        const int n0 = cb + 2 * b8, n1 = n0 + 1;
        int id0 = -1, id1 = -1;
        if (!kUp) {
          if (n0 < nrows) id0 = g.sorted_ids[row0 + n0];
          if (n1 < nrows) id1 = g.sorted_ids[row0 + n1];
        }
#pragma unroll
        for (int part = 0; part < (kUp ? 1 : 2); ++part) {
          uint32_t w[8];
#pragma unroll
          for (int p = 0; p < 8; ++p) {
            if (kUp) {
              float hv[2];
#pragma unroll
              for (int u2 = 0; u2 < 2; ++u2) {
                const int qq = 2 * p + u2;
                const float gt = __uint_as_float(v0[i][qq]) * s0;
                const float ut = __uint_as_float(v1[i][qq]) * s1;
                hv[u2] = silu_mul(gt, ut);
              }
              w[p] = pack_bf16x2(hv[0], hv[1]);
              if (cb + 2 * p < nrows) hmax = fmaxf(hmax, fabsf(bf16_lo(w[p])));
              if (cb + 2 * p + 1 < nrows) hmax = fmaxf(hmax, fabsf(bf16_hi(w[p])));
            } else {
              const uint32_t* v = part == 0 ? v0[i] : v1[i];
              const float sc = part == 0 ? s0 : s1;
              w[p] = pack_bf16x2(__uint_as_float(v[2 * p]) * sc, __uint_as_float(v[2 * p + 1]) * sc);
            }
          }
          transpose8x8(w, b8);
          const uint4 r0 = make_uint4(__byte_perm(w[0], w[1], 0x5410), __byte_perm(w[2], w[3], 0x5410),
                                      __byte_perm(w[4], w[5], 0x5410), __byte_perm(w[6], w[7], 0x5410));
          const uint4 r1 = make_uint4(__byte_perm(w[0], w[1], 0x7632), __byte_perm(w[2], w[3], 0x7632),
                                      __byte_perm(w[4], w[5], 0x7632), __byte_perm(w[6], w[7], 0x7632));
          if (kUp) {
            if (n0 < nrows) *reinterpret_cast<uint4*>(g.out + static_cast<size_t>(row0 + n0) * g.out_ld + col8) = r0;
            if (n1 < nrows) *reinterpret_cast<uint4*>(g.out + static_cast<size_t>(row0 + n1) * g.out_ld + col8) = r1;
          } else {
            const int cc = col8 + part * kBM;
            if (n0 < nrows && id0 >= 0 && id0 < nslots)
              *reinterpret_cast<uint4*>(g.out + static_cast<size_t>(id0) * g.out_ld + cc) = r0;
            if (n1 < nrows && id1 >= 0 && id1 < nslots)
              *reinterpret_cast<uint4*>(g.out + static_cast<size_t>(id1) * g.out_ld + cc) = r1;
          }
        }
      }
    }
    if (kUp && args.out_amax != nullptr) {
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) hmax = fmaxf(hmax, __shfl_xor_sync(0xffffffffu, hmax, off));
      if (lane == 0 && hmax > 0.0f) atomicMax(args.out_amax, __float_as_uint(hmax));
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <bool kUp>
cudaError_t launch_nvfp4_variant(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b,
                                 const Nvfp4GemmArgs& args, int num_sms, cudaStream_t stream) {
  auto kern = persistent_nvfp4_kernel<kUp>;
  int dev = 0;
  cudaError_t st = cudaGetDevice(&dev);
  if (st != cudaSuccess) return st;
  static bool done[64] = {};
  if (dev < 64 && !done[dev]) {
    st = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (st != cudaSuccess) return st;
    done[dev] = true;
  }
  kern<<<num_sms, kThreads, kSmem, stream>>>(a0, a1, b, args);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_nvfp4_quantize(const uint16_t* src, int64_t n_mats, int64_t rows, int64_t cols, uint8_t* codes,
                                  uint8_t* scales, float* gs, unsigned* amax_bits, cudaStream_t stream) {
  cudaError_t st = cudaMemsetAsync(amax_bits, 0, sizeof(unsigned) * n_mats, stream);
  if (st != cudaSuccess) return st;
  const int64_t per = rows * cols;
  const int64_t bx = std::min<int64_t>(1024, (per / 8 + 255) / 256);
  amax_kernel<<<dim3(static_cast<unsigned>(std::max<int64_t>(bx, 1)), static_cast<unsigned>(n_mats)), 256, 0,
                stream>>>(src, per, amax_bits);
  if ((st = cudaGetLastError()) != cudaSuccess) return st;
  global_scale_kernel<<<static_cast<unsigned>((n_mats + 255) / 256), 256, 0, stream>>>(
      amax_bits, static_cast<int>(n_mats), gs);
  if ((st = cudaGetLastError()) != cudaSuccess) return st;
  const int64_t total_blocks = n_mats * rows * (cols / 16);
  const int64_t grid = std::min<int64_t>((total_blocks + 255) / 256, 148 * 16);
  quantize_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(src, total_blocks, cols / 16, rows, amax_bits,
                                                                   codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_nvfp4_scales_to_atoms(const uint8_t* scales, int64_t rows, int64_t cols, uint8_t* atoms,
                                         cudaStream_t stream) {
  const int64_t n = rows * (cols / 16);
  const int64_t grid = std::min<int64_t>((n + 255) / 256, 148 * 16);
  scales_to_atoms_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(scales, rows, static_cast<int>(cols / 16),
                                                                          atoms);
  return cudaGetLastError();
}

cudaError_t launch_amax_all(const uint16_t* src, int64_t n, unsigned* amax_bits, cudaStream_t stream) {
  const int64_t bx = std::min<int64_t>(1024, (n / 8 + 255) / 256);
  amax_kernel<<<dim3(static_cast<unsigned>(std::max<int64_t>(bx, 1)), 1), 256, 0, stream>>>(src, n, amax_bits);
  return cudaGetLastError();
}

cudaError_t launch_amax_plan_rows(const uint16_t* h, const int32_t* sorted_ids, const int32_t* ntpp, int nslots,
                                  int cols, int cap, unsigned* amax_bits, cudaStream_t stream) {
  plan_rows_amax_kernel<<<(cap + 7) / 8, 256, 0, stream>>>(h, sorted_ids, ntpp, nslots, cols, cap, amax_bits);
  return cudaGetLastError();
}

cudaError_t launch_quantize_tiles(const uint16_t* src, const int32_t* counts, const int32_t* offsets, int E, int cols,
                                  int tiles_ub, const unsigned* amax_bits, uint8_t* codes, uint8_t* atoms,
                                  cudaStream_t stream) {
  const int slices = std::max(1, cols / 512);  // 8 groups of 64 elements per CTA and row
  quantize_tiles_kernel<<<dim3(tiles_ub, slices), 256, 0, stream>>>(src, counts, offsets, E, cols, amax_bits, codes,
                                                                    atoms);
  return cudaGetLastError();
}

cudaError_t launch_quantize_rows(const uint16_t* src, int64_t rows, int64_t cols, const unsigned* amax_bits,
                                 uint8_t* codes, uint8_t* scales, cudaStream_t stream) {
  const int64_t total_blocks = rows * (cols / 16);
  const int64_t grid = std::min<int64_t>((total_blocks + 255) / 256, 148 * 16);
  quantize_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(src, total_blocks, cols / 16, rows, amax_bits,
                                                                   codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_gather_tiles(const uint8_t* tok_codes, const uint8_t* tok_scales, const int32_t* sorted_ids,
                                const int32_t* counts, const int32_t* offsets, int E, int top_k, int nslots, int cols,
                                int tiles_ub, uint8_t* codes, uint8_t* atoms, cudaStream_t stream) {
  gather_tiles_kernel<<<dim3(tiles_ub, 8), 256, 0, stream>>>(tok_codes, tok_scales, sorted_ids, counts, offsets, E, top_k,
                                                    nslots, cols, codes, atoms);
  return cudaGetLastError();
}

cudaError_t launch_nvfp4_up(const CUtensorMap& gate_codes, const CUtensorMap& up_codes, const CUtensorMap& x_codes,
                            const Nvfp4GemmArgs& args, int num_sms, cudaStream_t stream) {
  return launch_nvfp4_variant<true>(gate_codes, up_codes, x_codes, args, num_sms, stream);
}

cudaError_t launch_nvfp4_down(const CUtensorMap& down_codes, const CUtensorMap& h_codes, const Nvfp4GemmArgs& args,
                              int num_sms, cudaStream_t stream) {
  return launch_nvfp4_variant<false>(down_codes, down_codes, h_codes, args, num_sms, stream);
}

}  // namespace moe
