// NVFP4 expert projections on 2-SM pairs ("[flashinfer] ... AlphaMoE NVFP4
// 커널 최적화", flashinfer PR #6511 analysis: e2m1 weights and activations
// with e4m3 block-16 scales, intro and §2; the up / down kernels of the route
// chain, §6).
//
// The operands and their layouts are those of the single-SM NVFP4 kernel
// (nvfp4.cu): weight codes [rows, kdim/2] read in 128-row x 128-byte boxes,
// scale atoms of 128 rows x 64 elements (512 bytes, the tcgen05.cp 32x128b
// source layout), and a tile-aligned copy of the activations (token tile ti =
// rows [128 ti, 128 ti + 128), its scale factors whole atoms).  What changes
// is the MMA: one tcgen05.mma.cta_group::2 of M = 256 weight rows per pair of
// SMs, as in the bf16 pair kernels (gemm_pair.cu), so per SM the activation
// bytes per weight byte and the block-scaled MMA instructions per weight byte
// halve.
//
// Scale factors in the pair: each CTA keeps in its own tensor memory the
// scales of its 128 weight rows and those of the whole token tile (all N
// columns of B); the leader copies both CTAs' scales with one
// tcgen05.cp.cta_group::2 per 32-row block (each CTA's shared memory into its
// own tensor memory).  All copies are 2-D TMA loads with cta_group::2 that
// complete on the leader's mbarriers (scale atoms through a tensor map of
// 256-byte rows, no swizzle); no load uses multicast.
//
// Tiles: (expert e, weight block w, token tile t), ordered e, w, t, a static
// round-robin list per pair; a token tile holds up to 128 plan rows, N = rows
// rounded up to 16, CTA r loads plan rows [r N/2, (r+1) N/2).
//   up:   weight block w = rows 256w..256w+255 of W_gate and of W_up; CTA r
//         holds rows 256w + 128r..+127 of both; h = bf16(silu(gate) * up).
//   down: weight block w = rows 512w..512w+511 of W_down as two M = 256
//         halves; CTA r holds rows 512w + 128r.. and 512w + 256 + 128r..;
//         y[slot, col] = bf16(acc), scattered to the slot.
// The fp32 accumulators are multiplied by gs_weight[e] * gs_activation.
// Warp roles (384 threads per CTA): 0 = weight producer, 1 = MMA issuer
// (leader), 2 = activation producer, 3 = scale-factor copier into tensor
// memory (leader), 4..11 = epilogue.  All mbarrier waits are bounded; a
// timeout sets the error word and unwinds, and both CTAs still meet at the
// final cluster barrier.
#include "common.cuh"
#include "kernels.h"
#include "pair_ptx.cuh"
#include "tile_list.cuh"

namespace moe {
namespace {

// Global scale of the NVFP4 recipe: amax / (6 * 448), or 1 for an all-zero tensor.
__device__ __forceinline__ float pair_global_scale(float amax) { return amax == 0.0f ? 1.0f : amax / 2688.0f; }

constexpr int kBM = 128;                 // weight rows per CTA (MMA M = 256 per pair)
constexpr int kNmax = 128;               // token rows per tile (pair)
constexpr int kHalf = kNmax / 2;         // token rows per CTA
constexpr int kElemsPerStage = 256;      // e2m1 elements of one 128-byte stage row
constexpr int kBoxBytes = kBM * 128;     // 128 rows x 128 bytes
constexpr int kSfChunk = 4 * 512;        // 4 atoms: 128 rows x 256 elements of scales
constexpr int kSfRows = kSfChunk / 256;  // the chunk as rows of the 256-byte scale map
constexpr int kBRows = 32;    // rows per token-row box
constexpr int kEpiWarps = 8;
constexpr int kEpiWarp0 = 4;  // warps 0-3 have the producer, MMA and copier roles
constexpr int kThreads = 32 * kEpiWarp0 + 32 * kEpiWarps;
constexpr int kStagesA = 4;
constexpr int kStagesB = 4;
constexpr int kAStage = 2 * kBoxBytes + 2 * kSfChunk;  // two weight code boxes and their scales: 36 KB
constexpr int kBStage = kHalf * 128 + kSfChunk;        // a CTA's token rows and the tile's scales: 10 KB
constexpr int kMisc = 8704;                             // barriers, flags, counts and tile prefix (E <= 1024)
constexpr int kSfCols = 48;  // per slot: SFA0 [0,16), SFA1 [16,32), SFB [32,48)
constexpr int kSfSlots = 4;
static_assert(2 * kNmax + kSfSlots * kSfCols <= 512, "tensor memory");
static_assert(kAStage % 1024 == 0 && kBStage % 1024 == 0, "stages keep the 1024-byte alignment of the swizzled boxes");
static_assert(kHalf % kBRows == 0, "whole token-row boxes per CTA");

constexpr int kSmem = 1024 + kStagesA * kAStage + kStagesB * kBStage + kMisc;
static_assert(kSmem <= 227 * 1024, "shared memory");
static_assert(kSmem > 116 * 1024, "one CTA per SM: it owns all 512 tensor-memory columns");
static_assert(8 * (2 * kStagesA + 2 * kStagesB + 2 + 2 * kSfSlots) + 8 + 4 * (1024 + 1025) <= kMisc, "misc");

template <bool kUp>
__global__ void __launch_bounds__(kThreads, 1)
    nvfp4_pair_kernel(const __grid_constant__ CUtensorMap tm_a0, const __grid_constant__ CUtensorMap tm_a1,
                      const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_sfa0,
                      const __grid_constant__ CUtensorMap tm_sfa1, const __grid_constant__ CUtensorMap tm_sfb,
                      const Nvfp4GemmArgs args) {
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
  uint64_t* acc_empty = acc_full + 1;       // the leader's counts both CTAs' epilogue warps
  uint64_t* sf_full = acc_empty + 1;        // [kSfSlots] (leader)
  uint64_t* sf_empty = sf_full + kSfSlots;  // [kSfSlots] (leader)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sf_empty + kSfSlots);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* cnt = const_cast<int*>(abort_flag + 1);  // [E]
  int* prefix = cnt + 1024;                     // [E + 1]

  const GroupedGemmArgs& g = args.g;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cta_rank_in_cluster();
  const bool leader = rank == 0;
  const int pair = static_cast<int>(blockIdx.x) >> 1;
  const int npairs = static_cast<int>(gridDim.x) >> 1;
  const int E = g.E;
  // weight blocks per expert: up = 256 rows of gate and of up; down = 512 rows
  const int W = kUp ? g.rows_per_expert / (2 * kBM) : g.rows_per_expert / (4 * kBM);

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
    mbar_init(acc_empty, 2 * kEpiWarps);
    for (int q = 0; q < kSfSlots; ++q) {
      mbar_init(&sf_full[q], 1);
      mbar_init(&sf_empty[q], 1);
    }
    fence_mbar_init();
  }
  __syncthreads();
  const int total = prefix[E];
  // Both CTAs of a pair see the same tile count, so they leave together.
  if (pair >= total) return;
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before_sync();
  cluster_sync_all();  // the peer's barriers are initialised and both CTAs hold tensor memory
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int nk = g.kdim / kElemsPerStage;
  const int kblk64 = g.kdim / 64;  // scale atoms per 128 rows
  const int nslots = g.M * g.top_k;

  if (warp == 0) {
    // ------------------------------------------------ weight producer (codes + scales, both CTAs)
    // lane 0 waits for the slot (the leader's lane 0 also posts both CTAs' bytes); lanes 0-3 issue the
    // stage's two code boxes and two scale chunks.
    if (lane == 0) {
      prefetch_tensor_map(&tm_a0);
      prefetch_tensor_map(&tm_sfa0);
      if (kUp) {
        prefetch_tensor_map(&tm_a1);
        prefetch_tensor_map(&tm_sfa1);
      }
    }
    int ka = 0;
    bool alive = true;
    for (int tile = pair; tile < total && alive; tile += npairs) {
      const TileCoord c = decode_tile<kNmax>(prefix, cnt, E, tile);
      const uint64_t pol = cnt[c.e] <= kNmax ? l2_policy_evict_first() : l2_policy_evict_normal();
      const int base = c.e * g.rows_per_expert + static_cast<int>(rank) * kBM;
      const int row_a0 = kUp ? base + c.w * 2 * kBM : base + c.w * 4 * kBM;
      const int row_a1 = kUp ? row_a0 : row_a0 + 2 * kBM;
      // first 256-byte row of each 128-row block's scale atoms in the scale maps
      const int sf_row0 = (row_a0 / kBM) * kblk64 * 2;
      const int sf_row1 = (row_a1 / kBM) * kblk64 * 2;
      for (int k = 0; k < nk; ++k, ++ka) {
        const int s = ka % kStagesA;
        bool ok = true;
        if (lane == 0) {
          ok = mbar_wait_bounded(&a_empty[s], ((ka / kStagesA) & 1) ^ 1, abort_flag);
          if (ok && leader) mbar_arrive_expect_tx(&a_full[s], 2 * kAStage);
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
        const uint32_t bar = cluster_addr(&a_full[s], 0);
        if (lane == 0)
          tma_load_2d_pair(&tm_a0, bar, st, k * 128, row_a0, pol);
        else if (lane == 1)
          tma_load_2d_pair(kUp ? &tm_a1 : &tm_a0, bar, st + kBoxBytes, k * 128, row_a1, pol);
        else if (lane == 2)
          tma_load_2d_pair(&tm_sfa0, bar, st + 2 * kBoxBytes, 0, sf_row0 + k * kSfRows, pol);
        else if (lane == 3)
          tma_load_2d_pair(kUp ? &tm_sfa1 : &tm_sfa0, bar, st + 2 * kBoxBytes + kSfChunk, 0,
                           sf_row1 + k * kSfRows, pol);
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------ activation producer (both CTAs: half the rows, all scales)
    if (lane == 0) {
      prefetch_tensor_map(&tm_b);
      prefetch_tensor_map(&tm_sfb);
    }
    const uint64_t pol_b = l2_policy_evict_normal();
    int kb = 0;
    bool alive = true;
    for (int tile = pair; tile < total && alive; tile += npairs) {
      const TileCoord c = decode_tile<kNmax>(prefix, cnt, E, tile);
      const int nrows = min(kNmax, cnt[c.e] - c.t * kNmax);
      const int N = (nrows + 15) & ~15;
      const int half = N / 2;
      const int ti = prefix[c.e] / W + c.t;  // global token-tile index
      const int row0 = ti * kNmax + static_cast<int>(rank) * half;
      const int nbox = (half + kBRows - 1) / kBRows;
      const int sfb_row = ti * kblk64 * 2;
      const uint32_t b_bytes = 2u * (nbox * kBRows * 128 + kSfChunk);
      for (int k = 0; k < nk; ++k, ++kb) {
        const int s = kb % kStagesB;
        bool ok = true;
        if (lane == 0) {
          ok = mbar_wait_bounded(&b_empty[s], ((kb / kStagesB) & 1) ^ 1, abort_flag);
          if (ok && leader) mbar_arrive_expect_tx(&b_full[s], b_bytes);
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
        const uint32_t bar = cluster_addr(&b_full[s], 0);
        if (lane < nbox)
          tma_load_2d_pair(&tm_b, bar, st + lane * kBRows * 128, k * 128, row0 + lane * kBRows, pol_b);
        else if (lane == 31)
          tma_load_2d_pair(&tm_sfb, bar, st + kHalf * 128, 0, sfb_row + k * kSfRows, pol_b);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (leader only)
    if (leader && lane == 0) {
      int ka = 0, kb = 0, j = 0, step = 0;
      bool alive = true;
      for (int tile = pair; tile < total && alive; tile += npairs, ++j) {
        const TileCoord c = decode_tile<kNmax>(prefix, cnt, E, tile);
        const int nrows = min(kNmax, cnt[c.e] - c.t * kNmax);
        const int N = (nrows + 15) & ~15;
        const uint32_t idesc = umma_idesc_nvfp4(2 * kBM, N);
        if (!mbar_wait_bounded(acc_empty, (j & 1) ^ 1, abort_flag)) {
          *abort_flag = 1;
          set_error(g.err, kErrTimeout);
          break;
        }
        tc_fence_after_sync();
        const uint32_t d0 = tmem, d1 = tmem + kNmax;
        for (int k = 0; k < nk; ++k, ++ka, ++kb, ++step) {
          const int sa = ka % kStagesA, sb = kb % kStagesB;
          const int slot = step % kSfSlots;
          if (!mbar_wait_bounded(&a_full[sa], (ka / kStagesA) & 1, abort_flag) ||
              !mbar_wait_bounded(&b_full[sb], (kb / kStagesB) & 1, abort_flag) ||
              !mbar_wait_bounded(&sf_full[slot], (step / kSfSlots) & 1, abort_flag)) {
            *abort_flag = 1;
            set_error(g.err, kErrTimeout);
            alive = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t sf = tmem + 2 * kNmax + slot * kSfCols;
          const uint64_t da0 = umma_desc_sw128(a_ring + sa * kAStage);
          const uint64_t da1 = umma_desc_sw128(a_ring + sa * kAStage + kBoxBytes);
          const uint64_t db = umma_desc_sw128(b_ring + sb * kBStage);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (k | kk) != 0 ? 1u : 0u;
            umma_nvfp4_pair(d0, da0 + 2 * kk, db + 2 * kk, idesc, sf + 4 * kk, sf + 32 + 4 * kk, acc);
            umma_nvfp4_pair(d1, da1 + 2 * kk, db + 2 * kk, idesc, sf + 16 + 4 * kk, sf + 32 + 4 * kk, acc);
          }
          umma_commit_pair(&a_empty[sa]);
          umma_commit_pair(&b_empty[sb]);
          umma_commit_pair_mask(&sf_empty[slot], 0x1);
        }
        umma_commit_pair(acc_full);  // also on an abort, so neither epilogue is left waiting
      }
    }
    __syncwarp();
  } else if (warp == 3) {
    // ------------------------------------------------ scale-factor copier (leader; runs ahead of the MMAs)
    if (leader && lane == 0) {
      int st = 0;
      bool alive = true;
      for (int tile = pair; tile < total && alive; tile += npairs) {
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
            tmem_copy_32x16B_x4_pair(sf + 4 * kk, smem_desc_32x16B(ast + 2 * kBoxBytes + kk * 512));
            tmem_copy_32x16B_x4_pair(sf + 16 + 4 * kk, smem_desc_32x16B(ast + 2 * kBoxBytes + kSfChunk + kk * 512));
            tmem_copy_32x16B_x4_pair(sf + 32 + 4 * kk, smem_desc_32x16B(bst + kHalf * 128 + kk * 512));
          }
          umma_commit_pair_mask(&sf_full[slot], 0x1);
        }
      }
    }
    __syncwarp();
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------ epilogue (both CTAs: their own 128 rows)
    const int q = warp & 3;  // tensor-memory lane quarter this warp may read
    const int part_c = (warp - kEpiWarp0) >> 2;  // which of the two 16-column chunks of every 32 this warp drains
    const float act_gs = pair_global_scale(__uint_as_float(*args.act_amax));
    float hmax = 0.0f;  // up: max |h| of the values this thread stores
    int j = 0;
    for (int tile = pair; tile < total; tile += npairs, ++j) {
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
      uint32_t v0[4][16], v1[4][16];  // this warp's chunks: 16 * (2i + part_c)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int cb = 16 * (2 * i + part_c);
        if (cb < N) {
          tmem_load_16(lane_base + cb, v0[i]);
          tmem_load_16(lane_base + kNmax + cb, v1[i]);
        }
      }
      tmem_load_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(cluster_addr(acc_empty, 0));  // tensor memory is free for the next tile
      const float s0 = args.gs_a0[c.e] * act_gs;
      const float s1 = args.gs_a1[c.e] * act_gs;
      // lane l holds weight row (col0 + l) for the 16 tokens of each chunk: pack token pairs as bf16,
      // transpose 8 x 8 inside each group of 8 lanes, and lane (8 g + b) writes tokens 2b and 2b + 1
      // at columns col0 + 8 g .. + 7 with one 16-byte store each
      const int g8 = lane >> 3, b8 = lane & 7;
      const int col8 = (kUp ? c.w * 2 * kBM : c.w * 4 * kBM) + static_cast<int>(rank) * kBM + q * 32 + 8 * g8;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int cb = 16 * (2 * i + part_c);
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
            const int cc = col8 + part * 2 * kBM;
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
  cluster_sync_all();  // neither CTA leaves while the other may still use its shared or tensor memory
  if (warp == 1) tmem_dealloc_pair(tmem, 512);
}

template <bool kUp>
cudaError_t launch_variant(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b, const CUtensorMap& sfa0,
                           const CUtensorMap& sfa1, const CUtensorMap& sfb, const Nvfp4GemmArgs& args, int num_sms,
                           cudaStream_t stream) {
  auto kern = nvfp4_pair_kernel<kUp>;
  int dev = 0;
  cudaError_t st = cudaGetDevice(&dev);
  if (st != cudaSuccess) return st;
  static bool done[64] = {};
  if (dev < 64 && !done[dev]) {
    st = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (st != cudaSuccess) return st;
    done[dev] = true;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms & ~1));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a0, a1, b, sfa0, sfa1, sfb, args);
}

}  // namespace

cudaError_t launch_nvfp4_pair_up(const CUtensorMap& gate_codes, const CUtensorMap& up_codes,
                                 const CUtensorMap& x_codes, const CUtensorMap& gate_sf, const CUtensorMap& up_sf,
                                 const CUtensorMap& x_sf, const Nvfp4GemmArgs& args, int num_sms,
                                 cudaStream_t stream) {
  if (args.g.rows_per_expert % (2 * kBM) != 0 || args.g.kdim % kElemsPerStage != 0) return cudaErrorInvalidValue;
  return launch_variant<true>(gate_codes, up_codes, x_codes, gate_sf, up_sf, x_sf, args, num_sms, stream);
}

cudaError_t launch_nvfp4_pair_down(const CUtensorMap& down_codes, const CUtensorMap& h_codes,
                                   const CUtensorMap& down_sf, const CUtensorMap& h_sf, const Nvfp4GemmArgs& args,
                                   int num_sms, cudaStream_t stream) {
  if (args.g.rows_per_expert % (4 * kBM) != 0 || args.g.kdim % kElemsPerStage != 0) return cudaErrorInvalidValue;
  return launch_variant<false>(down_codes, down_codes, h_codes, down_sf, down_sf, h_sf, args, num_sms, stream);
}

}  // namespace moe
