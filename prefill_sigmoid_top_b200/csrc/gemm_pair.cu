// Grouped expert projections on 2-SM pairs for batch and prefill shapes
// ("[flashinfer] ... AlphaMoE NVFP4 커널 최적화", flashinfer PR #6511 analysis:
// the up / down kernels of the route chain, §6; wide weight panels streamed by
// TMA, §2).
//
// Why: with one CTA per SM and 128-row token tiles the persistent kernel is
// bound by the operand feed into shared memory (each SM reads its weight tile
// and all the token rows of its tile for every stage).  Here two CTAs of a
// cluster run one tcgen05.mma.cta_group::2 of M = 256 weight rows: each CTA
// holds 128 weight rows (A) and half of the token rows (B) of the tile in its
// own shared memory, and each CTA's tensor memory receives its 128 rows of the
// product for all N tokens.  Per SM the token-row bytes per flop halve, and a
// token tile covers twice the weight rows per MMA instruction.
//
// Pair protocol (CTA rank 0 = leader, rank 1 = peer):
//   * both CTAs allocate tensor memory together (cta_group::2, same warp);
//   * each CTA's producers wait on their own "empty" barriers and load their
//     own halves; all copies complete on the leader's "full" barriers, for
//     which the leader alone posts the expected bytes of both CTAs;
//   * the leader's one MMA thread waits on its full barriers, issues the
//     MMAs, and its commits arrive on the empty barriers of both CTAs (the
//     commit's CTA mask) and on both CTAs' accumulator-full barriers;
//   * each CTA's epilogue drains its own tensor memory and arrives on the
//     leader's accumulator-empty barrier (the peer's arrive remotely).
// Copies are plain TMA loads with cta_group::2 (no multicast).
//
// Tiles: (expert e, weight block w, token tile t) over a static round-robin
// list of tiles per pair, ordered e, w, t.  A token tile holds up to kNmax
// plan rows; N = rows rounded up to 16; CTA r loads plan rows [r N/2, (r+1) N/2).
//   up:   weight block w = rows 256w..256w+255 of W_gate and of W_up; CTA r
//         holds rows 256w + 128r..+127 of both; h[row, 256w + 128r + i] =
//         bf16(silu(gate) * up) from its two accumulators.
//   down: weight block w = rows 512w..512w+511 of W_down as two M = 256
//         halves; CTA r holds rows 512w + 128r.. and 512w + 256 + 128r..;
//         y[slot, col] = bf16(acc), scattered to the slot.
// Warp roles (640 threads per CTA): 0 = weight producer, 1 = MMA issuer
// (leader only), 2 = token-row producer, 3 = idle, 4..19 = epilogue.
// All mbarrier waits are bounded; a timeout sets the error word and unwinds,
// and both CTAs still meet at the final cluster barrier.
#include "common.cuh"
#include "kernels.h"
#include "pair_ptx.cuh"
#include "tile_list.cuh"

namespace moe {

#ifdef MOE_PAIR_TRACE
// Timeline build (MOE_PAIR_TRACE, a separate library made by build.py --trace; never the
// default): per tile, 8 stamps of the leader CTA -- [0] e | w << 12 | t << 20 | N << 28 | sm << 48,
// [1] MMA start (accumulator free), [2] first stage ready, [3] last MMA issued, [4] epilogue
// start, [5] accumulator released, [6] / [7] first / last weight stage issued; [up, down].
constexpr int kTraceTiles = 8192;
__device__ unsigned long long g_pair_trace[2][kTraceTiles][8];
#define MOE_TRACE_STAMP(kind, tile, slot, value) \
  (g_pair_trace[(kind)][(tile) < kTraceTiles ? (tile) : kTraceTiles - 1][(slot)] = (value))
#else
#define MOE_TRACE_STAMP(kind, tile, slot, value) ((void)0)
#endif

namespace {

constexpr int kBM = 128;                  // weight rows per CTA (MMA M = 256 per pair)
constexpr int kBK = 64;                   // contraction elements per stage
constexpr int kBoxBytes = kBM * kBK * 2;  // one 128 x 64 bf16 box: 16 KB
constexpr int kBRows = 32;                // rows per token-row box
constexpr int kEpiWarps = 16;  // four per tensor-memory lane quarter: the drain is latency-bound
constexpr int kThreads = 128 + 32 * kEpiWarps;

template <int kNmax, int kStagesA, int kStagesB>
struct QCfg {
  static constexpr int kHalf = kNmax / 2;  // token rows per CTA
  static constexpr int kAStage = 2 * kBoxBytes;
  static constexpr int kBStage = kHalf * kBK * 2;
  static constexpr int kAccCols = 2 * kNmax;
  static constexpr int kAccBufs = 512 / kAccCols;
  static constexpr int kMisc = 10240;  // barriers, flags, counts and tile prefix over experts (E <= 1024)
  static constexpr int kSmem = 1024 + kStagesA * kAStage + kStagesB * kBStage + kMisc;
  static_assert(kNmax == 128 || kNmax == 256, "pair token-tile widths");
  static_assert(kHalf % kBRows == 0, "whole token-row boxes per CTA");
  static_assert(kSmem <= 227 * 1024, "shared memory");
  static_assert(kSmem > 116 * 1024, "one CTA per SM: it owns all 512 tensor-memory columns");
};

// kGatherB (up only): the token rows are gathered from x by token id inside the GEMM (tile::gather4,
// four rows per copy, one copy per lane) instead of read as consecutive rows of x pre-gathered into
// plan order.
template <bool kUp, int kNmax, int kStagesA, int kStagesB, bool kGatherB = false>
__global__ void __launch_bounds__(kThreads, 1)
    pair_gemm_kernel(const __grid_constant__ CUtensorMap tm_a0, const __grid_constant__ CUtensorMap tm_a1,
                     const __grid_constant__ CUtensorMap tm_b, const GroupedGemmArgs args) {
  using C = QCfg<kNmax, kStagesA, kStagesB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_ring = smem;
  uint8_t* b_ring = a_ring + kStagesA * C::kAStage;
  uint8_t* misc = b_ring + kStagesB * C::kBStage;
  uint64_t* a_full = reinterpret_cast<uint64_t*>(misc);
  uint64_t* a_empty = a_full + kStagesA;
  uint64_t* b_full = a_empty + kStagesA;
  uint64_t* b_empty = b_full + kStagesB;
  uint64_t* acc_full = b_empty + kStagesB;  // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2] (the leader's counts both CTAs' epilogue warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* cnt = const_cast<int*>(abort_flag + 1);  // [E]
  int* prefix = cnt + 1024;                     // [E + 1]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cta_rank_in_cluster();
  const bool leader = rank == 0;
  const int pair = static_cast<int>(blockIdx.x) >> 1;
  const int npairs = static_cast<int>(gridDim.x) >> 1;
  const int E = args.E;
  // weight blocks per expert: up = 256 rows of gate and of up; down = 512 rows
  const int W = kUp ? args.rows_per_expert / (2 * kBM) : args.rows_per_expert / (4 * kBM);

  for (int e = tid; e < E; e += kThreads) cnt[e] = args.expert_counts[e];
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
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * kEpiWarps);
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
  const int nk = args.kdim / kBK;
  const int nslots = args.M * args.top_k;

  if (warp == 0) {
    // ------------------------------------------------ weight producer (both CTAs)
    if (lane == 0) {
      prefetch_tensor_map(&tm_a0);
      if (kUp) prefetch_tensor_map(&tm_a1);
    }
    int ka = 0;
    bool alive = true;
    for (int tile = pair; tile < total && alive; tile += npairs) {
      const TileCoord c = decode_tile<kNmax>(prefix, cnt, E, tile);
      const bool single_use = cnt[c.e] <= kNmax;
      const uint64_t pol = single_use ? l2_policy_evict_first() : l2_policy_evict_normal();
      const int base = c.e * args.rows_per_expert + static_cast<int>(rank) * kBM;
      const int row_a0 = kUp ? base + c.w * 2 * kBM : base + c.w * 4 * kBM;
      const int row_a1 = kUp ? row_a0 : row_a0 + 2 * kBM;
      for (int k = 0; k < nk; ++k, ++ka) {
        const int s = ka % kStagesA;
        bool ok = true;
        if (lane == 0) {
          ok = mbar_wait_bounded(&a_empty[s], ((ka / kStagesA) & 1) ^ 1, abort_flag);
          if (ok && leader) mbar_arrive_expect_tx(&a_full[s], 2 * C::kAStage);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          if (lane == 0) {
            *abort_flag = 1;
            set_error(args.err, kErrTimeout);
          }
          alive = false;
          break;
        }
        if (lane == 0 && leader && (k == 0 || k == nk - 1))
          MOE_TRACE_STAMP(kUp ? 0 : 1, tile, k == 0 ? 6 : 7, global_timer_ns());
        uint8_t* st = a_ring + s * C::kAStage;
        const uint32_t bar = cluster_addr(&a_full[s], 0);
        if (lane == 0)
          tma_load_2d_pair(&tm_a0, bar, st, k * kBK, row_a0, pol);
        else if (lane == 1)
          tma_load_2d_pair(kUp ? &tm_a1 : &tm_a0, bar, st + kBoxBytes, k * kBK, row_a1, pol);
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------ token-row producer (both CTAs)
    if (lane == 0) prefetch_tensor_map(&tm_b);
    const uint64_t pol_b = l2_policy_evict_normal();
    int kb = 0;
    bool alive = true;
    for (int tile = pair; tile < total && alive; tile += npairs) {
      const TileCoord c = decode_tile<kNmax>(prefix, cnt, E, tile);
      const int nrows = min(kNmax, cnt[c.e] - c.t * kNmax);
      const int N = (nrows + 15) & ~15;
      const int half = N / 2;
      const int row0 = args.expert_offsets[c.e] + c.t * kNmax + static_cast<int>(rank) * half;
      const int nbox = (half + kBRows - 1) / kBRows;
      // gathered: lane i copies rows 4i .. 4i + 3 of this CTA's half (rows past the expert's count take
      // token 0; their columns of the product are never stored)
      int tok[4] = {0, 0, 0, 0};
      if (kGatherB) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int r = 4 * lane + u;
          if (r < half && static_cast<int>(rank) * half + r < nrows) {
            const int id = args.sorted_ids[row0 + r];
            tok[u] = (id >= 0 && id < nslots) ? id / args.top_k : 0;
          }
        }
      }
      const uint32_t b_bytes = kGatherB ? 2u * half * kBK * 2 : 2u * nbox * kBRows * kBK * 2;
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
            set_error(args.err, kErrTimeout);
          }
          alive = false;
          break;
        }
        uint8_t* st = b_ring + s * C::kBStage;
        if (kGatherB) {
          if (4 * lane < half)
            tma_gather4_pair(&tm_b, cluster_addr(&b_full[s], 0), st + lane * 4 * kBK * 2, k * kBK, tok[0], tok[1],
                             tok[2], tok[3], pol_b);
        } else if (lane < nbox) {
          tma_load_2d_pair(&tm_b, cluster_addr(&b_full[s], 0), st + lane * kBRows * kBK * 2, k * kBK,
                           row0 + lane * kBRows, pol_b);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (leader only)
    if (leader && lane == 0) {
      int ka = 0, kb = 0, j = 0;
      bool alive = true;
      for (int tile = pair; tile < total && alive; tile += npairs, ++j) {
        const TileCoord c = decode_tile<kNmax>(prefix, cnt, E, tile);
        const int nrows = min(kNmax, cnt[c.e] - c.t * kNmax);
        const int N = (nrows + 15) & ~15;
        const uint32_t idesc = umma_idesc_bf16(2 * kBM, N);
#ifdef MOE_PAIR_TRACE
        {
          unsigned smid;
          asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
          MOE_TRACE_STAMP(kUp ? 0 : 1, tile, 0,
                          static_cast<unsigned long long>(c.e) | (static_cast<unsigned long long>(c.w) << 12) |
                              (static_cast<unsigned long long>(c.t) << 20) |
                              (static_cast<unsigned long long>(N) << 28) |
                              (static_cast<unsigned long long>(smid) << 48));
        }
#endif
        const int buf = j % C::kAccBufs;
        const int use = j / C::kAccBufs;
        if (!mbar_wait_bounded(&acc_empty[buf], (use & 1) ^ 1, abort_flag)) {
          *abort_flag = 1;
          set_error(args.err, kErrTimeout);
          break;
        }
        tc_fence_after_sync();
        MOE_TRACE_STAMP(kUp ? 0 : 1, tile, 1, global_timer_ns());
        const uint32_t d0 = tmem + buf * C::kAccCols;
        const uint32_t d1 = d0 + kNmax;
        for (int k = 0; k < nk; ++k, ++ka, ++kb) {
          const int sa = ka % kStagesA, sb = kb % kStagesB;
          if (!mbar_wait_bounded(&a_full[sa], (ka / kStagesA) & 1, abort_flag) ||
              !mbar_wait_bounded(&b_full[sb], (kb / kStagesB) & 1, abort_flag)) {
            *abort_flag = 1;
            set_error(args.err, kErrTimeout);
            alive = false;
            break;
          }
          tc_fence_after_sync();
          if (k == 0) MOE_TRACE_STAMP(kUp ? 0 : 1, tile, 2, global_timer_ns());
          const uint64_t da0 = umma_desc_sw128(a_ring + sa * C::kAStage);
          const uint64_t da1 = umma_desc_sw128(a_ring + sa * C::kAStage + kBoxBytes);
          const uint64_t db = umma_desc_sw128(b_ring + sb * C::kBStage);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint32_t acc = (k | kk) != 0 ? 1u : 0u;
            umma_bf16_pair(d0, da0 + 2 * kk, db + 2 * kk, idesc, acc);
            umma_bf16_pair(d1, da1 + 2 * kk, db + 2 * kk, idesc, acc);
          }
          umma_commit_pair(&a_empty[sa]);
          umma_commit_pair(&b_empty[sb]);
        }
        MOE_TRACE_STAMP(kUp ? 0 : 1, tile, 3, global_timer_ns());
        umma_commit_pair(&acc_full[buf]);  // also on an abort, so neither epilogue is left waiting
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------ epilogue (both CTAs: their own 128 rows)
    const int q = warp & 3;
    const int part_c = (warp - 4) >> 2;  // which of the four 16-column chunks of every 64 this warp drains
    int j = 0;
    for (int tile = pair; tile < total; tile += npairs, ++j) {
      const TileCoord c = decode_tile<kNmax>(prefix, cnt, E, tile);
      const int nrows = min(kNmax, cnt[c.e] - c.t * kNmax);
      const int N = (nrows + 15) & ~15;
      const int row0 = args.expert_offsets[c.e] + c.t * kNmax;
      const int buf = j % C::kAccBufs;
      bool ok = true;
      if (lane == 0) ok = mbar_wait_bounded(&acc_full[buf], (j / C::kAccBufs) & 1, abort_flag);
      if (lane == 0 && warp == 4 && leader) MOE_TRACE_STAMP(kUp ? 0 : 1, tile, 4, global_timer_ns());
      ok = __shfl_sync(0xffffffffu, ok, 0);
      tc_fence_after_sync();
      const bool go = __shfl_sync(0xffffffffu, ok && !*abort_flag, 0);
      if (!go) {
        if (lane == 0 && !ok) set_error(args.err, kErrTimeout);
        break;
      }
      const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16) + buf * C::kAccCols;
      const int colbase = kUp ? c.w * 2 * kBM + static_cast<int>(rank) * kBM
                              : c.w * 4 * kBM + static_cast<int>(rank) * kBM;
      // 1. drain: lane l holds column col0 + l (its tensor-memory lane) for the tokens of each of the
      //    warp's 16-column chunks; the results are packed as bf16 token pairs in registers and the
      //    accumulator is released at once, so the next tile's MMAs run while this tile is stored
      constexpr int kChunks = kNmax / 64;
      constexpr int kWords = kUp ? 8 : 16;  // bf16 token pairs per chunk (down: both 256-row halves)
      uint32_t pk[kChunks][kWords];
#pragma unroll
      for (int i = 0; i < kChunks; ++i) {
        const int cb = 16 * part_c + 64 * i;
        if (cb >= N) break;
        uint32_t v0[16], v1[16];
        tmem_load_16(lane_base + cb, v0);
        tmem_load_16(lane_base + kNmax + cb, v1);
        tmem_load_wait();
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          if (kUp) {
            pk[i][p] = pack_bf16x2(silu_mul(__uint_as_float(v0[2 * p]), __uint_as_float(v1[2 * p])),
                                   silu_mul(__uint_as_float(v0[2 * p + 1]), __uint_as_float(v1[2 * p + 1])));
          } else {
            pk[i][p] = pack_bf16x2(__uint_as_float(v0[2 * p]), __uint_as_float(v0[2 * p + 1]));
            pk[i][8 + p] = pack_bf16x2(__uint_as_float(v1[2 * p]), __uint_as_float(v1[2 * p + 1]));
          }
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0 && warp == 4 && leader) MOE_TRACE_STAMP(kUp ? 0 : 1, tile, 5, global_timer_ns());
      if (lane == 0) mbar_arrive_cluster(cluster_addr(&acc_empty[buf], 0));
      // 2. store: an 8 x 8 transpose of the packed words inside each group of 8 lanes gives lane
      //    (8 g + b) tokens 2b and 2b + 1 of the chunk at columns col0 + 8 g .. + 7: two 16-byte
      //    row stores per lane per 16 tokens
      const int g8 = lane >> 3, b8 = lane & 7;
      const int col8 = colbase + q * 32 + 8 * g8;
#pragma unroll
      for (int i = 0; i < kChunks; ++i) {
        const int cb = 16 * part_c + 64 * i;
        if (cb >= N) break;
        const int n0 = cb + 2 * b8, n1 = n0 + 1;
        int id0 = -1, id1 = -1;  // down: the slots these two tokens' rows go to
        if (!kUp) {
          if (n0 < nrows) id0 = args.sorted_ids[row0 + n0];
          if (n1 < nrows) id1 = args.sorted_ids[row0 + n1];
        }
#pragma unroll
        for (int half = 0; half < (kUp ? 1 : 2); ++half) {
          uint32_t w[8];
#pragma unroll
          for (int p = 0; p < 8; ++p) w[p] = pk[i][8 * half + p];
          transpose8x8(w, b8);
          const uint4 r0 = make_uint4(__byte_perm(w[0], w[1], 0x5410), __byte_perm(w[2], w[3], 0x5410),
                                      __byte_perm(w[4], w[5], 0x5410), __byte_perm(w[6], w[7], 0x5410));
          const uint4 r1 = make_uint4(__byte_perm(w[0], w[1], 0x7632), __byte_perm(w[2], w[3], 0x7632),
                                      __byte_perm(w[4], w[5], 0x7632), __byte_perm(w[6], w[7], 0x7632));
          if (kUp) {
            if (n0 < nrows)
              *reinterpret_cast<uint4*>(args.out + static_cast<size_t>(row0 + n0) * args.out_ld + col8) = r0;
            if (n1 < nrows)
              *reinterpret_cast<uint4*>(args.out + static_cast<size_t>(row0 + n1) * args.out_ld + col8) = r1;
          } else {
            const int cc = col8 + half * 2 * kBM;
            if (n0 < nrows && id0 >= 0 && id0 < nslots)
              *reinterpret_cast<uint4*>(args.out + static_cast<size_t>(id0) * args.out_ld + cc) = r0;
            if (n1 < nrows && id1 >= 0 && id1 < nslots)
              *reinterpret_cast<uint4*>(args.out + static_cast<size_t>(id1) * args.out_ld + cc) = r1;
          }
        }
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync_all();  // neither CTA leaves while the other may still use its shared or tensor memory
  if (warp == 1) tmem_dealloc_pair(tmem, 512);
}

template <bool kUp, int kNmax, int kStagesA, int kStagesB, bool kGatherB = false>
cudaError_t launch_pair(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b, const GroupedGemmArgs& args,
                        int num_sms, cudaStream_t stream) {
  using C = QCfg<kNmax, kStagesA, kStagesB>;
  auto kern = pair_gemm_kernel<kUp, kNmax, kStagesA, kStagesB, kGatherB>;
  int dev = 0;
  cudaError_t st = cudaGetDevice(&dev);
  if (st != cudaSuccess) return st;
  static bool done[64] = {};
  if (dev < 64 && !done[dev]) {
    st = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (st != cudaSuccess) return st;
    done[dev] = true;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms & ~1));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a0, a1, b, args);
}

}  // namespace

cudaError_t launch_pair_up(const CUtensorMap& w_gate, const CUtensorMap& w_up, const CUtensorMap& x_rows,
                           const GroupedGemmArgs& args, int nmax, int num_sms, cudaStream_t stream, bool gather_b) {
  if (args.rows_per_expert % (2 * kBM) != 0) return cudaErrorInvalidValue;
  if (gather_b) {
    if (nmax >= 256) return launch_pair<true, 256, 5, 3, true>(w_gate, w_up, x_rows, args, num_sms, stream);
    return launch_pair<true, 128, 5, 6, true>(w_gate, w_up, x_rows, args, num_sms, stream);
  }
  if (nmax >= 256) return launch_pair<true, 256, 5, 3>(w_gate, w_up, x_rows, args, num_sms, stream);
  return launch_pair<true, 128, 5, 6>(w_gate, w_up, x_rows, args, num_sms, stream);
}

cudaError_t launch_pair_down(const CUtensorMap& w_down, const CUtensorMap& h_rows, const GroupedGemmArgs& args,
                             int nmax, int num_sms, cudaStream_t stream) {
  if (args.rows_per_expert % (4 * kBM) != 0) return cudaErrorInvalidValue;
  if (nmax >= 256) return launch_pair<false, 256, 5, 3>(w_down, w_down, h_rows, args, num_sms, stream);
  return launch_pair<false, 128, 5, 6>(w_down, w_down, h_rows, args, num_sms, stream);
}

}  // namespace moe

#ifdef MOE_PAIR_TRACE
// Host access to the timeline of the last pair launches (trace build only).
extern "C" __attribute__((visibility("default"))) int moe_pair_trace_read(void* host, size_t bytes) {
  return cudaMemcpyFromSymbol(host, moe::g_pair_trace, bytes) == cudaSuccess ? 0 : 1;
}
extern "C" __attribute__((visibility("default"))) int moe_pair_trace_clear() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, moe::g_pair_trace) != cudaSuccess) return 1;
  return cudaMemset(p, 0, sizeof(moe::g_pair_trace)) == cudaSuccess ? 0 : 1;
}
#endif
