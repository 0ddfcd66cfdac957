// Persistent grouped expert projections for batch and prefill shapes
// ("[flashinfer] ... AlphaMoE NVFP4 커널 최적화", flashinfer PR #6511 analysis:
// the up / down kernels of the route chain, §6; wide weight panels streamed
// by TMA, §2; activation rows taken in plan order inside the GEMM, §4).
//
// Why a second kernel: when ~128 tokens route to each expert the weight panel
// of a CTA is used by a 128-wide token tile, and the weight stream only stays
// at HBM speed if enough weight bytes are in flight on every SM (bytes in
// flight / memory latency).  This kernel runs one CTA per SM over a static
// round-robin list of tiles and keeps the two operands in separate rings:
//
//   weights  A ring: kStagesA x (2 boxes of 128 rows x 64 bf16) = 32 KB a stage
//   tokens   B ring: kStagesB x (up to 128 plan rows x 64 bf16)  = 16 KB a stage
//
// each filled by its own producer warp, so the weight ring runs kStagesA
// stages ahead no matter how the token rows (L2 hits) arrive.  The MMA warp
// alternates between two accumulator sets in tensor memory (2 x 256 columns)
// and the epilogue warps drain one set while the next tile accumulates into
// the other, so the weight stream never stops between tiles (128-row tiles;
// 256-row tiles fill tensor memory and the rings keep streaming meanwhile).
//
// A tile = (expert e, weight tile w, token tile t), ordered e, then w, then t
// (fastest): consecutive CTAs work on the token tiles that share a weight
// panel at the same time, so the panel comes from HBM once.  Each tile
// computes two 128 x N accumulators:
//   up:   acc0 = x W_gate[e][128w..]^T, acc1 = x W_up[e][128w..]^T,
//         h[r, 128w + i] = bf16(silu(acc0) * acc1)
//   down: acc0 / acc1 = h W_down[e][256w.. / 256w+128..]^T,
//         y[slot, 256w + j] = bf16(acc)
// The token rows (B operand) are consecutive plan rows of a tensor already in
// plan order: x gathered by gather_rows_kernel (up) or h (down).
//
// Warp roles (384 threads): 0 = weight producer, 1 = MMA issuer (one lane),
// 2 = token-row producer, 3 = idle, 4..11 = epilogue (warp w reads tensor
// memory lanes 32(w%4)..+31, every other 16-column chunk).  All waits are
// bounded.
#include "common.cuh"
#include "kernels.h"
#include "tile_list.cuh"

namespace moe {
namespace {

constexpr int kBM = 128;                 // rows of one accumulator (MMA M)
constexpr int kBK = 64;                  // contraction elements per stage
constexpr int kBoxBytes = kBM * kBK * 2;  // one 128 x 64 bf16 box: 16 KB
constexpr int kBRows = 32;               // rows per token-row box
constexpr int kEpiWarps = 8;             // two warps per tensor-memory lane quarter
constexpr int kThreads = 128 + 32 * kEpiWarps;

// kNmax token rows per tile.  A tile's two accumulators take 2*kNmax
// tensor-memory columns, so 128-row tiles are double-buffered (the epilogue
// of one tile overlaps the next tile's mainloop) and 256-row tiles are not.
template <int kNmax, int kStagesA, int kStagesB>
struct PCfg {
  static constexpr int kAStage = 2 * kBoxBytes;
  static constexpr int kBStage = kNmax * kBK * 2;
  static constexpr int kAccCols = 2 * kNmax;
  static constexpr int kAccBufs = 512 / kAccCols;
  static constexpr int kMisc = 10240;    // barriers, flags, counts and tile prefix over experts (E <= 1024)
  static constexpr int kSmem = 1024 + kStagesA * kAStage + kStagesB * kBStage + kMisc;
  static_assert(kNmax == 128 || kNmax == 256, "tile widths");
  static_assert(kSmem <= 227 * 1024, "shared memory");
  static_assert(kSmem > 116 * 1024, "one CTA per SM: it owns all 512 tensor-memory columns");
};

// kGatherB (up only): the token-row producer gathers the rows of x itself
// with tile::gather4 (x stays in L2); otherwise tm_b maps a plan-ordered
// tensor read in 32-row boxes.
template <bool kUp, int kNmax, int kStagesA, int kStagesB, bool kGatherB>
__global__ void __launch_bounds__(kThreads, 1)
    persistent_gemm_kernel(const __grid_constant__ CUtensorMap tm_a0, const __grid_constant__ CUtensorMap tm_a1,
                           const __grid_constant__ CUtensorMap tm_b, const GroupedGemmArgs args) {
  using C = PCfg<kNmax, kStagesA, kStagesB>;
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
  uint64_t* acc_empty = acc_full + 2;       // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* cnt = const_cast<int*>(abort_flag + 1);  // [E]
  int* prefix = cnt + 1024;                     // [E + 1]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = args.E;
  // weight tiles per expert: up = 128 rows of gate and of up; down = 256 rows
  const int W = kUp ? args.rows_per_expert / kBM : args.rows_per_expert / (2 * kBM);

  // ---- per-expert tile counts and their prefix (the tile list)
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
      mbar_init(&acc_empty[b], kEpiWarps);  // one arrival per epilogue warp
    }
    fence_mbar_init();
  }
  __syncthreads();
  const int total = prefix[E];
  if (static_cast<int>(blockIdx.x) >= total) return;  // nothing for this CTA: leave before any async work
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int nk = args.kdim / kBK;
  const int nslots = args.M * args.top_k;

  if (warp == 0) {
    // ------------------------------------------------ weight producer
    // lane 0 waits for the slot and posts the byte count; lanes 0 and 1 then
    // issue one box each, so the two copies of a stage are issued in parallel.
    if (lane == 0) {
      prefetch_tensor_map(&tm_a0);
      if (kUp) prefetch_tensor_map(&tm_a1);
    }
    int ka = 0;
    bool alive = true;
    for (int tile = blockIdx.x; tile < total && alive; tile += gridDim.x) {
      const TileCoord c = decode_tile<kNmax>(prefix, cnt, E, tile);
      const bool single_use = cnt[c.e] <= kNmax;
      const uint64_t pol = single_use ? l2_policy_evict_first() : l2_policy_evict_normal();
      const int row_a0 = kUp ? c.e * args.rows_per_expert + c.w * kBM : c.e * args.rows_per_expert + c.w * 2 * kBM;
      const int row_a1 = kUp ? row_a0 : row_a0 + kBM;
      for (int k = 0; k < nk; ++k, ++ka) {
        const int s = ka % kStagesA;
        bool ok = true;
        if (lane == 0) {
          ok = mbar_wait_bounded(&a_empty[s], ((ka / kStagesA) & 1) ^ 1, abort_flag);
          if (ok) mbar_arrive_expect_tx(&a_full[s], C::kAStage);
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
        uint8_t* st = a_ring + s * C::kAStage;
        if (lane == 0)
          tma_load_2d_hint(&tm_a0, &a_full[s], st, k * kBK, row_a0, pol);
        else if (lane == 1)
          tma_load_2d_hint(kUp ? &tm_a1 : &tm_a0, &a_full[s], st + kBoxBytes, k * kBK, row_a1, pol);
      }
    }
    __syncwarp();
  } else if (warp == 2 && kGatherB) {
    // ------------------------------------------------ token-row producer (gather from x)
    // lane l owns plan rows 4l..4l+3 of the tile (two groups for 256-row tiles)
    constexpr int kGroups = kNmax / 128;
    if (lane == 0) prefetch_tensor_map(&tm_b);
    int kb = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const TileCoord c = decode_tile<kNmax>(prefix, cnt, E, tile);
      const int nrows = min(kNmax, cnt[c.e] - c.t * kNmax);
      const int N = (nrows + 15) & ~15;
      const int row0 = args.expert_offsets[c.e] + c.t * kNmax;
      int rows[kGroups][4];
#pragma unroll
      for (int g = 0; g < kGroups; ++g)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int n = 128 * g + 4 * lane + i;
          int r = 0;  // padding rows read token 0; their columns are never stored
          if (n < nrows) {
            const int id = args.sorted_ids[row0 + n];
            if (id >= 0 && id < nslots) r = id / args.top_k;
          }
          rows[g][i] = r;
        }
      bool alive = true;
      for (int k = 0; k < nk; ++k, ++kb) {
        const int s = kb % kStagesB;
        bool ok = true;
        if (lane == 0) {
          ok = mbar_wait_bounded(&b_empty[s], ((kb / kStagesB) & 1) ^ 1, abort_flag);
          if (ok) mbar_arrive_expect_tx(&b_full[s], N * kBK * 2);
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
#pragma unroll
        for (int g = 0; g < kGroups; ++g)
          if (128 * g + 4 * lane < N)
            tma_gather4(&tm_b, &b_full[s], st + (128 * g + 4 * lane) * kBK * 2, k * kBK, rows[g][0], rows[g][1],
                        rows[g][2], rows[g][3]);
      }
      if (!alive) break;
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------ token-row producer (plan-ordered rows)
    // lane 0 waits and posts the byte count; lane i issues box i.
    if (lane == 0) prefetch_tensor_map(&tm_b);
    int kb = 0;
    bool alive = true;
    for (int tile = blockIdx.x; tile < total && alive; tile += gridDim.x) {
      const TileCoord c = decode_tile<kNmax>(prefix, cnt, E, tile);
      const int nrows = min(kNmax, cnt[c.e] - c.t * kNmax);
      const int row0 = args.expert_offsets[c.e] + c.t * kNmax;
      const int nbox = (nrows + kBRows - 1) / kBRows;
      for (int k = 0; k < nk; ++k, ++kb) {
        const int s = kb % kStagesB;
        bool ok = true;
        if (lane == 0) {
          ok = mbar_wait_bounded(&b_empty[s], ((kb / kStagesB) & 1) ^ 1, abort_flag);
          if (ok) mbar_arrive_expect_tx(&b_full[s], nbox * kBRows * kBK * 2);
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
        if (lane < nbox)
          tma_load_2d(&tm_b, &b_full[s], st + lane * kBRows * kBK * 2, k * kBK, row0 + lane * kBRows);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      int ka = 0, kb = 0, j = 0;
      bool alive = true;
      for (int tile = blockIdx.x; tile < total && alive; tile += gridDim.x, ++j) {
        const TileCoord c = decode_tile<kNmax>(prefix, cnt, E, tile);
        const int nrows = min(kNmax, cnt[c.e] - c.t * kNmax);
        const int N = (nrows + 15) & ~15;
        const uint32_t idesc = umma_idesc_bf16(kBM, N);
        const int buf = j % C::kAccBufs;
        const int use = j / C::kAccBufs;
        if (!mbar_wait_bounded(&acc_empty[buf], (use & 1) ^ 1, abort_flag)) {
          *abort_flag = 1;
          set_error(args.err, kErrTimeout);
          break;
        }
        tc_fence_after_sync();
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
          const uint64_t da0 = umma_desc_sw128(a_ring + sa * C::kAStage);
          const uint64_t da1 = umma_desc_sw128(a_ring + sa * C::kAStage + kBoxBytes);
          const uint64_t db = umma_desc_sw128(b_ring + sb * C::kBStage);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint32_t acc = (k | kk) != 0 ? 1u : 0u;
            umma_bf16_ss(d0, da0 + 2 * kk, db + 2 * kk, idesc, acc);
            umma_bf16_ss(d1, da1 + 2 * kk, db + 2 * kk, idesc, acc);
          }
          umma_commit(&a_empty[sa]);
          umma_commit(&b_empty[sb]);
        }
        umma_commit(&acc_full[buf]);  // also on an abort, so the epilogue is not left waiting
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------ epilogue
    const int q = warp & 3;             // tensor-memory lane quarter this warp may read
    const int half = (warp - 4) >> 2;   // which 16-column chunks: 2i + half
    int j = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++j) {
      const TileCoord c = decode_tile<kNmax>(prefix, cnt, E, tile);
      const int nrows = min(kNmax, cnt[c.e] - c.t * kNmax);
      const int N = (nrows + 15) & ~15;
      const int row0 = args.expert_offsets[c.e] + c.t * kNmax;
      const int buf = j % C::kAccBufs;
      bool ok = true;
      if (lane == 0) ok = mbar_wait_bounded(&acc_full[buf], (j / C::kAccBufs) & 1, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      tc_fence_after_sync();
      const bool go = __shfl_sync(0xffffffffu, ok && !*abort_flag, 0);
      if (!go) {
        if (lane == 0 && !ok) set_error(args.err, kErrTimeout);
        break;
      }
      const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16) + buf * C::kAccCols;
      int ids[kNmax / 32];  // lane l holds the slot ids of rows l, l+32, ...
      if (!kUp) {
#pragma unroll
        for (int i = 0; i < kNmax / 32; ++i) {
          const int n = lane + 32 * i;
          ids[i] = (n < nrows) ? args.sorted_ids[row0 + n] : -1;
        }
      }
      auto* out = reinterpret_cast<__nv_bfloat16*>(args.out);
      for (int cb = 16 * half; cb < N; cb += 32) {
        uint32_t v0[16], v1[16];
        tmem_load_16(lane_base + cb, v0);
        tmem_load_16(lane_base + kNmax + cb, v1);
        tmem_load_wait();
        const int id_word = kUp ? 0 : pick<kNmax / 32>(ids, cb >> 5);
#pragma unroll
        for (int qq = 0; qq < 16; ++qq) {
          const int n = cb + qq;
          if (kUp) {
            if (n < nrows) {
              const float g = __uint_as_float(v0[qq]);
              const float u = __uint_as_float(v1[qq]);
              const int col = c.w * kBM + q * 32 + lane;
              out[static_cast<size_t>(row0 + n) * args.out_ld + col] = __float2bfloat16_rn(g / (1.0f + expf(-g)) * u);
            }
          } else {
            const int id = __shfl_sync(0xffffffffu, id_word, (cb & 31) + qq);
            if (n < nrows && id >= 0 && id < nslots) {
              const int col = c.w * 2 * kBM + q * 32 + lane;
              out[static_cast<size_t>(id) * args.out_ld + col] = __float2bfloat16_rn(__uint_as_float(v0[qq]));
              out[static_cast<size_t>(id) * args.out_ld + col + kBM] = __float2bfloat16_rn(__uint_as_float(v1[qq]));
            }
          }
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_one(&acc_empty[buf]);
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <bool kUp, int kNmax, int kStagesA, int kStagesB, bool kGatherB>
cudaError_t launch_persistent(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b,
                              const GroupedGemmArgs& args, int num_sms, cudaStream_t stream) {
  using C = PCfg<kNmax, kStagesA, kStagesB>;
  auto kern = persistent_gemm_kernel<kUp, kNmax, kStagesA, kStagesB, kGatherB>;
  int dev = 0;
  cudaError_t st = cudaGetDevice(&dev);
  if (st != cudaSuccess) return st;
  static bool done[64] = {};
  if (dev < 64 && !done[dev]) {
    st = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (st != cudaSuccess) return st;
    done[dev] = true;
  }
  kern<<<num_sms, kThreads, C::kSmem, stream>>>(a0, a1, b, args);
  return cudaGetLastError();
}

}  // namespace

// Ring shapes: `deep_b` trades one weight stage for two more token-row stages.
cudaError_t launch_persistent_up(const CUtensorMap& w_gate, const CUtensorMap& w_up, const CUtensorMap& x_rows,
                                 const GroupedGemmArgs& args, int nmax, bool gather, bool deep_b, int num_sms,
                                 cudaStream_t stream) {
  if (nmax >= 256) {
    if (gather) return launch_persistent<true, 256, 4, 2, true>(w_gate, w_up, x_rows, args, num_sms, stream);
    return launch_persistent<true, 256, 4, 2, false>(w_gate, w_up, x_rows, args, num_sms, stream);
  }
  if (gather) {
    if (deep_b) return launch_persistent<true, 128, 4, 5, true>(w_gate, w_up, x_rows, args, num_sms, stream);
    return launch_persistent<true, 128, 5, 3, true>(w_gate, w_up, x_rows, args, num_sms, stream);
  }
  if (deep_b) return launch_persistent<true, 128, 4, 5, false>(w_gate, w_up, x_rows, args, num_sms, stream);
  return launch_persistent<true, 128, 5, 3, false>(w_gate, w_up, x_rows, args, num_sms, stream);
}

cudaError_t launch_persistent_down(const CUtensorMap& w_down, const CUtensorMap& h_rows, const GroupedGemmArgs& args,
                                   int nmax, bool deep_b, int num_sms, cudaStream_t stream) {
  if (nmax >= 256) return launch_persistent<false, 256, 4, 2, false>(w_down, w_down, h_rows, args, num_sms, stream);
  if (deep_b) return launch_persistent<false, 128, 4, 5, false>(w_down, w_down, h_rows, args, num_sms, stream);
  return launch_persistent<false, 128, 5, 3, false>(w_down, w_down, h_rows, args, num_sms, stream);
}

}  // namespace moe
