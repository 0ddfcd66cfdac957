// Grouped expert projections on the 5th-generation tensor cores (tcgen05 +
// tensor memory), fed by TMA, over the expert-major plan
// ("[flashinfer] ... AlphaMoE NVFP4 커널 최적화", flashinfer PR #6511 analysis:
// §3-§4 the up kernels, §1-§2 the down kernels, §6 the route chain
// up -> down -> finalize over the plan of §5).
//
// Orientation ("swap AB"): the weight rows are the MMA's M side (128 rows of
// one expert's W per CTA) and the routed tokens are its N side, so one CTA
// streams a 128 x K panel of weights through shared memory once and applies
// it to every token of its tile.  For decode-sized problems the token side is
// 16..32 wide and the kernel is a weight stream at HBM speed; for prefill the
// token side grows to 128 and the same kernel becomes a dense contraction.
//
// Work unit = (token tile, weight tile).  Token tiles are consecutive plan
// rows of one expert, at most NMAX wide: expert e owns ceil(count[e]/NMAX)
// tiles over its real rows (padding rows of the plan are never computed; the
// MMA width N is the tile's row count rounded up to 16, which stays inside
// the expert's padded segment because the block size is a multiple of 16).
// grid.x = weight tiles (fastest, so CTAs launched together share the token
// tile in L2), grid.y = an upper bound on the token tiles computed on the host
// without reading the plan back; CTAs past the real count exit at once.
//
// Roles in a 128-thread CTA:
//   warp 0       TMA producer: waits for a free stage, posts the expected
//                bytes, loads the weight tile(s) (one 128x64 bf16 box each) and
//                the token rows: up = x rows gathered by token id with
//                tile::gather4 (4 rows per copy), down = h rows (contiguous
//                plan rows, 16-row boxes).
//   warp 1 / t0  MMA issuer: 4 tcgen05.mma (K = 16 each) per 64-wide stage,
//                per accumulator; tcgen05.commit frees the stage.
//   warps 0-3    epilogue: tcgen05.ld of the fp32 accumulators (warp w owns
//                tensor-memory lanes 32w..32w+31 = weight rows), then
//                up:   h[row, i] = bf16(silu(gate) * up)   (fused SwiGLU)
//                down: y[slot, j] = bf16(acc), scattered to the slot id.
// Every wait is bounded; a timeout sets the error word and unwinds.
//
// Self-routing (kRoute, decode up only; flashinfer PR #6511 analysis, §6:
// the align launch folded into the first GEMM of the chain): instead of
// reading the plan, every CTA stages topk_ids (M*top_k <= kRouteMaxSlots) in
// shared memory, counts the slots per expert, finds its tile as above, takes
// the padded prefix of its expert and the slot ids of its token tile (one warp,
// ascending slot order, ballots), and writes its part of the plan: the rows
// and padding of its token tile (weight tile 0 only), and, in CTA 0, the
// counts, offsets, block -> expert map and padded total.  The plan is the one
// moe_align_block_size writes, bit for bit.
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kBM = 128;        // weight rows per CTA (MMA M)
constexpr int kBK = 64;         // contraction elements per stage = one 128-byte swizzle row
constexpr int kATile = kBM * kBK * 2;

constexpr int pow2_at_least(int v) {
  int p = 32;
  while (p < v) p <<= 1;
  return p;
}

template <bool kUp, int kNmax, int kStages>
struct Cfg {
  static constexpr int kBTile = kNmax * kBK * 2;
  static constexpr int kAPerStage = kUp ? 2 : 1;
  static constexpr int kStageBytes = kATile * kAPerStage + kBTile;
  static constexpr int kTmemCols = pow2_at_least(kUp ? 2 * kNmax : kNmax);
  static constexpr int kMiscBytes = (128 + 4 * kNmax + 1023) / 1024 * 1024;  // barriers, flags, token ids
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kMiscBytes;
  static_assert(kBTile % 1024 == 0, "token tile must keep 1024-byte alignment");
  static_assert(kNmax % 16 == 0 && kNmax <= 256, "MMA N limits");
  static_assert(kTmemCols <= 512, "tensor memory has 512 columns");
  // A CTA that takes more than half of tensor memory must also take more than
  // half of shared memory, so that no second CTA is resident to wait on it.
  static_assert(kTmemCols <= 256 || kSmemBytes > 116 * 1024, "tensor memory / occupancy mismatch");
};

// kGatherB: the token rows of the B operand are gathered from x by token id
// (tile::gather4); otherwise they are consecutive plan rows of a tensor that
// is already in plan order (h, or x gathered by gather_rows_kernel).
template <bool kUp, int kNmax, int kStages, bool kGatherB, bool kRoute>
__global__ void __launch_bounds__(128, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_a0, const __grid_constant__ CUtensorMap tm_a1,
                        const __grid_constant__ CUtensorMap tm_b, const GroupedGemmArgs args) {
  using C = Cfg<kUp, kNmax, kStages>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint8_t* misc = smem + kStages * C::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(misc);
  uint64_t* empty = full + kStages;
  uint64_t* accf = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* info = const_cast<int*>(reinterpret_cast<volatile int*>(abort_flag + 1));  // expert, token tile, weight tile
  int* tok = info + 4;                                                           // [kNmax]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = args.E;
  const int W = args.rows_per_expert / kBM;  // weight tiles per expert

  // ---- which (expert, weight tile, token tile) this CTA computes.  CTAs are
  // ordered expert by expert, then weight tile, then token tile (fastest), so
  // the token tiles that stream the same weight panel start together and the
  // panel is fetched from HBM once and shared through L2.
  int* cnt = reinterpret_cast<int*>(stages);  // scratch before the pipeline starts (E <= 1024)
  int* ids_s = cnt + 1024;                    // self-routing: topk_ids [M*top_k]
  int* pre = ids_s + kRouteMaxSlots;          // self-routing, CTA 0: padded prefix [E+1]
  int* slot_s = pre + 1025;                   // self-routing: slot ids of this token tile [kNmax]
  const int nslots = args.M * args.top_k;
  if (kRoute) {
    for (int e = tid; e < E; e += 128) cnt[e] = 0;
  } else {
    for (int e = tid; e < E; e += 128) cnt[e] = args.expert_counts[e];
  }
  if (tid == 0) {
    info[0] = -1;
    info[1] = 0;
    info[2] = 0;
    info[3] = 0;
    *abort_flag = 0;
  }
  __syncthreads();
  if (kRoute) {
    for (int f = tid; f < nslots; f += 128) {
      const int id = args.topk_ids[f];
      ids_s[f] = id;
      if (id >= 0 && id < E)
        atomicAdd(&cnt[id], 1);
      else
        set_error(args.err, kErrInvalidInput);
    }
    __syncthreads();
    const int B = args.block_size;
    if (blockIdx.x == 0) {
      // the plan header: counts, padded exclusive prefix, total, block -> expert
      if (warp == 0) {
        const int per = (E + 31) / 32;
        const int lo = min(E, lane * per), hi = min(E, lo + per);
        int sum = 0;
        for (int e = lo; e < hi; ++e) sum += (cnt[e] + B - 1) / B * B;
        int incl = sum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += v;
        }
        int run = incl - sum;
        for (int e = lo; e < hi; ++e) {
          pre[e] = run;
          run += (cnt[e] + B - 1) / B * B;
        }
        if (lane == 31) pre[E] = incl;
      }
      __syncthreads();
      for (int e = tid; e <= E; e += 128) args.plan_offsets[e] = pre[e];
      for (int e = tid; e < E; e += 128) {
        args.plan_counts[e] = cnt[e];
        for (int b = pre[e] / B; b < pre[e + 1] / B; ++b) args.plan_block_expert[b] = e;
      }
      if (tid == 0) *args.plan_ntpp = pre[E];
    }
  }
  if (warp == 0) {
    const int linear = blockIdx.x;
    const int per = (E + 31) / 32;
    const int lo = min(E, lane * per), hi = min(E, lo + per);
    int sum = 0;
    for (int e = lo; e < hi; ++e) sum += W * ((cnt[e] + kNmax - 1) / kNmax);
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    const int excl = incl - sum;
    if (linear >= excl && linear < incl) {
      int t = excl;
      for (int e = lo; e < hi; ++e) {
        const int ntiles = (cnt[e] + kNmax - 1) / kNmax;
        if (linear < t + W * ntiles) {
          const int rel = linear - t;
          info[0] = e;
          info[1] = rel % ntiles;
          info[2] = rel / ntiles;
          break;
        }
        t += W * ntiles;
      }
    }
  }
  __syncthreads();
  const int e = info[0];
  if (e < 0) return;  // past the real tile count: the whole CTA leaves before any async work
  const int local = info[1];
  const int wt = info[2];
  const int count_e = cnt[e];
  const int nrows = min(kNmax, count_e - local * kNmax);
  if (kRoute) {
    const int B = args.block_size;
    if (warp == 0) {
      // padded offset of expert e
      const int per = (E + 31) / 32;
      const int lo = min(e, lane * per), hi = min(e, lo + per);
      int sum = 0;
      for (int q = lo; q < hi; ++q) sum += (cnt[q] + B - 1) / B * B;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      if (lane == 0) info[3] = sum;
      // slot ids of token tile `local` of expert e, in ascending slot order
      const unsigned lt_mask = (1u << lane) - 1u;
      const int first = local * kNmax;
      int seen = 0;
      for (int base = 0; base < nslots && seen < first + nrows; base += 32) {
        const int f = base + lane;
        const bool m = f < nslots && ids_s[f] == e;
        const unsigned bal = __ballot_sync(0xffffffffu, m);
        const int pos = seen + __popc(bal & lt_mask);
        if (m && pos >= first && pos < first + nrows) slot_s[pos - first] = f;
        seen += __popc(bal);
      }
    }
    __syncthreads();
  }
  const int off_e = kRoute ? info[3] : args.expert_offsets[e];
  const int row0 = off_e + local * kNmax;
  const int N = (nrows + 15) & ~15;
  if (kRoute && wt == 0) {
    // this token tile's rows of the plan, and the expert's padding after its last tile
    for (int n = tid; n < nrows; n += 128) args.plan_sorted_ids[row0 + n] = slot_s[n];
    if (local == (count_e - 1) / kNmax) {
      const int B = args.block_size;
      const int pad_end = off_e + (count_e + B - 1) / B * B;
      for (int p = off_e + count_e + tid; p < pad_end; p += 128) args.plan_sorted_ids[p] = nslots;
    }
  }
  for (int n = tid; n < N; n += 128) {
    int v = (kUp && kGatherB) ? 0 : -1;
    if (n < nrows) {
      const int id = kRoute ? slot_s[n] : args.sorted_ids[row0 + n];
      if (id >= 0 && id < nslots) {
        v = (kUp && kGatherB) ? id / args.top_k : id;
      } else {
        set_error(args.err, kErrInvalidInput);
      }
    }
    tok[n] = v;
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();  // also retires the use of `cnt` before TMA writes the stages
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  const int nk = args.kdim / kBK;
  const int a_row = e * args.rows_per_expert + wt * kBM;
  const uint32_t b_bytes = static_cast<uint32_t>(N) * kBK * 2;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensor_map(&tm_a0);
      if (kUp) prefetch_tensor_map(&tm_a1);
      prefetch_tensor_map(&tm_b);
    }
    // A weight panel used by one token tile only is streamed with an
    // evict-first hint; an expert with several token tiles re-reads its panel
    // from L2, so those loads keep the normal policy.
    const bool single_use = count_e <= kNmax;
    const uint64_t pol_w = single_use ? l2_policy_evict_first() : l2_policy_evict_normal();
    int issued = 0;
    for (int k = 0; k < nk; ++k) {
      const int s = k % kStages;
      const uint32_t ph = (k / kStages) & 1;
      bool free_slot = true;
      if (lane == 0) free_slot = mbar_wait_bounded(&empty[s], ph ^ 1, abort_flag);
      free_slot = __shfl_sync(0xffffffffu, free_slot, 0);  // one decision for the whole warp
      if (!free_slot) {
        if (lane == 0) {
          *abort_flag = 1;
          set_error(args.err, kErrTimeout);
        }
        break;
      }
      uint8_t* st = stages + s * C::kStageBytes;
      uint8_t* bt = st + kATile * C::kAPerStage;
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[s], kATile * C::kAPerStage + b_bytes);
        tma_load_2d_hint(&tm_a0, &full[s], st, k * kBK, a_row, pol_w);
        if (kUp) tma_load_2d_hint(&tm_a1, &full[s], st + kATile, k * kBK, a_row, pol_w);
      }
      __syncwarp();
      if (kGatherB) {
        for (int i = lane; i < N / 4; i += 32)
          tma_gather4(&tm_b, &full[s], bt + i * 4 * (kBK * 2), k * kBK, tok[4 * i], tok[4 * i + 1], tok[4 * i + 2],
                      tok[4 * i + 3]);
      } else {
        for (int i = lane; i < N / 16; i += 32)
          tma_load_2d(&tm_b, &full[s], bt + i * 16 * (kBK * 2), k * kBK, row0 + 16 * i);
      }
      issued = k + 1;
    }
    // Do not leave while copies issued by this CTA may still land.
    if (lane == 0) {
      for (int k = max(0, issued - kStages); k < issued; ++k) {
        const int s = k % kStages;
        if (!mbar_wait_bounded(&full[s], (k / kStages) & 1, nullptr)) {
          set_error(args.err, kErrTimeout);
          break;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(kBM, N);
      for (int k = 0; k < nk; ++k) {
        const int s = k % kStages;
        const uint32_t ph = (k / kStages) & 1;
        if (!mbar_wait_bounded(&full[s], ph, abort_flag)) {
          *abort_flag = 1;
          set_error(args.err, kErrTimeout);
          break;
        }
        tc_fence_after_sync();
        uint8_t* st = stages + s * C::kStageBytes;
        const uint64_t da0 = umma_desc_sw128(st);
        const uint64_t db = umma_desc_sw128(st + kATile * C::kAPerStage);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint32_t acc = (k | kk) != 0 ? 1u : 0u;
          umma_bf16_ss(tmem, da0 + 2 * kk, db + 2 * kk, idesc, acc);
          if (kUp) {
            const uint64_t da1 = umma_desc_sw128(st + kATile);
            umma_bf16_ss(tmem + kNmax, da1 + 2 * kk, db + 2 * kk, idesc, acc);
          }
        }
        umma_commit(&empty[s]);
      }
      umma_commit(accf);
    }
    __syncwarp();
  }

  // ---------------------------------------------------- epilogue (all warps)
  bool ok = true;
  if (lane == 0) ok = mbar_wait_bounded(accf, 0, nullptr);
  ok = __shfl_sync(0xffffffffu, ok, 0);
  tc_fence_after_sync();
  if (!ok && lane == 0) set_error(args.err, kErrTimeout);
  const bool go = __shfl_sync(0xffffffffu, ok && !*abort_flag, 0);
  if (go) {
    const int wrow = wt * kBM + warp * 32 + lane;  // output column: I index (up) or H index (down)
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    for (int c = 0; c < N; c += 16) {
      uint32_t d0[16];
      tmem_load_16(lane_base + c, d0);
      if (kUp) {
        uint32_t d1[16];
        tmem_load_16(lane_base + kNmax + c, d1);
        tmem_load_wait();
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const int n = c + q;
          if (n < nrows) {
            const float g = __uint_as_float(d0[q]);
            const float u = __uint_as_float(d1[q]);
            const float hv = g / (1.0f + expf(-g)) * u;
            reinterpret_cast<__nv_bfloat16*>(args.out)[static_cast<size_t>(row0 + n) * args.out_ld + wrow] =
                __float2bfloat16_rn(hv);
          }
        }
      } else {
        tmem_load_wait();
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const int n = c + q;
          if (n < nrows) {
            const int slot = tok[n];
            if (slot >= 0)
              reinterpret_cast<__nv_bfloat16*>(args.out)[static_cast<size_t>(slot) * args.out_ld + wrow] =
                  __float2bfloat16_rn(__uint_as_float(d0[q]));
          }
        }
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

template <bool kUp, int kNmax, int kStages, bool kGatherB, bool kRoute = false>
cudaError_t launch_variant(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b,
                           const GroupedGemmArgs& args, cudaStream_t stream) {
  using C = Cfg<kUp, kNmax, kStages>;
  static_assert(!kRoute || (kUp && kGatherB), "self-routing: up projection with gathered x rows only");
  static_assert(!kRoute || (1024 + kRouteMaxSlots + 1025 + kNmax) * 4 <= kStages * C::kStageBytes,
                "self-routing scratch fits in the stage buffers");
  auto kern = grouped_gemm_kernel<kUp, kNmax, kStages, kGatherB, kRoute>;
  int dev = 0;
  cudaError_t st = cudaGetDevice(&dev);
  if (st != cudaSuccess) return st;
  static bool done[64] = {};
  if (dev < 64 && !done[dev]) {
    st = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (st != cudaSuccess) return st;
    done[dev] = true;
  }
  const long long mk = static_cast<long long>(args.M) * args.top_k;
  const long long tiles_ub = mk / kNmax + (mk < args.E ? mk : args.E);
  const unsigned grid = static_cast<unsigned>((args.rows_per_expert / kBM) * tiles_ub);
  kern<<<grid, 128, C::kSmemBytes, stream>>>(a0, a1, b, args);
  return cudaGetLastError();
}

// xg[r, :] = x[sorted_ids[r] / top_k, :] for every real plan row r (padding
// rows are skipped): one warp per row, 16-byte loads and stores, issued in
// batches of kGatherBatch loads per lane before their stores, so that a lane
// has that many reads in flight instead of one (a row of 7168 bf16 is 28
// loads per lane).
constexpr int kGatherBatch = 7;

__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ x, const int32_t* sorted_ids,
                                                          const int32_t* ntpp, int nslots, int top_k, int row_vecs,
                                                          int cap, uint4* __restrict__ xg) {
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= cap || r >= *ntpp) return;
  const int id = sorted_ids[r];
  if (id < 0 || id >= nslots) return;
  const uint4* src = x + static_cast<size_t>(id / top_k) * row_vecs;
  uint4* dst = xg + static_cast<size_t>(r) * row_vecs;
  for (int i0 = lane; i0 < row_vecs; i0 += 32 * kGatherBatch) {
    uint4 v[kGatherBatch];
#pragma unroll
    for (int b = 0; b < kGatherBatch; ++b) {
      const int i = i0 + 32 * b;
      if (i < row_vecs) v[b] = src[i];
    }
#pragma unroll
    for (int b = 0; b < kGatherBatch; ++b) {
      const int i = i0 + 32 * b;
      if (i < row_vecs) dst[i] = v[b];
    }
  }
}

}  // namespace

cudaError_t launch_grouped_up(const CUtensorMap& w_gate, const CUtensorMap& w_up, const CUtensorMap& x_rows,
                              const GroupedGemmArgs& args, int nmax, bool gathered, cudaStream_t stream) {
  if (gathered) {
    if (nmax <= 32) return launch_variant<true, 32, 3, false>(w_gate, w_up, x_rows, args, stream);
    if (nmax <= 128) return launch_variant<true, 128, 2, false>(w_gate, w_up, x_rows, args, stream);
    return launch_variant<true, 256, 3, false>(w_gate, w_up, x_rows, args, stream);
  }
  if (nmax <= 32) return launch_variant<true, 32, 3, true>(w_gate, w_up, x_rows, args, stream);
  if (nmax <= 128) return launch_variant<true, 128, 2, true>(w_gate, w_up, x_rows, args, stream);
  return launch_variant<true, 256, 3, true>(w_gate, w_up, x_rows, args, stream);
}

cudaError_t launch_grouped_up_routed(const CUtensorMap& w_gate, const CUtensorMap& w_up, const CUtensorMap& x_rows,
                                     const GroupedGemmArgs& args, cudaStream_t stream) {
  if (args.M * args.top_k > kRouteMaxSlots || args.E > 1024) return cudaErrorInvalidValue;
  return launch_variant<true, 32, 3, true, true>(w_gate, w_up, x_rows, args, stream);
}

cudaError_t launch_grouped_down(const CUtensorMap& w_down, const CUtensorMap& h_rows, const GroupedGemmArgs& args,
                                int nmax, cudaStream_t stream) {
  if (nmax <= 32) return launch_variant<false, 32, 5, false>(w_down, w_down, h_rows, args, stream);
  if (nmax <= 128) return launch_variant<false, 128, 3, false>(w_down, w_down, h_rows, args, stream);
  return launch_variant<false, 256, 4, false>(w_down, w_down, h_rows, args, stream);
}

cudaError_t launch_gather_rows(const uint16_t* x, const int32_t* sorted_ids, const int32_t* ntpp, int M, int top_k,
                               int H, int cap, uint16_t* xg, cudaStream_t stream) {
  gather_rows_kernel<<<(cap + 7) / 8, 256, 0, stream>>>(reinterpret_cast<const uint4*>(x), sorted_ids, ntpp,
                                                        M * top_k, top_k, H / 8, cap, reinterpret_cast<uint4*>(xg));
  return cudaGetLastError();
}

}  // namespace moe
