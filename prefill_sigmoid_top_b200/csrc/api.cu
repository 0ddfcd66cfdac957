// C-ABI entry points of libmoe_b200.so (declared and documented in
// include/moe_b200.h): host-side validation, TMA tensor-map encoding,
// workspace layout, and the launch sequence of the layer.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "moe_b200.h"
#include "moe_b200_tp.h"
#include "common.cuh"
#include "kernels.h"

namespace {

using moe::GroupedGemmArgs;

constexpr size_t kAlign = 256;

size_t align_up(size_t v, size_t a = kAlign) { return (v + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

moe_status_t check_shape(const moe_shape_t& s) {
  if (s.M < 1 || s.H < 256 || s.I < 128 || s.E < 1 || s.top_k < 1 || s.block_size < 1) return MOE_ERR_UNSUPPORTED;
  if (s.H % 256 != 0 || s.H > 8192) return MOE_ERR_UNSUPPORTED;
  if (s.I % 128 != 0 || s.I > 65536) return MOE_ERR_UNSUPPORTED;
  if (s.E > 1024 || s.top_k > s.E || s.top_k > 32) return MOE_ERR_UNSUPPORTED;
  if (!is_pow2(s.block_size) || s.block_size < 16 || s.block_size > 256) return MOE_ERR_UNSUPPORTED;
  const long long mk = static_cast<long long>(s.M) * s.top_k;
  const long long cap = mk + static_cast<long long>(s.E) * (s.block_size - 1);
  if (cap >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// ------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 tensor [rows, cols] (cols contiguous) read in boxes of
// box_rows x 64 elements (128 bytes) with the 128-byte swizzle.
bool make_map_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D byte tensor [rows, cols_bytes] read in boxes of box_rows x 128 bytes
// with the 128-byte swizzle (packed e2m1 codes: 256 elements per box row).
bool make_map_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols_bytes, uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols_bytes, rows};
  cuuint64_t strides[1] = {cols_bytes};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// NVFP4 scale atoms ([blocks][kdim/64][512 bytes]) as a 2-D byte tensor of
// 256-byte rows, read in boxes of 8 rows (one stage's four atoms, 2 KB) with
// no swizzle: the shared-memory copy is the global bytes in order.
bool make_map_sf(CUtensorMap* map, const void* base, uint64_t bytes, uint32_t box_rows = 8) {
  auto fn = encode_fn();
  if (fn == nullptr || bytes % (256 * box_rows) != 0) return false;
  cuuint64_t dims[2] = {256, bytes / 256};
  cuuint64_t strides[1] = {256};
  cuuint32_t box[2] = {256, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Token-tile width of the single-SM grouped kernels, from the mean routed rows
// per expert (known on the host without reading the plan back): decode shapes
// (<= 24) use 32-row tiles, larger ones 128-row tiles (which also selects the
// persistent path; there the 2-SM pair kernels pick their own width, see
// pair_nmax).  Single-SM 256-row tiles measured slower on the batch and
// prefill workloads (one accumulator set fills tensor memory), so they run
// only when asked for.  MOE_GEMM_NMAX=32|128|256 overrides (the tests cover
// every variant).
int choose_nmax(const moe_shape_t& s) {
  if (const char* env = std::getenv("MOE_GEMM_NMAX")) {
    const int v = std::atoi(env);
    if (v == 32 || v == 128 || v == 256) return v;
  }
  const double per_expert = static_cast<double>(s.M) * s.top_k / s.E;
  return per_expert <= 24.0 ? 32 : 128;
}

size_t cap_rows(const moe_shape_t& s) {
  return static_cast<size_t>(s.M) * s.top_k + static_cast<size_t>(s.E) * (s.block_size - 1);
}

// Whether the up projection first gathers x into plan order (one pass over
// the routed rows) and then reads it as contiguous 16-row boxes, instead of
// gathering the rows inside the GEMM with tile::gather4.  The in-GEMM gather
// issues one copy per 4 rows per 64-column stage, which limits the wide
// token tiles; the decode tiles (<= 32 rows) keep it.  MOE_UP_GATHER=tma |
// pregather overrides.
bool want_pregather(const moe_shape_t& s) {
  if (const char* env = std::getenv("MOE_UP_GATHER")) {
    if (std::strcmp(env, "tma") == 0) return false;
    if (std::strcmp(env, "pregather") == 0) return true;
  }
  return choose_nmax(s) >= 128;
}

size_t pregather_bytes(const moe_shape_t& s) { return align_up(cap_rows(s) * s.H * sizeof(uint16_t)); }

// ---------------------------------------------------------------- NVFP4 sizes
// Upper bound on 128-row token tiles (sum over experts of ceil(count/128)).
int nvfp4_tiles_ub(const moe_shape_t& s) {
  const long long mk = static_cast<long long>(s.M) * s.top_k;
  return static_cast<int>(mk / 128 + (mk < s.E ? mk : s.E));
}
// Tile-aligned NVFP4 activation copy of `cols`-wide rows: amax word, codes,
// scale atoms; for x (per_token) also the per-token codes and scales it is
// gathered from.
struct ActLayout {
  size_t amax, codes, atoms, tok_codes, tok_scales, total;
};
ActLayout act_layout(const moe_shape_t& s, int cols, bool per_token) {
  ActLayout L{};
  const size_t rows = static_cast<size_t>(nvfp4_tiles_ub(s)) * 128;
  L.amax = 0;
  L.codes = kAlign;
  L.atoms = align_up(L.codes + rows * cols / 2);
  L.tok_codes = align_up(L.atoms + static_cast<size_t>(nvfp4_tiles_ub(s)) * (cols / 64) * 512);
  L.tok_scales = per_token ? align_up(L.tok_codes + static_cast<size_t>(s.M) * cols / 2) : L.tok_codes;
  L.total = per_token ? align_up(L.tok_scales + static_cast<size_t>(s.M) * cols / 16) : L.tok_codes;
  return L;
}
ActLayout x_act_layout(const moe_shape_t& s) { return act_layout(s, s.H, true); }
ActLayout h_act_layout(const moe_shape_t& s) { return act_layout(s, s.I, false); }
// Blob of one projection: codes [rows, cols/2] then scale atoms.
void blob_dims(const moe_shape_t& s, int which, int64_t* rows, int64_t* cols) {
  *rows = static_cast<int64_t>(s.E) * (which == 2 ? s.H : s.I);
  *cols = which == 2 ? s.I : s.H;
}
size_t blob_codes_bytes(const moe_shape_t& s, int which) {
  int64_t r, c;
  blob_dims(s, which, &r, &c);
  return static_cast<size_t>(r) * c / 2;
}

// Whether the batch/prefill shapes take the persistent path (one CTA per SM,
// or one cluster per two SMs; deep weight ring): the pair kernels by default, the
// single-SM persistent kernels for shapes the pairs do not take or with
// MOE_GEMM_PAIR=0.  MOE_GEMM_PERSISTENT=0|1 overrides; the up projection also
// needs the plan-ordered copy of x, so it only takes this path when the
// caller provides that workspace.
bool want_persistent(const moe_shape_t& s) {
  if (const char* env = std::getenv("MOE_GEMM_PERSISTENT")) {
    if (std::strcmp(env, "0") == 0) return false;
    if (std::strcmp(env, "1") == 0) return true;
  }
  return choose_nmax(s) >= 128;
}

// Ring shape of the persistent kernels (MOE_PGEMM_DEEP_B=1: 4 weight + 5
// token-row stages; default 5 + 3).
bool deep_token_ring() {
  const char* env = std::getenv("MOE_PGEMM_DEEP_B");
  return env != nullptr && std::strcmp(env, "1") == 0;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  static int cached[64] = {};
  if (dev < 64 && cached[dev] > 0) return cached[dev];
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev < 64) cached[dev] = n;
  return n;
}

moe_status_t check_plan(const moe_plan_t* p) {
  if (p == nullptr || p->sorted_ids == nullptr || p->expert_counts == nullptr || p->expert_offsets == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(p->sorted_ids)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

moe_status_t check_weights(const moe_weights_t* w, const moe_shape_t& s) {
  if (w == nullptr) return MOE_ERR_INVALID_ARG;
  if (w->dtype != MOE_W_BF16 && w->dtype != MOE_W_NVFP4) return MOE_ERR_UNSUPPORTED;
  if (w->dtype == MOE_W_NVFP4) {
    if (!w->gate_gs || !w->up_gs || !w->down_gs) return MOE_ERR_INVALID_ARG;
    if (s.I % 256 != 0) return MOE_ERR_UNSUPPORTED;  // the NVFP4 kernels step 256 elements along I
  }
  return MOE_OK;
}

// NVFP4 up: amax of x -> tile-aligned NVFP4 copy of the routed x rows -> block-scaled GEMM.
// h_amax (nullable): word the up epilogue atomically maxes |h| into (the caller zeroes it first).
moe_status_t run_up_nvfp4(const moe_bf16_t* x, const moe_weights_t* w, const moe_plan_t* plan,
                          const moe_shape_t& s, moe_bf16_t* h, void* ws, int32_t* err, cudaStream_t stream,
                          unsigned* h_amax = nullptr);
// amax_ready: ws's amax word already holds max |h| (from the up epilogue); otherwise it is computed here.
moe_status_t run_down_nvfp4(const moe_bf16_t* h, const moe_weights_t* w, const moe_plan_t* plan,
                            const moe_shape_t& s, moe_bf16_t* y, void* ws, int32_t* err, cudaStream_t stream,
                            bool amax_ready = false);

// Token-tile width of the 2-SM pair kernels on the persistent path, or 0 for
// the single-SM persistent kernels.  Pairs measured faster on the batch and
// prefill workloads (the operand feed per SM is the limit there): 256-row
// tiles from 96 routed rows per expert on average, 128-row tiles below.
// MOE_GEMM_PAIR=0|128|256 overrides (the tests cover every variant).
int pair_nmax(const moe_shape_t& s) {
  if (const char* env = std::getenv("MOE_GEMM_PAIR")) {
    const int v = std::atoi(env);
    return (v == 128 || v == 256) ? v : 0;
  }
  const double per_expert = static_cast<double>(s.M) * s.top_k / s.E;
  return per_expert >= 96.0 ? 256 : 128;
}

// Whether the 2-SM pair up kernel gathers its x rows itself (tile::gather4 by token id, one copy of four
// rows per lane) instead of reading x pre-gathered into plan order by a separate launch.  It pays with
// 128-row token tiles (batch: up 2336 -> 2220 us, the gather launch gone) and not with 256-row tiles,
// where 32 gather copies per stage and CTA hold the producer back (prefill up 2957 -> 3684 us).
// MOE_PAIR_GATHER=0|1 overrides (the tests cover both).
bool want_pair_gather(const moe_shape_t& s) {
  if (const char* env = std::getenv("MOE_PAIR_GATHER")) return std::strcmp(env, "1") == 0;
  return pair_nmax(s) == 128;
}

// Whether the layer routes through the screened path (router_screen.cu), with the y region of its
// workspace as scratch.
bool route_screens(const moe_shape_t& s) {
  if (!moe::screen_eligible(s.M, s.H, s.E, s.top_k)) return false;
  return moe::screen_scratch_bytes(s.M, s.H, s.E) <= static_cast<size_t>(s.M) * s.top_k * s.H * sizeof(uint16_t);
}

// Whether the up projection of this shape launches the x gather into plan order first.
bool up_pregathers(const moe_shape_t& s) {
  if (!want_pregather(s)) return false;
  const bool pair_path = want_persistent(s) && pair_nmax(s) != 0 && s.I % 256 == 0;
  return !(pair_path && want_pair_gather(s));
}

moe_status_t run_up(const moe_bf16_t* x, const moe_weights_t* w, const moe_plan_t* plan, const moe_shape_t& s,
                    moe_bf16_t* h, void* ws, size_t ws_bytes, int32_t* err, cudaStream_t stream) {
  CUtensorMap mg, mu, mx;
  const uint64_t rows = static_cast<uint64_t>(s.E) * s.I;
  const bool have_ws = ws != nullptr && ws_bytes >= pregather_bytes(s) && aligned16(ws) &&
                       plan->num_tokens_post_padded != nullptr;
  const bool persistent = want_persistent(s);
  const bool gathered = want_pregather(s) && have_ws;
  if (!make_map_bf16(&mg, w->gate, rows, s.H, 128) || !make_map_bf16(&mu, w->up, rows, s.H, 128))
    return MOE_ERR_CUDA;
  if (persistent && gathered && pair_nmax(s) != 0 && s.I % 256 == 0 && want_pair_gather(s)) {
    if (!make_map_bf16(&mx, x, s.M, s.H, 1)) return MOE_ERR_CUDA;
    GroupedGemmArgs a{};
    a.sorted_ids = plan->sorted_ids;
    a.expert_counts = plan->expert_counts;
    a.expert_offsets = plan->expert_offsets;
    a.out = h;
    a.err = err;
    a.M = s.M;
    a.E = s.E;
    a.top_k = s.top_k;
    a.rows_per_expert = s.I;
    a.kdim = s.H;
    a.out_ld = s.I;
    return cuda_status(moe::launch_pair_up(mg, mu, mx, a, pair_nmax(s), num_sms(), stream, true));
  }
  if (gathered) {
    auto* xg = static_cast<moe_bf16_t*>(ws);
    const cudaError_t e = moe::launch_gather_rows(x, plan->sorted_ids, plan->num_tokens_post_padded, s.M, s.top_k,
                                                  s.H, static_cast<int>(cap_rows(s)), xg, stream);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    if (!make_map_bf16(&mx, xg, cap_rows(s), s.H, persistent ? 32 : 16)) return MOE_ERR_CUDA;
  } else if (!make_map_bf16(&mx, x, s.M, s.H, 1)) {
    return MOE_ERR_CUDA;
  }
  GroupedGemmArgs a{};
  a.sorted_ids = plan->sorted_ids;
  a.expert_counts = plan->expert_counts;
  a.expert_offsets = plan->expert_offsets;
  a.out = h;
  a.err = err;
  a.M = s.M;
  a.E = s.E;
  a.top_k = s.top_k;
  a.rows_per_expert = s.I;
  a.kdim = s.H;
  a.out_ld = s.I;
  if (persistent && gathered && pair_nmax(s) != 0 && s.I % 256 == 0)
    return cuda_status(moe::launch_pair_up(mg, mu, mx, a, pair_nmax(s), num_sms(), stream));
  if (persistent)
    return cuda_status(
        moe::launch_persistent_up(mg, mu, mx, a, choose_nmax(s), !gathered, deep_token_ring(), num_sms(), stream));
  return cuda_status(moe::launch_grouped_up(mg, mu, mx, a, choose_nmax(s), gathered, stream));
}

// Whether the layer folds the align step into the up projection: bf16
// weights on the decode path (32-row token tiles, x gathered by token id) and
// few enough routed slots for one warp per CTA to scan.  MOE_SELF_ROUTE=0
// turns it off (the tests cover both).
bool want_self_route(const moe_shape_t& s, moe_wdtype_t dt) {
  if (const char* env = std::getenv("MOE_SELF_ROUTE"))
    if (std::strcmp(env, "0") == 0) return false;
  return dt == MOE_W_BF16 && !want_persistent(s) && choose_nmax(s) == 32 && !want_pregather(s) &&
         static_cast<long long>(s.M) * s.top_k <= moe::kRouteMaxSlots;
}

// Whether moe_layer runs as one launch (layer_fused.cu): the decode shapes of
// the self-routing path with at most 256 experts.  MOE_FUSED_LAYER=0 turns it
// off (the tests cover both).
bool want_fused_layer(const moe_shape_t& s, moe_wdtype_t dt) {
  if (const char* env = std::getenv("MOE_FUSED_LAYER"))
    if (std::strcmp(env, "0") == 0) return false;
  return want_self_route(s, dt) && s.E <= 256;
}

moe_status_t run_layer_fused(const moe_bf16_t* x, const moe_bf16_t* w_router, const float* bias,
                             const moe_weights_t* w, const moe_bf16_t* gamma, float eps, const moe_shape_t& s,
                             moe_bf16_t* out, moe_bf16_t* residual_out, int32_t* ids, float* tw, uint8_t* base,
                             const moe_layer_ws_layout_t& L, cudaStream_t stream) {
  CUtensorMap mg, mu, md, mx, mh;
  const uint64_t rows = static_cast<uint64_t>(s.E) * s.I;
  auto* h = reinterpret_cast<moe_bf16_t*>(base + L.h);
  if (!make_map_bf16(&mg, w->gate, rows, s.H, 128) || !make_map_bf16(&mu, w->up, rows, s.H, 128) ||
      !make_map_bf16(&md, w->down, static_cast<uint64_t>(s.E) * s.H, s.I, 128) ||
      !make_map_bf16(&mx, x, s.M, s.H, 1) || !make_map_bf16(&mh, h, cap_rows(s), s.I, 16))
    return MOE_ERR_CUDA;
  moe::FusedLayerArgs a{};
  a.x = x;
  a.w_router = w_router;
  a.bias = bias;
  a.gamma = gamma;
  a.eps = eps;
  a.M = s.M;
  a.H = s.H;
  a.I = s.I;
  a.E = s.E;
  a.top_k = s.top_k;
  a.block_size = s.block_size;
  a.logits = reinterpret_cast<float*>(base + L.logits);
  a.topk_ids = ids;
  a.topk_w = tw;
  a.sorted_ids = reinterpret_cast<int32_t*>(base + L.sorted_ids);
  a.block_expert = reinterpret_cast<int32_t*>(base + L.block_expert);
  a.counts = reinterpret_cast<int32_t*>(base + L.expert_counts);
  a.offsets = reinterpret_cast<int32_t*>(base + L.expert_offsets);
  a.ntpp = reinterpret_cast<int32_t*>(base + L.num_tokens_post_padded);
  a.h = h;
  a.y = reinterpret_cast<moe_bf16_t*>(base + L.y);
  a.out = out;
  a.residual_out = residual_out;
  a.err = reinterpret_cast<int32_t*>(base + L.err_flag);
  a.sync = reinterpret_cast<unsigned*>(base + L.sync);
  const cudaError_t e = moe::launch_layer_fused(mg, mu, md, mx, mh, a, num_sms(), stream);
  if (e == cudaErrorCooperativeLaunchTooLarge || e == cudaErrorInvalidConfiguration || e == cudaErrorInvalidValue) {
    // nothing was launched (e.g. the GPU is shared and cannot hold one CTA per SM at once): the caller
    // runs the separate launches instead
    (void)cudaGetLastError();
    return MOE_ERR_UNSUPPORTED;
  }
  return cuda_status(e);
}

moe_status_t run_up_routed(const moe_bf16_t* x, const moe_weights_t* w, const int32_t* topk_ids,
                           const moe_shape_t& s, int32_t* sorted_ids, int32_t* block_expert, int32_t* counts,
                           int32_t* offsets, int32_t* ntpp, moe_bf16_t* h, int32_t* err, cudaStream_t stream) {
  CUtensorMap mg, mu, mx;
  const uint64_t rows = static_cast<uint64_t>(s.E) * s.I;
  if (!make_map_bf16(&mg, w->gate, rows, s.H, 128) || !make_map_bf16(&mu, w->up, rows, s.H, 128) ||
      !make_map_bf16(&mx, x, s.M, s.H, 1))
    return MOE_ERR_CUDA;
  GroupedGemmArgs a{};
  a.out = h;
  a.err = err;
  a.M = s.M;
  a.E = s.E;
  a.top_k = s.top_k;
  a.rows_per_expert = s.I;
  a.kdim = s.H;
  a.out_ld = s.I;
  a.topk_ids = topk_ids;
  a.block_size = s.block_size;
  a.plan_sorted_ids = sorted_ids;
  a.plan_block_expert = block_expert;
  a.plan_counts = counts;
  a.plan_offsets = offsets;
  a.plan_ntpp = ntpp;
  return cuda_status(moe::launch_grouped_up_routed(mg, mu, mx, a, stream));
}

moe_status_t run_down(const moe_bf16_t* h, const moe_weights_t* w, const moe_plan_t* plan, const moe_shape_t& s,
                      moe_bf16_t* y, int32_t* err, cudaStream_t stream) {
  CUtensorMap md, mh;
  const bool persistent = want_persistent(s);
  if (!make_map_bf16(&md, w->down, static_cast<uint64_t>(s.E) * s.H, s.I, 128) ||
      !make_map_bf16(&mh, h, cap_rows(s), s.I, persistent ? 32 : 16))
    return MOE_ERR_CUDA;
  GroupedGemmArgs a{};
  a.sorted_ids = plan->sorted_ids;
  a.expert_counts = plan->expert_counts;
  a.expert_offsets = plan->expert_offsets;
  a.out = y;
  a.err = err;
  a.M = s.M;
  a.E = s.E;
  a.top_k = s.top_k;
  a.rows_per_expert = s.H;
  a.kdim = s.I;
  a.out_ld = s.H;
  if (persistent && pair_nmax(s) != 0 && s.H % 512 == 0)
    return cuda_status(moe::launch_pair_down(md, mh, a, pair_nmax(s), num_sms(), stream));
  if (persistent)
    return cuda_status(moe::launch_persistent_down(md, mh, a, choose_nmax(s), deep_token_ring(), num_sms(), stream));
  return cuda_status(moe::launch_grouped_down(md, mh, a, choose_nmax(s), stream));
}

int num_sms();

// Whether the NVFP4 projections run on 2-SM pairs (nvfp4_pair.cu): whenever the weight blocks of a pair
// divide the expert (up: I a multiple of 256, down: H a multiple of 512).  MOE_NVFP4_PAIR=0 keeps the
// single-SM kernels (the tests cover both).
bool want_nvfp4_pair(const moe_shape_t& s, bool up) {
  if (const char* env = std::getenv("MOE_NVFP4_PAIR"))
    if (std::strcmp(env, "0") == 0) return false;
  return up ? s.I % 256 == 0 : s.H % 512 == 0;
}

moe_status_t run_up_nvfp4(const moe_bf16_t* x, const moe_weights_t* w, const moe_plan_t* plan,
                          const moe_shape_t& s, moe_bf16_t* h, void* ws, int32_t* err, cudaStream_t stream,
                          unsigned* h_amax) {
  const ActLayout L = x_act_layout(s);
  auto* base = static_cast<uint8_t*>(ws);
  auto* amax = reinterpret_cast<unsigned*>(base + L.amax);
  const int tiles = nvfp4_tiles_ub(s);
  if (cudaMemsetAsync(amax, 0, sizeof(unsigned), stream) != cudaSuccess) return MOE_ERR_CUDA;
  if (moe::launch_amax_all(x, static_cast<int64_t>(s.M) * s.H, amax, stream) != cudaSuccess) return MOE_ERR_CUDA;
  if (moe::launch_quantize_rows(x, s.M, s.H, amax, base + L.tok_codes, base + L.tok_scales, stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (moe::launch_gather_tiles(base + L.tok_codes, base + L.tok_scales, plan->sorted_ids, plan->expert_counts,
                               plan->expert_offsets, s.E, s.top_k, s.M * s.top_k, s.H, tiles, base + L.codes,
                               base + L.atoms, stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  CUtensorMap mg, mu, mx;
  const uint64_t wrows = static_cast<uint64_t>(s.E) * s.I;
  if (!make_map_u8(&mg, w->gate, wrows, s.H / 2, 128) || !make_map_u8(&mu, w->up, wrows, s.H / 2, 128) ||
      !make_map_u8(&mx, base + L.codes, static_cast<uint64_t>(tiles) * 128, s.H / 2, 32))
    return MOE_ERR_CUDA;
  moe::Nvfp4GemmArgs a{};
  a.g.sorted_ids = plan->sorted_ids;
  a.g.expert_counts = plan->expert_counts;
  a.g.expert_offsets = plan->expert_offsets;
  a.g.out = h;
  a.g.err = err;
  a.g.M = s.M;
  a.g.E = s.E;
  a.g.top_k = s.top_k;
  a.g.rows_per_expert = s.I;
  a.g.kdim = s.H;
  a.g.out_ld = s.I;
  a.sfa0 = static_cast<const uint8_t*>(w->gate) + blob_codes_bytes(s, 0);
  a.sfa1 = static_cast<const uint8_t*>(w->up) + blob_codes_bytes(s, 1);
  a.sfb = base + L.atoms;
  a.gs_a0 = w->gate_gs;
  a.gs_a1 = w->up_gs;
  a.act_amax = amax;
  a.out_amax = h_amax;
  if (want_nvfp4_pair(s, true)) {
    CUtensorMap sg, su, sx;
    const uint64_t wsf = static_cast<uint64_t>(s.E) * (s.I / 128) * (s.H / 64) * 512;
    if (!make_map_sf(&sg, a.sfa0, wsf) || !make_map_sf(&su, a.sfa1, wsf) ||
        !make_map_sf(&sx, a.sfb, static_cast<uint64_t>(tiles) * (s.H / 64) * 512))
      return MOE_ERR_CUDA;
    return cuda_status(moe::launch_nvfp4_pair_up(mg, mu, mx, sg, su, sx, a, num_sms(), stream));
  }
  return cuda_status(moe::launch_nvfp4_up(mg, mu, mx, a, num_sms(), stream));
}

moe_status_t run_down_nvfp4(const moe_bf16_t* h, const moe_weights_t* w, const moe_plan_t* plan,
                            const moe_shape_t& s, moe_bf16_t* y, void* ws, int32_t* err, cudaStream_t stream,
                            bool amax_ready) {
  const ActLayout L = h_act_layout(s);
  auto* base = static_cast<uint8_t*>(ws);
  auto* amax = reinterpret_cast<unsigned*>(base + L.amax);
  const int tiles = nvfp4_tiles_ub(s);
  if (!amax_ready) {
    if (cudaMemsetAsync(amax, 0, sizeof(unsigned), stream) != cudaSuccess) return MOE_ERR_CUDA;
    if (moe::launch_amax_plan_rows(h, plan->sorted_ids, plan->num_tokens_post_padded, s.M * s.top_k, s.I,
                                   static_cast<int>(cap_rows(s)), amax, stream) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  if (moe::launch_quantize_tiles(h, plan->expert_counts, plan->expert_offsets, s.E, s.I, tiles, amax, base + L.codes,
                                 base + L.atoms, stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  CUtensorMap md, mh;
  if (!make_map_u8(&md, w->down, static_cast<uint64_t>(s.E) * s.H, s.I / 2, 128) ||
      !make_map_u8(&mh, base + L.codes, static_cast<uint64_t>(tiles) * 128, s.I / 2, 32))
    return MOE_ERR_CUDA;
  moe::Nvfp4GemmArgs a{};
  a.g.sorted_ids = plan->sorted_ids;
  a.g.expert_counts = plan->expert_counts;
  a.g.expert_offsets = plan->expert_offsets;
  a.g.out = y;
  a.g.err = err;
  a.g.M = s.M;
  a.g.E = s.E;
  a.g.top_k = s.top_k;
  a.g.rows_per_expert = s.H;
  a.g.kdim = s.I;
  a.g.out_ld = s.H;
  a.sfa0 = static_cast<const uint8_t*>(w->down) + blob_codes_bytes(s, 2);
  a.sfa1 = a.sfa0;
  a.sfb = base + L.atoms;
  a.gs_a0 = w->down_gs;
  a.gs_a1 = w->down_gs;
  a.act_amax = amax;
  if (want_nvfp4_pair(s, false)) {
    CUtensorMap sd, sh;
    if (!make_map_sf(&sd, a.sfa0, static_cast<uint64_t>(s.E) * (s.H / 128) * (s.I / 64) * 512) ||
        !make_map_sf(&sh, a.sfb, static_cast<uint64_t>(tiles) * (s.I / 64) * 512))
      return MOE_ERR_CUDA;
    return cuda_status(moe::launch_nvfp4_pair_down(md, mh, sd, sh, a, num_sms(), stream));
  }
  return cuda_status(moe::launch_nvfp4_down(md, mh, a, num_sms(), stream));
}

// Counters of the single-launch layer: grid barrier, work counter, finalize
// count, one up-tile count per expert, and (up to 64 tokens) one slice count
// and 8 partial sums of squares per token.
size_t fused_sync_words(const moe_shape_t& s) {
  return 3 + static_cast<size_t>(s.E) + (s.M <= 64 ? 9 * static_cast<size_t>(s.M) : 0);
}

moe_layer_ws_layout_t layer_layout(const moe_shape_t& s, moe_wdtype_t dt) {
  moe_layer_ws_layout_t L{};
  const size_t mk = static_cast<size_t>(s.M) * s.top_k;
  const size_t cap = cap_rows(s);
  size_t off = 0;
  L.err_flag = off;
  L.sync = off + 16;  // zeroed with the error word before every layer call
  off = align_up(L.sync + fused_sync_words(s) * sizeof(uint32_t));
  L.logits = off;
  off = align_up(off + static_cast<size_t>(s.M) * s.E * sizeof(float));
  L.topk_ids = off;
  off = align_up(off + mk * sizeof(int32_t));
  L.topk_w = off;
  off = align_up(off + mk * sizeof(float));
  L.sorted_ids = off;
  off = align_up(off + cap * sizeof(int32_t));
  L.block_expert = off;
  off = align_up(off + (cap / s.block_size + 1) * sizeof(int32_t));
  L.expert_counts = off;
  off = align_up(off + s.E * sizeof(int32_t));
  L.expert_offsets = off;
  off = align_up(off + (s.E + 1) * sizeof(int32_t));
  L.num_tokens_post_padded = off;
  off = align_up(off + sizeof(int32_t));
  L.h = off;
  off = align_up(off + cap * s.I * sizeof(uint16_t));
  L.y = off;
  off = align_up(off + mk * s.H * sizeof(uint16_t));
  L.act_scratch = off;  // bf16: x gathered into plan order; NVFP4: the two tile-aligned activation copies
  if (dt == MOE_W_NVFP4)
    off = align_up(off + x_act_layout(s).total + h_act_layout(s).total);
  else
    off = align_up(off + pregather_bytes(s));
  L.total = off;
  return L;
}

moe_status_t check_layer_args(const moe_bf16_t* x, const moe_bf16_t* w_router, const moe_weights_t* w,
                              const moe_bf16_t* gamma, float eps, const moe_shape_t& s, const moe_bf16_t* out,
                              const moe_bf16_t* residual_out) {
  moe_status_t st = check_shape(s);
  if (st != MOE_OK) return st;
  if (!w) return MOE_ERR_INVALID_ARG;
  if ((st = check_weights(w, s)) != MOE_OK) return st;
  if (!x || !w_router || !gamma || !out || !w->gate || !w->up || !w->down) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(gamma) || !aligned16(out) || !aligned16(w->gate) ||
      !aligned16(w->up) || !aligned16(w->down) || (residual_out && !aligned16(residual_out)))
    return MOE_ERR_INVALID_ARG;
  if (!(eps >= 0.0f)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

// Route -> plan -> up -> down of the layer as separate launches, leaving y [M*K, H] in the workspace
// (the finalize is the caller's: single-GPU or fused with the exchange across ranks).
moe_status_t run_layer_to_y(const moe_bf16_t* x, const moe_bf16_t* w_router, const float* bias,
                            const moe_weights_t* w, const moe_shape_t& s, uint8_t* base,
                            const moe_layer_ws_layout_t& L, int32_t* ids, float* tw, cudaStream_t cs) {
  moe_status_t st;
  auto* err = reinterpret_cast<int32_t*>(base + L.err_flag);
  auto* sorted = reinterpret_cast<int32_t*>(base + L.sorted_ids);
  auto* bexp = reinterpret_cast<int32_t*>(base + L.block_expert);
  auto* counts = reinterpret_cast<int32_t*>(base + L.expert_counts);
  auto* offs = reinterpret_cast<int32_t*>(base + L.expert_offsets);
  auto* ntpp = reinterpret_cast<int32_t*>(base + L.num_tokens_post_padded);
  auto* h = reinterpret_cast<moe_bf16_t*>(base + L.h);
  auto* y = reinterpret_cast<moe_bf16_t*>(base + L.y);
  float* logits = reinterpret_cast<float*>(base + L.logits);
  if (route_screens(s)) {  // its scratch: the y region, written only by the down projection
    if ((st = cuda_status(moe::launch_route_screened(x, w_router, bias, s.M, s.H, s.E, s.top_k, base + L.y, ids,
                                                     tw, err, cs))) != MOE_OK)
      return st;
  } else {
    if ((st = cuda_status(moe::launch_router_logits(x, w_router, bias, s.M, s.H, s.E, logits, cs))) != MOE_OK)
      return st;
    if ((st = cuda_status(moe::launch_router_topk(logits, s.M, s.E, s.top_k, ids, tw, cs))) != MOE_OK) return st;
  }
  moe_plan_t plan{sorted, bexp, counts, offs, ntpp};
  if (want_self_route(s, w->dtype)) {
    if ((st = run_up_routed(x, w, ids, s, sorted, bexp, counts, offs, ntpp, h, err, cs)) != MOE_OK) return st;
    return run_down(h, w, &plan, s, y, err, cs);
  }
  if ((st = cuda_status(moe::launch_align(ids, s.M, s.top_k, s.E, s.block_size, sorted, bexp, counts, offs, ntpp,
                                          err, cs))) != MOE_OK)
    return st;
  if (w->dtype == MOE_W_NVFP4) {
    // max |h| comes out of the up kernel's epilogue into the down activation copy's amax word
    uint8_t* act = base + L.act_scratch;
    uint8_t* act_h = act + x_act_layout(s).total;
    auto* h_amax = reinterpret_cast<unsigned*>(act_h + h_act_layout(s).amax);
    if ((st = cuda_status(cudaMemsetAsync(h_amax, 0, sizeof(unsigned), cs))) != MOE_OK) return st;
    if ((st = run_up_nvfp4(x, w, &plan, s, h, act, err, cs, h_amax)) != MOE_OK) return st;
    return run_down_nvfp4(h, w, &plan, s, y, act_h, err, cs, true);
  }
  if ((st = run_up(x, w, &plan, s, h, base + L.act_scratch, L.total - L.act_scratch, err, cs)) != MOE_OK) return st;
  return run_down(h, w, &plan, s, y, err, cs);
}

}  // namespace

namespace moe {
bool encode_map_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  return make_map_bf16(map, base, rows, cols, box_rows);
}
bool encode_map_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols_bytes, uint32_t box_rows) {
  return make_map_u8(map, base, rows, cols_bytes, box_rows);
}
bool encode_map_sf_rows(CUtensorMap* map, const void* base, uint64_t bytes, uint32_t box_rows) {
  return make_map_sf(map, base, bytes, box_rows);
}

int check_route_args(const moe_shape_t& s, const void* x, const void* w_router, const void* topk_ids,
                     const void* topk_w) {
  const moe_status_t st = check_shape(s);
  if (st != MOE_OK) return st;
  if (!x || !w_router || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}
}  // namespace moe

extern "C" {

const char* moe_status_string(moe_status_t st) {
  switch (st) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: null, misaligned or out-of-range argument";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: shape or dtype outside the accepted set";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace missing or too small";
    case MOE_ERR_INVALID_INPUT: return "MOE_ERR_INVALID_INPUT: device found an expert id outside [0, E)";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT: a bounded wait inside a kernel expired";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA call or kernel launch failed";
  }
  return "unknown moe_status_t";
}

size_t moe_align_capacity(moe_shape_t s) {
  if (check_shape(s) != MOE_OK) return 0;
  return cap_rows(s);
}

size_t moe_route_workspace_size(moe_shape_t s) {
  if (check_shape(s) != MOE_OK) return 0;
  const size_t logits = align_up(static_cast<size_t>(s.M) * s.E * sizeof(float));
  return logits + (moe::screen_shape_ok(s.M, s.H, s.E, s.top_k) ? moe::screen_scratch_bytes(s.M, s.H, s.E) : 0);
}

size_t moe_up_workspace_size(moe_shape_t s, moe_wdtype_t dtype) {
  if (check_shape(s) != MOE_OK) return 0;
  if (dtype == MOE_W_NVFP4) return x_act_layout(s).total;
  return (want_pregather(s) || want_persistent(s)) ? pregather_bytes(s) : 0;
}

size_t moe_down_workspace_size(moe_shape_t s, moe_wdtype_t dtype) {
  if (check_shape(s) != MOE_OK) return 0;
  return dtype == MOE_W_NVFP4 ? h_act_layout(s).total : 0;
}

moe_status_t moe_route(const moe_bf16_t* x, const moe_bf16_t* w_router, const float* bias, moe_shape_t s,
                       int32_t* topk_ids, float* topk_w, void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status_t st = check_shape(s);
  if (st != MOE_OK) return st;
  if (!x || !w_router || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router)) return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < moe_route_workspace_size(s)) return MOE_ERR_WORKSPACE;
  auto cs = static_cast<cudaStream_t>(stream);
  float* logits = static_cast<float*>(ws);
  if (moe::screen_eligible(s.M, s.H, s.E, s.top_k) && aligned16(ws)) {
    uint8_t* scratch = static_cast<uint8_t*>(ws) + align_up(static_cast<size_t>(s.M) * s.E * sizeof(float));
    return cuda_status(moe::launch_route_screened(x, w_router, bias, s.M, s.H, s.E, s.top_k, scratch, topk_ids,
                                                  topk_w, nullptr, cs));
  }
  st = cuda_status(moe::launch_router_logits(x, w_router, bias, s.M, s.H, s.E, logits, cs));
  if (st != MOE_OK) return st;
  return cuda_status(moe::launch_router_topk(logits, s.M, s.E, s.top_k, topk_ids, topk_w, cs));
}

moe_status_t moe_route_ex(const moe_bf16_t* x, const moe_bf16_t* w_router, const float* bias, moe_shape_t s,
                          const moe_route_opts_t* opts, int32_t* topk_ids, float* topk_w, void* ws, size_t ws_bytes,
                          moe_stream_t stream) {
  moe_status_t st = check_shape(s);
  if (st != MOE_OK) return st;
  if (!x || !w_router || !topk_ids || !topk_w || !opts) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router)) return MOE_ERR_INVALID_ARG;
  if (opts->scoring != MOE_SCORE_SOFTMAX && opts->scoring != MOE_SCORE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (!(opts->routed_scale > 0.0f) || !std::isfinite(opts->routed_scale)) return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < moe_route_workspace_size(s)) return MOE_ERR_WORKSPACE;
  auto cs = static_cast<cudaStream_t>(stream);
  float* logits = static_cast<float*>(ws);
  const bool sel_only = bias != nullptr && opts->bias_in_score == 0;
  st = cuda_status(moe::launch_router_logits(x, w_router, sel_only ? nullptr : bias, s.M, s.H, s.E, logits, cs));
  if (st != MOE_OK) return st;
  return cuda_status(moe::launch_router_topk_ext(logits, sel_only ? bias : nullptr, s.M, s.E, s.top_k, opts->scoring,
                                                 opts->renormalize != 0 ? 1 : 0, opts->routed_scale, topk_ids,
                                                 topk_w, cs));
}

moe_status_t moe_align_block_size(const int32_t* topk_ids, moe_shape_t s, int32_t* sorted_ids, int32_t* block_expert,
                                  int32_t* expert_counts, int32_t* expert_offsets, int32_t* num_tokens_post_padded,
                                  int32_t* err_flag, moe_stream_t stream) {
  moe_status_t st = check_shape(s);
  if (st != MOE_OK) return st;
  if (!topk_ids || !sorted_ids || !block_expert || !expert_counts || !expert_offsets || !num_tokens_post_padded)
    return MOE_ERR_INVALID_ARG;
  return cuda_status(moe::launch_align(topk_ids, s.M, s.top_k, s.E, s.block_size, sorted_ids, block_expert,
                                       expert_counts, expert_offsets, num_tokens_post_padded, err_flag,
                                       static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_grouped_up_swiglu(const moe_bf16_t* x, const moe_weights_t* w, const moe_plan_t* plan,
                                   moe_shape_t s, moe_bf16_t* h, void* ws, size_t ws_bytes, int32_t* err_flag,
                                   moe_stream_t stream) {
  moe_status_t st = check_shape(s);
  if (st != MOE_OK) return st;
  if ((st = check_weights(w, s)) != MOE_OK) return st;
  if ((st = check_plan(plan)) != MOE_OK) return st;
  if (!x || !h || !w->gate || !w->up) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(h) || !aligned16(w->gate) || !aligned16(w->up)) return MOE_ERR_INVALID_ARG;
  if (w->dtype == MOE_W_NVFP4) {
    if (!ws || ws_bytes < moe_up_workspace_size(s, MOE_W_NVFP4) || !aligned16(ws) || !plan->num_tokens_post_padded)
      return MOE_ERR_WORKSPACE;
    return run_up_nvfp4(x, w, plan, s, h, ws, err_flag, static_cast<cudaStream_t>(stream));
  }
  return run_up(x, w, plan, s, h, ws, ws_bytes, err_flag, static_cast<cudaStream_t>(stream));
}

static_assert(MOE_ROUTED_UP_MAX_SLOTS == moe::kRouteMaxSlots, "header and kernel agree on the slot limit");

moe_status_t moe_grouped_up_swiglu_routed(const moe_bf16_t* x, const moe_weights_t* w, const int32_t* topk_ids,
                                          moe_shape_t s, int32_t* sorted_ids, int32_t* block_expert,
                                          int32_t* expert_counts, int32_t* expert_offsets,
                                          int32_t* num_tokens_post_padded, moe_bf16_t* h, int32_t* err_flag,
                                          moe_stream_t stream) {
  moe_status_t st = check_shape(s);
  if (st != MOE_OK) return st;
  if (!w) return MOE_ERR_INVALID_ARG;
  if (w->dtype != MOE_W_BF16) return MOE_ERR_UNSUPPORTED;
  if ((st = check_weights(w, s)) != MOE_OK) return st;
  if (static_cast<long long>(s.M) * s.top_k > moe::kRouteMaxSlots) return MOE_ERR_UNSUPPORTED;
  if (!x || !topk_ids || !h || !w->gate || !w->up || !sorted_ids || !block_expert || !expert_counts ||
      !expert_offsets || !num_tokens_post_padded)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(h) || !aligned16(w->gate) || !aligned16(w->up)) return MOE_ERR_INVALID_ARG;
  return run_up_routed(x, w, topk_ids, s, sorted_ids, block_expert, expert_counts, expert_offsets,
                       num_tokens_post_padded, h, err_flag, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_grouped_down(const moe_bf16_t* h, const moe_weights_t* w, const moe_plan_t* plan, moe_shape_t s,
                              moe_bf16_t* y, void* ws, size_t ws_bytes, int32_t* err_flag, moe_stream_t stream) {
  moe_status_t st = check_shape(s);
  if (st != MOE_OK) return st;
  if ((st = check_weights(w, s)) != MOE_OK) return st;
  if ((st = check_plan(plan)) != MOE_OK) return st;
  if (!h || !y || !w->down) return MOE_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(y) || !aligned16(w->down)) return MOE_ERR_INVALID_ARG;
  if (w->dtype == MOE_W_NVFP4) {
    if (!ws || ws_bytes < moe_down_workspace_size(s, MOE_W_NVFP4) || !aligned16(ws) || !plan->num_tokens_post_padded)
      return MOE_ERR_WORKSPACE;
    return run_down_nvfp4(h, w, plan, s, y, ws, err_flag, static_cast<cudaStream_t>(stream));
  }
  return run_down(h, w, plan, s, y, err_flag, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_finalize_rmsnorm(const moe_bf16_t* x, const moe_bf16_t* y, const float* topk_w,
                                  const moe_bf16_t* gamma, float eps, moe_shape_t s, moe_bf16_t* out,
                                  moe_bf16_t* residual_out, moe_stream_t stream) {
  moe_status_t st = check_shape(s);
  if (st != MOE_OK) return st;
  if (!x || !y || !topk_w || !gamma || !out) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y) || !aligned16(gamma) || !aligned16(out) ||
      (residual_out && !aligned16(residual_out)))
    return MOE_ERR_INVALID_ARG;
  if (!(eps >= 0.0f)) return MOE_ERR_INVALID_ARG;
  return cuda_status(moe::launch_finalize(x, y, topk_w, gamma, eps, s.M, s.top_k, s.H, out, residual_out,
                                          static_cast<cudaStream_t>(stream)));
}

size_t moe_layer_workspace_size(moe_shape_t s, moe_wdtype_t dtype) {
  if (check_shape(s) != MOE_OK) return 0;
  return layer_layout(s, dtype).total;
}

moe_status_t moe_layer_workspace_layout(moe_shape_t s, moe_wdtype_t dtype, moe_layer_ws_layout_t* layout) {
  moe_status_t st = check_shape(s);
  if (st != MOE_OK) return st;
  if (!layout) return MOE_ERR_INVALID_ARG;
  *layout = layer_layout(s, dtype);
  return MOE_OK;
}

moe_status_t moe_layer(const moe_bf16_t* x, const moe_bf16_t* w_router, const float* bias, const moe_weights_t* w,
                       const moe_bf16_t* gamma, float eps, moe_shape_t s, moe_bf16_t* out, moe_bf16_t* residual_out,
                       int32_t* topk_ids_out, float* topk_w_out, void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status_t st = check_layer_args(x, w_router, w, gamma, eps, s, out, residual_out);
  if (st != MOE_OK) return st;
  const moe_layer_ws_layout_t L = layer_layout(s, w->dtype);
  if (!ws || ws_bytes < L.total || !aligned16(ws)) return MOE_ERR_WORKSPACE;
  auto cs = static_cast<cudaStream_t>(stream);
  auto* base = static_cast<uint8_t*>(ws);
  auto* err = reinterpret_cast<int32_t*>(base + L.err_flag);
  int32_t* ids = topk_ids_out ? topk_ids_out : reinterpret_cast<int32_t*>(base + L.topk_ids);
  float* tw = topk_w_out ? topk_w_out : reinterpret_cast<float*>(base + L.topk_w);
  auto* y = reinterpret_cast<moe_bf16_t*>(base + L.y);

  // the error word and the single-launch layer's counters, in one region
  if ((st = cuda_status(cudaMemsetAsync(err, 0, L.logits - L.err_flag, cs))) != MOE_OK) return st;
  if (want_fused_layer(s, w->dtype)) {
    st = run_layer_fused(x, w_router, bias, w, gamma, eps, s, out, residual_out, ids, tw, base, L, cs);
    if (st != MOE_ERR_UNSUPPORTED) return st;
  }
  if ((st = run_layer_to_y(x, w_router, bias, w, s, base, L, ids, tw, cs)) != MOE_OK) return st;
  return cuda_status(moe::launch_finalize(x, y, tw, gamma, eps, s.M, s.top_k, s.H, out, residual_out, cs));
}

size_t moe_tp_layer_workspace_size(moe_shape_t s) { return moe_layer_workspace_size(s, MOE_W_BF16); }

moe_status_t moe_tp_layer(const moe_bf16_t* x, const moe_bf16_t* w_router, const float* bias, const moe_weights_t* w,
                          const moe_bf16_t* gamma, float eps, moe_shape_t s, const moe_tp_group_t* g,
                          moe_bf16_t* out, moe_bf16_t* residual_out, int32_t* topk_ids_out, float* topk_w_out,
                          void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status_t st = check_layer_args(x, w_router, w, gamma, eps, s, out, residual_out);
  if (st != MOE_OK) return st;
  if (w->dtype != MOE_W_BF16) return MOE_ERR_UNSUPPORTED;
  if (g == nullptr || g->rank < 0 || g->rank >= g->world) return MOE_ERR_INVALID_ARG;
  if (g->world < 1 || g->world > MOE_TP_MAX_RANKS || s.M > g->max_tokens || s.H != g->hidden)
    return MOE_ERR_UNSUPPORTED;
  if (g->world > 1)
    for (int r = 0; r < g->world; ++r)
      if (g->bufs[r] == nullptr || (reinterpret_cast<uintptr_t>(g->bufs[r]) & 255u) != 0) return MOE_ERR_INVALID_ARG;
  const moe_layer_ws_layout_t L = layer_layout(s, MOE_W_BF16);
  if (!ws || ws_bytes < L.total || !aligned16(ws)) return MOE_ERR_WORKSPACE;
  auto cs = static_cast<cudaStream_t>(stream);
  auto* base = static_cast<uint8_t*>(ws);
  auto* err = reinterpret_cast<int32_t*>(base + L.err_flag);
  int32_t* ids = topk_ids_out ? topk_ids_out : reinterpret_cast<int32_t*>(base + L.topk_ids);
  float* tw = topk_w_out ? topk_w_out : reinterpret_cast<float*>(base + L.topk_w);
  const auto* y = reinterpret_cast<const uint16_t*>(base + L.y);
  if ((st = cuda_status(cudaMemsetAsync(err, 0, L.logits - L.err_flag, cs))) != MOE_OK) return st;
  // this rank's partial expert rows (its slice of I), then the finalize fused with the exchange
  if ((st = run_layer_to_y(x, w_router, bias, w, s, base, L, ids, tw, cs)) != MOE_OK) return st;
  const uint16_t* ys[1] = {y};
  uint16_t* outs[1] = {out};
  uint16_t* rs[1] = {residual_out};
  return cuda_status(moe::launch_tp_finalize(x, ys, tw, gamma, eps, s.M, s.top_k, s.H, g->world, g->max_tokens,
                                             g->rank, 1, g->bufs, outs, rs, err, cs));
}

int moe_layer_kernel_count(moe_shape_t s, moe_wdtype_t dtype) {
  if (check_shape(s) != MOE_OK || (dtype != MOE_W_BF16 && dtype != MOE_W_NVFP4)) return -1;
  // routing: logits + top-k, or screened: digits, integer partial logits, candidates + exact logits + top-k
  const int route = route_screens(s) ? 3 : 2;
  if (dtype == MOE_W_NVFP4)  // routing, align, amax x, quantize x, gather tiles, up (+ amax h), quantize h, down, finalize
    return route + 8;
  if (want_fused_layer(s, dtype)) return 1;      // the whole layer in one launch
  if (want_self_route(s, dtype)) return route + 3;  // routing, up with the plan, down, finalize
  return route + 4 + (up_pregathers(s) ? 1 : 0);   // routing, align, [gather x], up, down, finalize
}

moe_status_t moe_quantize_nvfp4(const moe_bf16_t* src, int64_t n_mats, int64_t rows, int64_t cols, uint8_t* codes,
                                uint8_t* scales, float* gs, void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (n_mats < 1 || rows < 1 || cols < 16 || cols % 16 != 0) return MOE_ERR_UNSUPPORTED;
  if (!src || !codes || !scales || !gs) return MOE_ERR_INVALID_ARG;
  if (!aligned16(src) || !aligned16(codes) || !aligned16(scales)) return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < moe_nvfp4_quantize_workspace_size(n_mats) || !aligned16(ws)) return MOE_ERR_WORKSPACE;
  return cuda_status(moe::launch_nvfp4_quantize(src, n_mats, rows, cols, codes, scales, gs,
                                                static_cast<unsigned*>(ws), static_cast<cudaStream_t>(stream)));
}

size_t moe_nvfp4_quantize_workspace_size(int64_t n_mats) {
  return n_mats < 1 ? 0 : align_up(static_cast<size_t>(n_mats) * 4);
}

moe_status_t moe_prepare_nvfp4_weights(const uint8_t* codes, const uint8_t* scales, moe_shape_t s, int which,
                                       void* blob, size_t blob_bytes, moe_stream_t stream) {
  moe_status_t st = check_shape(s);
  if (st != MOE_OK) return st;
  if (which < 0 || which > 2) return MOE_ERR_INVALID_ARG;
  if (!codes || !scales || !blob || !aligned16(codes) || !aligned16(blob)) return MOE_ERR_INVALID_ARG;
  if (blob_bytes < moe_nvfp4_blob_bytes(s, which)) return MOE_ERR_WORKSPACE;
  int64_t rows, cols;
  blob_dims(s, which, &rows, &cols);
  auto cs = static_cast<cudaStream_t>(stream);
  auto* b = static_cast<uint8_t*>(blob);
  if (cudaMemcpyAsync(b, codes, static_cast<size_t>(rows) * cols / 2, cudaMemcpyDeviceToDevice, cs) != cudaSuccess)
    return MOE_ERR_CUDA;
  return cuda_status(moe::launch_nvfp4_scales_to_atoms(scales, rows, cols, b + blob_codes_bytes(s, which), cs));
}

size_t moe_nvfp4_blob_bytes(moe_shape_t s, int which) {
  if (check_shape(s) != MOE_OK || which < 0 || which > 2) return 0;
  int64_t rows, cols;
  blob_dims(s, which, &rows, &cols);
  return static_cast<size_t>(rows) * cols / 2 + static_cast<size_t>(rows) * cols / 16;
}

moe_status_t moe_selftest_wait_timeout(int32_t* err_flag, uint32_t limit_us, moe_stream_t stream) {
  if (!err_flag) return MOE_ERR_INVALID_ARG;
  if (limit_us == 0 || limit_us > 1000000u) return MOE_ERR_INVALID_ARG;
  return cuda_status(moe::launch_wait_timeout_selftest(err_flag, static_cast<uint64_t>(limit_us) * 1000ull,
                                                       static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_get_device_error(const int32_t* err_flag, moe_stream_t stream, int32_t* host_code) {
  if (!err_flag || !host_code) return MOE_ERR_INVALID_ARG;
  int32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, err_flag, sizeof(v), cudaMemcpyDeviceToHost, static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  if (v & moe::kErrTimeout)
    *host_code = MOE_ERR_TIMEOUT;
  else if (v & moe::kErrInvalidInput)
    *host_code = MOE_ERR_INVALID_INPUT;
  else if (v & moe::kErrUnsupported)
    *host_code = MOE_ERR_UNSUPPORTED;
  else
    *host_code = MOE_OK;
  return MOE_OK;
}

}  // extern "C"
