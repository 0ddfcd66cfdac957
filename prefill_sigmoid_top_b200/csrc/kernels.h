// Internal launchers shared between the kernel files and the C-ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe_b200.h"

namespace moe {

// api.cu: validation of moe_route's arguments (a moe_status_t value).
// 2-D bf16 tensor map [rows, cols] with boxes of box_rows x 64 elements and the 128-byte swizzle.
bool encode_map_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);
// 2-D byte tensor map [rows, cols_bytes] with boxes of box_rows x 128 bytes and the 128-byte swizzle.
bool encode_map_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols_bytes, uint32_t box_rows);
// Bytes as a [bytes / 256, 256] tensor read in unswizzled boxes of box_rows x 256 bytes (NVFP4 scale atoms).
bool encode_map_sf_rows(CUtensorMap* map, const void* base, uint64_t bytes, uint32_t box_rows);

// router_screen.cu: routing of many tokens from exact canonical logits of the candidate experts only
// (the same ids and weights as launch_router_logits + launch_router_topk).
bool screen_shape_ok(int M, int H, int E, int K);   // shapes it takes (sizes the workspaces)
bool screen_eligible(int M, int H, int E, int K);   // shapes it takes, unless MOE_ROUTER_SCREEN=0
size_t screen_scratch_bytes(int M, int H, int E);   // device scratch it needs (16-byte aligned base)
cudaError_t launch_route_screened(const uint16_t* x, const uint16_t* w_router, const float* bias, int M, int H, int E,
                                  int K, uint8_t* scratch, int32_t* topk_ids, float* topk_w, int32_t* err,
                                  cudaStream_t stream);

int check_route_args(const moe_shape_t& s, const void* x, const void* w_router, const void* topk_ids,
                     const void* topk_w);

// router.cu
cudaError_t launch_router_logits(const uint16_t* x, const uint16_t* w_router, const float* bias, int M, int H, int E,
                                 float* logits, cudaStream_t stream);
cudaError_t launch_router_topk(const float* logits, int M, int E, int K, int32_t* topk_ids, float* topk_w,
                               cudaStream_t stream);
cudaError_t launch_router_topk_ext(const float* logits, const float* sel_bias, int M, int E, int K, int scoring,
                                   int renormalize, float scale, int32_t* topk_ids, float* topk_w,
                                   cudaStream_t stream);

// align.cu
cudaError_t launch_align(const int32_t* topk_ids, int M, int K, int E, int B, int32_t* sorted_ids,
                         int32_t* block_expert, int32_t* expert_counts, int32_t* expert_offsets, int32_t* ntpp,
                         int32_t* err, cudaStream_t stream);

// finalize.cu
cudaError_t launch_finalize(const uint16_t* x, const uint16_t* y, const float* topk_w, const uint16_t* gamma,
                            float eps, int M, int K, int H, uint16_t* out, uint16_t* residual_out,
                            cudaStream_t stream);

// tp_finalize.cu: the tensor-parallel finalize (reduction across ranks fused with the norm).
// `rows` CTA rows play ranks rank0 .. rank0 + rows - 1 (1 for a real rank; G when all ranks
// are emulated on one GPU); ys / outs / residual_outs hold one pointer per row, bufs one
// group buffer per rank (null when G == 1).
cudaError_t launch_tp_finalize(const uint16_t* x, const uint16_t* const* ys, const float* topk_w,
                               const uint16_t* gamma, float eps, int M, int K, int H, int G, int max_tokens,
                               int rank0, int rows, void* const* bufs, uint16_t* const* outs,
                               uint16_t* const* residual_outs, int32_t* err, cudaStream_t stream);
size_t tp_buffer_bytes(int G, int max_tokens, int H);
int tp_protocol(int M, int G, int max_tokens);

// finalize.cu: one-warp kernel whose bounded wait can never be satisfied.
cudaError_t launch_wait_timeout_selftest(int32_t* err, uint64_t limit_ns, cudaStream_t stream);

// gemm_bf16.cu: grouped projections over the expert-major plan.
struct GroupedGemmArgs {
  const int32_t* sorted_ids;
  const int32_t* expert_counts;
  const int32_t* expert_offsets;
  uint16_t* out;       // up: h [cap, I]; down: y [M*K, H]
  int32_t* err;        // device error word (nullable)
  int M, E, top_k;
  int rows_per_expert; // up: I; down: H  (weight rows of one expert)
  int kdim;            // up: H; down: I  (contraction length)
  int out_ld;          // up: I; down: H
  // Self-routing up only (null otherwise): the routed ids it reads instead of
  // the plan, and the plan it writes for the kernels that follow.
  const int32_t* topk_ids;
  int block_size;
  int32_t* plan_sorted_ids;
  int32_t* plan_block_expert;
  int32_t* plan_counts;
  int32_t* plan_offsets;
  int32_t* plan_ntpp;
};

// Largest M*top_k the self-routing up kernel accepts (the ids are staged in
// shared memory and scanned by one warp per CTA).
constexpr int kRouteMaxSlots = 1024;

// `nmax` selects the token-tile width (32 or 128).  Tensor maps: a0/a1 are
// the weight matrices viewed as 2-D [E*rows_per_expert, kdim]; b is x [M,H]
// (up, row gather) or h [cap, I] (down, contiguous rows).
// `gathered`: x_rows maps x already gathered into plan order ([cap, H],
// 16-row boxes); otherwise x itself ([M, H], one-row boxes for tile::gather4).
cudaError_t launch_grouped_up(const CUtensorMap& w_gate, const CUtensorMap& w_up, const CUtensorMap& x_rows,
                              const GroupedGemmArgs& args, int nmax, bool gathered, cudaStream_t stream);
// xg[r] = x[sorted_ids[r] / top_k] for the real plan rows r < ntpp.
cudaError_t launch_gather_rows(const uint16_t* x, const int32_t* sorted_ids, const int32_t* ntpp, int M, int top_k,
                               int H, int cap, uint16_t* xg, cudaStream_t stream);
// 2-SM pair variants of the persistent kernels (gemm_pair.cu): token tiles of
// `nmax` plan rows (128 or 256) split over the two CTAs of a cluster; the
// token-row tensor is plan-ordered (x gathered, or h) in 32-row boxes.
cudaError_t launch_pair_up(const CUtensorMap& w_gate, const CUtensorMap& w_up, const CUtensorMap& x_rows,
                           const GroupedGemmArgs& args, int nmax, int num_sms, cudaStream_t stream,
                           bool gather_b = false);
cudaError_t launch_pair_down(const CUtensorMap& w_down, const CUtensorMap& h_rows, const GroupedGemmArgs& args,
                             int nmax, int num_sms, cudaStream_t stream);

// Decode up projection that builds the plan itself from topk_ids (32-row
// token tiles, x rows gathered by token id) and writes it for the down and
// finalize kernels: the align step folded into the up kernel.
cudaError_t launch_grouped_up_routed(const CUtensorMap& w_gate, const CUtensorMap& w_up, const CUtensorMap& x_rows,
                                     const GroupedGemmArgs& args, cudaStream_t stream);
cudaError_t launch_grouped_down(const CUtensorMap& w_down, const CUtensorMap& h_rows, const GroupedGemmArgs& args,
                                int nmax, cudaStream_t stream);

// gemm_persistent.cu: one CTA per SM over a static tile list, 128-row token
// tiles.  xg_rows / h_rows: plan-ordered [cap, kdim] tensors in 32-row boxes.
// Weight tiles: up = 128 rows of gate and of up; down = 256 rows of W_down.
// gather: x_rows maps x itself ([M,H], one-row boxes) and the kernel gathers
// token rows with tile::gather4; otherwise x_rows is x in plan order.
// deep_b: 4 weight stages + 5 token-row stages instead of 5 + 3.
cudaError_t launch_persistent_up(const CUtensorMap& w_gate, const CUtensorMap& w_up, const CUtensorMap& x_rows,
                                 const GroupedGemmArgs& args, int nmax, bool gather, bool deep_b, int num_sms,
                                 cudaStream_t stream);
cudaError_t launch_persistent_down(const CUtensorMap& w_down, const CUtensorMap& h_rows, const GroupedGemmArgs& args,
                                   int nmax, bool deep_b, int num_sms, cudaStream_t stream);

// Device error bit of a kernel that cannot run as launched (layer_fused.cu:
// a dynamic shared-memory base that is not 1024-byte aligned): MOE_ERR_UNSUPPORTED.
constexpr int32_t kErrUnsupported = 1 << 2;

// layer_fused.cu: the decode-shaped layer (route, plan, up, down, finalize)
// in one cooperative launch.  `sync` points at 3 + E (+ 9 M when M <= 64)
// words that are zero when the launch starts: grid barrier, work counter,
// finalize count, one up-tile count per expert, then per token a count of
// finalize slices and their 8 partial sums of squares.
struct FusedLayerArgs {
  const uint16_t* x;         // [M, H]
  const uint16_t* w_router;  // [E, H]
  const float* bias;         // [E] or null
  const uint16_t* gamma;     // [H]
  float eps;
  int M, H, I, E, top_k, block_size;
  float* logits;             // [M, E] scratch
  int32_t* topk_ids;         // [M, top_k]
  float* topk_w;             // [M, top_k]
  int32_t* sorted_ids;       // the plan, as moe_align_block_size writes it
  int32_t* block_expert;
  int32_t* counts;
  int32_t* offsets;
  int32_t* ntpp;
  uint16_t* h;               // [cap, I]
  uint16_t* y;               // [M*top_k, H]
  uint16_t* out;             // [M, H]
  uint16_t* residual_out;    // [M, H] or null
  int32_t* err;
  unsigned* sync;
};
// Tensor maps: W_gate / W_up as [E*I, H] and W_down as [E*H, I] in 128-row
// boxes, x as [M, H] in one-row boxes (tile::gather4), h as [cap, I] in
// 16-row boxes.
cudaError_t launch_layer_fused(const CUtensorMap& w_gate, const CUtensorMap& w_up, const CUtensorMap& w_down,
                               const CUtensorMap& x_rows, const CUtensorMap& h_rows, const FusedLayerArgs& args,
                               int num_sms, cudaStream_t stream);
int layer_fused_smem_bytes(int E, int nslots);

// nvfp4.cu ------------------------------------------------------------------
struct Nvfp4GemmArgs {
  GroupedGemmArgs g;      // kdim in elements; out / plan / shape as for bf16
  const uint8_t* sfa0;    // weight scale atoms of the tm_a0 rows ([rows/128][kdim/64][512])
  const uint8_t* sfa1;    // of the tm_a1 rows (up: W_up; down: W_down again)
  const uint8_t* sfb;     // activation scale atoms, tile-aligned ([tiles][kdim/64][512])
  const float* gs_a0;     // [E] global scales of the tm_a0 matrix
  const float* gs_a1;     // [E]
  const unsigned* act_amax;  // activation amax (fp32 bits); gs = amax / 2688
  unsigned* out_amax;        // up only, nullable: max |h| over the h values written (fp32 bits, atomic max)
};

// Quantise n_mats matrices [rows, cols] (bf16, back to back) to NVFP4 codes /
// row-major e4m3 scales / per-matrix global scales; amax_bits: n_mats words.
cudaError_t launch_nvfp4_quantize(const uint16_t* src, int64_t n_mats, int64_t rows, int64_t cols, uint8_t* codes,
                                  uint8_t* scales, float* gs, unsigned* amax_bits, cudaStream_t stream);
cudaError_t launch_nvfp4_scales_to_atoms(const uint8_t* scales, int64_t rows, int64_t cols, uint8_t* atoms,
                                         cudaStream_t stream);
// *amax_bits = max(*amax_bits, max |src[0..n)|) (bits of a non-negative float).
cudaError_t launch_amax_all(const uint16_t* src, int64_t n, unsigned* amax_bits, cudaStream_t stream);
cudaError_t launch_amax_plan_rows(const uint16_t* h, const int32_t* sorted_ids, const int32_t* ntpp, int nslots,
                                  int cols, int cap, unsigned* amax_bits, cudaStream_t stream);
// h (plan order) -> tile-aligned NVFP4 codes / scale atoms (global scale from *amax_bits).
cudaError_t launch_quantize_tiles(const uint16_t* src, const int32_t* counts, const int32_t* offsets, int E, int cols,
                                  int tiles_ub, const unsigned* amax_bits, uint8_t* codes, uint8_t* atoms,
                                  cudaStream_t stream);
// rows x cols bf16 -> codes [rows, cols/2], row-major scales [rows, cols/16] (global scale from *amax_bits).
cudaError_t launch_quantize_rows(const uint16_t* src, int64_t rows, int64_t cols, const unsigned* amax_bits,
                                 uint8_t* codes, uint8_t* scales, cudaStream_t stream);
// per-token codes / scales -> tile-aligned copy of the routed slots (row r of tile ti <- token sorted_ids[..] / top_k).
cudaError_t launch_gather_tiles(const uint8_t* tok_codes, const uint8_t* tok_scales, const int32_t* sorted_ids,
                                const int32_t* counts, const int32_t* offsets, int E, int top_k, int nslots, int cols,
                                int tiles_ub, uint8_t* codes, uint8_t* atoms, cudaStream_t stream);
cudaError_t launch_nvfp4_up(const CUtensorMap& gate_codes, const CUtensorMap& up_codes, const CUtensorMap& x_codes,
                            const Nvfp4GemmArgs& args, int num_sms, cudaStream_t stream);
cudaError_t launch_nvfp4_down(const CUtensorMap& down_codes, const CUtensorMap& h_codes, const Nvfp4GemmArgs& args,
                              int num_sms, cudaStream_t stream);

// nvfp4_pair.cu: the same projections on 2-SM pairs; the *_sf maps read the scale atoms of the matching
// operand as 256-byte rows (up: I % 256 == 0; down: H % 512 == 0).
cudaError_t launch_nvfp4_pair_up(const CUtensorMap& gate_codes, const CUtensorMap& up_codes,
                                 const CUtensorMap& x_codes, const CUtensorMap& gate_sf, const CUtensorMap& up_sf,
                                 const CUtensorMap& x_sf, const Nvfp4GemmArgs& args, int num_sms, cudaStream_t stream);
cudaError_t launch_nvfp4_pair_down(const CUtensorMap& down_codes, const CUtensorMap& h_codes,
                                   const CUtensorMap& down_sf, const CUtensorMap& h_sf, const Nvfp4GemmArgs& args,
                                   int num_sms, cudaStream_t stream);

}  // namespace moe
