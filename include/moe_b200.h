/*
 * moe_b200.h -- C ABI of libmoe_b200.so: one routed Mixture-of-Experts layer
 * with sigmoid top-k routing on an NVIDIA B200 (sm_100a).
 *
 * The layer, step by step (the pages that describe the method, cited by page
 * title and section):
 *   1. route     sigmoid scores over E experts, top-k, weights renormalised to
 *                sum to 1 ("[sglang] [NPU] GLM-4.7-Flash 성능 최적화",
 *                sglang PR #29509 analysis, §2 "MoE TopK Scoring Function").
 *   2. align     expert-major block plan: per-expert histogram, prefix scan,
 *                padding to the block size, block -> expert by search
 *                ("[flashinfer] ... AlphaMoE NVFP4 커널 최적화", flashinfer
 *                PR #6511 analysis, §5 "moe_align_block_size_kernel 동기화 개선").
 *   3. up        grouped gate/up projection with SwiGLU fused in the epilogue
 *                (same page, §3-§4, the "up" kernels of the route chain, §6).
 *   4. down      grouped down projection (same page, §1-§2, the "down" kernels).
 *   5. finalize  top-k weighted sum + residual add + RMSNorm, one pass, no
 *                intermediate in HBM ("[flashinfer] Kimi K3를 위한 초고속 통신
 *                최적화", flashinfer PR #5701 analysis, intro and §2 HT preset:
 *                H=7168 = 896 bf16x8 packs; §3: RMS_EPS=1e-5, WEIGHT_BIAS=0).
 *   moe_layer    runs 1-5 on one stream (PR #6511 analysis, §6 route chain);
 *                on decode shapes as a single launch.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers to caller-allocated memory,
 *    row-major, 16-byte aligned.  The library allocates nothing and keeps no
 *    state between calls other than cached device properties.
 *  - bf16 tensors are passed as moe_bf16_t (raw bfloat16 bits).
 *  - Every call validates its arguments on the host first; on a problem it
 *    returns a status and launches nothing.  Otherwise it enqueues its kernels
 *    asynchronously on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and returns MOE_OK, or MOE_ERR_CUDA if a launch failed.
 *  - Problems only visible on the device (e.g. an expert id outside [0,E))
 *    never trap: the kernel ORs a bit into the int32 word at `err_flag`
 *    (nullable: then they are silently ignored) and the affected outputs are
 *    unspecified.  Read it with moe_get_device_error().  Bit (1 << status)
 *    is set for status MOE_ERR_INVALID_INPUT or MOE_ERR_TIMEOUT, or
 *    MOE_ERR_UNSUPPORTED for a launch the kernel found it cannot run (the
 *    single-launch layer given shared memory without 1024-byte alignment).
 *  - Waits inside kernels are bounded (0.5 s each); on expiry the kernel
 *    sets the MOE_ERR_TIMEOUT bit and returns.
 *  - Accepted shapes: M >= 1; H % 256 == 0 and H <= 8192; I % 128 == 0
 *    (I % 256 == 0 with MOE_W_NVFP4 weights);
 *    1 <= top_k <= min(E, 32); 1 <= E <= 1024; block_size a power of two in
 *    [16, 256]; M * top_k < 2^31.  Others return MOE_ERR_UNSUPPORTED.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad scalar */
  MOE_ERR_UNSUPPORTED = 2,   /* shape or dtype outside the accepted set */
  MOE_ERR_WORKSPACE = 3,     /* workspace missing or too small */
  MOE_ERR_INVALID_INPUT = 4, /* device-detected: expert id out of range */
  MOE_ERR_TIMEOUT = 5,       /* device-detected: a bounded wait expired */
  MOE_ERR_CUDA = 6           /* a CUDA runtime call or launch failed */
} moe_status_t;

typedef uint16_t moe_bf16_t; /* raw bfloat16 bits */
typedef void* moe_stream_t;  /* cudaStream_t */

/* M tokens, hidden H, expert intermediate I, E experts, top_k, align block size. */
typedef struct {
  int32_t M, H, I, E, top_k, block_size;
} moe_shape_t;

typedef enum { MOE_W_BF16 = 0, MOE_W_NVFP4 = 1 } moe_wdtype_t;

/* Expert weights.
 * MOE_W_BF16:  gate, up: bf16 [E, I, H]; down: bf16 [E, H, I] (the contraction
 *              dimension is contiguous); the *_gs pointers are ignored.
 * MOE_W_NVFP4: gate, up, down: blobs written by moe_prepare_nvfp4_weights
 *              (from moe_quantize_nvfp4 of W_gate/W_up as E matrices [I,H] and
 *              W_down as E matrices [H,I]); gate_gs, up_gs, down_gs: the device
 *              fp32 [E] per-expert global scales that moe_quantize_nvfp4 wrote. */
typedef struct {
  moe_wdtype_t dtype;
  const void* gate;
  const void* up;
  const void* down;
  const float* gate_gs;
  const float* up_gs;
  const float* down_gs;
} moe_weights_t;

/* The expert-major plan written by moe_align_block_size (device pointers). */
typedef struct {
  const int32_t* sorted_ids;             /* [cap]: flat slot ids t*top_k+k, pad = M*top_k */
  const int32_t* block_expert;           /* [cap / block_size] */
  const int32_t* expert_counts;          /* [E] */
  const int32_t* expert_offsets;         /* [E+1], multiples of block_size */
  const int32_t* num_tokens_post_padded; /* [1] = expert_offsets[E] */
} moe_plan_t;

/* ---------------------------------------------------------------- route --
 * Sigmoid top-k routing (sglang PR #29509 analysis, §2).
 *   z[t,e]  = sum_h x[t,h] * w_router[e,h] + bias[e], fp32 in a fixed order:
 *             32 partial sums, partial l accumulating (one fma per element, in
 *             increasing h) every h with floor(h/8) % 32 == l; partials
 *             combined pairwise l += l+16, +8, +4, +2, +1; then + bias[e].
 *   topk_ids[t,0..K) = the K largest z[t,:], descending, ties -> lower id.
 *   topk_w[t,k] = s_k / sum_j s_j with s = 1 / (1 + exp(-z)).
 * x: bf16 [M,H]; w_router: bf16 [E,H]; bias: fp32 [E] (nullable -> 0);
 * topk_ids: int32 [M,K]; topk_w: fp32 [M,K];
 * ws: device scratch of at least moe_route_workspace_size(s) bytes. */
MOE_API moe_status_t moe_route(const moe_bf16_t* x, const moe_bf16_t* w_router, const float* bias, moe_shape_t s,
                       int32_t* topk_ids, float* topk_w, void* ws, size_t ws_bytes, moe_stream_t stream);
MOE_API size_t moe_route_workspace_size(moe_shape_t s);

/* -------------------------------------------------------- route variants --
 * The routing variants of the same fused top-k (sglang PR #29509 analysis,
 * §2: its norm_type selects softmax (0) or sigmoid (1) scores).
 * The selection key is z as above, except that with bias_in_score == 0 the
 * bias is left out of z and added to the key only: key = fp32(z + bias[e]).
 * topk_ids = the K largest keys, descending, ties -> lower id.  With z_k the
 * logit (bias_in_score == 0: without the bias) of the k-th selected expert:
 *   scoring SIGMOID: p_k = 1 / (1 + exp(-z_k))
 *   scoring SOFTMAX: p_k = exp(z_k) / sum_e exp(z[t,e]), over all E experts
 *   w_k = (renormalize ? p_k / sum_j p_j : p_k) * routed_scale
 * {SIGMOID, renormalize 1, bias_in_score 1, routed_scale 1} is moe_route.
 * Arguments, layouts, workspace and errors as moe_route; opts is a host
 * pointer, read during the call; INVALID_ARG for a null opts, an unknown
 * scoring, or a routed_scale that is not finite and > 0. */
typedef enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 } moe_score_t;
typedef struct {
  int32_t scoring;       /* moe_score_t */
  int32_t renormalize;   /* nonzero: renormalise over the K selected */
  int32_t bias_in_score; /* nonzero: bias is part of z; zero: it shifts the selection key only */
  float routed_scale;    /* multiplies every weight */
} moe_route_opts_t;
MOE_API moe_status_t moe_route_ex(const moe_bf16_t* x, const moe_bf16_t* w_router, const float* bias, moe_shape_t s,
                                  const moe_route_opts_t* opts, int32_t* topk_ids, float* topk_w, void* ws,
                                  size_t ws_bytes, moe_stream_t stream);

/* ---------------------------------------------------------------- align --
 * Expert-major block plan (flashinfer PR #6511 analysis, §5).
 *   expert_counts[e]      = #{f : topk_ids[f] == e}, f = t*K + k
 *   expert_offsets[0] = 0, expert_offsets[e+1] = expert_offsets[e] + roundup(count[e], B)
 *   sorted_ids[offsets[e] + j] = the j-th f (ascending) with topk_ids[f] == e,
 *                         for j < count[e]; the rest of the segment = M*K
 *   block_expert[b]       = e with offsets[e] <= b*B < offsets[e+1]
 *   num_tokens_post_padded[0] = offsets[E]
 * Output sizes: sorted_ids holds moe_align_capacity(s) ints, block_expert
 * moe_align_capacity(s)/B ints; only sorted_ids[0, ntpp) and
 * block_expert[0, ntpp/B) are written.  An id outside [0,E) sets
 * MOE_ERR_INVALID_INPUT in err_flag and the plan is unspecified. */
MOE_API moe_status_t moe_align_block_size(const int32_t* topk_ids, moe_shape_t s, int32_t* sorted_ids,
                                  int32_t* block_expert, int32_t* expert_counts, int32_t* expert_offsets,
                                  int32_t* num_tokens_post_padded, int32_t* err_flag, moe_stream_t stream);
MOE_API size_t moe_align_capacity(moe_shape_t s); /* M*top_k + E*(block_size-1) */

/* ---------------------------------------------------------------- up -----
 * Grouped gate/up projection with fused SwiGLU, in plan order (flashinfer
 * PR #6511 analysis, §3-§4).  For every plan row r < ntpp that is not padding,
 * with e the expert of its segment and t = sorted_ids[r] / K:
 *   g = x[t] . w.gate[e]^T,  u = x[t] . w.up[e]^T   (fp32 accumulation)
 *   h[r, :] = bf16(silu(g) * u),   silu(g) = g / (1 + exp(-g))
 * h: bf16 [moe_align_capacity(s), I]; padding rows are not written.
 * ws (nullable): moe_up_workspace_size(s, dtype) bytes of device scratch.  With
 * it, wide token tiles first gather x into plan order there and read it as
 * contiguous rows; without it the rows are gathered inside the GEMM.  Both
 * give the same result.  MOE_W_NVFP4: x is quantised on the fly (global scale
 * from the amax over all of x) into ws (required), and the accumulators are
 * scaled by gs_gate[e] * gs_x and gs_up[e] * gs_x before SwiGLU; the block-
 * scaled GEMM runs on 2-SM pairs (cta_group::2) when I % 256 == 0 and on
 * single SMs otherwise or with MOE_NVFP4_PAIR=0 in the environment, with the
 * same bits either way. */
MOE_API moe_status_t moe_grouped_up_swiglu(const moe_bf16_t* x, const moe_weights_t* w, const moe_plan_t* plan,
                                   moe_shape_t s, moe_bf16_t* h, void* ws, size_t ws_bytes, int32_t* err_flag,
                                   moe_stream_t stream);
MOE_API size_t moe_up_workspace_size(moe_shape_t s, moe_wdtype_t dtype);

/* ------------------------------------------------------ self-routing up --
 * moe_align_block_size and moe_grouped_up_swiglu in one launch (flashinfer
 * PR #6511 analysis, §6: the align step folded into the first GEMM of the
 * route chain, one launch fewer).  Every CTA of the up projection builds what
 * it needs of the expert-major plan from topk_ids itself, computes its tile
 * exactly as moe_grouped_up_swiglu does (32-row token tiles, x rows gathered
 * by token id), and writes its part of the plan, so that on return the plan
 * arrays hold exactly what moe_align_block_size writes and h exactly what
 * moe_grouped_up_swiglu writes for that plan.
 * x: bf16 [M,H]; w: MOE_W_BF16 weights; topk_ids: int32 [M,top_k] (device);
 * plan outputs (device, sizes as moe_align_block_size); h: bf16 [cap, I];
 * err_flag: device int32 (nullable), MOE_ERR_INVALID_INPUT if an id lies
 * outside [0,E) (outputs then unspecified).
 * Limit: M*top_k <= MOE_ROUTED_UP_MAX_SLOTS, else MOE_ERR_UNSUPPORTED;
 * NVFP4 weights: MOE_ERR_UNSUPPORTED.  moe_layer takes this path by itself on
 * decode shapes. */
#define MOE_ROUTED_UP_MAX_SLOTS 1024
MOE_API moe_status_t moe_grouped_up_swiglu_routed(const moe_bf16_t* x, const moe_weights_t* w,
                                                  const int32_t* topk_ids, moe_shape_t s, int32_t* sorted_ids,
                                                  int32_t* block_expert, int32_t* expert_counts,
                                                  int32_t* expert_offsets, int32_t* num_tokens_post_padded,
                                                  moe_bf16_t* h, int32_t* err_flag, moe_stream_t stream);

/* ---------------------------------------------------------------- down ---
 * Grouped down projection (flashinfer PR #6511 analysis, §1-§2).  For every
 * non-padding plan row r of expert e, with f = sorted_ids[r]:
 *   y[f, :] = bf16(h[r] . w.down[e]^T)   (fp32 accumulation)
 * h: bf16 [cap, I]; y: bf16 [M*top_k, H] (slot-major: y[t, k, :]).
 * MOE_W_NVFP4: h is quantised on the fly (global scale from the amax over the
 * real plan rows of h) into ws, moe_down_workspace_size(s, MOE_W_NVFP4) bytes
 * (required); the accumulators are scaled by gs_down[e] * gs_h; 2-SM pairs
 * when H % 512 == 0 (MOE_NVFP4_PAIR=0: single SMs), the same bits either way. */
MOE_API moe_status_t moe_grouped_down(const moe_bf16_t* h, const moe_weights_t* w, const moe_plan_t* plan,
                              moe_shape_t s, moe_bf16_t* y, void* ws, size_t ws_bytes, int32_t* err_flag,
                              moe_stream_t stream);
MOE_API size_t moe_down_workspace_size(moe_shape_t s, moe_wdtype_t dtype);

/* ---------------------------------------------------------------- finalize
 * Top-k weighted sum fused with residual add and RMSNorm (flashinfer PR #5701
 * analysis; WEIGHT_BIAS = 0, so gamma multiplies as is):
 *   s[t,:] = x[t,:] + sum_k topk_w[t,k] * y[t,k,:]                 (fp32)
 *   out[t,:] = bf16( s * rsqrt(mean_h(s^2) + eps) * gamma )
 *   residual_out[t,:] = bf16(s)                    (residual_out nullable)
 * x: bf16 [M,H]; y: bf16 [M,K,H]; topk_w: fp32 [M,K]; gamma: bf16 [H]. */
MOE_API moe_status_t moe_finalize_rmsnorm(const moe_bf16_t* x, const moe_bf16_t* y, const float* topk_w,
                                  const moe_bf16_t* gamma, float eps, moe_shape_t s, moe_bf16_t* out,
                                  moe_bf16_t* residual_out, moe_stream_t stream);

/* ---------------------------------------------------------------- layer --
 * The whole layer on one stream: route -> align -> up -> down -> finalize
 * (flashinfer PR #6511 analysis, §6 route chain), with the same results as
 * calling those entry points in turn.  On decode shapes (MOE_W_BF16, at most
 * 24 routed rows per expert on average, M*top_k <= MOE_ROUTED_UP_MAX_SLOTS,
 * E <= 256) the layer is ONE cooperative launch (one 192-thread CTA per SM: the
 * router, a grid barrier, the plan, the up and down tiles handed out by a
 * device-side counter with the down tiles of an expert waiting for its up
 * tiles, then the finalize; the megakernel of "AWS Trainium2에서 GLM-5.3-Flash를
 * 위한 NKI 레이어 메가커널"), bit-identical to the separate entry points;
 * MOE_FUSED_LAYER=0 in the environment selects the 5-launch form instead, in
 * which the align step runs inside the up projection
 * (moe_grouped_up_swiglu_routed); moe_layer also takes it by itself when the
 * single launch cannot be made (a GPU shared with other work that cannot
 * hold one CTA per SM at once).
 * Intermediates live in ws (moe_layer_workspace_size bytes, 256-byte aligned);
 * the first int32 of ws is the layer's device error word (cleared by each
 * call; read it with moe_get_device_error((const int32_t*)ws, ...)).
 * topk_ids_out / topk_w_out (nullable) receive the routing.  residual_out is
 * nullable.  All work is enqueued on `stream` (capturable in a CUDA graph). */
MOE_API moe_status_t moe_layer(const moe_bf16_t* x, const moe_bf16_t* w_router, const float* bias,
                       const moe_weights_t* w, const moe_bf16_t* gamma, float eps, moe_shape_t s,
                       moe_bf16_t* out, moe_bf16_t* residual_out, int32_t* topk_ids_out, float* topk_w_out,
                       void* ws, size_t ws_bytes, moe_stream_t stream);
MOE_API size_t moe_layer_workspace_size(moe_shape_t s, moe_wdtype_t dtype);

/* Number of kernels one moe_layer call launches for this shape and weight
 * type (the stream-ordered memsets of its error and scale words not counted);
 * -1 for an unsupported shape or dtype.  Host only, no CUDA call. */
MOE_API int moe_layer_kernel_count(moe_shape_t s, moe_wdtype_t dtype);

/* Byte offsets of the layer's intermediates inside ws (for inspection). */
typedef struct {
  size_t err_flag, logits, topk_ids, topk_w, sorted_ids, block_expert, expert_counts, expert_offsets,
      num_tokens_post_padded, h, y, act_scratch,
      sync, /* uint32 counters of the single-launch layer (3 + E, + 9 M for M <= 64), cleared with the error word */
      total;
} moe_layer_ws_layout_t;
MOE_API moe_status_t moe_layer_workspace_layout(moe_shape_t s, moe_wdtype_t dtype, moe_layer_ws_layout_t* layout);

/* ---------------------------------------------------------------- NVFP4 --
 * Weight preparation for MOE_W_NVFP4 (flashinfer PR #6511 analysis, intro:
 * e2m1 values with e4m3 per-16 block scales; §2: weights repacked offline by
 * a separate preparation step).  Quantises `n_mats` bf16 matrices of
 * [rows, cols] (cols % 16 == 0; blocks of 16 along cols) stored back to back:
 *   gs[m]   = amax(matrix m) / (6*448)   (1 if amax == 0)
 *   sb      = e4m3_rn_satfinite(blockamax / 6 / gs)
 *   q       = e2m1_rn_satfinite(v / (sb * gs))   (0 if sb == 0)
 * all in fp32.  codes: uint8 [n_mats, rows, cols/2] (two codes per byte, the
 * even column in the low nibble); scales: uint8 e4m3 [n_mats, rows, cols/16];
 * gs: fp32 [n_mats].  ws: moe_nvfp4_quantize_workspace_size(n_mats) bytes. */
MOE_API moe_status_t moe_quantize_nvfp4(const moe_bf16_t* src, int64_t n_mats, int64_t rows, int64_t cols,
                                uint8_t* codes, uint8_t* scales, float* gs, void* ws, size_t ws_bytes,
                                moe_stream_t stream);
MOE_API size_t moe_nvfp4_quantize_workspace_size(int64_t n_mats);

/* Repack quantised expert weights (codes/scales as written by
 * moe_quantize_nvfp4 for all E experts of one projection) into the blob the
 * grouped kernels read: the codes unchanged, then the scales regrouped into
 * 512-byte atoms of 128 rows x 64 columns (row r, column block j at byte
 * (r%32)*16 + ((r%128)/32)*4 + j%4 of atom [r/128][j/4]), the layout the
 * block-scaled tensor-core MMA takes its scale factors in.
 * which: 0 gate, 1 up, 2 down; blob: moe_nvfp4_blob_bytes(s, which) bytes. */
MOE_API moe_status_t moe_prepare_nvfp4_weights(const uint8_t* codes, const uint8_t* scales, moe_shape_t s, int which,
                                       void* blob, size_t blob_bytes, moe_stream_t stream);
MOE_API size_t moe_nvfp4_blob_bytes(moe_shape_t s, int which);

/* ---------------------------------------------------------------- route, no allocation
 * No counterpart on the pages: this entry point exists for callers that cannot
 * allocate device memory themselves, for example a plugin running inside a
 * host framework that owns every device allocation through its own pool, or a
 * caller with a fixed, pre-budgeted memory footprint.  moe_route needs a
 * caller-provided scratch buffer for the [M,E] fp32 router logits;
 * moe_route_noalloc computes exactly the same routing (same kernels, same
 * results) but keeps those logits in an array inside the library instead.
 *  - Limit: M * E <= MOE_ROUTE_NOALLOC_MAX_LOGITS (4 MiB of fp32 logits, e.g.
 *    M = 4096 tokens at E = 256); larger shapes return MOE_ERR_UNSUPPORTED
 *    without launching anything.
 *  - The array is a fixed 4 MiB device allocation made when the library is
 *    loaded; every GPU the process uses holds one until the process exits.
 *  - Every call looks up the array's device address on the current device
 *    (cudaGetSymbolAddress, which allocates nothing), so the address stays
 *    right after a device reset or a new primary context.  The first call
 *    on a device may load the library's device code there, so that first
 *    call should come before any stream capture on the device.
 *  - All calls share the one array: calls whose kernels may overlap on the
 *    GPU (other streams, other host threads) race and give wrong results, so
 *    serialise them.  Nothing needs clearing between calls: each call writes
 *    all M*E logits before it reads them.
 *  - It allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * Arguments, layouts and errors as moe_route, without ws / ws_bytes. */
#define MOE_ROUTE_NOALLOC_MAX_LOGITS (1 << 20)
MOE_API moe_status_t moe_route_noalloc(const moe_bf16_t* x, const moe_bf16_t* w_router, const float* bias,
                                       moe_shape_t s, int32_t* topk_ids, float* topk_w, moe_stream_t stream);

/* ---------------------------------------------------------------- errors -
 * Synchronises `stream`, reads the device error word and returns, in
 * *host_code, MOE_OK or the most severe device-detected status
 * (MOE_ERR_TIMEOUT before MOE_ERR_INVALID_INPUT before MOE_ERR_UNSUPPORTED).
 * Clears nothing. */
MOE_API moe_status_t moe_get_device_error(const int32_t* err_flag, moe_stream_t stream, int32_t* host_code);

/* Failure-path self-test: launches one warp whose bounded wait (the same wait
 * the pipelined kernels use on their mbarriers) can never be satisfied; after
 * limit_us (1 .. 1,000,000) it ORs the MOE_ERR_TIMEOUT bit into *err_flag and
 * returns.  Nothing faults, traps or hangs; the stream stays usable. */
MOE_API moe_status_t moe_selftest_wait_timeout(int32_t* err_flag, uint32_t limit_us, moe_stream_t stream);
MOE_API const char* moe_status_string(moe_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
