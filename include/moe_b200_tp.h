/*
 * moe_b200_tp.h -- the tensor-parallel form of the routed-MoE layer: the
 * expert intermediate dimension I split over G GPUs of one NVLink/NVSwitch
 * node, and the finalize fused with the reduction across the GPUs and the
 * RMSNorm ("[flashinfer] Kimi K3를 위한 초고속 통신 최적화", flashinfer PR
 * #5701 analysis: intro -- the MoE finalize, the all-reduce and the RMSNorm
 * as one kernel; §2 -- the exchange protocol chosen by the token count M,
 * low-latency for M <= 24, bulk transfers above).
 *
 * Partitioning.  Rank r of G holds, for every expert e, rows
 * [r*I/G, (r+1)*I/G) of W_gate[e] and W_up[e] (its slice of h's columns) and
 * the same columns of W_down[e] (its slice of the down contraction).  Routing,
 * the plan and x are replicated: every rank computes them identically.  Rank r
 * computes y_r[t,k] = bf16(h_r[t,k] . W_down_r[e]^T), a partial down
 * projection, and then every rank obtains
 *   s[t]   = sum_{r=0..G-1} p_r[t]            (fp32, added in rank order)
 *   p_0[t] = x[t] + sum_k w[t,k] * y_0[t,k]    (the residual enters once, on rank 0)
 *   p_r[t] =        sum_k w[t,k] * y_r[t,k]    (r > 0; fp32, k in order)
 *   out[t] = bf16(s * rsqrt(mean_h(s^2) + eps) * gamma),  residual_out[t] = bf16(s)
 * With G = 1 this is exactly moe_finalize_rmsnorm (the same arithmetic, in
 * the same order), so moe_tp_layer at G = 1 returns moe_layer's bits.
 *
 * Exchange.  Each rank owns one "group buffer" of moe_tp_buffer_bytes()
 * bytes, which every other rank of the node maps (CUDA IPC: moe_tp_ipc_*).
 * The finalize kernel stores its fp32 partial rows straight into the peers'
 * buffers over NVLink (plain 16-byte peer stores, no multicast), then sets a
 * per-(source, token) flag there with a system-scope release; readers wait on
 * their own buffer's flags (system-scope acquire, bounded).
 *  - ONESHOT (M <= 24, or MOE_TP_PROTOCOL=oneshot): every rank sends its whole
 *    partial to every rank, and every rank reduces and normalises every token.
 *    One exchange round: the latency protocol.
 *  - TWOSHOT (M > 24): token t is owned by rank t % G.  Every rank sends its
 *    partial row of t to the owner only; the owner reduces, normalises and
 *    sends the finished bf16 row (and residual row) to every other rank.  Each
 *    rank moves (G-1)/G of the fp32 partials and (G-1)/G of the bf16 rows:
 *    the bandwidth protocol.
 * The call number lives in the group buffer (the kernel advances it), data
 * areas alternate by its parity and flags carry it, so buffers are reused
 * across calls without clearing and the calls can be replayed from a CUDA
 * graph.  Every rank must make the same calls, in the same order, with the
 * same M.  The finalize kernel is a cooperative launch (all CTAs resident),
 * pushes everything it sends before it waits for anything, and bounds every
 * wait (2 s); an expired wait sets MOE_ERR_TIMEOUT in err_flag, after which
 * the group is out of step and must be rebuilt (buffers zeroed on every rank).
 */
#ifndef MOE_B200_TP_H
#define MOE_B200_TP_H

#include "moe_b200.h"

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_TP_MAX_RANKS 8
#define MOE_TP_ONESHOT_MAX_TOKENS 24
#define MOE_TP_IPC_HANDLE_BYTES 72

/* One rank's view of the group.
 * bufs[r]: rank r's group buffer as mapped in this process (bufs[rank] is this
 * rank's own buffer, allocated by the caller with moe_tp_buffer_bytes() bytes,
 * 256-byte aligned, zeroed once before first use; the others come from
 * moe_tp_ipc_open).  With world == 1 the buffers are not used and may be null.
 * max_tokens and hidden are the sizes the buffers were made for; every call
 * needs M <= max_tokens and H == hidden. */
typedef struct {
  int32_t rank, world, max_tokens, hidden;
  void* bufs[MOE_TP_MAX_RANKS];
} moe_tp_group_t;

/* Bytes of one rank's group buffer (0 for an unsupported size: world outside
 * 1..MOE_TP_MAX_RANKS, max_tokens < 1, hidden not a multiple of 256 or above 8192). */
MOE_API size_t moe_tp_buffer_bytes(int32_t world, int32_t max_tokens, int32_t hidden);

/* The protocol a call with M tokens takes on `world` ranks: 0 = ONESHOT,
 * 1 = TWOSHOT (host only; MOE_TP_PROTOCOL=oneshot|twoshot overrides when the
 * buffer allows it). */
MOE_API int moe_tp_protocol(int32_t M, int32_t world, int32_t max_tokens);

/* The fused finalize: top-k weighted sum of this rank's partial expert rows,
 * reduction across the G ranks, residual add and RMSNorm, as defined above.
 * x: bf16 [M,H] (replicated); y_partial: bf16 [M,top_k,H], this rank's y_r;
 * topk_w: fp32 [M,top_k]; gamma: bf16 [H]; out, residual_out (nullable): bf16
 * [M,H], written on every rank (the same bits everywhere); residual_out must
 * be given on every rank or on none.  s.I is ignored.
 * err_flag (nullable): device int32, MOE_ERR_TIMEOUT if a wait expired.
 * UNSUPPORTED for M > g->max_tokens, H != g->hidden or world outside
 * 1..MOE_TP_MAX_RANKS; INVALID_ARG for a null or misaligned pointer or a
 * missing buffer (world > 1). */
MOE_API moe_status_t moe_tp_finalize_allreduce_rmsnorm(const moe_bf16_t* x, const moe_bf16_t* y_partial,
                                                       const float* topk_w, const moe_bf16_t* gamma, float eps,
                                                       moe_shape_t s, const moe_tp_group_t* g, moe_bf16_t* out,
                                                       moe_bf16_t* residual_out, int32_t* err_flag,
                                                       moe_stream_t stream);

/* The whole tensor-parallel layer on this rank: route -> align -> up (this
 * rank's slice) -> down (this rank's slice) -> the fused finalize above.
 * s.I is this rank's slice of the intermediate dimension (I / G; a multiple of
 * 128); w: MOE_W_BF16 weights of the slice, gate/up [E, I/G, H], down
 * [E, H, I/G] (MOE_W_NVFP4: UNSUPPORTED).  Other arguments as moe_layer;
 * ws: moe_tp_layer_workspace_size(s) bytes, 256-byte aligned, whose first
 * int32 is the call's device error word (cleared by each call).  At world == 1
 * the result is moe_layer's, bit for bit. */
MOE_API moe_status_t moe_tp_layer(const moe_bf16_t* x, const moe_bf16_t* w_router, const float* bias,
                                  const moe_weights_t* w, const moe_bf16_t* gamma, float eps, moe_shape_t s,
                                  const moe_tp_group_t* g, moe_bf16_t* out, moe_bf16_t* residual_out,
                                  int32_t* topk_ids_out, float* topk_w_out, void* ws, size_t ws_bytes,
                                  moe_stream_t stream);
MOE_API size_t moe_tp_layer_workspace_size(moe_shape_t s);

/* All G ranks of a group emulated on this one GPU: the same kernel and the
 * same exchange as G separate launches, run as ONE cooperative launch whose
 * CTAs play every rank (ranks that wait for one another must run at the same
 * time, which separate launches on one GPU do not guarantee).  bufs, y_partials,
 * outs and residual_outs are host arrays of `world` device pointers (one group
 * buffer of moe_tp_buffer_bytes(world, max_tokens, H) bytes per emulated rank,
 * all on this device; residual_outs nullable as a whole); x, topk_w, gamma as
 * above.  Used to check the exchange protocols on one GPU. */
MOE_API moe_status_t moe_tp_finalize_emulated(const moe_bf16_t* x, const moe_bf16_t* const* y_partials,
                                              const float* topk_w, const moe_bf16_t* gamma, float eps,
                                              moe_shape_t s, int32_t world, int32_t max_tokens, void* const* bufs,
                                              moe_bf16_t* const* outs, moe_bf16_t* const* residual_outs,
                                              int32_t* err_flag, moe_stream_t stream);

/* CUDA IPC plumbing for the group buffers (host calls, not on the hot path):
 * the handle of a buffer this process allocated (MOE_TP_IPC_HANDLE_BYTES bytes
 * into handle_out: the allocation's IPC handle and the buffer's offset inside
 * that allocation; exchange them with any host transport), the mapping of a
 * peer's buffer into this process (peer access enabled lazily; *buf_out points
 * at the buffer, not at its allocation's start), and its release. */
MOE_API moe_status_t moe_tp_ipc_handle(const void* buf, void* handle_out);
MOE_API moe_status_t moe_tp_ipc_open(const void* handle, void** buf_out);
MOE_API moe_status_t moe_tp_ipc_close(void* buf);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_TP_H */
