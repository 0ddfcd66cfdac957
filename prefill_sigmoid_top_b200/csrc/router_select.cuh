// The per-token top-k and sigmoid weights of the router ("[sglang] [NPU] GLM-4.7-Flash 성능 최적화", §2:
// sigmoid scores, renormalised over the selected experts), shared by the router's top-k kernel and the
// screened router, so that both give the same ids and the same weight bits from the same logits.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// (value, id) ordering of the selection: larger value first, then lower id.
__device__ __forceinline__ bool better(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// A NaN logit enters the selection (and its score) as -inf: it ranks below
// every other logit, so a selected id always lies in [0, E).
__device__ __forceinline__ float selection_key(float z) { return isnan(z) ? -INFINITY : z; }

// One warp, one token: expert lane + 32 i is held by lane `lane` (i < kPerLane); logit(e) gives its
// logit.  K rounds of a warp argmax pick the K largest (descending, equal ones: lower id); lane k < K
// then writes ids[k] and w[k] = s_k / sum_j s_j with s = 1 / (1 + exp(-z)).
template <int kPerLane, class Logit>
__device__ __forceinline__ void topk_sigmoid_token(Logit logit, int E, int K, int lane, int32_t* ids, float* w) {
  float v[kPerLane];
  bool live[kPerLane];
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    const int e = lane + 32 * i;
    live[i] = e < E;
    v[i] = live[i] ? selection_key(logit(e)) : -INFINITY;
  }
  float sel_v = 0.0f;
  int sel_id = 0;
  for (int k = 0; k < K; ++k) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i)
      if (live[i] && better(v[i], lane + 32 * i, bv, bi)) {
        bv = v[i];
        bi = lane + 32 * i;
      }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (better(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
    }
#pragma unroll
    for (int i = 0; i < kPerLane; ++i)  // the owner retires the winner
      if (lane + 32 * i == bi) live[i] = false;
    if (lane == k) {
      sel_v = bv;
      sel_id = bi;
    }
  }
  const float s = (lane < K) ? 1.0f / (1.0f + expf(-sel_v)) : 0.0f;
  float total = s;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) total += __shfl_xor_sync(0xffffffffu, total, off);
  if (lane < K) {
    ids[lane] = sel_id;
    w[lane] = s / total;
  }
}

}  // namespace moe
