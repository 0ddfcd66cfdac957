// The multiply-add step of the router logit ("[sglang] [NPU] GLM-4.7-Flash
// 성능 최적화", §2 "MoE TopK Scoring Function": z = x . w_router + bias before
// the sigmoid), shared by the router kernels and the single-launch layer so
// that both take every element of the canonical order with the same fma.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// fp32 fma with bf16 multiplicands: c + a*b rounded once, a and b taken
// exactly (a product of two bf16 values is exact in fp32), so the result is
// the same as fmaf(float(a), float(b), c) without the two conversions.
// kHi selects the high or the low bf16 half of each 32-bit word.
template <bool kHi>
__device__ __forceinline__ float fma_bf16(uint32_t aw, uint32_t bw, float c) {
  float d = c;
  if (kHi)
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, ah, bh, %0;\n\t}"
        : "+f"(d)
        : "r"(aw), "r"(bw));
  else
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, al, bl, %0;\n\t}"
        : "+f"(d)
        : "r"(aw), "r"(bw));
  return d;
}

__device__ __forceinline__ uint32_t word(const uint4& v, int w) {
  return w == 0 ? v.x : w == 1 ? v.y : w == 2 ? v.z : v.w;
}

}  // namespace moe
