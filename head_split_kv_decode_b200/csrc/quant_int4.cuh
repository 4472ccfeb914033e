// Asymmetric 4-bit quantisation of one (token, KV head) row, K or V, by one
// warp.  Used by the append kernel and by the fused decode step, so that both
// write the same codes.
//
// Pages: "DuoAttention: Efficient Long-Context LLM Inference with Retrieval and
// Streaming Heads" (hotpaper.ai), section "기술적 접근법": the method combines
// with a 4-bit KV cache.  The pages give no scheme; this one is min/max per
// row of head_dim channels with fp16 scale and zero, every step a correctly
// rounded fp32 operation, in this order:
//   span = mx - mn; sc = fp16(span / 15); zp = fp16(mn);
//   u = clamp(rint((x - zp) / sc), 0, 15), u = 0 when sc == 0.
#pragma once

#include "common.cuh"

namespace duo {

// Lane l holds channels [l*CPL, l*CPL + CPL) of the row in x.  Returns this
// lane's codes packed low nibble first (channel l*CPL + j in nibble j) and
// the row's fp16 scale and zero (the same in every lane).
template <int CPL>
__device__ __forceinline__ uint32_t quantize_row_int4(const float (&x)[CPL], __half *sch_out,
                                                      __half *zph_out) {
  float mn = INFINITY, mx = -INFINITY;
#pragma unroll
  for (int j = 0; j < CPL; ++j) {
    mn = fminf(mn, x[j]);
    mx = fmaxf(mx, x[j]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const __half sch = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), 15.0f));
  const __half zph = __float2half_rn(mn);
  const float scf = __half2float(sch);
  const float zpf = __half2float(zph);
  uint32_t packed = 0;
#pragma unroll
  for (int j = 0; j < CPL; ++j) {
    float q = 0.0f;
    if (scf != 0.0f) q = fminf(15.0f, fmaxf(0.0f, rintf(__fdiv_rn(__fsub_rn(x[j], zpf), scf))));
    packed |= (uint32_t)q << (4 * j);
  }
  *sch_out = sch;
  *zph_out = zph;
  return packed;
}

}  // namespace duo
