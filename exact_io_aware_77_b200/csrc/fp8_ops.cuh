// Device primitives of the FP8 (E4M3) forward: the kind::f8f6f4 tensor-core MMA and the fp32 ->
// E4M3 conversion.
#pragma once

#include <cstdint>
#include <cuda_fp8.h>

namespace fa {

// D[tmem] (+)= A[smem] * B[smem]^T with E4M3 A and B (K-major, 32 elements per k-step) and fp32
// D; warp-uniform: one elected lane issues.
__device__ __forceinline__ void mma_e4m3_ss_w(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Two fp32 values as E4M3 codes (round to nearest even, saturating to the largest finite
// value); lo in the low byte.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  return uint32_t(__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

}  // namespace fa
