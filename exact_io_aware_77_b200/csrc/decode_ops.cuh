// Device primitives of the split-key decode kernel: 8x8 matrix loads from shared memory into
// warp MMA operand registers, and the m16n8k16 bf16 (or f16) warp MMA with fp32 accumulators.
// These are warp-level instructions: the decode kernel's rows are too few (16) for a tcgen05
// MMA tile, and its time goes to reading K and V from HBM.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

namespace fa {

// The kernel's dynamic shared memory.
__device__ __forceinline__ unsigned char* dec_dyn_smem() {
  extern __shared__ __align__(128) unsigned char dec_smem_raw[];
  return dec_smem_raw;
}

// Four 8x8 b16 matrices; lane l gives the address of row l % 8 of matrix l / 8, and receives
// in r[m] the pair (row l / 4, columns 2 (l % 4) and 2 (l % 4) + 1) of matrix m.
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void* row) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(row))
               : "memory");
}
// The same, transposed: r[m] holds (rows 2 (l % 4) and 2 (l % 4) + 1, column l / 4) of matrix m.
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], const void* row) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(row))
               : "memory");
}

// d += a b for a 16x16 bf16 A (row-major fragment), a 16x8 bf16 B (column fragment) and a
// 16x8 fp32 accumulator, over one warp.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The same MMA on f16 operands (the FP8 K/V path: e4m3 converts to f16 exactly).
__device__ __forceinline__ void mma_16816_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two fp32 values as f16x2 (round to nearest even; lo in the low half).
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Two E4M3 codes (lo in the low byte) as f16x2; the conversion is exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two_codes & 0xffffu), __NV_E4M3);
  return uint32_t(h.x) | (uint32_t(h.y) << 16);
}

// A bf16x2 word as f16x2, each value clamped to the finite f16 range first.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_sat(uint32_t w) {
  constexpr float kMax = 65504.f;
  const float lo = fminf(fmaxf(__uint_as_float(w << 16), -kMax), kMax);
  const float hi = fminf(fmaxf(__uint_as_float(w & 0xffff0000u), -kMax), kMax);
  return pack_f16x2(lo, hi);
}

__device__ __forceinline__ uint32_t ld_global_u32(const void* p) {
  return *reinterpret_cast<const uint32_t*>(p);
}

// Programmatic dependent launch.  A grid launched with programmatic stream serialization may be
// scheduled before the previous grid on its stream has finished: grid_dep_wait blocks until that
// grid has completed and its memory operations are visible to this one (at once when the grid was
// launched without the attribute).  grid_dep_launch_dependents lets the next grid be scheduled as
// soon as every CTA of this grid has issued it or exited.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

}  // namespace fa
