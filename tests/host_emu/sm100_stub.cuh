// TEST INFRASTRUCTURE ONLY: host stand-ins for the device helpers the decode kernel takes from
// sm100.cuh and decode_ops.cuh.  The test copies this file next to decode_kernel.cuh under the
// name sm100.cuh.  ldmatrix and mma.sync are emulated from the fragment layouts the PTX ISA
// documents (m8n8 b16 matrices; m16n8k16 row.col bf16 with fp32 accumulators); cp.async is a
// synchronous copy (zero-fill when the source size is 0); ex2 / lg2 are std::exp2 / std::log2;
// bf16 and f16 rounding is round-to-nearest-even (f16 with subnormals and overflow to
// infinity); E4M3 codes decode by the format's definition (they are all f16 values).
#pragma once
#include "emu.h"

namespace fa {
struct Strides {
  long long b, h, n;
  long long at(int b_, int h_, int n_) const { return (long long)b_ * b + (long long)h_ * h + (long long)n_ * n; }
};
inline float ex2_approx(float x) { return std::exp2(x); }
inline float lg2_approx(float x) { return std::log2(x); }
inline uint16_t f2bf(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if (std::isnan(f)) return 0x7fc0;
  u += 0x7fffu + ((u >> 16) & 1u);
  return uint16_t(u >> 16);
}
inline float bf2f(uint16_t h) {
  uint32_t u = uint32_t(h) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}
inline uint32_t pack_bf16x2(float lo, float hi) { return uint32_t(f2bf(lo)) | (uint32_t(f2bf(hi)) << 16); }
inline uint16_t f2h(float f) {
  uint32_t x;
  std::memcpy(&x, &f, 4);
  const uint32_t sign = (x >> 16) & 0x8000u, ax = x & 0x7fffffffu;
  if (ax >= 0x7f800000u) return uint16_t(sign | (ax > 0x7f800000u ? 0x7e00u : 0x7c00u));
  if (ax >= 0x477ff000u) return uint16_t(sign | 0x7c00u);   // >= 65520 rounds to infinity
  if (ax < 0x38800000u) {                                    // below 2^-14: subnormal
    float v;
    std::memcpy(&v, &ax, 4);
    return uint16_t(sign | uint32_t(std::nearbyint(v * 16777216.0f)));
  }
  const uint32_t m = ax & 0x7fffffu;
  uint32_t h = (((ax >> 23) - 112u) << 10) | (m >> 13);
  const uint32_t rem = m & 0x1fffu;
  if (rem > 0x1000u || (rem == 0x1000u && (h & 1u))) h += 1;
  return uint16_t(sign | h);
}
inline float h2f(uint16_t h) {
  const int e = (h >> 10) & 0x1f, m = h & 0x3ff;
  float v;
  if (e == 0) v = std::ldexp(float(m), -24);
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = std::ldexp(float(1024 + m), e - 25);
  return (h & 0x8000) ? -v : v;
}
inline float e4m3_to_f(uint8_t c) {
  const int e = (c >> 3) & 0xf, m = c & 7;
  float v;
  if (e == 0) v = std::ldexp(float(m), -9);
  else if (e == 15 && m == 7) v = NAN;
  else v = std::ldexp(float(8 + m), e - 10);
  return (c & 0x80) ? -v : v;
}
inline uint32_t pack_f16x2(float lo, float hi) { return uint32_t(f2h(lo)) | (uint32_t(f2h(hi)) << 16); }
inline uint32_t e4m3x2_to_f16x2(uint32_t two) {
  return uint32_t(f2h(e4m3_to_f(uint8_t(two & 0xff)))) | (uint32_t(f2h(e4m3_to_f(uint8_t((two >> 8) & 0xff)))) << 16);
}
inline uint32_t bf16x2_to_f16x2_sat(uint32_t w) {
  const float lo = std::fmin(std::fmax(bf2f(uint16_t(w & 0xffff)), -65504.f), 65504.f);
  const float hi = std::fmin(std::fmax(bf2f(uint16_t(w >> 16)), -65504.f), 65504.f);
  return pack_f16x2(lo, hi);
}
inline unsigned char* dec_dyn_smem() { return g_blk->smem; }
inline void cp_async_16(void* dst, const void* src, int n) {
  if (n == 16) std::memcpy(dst, src, 16);
  else if (n == 0) std::memset(dst, 0, 16);
  else { std::fprintf(stderr, "bad cp.async size %d\n", n); std::abort(); }
}
inline void cp_async_commit() {}
template <int N> inline void cp_async_wait() {}
inline uint32_t ld_global_u32(const void* p) {
  if (reinterpret_cast<uintptr_t>(p) % 4) { std::fprintf(stderr, "misaligned u32 load\n"); std::abort(); }
  uint32_t v;
  std::memcpy(&v, p, 4);
  return v;
}
inline void check_row_addr(const void* row) {
  if (reinterpret_cast<uintptr_t>(row) % 16) { std::fprintf(stderr, "ldmatrix row not 16-byte aligned\n"); std::abort(); }
}
inline void ldmatrix_x4(uint32_t (&r)[4], const void* row) {
  check_row_addr(row);
  WarpCtx& w = my_warp();
  int l = lane_id();
  w.addr[l] = row;
  w.bar->arrive_and_wait();
  for (int m = 0; m < 4; ++m) {
    const unsigned char* a = static_cast<const unsigned char*>(w.addr[m * 8 + l / 4]);
    std::memcpy(&r[m], a + 4 * (l % 4), 4);
  }
  w.bar->arrive_and_wait();
}
inline void ldmatrix_x4_trans(uint32_t (&r)[4], const void* row) {
  check_row_addr(row);
  WarpCtx& w = my_warp();
  int l = lane_id();
  w.addr[l] = row;
  w.bar->arrive_and_wait();
  for (int m = 0; m < 4; ++m) {
    const unsigned char* r0 = static_cast<const unsigned char*>(w.addr[m * 8 + 2 * (l % 4)]);
    const unsigned char* r1 = static_cast<const unsigned char*>(w.addr[m * 8 + 2 * (l % 4) + 1]);
    uint16_t lo, hi;
    std::memcpy(&lo, r0 + 2 * (l / 4), 2);
    std::memcpy(&hi, r1 + 2 * (l / 4), 2);
    r[m] = uint32_t(lo) | (uint32_t(hi) << 16);
  }
  w.bar->arrive_and_wait();
}
template <class Dec>
inline void mma_emu(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1, Dec dec) {
  WarpCtx& w = my_warp();
  int l = lane_id();
  for (int i = 0; i < 4; ++i) w.xch[l][i] = a[i];
  w.xch[l][4] = b0;
  w.xch[l][5] = b1;
  for (int i = 0; i < 4; ++i) std::memcpy(&w.xch[l][6 + i], &d[i], 4);
  w.bar->arrive_and_wait();
  float A[16][16], B[16][8], C[16][8];
  for (int L = 0; L < 32; ++L) {
    const int g = L >> 2, t = L & 3;
    const uint32_t* x = w.xch[L];
    auto lo = [&](uint32_t v) { return dec(uint16_t(v & 0xffff)); };
    auto hi = [&](uint32_t v) { return dec(uint16_t(v >> 16)); };
    A[g][2 * t] = lo(x[0]); A[g][2 * t + 1] = hi(x[0]);
    A[g + 8][2 * t] = lo(x[1]); A[g + 8][2 * t + 1] = hi(x[1]);
    A[g][2 * t + 8] = lo(x[2]); A[g][2 * t + 9] = hi(x[2]);
    A[g + 8][2 * t + 8] = lo(x[3]); A[g + 8][2 * t + 9] = hi(x[3]);
    B[2 * t][g] = lo(x[4]); B[2 * t + 1][g] = hi(x[4]);
    B[2 * t + 8][g] = lo(x[5]); B[2 * t + 9][g] = hi(x[5]);
    float c[4];
    std::memcpy(c, &x[6], 16);
    C[g][2 * t] = c[0]; C[g][2 * t + 1] = c[1];
    C[g + 8][2 * t] = c[2]; C[g + 8][2 * t + 1] = c[3];
  }
  const int g = l >> 2, t = l & 3;
  const int rr[4] = {g, g, g + 8, g + 8}, cc[4] = {2 * t, 2 * t + 1, 2 * t, 2 * t + 1};
  for (int i = 0; i < 4; ++i) {
    float s = C[rr[i]][cc[i]];
    for (int k = 0; k < 16; ++k) s += A[rr[i]][k] * B[k][cc[i]];
    d[i] = s;
  }
  w.bar->arrive_and_wait();
}
inline void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  mma_emu(d, a, b0, b1, [](uint16_t h) { return bf2f(h); });
}
inline void mma_16816_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  mma_emu(d, a, b0, b1, [](uint16_t h) { return h2f(h); });
}
}  // namespace fa
