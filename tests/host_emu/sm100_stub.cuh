// TEST INFRASTRUCTURE ONLY: host stand-ins for the device helpers the decode and forward
// kernels take from sm100.cuh and decode_ops.cuh.  The tests copy this file next to the kernel
// under the name sm100.cuh, with sm100_extracted.inc: the pure helpers (descriptor encoders,
// the FMA-pipe exponential) cut from the real sm100.cuh, so their encodings are not restated.
//
// tcgen05, TMA and mbarriers are emulated from their documented behaviour:
//   mbarrier    phases with an arrival count and a transaction-byte count; try_wait.parity(P)
//               succeeds once the phase of parity P has completed.
//   TMA         a 4-D tiled load of a 64-element x rows box, zero outside the tensor, written
//               with the 128-byte swizzle (16-byte chunk c of a 128-byte row r lands at chunk
//               c ^ (r % 8) of its 1024-byte atom), completing its bytes on the barrier.
//   TMEM        128 lanes x 512 32-bit columns; address = lane << 16 | column; a warp's
//               32x32b loads and stores reach only the lane quadrant 32 (warp % 4).
//   MMA         kind::f16 bf16 x bf16 -> fp32, M = 128, K = 16, N from the instruction
//               descriptor; operands read through SW128 shared-memory descriptors (K-major:
//               8-row atoms SBO apart; MN-major: 64 MN-contiguous elements per row, 8-k atoms
//               SBO apart, the next 64 MN elements LBO apart) or A from TMEM (bf16 pairs);
//               queued when issued and executed, in issue order, at the issuing thread's
//               next tcgen05.commit (a legal schedule: the hardware runs them asynchronously,
//               in order, and the commit's barrier tracks their completion).
// TMA and bulk copies likewise land only when some thread tests the barrier that tracks them,
// so a consumer that reads shared memory or TMEM without waiting on the right barrier sees
// stale (NaN-filled) data.  ldmatrix and mma.sync are emulated from the fragment layouts the PTX ISA
// documents (m8n8 b16 matrices; m16n8k16 row.col bf16 with fp32 accumulators); ex2 / lg2 are std::exp2 / std::log2;
// bf16 and f16 rounding is round-to-nearest-even (f16 with subnormals and overflow to
// infinity); E4M3 codes decode by the format's definition (they are all f16 values).
#pragma once
#include <atomic>
#include <deque>
#include <functional>
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
struct __nv_bfloat162 { uint16_t x, y; };
inline __nv_bfloat16 __float2bfloat16_rn(float f) { return __nv_bfloat16{f2bf(f)}; }
inline float2 __bfloat1622float2(__nv_bfloat162 h) { return {bf2f(h.x), bf2f(h.y)}; }
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
// programmatic dependent launch: the emulation runs grids one after another, so both are no-ops
inline void grid_dep_wait() {}
inline void grid_dep_launch_dependents() {}

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
// ------------------------------------------------------------ shared memory addresses
inline uint32_t smem_u32(const void* p) {
  const long long off = static_cast<const unsigned char*>(p) - g_blk->smem;
  if (off < 0 || size_t(off) >= g_blk->smem_bytes) { std::fprintf(stderr, "smem_u32 outside shared memory\n"); std::abort(); }
  return uint32_t(off);
}
inline unsigned char* smem_at(uint32_t a, size_t bytes) {
  if (size_t(a) + bytes > g_blk->smem_bytes) { std::fprintf(stderr, "shared access past the end: %u\n", a); std::abort(); }
  return g_blk->smem + a;
}
inline uint64_t global_timer_ns() {
  return uint64_t(std::chrono::duration_cast<std::chrono::nanoseconds>(
                      std::chrono::steady_clock::now().time_since_epoch()).count());
}
inline int g_status = 0;
constexpr int FA_DEVICE_TIMEOUT = 1;

// ------------------------------------------------------------ mbarriers
inline BarState& bar_state(uint32_t bar) {
  auto it = g_blk->bars->find(bar);
  if (it == g_blk->bars->end()) { std::fprintf(stderr, "mbarrier %u used before init\n", bar); std::abort(); }
  return it->second;
}
inline void bar_flip_if_done(BarState& b) {
  if (b.pending == 0 && b.tx == 0) {
    b.phase ^= 1u;
    b.pending = b.expected;
  }
}
inline void mbar_init(uint32_t bar, uint32_t count) {
  std::lock_guard<std::mutex> lk(*g_blk->mu);
  (*g_blk->bars)[bar] = BarState{count, count, 0, 0};
}
inline void fence_mbar_init() {}
inline void mbar_arrive(uint32_t bar) {
  std::lock_guard<std::mutex> lk(*g_blk->mu);
  BarState& b = bar_state(bar);
  if (b.pending == 0) { std::fprintf(stderr, "mbarrier %u: too many arrivals\n", bar); std::abort(); }
  b.pending -= 1;
  bar_flip_if_done(b);
}
inline void mbar_expect_tx(uint32_t bar, uint32_t bytes) {   // arrive.expect_tx
  std::lock_guard<std::mutex> lk(*g_blk->mu);
  BarState& b = bar_state(bar);
  if (b.pending == 0) { std::fprintf(stderr, "mbarrier %u: too many arrivals\n", bar); std::abort(); }
  b.tx += bytes;
  b.pending -= 1;
  bar_flip_if_done(b);
}
inline void bar_complete_tx(uint32_t bar, uint32_t bytes) {
  std::lock_guard<std::mutex> lk(*g_blk->mu);
  BarState& b = bar_state(bar);
  b.tx -= bytes;
  bar_flip_if_done(b);
}
inline void land_copies(uint32_t bar);
inline bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  land_copies(bar);
  std::lock_guard<std::mutex> lk(*g_blk->mu);
  return bar_state(bar).phase != (parity & 1u);
}
inline bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort, uint64_t limit_ns) {
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (global_timer_ns() - t0 > limit_ns) {
      *abort = 1;
      atomicOr(&g_status, FA_DEVICE_TIMEOUT);
      return false;
    }
    std::this_thread::yield();
  }
}
inline bool mbar_wait_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  int never = 0;
  return mbar_wait(bar, parity, &never, limit_ns);
}
// the inline forms the warpgroup-budget kernels use, and the budget moves (no effect on the host)
inline bool mbar_wait_inl(uint32_t bar, uint32_t parity, volatile int* abort, uint64_t limit_ns) {
  return mbar_wait(bar, parity, abort, limit_ns);
}
inline bool mbar_wait_drain_inl(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  return mbar_wait_drain(bar, parity, limit_ns);
}
template <uint32_t N>
inline void regs_lower() {}
template <uint32_t N>
inline void regs_raise() {}

// ------------------------------------------------------------ TMA
struct CUtensorMap {
  const unsigned char* base;
  uint64_t dims[4];      // x (contiguous), rows, heads, batch (elements)
  uint64_t strides[3];   // bytes: rows, heads, batch
  uint32_t box_x, box_rows;
  uint32_t esize = 2;      // bytes per element; box_x * esize is the 128-byte swizzle row
  uint32_t swizzle = 128;  // 128: the 128-byte swizzle; 0: plain rows of box_x * esize bytes
};
inline void tma_prefetch_desc(const CUtensorMap*) {}
inline uint32_t sw128(uint32_t addr) { return addr ^ (((addr >> 7) & 7u) << 4); }
// performs the copies issued so far that `bar` tracks (each completes its bytes on it)
inline void land_copies(uint32_t bar) {
  std::vector<std::function<void()>> todo;
  {
    std::lock_guard<std::mutex> lk(*g_blk->mu);
    auto& q = *g_blk->copies;
    for (auto it = q.begin(); it != q.end();) {
      if (it->bar == bar) {
        todo.push_back(std::move(it->run));
        it = q.erase(it);
      } else {
        ++it;
      }
    }
  }
  for (auto& f : todo) f();
}
// By default a copy lands only when its barrier is tested (late: a consumer that skips its wait
// reads stale data).  Built with EMU_EAGER_COPIES it lands at issue instead (early: a producer
// that skips its wait for the consumers' release overwrites data they still need).  Both are
// schedules the hardware may take.
inline void queue_copy(uint32_t bar, std::function<void()> f) {
#ifdef EMU_EAGER_COPIES
  f();
  return;
#endif
  std::lock_guard<std::mutex> lk(*g_blk->mu);
  g_blk->copies->push_back(PendingOp{bar, std::move(f)});
}
inline void tma_copy_now(uint32_t dst, CUtensorMap map, uint32_t bar, int x, int row, int head, int batch);
inline void tma_load_rows(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int row, int head, int batch) {
  if ((x * int(map->esize)) % 16) { std::fprintf(stderr, "TMA x coordinate not 16-byte aligned\n"); std::abort(); }
  const uint32_t row_bytes = map->box_x * map->esize;
  if (map->swizzle == 128 ? row_bytes != 128 : (map->swizzle != 0 || row_bytes % 16 != 0)) {
    std::fprintf(stderr, "TMA box row does not fit the swizzle mode\n");
    std::abort();
  }
  if (dst % (map->swizzle == 128 ? 1024u : 16u)) { std::fprintf(stderr, "TMA destination misaligned\n"); std::abort(); }
  smem_at(dst, size_t(map->box_rows) * row_bytes);   // the destination must lie in shared memory
  const CUtensorMap m = *map;
  BlockCtx* blk = g_blk;
  queue_copy(bar, [=] {
    BlockCtx* saved = g_blk;
    g_blk = blk;
    tma_copy_now(dst, m, bar, x, row, head, batch);
    g_blk = saved;
  });
}
inline void tma_copy_now(uint32_t dst, CUtensorMap mm, uint32_t bar, int x, int row, int head, int batch) {
  const CUtensorMap* map = &mm;
  for (uint32_t r = 0; r < map->box_rows; ++r)
    for (uint32_t c = 0; c < map->box_x; ++c) {
      const long long gx = (long long)x + c, gr = (long long)row + r;
      const uint32_t es = map->esize;
      uint16_t val = 0;
      if (gx >= 0 && gr >= 0 && head >= 0 && batch >= 0 && uint64_t(gx) < map->dims[0] &&
          uint64_t(gr) < map->dims[1] && uint64_t(head) < map->dims[2] && uint64_t(batch) < map->dims[3])
        std::memcpy(&val, map->base + uint64_t(batch) * map->strides[2] + uint64_t(head) * map->strides[1] +
                              uint64_t(gr) * map->strides[0] + uint64_t(gx) * es, es);
      const uint32_t at = dst + r * map->box_x * es + c * es;
      std::memcpy(smem_at(map->swizzle == 128 ? sw128(at) : at, es), &val, es);
    }
  bar_complete_tx(bar, map->box_x * map->box_rows * map->esize);
}

// cp.reduce.async.bulk.tensor .add (fp32): the reduction joins this thread's open bulk group;
// a group's reductions run (read the shared-memory box, add atomically into the tensor) only
// when a bulk wait retires the group -- late, so that a box rewritten before its wait shows up
// as wrong sums.  Reductions still in flight when the thread ends abort the run.
inline thread_local std::vector<std::function<void()>> t_bulk_open;
inline thread_local std::deque<std::vector<std::function<void()>>> t_bulk_groups;
inline void tma_reduce_add_rows(const CUtensorMap* map, uint32_t src, int x, int row, int head, int batch) {
  if (map->esize != 4) { std::fprintf(stderr, "TMA reduce: only fp32 tensors are emulated\n"); std::abort(); }
  if ((x * int(map->esize)) % 16) { std::fprintf(stderr, "TMA x coordinate not 16-byte aligned\n"); std::abort(); }
  if (map->box_x * map->esize != 128) { std::fprintf(stderr, "TMA box row is not 128 bytes\n"); std::abort(); }
  if (src % 128) { std::fprintf(stderr, "TMA reduce source not 128-byte aligned\n"); std::abort(); }
  smem_at(src, size_t(map->box_rows) * 128);
  const CUtensorMap m = *map;
  BlockCtx* blk = g_blk;
  t_bulk_open.push_back([=] {
    BlockCtx* saved = g_blk;
    g_blk = blk;
    for (uint32_t r = 0; r < m.box_rows; ++r)
      for (uint32_t c = 0; c < m.box_x; ++c) {
        const long long gx = (long long)x + c, gr = (long long)row + r;
        if (gx < 0 || gr < 0 || head < 0 || batch < 0 || uint64_t(gx) >= m.dims[0] || uint64_t(gr) >= m.dims[1] ||
            uint64_t(head) >= m.dims[2] || uint64_t(batch) >= m.dims[3])
          continue;   // outside the tensor: skipped
        float val;
        std::memcpy(&val, smem_at(sw128(src + r * 128 + c * 4), 4), 4);
        float* dst = reinterpret_cast<float*>(const_cast<unsigned char*>(m.base) + uint64_t(batch) * m.strides[2] +
                                              uint64_t(head) * m.strides[1] + uint64_t(gr) * m.strides[0] +
                                              uint64_t(gx) * 4);
        std::atomic_ref<float>(*dst).fetch_add(val);
      }
    g_blk = saved;
  });
}
// cp.async.bulk.tensor (shared -> global) tiled store: like the reduction above, it joins the
// thread's open bulk group and runs (reads the box, writes the rows inside the tensor) only when
// a bulk wait retires the group.
inline void tma_store_rows(const CUtensorMap* map, uint32_t src, int x, int row, int head, int batch) {
  if ((x * int(map->esize)) % 16) { std::fprintf(stderr, "TMA x coordinate not 16-byte aligned\n"); std::abort(); }
  if (map->box_x * map->esize != 128) { std::fprintf(stderr, "TMA box row is not 128 bytes\n"); std::abort(); }
  if (src % 128) { std::fprintf(stderr, "TMA store source not 128-byte aligned\n"); std::abort(); }
  if (x < 0 || row < 0 || head < 0 || batch < 0) { std::fprintf(stderr, "TMA store at a negative coordinate\n"); std::abort(); }
  smem_at(src, size_t(map->box_rows) * 128);
  const CUtensorMap m = *map;
  BlockCtx* blk = g_blk;
  t_bulk_open.push_back([=] {
    BlockCtx* saved = g_blk;
    g_blk = blk;
    for (uint32_t r = 0; r < m.box_rows; ++r)
      for (uint32_t c = 0; c < m.box_x; ++c) {
        const uint64_t gx = uint64_t(x) + c, gr = uint64_t(row) + r;
        if (gx >= m.dims[0] || gr >= m.dims[1] || uint64_t(head) >= m.dims[2] || uint64_t(batch) >= m.dims[3]) continue;
        std::memcpy(const_cast<unsigned char*>(m.base) + uint64_t(batch) * m.strides[2] + uint64_t(head) * m.strides[1] +
                        gr * m.strides[0] + gx * m.esize,
                    smem_at(sw128(src + r * 128 + c * m.esize), m.esize), m.esize);
      }
    g_blk = saved;
  });
}
inline void bulk_commit_group() {
  t_bulk_groups.push_back(std::move(t_bulk_open));
  t_bulk_open.clear();
}
template <int N>
inline void bulk_wait_group_read() {
  while (t_bulk_groups.size() > size_t(N)) {
    for (auto& f : t_bulk_groups.front()) f();
    t_bulk_groups.pop_front();
  }
}
template <int N>
inline void bulk_wait_group() {
  bulk_wait_group_read<N>();
}
inline void bulk_exit_check() {
  if (!t_bulk_open.empty() || !t_bulk_groups.empty()) {
    std::fprintf(stderr, "thread %u of CTA %u ends with bulk operations (tensor reductions or stores) in flight\n", threadIdx.x, blockIdx.x);
    std::abort();
  }
}

// ------------------------------------------------------------ tensor memory
inline uint32_t& tmem_cell(uint32_t lane, uint32_t col) {
  if (lane >= 128 || col >= 512) { std::fprintf(stderr, "TMEM access out of range (%u, %u)\n", lane, col); std::abort(); }
  return g_blk->tmem[lane * 512 + col];
}
inline void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  if (ncols < 32 || ncols > 512 || (ncols & (ncols - 1))) { std::fprintf(stderr, "bad TMEM allocation\n"); std::abort(); }
  if (lane_id() == 0) {
    const uint32_t base = 0;
    std::memcpy(smem_at(dst_smem, 4), &base, 4);
  }
  __syncwarp();
}
inline void tmem_relinquish() {}
inline void tmem_dealloc(uint32_t, uint32_t) {}
inline void tc_fence_before() {}
inline void tc_fence_after() {}
inline void fence_proxy_async_smem() {}
// the lane quadrant a warp may access: lanes 32 (warp % 4) .. + 31
inline uint32_t tmem_row(uint32_t taddr) {
  const uint32_t base = taddr >> 16, warp = threadIdx.x >> 5;
  if (base != 32u * (warp % 4u)) { std::fprintf(stderr, "TMEM lane base %u outside warp %u's quadrant\n", base, warp); std::abort(); }
  return base + uint32_t(lane_id());
}
template <int N>
inline void tmem_ld_n(uint32_t taddr, uint32_t* r) {
  const uint32_t row = tmem_row(taddr), col = taddr & 0xffffu;
  std::lock_guard<std::mutex> lk(*g_blk->mu);
  for (int i = 0; i < N; ++i) r[i] = tmem_cell(row, col + i);
}
template <int N>
inline void tmem_st_n(uint32_t taddr, const uint32_t* r) {
  const uint32_t row = tmem_row(taddr), col = taddr & 0xffffu;
  std::lock_guard<std::mutex> lk(*g_blk->mu);
  for (int i = 0; i < N; ++i) tmem_cell(row, col + i) = r[i];
}
inline void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) { tmem_ld_n<32>(taddr, r); }
inline void tmem_ld32_async(uint32_t taddr, uint32_t* r) { tmem_ld_n<32>(taddr, r); }
inline void tmem_ld_wait() {}
template <int N>
inline void reg_fence(uint32_t*) {}
inline void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) { tmem_st_n<32>(taddr, r); }
inline void tmem_st16(uint32_t taddr, const uint32_t* r) { tmem_st_n<16>(taddr, r); }
inline void tmem_st_wait() {}

// bf16 element (i along M or N, k along K) of a 128-byte-swizzled shared-memory operand
inline float sw128_operand(uint64_t desc, bool mn_major, uint32_t i, uint32_t k) {
  if ((desc >> 61) != 2u) { std::fprintf(stderr, "descriptor layout is not the 128-byte swizzle\n"); std::abort(); }
  const uint32_t start = uint32_t(desc & 0x3fffu) << 4, lbo = uint32_t((desc >> 16) & 0x3fffu) << 4,
                 sbo = uint32_t((desc >> 32) & 0x3fffu) << 4;
  const uint32_t addr = mn_major ? start + (i / 64) * lbo + (k / 8) * sbo + (k % 8) * 128 + (i % 64) * 2
                                 : start + (i / 8) * sbo + (i % 8) * 128 + k * 2;
  uint16_t h;
  std::memcpy(&h, smem_at(sw128(addr), 2), 2);
  return bf2f(h);
}
// D (+)= A B^T with A 128 x 16 (shared memory, or TMEM when a_tmem_addr != ~0u), B N x 16
inline void mma_exec(uint32_t d_tmem, uint64_t a_desc, uint32_t a_tmem_addr, uint64_t b_desc, uint32_t idesc,
                     uint32_t accumulate) {
  if (((idesc >> 4) & 3u) != 1u || ((idesc >> 7) & 7u) != 1u || ((idesc >> 10) & 7u) != 1u) {
    std::fprintf(stderr, "instruction descriptor is not bf16 x bf16 -> f32\n");
    std::abort();
  }
  const uint32_t M = ((idesc >> 24) & 0x1fu) << 4, N = ((idesc >> 17) & 0x3fu) << 3;
  const bool a_mn = (idesc >> 15) & 1u, b_mn = (idesc >> 16) & 1u;
  if (M != 128 || N < 8 || N > 256 || N % 16) { std::fprintf(stderr, "unsupported MMA shape\n"); std::abort(); }
  std::lock_guard<std::mutex> lk(*g_blk->mu);
  static thread_local std::vector<float> A, B;
  A.assign(128 * 16, 0.f);
  B.assign(N * 16, 0.f);
  for (uint32_t m = 0; m < 128; ++m)
    for (uint32_t k = 0; k < 16; ++k) {
      if (a_tmem_addr != ~0u) {
        const uint32_t w = tmem_cell((a_tmem_addr >> 16) + m, (a_tmem_addr & 0xffffu) + k / 2);
        A[m * 16 + k] = bf2f(uint16_t((k & 1) ? (w >> 16) : (w & 0xffffu)));
      } else {
        A[m * 16 + k] = sw128_operand(a_desc, a_mn, m, k);
      }
    }
  for (uint32_t n = 0; n < N; ++n)
    for (uint32_t k = 0; k < 16; ++k) B[n * 16 + k] = sw128_operand(b_desc, b_mn, n, k);
  const uint32_t lane0 = d_tmem >> 16, col0 = d_tmem & 0xffffu;
  for (uint32_t m = 0; m < 128; ++m)
    for (uint32_t n = 0; n < N; ++n) {
      uint32_t& cell = tmem_cell(lane0 + m, col0 + n);
      float acc = accumulate ? __uint_as_float(cell) : 0.f;
      for (uint32_t k = 0; k < 16; ++k) acc += A[m * 16 + k] * B[n * 16 + k];
      cell = __float_as_uint(acc);
    }
}
// By default an MMA runs at its issuing thread's next commit.  Built with EMU_EAGER_MMA it runs
// at issue instead, the other legal extreme: an MMA issued before its operands are ready (a P
// in TMEM, a tile in shared memory) then reads them too early.
inline void queue_mma(std::function<void()> f) {
#ifdef EMU_EAGER_MMA
  f();
  return;
#endif
  std::lock_guard<std::mutex> lk(*g_blk->mu);
  g_blk->mmas->push_back(PendingOp{0, std::move(f)});
}
// kind::f8f6f4 with E4M3 A and B (type code 0), fp32 D, M = 128, K = 32: byte elements of
// K-major 128-byte-swizzled shared-memory operands
inline float sw128_operand_u8(uint64_t desc, uint32_t i, uint32_t k) {
  if ((desc >> 61) != 2u) { std::fprintf(stderr, "descriptor layout is not the 128-byte swizzle\n"); std::abort(); }
  const uint32_t start = uint32_t(desc & 0x3fffu) << 4, sbo = uint32_t((desc >> 32) & 0x3fffu) << 4;
  const uint32_t addr = start + (i / 8) * sbo + (i % 8) * 128 + k;
  return e4m3_to_f(*smem_at(sw128(addr), 1));
}
inline void mma_f8_exec(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
  if (((idesc >> 4) & 3u) != 1u || ((idesc >> 7) & 7u) != 0u || ((idesc >> 10) & 7u) != 0u ||
      ((idesc >> 15) & 3u) != 0u) {
    std::fprintf(stderr, "instruction descriptor is not K-major E4M3 x E4M3 -> f32\n");
    std::abort();
  }
  const uint32_t M = ((idesc >> 24) & 0x1fu) << 4, N = ((idesc >> 17) & 0x3fu) << 3;
  if (M != 128 || N < 8 || N > 256 || N % 16) { std::fprintf(stderr, "unsupported MMA shape\n"); std::abort(); }
  std::lock_guard<std::mutex> lk(*g_blk->mu);
  std::vector<float> A(128 * 32), B(N * 32);
  for (uint32_t m = 0; m < 128; ++m)
    for (uint32_t k = 0; k < 32; ++k) A[m * 32 + k] = sw128_operand_u8(a_desc, m, k);
  for (uint32_t n = 0; n < N; ++n)
    for (uint32_t k = 0; k < 32; ++k) B[n * 32 + k] = sw128_operand_u8(b_desc, n, k);
  const uint32_t lane0 = d_tmem >> 16, col0 = d_tmem & 0xffffu;
  for (uint32_t m = 0; m < 128; ++m)
    for (uint32_t n = 0; n < N; ++n) {
      uint32_t& cell = tmem_cell(lane0 + m, col0 + n);
      float acc = accumulate ? __uint_as_float(cell) : 0.f;
      for (uint32_t k = 0; k < 32; ++k) acc += A[m * 32 + k] * B[n * 32 + k];
      cell = __float_as_uint(acc);
    }
}
inline void mma_bf16_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  queue_mma([=] { mma_exec(d, a, ~0u, b, idesc, acc); });
}
inline void mma_bf16_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  queue_mma([=] { mma_exec(d, 0, a, b, idesc, acc); });
}
// the MMAs issued so far complete, in order, then the barrier sees one arrival
inline void mma_commit(uint32_t bar) {
  std::vector<PendingOp> todo;
  {
    std::lock_guard<std::mutex> lk(*g_blk->mu);
    todo.swap(*g_blk->mmas);
  }
  for (auto& op : todo) op.run();
  mbar_arrive(bar);
}
// warp-uniform forms: one elected lane issues
inline void mma_bf16_ss_w(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  if (lane_id() == 0) mma_bf16_ss(d, a, b, idesc, acc);
}
inline void mma_bf16_ts_w(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  if (lane_id() == 0) mma_bf16_ts(d, a, b, idesc, acc);
}
inline void mma_commit_w(uint32_t bar) {
  if (lane_id() == 0) mma_commit(bar);
}
inline void mma_e4m3_ss_w(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  if (lane_id() == 0) queue_mma([=] { mma_f8_exec(d, a, b, idesc, acc); });
}
// two fp32 values as E4M3 codes (round to nearest even, saturating to +-448; lo in the low byte)
inline uint8_t f2e4m3(float f) {
  if (std::isnan(f)) return 0x7f;
  const uint8_t sign = std::signbit(f) ? 0x80 : 0;
  float a = std::fabs(f);
  if (a >= 448.f) return sign | 0x7e;
  // find the nearest representable magnitude by search over the 127 finite codes (exact and simple)
  uint8_t best = 0;
  float bd = INFINITY;
  for (int c = 0; c <= 0x7e; ++c) {
    const float v = e4m3_to_f(uint8_t(c));
    const float dd = std::fabs(v - a);
    if (dd < bd || (dd == bd && (c & 1) == 0 && (best & 1) == 1)) { bd = dd; best = uint8_t(c); }
  }
  return sign | best;
}
inline uint32_t f32x2_to_e4m3x2(float lo, float hi) { return uint32_t(f2e4m3(lo)) | (uint32_t(f2e4m3(hi)) << 8); }

// ------------------------------------------------------------ shared vectors, bulk copies, reductions
inline uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  std::memcpy(&v, smem_at(addr, 16), 16);
  return v;
}
inline void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  const uint4 v{a, b, c, d};
  std::memcpy(smem_at(addr, 16), &v, 16);
}
// the untiled bulk copy global -> shared, completing its bytes on the barrier
inline void emu_bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  if (dst % 16 || bytes % 16 || reinterpret_cast<uintptr_t>(src) % 16) {
    std::fprintf(stderr, "bulk copy not 16-byte aligned\n");
    std::abort();
  }
  smem_at(dst, bytes);
  queue_copy(bar, [=] {
    std::memcpy(smem_at(dst, bytes), src, bytes);
    bar_complete_tx(bar, bytes);
  });
}
// red.global.add.v4.f32: four fp32 adds done atomically at the target
inline void red_add_v4(float* addr, uint4 v) {
  if (reinterpret_cast<uintptr_t>(addr) % 16) { std::fprintf(stderr, "vector reduction not 16-byte aligned\n"); std::abort(); }
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  for (int i = 0; i < 4; ++i) std::atomic_ref<float>(addr[i]).fetch_add(__uint_as_float(w[i]));
}

// ------------------------------------------------------------ packed fp32 pairs, max
inline uint64_t f2(float lo, float hi) { return uint64_t(__float_as_uint(lo)) | (uint64_t(__float_as_uint(hi)) << 32); }
inline void f2_split(uint64_t v, float& lo, float& hi) {
  lo = __uint_as_float(uint32_t(v));
  hi = __uint_as_float(uint32_t(v >> 32));
}
inline uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  float a0, a1, b0, b1, c0, c1;
  f2_split(a, a0, a1);
  f2_split(b, b0, b1);
  f2_split(c, c0, c1);
  return f2(std::fma(a0, b0, c0), std::fma(a1, b1, c1));
}
inline uint64_t f2_mul(uint64_t a, uint64_t b) {
  float a0, a1, b0, b1;
  f2_split(a, a0, a1);
  f2_split(b, b0, b1);
  return f2(a0 * b0, a1 * b1);
}
inline uint64_t f2_add(uint64_t a, uint64_t b) {
  float a0, a1, b0, b1;
  f2_split(a, a0, a1);
  f2_split(b, b0, b1);
  return f2(a0 + b0, a1 + b1);
}
inline float max3f(float a, float b, float c) { return std::fmax(std::fmax(a, b), c); }

#include "sm100_extracted.inc"

}  // namespace fa

// emu.h's end-of-thread hook
inline void emu_thread_exit() { fa::bulk_exit_check(); }
