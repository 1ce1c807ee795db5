// TEST INFRASTRUCTURE ONLY (tests/test_decode_emulated.py, tests/test_fwd_emulated.py): a
// host emulation of the CUDA built-ins the decode and forward kernels use, so that their own
// source can run on the CPU under AddressSanitizer.  Each CUDA thread is a std::thread; __syncthreads and __syncwarp are
// barriers; warp shuffles exchange through a per-warp buffer.  CTAs run one after another.
// Shared memory starts as 0xFF bytes (bf16 NaN), so a read of a byte nothing wrote shows up
// in the results.  Nothing in the library uses this.
#pragma once
#include <algorithm>
#include <barrier>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <chrono>
#include <functional>
#include <memory>
#include <mutex>
#include <thread>
#include <unordered_map>
#include <vector>

#define __global__
#define __device__
#define __host__
#define __forceinline__ inline
#define __launch_bounds__(...)
#define __restrict__
#define __noinline__
#define __grid_constant__
#define __shared__
#define __align__(x) __attribute__((aligned(x)))
using std::max;
using std::min;

struct dim3s { unsigned x = 0, y = 0, z = 0; };
inline thread_local dim3s threadIdx, blockIdx;
inline dim3s gridDim, blockDim;   // set by emu_launch for the whole grid
struct float2 { float x, y; };
struct float4 { float x, y, z, w; };
inline float4 make_float4(float a, float b, float c, float d) { return {a, b, c, d}; }
struct uint2 { uint32_t x, y; };
struct uint4 { uint32_t x, y, z, w; };
inline float2 make_float2(float a, float b) { return {a, b}; }
inline uint4 make_uint4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) { return {a, b, c, d}; }
inline float __uint_as_float(uint32_t u) {
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}
inline uint32_t __float_as_uint(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  return u;
}
inline int atomicOr(int* p, int v) { return __atomic_fetch_or(p, v, __ATOMIC_SEQ_CST); }
struct __nv_bfloat16 { uint16_t x; };

struct WarpCtx {
  std::barrier<>* bar;
  uint32_t xch[32][12];
  const void* addr[32];
};
// mbarrier state, kept beside shared memory (keyed by the barrier's shared-memory offset)
struct BarState {
  uint32_t expected = 0, pending = 0, phase = 0;
  long long tx = 0;
};
// an asynchronous operation (TMA or bulk copy, MMA) not yet performed
struct PendingOp {
  uint32_t bar;                    // copies: the barrier that tracks them
  std::function<void()> run;
};
struct BlockCtx {
  std::barrier<>* bar;
  unsigned char* smem;
  std::vector<WarpCtx>* warps;
  size_t smem_bytes;
  std::mutex* mu;                                    // guards bars
  std::unordered_map<uint32_t, BarState>* bars;
  uint32_t* tmem;                                    // 128 lanes x 512 columns
  std::vector<PendingOp>* copies;                    // TMA / bulk copies issued, not yet landed
  std::vector<PendingOp>* mmas;                      // MMAs issued, not yet executed (in order)
};
inline thread_local BlockCtx* g_blk = nullptr;
inline int lane_id() { return threadIdx.x & 31; }
inline WarpCtx& my_warp() { return (*g_blk->warps)[threadIdx.x >> 5]; }
inline void __syncthreads() { g_blk->bar->arrive_and_wait(); }
inline void __syncwarp(unsigned = 0xffffffffu) { my_warp().bar->arrive_and_wait(); }
inline float __shfl_xor_sync(unsigned, float v, int m) {
  WarpCtx& w = my_warp();
  int l = lane_id();
  std::memcpy(&w.xch[l][0], &v, 4);
  w.bar->arrive_and_wait();
  float r;
  std::memcpy(&r, &w.xch[l ^ m][0], 4);
  w.bar->arrive_and_wait();
  return r;
}

// width-limited xor shuffle: the partner is lane ^ m inside the lane's segment of `width`
inline float __shfl_xor_sync(unsigned mask, float v, int m, int width) {
  if (m >= width) { std::fprintf(stderr, "shuffle mask leaves its segment\n"); std::abort(); }
  return __shfl_xor_sync(mask, v, m);
}
inline int __all_sync(unsigned, int pred) {
  WarpCtx& w = my_warp();
  int l = lane_id();
  w.xch[l][0] = pred ? 1u : 0u;
  w.bar->arrive_and_wait();
  int all = 1;
  for (int i = 0; i < 32; ++i) all &= int(w.xch[i][0]);
  w.bar->arrive_and_wait();
  return all;
}
inline int __any_sync(unsigned, int pred) {
  WarpCtx& w = my_warp();
  int l = lane_id();
  w.xch[l][0] = pred ? 1u : 0u;
  w.bar->arrive_and_wait();
  int any = 0;
  for (int i = 0; i < 32; ++i) any |= int(w.xch[i][0]);
  w.bar->arrive_and_wait();
  return any;
}
inline float __shfl_sync(unsigned, float v, int src) {
  WarpCtx& w = my_warp();
  int l = lane_id();
  std::memcpy(&w.xch[l][0], &v, 4);
  w.bar->arrive_and_wait();
  float r;
  std::memcpy(&r, &w.xch[src & 31][0], 4);
  w.bar->arrive_and_wait();
  return r;
}

// checks the stub makes on every emulated thread as it ends (bulk operations it left in flight)
inline void emu_thread_exit();

// Runs the grid one CTA after another.  `external_smem` (for kernels that declare their own
// extern shared array) is refilled with 0xFF before every CTA; otherwise each CTA gets a fresh
// buffer of exactly smem_bytes.
template <class F>
void emu_launch(unsigned grid, unsigned block, size_t smem_bytes, F call, unsigned char* external_smem = nullptr) {
  gridDim = dim3s{grid, 1, 1};
  blockDim = dim3s{block, 1, 1};
  for (unsigned bx = 0; bx < grid; ++bx) {
    std::vector<unsigned char> own(external_smem ? 1 : (smem_bytes ? smem_bytes : 1), 0xFF);   // NaN-filled
    unsigned char* smem = external_smem ? external_smem : own.data();
    if (external_smem) std::memset(external_smem, 0xFF, smem_bytes);
    std::mutex mu;
    std::unordered_map<uint32_t, BarState> bars;
    std::vector<uint32_t> tmem(128 * 512, 0x7fc07fc0u);
    std::vector<PendingOp> copies, mmas;
    std::barrier<> bar(block);
    std::vector<WarpCtx> warps(block / 32);
    std::vector<std::unique_ptr<std::barrier<>>> wb;
    for (auto& w : warps) {
      wb.emplace_back(new std::barrier<>(32));
      w.bar = wb.back().get();
    }
    BlockCtx ctx{&bar, smem, &warps, smem_bytes, &mu, &bars, tmem.data(), &copies, &mmas};
    std::vector<std::thread> th;
    th.reserve(block);
    for (unsigned tx = 0; tx < block; ++tx)
      th.emplace_back([&, tx] {
        threadIdx.x = tx;
        blockIdx.x = bx;
        g_blk = &ctx;
        call();
        emu_thread_exit();
      });
    for (auto& t : th) t.join();
  }
}
