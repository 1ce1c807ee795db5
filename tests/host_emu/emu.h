// TEST INFRASTRUCTURE ONLY (tests/test_decode_emulated.py): a host emulation of the few CUDA
// built-ins the decode kernel uses, so that the kernel's own source can run on the CPU under
// AddressSanitizer.  Each CUDA thread is a std::thread; __syncthreads and __syncwarp are
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
#include <memory>
#include <thread>
#include <vector>

#define __global__
#define __device__
#define __host__
#define __forceinline__ inline
#define __launch_bounds__(...)
#define __restrict__
using std::max;
using std::min;

struct dim3s { unsigned x = 0, y = 0, z = 0; };
inline thread_local dim3s threadIdx, blockIdx;
struct float2 { float x, y; };
struct float4 { float x, y, z, w; };
struct uint2 { uint32_t x, y; };
struct uint4 { uint32_t x, y, z, w; };
inline float2 make_float2(float a, float b) { return {a, b}; }
struct __nv_bfloat16 { uint16_t x; };

struct WarpCtx {
  std::barrier<>* bar;
  uint32_t xch[32][12];
  const void* addr[32];
};
struct BlockCtx {
  std::barrier<>* bar;
  unsigned char* smem;
  std::vector<WarpCtx>* warps;
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

template <class F>
void emu_launch(unsigned grid, unsigned block, size_t smem_bytes, F call) {
  for (unsigned bx = 0; bx < grid; ++bx) {
    std::vector<unsigned char> smem(smem_bytes ? smem_bytes : 1, 0xFF);   // NaN-filled
    std::barrier<> bar(block);
    std::vector<WarpCtx> warps(block / 32);
    std::vector<std::unique_ptr<std::barrier<>>> wb;
    for (auto& w : warps) {
      wb.emplace_back(new std::barrier<>(32));
      w.bar = wb.back().get();
    }
    BlockCtx ctx{&bar, smem.data(), &warps};
    std::vector<std::thread> th;
    th.reserve(block);
    for (unsigned tx = 0; tx < block; ++tx)
      th.emplace_back([&, tx] {
        threadIdx.x = tx;
        blockIdx.x = bx;
        g_blk = &ctx;
        call();
      });
    for (auto& t : th) t.join();
  }
}
