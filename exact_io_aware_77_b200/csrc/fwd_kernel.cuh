// Forward pass of exact attention, fused in one kernel:
//   O = softmax(scale * Q K^T + mask) V  and  L = row logsumexp (natural log).
//
// The method is the IO-aware one of the FlashAttention pages: Q, K and V are cut
// into tiles that fit on chip and streamed through (FlashAttention (NL), "Tiling en
// blokgewijze verwerking"), the softmax is computed online from a running row maximum
// and a running sum of exponentials (same page, "Online berekening van Softmax"), and
// QK^T, masking, softmax and the product with V run in one kernel that writes only the
// final result (same page, "Samensmelting van bewerkingen in een CUDA-kernel").  The
// N x N score matrix never leaves the SM.
//
// sm_100a mapping (one CTA per 128-row query tile of one head):
//   warp 4      TMA producer: Q tile once, then K_j / V_j tiles into 2-stage rings.
//   warp 5      MMA issuer:   S_j = Q K_j^T into TMEM (double-buffered), O += P_j V_j in TMEM.
//   warps 0-3   softmax:      thread t owns query row t = TMEM lane t; reads S_j with
//                              tcgen05.ld, applies scale/mask, updates the running max m and
//                              sum l, writes P_j (bf16) to shared memory, rescales O in TMEM
//                              when m grows, and finally writes O / l and L.
// TMEM columns: [0,128) S buffer 0, [128,256) S buffer 1, [256, 256 + D) O accumulator.
#pragma once

#include "sm100.cuh"

namespace fa {

constexpr int kBlockM = 128;   // query rows per CTA
constexpr int kBlockN = 128;   // keys per KV tile
constexpr int kStages = 2;     // K/V shared-memory ring depth
constexpr int kFwdThreads = 192;
constexpr int kWarpTma = 4;
constexpr int kWarpMma = 5;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 256;

struct FwdParams {
  __nv_bfloat16* o;   // [BH, N, D]
  float* lse;         // [BH, N]
  int N;
  int BH;
  int n_q_tiles;
  int causal;
  int window;
  float scale_log2;   // scale * log2(e)
  unsigned long long wait_limit_ns;
};

template <int D>
struct FwdSmem {
  static constexpr int kChunks = D / 64;                 // 64-element (128-byte) column chunks
  static constexpr uint32_t kTileBytes = kBlockN * D * 2;  // one Q, K or V tile
  alignas(1024) uint8_t q[kBlockM * D * 2];
  alignas(1024) uint8_t k[kStages][kTileBytes];
  alignas(1024) uint8_t v[kStages][kTileBytes];
  alignas(1024) uint8_t p[kBlockM * kBlockN * 2];
  alignas(8) uint64_t q_full;
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full, o_done, mma_drain;
  uint32_t tmem_base;
  int abort;
};

// Range of KV tiles a query tile needs: causal stops at the diagonal, a window starts at
// the first tile that holds key q0 - W + 1.
__device__ __forceinline__ void kv_tile_range(int q0, int N, int causal, int window, int& t_begin, int& t_end) {
  const int kv_end = causal ? min(N, q0 + kBlockM) : N;
  t_end = (kv_end + kBlockN - 1) / kBlockN;
  const int kv_begin = window > 0 ? max(0, q0 - window + 1) : 0;
  t_begin = kv_begin / kBlockN;
}

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const FwdParams prm) {
  using Smem = FwdSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q_tile = prm.n_q_tiles - 1 - int(blockIdx.x / prm.BH);   // longest causal tiles first
  const int bh = int(blockIdx.x % prm.BH);
  const int q0 = q_tile * kBlockM;
  int t_begin, t_end;
  kv_tile_range(q0, prm.N, prm.causal, prm.window, t_begin, t_end);
  const int n_tiles = t_end - t_begin;   // >= 1: the diagonal tile is always needed
  volatile int* abort = &sm.abort;
  const uint64_t lim = prm.wait_limit_ns;

  if (threadIdx.x == 0) {
    sm.abort = 0;
    mbar_init(smem_u32(&sm.q_full), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&sm.k_full[s]), 1);
      mbar_init(smem_u32(&sm.k_empty[s]), 1);
      mbar_init(smem_u32(&sm.v_full[s]), 1);
      mbar_init(smem_u32(&sm.v_empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&sm.s_full[b]), 1);
      mbar_init(smem_u32(&sm.s_empty[b]), kBlockM);
    }
    mbar_init(smem_u32(&sm.p_full), kBlockM);
    mbar_init(smem_u32(&sm.o_done), 1);
    mbar_init(smem_u32(&sm.mma_drain), 1);
    fence_mbar_init();
  }
  if (warp == kWarpTma && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == kWarpTma) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint32_t qb = smem_u32(&sm.q_full);
      int k_issued = 0, v_issued = 0;
      mbar_expect_tx(qb, Smem::kTileBytes);
      for (int c = 0; c < Smem::kChunks; ++c)
        tma_load_3d(smem_u32(sm.q) + c * 16384, &tm_q, qb, c * 64, q0, bh);
      for (int t = 0; t < n_tiles; ++t) {
        const int s = t & 1;
        const uint32_t ph = (t >> 1) & 1;
        const int kv0 = (t_begin + t) * kBlockN;
        if (!mbar_wait(smem_u32(&sm.k_empty[s]), ph ^ 1, abort, lim)) break;
        const uint32_t kb = smem_u32(&sm.k_full[s]);
        mbar_expect_tx(kb, Smem::kTileBytes);
        for (int c = 0; c < Smem::kChunks; ++c)
          tma_load_3d(smem_u32(sm.k[s]) + c * 16384, &tm_k, kb, c * 64, kv0, bh);
        k_issued = t + 1;
        if (!mbar_wait(smem_u32(&sm.v_empty[s]), ph ^ 1, abort, lim)) break;
        const uint32_t vb = smem_u32(&sm.v_full[s]);
        mbar_expect_tx(vb, Smem::kTileBytes);
        for (int c = 0; c < Smem::kChunks; ++c)
          tma_load_3d(smem_u32(sm.v[s]) + c * 16384, &tm_v, vb, c * 64, kv0, bh);
        v_issued = t + 1;
      }
      // Let every copy this CTA started land before the CTA can exit (matters only when
      // aborting; on the normal path each one has been consumed already).
      mbar_wait_drain(qb, 0, lim);
      for (int t = max(0, k_issued - kStages); t < k_issued; ++t)
        mbar_wait_drain(smem_u32(&sm.k_full[t & 1]), (t >> 1) & 1, lim);
      for (int t = max(0, v_issued - kStages); t < v_issued; ++t)
        mbar_wait_drain(smem_u32(&sm.v_full[t & 1]), (t >> 1) & 1, lim);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kBlockM, kBlockN, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(kBlockM, D, false, true);
      const uint32_t q_addr = smem_u32(sm.q);
      const uint32_t p_addr = smem_u32(sm.p);
      bool ok = mbar_wait(smem_u32(&sm.q_full), 0, abort, lim);
      for (int t = 0; ok && t <= n_tiles; ++t) {
        if (t < n_tiles) {
          const int s = t & 1;
          const uint32_t ph = (t >> 1) & 1;
          if (!mbar_wait(smem_u32(&sm.k_full[s]), ph, abort, lim)) break;
          if (!mbar_wait(smem_u32(&sm.s_empty[s]), ph ^ 1, abort, lim)) break;
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sm.k[s]);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            // K-major operands: 16-element k-steps are 32 bytes apart inside a 128-byte row,
            // 64-element chunks are separate 16 KB tiles.
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_bf16_ss(tmem + s * kBlockN, sw128_desc(q_addr + off, 16, 1024), sw128_desc(k_addr + off, 16, 1024),
                        idesc_s, kk > 0);
          }
          mma_commit(smem_u32(&sm.s_full[s]));
          mma_commit(smem_u32(&sm.k_empty[s]));
        }
        if (t > 0) {
          const int u = t - 1;
          const int su = u & 1;
          if (!mbar_wait(smem_u32(&sm.p_full), u & 1, abort, lim)) break;
          if (!mbar_wait(smem_u32(&sm.v_full[su]), (u >> 1) & 1, abort, lim)) break;
          tc_fence_after();
          const uint32_t v_addr = smem_u32(sm.v[su]);
#pragma unroll
          for (int kk = 0; kk < kBlockN / 16; ++kk) {
            // A = P (K-major, like Q); B = V is MN-major: 16 keys = 16 rows of 128 bytes,
            // the next 64 head-dim columns sit one 16 KB chunk (LBO) further.
            const uint32_t a_off = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_bf16_ss(tmem + kTmemO, sw128_desc(p_addr + a_off, 16, 1024),
                        sw128_desc(v_addr + kk * 2048, 16384, 1024), idesc_o, (u > 0 || kk > 0));
          }
          mma_commit(smem_u32(&sm.o_done));
          mma_commit(smem_u32(&sm.v_empty[su]));
        }
      }
      // every MMA issued above completes before TMEM is released
      mma_commit(smem_u32(&sm.mma_drain));
      mbar_wait_drain(smem_u32(&sm.mma_drain), 0, lim);
    }
  } else {
    // ------------------------------------------------------------------ softmax warps 0-3
    const int row = threadIdx.x;                 // 0..127 == TMEM lane
    const int qi = q0 + row;
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const float c = prm.scale_log2;
    float m = -INFINITY;                         // running max of scaled scores (log2 units)
    float l = 0.f;                               // running sum of exponentials
    const uint32_t p_row = smem_u32(sm.p) + row * 128;
    const uint32_t sw = row & 7;
    bool ok = true;
    for (int t = 0; t < n_tiles; ++t) {
      const int s = t & 1;
      const int kv0 = (t_begin + t) * kBlockN;
      // the vote keeps every lane of the warp on the same path into the .sync.aligned TMEM ops
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.s_full[s]), (t >> 1) & 1, abort, lim))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[kBlockN];
#pragma unroll
      for (int ch = 0; ch < kBlockN / 32; ++ch) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + s * kBlockN + ch * 32, r);
#pragma unroll
        for (int j = 0; j < 32; ++j) sv[ch * 32 + j] = __uint_as_float(r[j]);
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&sm.s_empty[s]));

      const bool need_mask = (kv0 + kBlockN > prm.N) || (prm.causal && kv0 + kBlockN - 1 > q0) ||
                             (prm.window > 0 && kv0 < q0 + kBlockM - prm.window);
      if (need_mask) {
        const int hi = prm.causal ? min(qi, prm.N - 1) : prm.N - 1;       // last allowed key
        const int lo = prm.window > 0 ? qi - prm.window + 1 : 0;           // first allowed key
#pragma unroll
        for (int j = 0; j < kBlockN; ++j) {
          const int key = kv0 + j;
          if (key > hi || key < lo) sv[j] = -INFINITY;
        }
      }
      float mx = sv[0];
#pragma unroll
      for (int j = 1; j < kBlockN; ++j) mx = fmaxf(mx, sv[j]);
      const float m_new = fmaxf(m, mx * c);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;   // a row with no key yet stays at 0
      const float alpha = ex2_approx(m - m_use);
      float sum = 0.f;
      uint32_t pk[kBlockN / 2];
#pragma unroll
      for (int j = 0; j < kBlockN; j += 2) {
        const float p0 = ex2_approx(fmaf(sv[j], c, -m_use));
        const float p1 = ex2_approx(fmaf(sv[j + 1], c, -m_use));
        sum += p0 + p1;
        pk[j / 2] = pack_bf16x2(p0, p1);
      }
      l = l * alpha + sum;
      m = m_new;

      if (t > 0) {
        // PV of the previous tile must be complete: it read the P buffer, and O is rescaled now.
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.o_done), (t - 1) & 1, abort, lim))) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      // P row -> shared memory, 128B-swizzled K-major layout (two 64-key chunks of 16 KB)
#pragma unroll
      for (int c16 = 0; c16 < kBlockN / 8; ++c16) {
        const uint32_t addr = p_row + (c16 >> 3) * 16384 + (((c16 & 7) ^ sw) << 4);
        st_shared_v4(addr, pk[c16 * 4 + 0], pk[c16 * 4 + 1], pk[c16 * 4 + 2], pk[c16 * 4 + 3]);
      }
      if (t > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t r[32];
          const uint32_t ta = tmem + lane_base + kTmemO + ch * 32;
          tmem_ld32(ta, r);
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * alpha);
          tmem_st32(ta, r);
        }
        tmem_st_wait();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(smem_u32(&sm.p_full));
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.o_done), (n_tiles - 1) & 1, abort, lim))) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool in_range = qi < prm.N;
      __nv_bfloat16* orow = prm.o + (size_t(bh) * prm.N + (in_range ? qi : 0)) * D;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + kTmemO + ch * 32, r);
        uint32_t w[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          w[j] = pack_bf16x2(__uint_as_float(r[2 * j]) * inv_l, __uint_as_float(r[2 * j + 1]) * inv_l);
        if (in_range) {
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
          for (int j = 0; j < 4; ++j) dst[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
        }
      }
      if (in_range) prm.lse[size_t(bh) * prm.N + qi] = (m + lg2_approx(l)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace fa
