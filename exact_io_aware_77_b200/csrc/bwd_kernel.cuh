// Backward pass of exact attention with recomputation.
//
// The pages say only that intermediates are recomputed when needed instead of being
// stored (memory-optimized flash attention page, "How it works"); the forward keeps just
// O and the row logsumexp L, so the backward rebuilds P tile by tile from L:
//   P = exp(scale * Q K^T - L),  dV = P^T dO,  dP = dO V^T,
//   D_i = rowsum(dO_i o O_i)  (= sum_j P_ij dP_ij),  dS = P o (dP - D),
//   dQ = scale * dS K,  dK = scale * dS^T Q.
// No N x N buffer ever reaches device memory.
//
// Three kernels on one stream:
//   fa_bwd_prep      D (fp32), L in log2 units (padded rows get +inf so their P is 0),
//                    and a zeroed fp32 dQ accumulator.
//   fa_bwd_kernel    one CTA per 128-key tile of one head; loops over 64-row query tiles.
//   fa_bwd_dq_final  dQ = scale * accumulator, rounded to bf16.
//
// fa_bwd_kernel roles (320 threads):
//   warp 8      TMA producer: K_j, V_j once; Q_i, dO_i (+ their L and D rows) into a 3-stage ring.
//   warp 9      MMA issuer:   S^T = K Q_i^T and dP^T = V dO_i^T (N = 64), then
//                              dV += P^T dO_i and dK += dS^T Q_i with A read from TMEM,
//                              and dQ_i^T = K^T dS^T (A, B from shared memory).
//   warps 0-3   thread t owns key kv0 + t (TMEM lane t): P^T = exp2(S^T c - L), dS^T =
//               P^T o (dP^T - D) with the causal/window mask; P^T and dS^T go back to TMEM
//               as bf16 (A operands of the dV/dK MMAs) and dS^T also to shared memory (B
//               operand of the dQ^T MMA).  At the end they write dK and dV.
//   warps 4-7   thread t owns head-dim column t of dQ_i^T (TMEM lane t) and adds its 64
//               values into the fp32 accumulator with coalesced reductions.
// TMEM columns: [0,128) dK, [128,256) dV, [256,320)/[320,384) S^T buffers (later P^T in the
// first 32 columns and dS^T in the next 32), [384,448) dP^T, [448,512) dQ^T.
#pragma once

#include "sm100.cuh"

namespace fa {

constexpr int kBwdKeys = 128;    // keys per CTA
constexpr int kBwdRows = 64;     // queries per iteration
constexpr int kBwdQStages = 3;
constexpr int kBwdThreads = 320;
constexpr int kBwdWarpTma = 8;
constexpr int kBwdWarpMma = 9;
constexpr uint32_t kTdK = 0, kTdV = 128, kTS = 256, kTdP = 384, kTdQ = 448;

struct BwdParams {
  const float* lp;        // [BH, Np] L * log2(e), +inf on padded rows
  const float* dd;        // [BH, Np] D
  float* dq_acc;          // [BH, Np, D]
  __nv_bfloat16* dk;      // [BH, N, D]
  __nv_bfloat16* dv;      // [BH, N, D]
  int N, Np, BH, n_kv_tiles, causal, window;
  float scale_log2;       // scale * log2(e)
  float scale;
  unsigned long long wait_limit_ns;
};

template <int D>
struct BwdSmem {
  static constexpr int kChunks = D / 64;
  static constexpr uint32_t kKVBytes = kBwdKeys * D * 2;   // K or V tile
  static constexpr uint32_t kQBytes = kBwdRows * D * 2;    // Q or dO tile
  static constexpr uint32_t kDsBytes = kBwdKeys * kBwdRows * 2;
  alignas(1024) uint8_t k[kKVBytes];
  alignas(1024) uint8_t v[kKVBytes];
  alignas(1024) uint8_t q[kBwdQStages][kQBytes];
  alignas(1024) uint8_t dout[kBwdQStages][kQBytes];
  alignas(1024) uint8_t ds[2][kDsBytes];
  alignas(16) float lp[kBwdQStages][kBwdRows];
  alignas(16) float dd[kBwdQStages][kBwdRows];
  alignas(8) uint64_t kv_full;
  uint64_t q_full[kBwdQStages], q_empty[kBwdQStages];
  uint64_t s_full[2], s_free[2], ds_full[2], ds_free[2];
  uint64_t dp_full, dp_free, dq_full, dq_free, mma_final, mma_drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

// query tiles (of 64 rows) that can see some key of the tile [kv0, kv0 + 128)
__device__ __forceinline__ void q_tile_range(int kv0, int N, int causal, int window, int& i_begin, int& i_end) {
  const int n_q = (N + kBwdRows - 1) / kBwdRows;
  i_begin = causal ? kv0 / kBwdRows : 0;
  i_end = n_q;
  if (window > 0) {
    const long long last_q = (long long)kv0 + kBwdKeys - 1 + window - 1;   // last query whose band reaches the tile
    i_end = (int)min((long long)n_q, last_q / kBwdRows + 1);
  }
}

// ----------------------------------------------------------------------------- preprocess
// One group of D/8 threads per (padded) row: D_i = sum_c dO_ic O_ic, L_i * log2(e), zero dQacc.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_prep(const __nv_bfloat16* __restrict__ o,
                                                   const __nv_bfloat16* __restrict__ dout,
                                                   const float* __restrict__ lse, float* __restrict__ lp,
                                                   float* __restrict__ dd, float* __restrict__ dq_acc, int N, int Np,
                                                   long long total_rows) {
  constexpr int G = D / 8;                      // threads per row
  const long long g = (long long)blockIdx.x * (256 / G) + threadIdx.x / G;
  const int c = threadIdx.x % G;
  if (g >= total_rows) return;
  const long long bh = g / Np;
  const int n = int(g % Np);
  float dot = 0.f;
  if (n < N) {
    const size_t off = (size_t(bh) * N + n) * D + c * 8;
    const uint4 a = *reinterpret_cast<const uint4*>(o + off);
    const uint4 b = *reinterpret_cast<const uint4*>(dout + off);
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 fa = __bfloat1622float2(pa[j]);
      const float2 fb = __bfloat1622float2(pb[j]);
      dot = fmaf(fa.x, fb.x, dot);
      dot = fmaf(fa.y, fb.y, dot);
    }
  }
#pragma unroll
  for (int w = G / 2; w >= 1; w >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, w, G);
  if (c == 0) {
    dd[g] = dot;
    lp[g] = n < N ? lse[size_t(bh) * N + n] * 1.4426950408889634f : INFINITY;
  }
  float4* acc = reinterpret_cast<float4*>(dq_acc + size_t(g) * D + c * 8);
  acc[0] = make_float4(0.f, 0.f, 0.f, 0.f);
  acc[1] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ----------------------------------------------------------------------------- dQ finalise
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_dq_final(const float* __restrict__ dq_acc,
                                                       __nv_bfloat16* __restrict__ dq, int N, int Np, float scale,
                                                       long long total_rows) {
  constexpr int G = D / 8;
  const long long g = (long long)blockIdx.x * (256 / G) + threadIdx.x / G;   // row of [BH, N]
  const int c = threadIdx.x % G;
  if (g >= total_rows) return;
  const long long bh = g / N;
  const int n = int(g % N);
  const float4* src = reinterpret_cast<const float4*>(dq_acc + (size_t(bh) * Np + n) * D + c * 8);
  const float4 a = src[0], b = src[1];
  uint4 out;
  out.x = pack_bf16x2(a.x * scale, a.y * scale);
  out.y = pack_bf16x2(a.z * scale, a.w * scale);
  out.z = pack_bf16x2(b.x * scale, b.y * scale);
  out.w = pack_bf16x2(b.z * scale, b.w * scale);
  *reinterpret_cast<uint4*>(dq + size_t(g) * D + c * 8) = out;
}

// ----------------------------------------------------------------------------- main kernel
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const BwdParams prm) {
  using Smem = BwdSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = int(blockIdx.x / prm.n_kv_tiles);
  const int kv_tile = int(blockIdx.x % prm.n_kv_tiles);    // longest causal tiles first within a head
  const int kv0 = kv_tile * kBwdKeys;
  int i_begin, i_end;
  q_tile_range(kv0, prm.N, prm.causal, prm.window, i_begin, i_end);
  const int n_it = i_end - i_begin;                        // >= 1
  volatile int* abort = &sm.abort;
  const uint64_t lim = prm.wait_limit_ns;

  if (threadIdx.x == 0) {
    sm.abort = 0;
    mbar_init(smem_u32(&sm.kv_full), 1);
    for (int s = 0; s < kBwdQStages; ++s) {
      mbar_init(smem_u32(&sm.q_full[s]), 1);
      mbar_init(smem_u32(&sm.q_empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&sm.s_full[b]), 1);
      mbar_init(smem_u32(&sm.s_free[b]), 1);
      mbar_init(smem_u32(&sm.ds_full[b]), 128);
      mbar_init(smem_u32(&sm.ds_free[b]), 1);
    }
    mbar_init(smem_u32(&sm.dp_full), 1);
    mbar_init(smem_u32(&sm.dp_free), 128);
    mbar_init(smem_u32(&sm.dq_full), 1);
    mbar_init(smem_u32(&sm.dq_free), D);
    mbar_init(smem_u32(&sm.mma_final), 1);
    mbar_init(smem_u32(&sm.mma_drain), 1);
    fence_mbar_init();
  }
  if (warp == kBwdWarpTma && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
  }
  if (warp == kBwdWarpMma) {
    tmem_alloc(smem_u32(&sm.tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == kBwdWarpTma) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint32_t kvb = smem_u32(&sm.kv_full);
      mbar_expect_tx(kvb, 2 * Smem::kKVBytes);
      for (int c = 0; c < Smem::kChunks; ++c) {
        tma_load_3d(smem_u32(sm.k) + c * 16384, &tm_k, kvb, c * 64, kv0, bh);
        tma_load_3d(smem_u32(sm.v) + c * 16384, &tm_v, kvb, c * 64, kv0, bh);
      }
      int issued = 0;
      for (int it = 0; it < n_it; ++it) {
        const int qs = it % kBwdQStages;
        const uint32_t ph = (it / kBwdQStages) & 1;
        const int q0 = (i_begin + it) * kBwdRows;
        if (!mbar_wait(smem_u32(&sm.q_empty[qs]), ph ^ 1, abort, lim)) break;
        const uint32_t qb = smem_u32(&sm.q_full[qs]);
        mbar_expect_tx(qb, 2 * Smem::kQBytes + 2 * kBwdRows * 4);
        for (int c = 0; c < Smem::kChunks; ++c) {
          tma_load_3d(smem_u32(sm.q[qs]) + c * 8192, &tm_q, qb, c * 64, q0, bh);
          tma_load_3d(smem_u32(sm.dout[qs]) + c * 8192, &tm_do, qb, c * 64, q0, bh);
        }
        const size_t row = size_t(bh) * prm.Np + q0;
        bulk_load(smem_u32(sm.lp[qs]), prm.lp + row, kBwdRows * 4, qb);
        bulk_load(smem_u32(sm.dd[qs]), prm.dd + row, kBwdRows * 4, qb);
        issued = it + 1;
      }
      mbar_wait_drain(kvb, 0, lim);
      for (int it = max(0, issued - kBwdQStages); it < issued; ++it)
        mbar_wait_drain(smem_u32(&sm.q_full[it % kBwdQStages]), (it / kBwdQStages) & 1, lim);
    }
  } else if (warp == kBwdWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, kBwdRows, false, false);   // S^T, dP^T
      constexpr uint32_t idesc_kv = idesc_bf16_f32(128, D, false, true);          // dV, dK (A in TMEM)
      constexpr uint32_t idesc_q = idesc_bf16_f32(128, kBwdRows, true, true);     // dQ^T
      const uint32_t k_addr = smem_u32(sm.k);
      const uint32_t v_addr = smem_u32(sm.v);
      bool ok = mbar_wait(smem_u32(&sm.kv_full), 0, abort, lim);
      for (int it = 0; ok && it <= n_it; ++it) {
        if (it < n_it) {
          const int qs = it % kBwdQStages;
          const int st = it & 1;
          if (!mbar_wait(smem_u32(&sm.q_full[qs]), (it / kBwdQStages) & 1, abort, lim)) break;
          if (!mbar_wait(smem_u32(&sm.s_free[st]), ((it >> 1) & 1) ^ 1, abort, lim)) break;
          tc_fence_after();
          const uint32_t q_addr = smem_u32(sm.q[qs]);
          const uint32_t do_addr = smem_u32(sm.dout[qs]);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t a_off = (kk >> 2) * 16384 + (kk & 3) * 32;
            const uint32_t b_off = (kk >> 2) * 8192 + (kk & 3) * 32;
            mma_bf16_ss(tmem + kTS + st * 64, sw128_desc(k_addr + a_off, 16, 1024),
                        sw128_desc(q_addr + b_off, 16, 1024), idesc_s, kk > 0);
          }
          mma_commit(smem_u32(&sm.s_full[st]));
          if (!mbar_wait(smem_u32(&sm.dp_free), (it & 1) ^ 1, abort, lim)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t a_off = (kk >> 2) * 16384 + (kk & 3) * 32;
            const uint32_t b_off = (kk >> 2) * 8192 + (kk & 3) * 32;
            mma_bf16_ss(tmem + kTdP, sw128_desc(v_addr + a_off, 16, 1024), sw128_desc(do_addr + b_off, 16, 1024),
                        idesc_s, kk > 0);
          }
          mma_commit(smem_u32(&sm.dp_full));
        }
        if (it > 0) {
          const int u = it - 1;
          const int qsu = u % kBwdQStages;
          const int su = u & 1;
          if (!mbar_wait(smem_u32(&sm.ds_full[su]), (u >> 1) & 1, abort, lim)) break;
          tc_fence_after();
          const uint32_t q_addr = smem_u32(sm.q[qsu]);
          const uint32_t do_addr = smem_u32(sm.dout[qsu]);
#pragma unroll
          for (int kk = 0; kk < kBwdRows / 16; ++kk) {
            // B = dO_i / Q_i as MN-major [queries x D]: 16 queries per k-step = 2 KB, the next
            // 64 head-dim columns one 8 KB chunk (LBO) further.
            mma_bf16_ts(tmem + kTdV, tmem + kTS + su * 64 + kk * 8, sw128_desc(do_addr + kk * 2048, 8192, 1024),
                        idesc_kv, (u > 0 || kk > 0));
          }
#pragma unroll
          for (int kk = 0; kk < kBwdRows / 16; ++kk) {
            mma_bf16_ts(tmem + kTdK, tmem + kTS + su * 64 + 32 + kk * 8,
                        sw128_desc(q_addr + kk * 2048, 8192, 1024), idesc_kv, (u > 0 || kk > 0));
          }
          mma_commit(smem_u32(&sm.s_free[su]));
          if (!mbar_wait(smem_u32(&sm.dq_free), (u & 1) ^ 1, abort, lim)) break;
          tc_fence_after();
          const uint32_t ds_addr = smem_u32(sm.ds[su]);
#pragma unroll
          for (int kk = 0; kk < kBwdKeys / 16; ++kk) {
            // A = K^T (MN-major over the head dim: 64-column chunks 16 KB apart), B = dS^T
            // (MN-major over the 64 queries); 16 keys per k-step = 2 KB in both.
            mma_bf16_ss(tmem + kTdQ, sw128_desc(k_addr + kk * 2048, 16384, 1024),
                        sw128_desc(ds_addr + kk * 2048, 8192, 1024), idesc_q, kk > 0);
          }
          mma_commit(smem_u32(&sm.dq_full));
          mma_commit(smem_u32(&sm.ds_free[su]));
          mma_commit(smem_u32(&sm.q_empty[qsu]));
        }
      }
      mma_commit(smem_u32(&sm.mma_final));
      mma_commit(smem_u32(&sm.mma_drain));
      mbar_wait_drain(smem_u32(&sm.mma_drain), 0, lim);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------------ P^T / dS^T warps
    const int r = threadIdx.x;                 // key row within the tile == TMEM lane
    const int key = kv0 + r;
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const float c = prm.scale_log2;
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int qs = it % kBwdQStages;
      const int st = it & 1;
      const int q0 = (i_begin + it) * kBwdRows;
      bool w_ok = mbar_wait(smem_u32(&sm.q_full[qs]), (it / kBwdQStages) & 1, abort, lim);
      w_ok = w_ok && mbar_wait(smem_u32(&sm.s_full[st]), (it >> 1) & 1, abort, lim);
      if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
      tc_fence_after();
      float s[kBwdRows], dp[kBwdRows];
      {
        uint32_t ra[32], rb[32];
        tmem_ld32(tmem + lane_base + kTS + st * 64, ra);
        tmem_ld32(tmem + lane_base + kTS + st * 64 + 32, rb);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          s[j] = __uint_as_float(ra[j]);
          s[32 + j] = __uint_as_float(rb[j]);
        }
      }
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.dp_full), it & 1, abort, lim))) { ok = false; break; }
      tc_fence_after();
      {
        uint32_t ra[32], rb[32];
        tmem_ld32(tmem + lane_base + kTdP, ra);
        tmem_ld32(tmem + lane_base + kTdP + 32, rb);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          dp[j] = __uint_as_float(ra[j]);
          dp[32 + j] = __uint_as_float(rb[j]);
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&sm.dp_free));

      const float* lp = sm.lp[qs];
      const float* dd = sm.dd[qs];
      const bool need_mask = (prm.causal && kv0 + kBwdKeys - 1 > q0) ||
                             (prm.window > 0 && kv0 < q0 + kBwdRows - prm.window) || (kv0 + kBwdKeys > prm.N);
      uint32_t pp[kBwdRows / 2], pd[kBwdRows / 2];
#pragma unroll
      for (int j = 0; j < kBwdRows; j += 2) {
        float p0 = ex2_approx(fmaf(s[j], c, -lp[j]));
        float p1 = ex2_approx(fmaf(s[j + 1], c, -lp[j + 1]));
        if (need_mask) {
          const int qa = q0 + j, qb = q0 + j + 1;
          const bool oka = key < prm.N && (!prm.causal || key <= qa) && (prm.window == 0 || key > qa - prm.window);
          const bool okb = key < prm.N && (!prm.causal || key <= qb) && (prm.window == 0 || key > qb - prm.window);
          p0 = oka ? p0 : 0.f;
          p1 = okb ? p1 : 0.f;
        }
        const float d0 = p0 * (dp[j] - dd[j]);
        const float d1 = p1 * (dp[j + 1] - dd[j + 1]);
        pp[j / 2] = pack_bf16x2(p0, p1);
        pd[j / 2] = pack_bf16x2(d0, d1);
      }
      // P^T and dS^T into this S buffer's columns (A operands of the dV / dK MMAs)
      tmem_st32(tmem + lane_base + kTS + st * 64, pp);
      tmem_st32(tmem + lane_base + kTS + st * 64 + 32, pd);
      // dS^T into shared memory for the dQ^T MMA; the buffer is free once the dQ^T MMA of
      // iteration it - 2 has completed
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.ds_free[st]), ((it >> 1) & 1) ^ 1, abort, lim))) {
        ok = false;
        break;
      }
      const uint32_t row_addr = smem_u32(sm.ds[st]) + r * 128;
#pragma unroll
      for (int c16 = 0; c16 < 8; ++c16)
        st_shared_v4(row_addr + ((c16 ^ (r & 7)) << 4), pd[4 * c16], pd[4 * c16 + 1], pd[4 * c16 + 2],
                     pd[4 * c16 + 3]);
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(smem_u32(&sm.ds_full[st]));
    }
    // epilogue: dK = scale * acc, dV = acc, rows of keys < N
    if (ok && __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.mma_final), 0, abort, lim))) {
      tc_fence_after();
      const bool in_range = key < prm.N;
      const size_t row_off = (size_t(bh) * prm.N + (in_range ? key : 0)) * D;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        __nv_bfloat16* dst_row = (which == 0 ? prm.dk : prm.dv) + row_off;
        const float mul = which == 0 ? prm.scale : 1.f;
        const uint32_t col0 = which == 0 ? kTdK : kTdV;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t rr[32];
          tmem_ld32(tmem + lane_base + col0 + ch * 32, rr);
          uint32_t w[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            w[j] = pack_bf16x2(__uint_as_float(rr[2 * j]) * mul, __uint_as_float(rr[2 * j + 1]) * mul);
          if (in_range) {
            uint4* dst = reinterpret_cast<uint4*>(dst_row + ch * 32);
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
          }
        }
      }
    }
  } else if (warp < 8 && (warp - 4) * 32 < D) {
    // ------------------------------------------------------------------ dQ warps
    const int dcol = (warp - 4) * 32 + lane;    // head-dim column == TMEM lane of dQ^T
    const uint32_t lane_base = uint32_t((warp - 4) * 32) << 16;
    for (int it = 0; it < n_it; ++it) {
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.dq_full), it & 1, abort, lim))) break;
      tc_fence_after();
      uint32_t ra[32], rb[32];
      tmem_ld32(tmem + lane_base + kTdQ, ra);
      tmem_ld32(tmem + lane_base + kTdQ + 32, rb);
      tc_fence_before();
      mbar_arrive(smem_u32(&sm.dq_free));
      const int q0 = (i_begin + it) * kBwdRows;
      float* acc = prm.dq_acc + (size_t(bh) * prm.Np + q0) * D + dcol;
#pragma unroll
      for (int j = 0; j < 32; ++j) atomicAdd(acc + size_t(j) * D, __uint_as_float(ra[j]));
#pragma unroll
      for (int j = 0; j < 32; ++j) atomicAdd(acc + size_t(32 + j) * D, __uint_as_float(rb[j]));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kBwdWarpMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa
