// Backward pass of exact attention at head dimension 256: the same gradients as fa_bwd_kernel
// (bwd_kernel.cuh), with a plan that fits d = 256.
//
// At d = 256 the dK and dV accumulators of a 128-key tile alone fill the 512 TMEM columns, and
// full-width 128-key K and V tiles take 128 KB of shared memory.  Here each CTA owns a 64-key
// tile of one K/V head and loops over the 128-row query tiles (of every query head that reads
// the K/V head):
//   S  = Q K^T,  dP = dO V^T             full d, M = 128 queries, N = 64 keys
//   P  = exp2(S c - L log2 e) (masked),  dS = P o (dP - D)           compute warps
//   dV^T_c += dO_c^T P,  dK^T_c += Q_c^T dS   for both head-dim halves c (columns 128c ..),
//                                        M = 128 head-dim columns, N = 64 keys, K = 128
//                                        queries: dO and Q as MN-major A operands (the same
//                                        tiles the first products read K-major), P and dS
//                                        staged in shared memory as MN-major B operands
//   dQ_c = dS K_c                        M = 128 queries, N = 128, K = 64 keys; K_c MN-major;
//                                        dQ_0 in its own columns, dQ_1 over those of S and dP
//                                        (read by then), both right after dV^T and dK^T.
// Each compute warp loads its 32 rows of dQ_c from TMEM at once (freeing the columns for the
// next product), then stages them 32 columns at a time in 4 KB slots in the 128-byte swizzled
// layout and adds each 32 x 32 block into the fp32 accumulator with one TMA tensor reduction
// (whole 128-byte lines at the L2).  The slots are the warp's own 32 rows of the dS and P tiles,
// in turn: both are free once dQ_1 is complete (every MMA that reads them came first).  The warp
// writes those rows again (the next tile's P and dS) only after the reductions have read them.
// Roles (192 threads): warps 0-3 compute (thread t of warp w owns TMEM lane 32w + t: a query
// row of S, dP and dQ, and at the end a head-dim column of each half of dV^T and dK^T), warp 4
// TMA, warp 5 MMA.  TMEM columns: S [0, 64), dP [64, 128), dV^T_0 [128, 192), dV^T_1 [192, 256),
// dK^T_0 [256, 320), dK^T_1 [320, 384), dQ_0 [384, 512), dQ_1 [0, 128): the next tile's S and dP
// wait until dQ_1 has been read out.
// One stage of Q and dO: the next query tile loads once the dV and dK MMAs of this one are
// done, while dQ is computed and read out.
#pragma once

#include <type_traits>

#include "bwd_kernel.cuh"

namespace fa {

constexpr int kB256Keys = 64;     // keys per CTA
constexpr int kB256Rows = 128;    // query rows per iteration
constexpr int kB256Threads = 192;
constexpr int kB256WarpTma = 4;
constexpr int kB256WarpMma = 5;
constexpr uint32_t kT256S = 0, kT256dP = 64, kT256dV = 128, kT256dK = 256;   // dV^T_c, dK^T_c at + 64c
constexpr uint32_t kT256dQ0 = 384, kT256dQ1 = 0;

struct Bwd256Smem {
  static constexpr uint32_t kQChunk = kB256Rows * 128;   // 64 head-dim columns of 128 rows
  static constexpr uint32_t kKChunk = kB256Keys * 128;   // 64 head-dim columns of 64 keys
  alignas(1024) uint8_t q[4 * kQChunk];
  alignas(1024) uint8_t dout[4 * kQChunk];
  alignas(1024) uint8_t k[4 * kKChunk];
  alignas(1024) uint8_t v[4 * kKChunk];
  alignas(1024) uint8_t p[kB256Rows * 128];    // P  [query][key], 128-byte swizzled rows
  alignas(1024) uint8_t ds[kB256Rows * 128];   // dS [query][key]
  alignas(16) float lp[kB256Rows];
  alignas(16) float dd[kB256Rows];
  // q_empty: Q and dO read by this tile's last MMAs that use them (dV^T, dK^T)
  alignas(8) uint64_t kv_full, q_full, q_empty, s_full, p_full, dq_full, dq_free0, dq_free1, mma_final, mma_drain;
  uint32_t tmem_base;
  int abort;
};

// query tiles (of 128 rows) that can see some key of [kv0, kv0 + 64)
__device__ __forceinline__ void q_tile_range256(int kv0, int N, int causal, int window, int& i_begin, int& i_end) {
  const int n_q = (N + kB256Rows - 1) / kB256Rows;
  i_begin = causal ? kv0 / kB256Rows : (window > 0 ? max(0, kv0 - window + 1) / kB256Rows : 0);
  i_end = n_q;
  if (window > 0) {
    const long long last_q = (long long)kv0 + kB256Keys - 1 + window - 1;
    i_end = (int)min((long long)n_q, last_q / kB256Rows + 1);
  }
}

// One CTA per (K/V head, 64-key tile), in grid_item's chunked order.
// prm.n_kv_tiles counts 64-key tiles here.
__global__ void __launch_bounds__(kB256Threads, 1)
    fa_bwd256_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_dq, const BwdParams prm) {
  using Smem = Bwd256Smem;
  constexpr int D = 256;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((reinterpret_cast<uintptr_t>(smem_raw) & 1023) != 0) {
    if (threadIdx.x == 0) atomicOr(&g_status, FA_DEVICE_SMEM_ALIGN);
    return;
  }
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int bh, tile;   // K/V head (b * H_kv + h_kv) and key tile
  grid_item(int(blockIdx.x), prm.BH / prm.group, prm.n_kv_tiles, kBwdChunkHeads, bh, tile);
  const int b_idx = bh / prm.H_kv, h_kv = bh % prm.H_kv;
  const int bh_q0 = b_idx * prm.H + h_kv * prm.group;       // first query head of the group
  const int kv0 = tile * kB256Keys;
  int i_begin, i_end;
  q_tile_range256(kv0, prm.N, prm.causal, prm.window, i_begin, i_end);
  const int n_i = i_end - i_begin;
  const int n_it = n_i * prm.group;
  auto q_tile = [&](int it) { return i_begin + it % n_i; };
  auto q_head = [&](int it) { return bh_q0 + it / n_i; };
  volatile int* abort = &sm.abort;
  const uint64_t lim = prm.wait_limit_ns;

  if (threadIdx.x == 0) {
    sm.abort = 0;
    mbar_init(smem_u32(&sm.kv_full), 1);
    mbar_init(smem_u32(&sm.q_full), 1);
    mbar_init(smem_u32(&sm.q_empty), 1);
    mbar_init(smem_u32(&sm.s_full), 1);
    mbar_init(smem_u32(&sm.p_full), kB256Rows);
    mbar_init(smem_u32(&sm.dq_full), 1);            // dQ_0 and dQ_1 complete
    mbar_init(smem_u32(&sm.dq_free0), kB256Rows);   // dQ_0 read out of TMEM
    mbar_init(smem_u32(&sm.dq_free1), kB256Rows);   // dQ_1 read out of TMEM (S and dP may be written)
    mbar_init(smem_u32(&sm.mma_final), 1);
    mbar_init(smem_u32(&sm.mma_drain), 1);
    fence_mbar_init();
  }
  if (warp == kB256WarpTma) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_dq);
    }
    __syncwarp();
    tmem_alloc(smem_u32(&sm.tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == kB256WarpTma) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && n_it > 0) {
      const uint32_t kvb = smem_u32(&sm.kv_full);
      mbar_expect_tx(kvb, 2 * 4 * Smem::kKChunk);
      for (int c = 0; c < 4; ++c) {
        tma_load_rows(smem_u32(sm.k) + c * Smem::kKChunk, &tm_k, kvb, c * 64, kv0, h_kv, b_idx);
        tma_load_rows(smem_u32(sm.v) + c * Smem::kKChunk, &tm_v, kvb, c * 64, kv0, h_kv, b_idx);
      }
      const uint32_t qb = smem_u32(&sm.q_full);
      int issued = 0;
      for (int it = 0; it < n_it; ++it) {
        if (it > 0 && !mbar_wait(smem_u32(&sm.q_empty), (it - 1) & 1, abort, lim)) break;
        const int q0 = q_tile(it) * kB256Rows, hq = q_head(it);
        const int hq_b = hq % prm.H;   // query head within its batch entry
        mbar_expect_tx(qb, 2 * 4 * Smem::kQChunk + 2 * kB256Rows * 4);
        for (int c = 0; c < 4; ++c) {
          tma_load_rows(smem_u32(sm.q) + c * Smem::kQChunk, &tm_q, qb, c * 64, q0, hq_b, b_idx);
          tma_load_rows(smem_u32(sm.dout) + c * Smem::kQChunk, &tm_do, qb, c * 64, q0, hq_b, b_idx);
        }
        bulk_load(smem_u32(sm.lp), prm.lp + size_t(hq) * prm.Np + q0, kB256Rows * 4, qb);
        bulk_load(smem_u32(sm.dd), prm.dd + size_t(hq) * prm.Np + q0, kB256Rows * 4, qb);
        issued = it + 1;
      }
      mbar_wait_drain(kvb, 0, lim);
      if (issued > 0) mbar_wait_drain(qb, (issued - 1) & 1, lim);
    }
  } else if (warp == kB256WarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    auto wait = [&](uint32_t bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, lim));
    };
    constexpr uint32_t idesc_s = idesc_bf16_f32(kB256Rows, kB256Keys, false, false);    // S, dP
    constexpr uint32_t idesc_t = idesc_bf16_f32(128, kB256Keys, true, true);            // dV^T, dK^T
    constexpr uint32_t idesc_q = idesc_bf16_f32(kB256Rows, 128, false, true);           // dQ
    // K-major views (rows of 128 bytes, 8-row atoms 1024 bytes apart)
    const uint64_t dq_k = sw128_desc(smem_u32(sm.q), 16, 1024);
    const uint64_t ddo_k = sw128_desc(smem_u32(sm.dout), 16, 1024);
    const uint64_t dk_k = sw128_desc(smem_u32(sm.k), 16, 1024);
    const uint64_t dv_k = sw128_desc(smem_u32(sm.v), 16, 1024);
    const uint64_t dds_k = sw128_desc(smem_u32(sm.ds), 16, 1024);
    // MN-major views of head-dim half c: 64 columns per 128-byte row, one row per query (or
    // key), 8-row atoms 1024 bytes apart, the next 64 columns one chunk (LBO) further
    auto dq_t = [&](int c) { return sw128_desc(smem_u32(sm.q) + 2 * c * Smem::kQChunk, Smem::kQChunk, 1024); };
    auto ddo_t = [&](int c) { return sw128_desc(smem_u32(sm.dout) + 2 * c * Smem::kQChunk, Smem::kQChunk, 1024); };
    auto dk_t = [&](int c) { return sw128_desc(smem_u32(sm.k) + 2 * c * Smem::kKChunk, Smem::kKChunk, 1024); };
    const uint64_t dp_t = sw128_desc(smem_u32(sm.p), Smem::kQChunk, 1024);
    const uint64_t dds_t = sw128_desc(smem_u32(sm.ds), Smem::kQChunk, 1024);
    bool ok = n_it > 0 && wait(smem_u32(&sm.kv_full), 0);
    for (int it = 0; ok && it < n_it; ++it) {
      if (!wait(smem_u32(&sm.q_full), it & 1)) break;
      if (it > 0 && !wait(smem_u32(&sm.dq_free1), (it - 1) & 1)) break;   // dQ_1 left S and dP's columns
      tc_fence_after();
      // S = Q K^T and dP = dO V^T over the full head dimension
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t qo = (kk >> 2) * Smem::kQChunk + (kk & 3) * 32;
        const uint32_t ko = (kk >> 2) * Smem::kKChunk + (kk & 3) * 32;
        mma_bf16_ss_w(tmem + kT256S, desc_advance(dq_k, qo), desc_advance(dk_k, ko), idesc_s, kk > 0);
        mma_bf16_ss_w(tmem + kT256dP, desc_advance(ddo_k, qo), desc_advance(dv_k, ko), idesc_s, kk > 0);
      }
      mma_commit_w(smem_u32(&sm.s_full));
      if (!wait(smem_u32(&sm.p_full), it & 1)) break;
      tc_fence_after();
      // dV^T_c += dO_c^T P and dK^T_c += Q_c^T dS for both halves: 16 queries per k-step = 16
      // rows of 128 bytes
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const uint64_t dot = ddo_t(c), qt = dq_t(c);
#pragma unroll
        for (int kk = 0; kk < kB256Rows / 16; ++kk) {
          const uint32_t acc = (it > 0 || kk > 0) ? 1u : 0u;
          mma_bf16_ss_w(tmem + kT256dV + 64 * c, desc_advance(dot, kk * 2048), desc_advance(dp_t, kk * 2048),
                        idesc_t, acc);
          mma_bf16_ss_w(tmem + kT256dK + 64 * c, desc_advance(qt, kk * 2048), desc_advance(dds_t, kk * 2048),
                        idesc_t, acc);
        }
      }
      mma_commit_w(smem_u32(&sm.q_empty));   // the next Q and dO may load now
      // dQ_c = dS K_c: 16 keys per k-step (32 bytes along dS's rows, 16 rows of K).  dQ_0 waits
      // until the previous tile's dQ_0 has been read out of its columns
      if (it > 0 && !wait(smem_u32(&sm.dq_free0), (it - 1) & 1)) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const uint64_t kt = dk_t(c);
        const uint32_t dst = c == 0 ? kT256dQ0 : kT256dQ1;
#pragma unroll
        for (int kk = 0; kk < kB256Keys / 16; ++kk)
          mma_bf16_ss_w(tmem + dst, desc_advance(dds_k, kk * 32), desc_advance(kt, kk * 2048), idesc_q, kk > 0);
      }
      mma_commit_w(smem_u32(&sm.dq_full));
    }
    mma_commit_w(smem_u32(&sm.mma_final));
    mma_commit_w(smem_u32(&sm.mma_drain));
    mbar_wait_drain(smem_u32(&sm.mma_drain), 0, lim);
  } else {
    // ------------------------------------------------------------------ compute warps
    const int row = threadIdx.x;   // TMEM lane: a query row of S, dP, dQ; head-dim column row (+ 128) of dV^T, dK^T
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const uint32_t slot_p = smem_u32(sm.p) + uint32_t(warp) * 4096;    // my 32 rows of P and of dS:
    const uint32_t slot_ds = smem_u32(sm.ds) + uint32_t(warp) * 4096;  // dQ staging slots
    const float c = prm.scale_log2;
    bool ok = true;
    for (int it = 0; ok && it < n_it; ++it) {
      const int q0 = q_tile(it) * kB256Rows, hq = q_head(it);
      const int qi = q0 + row;
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.s_full), it & 1, abort, lim));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[kB256Keys], pr[kB256Keys];
      tmem_ld32_async(tmem + lane_base + kT256S, sr);
      tmem_ld32_async(tmem + lane_base + kT256S + 32, sr + 32);
      tmem_ld32_async(tmem + lane_base + kT256dP, pr);
      tmem_ld32_async(tmem + lane_base + kT256dP + 32, pr + 32);
      tmem_ld_wait();
      reg_fence<kB256Keys>(sr);
      reg_fence<kB256Keys>(pr);
      // this row's keys: [lo, hi] from the mask, and below N
      const int hi = prm.causal ? min(qi, prm.N - 1)
                                : (prm.window > 0 ? min(qi + prm.window - 1, prm.N - 1) : prm.N - 1);
      const int lo = prm.window > 0 ? qi - prm.window + 1 : 0;
      const float lrow = sm.lp[row];   // L log2(e); +inf on rows past N, so P = 0 there
      const float drow = sm.dd[row];
      uint32_t pk[kB256Keys / 2], dk2[kB256Keys / 2];
#pragma unroll
      for (int j = 0; j < kB256Keys; j += 2) {
        float p2[2], d2[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int key = kv0 + j + e;
          const bool in = key >= lo && key <= hi;
          const float p = in ? ex2_approx(__uint_as_float(sr[j + e]) * c - lrow) : 0.f;
          p2[e] = p;
          d2[e] = p * (__uint_as_float(pr[j + e]) - drow);
        }
        pk[j / 2] = pack_bf16x2(p2[0], p2[1]);
        dk2[j / 2] = pack_bf16x2(d2[0], d2[1]);
      }
      // P and dS of the previous query tile have been read by its MMAs: this warp saw its dQ
      // complete, and the MMAs finish in issue order.  My rows of both must also have
      // been read by the tensor reductions that staged dQ there.
      if (it > 0) {
        if (lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
      }
      // row `row` of the P and dS tiles: 8 chunks of 16 bytes, chunk j at j ^ (row % 8)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t off = uint32_t(row) * 128 + uint32_t((j ^ (row & 7)) * 16);
        st_shared_v4(smem_u32(sm.p) + off, pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
        st_shared_v4(smem_u32(sm.ds) + off, dk2[4 * j], dk2[4 * j + 1], dk2[4 * j + 2], dk2[4 * j + 3]);
      }
      fence_proxy_async_smem();   // the MMAs read P and dS through the async proxy
      tc_fence_before();
      mbar_arrive(smem_u32(&sm.p_full));
      // dQ_1 first (its columns are the next tile's S and dP), then dQ_0: my 32 rows into
      // registers, then 32 columns a pass through the dS and P slots in turn into the
      // accumulator rows q0 + 32 warp ..
      const int q_row = q0 + warp * 32;
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.dq_full), it & 1, abort, lim));
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int c = 1; c >= 0; --c) {
        uint32_t r[128];
        const uint32_t src = c == 0 ? kT256dQ0 : kT256dQ1;
#pragma unroll
        for (int ps = 0; ps < 4; ++ps) tmem_ld32_async(tmem + lane_base + src + ps * 32, r + 32 * ps);
        tmem_ld_wait();
        reg_fence<128>(r);
        tc_fence_before();
        mbar_arrive(smem_u32(c == 0 ? &sm.dq_free0 : &sm.dq_free1));   // the MMA warp may overwrite dQ_c
#pragma unroll
        for (int ps = 0; ps < 4; ++ps) {
          // even passes through the dS rows, odd ones through the P rows, each after the read
          // of the pass before the previous one
          const uint32_t slot = (ps & 1) ? slot_p : slot_ds;
          if (lane == 0) bulk_wait_group_read<1>();
          __syncwarp();
          // row `lane`, 16-byte chunk j at lane * 128 + (j ^ (lane & 7)) * 16
#pragma unroll
          for (int j = 0; j < 8; ++j)
            st_shared_v4(slot + lane * 128 + ((j ^ (lane & 7)) << 4), r[32 * ps + 4 * j], r[32 * ps + 4 * j + 1],
                         r[32 * ps + 4 * j + 2], r[32 * ps + 4 * j + 3]);
          fence_proxy_async_smem();   // the tensor reduction reads the slot through the async proxy
          __syncwarp();
          if (lane == 0) {
            tma_reduce_add_rows(&tm_dq, slot, c * 128 + ps * 32, q_row, hq, 0);
            bulk_commit_group();
          }
        }
      }
    }
    // dV and dK of this tile's keys, head-dim columns row and 128 + row
    if (ok && __all_sync(0xffffffffu, n_it == 0 || mbar_wait(smem_u32(&sm.mma_final), 0, abort, lim))) {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t vr[kB256Keys], kr[kB256Keys];
        if (n_it > 0) {
          tmem_ld32_async(tmem + lane_base + kT256dV + 64 * c, vr);
          tmem_ld32_async(tmem + lane_base + kT256dV + 64 * c + 32, vr + 32);
          tmem_ld32_async(tmem + lane_base + kT256dK + 64 * c, kr);
          tmem_ld32_async(tmem + lane_base + kT256dK + 64 * c + 32, kr + 32);
          tmem_ld_wait();
          reg_fence<kB256Keys>(vr);
          reg_fence<kB256Keys>(kr);
        } else {
#pragma unroll
          for (int j = 0; j < kB256Keys; ++j) vr[j] = kr[j] = 0u;
        }
        const int col = c * 128 + row;
#pragma unroll
        for (int j = 0; j < kB256Keys; ++j) {
          const int key = kv0 + j;
          if (key < prm.N) {
            prm.dv[prm.dv_st.at(b_idx, h_kv, key) + col] = __float2bfloat16_rn(__uint_as_float(vr[j]));
            prm.dk[prm.dk_st.at(b_idx, h_kv, key) + col] = __float2bfloat16_rn(__uint_as_float(kr[j]) * prm.scale);
          }
        }
      }
    }
    // every reduction this warp issued has read its slot before the CTA's shared memory is
    // released (the adds complete with the grid, before the finalise kernel runs)
    if (lane == 0) bulk_wait_group_read<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kB256WarpTma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa
