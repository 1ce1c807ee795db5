// Persistent form of fa_bwd_kernel: gridDim.x CTAs (one per SM) loop over the work items
// (K/V head, 128-key tile), so that one item's K/V load and first S^T, dP^T products overlap the
// previous item's dK/dV write and its last dQ reductions, instead of waiting for a new CTA's
// launch, barrier setup and TMEM allocation.
//
// The per-item work is fa_bwd_kernel's (same roles, TMEM columns, rings, phases A and B, dQ
// staging and reductions).  What changes is bookkeeping across items:
//   * every ring keeps its phase across items: the query iterations (Q stages, dO, S^T, dP^T,
//     P^T, dS^T, dQ and its staging slots) are numbered over the CTA's whole run;
//   * kv_empty (committed after an item's last MMA) lets the TMA warp load the next item's K, V;
//   * mma_final is committed once per item, and the compute warps wait for it every item before
//     they read dK and dV;
//   * the next item's first dV (and dK) product, which overwrites the accumulator, waits for
//     pa_full (ds_full): every compute warp arrives there only after its dK/dV readout of the
//     previous item, so the accumulators need no barrier of their own;
//   * the next item's first dP^T overwrites the dQ columns: it waits for dq_free of the previous
//     item's last readout.
// Every item runs at least one query tile, so no role skips an item's handshakes.
#pragma once

#include <type_traits>

#include "bwd_kernel.cuh"
#include "persist_sched.cuh"

namespace fa {

template <int D>
struct BwdPersistSmem {
  static constexpr int kChunks = D / 64;
  static constexpr uint32_t kTileBytes = 128 * D * 2;
  alignas(1024) uint8_t k[kTileBytes];
  alignas(1024) uint8_t v[kTileBytes];
  alignas(1024) uint8_t q[kBwdQStages][kTileBytes];
  alignas(1024) uint8_t dout[kTileBytes];
  alignas(1024) uint8_t ds[kBwdKeys * kBwdRows * 2];
  alignas(1024) uint8_t stage[8][32 * 32 * 4];
  alignas(16) float lp[kBwdQStages][kBwdRows];
  alignas(16) float dd[kBwdQStages][kBwdRows];
  alignas(8) uint64_t kv_full, kv_empty;
  uint64_t q_full[kBwdQStages], q_empty[kBwdQStages], do_full, do_empty;
  uint64_t s_full, dp_full, pa_full, ds_full, dq_full, dq_free, mma_final, mma_drain;
  uint64_t st_full[8], st_free[8];
  uint32_t tmem_base;
  int abort;
};

// The item at position `pos` of `order`: its K/V head and key tile, and the query tiles (of each
// query head of its group) that see the tile.  Cost-major is key-tile-major from tile 0, the
// longest under a causal mask.
struct BwdItem {
  int b_idx, h_kv, kv0, i_begin, n_i, n_it, bh_q0;
};
__device__ __forceinline__ BwdItem bwd_item(const BwdParams& prm, int order, int pos) {
  const int bh_kv_count = prm.BH / prm.group;
  const int bh = order == kOrderPairMajor ? pos % bh_kv_count : pos / prm.n_kv_tiles;
  const int tile = order == kOrderPairMajor ? pos / bh_kv_count : pos % prm.n_kv_tiles;
  BwdItem it;
  it.b_idx = bh / prm.H_kv;
  it.h_kv = bh % prm.H_kv;
  it.kv0 = tile * kBwdKeys;
  int i_end;
  q_tile_range(it.kv0, prm.N, prm.causal, prm.window, it.i_begin, i_end);
  it.n_i = i_end - it.i_begin;   // >= 1
  it.n_it = it.n_i * prm.group;
  it.bh_q0 = it.b_idx * prm.H + it.h_kv * prm.group;   // first query head of the group
  return it;
}
// query tile and query head of the item's iteration `it`
__device__ __forceinline__ int bwd_q_tile(const BwdItem& w, int group, int it) {
  return group == 1 ? w.i_begin + it : w.i_begin + it % w.n_i;
}
__device__ __forceinline__ int bwd_q_head(const BwdItem& w, int group, int it) {
  return group == 1 ? w.bh_q0 : w.bh_q0 + it / w.n_i;
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_persist_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                          const BwdParams prm, const int order) {
  using Smem = BwdPersistSmem<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicOr(&g_status, FA_DEVICE_SMEM_ALIGN);
    return;
  }
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_items = prm.n_kv_tiles * (prm.BH / prm.group);
  volatile int* abort = &sm.abort;
  const uint64_t lim = prm.wait_limit_ns;

  if (threadIdx.x == 0) {
    sm.abort = 0;
    mbar_init(smem_u32(&sm.kv_full), 1);
    mbar_init(smem_u32(&sm.kv_empty), 1);
    for (int s = 0; s < kBwdQStages; ++s) {
      mbar_init(smem_u32(&sm.q_full[s]), 1);
      mbar_init(smem_u32(&sm.q_empty[s]), 1);
    }
    mbar_init(smem_u32(&sm.s_full), 1);
    mbar_init(smem_u32(&sm.dp_full), 1);
    mbar_init(smem_u32(&sm.pa_full), 256);
    mbar_init(smem_u32(&sm.ds_full), 256);
    mbar_init(smem_u32(&sm.dq_full), 1);
    mbar_init(smem_u32(&sm.dq_free), 256);
    mbar_init(smem_u32(&sm.mma_final), 1);
    mbar_init(smem_u32(&sm.mma_drain), 1);
    mbar_init(smem_u32(&sm.do_full), 1);
    mbar_init(smem_u32(&sm.do_empty), 1);
    for (int w = 0; w < 8; ++w) {
      mbar_init(smem_u32(&sm.st_full[w]), 32);
      mbar_init(smem_u32(&sm.st_free[w]), 32);
    }
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
      int issued = 0, issued_do = 0;   // Q (with L, D rows) and dO loads over the run
      int n_local = 0;
      bool ok = true;
      for (int pos; ok && (pos = persist_item(n_items, n_local)) >= 0; ++n_local) {
        const BwdItem w = bwd_item(prm, order, pos);
        // the previous item's MMAs have read K and V
        if (n_local > 0 && !mbar_wait(smem_u32(&sm.kv_empty), (n_local - 1) & 1, abort, lim)) break;
        mbar_expect_tx(kvb, 2 * Smem::kTileBytes);
        for (int c = 0; c < Smem::kChunks; ++c) {
          tma_load_rows(smem_u32(sm.k) + c * 16384, &tm_k, kvb, c * 64, w.kv0, w.h_kv, w.b_idx);
          tma_load_rows(smem_u32(sm.v) + c * 16384, &tm_v, kvb, c * 64, w.kv0, w.h_kv, w.b_idx);
        }
        for (int it = 0; it < w.n_it; ++it) {
          const int ir = issued;   // this iteration's number over the run
          const int qs = ir % kBwdQStages;
          const uint32_t ph = (ir / kBwdQStages) & 1;
          const int q0 = bwd_q_tile(w, prm.group, it) * kBwdRows;
          const int bq = bwd_q_head(w, prm.group, it);
          if (!mbar_wait(smem_u32(&sm.q_empty[qs]), ph ^ 1, abort, lim)) {
            ok = false;
            break;
          }
          const uint32_t qb = smem_u32(&sm.q_full[qs]);
          mbar_expect_tx(qb, Smem::kTileBytes + 2 * kBwdRows * 4);
          for (int c = 0; c < Smem::kChunks; ++c)
            tma_load_rows(smem_u32(sm.q[qs]) + c * 16384, &tm_q, qb, c * 64, q0, bq - w.b_idx * prm.H, w.b_idx);
          const size_t row = size_t(bq) * prm.Np + q0;
          bulk_load(smem_u32(sm.lp[qs]), prm.lp + row, kBwdRows * 4, qb);
          bulk_load(smem_u32(sm.dd[qs]), prm.dd + row, kBwdRows * 4, qb);
          issued = ir + 1;
          if (!mbar_wait(smem_u32(&sm.do_empty), (ir & 1) ^ 1, abort, lim)) {
            ok = false;
            break;
          }
          const uint32_t db = smem_u32(&sm.do_full);
          mbar_expect_tx(db, Smem::kTileBytes);
          for (int c = 0; c < Smem::kChunks; ++c)
            tma_load_rows(smem_u32(sm.dout) + c * 16384, &tm_do, db, c * 64, q0, bq - w.b_idx * prm.H, w.b_idx);
          issued_do = ir + 1;
        }
      }
      // let every copy this CTA started land before the CTA may exit
      if (n_local > 0) mbar_wait_drain(kvb, (n_local - 1) & 1, lim);
      for (int ir = max(0, issued - kBwdQStages); ir < issued; ++ir)
        mbar_wait_drain(smem_u32(&sm.q_full[ir % kBwdQStages]), (ir / kBwdQStages) & 1, lim);
      if (issued_do > 0) mbar_wait_drain(smem_u32(&sm.do_full), (issued_do - 1) & 1, lim);
    }
  } else if (warp == kBwdWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    auto wait = [&](uint32_t bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, lim));
    };
    constexpr uint32_t idesc_t = idesc_bf16_f32(128, kBwdRows, false, false);   // S^T, dP^T
    constexpr uint32_t idesc_kv = idesc_bf16_f32(128, D, false, true);          // dV, dK (A in TMEM)
    constexpr uint32_t idesc_q = idesc_bf16_f32(kBwdRows, D, true, true);       // dQ
    const uint64_t dk_kmaj = sw128_desc(smem_u32(sm.k), 16, 1024);
    const uint64_t dv_kmaj = sw128_desc(smem_u32(sm.v), 16, 1024);
    const uint64_t dk_mn = sw128_desc(smem_u32(sm.k), 16384, 1024);
    const uint64_t dds_mn = sw128_desc(smem_u32(sm.ds), 16384, 1024);
    auto issue_t = [&](uint64_t a, const uint8_t* b_tile, uint32_t d_col) {
      const uint64_t b = sw128_desc(smem_u32(b_tile), 16, 1024);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        mma_bf16_ss_w(tmem + d_col, desc_advance(a, off), desc_advance(b, off), idesc_t, kk > 0);
      }
    };
    auto issue_kv = [&](uint32_t a_col, const uint8_t* b_tile, uint32_t d_col, bool first) {
      const uint64_t b = sw128_desc(smem_u32(b_tile), 16384, 1024);
#pragma unroll
      for (int kk = 0; kk < kBwdRows / 16; ++kk)
        mma_bf16_ts_w(tmem + d_col, tmem + a_col + (kk >> 2) * 64 + (kk & 3) * 8, desc_advance(b, kk * 2048),
                      idesc_kv, (first && kk == 0) ? 0u : 1u);
    };
    int it_run = 0;   // query iterations of the finished items
    int n_local = 0;
    bool ok = true;
    for (int pos; ok && (pos = persist_item(n_items, n_local)) >= 0; ++n_local) {
      const BwdItem w = bwd_item(prm, order, pos);
      const int q_first = it_run % kBwdQStages;
      ok = wait(smem_u32(&sm.kv_full), n_local & 1) &&
           wait(smem_u32(&sm.q_full[q_first]), (it_run / kBwdQStages) & 1);
      if (ok) {
        tc_fence_after();
        issue_t(dk_kmaj, sm.q[q_first], kTS);
        mma_commit_w(smem_u32(&sm.s_full));
        // the first dP^T overwrites the dQ columns the previous item's last readout read
        ok = (it_run == 0 || wait(smem_u32(&sm.dq_free), (it_run - 1) & 1)) &&
             wait(smem_u32(&sm.do_full), it_run & 1);
      }
      if (ok) {
        tc_fence_after();
        issue_t(dv_kmaj, sm.dout, kTdP);
        mma_commit_w(smem_u32(&sm.dp_full));
      }
      for (int it = 0; ok && it < w.n_it; ++it) {
        const int ir = it_run + it;
        const int qs = ir % kBwdQStages;
        const bool has_next = it + 1 < w.n_it;
        const int qn = (ir + 1) % kBwdQStages;
        // dV += P^T dO_i (the item's first overwrites the accumulator: every compute warp has
        // read the previous item's dV out before it arrived on pa_full)
        if (!wait(smem_u32(&sm.pa_full), ir & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_kv(kTP, sm.dout, kTdV, it == 0);
        mma_commit_w(smem_u32(&sm.do_empty));
        if (has_next) {
          if (!wait(smem_u32(&sm.q_full[qn]), ((ir + 1) / kBwdQStages) & 1)) {
            ok = false;
            break;
          }
          issue_t(dk_kmaj, sm.q[qn], kTS);
          mma_commit_w(smem_u32(&sm.s_full));
        }
        if (!wait(smem_u32(&sm.ds_full), ir & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_kv(kTdS, sm.q[qs], kTdK, it == 0);
        if (!wait(smem_u32(&sm.dq_free), (ir & 1) ^ 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBwdKeys / 16; ++kk)
          mma_bf16_ss_w(tmem + kTdQ, desc_advance(dds_mn, kk * 2048), desc_advance(dk_mn, kk * 2048), idesc_q, kk > 0);
        mma_commit_w(smem_u32(&sm.dq_full));
        mma_commit_w(smem_u32(&sm.q_empty[qs]));
        if (has_next) {
          if (!wait(smem_u32(&sm.dq_free), ir & 1) || !wait(smem_u32(&sm.do_full), (ir + 1) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_t(dv_kmaj, sm.dout, kTdP);
          mma_commit_w(smem_u32(&sm.dp_full));
        }
      }
      if (!ok) break;
      it_run += w.n_it;
      mma_commit_w(smem_u32(&sm.mma_final));   // dK, dV of the item are complete
      mma_commit_w(smem_u32(&sm.kv_empty));    // and K, V have been read
    }
    mma_commit_w(smem_u32(&sm.mma_drain));
    mbar_wait_drain(smem_u32(&sm.mma_drain), 0, lim);
  } else if (warp < 8) {
    // ------------------------------------------------------------------ compute warps
    const int quad = warp & 3;
    const int hq = warp >> 2;
    const int r = quad * 32 + lane;
    const uint32_t lane_base = uint32_t(quad * 32) << 16;
    const float c = prm.scale_log2;
    const uint32_t col_s = kTS + hq * 64;
    const uint32_t col_dp = kTdP + hq * 64;
    const uint32_t col_dq = kTdQ + hq * (D / 2);
    const uint32_t ds_row = smem_u32(sm.ds) + hq * 16384 + r * 128;
    const uint32_t sw = r & 7;
    const uint32_t stage = smem_u32(sm.stage[warp]);
    int n_pass = 0;   // dQ blocks staged over the run: their parity is the slot barriers' phase
    int it_run = 0;
    int n_local = 0;
    bool ok = true;
    for (int pos; ok && (pos = persist_item(n_items, n_local)) >= 0; ++n_local) {
      const BwdItem w = bwd_item(prm, order, pos);
      const int kv0 = w.kv0;
      const int key = kv0 + r;
      uint32_t pk[32];
      // phase A of the item's iteration it (run number it_run + it), as in fa_bwd_kernel
      auto phase_a = [&](int it, auto masked) -> bool {
        const int ir = it_run + it;
        const int qs = ir % kBwdQStages;
        const int q0 = bwd_q_tile(w, prm.group, it) * kBwdRows;
        bool w_ok = mbar_wait(smem_u32(&sm.q_full[qs]), (ir / kBwdQStages) & 1, abort, lim);
        w_ok = w_ok && mbar_wait(smem_u32(&sm.s_full), ir & 1, abort, lim);
        if (!__all_sync(0xffffffffu, w_ok)) return false;
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld32_async(tmem + lane_base + col_s, sr);
        tmem_ld32_async(tmem + lane_base + col_s + 32, sr + 32);
        tmem_ld_wait();
        reg_fence<64>(sr);
        const float* lp = sm.lp[qs] + hq * 64;
        float x[64];
        const uint64_t c2 = f2(c, c);
#pragma unroll
        for (int j2 = 0; j2 < 32; ++j2) {
          const float2 l2 = *reinterpret_cast<const float2*>(lp + 2 * j2);
          f2_split(f2_fma(f2(__uint_as_float(sr[2 * j2]), __uint_as_float(sr[2 * j2 + 1])), c2, f2(-l2.x, -l2.y)),
                   x[2 * j2], x[2 * j2 + 1]);
        }
        if constexpr (decltype(masked)::value) {
          const int qbase = q0 + hq * 64;
          const int a = prm.causal ? key - qbase : (prm.window > 0 ? key - prm.window + 1 - qbase : 0);
          const int b = key >= prm.N ? a : (prm.window > 0 ? key + prm.window - qbase : 64);
#pragma unroll
          for (int wd = 0; wd < 2; ++wd) {
            const int aw = min(max(a - 32 * wd, 0), 32), bw = min(max(b - 32 * wd, 0), 32);
            const uint32_t below_b = bw >= 32 ? 0xffffffffu : ((1u << bw) - 1u);
            const uint32_t below_a = aw >= 32 ? 0xffffffffu : ((1u << aw) - 1u);
            const uint32_t bits = below_b & ~below_a;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (!((bits >> j) & 1u)) x[32 * wd + j] = -INFINITY;
          }
        }
#pragma unroll
        for (int j2 = 0; j2 < 32; ++j2) pk[j2] = pack_bf16x2(ex2_approx(x[2 * j2]), ex2_approx(x[2 * j2 + 1]));
        tmem_st16(tmem + lane_base + col_s, pk);
        tmem_st16(tmem + lane_base + col_s + 16, pk + 16);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(smem_u32(&sm.pa_full));
        return true;
      };
      auto phase_b = [&](int it) -> bool {
        const int ir = it_run + it;
        const int qs = ir % kBwdQStages;
        const bool w_ok = mbar_wait(smem_u32(&sm.dp_full), ir & 1, abort, lim);
        if (!__all_sync(0xffffffffu, w_ok)) return false;
        tc_fence_after();
        uint32_t dr[64];
        tmem_ld32_async(tmem + lane_base + col_dp, dr);
        tmem_ld32_async(tmem + lane_base + col_dp + 32, dr + 32);
        tmem_ld_wait();
        reg_fence<64>(dr);
        const float* ddp = sm.dd[qs] + hq * 64;
        uint32_t pd[32];
#pragma unroll
        for (int j2 = 0; j2 < 32; ++j2) {
          const float2 d2 = *reinterpret_cast<const float2*>(ddp + 2 * j2);
          const uint32_t wv = pk[j2];
          const uint64_t p2 = f2(__uint_as_float(wv << 16), __uint_as_float(wv & 0xffff0000u));
          const uint64_t t2 =
              f2_add(f2(__uint_as_float(dr[2 * j2]), __uint_as_float(dr[2 * j2 + 1])), f2(-d2.x, -d2.y));
          float s0, s1;
          f2_split(f2_mul(t2, p2), s0, s1);
          pd[j2] = pack_bf16x2(s0, s1);
        }
        tmem_st16(tmem + lane_base + col_dp, pd);
        tmem_st16(tmem + lane_base + col_dp + 16, pd + 16);
#pragma unroll
        for (int c16 = 0; c16 < 8; ++c16)
          st_shared_v4(ds_row + ((c16 ^ sw) << 4), pd[4 * c16], pd[4 * c16 + 1], pd[4 * c16 + 2], pd[4 * c16 + 3]);
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(smem_u32(&sm.ds_full));
        return true;
      };
      auto readout = [&](int it) -> bool {
        const int ir = it_run + it;
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.dq_full), ir & 1, abort, lim))) return false;
        tc_fence_after();
        uint32_t v[D / 2];
#pragma unroll
        for (int ch = 0; ch < D / 64; ++ch) tmem_ld32_async(tmem + lane_base + col_dq + ch * 32, v + ch * 32);
        tmem_ld_wait();
        reg_fence<D / 2>(v);
        tc_fence_before();
        mbar_arrive(smem_u32(&sm.dq_free));
#pragma unroll
        for (int ps = 0; ps < D / 64; ++ps, ++n_pass) {
          if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.st_free[warp]), (n_pass & 1) ^ 1, abort, lim)))
            return false;
#pragma unroll
          for (int c16 = 0; c16 < 8; ++c16)
            st_shared_v4(stage + lane * 128 + ((c16 ^ (lane & 7)) << 4), v[32 * ps + 4 * c16],
                         v[32 * ps + 4 * c16 + 1], v[32 * ps + 4 * c16 + 2], v[32 * ps + 4 * c16 + 3]);
          mbar_arrive(smem_u32(&sm.st_full[warp]));
        }
        return true;
      };
      auto run_a = [&](int it) -> bool {
        const int qbase = bwd_q_tile(w, prm.group, it) * kBwdRows + hq * 64;
        const bool need_mask = (prm.causal && kv0 + kBwdKeys - 1 > qbase) ||
                               (prm.window > 0 && kv0 < qbase + 64 - prm.window) || (kv0 + kBwdKeys > prm.N) ||
                               (!prm.causal && prm.window > 0 && qbase + prm.window - 1 < kv0 + kBwdKeys - 1);
        return need_mask ? phase_a(it, std::true_type{}) : phase_a(it, std::false_type{});
      };
      ok = run_a(0);
      for (int it = 0; ok && it < w.n_it; ++it) {
        if (!phase_b(it)) {
          ok = false;
          break;
        }
        if (it + 1 < w.n_it && !run_a(it + 1)) {
          ok = false;
          break;
        }
        if (!readout(it)) {
          ok = false;
          break;
        }
      }
      if (!ok) break;
      it_run += w.n_it;
      // epilogue: warps of query half 0 write dK = scale * acc, those of half 1 write dV = acc
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.mma_final), n_local & 1, abort, lim))) break;
      tc_fence_after();
      const bool in_range = key < prm.N;
      const int krow = in_range ? key : 0;
      __nv_bfloat16* dst_row = hq == 0 ? prm.dk + prm.dk_st.at(w.b_idx, w.h_kv, krow)
                                       : prm.dv + prm.dv_st.at(w.b_idx, w.h_kv, krow);
      const float mul = hq == 0 ? prm.scale : 1.f;
      const uint32_t col0 = hq == 0 ? kTdK : kTdV;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t rr[32];
        tmem_ld32(tmem + lane_base + col0 + ch * 32, rr);
        uint32_t wv[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          wv[j] = pack_bf16x2(__uint_as_float(rr[2 * j]) * mul, __uint_as_float(rr[2 * j + 1]) * mul);
        if (in_range) {
          uint4* dst = reinterpret_cast<uint4*>(dst_row + ch * 32);
#pragma unroll
          for (int j = 0; j < 4; ++j) dst[j] = make_uint4(wv[4 * j], wv[4 * j + 1], wv[4 * j + 2], wv[4 * j + 3]);
        }
      }
      // (the next item's phase A arrives on pa_full only after these TMEM reads: tc_fence_before there)
    }
  }

  if (warp >= 10) {
    // ------------------------------------------------------------------ reduction warps
    const int first = (warp - 10) * 4;
    const int hq = first / 4;
    int it_run = 0;
    int n_local = 0;
    bool ok = true;
    for (int pos; ok && (pos = persist_item(n_items, n_local)) >= 0; ++n_local) {
      const BwdItem w = bwd_item(prm, order, pos);
      for (int it = 0; ok && it < w.n_it; ++it) {
        const int ir = it_run + it;
        for (int ps = 0; ok && ps < D / 64; ++ps) {
          const int n = ir * (D / 64) + ps;
          for (int qd = 0; qd < 4 && ok; ++qd) {
            const int wq = first + qd;
            ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.st_full[wq]), n & 1, abort, lim));
            if (!ok) break;
            const uint32_t slot = smem_u32(sm.stage[wq]);
            uint4 x[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int row = 4 * j + (lane >> 3), cc = lane & 7;
              x[j] = ld_shared_v4(slot + row * 128 + ((cc ^ (row & 7)) << 4));
            }
            mbar_arrive(smem_u32(&sm.st_free[wq]));
            const int q0 = bwd_q_tile(w, prm.group, it) * kBwdRows + qd * 32;
            float* acc = prm.dq_acc + (size_t(bwd_q_head(w, prm.group, it)) * prm.Np + q0) * D + hq * (D / 2) + 32 * ps;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int row = 4 * j + (lane >> 3), cc = lane & 7;
              red_add_v4(acc + size_t(row) * D + 4 * cc, x[j]);
            }
          }
        }
        if (*abort) ok = false;
      }
      it_run += w.n_it;
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
