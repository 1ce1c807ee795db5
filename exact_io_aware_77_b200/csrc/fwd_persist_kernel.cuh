// Persistent form of fa_fwd_kernel: one CTA per SM loops over the work items (pairs of query
// tiles of one head), so that an item's Q load and first S = Q K^T overlap the previous item's
// epilogue instead of waiting for a new CTA's launch, barrier setup and TMEM allocation.
//
// The per-item work is fa_fwd_kernel's (same warps, TMEM columns, ring, lazy rescale and
// masked / unmasked tile bodies).  What changes is bookkeeping across items:
//   * every barrier keeps its phase across items: loads are numbered over the CTA's whole run
//     (slot = L % 4), S commits and P arrivals are counted per query tile over the run;
//   * q_empty (committed after an item's last S) lets the TMA warp load the next item's Q;
//   * o_free[w] (128 arrivals per item, after the epilogue has read O_w) lets the MMA warp start
//     the next item's P V for tile w, whose first k-step overwrites O_w;
//   * o_final[w] is committed once per item after its last P V for tile w, and the softmax warps
//     of tile w wait for it every item, even one in which tile w has no keys: otherwise they could
//     arrive on o_free[w] two phases ahead of the MMA warp's wait, which a parity wait cannot tell
//     from the phase it wants.
// MMAs from one thread still run in order, so within an item the rescale and P/S reuse
// arguments of fa_fwd_kernel hold unchanged.
#pragma once

#include <type_traits>

#include "fwd_kernel.cuh"
#include "persist_sched.cuh"

namespace fa {

template <int D>
struct FwdPersistSmem {
  static constexpr int kChunks = D / 64;
  static constexpr uint32_t kTileBytes = kBlockN * D * 2;
  alignas(1024) uint8_t q[kQTiles][kTileBytes];
  alignas(1024) uint8_t kv[kSlots][kTileBytes];
  alignas(8) uint64_t q_full, q_empty;
  uint64_t slot_full[kSlots], slot_empty[kSlots];
  uint64_t s_full[kQTiles], p_full[kQTiles], o_final[kQTiles], o_free[kQTiles];
  uint64_t mma_drain;
  uint32_t tmem_base;
  int abort;
};

// The item at position `pos` of `order`: its head, first query row and the K/V tile ranges of
// its two query tiles.  Within a head, the longest (last) pair comes first.
struct FwdItem {
  int bh, b_idx, h_q, h_kv, q0, b0, e0, b1, e1, t_begin, t_end;
};
__device__ __forceinline__ FwdItem fwd_item(const FwdParams& prm, int order, int pos) {
  FwdItem it;
  const int rank = order == kOrderPairMajor ? pos / prm.BH : pos % prm.n_pairs;   // 0 = the longest pair
  it.bh = order == kOrderPairMajor ? pos % prm.BH : pos / prm.n_pairs;
  it.b_idx = it.bh / prm.H;
  it.h_q = it.bh % prm.H;
  it.h_kv = it.h_q / prm.group;
  const int pair = prm.n_pairs - 1 - rank;
  it.q0 = pair * (kQTiles * kBlockM);
  kv_tile_range(it.q0, prm.N, prm.causal, prm.window, it.b0, it.e0);
  kv_tile_range(it.q0 + kBlockM, prm.N, prm.causal, prm.window, it.b1, it.e1);
  if (it.e1 == 0) it.b1 = it.e1 = it.b0;
  it.t_begin = it.b0;
  it.t_end = max(it.e0, it.e1);
  return it;
}

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fa_fwd_persist_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const FwdParams prm, const int order) {
  using Smem = FwdPersistSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_items = prm.n_pairs * prm.BH;
  volatile int* abort = &sm.abort;
  const uint64_t lim = prm.wait_limit_ns;

  if (threadIdx.x == 0) {
    sm.abort = 0;
    mbar_init(smem_u32(&sm.q_full), 1);
    mbar_init(smem_u32(&sm.q_empty), 1);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(smem_u32(&sm.slot_full[s]), 1);
      mbar_init(smem_u32(&sm.slot_empty[s]), 1);
    }
    for (int w = 0; w < kQTiles; ++w) {
      mbar_init(smem_u32(&sm.s_full[w]), 1);
      mbar_init(smem_u32(&sm.p_full[w]), kBlockM);
      mbar_init(smem_u32(&sm.o_final[w]), 1);
      mbar_init(smem_u32(&sm.o_free[w]), kBlockM);
    }
    mbar_init(smem_u32(&sm.mma_drain), 1);
    fence_mbar_init();
  }
  if (warp == kWarpTma) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    __syncwarp();
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
      int L_run = 0;   // loads issued over the whole run: load L uses slot L % kSlots
      int n_local = 0;
      bool ok = true;
      for (int pos; ok && (pos = persist_item(n_items, n_local)) >= 0; ++n_local) {
        const FwdItem w_it = fwd_item(prm, order, pos);
        // the previous item's S products have read Q
        if (n_local > 0 && !mbar_wait(smem_u32(&sm.q_empty), (n_local - 1) & 1, abort, lim)) break;
        mbar_expect_tx(qb, kQTiles * Smem::kTileBytes);
        for (int w = 0; w < kQTiles; ++w)
          for (int c = 0; c < Smem::kChunks; ++c)
            tma_load_rows(smem_u32(sm.q[w]) + c * 16384, &tm_q, qb, c * 64, w_it.q0 + w * kBlockM, w_it.h_q,
                          w_it.b_idx);
        const int n_loads = 2 * (w_it.t_end - w_it.t_begin);
        for (int L = 0; L < n_loads; ++L, ++L_run) {
          const int slot = L_run % kSlots;
          if (!mbar_wait(smem_u32(&sm.slot_empty[slot]), ((L_run / kSlots) & 1) ^ 1, abort, lim)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&sm.slot_full[slot]);
          const int kv0 = (w_it.t_begin + (L >> 1)) * kBlockN;
          const CUtensorMap* map = (L & 1) ? &tm_v : &tm_k;
          mbar_expect_tx(fb, Smem::kTileBytes);
          for (int c = 0; c < Smem::kChunks; ++c)
            tma_load_rows(smem_u32(sm.kv[slot]) + c * 16384, map, fb, c * 64, kv0, w_it.h_kv, w_it.b_idx);
        }
      }
      // let every copy this CTA started land before the CTA may exit
      if (n_local > 0) mbar_wait_drain(qb, (n_local - 1) & 1, lim);
      for (int L = max(0, L_run - kSlots); L < L_run; ++L)
        mbar_wait_drain(smem_u32(&sm.slot_full[L % kSlots]), (L / kSlots) & 1, lim);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    auto wait = [&](uint32_t bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, lim));
    };
    constexpr uint32_t idesc_s = idesc_bf16_f32(kBlockM, kBlockN, false, false);
    constexpr uint32_t idesc_o = idesc_bf16_f32(kBlockM, D, false, true);
    const uint64_t dq[2] = {sw128_desc(smem_u32(sm.q[0]), 16, 1024), sw128_desc(smem_u32(sm.q[1]), 16, 1024)};
    const uint64_t dkv0 = sw128_desc(smem_u32(sm.kv[0]), 16, 1024);
    const uint64_t dv0 = sw128_desc(smem_u32(sm.kv[0]), 16384, 1024);
    int pv_run[2] = {0, 0};   // P V products over the run (p_full parity)
    int L_run = 0;
    int n_local = 0;
    bool ok = true;
    for (int pos; ok && (pos = persist_item(n_items, n_local)) >= 0; ++n_local) {
      const FwdItem w_it = fwd_item(prm, order, pos);
      const int bw[2] = {w_it.b0, w_it.b1}, ew[2] = {w_it.e0, w_it.e1};
      auto active = [&](int w, int t) { return t >= bw[w] && t < ew[w]; };
      int pv_item[2] = {0, 0};   // this item's P V products per tile (the first overwrites O)
      auto issue_s = [&](int w, uint32_t slot) {
        const uint64_t dk = desc_advance(dkv0, slot * Smem::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss_w(tmem + w * 128, desc_advance(dq[w], off), desc_advance(dk, off), idesc_s, kk > 0);
        }
        mma_commit_w(smem_u32(&sm.s_full[w]));
      };
      auto issue_pv = [&](int w, uint32_t slot) {
        const uint64_t dv = desc_advance(dv0, slot * Smem::kTileBytes);
        const uint32_t acc = pv_item[w] > 0;
#pragma unroll
        for (int kk = 0; kk < kBlockN / 16; ++kk)
          mma_bf16_ts_w(tmem + 256 + w * 128, tmem + w * 128 + kk * 8, desc_advance(dv, kk * 2048), idesc_o,
                        kk > 0 ? 1u : acc);
        ++pv_item[w];
        ++pv_run[w];
      };
      if (!wait(smem_u32(&sm.q_full), n_local & 1)) break;
      const int L0 = L_run;   // K of the item's first tile
      if (!wait(smem_u32(&sm.slot_full[L0 % kSlots]), (L0 / kSlots) & 1)) break;
      tc_fence_after();
#pragma unroll
      for (int w = 0; w < kQTiles; ++w)
        if (active(w, w_it.t_begin)) issue_s(w, L0 % kSlots);
      mma_commit_w(smem_u32(&sm.slot_empty[L0 % kSlots]));
      for (int t = w_it.t_begin; ok && t < w_it.t_end; ++t) {
        const int Lv = L0 + 2 * (t - w_it.t_begin) + 1;
        const int Lk = Lv + 1;
        const bool has_next = t + 1 < w_it.t_end;
        if (!wait(smem_u32(&sm.slot_full[Lv % kSlots]), (Lv / kSlots) & 1)) {
          ok = false;
          break;
        }
        if (has_next && !wait(smem_u32(&sm.slot_full[Lk % kSlots]), (Lk / kSlots) & 1)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int w = 0; w < kQTiles; ++w) {
          if (active(w, t)) {
            if (!wait(smem_u32(&sm.p_full[w]), pv_run[w] & 1)) {
              ok = false;
              break;
            }
            // the previous item's epilogue must have read O_w before this item's first P V
            if (pv_item[w] == 0 && n_local > 0 && !wait(smem_u32(&sm.o_free[w]), (n_local - 1) & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_pv(w, Lv % kSlots);
          }
          if (has_next && active(w, t + 1)) issue_s(w, Lk % kSlots);
        }
        if (!ok) break;
        if (has_next) mma_commit_w(smem_u32(&sm.slot_empty[Lk % kSlots]));
        mma_commit_w(smem_u32(&sm.slot_empty[Lv % kSlots]));
      }
      if (!ok) break;
      L_run += 2 * (w_it.t_end - w_it.t_begin);
      mma_commit_w(smem_u32(&sm.q_empty));   // every S of the item has been issued: Q may be reloaded
#pragma unroll
      for (int w = 0; w < kQTiles; ++w) {
        // a tile with no keys in this item still gets its O_w handshake from the previous item
        if (pv_item[w] == 0 && n_local > 0 && !wait(smem_u32(&sm.o_free[w]), (n_local - 1) & 1)) {
          ok = false;
          break;
        }
        mma_commit_w(smem_u32(&sm.o_final[w]));
      }
    }
    mma_commit_w(smem_u32(&sm.mma_drain));
    mbar_wait_drain(smem_u32(&sm.mma_drain), 0, lim);
  } else {
    // ------------------------------------------------------------------ softmax warpgroups
    const int w = warp >> 2;
    const int row = threadIdx.x & 127;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t s_col = tmem + lane_base + w * 128;
    const uint32_t o_col = tmem + lane_base + 256 + w * 128;
    const float c = prm.scale_log2;
    int s_run = 0;   // S tiles of this query tile consumed over the run (s_full parity)
    int n_local = 0;
    bool ok = true;
    for (int pos; ok && (pos = persist_item(n_items, n_local)) >= 0; ++n_local) {
      const FwdItem w_it = fwd_item(prm, order, pos);
      const int qw0 = w_it.q0 + w * kBlockM;
      const int qi = qw0 + row;
      const int tb = w == 0 ? w_it.b0 : w_it.b1;
      const int te = w == 0 ? w_it.e0 : w_it.e1;
      float m = -INFINITY;
      float l = 0.f;
      auto step = [&](const int t, auto masked) -> bool {
        const int k = t - tb;
        const int kv0 = t * kBlockN;
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.s_full[w]), s_run & 1, abort, lim))) return false;
        ++s_run;
        tc_fence_after();
        float sv[kBlockN];
        {
          uint32_t r[kBlockN];
#pragma unroll
          for (int ch = 0; ch < kBlockN / 32; ++ch) tmem_ld32_async(s_col + ch * 32, r + ch * 32);
          tmem_ld_wait();
          reg_fence<kBlockN>(r);
#pragma unroll
          for (int j = 0; j < kBlockN; ++j) sv[j] = __uint_as_float(r[j]);
        }
        if constexpr (decltype(masked)::value) {
          const int hi = prm.causal ? min(qi, prm.N - 1)
                                    : (prm.window > 0 ? min(qi + prm.window - 1, prm.N - 1) : prm.N - 1);
          const int lo = prm.window > 0 ? qi - prm.window + 1 : 0;
          const int a = lo - kv0, b = hi - kv0 + 1;
#pragma unroll
          for (int wd = 0; wd < kBlockN / 32; ++wd) {
            const int aw = min(max(a - 32 * wd, 0), 32), bw = min(max(b - 32 * wd, 0), 32);
            const uint32_t below_b = bw >= 32 ? 0xffffffffu : ((1u << bw) - 1u);
            const uint32_t below_a = aw >= 32 ? 0xffffffffu : ((1u << aw) - 1u);
            const uint32_t bits = below_b & ~below_a;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (!((bits >> j) & 1u)) sv[32 * wd + j] = -INFINITY;
          }
        }
        float mx16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) mx16[i] = sv[i];
#pragma unroll
        for (int j = 16; j < kBlockN; j += 16)
#pragma unroll
          for (int i = 0; i < 16; ++i) mx16[i] = fmaxf(mx16[i], sv[j + i]);
#pragma unroll
        for (int i = 0; i < 8; ++i) mx16[i] = fmaxf(mx16[i], mx16[i + 8]);
        const float mx = max3f(max3f(mx16[0], mx16[1], mx16[2]), max3f(mx16[3], mx16[4], mx16[5]),
                               fmaxf(mx16[6], mx16[7]));
        const float m_cand = fmaxf(m, mx * c);
        const bool grow = m_cand > m + kRescaleThreshold;
        const float m_new = grow ? m_cand : m;
        const float alpha = grow ? ex2_approx(m - m_new) : 1.f;
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        const uint64_t c2 = f2(c, c), nm2 = f2(-m_use, -m_use);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int ch = 0; ch < kBlockN / 32; ++ch) {
          uint32_t pk[16];
#pragma unroll
          for (int jp = 0; jp < 16; ++jp) {
            const int j = ch * 32 + 2 * jp;
            const uint64_t x = f2_fma(f2(sv[j], sv[j + 1]), c2, nm2);
            float p0, p1;
            if (jp < kEmuPairs) {
              exp2_poly_x2(x, p0, p1);
            } else {
              float x0, x1;
              f2_split(x, x0, x1);
              p0 = ex2_approx(x0);
              p1 = ex2_approx(x1);
            }
            acc[jp & 3] = f2_add(acc[jp & 3], f2(p0, p1));
            pk[jp] = pack_bf16x2(p0, p1);
          }
          tmem_st16(s_col + ch * 16, pk);
        }
        float sum;
        {
          const uint64_t a2 = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
          float lo2, hi2;
          f2_split(a2, lo2, hi2);
          sum = lo2 + hi2;
        }
        l = l * alpha + sum;
        m = m_new;
        if (k > 0 && __any_sync(0xffffffffu, grow)) {
          // PV of the previous tile of this item completed before this S did (in-order MMAs)
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t r[32];
            tmem_ld32(o_col + ch * 32, r);
#pragma unroll
            for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * alpha);
            tmem_st32(o_col + ch * 32, r);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(smem_u32(&sm.p_full[w]));
        return true;
      };
      const int band_lo_max = prm.window > 0 ? qw0 + kBlockM - prm.window : 0;
      const int band_hi_min =
          min(prm.N - 1, prm.causal ? qw0 : (prm.window > 0 ? qw0 + prm.window - 1 : prm.N - 1));
      for (int t = tb; t < te; ++t) {
        const int kv0 = t * kBlockN;
        const bool need_mask = kv0 < band_lo_max || kv0 + kBlockN - 1 > band_hi_min;
        ok = need_mask ? step(t, std::true_type{}) : step(t, std::false_type{});
        if (!ok) break;
      }
      if (!ok) break;
      // every item's o_final[w] (committed after the MMA warp's wait on the previous o_free[w])
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.o_final[w]), n_local & 1, abort, lim))) break;
      if (te > tb) {
        tc_fence_after();
        const float inv_l = 1.f / l;
        const bool in_range = qi < prm.N;
        __nv_bfloat16* orow = prm.o + prm.o_st.at(w_it.b_idx, w_it.h_q, in_range ? qi : 0);
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t r[32];
          tmem_ld32(o_col + ch * 32, r);
          uint32_t wv[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            wv[j] = pack_bf16x2(__uint_as_float(r[2 * j]) * inv_l, __uint_as_float(r[2 * j + 1]) * inv_l);
          if (in_range) {
            uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[j] = make_uint4(wv[4 * j], wv[4 * j + 1], wv[4 * j + 2], wv[4 * j + 3]);
          }
        }
        if (in_range) prm.lse[size_t(w_it.bh) * prm.N + qi] = (m + lg2_approx(l)) * 0.69314718055994531f;
        tc_fence_before();
      }
      // O_w has been read (or was not used): the next item's P V may overwrite it
      mbar_arrive(smem_u32(&sm.o_free[w]));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpTma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace fa
