// Persistent form of fa_fwd256_kernel: gridDim.x CTAs (one per SM) loop over the work items
// (128-row query tiles of one head), so that one item's Q load and first S = Q K^T overlap the
// previous item's last P V and its epilogue, instead of waiting for a new CTA's launch, barrier
// setup and TMEM allocation.
//
// The per-item work is fa_fwd256_kernel's (same warps, TMEM columns, two S buffers, ring, lazy
// rescale).  What changes is bookkeeping across items:
//   * the K/V loads are numbered over the CTA's whole run (slot = L % 4), and so are the key
//     tiles (steps): step s uses S buffer s % 2, and the s_full / p_full / pv_done phases follow
//     the run's step count;
//   * q_empty, committed right after an item's last S, lets the TMA warp load the next item's Q
//     while the item's last P V still runs;
//   * o_free (128 arrivals per item, after the epilogue has read O) lets the MMA warp issue the
//     next item's first P V, which overwrites O; the softmax warps wait for o_final every item.
// Every item has at least one key tile (the query tile's own diagonal), so no role skips an
// item's handshakes.
#pragma once

#include <type_traits>

#include "fwd256_kernel.cuh"
#include "persist_sched.cuh"

namespace fa {

struct Fwd256PersistSmem {
  static constexpr uint32_t kQBytes = Fwd256Smem::kQBytes;
  static constexpr uint32_t kTileBytes = Fwd256Smem::kTileBytes;
  static constexpr uint32_t kQChunk = Fwd256Smem::kQChunk;
  static constexpr uint32_t kKvChunk = Fwd256Smem::kKvChunk;
  alignas(1024) uint8_t q[kQBytes];
  alignas(1024) uint8_t kv[k256Slots][kTileBytes];
  alignas(8) uint64_t q_full, q_empty;
  uint64_t slot_full[k256Slots], slot_empty[k256Slots];
  uint64_t s_full[2], p_full[2], pv_done, o_final, o_free, mma_drain;
  uint32_t tmem_base;
  int abort;
};

// The item at position `pos` of `order` (prm.n_pairs = query tiles per head): its head and
// query tile, the longest (last) tile of a head first.  Cost-major is tile-major over all heads.
struct Fwd256Item {
  int bh, b_idx, h_q, h_kv, q0, t_begin, t_end;
};
__device__ __forceinline__ Fwd256Item fwd256_item(const FwdParams& prm, int order, int pos) {
  Fwd256Item it;
  const int rank = order == kOrderPairMajor ? pos / prm.BH : pos % prm.n_pairs;   // 0 = the longest tile
  it.bh = order == kOrderPairMajor ? pos % prm.BH : pos / prm.n_pairs;
  it.b_idx = it.bh / prm.H;
  it.h_q = it.bh % prm.H;
  it.h_kv = it.h_q / prm.group;
  it.q0 = (prm.n_pairs - 1 - rank) * k256BlockM;
  kv_tile_range256(it.q0, prm.N, prm.causal, prm.window, it.t_begin, it.t_end);
  return it;
}

__global__ void __launch_bounds__(k256Threads, 1)
    fa_fwd256_persist_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const FwdParams prm, const int order) {
  using Smem = Fwd256PersistSmem;
  constexpr int D = kD256;
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
    for (int s = 0; s < k256Slots; ++s) {
      mbar_init(smem_u32(&sm.slot_full[s]), 1);
      mbar_init(smem_u32(&sm.slot_empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&sm.s_full[b]), 1);
      mbar_init(smem_u32(&sm.p_full[b]), k256BlockM);
    }
    mbar_init(smem_u32(&sm.pv_done), 1);
    mbar_init(smem_u32(&sm.o_final), 1);
    mbar_init(smem_u32(&sm.o_free), k256BlockM);
    mbar_init(smem_u32(&sm.mma_drain), 1);
    fence_mbar_init();
  }
  if (warp == k256WarpTma) {
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

  if (warp == k256WarpTma) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint32_t qb = smem_u32(&sm.q_full);
      int L_run = 0;   // K/V loads issued over the run: load L uses slot L % k256Slots
      int n_local = 0;
      bool ok = true;
      for (int pos; ok && (pos = persist_item(n_items, n_local)) >= 0; ++n_local) {
        const Fwd256Item w = fwd256_item(prm, order, pos);
        // the previous item's S products have read Q
        if (n_local > 0 && !mbar_wait(smem_u32(&sm.q_empty), (n_local - 1) & 1, abort, lim)) break;
        mbar_expect_tx(qb, Smem::kQBytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_rows(smem_u32(sm.q) + c * Smem::kQChunk, &tm_q, qb, c * 64, w.q0, w.h_q, w.b_idx);
        const int n_loads = 2 * (w.t_end - w.t_begin);
        for (int L = 0; L < n_loads; ++L, ++L_run) {
          const int slot = L_run % k256Slots;
          if (!mbar_wait(smem_u32(&sm.slot_empty[slot]), ((L_run / k256Slots) & 1) ^ 1, abort, lim)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&sm.slot_full[slot]);
          const int kv0 = (w.t_begin + (L >> 1)) * k256BlockN;
          const CUtensorMap* map = (L & 1) ? &tm_v : &tm_k;
          mbar_expect_tx(fb, Smem::kTileBytes);
          for (int c = 0; c < D / 64; ++c)
            tma_load_rows(smem_u32(sm.kv[slot]) + c * Smem::kKvChunk, map, fb, c * 64, kv0, w.h_kv, w.b_idx);
        }
      }
      // let every copy this CTA started land before the CTA may exit
      if (n_local > 0) mbar_wait_drain(qb, (n_local - 1) & 1, lim);
      for (int L = max(0, L_run - k256Slots); L < L_run; ++L)
        mbar_wait_drain(smem_u32(&sm.slot_full[L % k256Slots]), (L / k256Slots) & 1, lim);
    }
  } else if (warp == k256WarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    auto wait = [&](uint32_t bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, lim));
    };
    constexpr uint32_t idesc_s = idesc_bf16_f32(k256BlockM, k256BlockN, false, false);
    constexpr uint32_t idesc_o = idesc_bf16_f32(k256BlockM, D, false, true);
    const uint64_t dq = sw128_desc(smem_u32(sm.q), 16, 1024);
    const uint64_t dk0 = sw128_desc(smem_u32(sm.kv[0]), 16, 1024);
    const uint64_t dv0 = sw128_desc(smem_u32(sm.kv[0]), Smem::kKvChunk, 1024);
    auto issue_s = [&](uint32_t slot, int buf) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t qoff = (kk >> 2) * Smem::kQChunk + (kk & 3) * 32;
        const uint32_t koff = slot * Smem::kTileBytes + (kk >> 2) * Smem::kKvChunk + (kk & 3) * 32;
        mma_bf16_ss_w(tmem + 64 * buf, desc_advance(dq, qoff), desc_advance(dk0, koff), idesc_s, kk > 0);
      }
      mma_commit_w(smem_u32(&sm.s_full[buf]));
    };
    auto issue_pv = [&](uint32_t slot, int buf, bool first) {
      const uint64_t dv = desc_advance(dv0, slot * Smem::kTileBytes);
#pragma unroll
      for (int kk = 0; kk < k256BlockN / 16; ++kk)
        mma_bf16_ts_w(tmem + 256, tmem + 64 * buf + kk * 8, desc_advance(dv, kk * 2048), idesc_o,
                      (kk > 0 || !first) ? 1u : 0u);
    };
    int L_run = 0;   // K/V loads consumed over the run
    int ks = 0;      // key tiles (steps) over the run: step s uses S buffer s % 2
    int n_local = 0;
    bool ok = true;
    for (int pos; ok && (pos = persist_item(n_items, n_local)) >= 0; ++n_local) {
      const Fwd256Item w = fwd256_item(prm, order, pos);
      const int n_t = w.t_end - w.t_begin;   // >= 1
      const int L0 = L_run;                  // K of the item's first tile
      ok = wait(smem_u32(&sm.q_full), n_local & 1) && wait(smem_u32(&sm.slot_full[L0 % k256Slots]),
                                                            (L0 / k256Slots) & 1);
      if (!ok) break;
      tc_fence_after();
      issue_s(L0 % k256Slots, ks & 1);
      mma_commit_w(smem_u32(&sm.slot_empty[L0 % k256Slots]));
      if (n_t == 1) mma_commit_w(smem_u32(&sm.q_empty));   // the item's only S has been issued
      for (int k = 0; k < n_t; ++k) {
        const int s = ks + k;            // this step's run number
        const int Lv = L0 + 2 * k + 1;   // V of tile k
        const int Lk = Lv + 1;           // K of tile k + 1
        if (k + 1 < n_t) {
          // S of the next tile into the other buffer, ahead of this tile's PV
          if (!wait(smem_u32(&sm.slot_full[Lk % k256Slots]), (Lk / k256Slots) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_s(Lk % k256Slots, (s + 1) & 1);
          mma_commit_w(smem_u32(&sm.slot_empty[Lk % k256Slots]));
          if (k + 2 == n_t) mma_commit_w(smem_u32(&sm.q_empty));   // the item's last S
        }
        if (!wait(smem_u32(&sm.slot_full[Lv % k256Slots]), (Lv / k256Slots) & 1) ||
            !wait(smem_u32(&sm.p_full[s & 1]), (s >> 1) & 1)) {
          ok = false;
          break;
        }
        // the previous item's epilogue must have read O before this item's first P V
        if (k == 0 && n_local > 0 && !wait(smem_u32(&sm.o_free), (n_local - 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_pv(Lv % k256Slots, s & 1, k == 0);
        mma_commit_w(smem_u32(&sm.pv_done));
        mma_commit_w(smem_u32(&sm.slot_empty[Lv % k256Slots]));
      }
      if (!ok) break;
      L_run += 2 * n_t;
      ks += n_t;
      mma_commit_w(smem_u32(&sm.o_final));
    }
    mma_commit_w(smem_u32(&sm.mma_drain));
    mbar_wait_drain(smem_u32(&sm.mma_drain), 0, lim);
  } else {
    // ------------------------------------------------------------------ softmax warps
    const int row = threadIdx.x;   // == TMEM lane
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const uint32_t o_col = tmem + lane_base + 256;
    const float c = prm.scale_log2;
    int ks = 0;   // steps of the finished items
    int n_local = 0;
    bool ok = true;
    for (int pos; ok && (pos = persist_item(n_items, n_local)) >= 0; ++n_local) {
      const Fwd256Item w = fwd256_item(prm, order, pos);
      const int qi = w.q0 + row;
      float m = -INFINITY;
      float l = 0.f;
      auto step = [&](const int t, auto masked) -> bool {
        const int k = t - w.t_begin;
        const int s = ks + k;
        const int kv0 = t * k256BlockN;
        const int buf = s & 1;
        const uint32_t s_col = tmem + lane_base + 64 * buf;
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.s_full[buf]), (s >> 1) & 1, abort, lim))) return false;
        tc_fence_after();
        float sv[k256BlockN];
        {
          uint32_t r[k256BlockN];
#pragma unroll
          for (int ch = 0; ch < k256BlockN / 32; ++ch) tmem_ld32_async(s_col + ch * 32, r + ch * 32);
          tmem_ld_wait();
          reg_fence<k256BlockN>(r);
#pragma unroll
          for (int j = 0; j < k256BlockN; ++j) sv[j] = __uint_as_float(r[j]);
        }
        if constexpr (decltype(masked)::value) {
          const int hi = prm.causal ? min(qi, prm.N - 1)
                                    : (prm.window > 0 ? min(qi + prm.window - 1, prm.N - 1) : prm.N - 1);
          const int lo = prm.window > 0 ? qi - prm.window + 1 : 0;
          const int a = lo - kv0, b = hi - kv0 + 1;
#pragma unroll
          for (int wd = 0; wd < k256BlockN / 32; ++wd) {
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
        for (int j = 16; j < k256BlockN; j += 16)
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
        for (int ch = 0; ch < k256BlockN / 32; ++ch) {
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
          // P V of this item's previous step (run step s - 1) must be done before O is touched
          if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.pv_done), (s - 1) & 1, abort, lim))) return false;
          tc_fence_after();
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
        mbar_arrive(smem_u32(&sm.p_full[buf]));
        return true;
      };
      const int band_lo_max = prm.window > 0 ? w.q0 + k256BlockM - prm.window : 0;
      const int band_hi_min =
          min(prm.N - 1, prm.causal ? w.q0 : (prm.window > 0 ? w.q0 + prm.window - 1 : prm.N - 1));
      for (int t = w.t_begin; t < w.t_end; ++t) {
        const int kv0 = t * k256BlockN;
        const bool need_mask = kv0 < band_lo_max || kv0 + k256BlockN - 1 > band_hi_min;
        ok = need_mask ? step(t, std::true_type{}) : step(t, std::false_type{});
        if (!ok) break;
      }
      if (!ok) break;
      ks += w.t_end - w.t_begin;
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.o_final), n_local & 1, abort, lim))) break;
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool in_range = qi < prm.N;
      __nv_bfloat16* orow = prm.o + prm.o_st.at(w.b_idx, w.h_q, in_range ? qi : 0);
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
      if (in_range) prm.lse[size_t(w.bh) * prm.N + qi] = (m + lg2_approx(l)) * 0.69314718055994531f;
      tc_fence_before();
      mbar_arrive(smem_u32(&sm.o_free));   // O has been read: the next item's first P V may overwrite it
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == k256WarpTma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace fa
