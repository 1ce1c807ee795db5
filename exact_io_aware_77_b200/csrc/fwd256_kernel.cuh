// Forward pass of exact attention at head dimension 256: the same method and results as
// fa_fwd_kernel (fwd_kernel.cuh), with a tile plan that fits d = 256.
//
// At d = 256 the two-query-tile plan of fa_fwd_kernel does not fit: its TMEM would hold two S
// tiles and two 256-column O accumulators (768 of 512 columns), and 128-key K/V tiles of 64 KB
// leave no room for a ring next to two Q tiles.  Here:
//   one CTA per 128-row query tile of one head (192 threads);
//   K/V tiles of 64 keys (32 KB), four of them in the shared-memory ring next to Q (64 KB);
//   TMEM: two S buffers, S_0 [0, 64) and S_1 [64, 128) (P over the first 32 columns of its S
//   as bf16 pairs), O [256, 512).  Tile j uses S_(j % 2).
//   warp 4      TMA producer and TMEM owner: Q once, then K_j, V_j through the ring.
//   warp 5      MMA issuer, per tile j: S(j+1) = Q K_{j+1}^T into the other buffer first
//               (16 k-steps, N = 64), so that it runs while the softmax works on S(j); then,
//               once P(j) is in TMEM, O += P(j) V_j (4 k-steps of 16 keys, N = 256).  MMAs from
//               one thread run in order, so S(j+1) overwrites S_(j+1 % 2) only after PV(j-1) has
//               read the P that was there.
//   warps 0-3   softmax: thread t owns row t (TMEM lane t), as in fa_fwd_kernel: running max
//               (updated lazily, O rescaled only when it grows by more than 2^8), running sum,
//               P = 2^(S c - m) to bf16 into TMEM, and at the end O / l and L.  Since S(j+1)
//               is issued before PV(j), S(j+1) completing no longer implies PV(j) completed: a
//               tile that rescales O first waits for the previous PV (pv_done).
// With one query tile per CTA the two S buffers take the place of fa_fwd_kernel's ping-pong
// between two query tiles: the tensor pipe computes S(j+1) during softmax(j) and PV(j) during
// softmax(j+1).
#pragma once

#include <type_traits>

#include "fwd_kernel.cuh"

namespace fa {

constexpr int kD256 = 256;
constexpr int k256BlockM = 128;   // query rows per CTA (one per TMEM lane)
constexpr int k256BlockN = 64;    // keys per K/V tile
constexpr int k256Slots = 4;      // ring slots (K and V alternate)
constexpr int k256Threads = 192;
constexpr int k256WarpTma = 4;
constexpr int k256WarpMma = 5;

struct Fwd256Smem {
  static constexpr uint32_t kQBytes = k256BlockM * kD256 * 2;   // 4 chunks of 128 rows x 128 B
  static constexpr uint32_t kTileBytes = k256BlockN * kD256 * 2;  // 4 chunks of 64 rows x 128 B
  static constexpr uint32_t kQChunk = k256BlockM * 128;
  static constexpr uint32_t kKvChunk = k256BlockN * 128;
  alignas(1024) uint8_t q[kQBytes];
  alignas(1024) uint8_t kv[k256Slots][kTileBytes];
  alignas(8) uint64_t q_full;
  uint64_t slot_full[k256Slots], slot_empty[k256Slots];
  uint64_t s_full[2], p_full[2], pv_done, o_final, mma_drain;
  uint32_t tmem_base;
  int abort;
};

// K/V tiles [t_begin, t_end) of 64 keys that the query tile starting at q0 needs.
__device__ __forceinline__ void kv_tile_range256(int q0, int N, int causal, int window, int& t_begin, int& t_end) {
  const int kv_end = causal ? min(N, q0 + k256BlockM)
                            : (window > 0 ? min(N, q0 + k256BlockM - 1 + window) : N);
  t_end = (kv_end + k256BlockN - 1) / k256BlockN;
  const int kv_begin = window > 0 ? max(0, q0 - window + 1) : 0;
  t_begin = kv_begin / k256BlockN;
}

// prm.n_pairs holds the number of 128-row query tiles per head here.
__global__ void __launch_bounds__(k256Threads, 1)
    fa_fwd256_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const FwdParams prm) {
  using Smem = Fwd256Smem;
  constexpr int D = kD256;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_tiles = prm.n_pairs;
  int bh, rank;
  grid_item(int(blockIdx.x), prm.BH, n_tiles, kFwdChunkHeads, bh, rank);
  const int b_idx = bh / prm.H, h_q = bh % prm.H, h_kv = h_q / prm.group;
  const int q0 = (n_tiles - 1 - rank) * k256BlockM;   // longest causal tiles of the chunk first
  int t_begin, t_end;
  kv_tile_range256(q0, prm.N, prm.causal, prm.window, t_begin, t_end);
  volatile int* abort = &sm.abort;
  const uint64_t lim = prm.wait_limit_ns;

  if (threadIdx.x == 0) {
    sm.abort = 0;
    mbar_init(smem_u32(&sm.q_full), 1);
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
      mbar_expect_tx(qb, Smem::kQBytes);
      for (int c = 0; c < D / 64; ++c) tma_load_rows(smem_u32(sm.q) + c * Smem::kQChunk, &tm_q, qb, c * 64, q0, h_q, b_idx);
      int issued = 0;
      const int n_loads = 2 * (t_end - t_begin);
      for (int L = 0; L < n_loads; ++L) {
        const int slot = L % k256Slots;
        if (!mbar_wait(smem_u32(&sm.slot_empty[slot]), ((L / k256Slots) & 1) ^ 1, abort, lim)) break;
        const uint32_t fb = smem_u32(&sm.slot_full[slot]);
        const int kv0 = (t_begin + (L >> 1)) * k256BlockN;
        const CUtensorMap* map = (L & 1) ? &tm_v : &tm_k;
        mbar_expect_tx(fb, Smem::kTileBytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_rows(smem_u32(sm.kv[slot]) + c * Smem::kKvChunk, map, fb, c * 64, kv0, h_kv, b_idx);
        issued = L + 1;
      }
      mbar_wait_drain(qb, 0, lim);
      for (int L = max(0, issued - k256Slots); L < issued; ++L)
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
    // V as the MN-major B operand: 64 head-dim columns per 128-byte row, the next 64 columns
    // one 8 KB chunk further (LBO), 8 keys per 1024-byte atom (SBO)
    const uint64_t dv0 = sw128_desc(smem_u32(sm.kv[0]), Smem::kKvChunk, 1024);
    int pv_count = 0;
    auto issue_s = [&](uint32_t slot, int buf) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        // 16-element k-steps are 32 bytes apart inside a 128-byte row; 64-element chunks are
        // separate 16 KB (Q) or 8 KB (K) blocks
        const uint32_t qoff = (kk >> 2) * Smem::kQChunk + (kk & 3) * 32;
        const uint32_t koff = slot * Smem::kTileBytes + (kk >> 2) * Smem::kKvChunk + (kk & 3) * 32;
        mma_bf16_ss_w(tmem + 64 * buf, desc_advance(dq, qoff), desc_advance(dk0, koff), idesc_s, kk > 0);
      }
      mma_commit_w(smem_u32(&sm.s_full[buf]));
    };
    auto issue_pv = [&](uint32_t slot, int buf) {
      const uint64_t dv = desc_advance(dv0, slot * Smem::kTileBytes);
      const uint32_t acc = pv_count > 0;
#pragma unroll
      for (int kk = 0; kk < k256BlockN / 16; ++kk)
        mma_bf16_ts_w(tmem + 256, tmem + 64 * buf + kk * 8, desc_advance(dv, kk * 2048), idesc_o, kk > 0 ? 1u : acc);
      ++pv_count;
    };
    bool ok = t_end > t_begin && wait(smem_u32(&sm.q_full), 0);
    if (ok) {
      ok = wait(smem_u32(&sm.slot_full[0]), 0);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        mma_commit_w(smem_u32(&sm.slot_empty[0]));
      }
    }
    for (int t = t_begin; ok && t < t_end; ++t) {
      const int k = t - t_begin;
      const int Lv = 2 * k + 1;   // V of tile t
      const int Lk = Lv + 1;      // K of tile t + 1
      if (t + 1 < t_end) {
        // S of the next tile into the other buffer, ahead of this tile's PV
        if (!wait(smem_u32(&sm.slot_full[Lk % k256Slots]), (Lk / k256Slots) & 1)) break;
        tc_fence_after();
        issue_s(Lk % k256Slots, (k + 1) & 1);
        mma_commit_w(smem_u32(&sm.slot_empty[Lk % k256Slots]));
      }
      if (!wait(smem_u32(&sm.slot_full[Lv % k256Slots]), (Lv / k256Slots) & 1)) break;
      if (!wait(smem_u32(&sm.p_full[k & 1]), (k >> 1) & 1)) break;
      tc_fence_after();
      issue_pv(Lv % k256Slots, k & 1);
      mma_commit_w(smem_u32(&sm.pv_done));
      mma_commit_w(smem_u32(&sm.slot_empty[Lv % k256Slots]));
    }
    mma_commit_w(smem_u32(&sm.o_final));
    mma_commit_w(smem_u32(&sm.mma_drain));
    mbar_wait_drain(smem_u32(&sm.mma_drain), 0, lim);
  } else {
    // ------------------------------------------------------------------ softmax warps
    const int row = threadIdx.x;   // == TMEM lane
    const int qi = q0 + row;
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const uint32_t o_col = tmem + lane_base + 256;
    const float c = prm.scale_log2;
    bool ok = true;
    float m = -INFINITY;
    float l = 0.f;
    auto step = [&](const int t, auto masked) -> bool {
      const int k = t - t_begin;
      const int kv0 = t * k256BlockN;
      const int buf = k & 1;
      const uint32_t s_col = tmem + lane_base + 64 * buf;
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.s_full[buf]), (k >> 1) & 1, abort, lim))) return false;
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
        tmem_st16(s_col + ch * 16, pk);   // P over the S columns already read
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
        // S(k) was issued before PV(k-1), so wait for PV(k-1) before touching O (S(k) completing
        // does imply PV(k-2) completed, so the phase of parity (k-1) & 1 is the right one)
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.pv_done), (k - 1) & 1, abort, lim))) return false;
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
    const int band_lo_max = prm.window > 0 ? q0 + k256BlockM - prm.window : 0;
    const int band_hi_min = min(prm.N - 1, prm.causal ? q0 : (prm.window > 0 ? q0 + prm.window - 1 : prm.N - 1));
    for (int t = t_begin; t < t_end; ++t) {
      const int kv0 = t * k256BlockN;
      const bool need_mask = kv0 < band_lo_max || kv0 + k256BlockN - 1 > band_hi_min;
      ok = need_mask ? step(t, std::true_type{}) : step(t, std::false_type{});
      if (!ok) break;
    }
    if (ok && t_end > t_begin && __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.o_final), 0, abort, lim))) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool in_range = qi < prm.N;
      __nv_bfloat16* orow = prm.o + prm.o_st.at(b_idx, h_q, in_range ? qi : 0);
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
      if (in_range) prm.lse[size_t(bh) * prm.N + qi] = (m + lg2_approx(l)) * 0.69314718055994531f;
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
