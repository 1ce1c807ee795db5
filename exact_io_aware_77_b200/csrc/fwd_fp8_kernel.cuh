// Forward pass of exact attention with FP8 (E4M3) Q, K and V and one scale per tensor:
//   Q = s_q E4M3(Q8), K = s_k E4M3(K8), V = s_v E4M3(V8),
//   O = softmax(scale Q K^T + mask) V,  L = row logsumexp,
// the FP8 forward the pages attribute to FlashAttention-3 (FlashAttention (NL), "Evolutie en
// verdere ontwikkelingen").  d = 128.
//
// The same CTA plan as fa_fwd_kernel (two 128-row query tiles per CTA in ping-pong, 128-key K/V
// tiles through a 4-slot ring, S and O in TMEM, lazy rescale), with both products on the
// kind::f8f6f4 tensor-core path (E4M3 x E4M3 -> fp32, 32 elements per k-step):
//   S = Q8 K8^T      A = Q8 [query][d], B = K8 [key][d], both K-major (a 128-byte row holds all
//                    128 head-dim codes); s_q s_k is folded into the softmax scale.
//   O += P8 V8       A = P8 [query][key] K-major, written to shared memory by the softmax warps
//                    as E4M3 codes of P (P <= 2^8 under the lazy rescale, inside E4M3's range);
//                    B = V8^T [d][key] K-major: V is taken transposed, [B, H_kv, d, N], so that
//                    both operands of the 8-bit product are K-major.  s_v multiplies O / l.
// l sums the fp32 P, so O carries the E4M3 rounding of P (relative 2^-4 per weight).
#pragma once

#include <type_traits>

#include "fwd_kernel.cuh"
#include "fp8_ops.cuh"

namespace fa {

constexpr int kF8D = 128;

// Instruction descriptor for kind::f8f6f4 with E4M3 A and B (type code 0), fp32 D, both
// operands K-major: bits 4-5 D format (1 = f32), 7-9 / 10-12 A / B type, 17-22 N >> 3, 24-28 M >> 4.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

struct FwdFp8Smem {
  static constexpr uint32_t kTileBytes = 128 * kF8D;   // 128 rows of 128 one-byte codes
  alignas(1024) uint8_t q[kQTiles][kTileBytes];
  alignas(1024) uint8_t kv[kSlots][kTileBytes];          // K8 tiles [key][d], V8^T tiles [d][key]
  alignas(1024) uint8_t p[kQTiles][kTileBytes];          // P8 [query][key] per query tile
  alignas(8) uint64_t q_full;
  uint64_t slot_full[kSlots], slot_empty[kSlots];
  uint64_t s_full[kQTiles], p_full[kQTiles], o_final[kQTiles];
  uint64_t mma_drain;
  uint32_t tmem_base;
  int abort;
};

// prm.scale_log2 = scale * s_q * s_k * log2(e); v_scale = s_v.
__global__ void __launch_bounds__(kFwdThreads, 1)
    fa_fwd_fp8_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_vt, const FwdParams prm, const float v_scale) {
  using Smem = FwdFp8Smem;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  int bh, rank;
  grid_item(int(blockIdx.x), prm.BH, prm.n_pairs, kFwdChunkHeads, bh, rank);
  const int b_idx = bh / prm.H, h_q = bh % prm.H, h_kv = h_q / prm.group;
  const int pair = prm.n_pairs - 1 - rank;
  const int q0 = pair * (kQTiles * kBlockM);
  int b0, e0, b1, e1;
  kv_tile_range(q0, prm.N, prm.causal, prm.window, b0, e0);
  kv_tile_range(q0 + kBlockM, prm.N, prm.causal, prm.window, b1, e1);
  if (e1 == 0) b1 = e1 = b0;
  const int t_begin = b0;
  const int t_end = max(e0, e1);
  volatile int* abort = &sm.abort;
  const uint64_t lim = prm.wait_limit_ns;

  if (threadIdx.x == 0) {
    sm.abort = 0;
    mbar_init(smem_u32(&sm.q_full), 1);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(smem_u32(&sm.slot_full[s]), 1);
      mbar_init(smem_u32(&sm.slot_empty[s]), 1);
    }
    for (int w = 0; w < kQTiles; ++w) {
      mbar_init(smem_u32(&sm.s_full[w]), 1);
      mbar_init(smem_u32(&sm.p_full[w]), kBlockM);
      mbar_init(smem_u32(&sm.o_final[w]), 1);
    }
    mbar_init(smem_u32(&sm.mma_drain), 1);
    fence_mbar_init();
  }
  if (warp == kWarpTma) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_vt);
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
      mbar_expect_tx(qb, kQTiles * Smem::kTileBytes);
      for (int w = 0; w < kQTiles; ++w) tma_load_rows(smem_u32(sm.q[w]), &tm_q, qb, 0, q0 + w * kBlockM, h_q, b_idx);
      int issued = 0;
      const int n_loads = 2 * (t_end - t_begin);
      for (int L = 0; L < n_loads; ++L) {
        const int slot = L % kSlots;
        if (!mbar_wait(smem_u32(&sm.slot_empty[slot]), ((L / kSlots) & 1) ^ 1, abort, lim)) break;
        const uint32_t fb = smem_u32(&sm.slot_full[slot]);
        const int kv0 = (t_begin + (L >> 1)) * kBlockN;
        mbar_expect_tx(fb, Smem::kTileBytes);
        if (L & 1)   // V8^T: x = key, rows = head-dim columns
          tma_load_rows(smem_u32(sm.kv[slot]), &tm_vt, fb, kv0, 0, h_kv, b_idx);
        else         // K8: x = head-dim column, rows = keys
          tma_load_rows(smem_u32(sm.kv[slot]), &tm_k, fb, 0, kv0, h_kv, b_idx);
        issued = L + 1;
      }
      mbar_wait_drain(qb, 0, lim);
      for (int L = max(0, issued - kSlots); L < issued; ++L)
        mbar_wait_drain(smem_u32(&sm.slot_full[L % kSlots]), (L / kSlots) & 1, lim);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    auto wait = [&](uint32_t bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, lim));
    };
    constexpr uint32_t idesc = idesc_e4m3_f32(kBlockM, kBlockN);   // S (N = keys) and O (N = d): both 128
    const int bw[2] = {b0, b1}, ew[2] = {e0, e1};
    auto active = [&](int w, int t) { return t >= bw[w] && t < ew[w]; };
    int pv_count[2] = {0, 0};
    bool o_done[2] = {false, false};   // o_final committed (right after the tile's last P V)
    const uint64_t dq[2] = {sw128_desc(smem_u32(sm.q[0]), 16, 1024), sw128_desc(smem_u32(sm.q[1]), 16, 1024)};
    const uint64_t dp[2] = {sw128_desc(smem_u32(sm.p[0]), 16, 1024), sw128_desc(smem_u32(sm.p[1]), 16, 1024)};
    const uint64_t dkv0 = sw128_desc(smem_u32(sm.kv[0]), 16, 1024);
    auto issue_s = [&](int w, uint32_t slot) {
      const uint64_t dk = desc_advance(dkv0, slot * Smem::kTileBytes);
#pragma unroll
      for (int kk = 0; kk < kF8D / 32; ++kk)   // 32 codes = 32 bytes per k-step
        mma_e4m3_ss_w(tmem + w * 128, desc_advance(dq[w], kk * 32), desc_advance(dk, kk * 32), idesc, kk > 0);
      mma_commit_w(smem_u32(&sm.s_full[w]));
    };
    auto issue_pv = [&](int w, uint32_t slot) {
      const uint64_t dvt = desc_advance(dkv0, slot * Smem::kTileBytes);
      const uint32_t acc = pv_count[w] > 0;
#pragma unroll
      for (int kk = 0; kk < kBlockN / 32; ++kk)   // 32 keys per k-step
        mma_e4m3_ss_w(tmem + 256 + w * 128, desc_advance(dp[w], kk * 32), desc_advance(dvt, kk * 32), idesc,
                      kk > 0 ? 1u : acc);
      ++pv_count[w];
    };
    bool ok = wait(smem_u32(&sm.q_full), 0);
    if (ok) {
      ok = wait(smem_u32(&sm.slot_full[0]), 0);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int w = 0; w < kQTiles; ++w)
          if (active(w, t_begin)) issue_s(w, 0);
        mma_commit_w(smem_u32(&sm.slot_empty[0]));
      }
    }
    for (int t = t_begin; ok && t < t_end; ++t) {
      const int Lv = 2 * (t - t_begin) + 1;
      const int Lk = Lv + 1;
      const bool has_next = t + 1 < t_end;
      if (!wait(smem_u32(&sm.slot_full[Lv % kSlots]), (Lv / kSlots) & 1)) break;
      if (has_next && !wait(smem_u32(&sm.slot_full[Lk % kSlots]), (Lk / kSlots) & 1)) break;
#pragma unroll
      for (int w = 0; w < kQTiles; ++w) {
        if (active(w, t)) {
          if (!wait(smem_u32(&sm.p_full[w]), pv_count[w] & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(w, Lv % kSlots);
          if (t + 1 == ew[w]) {
            // the tile's O is final once this P V completes: its epilogue overlaps the other
            // tile's last steps
            mma_commit_w(smem_u32(&sm.o_final[w]));
            o_done[w] = true;
          }
        }
        if (has_next && active(w, t + 1)) issue_s(w, Lk % kSlots);
      }
      if (!ok) break;
      if (has_next) mma_commit_w(smem_u32(&sm.slot_empty[Lk % kSlots]));
      mma_commit_w(smem_u32(&sm.slot_empty[Lv % kSlots]));
    }
#pragma unroll
    for (int w = 0; w < kQTiles; ++w)
      if (!o_done[w]) mma_commit_w(smem_u32(&sm.o_final[w]));   // a tile without keys, or after an abort
    mma_commit_w(smem_u32(&sm.mma_drain));
    mbar_wait_drain(smem_u32(&sm.mma_drain), 0, lim);
  } else {
    // ------------------------------------------------------------------ softmax warpgroups
    const int w = warp >> 2;
    const int row = threadIdx.x & 127;
    const int qw0 = q0 + w * kBlockM;
    const int qi = qw0 + row;
    const int tb = w == 0 ? b0 : b1;
    const int te = w == 0 ? e0 : e1;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t s_col = tmem + lane_base + w * 128;
    const uint32_t o_col = tmem + lane_base + 256 + w * 128;
    const uint32_t p_row = smem_u32(sm.p[w]) + uint32_t(row) * 128;
    const float c = prm.scale_log2;
    bool ok = true;
    float m = -INFINITY;
    float l = 0.f;
    auto step = [&](const int t, auto masked) -> bool {
      const int k = t - tb;
      const int kv0 = t * kBlockN;
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.s_full[w]), k & 1, abort, lim))) return false;
      tc_fence_after();
      // Two passes over the S columns in TMEM, as in fa_fwd_kernel: the row max from all 128,
      // then the exponentials 32 columns at a time (the next chunk's load in flight), so that the
      // exponentials' temporaries fit next to one chunk of scores rather than all 128.
      int a = 0, b = kBlockN;   // allowed columns of this row in the tile: [a, b)
      if constexpr (decltype(masked)::value) {
        const int hi = prm.causal ? min(qi, prm.N - 1)
                                  : (prm.window > 0 ? min(qi + prm.window - 1, prm.N - 1) : prm.N - 1);
        const int lo = prm.window > 0 ? qi - prm.window + 1 : 0;
        a = lo - kv0;
        b = hi - kv0 + 1;
      }
      float mx;
      if constexpr (!decltype(masked)::value) {
        uint32_t r[kBlockN];
#pragma unroll
        for (int ch = 0; ch < kBlockN / 32; ++ch) tmem_ld32_async(s_col + ch * 32, r + ch * 32);
        tmem_ld_wait();
        reg_fence<kBlockN>(r);
        float mx16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) mx16[i] = __uint_as_float(r[i]);
#pragma unroll
        for (int j = 16; j < kBlockN; j += 16)
#pragma unroll
          for (int i = 0; i < 16; ++i) mx16[i] = fmaxf(mx16[i], __uint_as_float(r[j + i]));
#pragma unroll
        for (int i = 0; i < 8; ++i) mx16[i] = fmaxf(mx16[i], mx16[i + 8]);
        mx = max3f(max3f(mx16[0], mx16[1], mx16[2]), max3f(mx16[3], mx16[4], mx16[5]), fmaxf(mx16[6], mx16[7]));
      } else {
        // the masked form takes the max 64 columns at a time (its masking temporaries would
        // not fit next to all 128 scores)
        float mx16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) mx16[i] = -INFINITY;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t r[64];
          tmem_ld32_async(s_col + half * 64, r);
          tmem_ld32_async(s_col + half * 64 + 32, r + 32);
          tmem_ld_wait();
          reg_fence<64>(r);
#pragma unroll
          for (int wd = 0; wd < 2; ++wd) {
            const int aw = min(max(a - 32 * (2 * half + wd), 0), 32), bw = min(max(b - 32 * (2 * half + wd), 0), 32);
            const uint32_t below_b = bw >= 32 ? 0xffffffffu : ((1u << bw) - 1u);
            const uint32_t below_a = aw >= 32 ? 0xffffffffu : ((1u << aw) - 1u);
            const uint32_t bits = below_b & ~below_a;   // allowed columns 32 (2 half + wd) + j
#pragma unroll
            for (int j = 0; j < 32; ++j)
              mx16[j & 15] = fmaxf(mx16[j & 15], ((bits >> j) & 1u) ? __uint_as_float(r[32 * wd + j]) : -INFINITY);
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) mx16[i] = fmaxf(mx16[i], mx16[i + 8]);
        mx = max3f(max3f(mx16[0], mx16[1], mx16[2]), max3f(mx16[3], mx16[4], mx16[5]), fmaxf(mx16[6], mx16[7]));
      }
      const float m_cand = fmaxf(m, mx * c);
      const bool grow = m_cand > m + kRescaleThreshold;
      const float m_new = grow ? m_cand : m;
      const float alpha = grow ? ex2_approx(m - m_new) : 1.f;
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const uint64_t c2 = f2(c, c), nm2 = f2(-m_use, -m_use);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
      // one 32-column chunk: P as E4M3 codes into this row of the P tile, 16-byte chunk j (keys
      // 16 j ..) at j ^ (row % 8)
      auto exp_chunk = [&](int ch, const uint32_t* cur) {
        float sv[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) sv[j] = __uint_as_float(cur[j]);
        if constexpr (decltype(masked)::value) {
          const int aw = a - 32 * ch, bw = b - 32 * ch;   // allowed columns j of the chunk: [aw, bw)
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < aw || j >= bw) sv[j] = -INFINITY;
        }
#pragma unroll
        for (int h16 = 0; h16 < 2; ++h16) {
          uint32_t words[4];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t codes = 0;
#pragma unroll
            for (int hp = 0; hp < 2; ++hp) {
              const int j = h16 * 16 + q4 * 4 + hp * 2;   // column in the chunk; pair jp = j / 2
              const uint64_t x = f2_fma(f2(sv[j], sv[j + 1]), c2, nm2);
              float p0, p1;
              if ((j >> 1) < kEmuPairs) {
                exp2_poly_x2(x, p0, p1);
              } else {
                float x0, x1;
                f2_split(x, x0, x1);
                p0 = ex2_approx(x0);
                p1 = ex2_approx(x1);
              }
              acc[(j >> 1) & 3] = f2_add(acc[(j >> 1) & 3], f2(p0, p1));
              codes |= f32x2_to_e4m3x2(p0, p1) << (16 * hp);
            }
            words[q4] = codes;
          }
          const int c16 = 2 * ch + h16;
          st_shared_v4(p_row + uint32_t((c16 ^ (row & 7)) * 16), words[0], words[1], words[2], words[3]);
        }
      };
      {
        uint32_t ra[32], rb[32];
        tmem_ld32_async(s_col, ra);
        tmem_ld_wait();
        reg_fence<32>(ra);
#pragma unroll
        for (int ch = 0; ch < kBlockN / 32; ++ch) {
          uint32_t* cur = (ch & 1) ? rb : ra;
          uint32_t* nxt = (ch & 1) ? ra : rb;
          if (ch + 1 < kBlockN / 32) tmem_ld32_async(s_col + (ch + 1) * 32, nxt);
          exp_chunk(ch, cur);
          if (ch + 1 < kBlockN / 32) {
            tmem_ld_wait();
            reg_fence<32>(nxt);
          }
        }
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
        // PV of the previous tile completed before this S did (in-order MMAs): O is stable
#pragma unroll
        for (int ch = 0; ch < kF8D / 32; ++ch) {
          uint32_t r[32];
          tmem_ld32(o_col + ch * 32, r);
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * alpha);
          tmem_st32(o_col + ch * 32, r);
        }
        tmem_st_wait();
      }
      fence_proxy_async_smem();   // the MMA reads P through the async proxy
      tc_fence_before();
      mbar_arrive(smem_u32(&sm.p_full[w]));
      return true;
    };
    const int band_lo_max = prm.window > 0 ? qw0 + kBlockM - prm.window : 0;
    const int band_hi_min = min(prm.N - 1, prm.causal ? qw0 : (prm.window > 0 ? qw0 + prm.window - 1 : prm.N - 1));
    for (int t = tb; t < te; ++t) {
      const int kv0 = t * kBlockN;
      const bool need_mask = kv0 < band_lo_max || kv0 + kBlockN - 1 > band_hi_min;
      ok = need_mask ? step(t, std::true_type{}) : step(t, std::false_type{});
      if (!ok) break;
    }
    if (ok && te > tb && __all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.o_final[w]), 0, abort, lim))) {
      tc_fence_after();
      const float inv_l = v_scale / l;
      const bool in_range = qi < prm.N;
      __nv_bfloat16* orow = prm.o + prm.o_st.at(b_idx, h_q, in_range ? qi : 0);
#pragma unroll
      for (int ch = 0; ch < kF8D / 32; ++ch) {
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
  if (warp == kWarpTma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace fa
