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
// sm_100a mapping: one CTA per pair of adjacent 128-row query tiles of one head, so every
// K/V tile brought on chip serves 256 query rows; the grid takes heads in chunks, the longest
// causal pairs of a chunk first (grid_item).
//   warp 8      TMA producer (and TMEM owner): both Q tiles once, then K_j, V_j through a
//               4-slot ring.
//   warp 9      MMA issuer (one thread), in the order PV0(j), S0(j+1), PV1(j), S1(j+1), so
//               the tensor pipe computes one tile's products while the other tile's softmax
//               runs (ping-pong).  S = Q K^T lands in TMEM; P is written back over the
//               consumed S columns as bf16 and O += P V reads it from TMEM.
//   warps 0-3   softmax of query tile 0, warps 4-7 of tile 1: thread t owns row t (TMEM
//               lane t): tcgen05.ld of S (twice: the row max, then the exponentials 32
//               columns at a time), scale and mask, running max m and sum l,
//               P = 2^(S c - m) packed to bf16 and stored to TMEM, and at the end O / l ->
//               bf16 (written through the tile's Q buffer by TMA tensor stores) and
//               L = (m + log2 l) ln 2.
// The running max is updated lazily: O in TMEM is rescaled only when a row's max grows by
// more than 2^8; otherwise the stale max keeps being used (P <= 256, exact after the final
// division by l).  MMAs issued by one thread execute in order, so S(j) completing means
// PV(j-1) of the same tile has completed: a rescale never races an MMA, and S(j+1) may be
// issued right behind PV(j) although it overwrites the TMEM columns PV(j) reads P from.
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256, 256+D), O1 [384, 384+D); P_w occupies
// the first 64 columns of S_w.  A tile's O is final (o_final) right after its own last P V, so
// its epilogue overlaps the other tile's last steps (under the causal mask the second tile
// has one more key tile than the first).
#pragma once

#include <type_traits>

#include "grid_sched.cuh"
#include "sm100.cuh"

namespace fa {

constexpr int kBlockM = 128;   // query rows per tile (one per TMEM lane)
constexpr int kBlockN = 128;   // keys per KV tile
constexpr int kQTiles = 2;     // query tiles per CTA
constexpr int kSlots = 4;      // K/V shared-memory ring slots (K and V alternate)
constexpr int kFwdThreads = 320;
constexpr int kWarpTma = 8;
constexpr int kWarpMma = 9;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;   // log2 units: rescale O only when m grows by > 2^8
#ifndef FA_FWD_EMU_PAIRS
#define FA_FWD_EMU_PAIRS 7
#endif
constexpr int kEmuPairs = FA_FWD_EMU_PAIRS;   // of every 16 exponential pairs, this many use the FMA pipe
// fa_fwd_kernel's own split per head dimension: measured on a B200 (20-step causal / GPT-2-like
// runs), 6 of 16 is best at d = 128 (0.2674 ms against 0.2691 at 7 and 0.2741 at 5) and 7 at
// d = 64 (127.3 us against 128.2 at 6 and 135.3 at 8); the other forwards use kEmuPairs
#ifdef FA_FWD_EMU_PAIRS_OVERRIDE
template <int D>
constexpr int kFwdEmuPairs = FA_FWD_EMU_PAIRS;
#else
template <int D>
constexpr int kFwdEmuPairs = D == 64 ? 7 : 6;
#endif

struct FwdParams {
  __nv_bfloat16* o;   // [B, H, N, D] with strides o_st
  float* lse;         // [BH, N]
  int N;
  int BH;             // query heads, B * H
  int H;              // query heads per batch entry
  int group;          // query heads per K/V head (H / H_kv)
  Strides o_st;       // element strides of O
  int n_pairs;        // ceil(ceil(N / 128) / 2)
  int causal;
  int window;
  float scale_log2;   // scale * log2(e)
  unsigned long long wait_limit_ns;
};

template <int D>
struct FwdSmem {
  static constexpr int kChunks = D / 64;                   // 64-element (128-byte) column chunks
  static constexpr uint32_t kTileBytes = kBlockN * D * 2;  // one Q, K or V tile
  alignas(1024) uint8_t q[kQTiles][kTileBytes];
  alignas(1024) uint8_t kv[kSlots][kTileBytes];
  alignas(8) uint64_t q_full;
  uint64_t slot_full[kSlots], slot_empty[kSlots];
  uint64_t s_full[kQTiles], p_full[kQTiles], o_final[kQTiles];
  uint64_t o_staged[kQTiles];   // a tile's 128 rows of O / l are in its Q buffer
  uint64_t mma_drain;
  uint32_t tmem_base;
  int abort;
};

// KV tiles [t_begin, t_end) one query tile starting at q0 needs: causal stops at the diagonal,
// a window starts at the tile holding key q0 - W + 1.  Empty when the tile is past N.
__device__ __forceinline__ void kv_tile_range(int q0, int N, int causal, int window, int& t_begin, int& t_end) {
  if (q0 >= N) {
    t_begin = t_end = 0;
    return;
  }
  // the tile's last query attends keys up to itself (causal), up to itself + W - 1 (two-sided
  // window), or all of them
  const int kv_end = causal ? min(N, q0 + kBlockM) : (window > 0 ? min(N, q0 + kBlockM - 1 + window) : N);
  t_end = (kv_end + kBlockN - 1) / kBlockN;
  const int kv_begin = window > 0 ? max(0, q0 - window + 1) : 0;
  t_begin = kv_begin / kBlockN;
}

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                  const FwdParams prm) {
  using Smem = FwdSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // chunks of heads (their K/V stay in L2), the longest causal pairs of a chunk first
  int bh, rank;
  grid_item(int(blockIdx.x), prm.BH, prm.n_pairs, kFwdChunkHeads, bh, rank);
  // batch entry, query head, and the K/V head it reads (heads share K/V in contiguous groups)
  const int b_idx = bh / prm.H, h_q = bh % prm.H, h_kv = h_q / prm.group;
  const int pair = prm.n_pairs - 1 - rank;
  const int q0 = pair * (kQTiles * kBlockM);
  int b0, e0, b1, e1;
  kv_tile_range(q0, prm.N, prm.causal, prm.window, b0, e0);
  kv_tile_range(q0 + kBlockM, prm.N, prm.causal, prm.window, b1, e1);
  if (e1 == 0) b1 = e1 = b0;   // second tile entirely past N: no work for it
  const int t_begin = b0;       // b1 >= b0 and e1 >= e0 whenever tile 1 has work
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
      mbar_init(smem_u32(&sm.o_staged[w]), kBlockM);
    }
    mbar_init(smem_u32(&sm.mma_drain), 1);
    fence_mbar_init();
  }
  if (warp == kWarpTma) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_o);
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
      for (int w = 0; w < kQTiles; ++w)
        for (int c = 0; c < Smem::kChunks; ++c)
          tma_load_rows(smem_u32(sm.q[w]) + c * 16384, &tm_q, qb, c * 64, q0 + w * kBlockM, h_q, b_idx);
      int issued = 0;   // loads issued: K_t is load 2(t - t_begin), V_t the next one
      const int n_loads = 2 * (t_end - t_begin);
      for (int L = 0; L < n_loads; ++L) {
        const int slot = L % kSlots;
        if (!mbar_wait(smem_u32(&sm.slot_empty[slot]), ((L / kSlots) & 1) ^ 1, abort, lim)) break;
        const uint32_t fb = smem_u32(&sm.slot_full[slot]);
        const int kv0 = (t_begin + (L >> 1)) * kBlockN;
        const CUtensorMap* map = (L & 1) ? &tm_v : &tm_k;
        mbar_expect_tx(fb, Smem::kTileBytes);
        for (int c = 0; c < Smem::kChunks; ++c)
          tma_load_rows(smem_u32(sm.kv[slot]) + c * 16384, map, fb, c * 64, kv0, h_kv, b_idx);
        issued = L + 1;
      }
      // let every copy this CTA started land before the CTA may exit
      mbar_wait_drain(qb, 0, lim);
      for (int L = max(0, issued - kSlots); L < issued; ++L)
        mbar_wait_drain(smem_u32(&sm.slot_full[L % kSlots]), (L / kSlots) & 1, lim);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    // the whole warp runs this loop (uniformly); each tcgen05 op is issued by one elected lane
    {
      auto wait = [&](uint32_t bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, lim));
      };
      constexpr uint32_t idesc_s = idesc_bf16_f32(kBlockM, kBlockN, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(kBlockM, D, false, true);
      const int bw[2] = {b0, b1}, ew[2] = {e0, e1};
      auto active = [&](int w, int t) { return t >= bw[w] && t < ew[w]; };
      int pv_count[2] = {0, 0};
      bool o_done[2] = {false, false};   // o_final committed (right after the tile's last P V)
      // descriptors are built once; each k-step only adds a constant to the start field
      const uint64_t dq[2] = {sw128_desc(smem_u32(sm.q[0]), 16, 1024), sw128_desc(smem_u32(sm.q[1]), 16, 1024)};
      const uint64_t dkv0 = sw128_desc(smem_u32(sm.kv[0]), 16, 1024);
      const uint64_t dv0 = sw128_desc(smem_u32(sm.kv[0]), 16384, 1024);
      auto issue_s = [&](int w, uint32_t slot) {
        const uint64_t dk = desc_advance(dkv0, slot * Smem::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // K-major operands: 16-element k-steps are 32 bytes apart inside a 128-byte row,
          // 64-element chunks are separate 16 KB tiles
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss_w(tmem + w * 128, desc_advance(dq[w], off), desc_advance(dk, off), idesc_s, kk > 0);
        }
        mma_commit_w(smem_u32(&sm.s_full[w]));
      };
      auto issue_pv = [&](int w, uint32_t slot) {
        const uint64_t dv = desc_advance(dv0, slot * Smem::kTileBytes);
        const uint32_t acc = pv_count[w] > 0;
#pragma unroll
        for (int kk = 0; kk < kBlockN / 16; ++kk) {
          // A = P from TMEM (16 keys = 8 packed columns per k-step); B = V MN-major: 16 keys =
          // 16 rows of 128 bytes, the next 64 head-dim columns one 16 KB chunk (LBO) further
          mma_bf16_ts_w(tmem + 256 + w * 128, tmem + w * 128 + kk * 8, desc_advance(dv, kk * 2048), idesc_o,
                      kk > 0 ? 1u : acc);
        }
        ++pv_count[w];
      };
      bool ok = wait(smem_u32(&sm.q_full), 0);
      // prologue: S of the first KV tile
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
        const int Lv = 2 * (t - t_begin) + 1;   // V of tile t
        const int Lk = Lv + 1;                  // K of tile t + 1
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
              // the tile's O is final once this P V completes: its softmax warps start the
              // epilogue while the other tile's last steps run
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
      // every MMA issued above completes before TMEM is released
      mma_commit_w(smem_u32(&sm.mma_drain));
      mbar_wait_drain(smem_u32(&sm.mma_drain), 0, lim);
    }
  } else {
    // ------------------------------------------------------------------ softmax warpgroups
    const int w = warp >> 2;                     // query tile of this warpgroup
    const int row = threadIdx.x & 127;           // == TMEM lane
    const int qw0 = q0 + w * kBlockM;
    const int qi = qw0 + row;
    const int tb = w == 0 ? b0 : b1;
    const int te = w == 0 ? e0 : e1;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t s_col = tmem + lane_base + w * 128;
    const uint32_t o_col = tmem + lane_base + 256 + w * 128;
    const float c = prm.scale_log2;
    bool ok = true;
    float m = -INFINITY;   // running max of scaled scores (log2 units)
    float l = 0.f;         // running sum of exponentials
    // One KV tile.  The masked and the unmasked form are separate instantiations: folded into
    // one body, the masking code is predicated rather than branched around and costs issue
    // slots on every tile.
    auto step = [&](const int t, auto masked) -> bool {
      {
        const int k = t - tb;
        const int kv0 = t * kBlockN;
        // the vote keeps every lane of the warp on the same path into the .sync.aligned TMEM ops
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.s_full[w]), k & 1, abort, lim))) return false;
        tc_fence_after();
        // Two passes over the S columns in TMEM: the row max from all 128, then the
        // exponentials 32 columns at a time, each chunk reloaded (the next one's load in flight
        // while this one is exponentiated).  Holding all 128 scores through the exponentials
        // would leave too few of the 168 registers for the exponentials' temporaries.
        // Allowed keys of this row form one range [lo, hi]; as columns of the tile, [a, b); the
        // masked form applies it in both passes.
        int a = 0, b = kBlockN;
        if constexpr (decltype(masked)::value) {
          const int hi = prm.causal ? min(qi, prm.N - 1)
                                    : (prm.window > 0 ? min(qi + prm.window - 1, prm.N - 1) : prm.N - 1);
          const int lo = prm.window > 0 ? qi - prm.window + 1 : 0;
          a = lo - kv0;
          b = hi - kv0 + 1;
        }
        // allowed columns 32 wd + j of the tile, as bits j
        auto allowed_bits = [&](int wd) -> uint32_t {
          const int aw = min(max(a - 32 * wd, 0), 32), bw = min(max(b - 32 * wd, 0), 32);
          const uint32_t below_b = bw >= 32 ? 0xffffffffu : ((1u << bw) - 1u);
          const uint32_t below_a = aw >= 32 ? 0xffffffffu : ((1u << aw) - 1u);
          return below_b & ~below_a;
        };
        float mx;
        if constexpr (!decltype(masked)::value) {
          uint32_t r[kBlockN];
#pragma unroll
          for (int ch = 0; ch < kBlockN / 32; ++ch) tmem_ld32_async(s_col + ch * 32, r + ch * 32);
          tmem_ld_wait();
          reg_fence<kBlockN>(r);
          // row max in 16 independent chains (one chain would be 127 dependent steps)
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
          // the masked form (diagonal and band-edge tiles) takes the max 64 columns at a time:
          // its masking temporaries would not fit next to all 128 scores
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
              const uint32_t bits = allowed_bits(2 * half + wd);
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
        const bool grow = m_cand > m + kRescaleThreshold;   // false while the row has no key
        const float m_new = grow ? m_cand : m;
        const float alpha = grow ? ex2_approx(m - m_new) : 1.f;   // 0 for the first keys of a row
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;   // a row with no key yet gives P = 0
        // P = 2^(S c - m): in every 16 pairs the first kFwdEmuPairs<D> go through the FMA-pipe
        // polynomial, the rest through MUFU ex2, so that neither unit limits the tile
        const uint64_t c2 = f2(c, c), nm2 = f2(-m_use, -m_use);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
        // one chunk's exponentials: S columns 32 ch .. of `cur`, P into packed columns 16 ch ..
        // (S columns already read), the sum into acc
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
          uint32_t pk[16];
#pragma unroll
          for (int jp = 0; jp < 16; ++jp) {
            const uint64_t x = f2_fma(f2(sv[2 * jp], sv[2 * jp + 1]), c2, nm2);
            float p0, p1;
            if (jp < kFwdEmuPairs<D>) {
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
        };
        {
          // chunk ch + 1 loads while chunk ch is exponentiated
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
          const uint64_t tot = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
          float lo, hi;
          f2_split(tot, lo, hi);
          sum = lo + hi;
        }
        l = l * alpha + sum;
        m = m_new;
        if (k > 0 && __any_sync(0xffffffffu, grow)) {
          // PV of the previous tile is complete (it was issued before this S), so O is stable;
          // done after P so that the S registers are free
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
      }
      return true;
    };
    // a KV tile needs the mask when some key lies outside some row's band: below the band of the
    // tile's last row, or above the band of its first row (or past N)
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
      const float inv_l = 1.f / l;
      // O / l as bf16, staged in this tile's Q buffer (every MMA has completed, so Q is read no
      // more) in the layout a TMA load of the tile leaves there: 64-column chunks of 16 KB,
      // 128-byte rows, 16-byte piece c of row r at c ^ (r % 8).  One thread then writes the tile
      // with TMA tensor stores, which skip the rows past N.
      const uint32_t stage = smem_u32(sm.q[w]);
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t r[32];
        tmem_ld32(o_col + ch * 32, r);
        uint32_t wv[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          wv[j] = pack_bf16x2(__uint_as_float(r[2 * j]) * inv_l, __uint_as_float(r[2 * j + 1]) * inv_l);
        const uint32_t row_addr = stage + (ch >> 1) * 16384 + row * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t c16 = (ch & 1) * 4 + j;
          st_shared_v4(row_addr + ((c16 ^ (row & 7)) << 4), wv[4 * j], wv[4 * j + 1], wv[4 * j + 2], wv[4 * j + 3]);
        }
      }
      fence_proxy_async_smem();   // the tensor store reads the rows through the async proxy
      mbar_arrive(smem_u32(&sm.o_staged[w]));
      if (qi < prm.N) prm.lse[size_t(bh) * prm.N + qi] = (m + lg2_approx(l)) * 0.69314718055994531f;
      if (row == 0 && mbar_wait(smem_u32(&sm.o_staged[w]), 0, abort, lim)) {
#pragma unroll
        for (int c = 0; c < Smem::kChunks; ++c) tma_store_rows(&tm_o, stage + c * 16384, c * 64, qw0, h_q, b_idx);
        bulk_commit_group();
        // the rows are read before the CTA's shared memory is released (the writes to global
        // memory complete with the grid)
        bulk_wait_group_read<0>();
      }
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
