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
//   fa_bwd_kernel    one CTA per 128-key tile of one head; loops over 128-row query tiles.
//   fa_bwd_dq_final  dQ = scale * accumulator, rounded to bf16.
//
// fa_bwd_kernel roles (512 threads), every MMA 128 x 128 (narrower ones cost as much time):
//   warp 12     TMA producer: K, V once; Q_i (+ its L and D rows) into a 2-stage ring, dO_i into
//               one stage.
//   warp 13     MMA issuer, per query tile i in the order
//                 dV += P_i^T dO_i, S_{i+1}^T = K Q_{i+1}^T, dK += dS_i^T Q_i, dQ_i = dS_i K,
//                 dP_{i+1}^T = V dO_{i+1}^T
//               (dV and dK read their A operand from TMEM; dQ reads dS from shared memory), so
//               that the exponentials of tile i+1 run while dK_i and dQ_i are computed, and dS
//               of tile i+1 while dV_{i+1} and S_{i+2} are.  The kDkSmem form (shared K/V
//               heads) swaps dK_i and dQ_i, dK reading dS from shared memory as well, so that
//               the readout of dQ_i runs while dK_i is computed.
//   warps 0-7   two per TMEM lane quadrant; warp w owns lanes 32 (w % 4).. and the query half
//               w / 4 of each tile.  Phase A: P^T = exp2(S^T c - L) with the causal/window mask,
//               stored to TMEM as bf16.  Phase B: dS^T = P^T o (dP^T - D) to shared memory (A of
//               dQ; and of dK in the kDkSmem form) and to TMEM (A of dK in the other form).
//               Order per tile: B(i), A(i+1).  At the end: dK
//               (half 0), dV (half 1), staged in the idle Q buffers and written by TMA tensor
//               stores.
//   warps 8-11  dQ readout, one per TMEM lane quadrant: all D columns of its 32 query rows of
//               dQ_i from TMEM as soon as the product completes, then 32 columns at a time
//               through two shared-memory staging slots, each block added into the fp32
//               accumulator by one TMA tensor reduction (cp.reduce.async.bulk.tensor .add), so
//               that the adds leave the SM as whole 128-byte lines and no warp waits for them.
//   warps 14-15 none (they complete the last warpgroup, whose registers go to the others:
//               setmaxnreg moves them from the TMA/MMA warpgroup to the compute and readout ones).
// TMEM columns: dK [0,128), dV [128,256), S^T [256,384) with P^T in [256,288) and [320,352)
// once read, dP^T [384,512) with dS^T in [384,416) and [448,480) once read (TMEM form), and
// dQ in [384,512).  MMAs of one thread run in order, which makes each reuse safe: S_{i+1} is
// issued after dV_i read P_i, dQ_i after dK_i read dS_i^T (TMEM form) or after phase B read
// dP_i^T; dP_{i+1} waits until the readout warps have read dQ_i out, and phase B of tile i+1
// rewrites the dS buffer only once dP_{i+1}, and so dQ_i and dK_i before it, has completed.
#pragma once

#include <type_traits>

#include "grid_sched.cuh"
#include "sm100.cuh"

namespace fa {

constexpr int kBwdKeys = 128;    // keys per CTA
constexpr int kBwdRows = 128;    // queries per iteration
constexpr int kBwdQStages = 2;
constexpr int kBwdThreads = 512;   // 8 compute warps, 4 dQ readout warps, TMA, MMA and 2 idle warps
constexpr int kBwdWarpRead = 8;    // warps 8-11: the dQ readout, one per TMEM lane quadrant
constexpr int kBwdWarpTma = 12;
constexpr int kBwdWarpMma = 13;    // warps 14-15 complete the TMA/MMA warpgroup and do nothing
// Registers per thread: 128 at launch (512 threads share the SM's 64K); the compute warpgroups
// raise themselves to kBwdRegsCompute and the readout warpgroup to kBwdRegsRead out of what the
// TMA/MMA warpgroup gives back by lowering itself to kBwdRegsOther.
constexpr int kBwdLaunchRegs = 65536 / kBwdThreads;
constexpr int kBwdRegsCompute = 152;
constexpr int kBwdRegsRead = 88;
constexpr int kBwdRegsOther = 4 * kBwdLaunchRegs - 2 * kBwdRegsCompute - kBwdRegsRead;
static_assert(kBwdRegsOther >= 24 && kBwdRegsOther % 8 == 0 &&
                  2 * kBwdRegsCompute + kBwdRegsRead + kBwdRegsOther <= 4 * kBwdLaunchRegs,
              "the warpgroups' register budgets must fit in the launch share");
// setmaxnreg.inc may only raise a warp's count and .dec only lower it: the compute warpgroups
// raise, the readout and TMA/MMA warpgroups lower
static_assert(kBwdRegsCompute >= kBwdLaunchRegs && kBwdRegsRead <= kBwdLaunchRegs &&
                  kBwdRegsOther <= kBwdLaunchRegs,
              "each warpgroup's budget moves in the direction of its setmaxnreg form");
constexpr uint32_t kTdK = 0, kTdV = 128, kTS = 256, kTP = 256, kTdP = 384, kTdS = 384, kTdQ = 384;
constexpr int FA_DEVICE_SMEM_ALIGN = 2;   // status bit: dynamic shared memory not 1 KB aligned

struct BwdParams {
  const float* lp;        // [BH, Np] L * log2(e), +inf on padded rows
  const float* dd;        // [BH, Np] D
  float* dq_acc;          // [BH, Np, D]
  __nv_bfloat16* dk;      // [BH, N, D]
  __nv_bfloat16* dv;      // [BH, N, D]
  int N, Np, BH, n_kv_tiles, causal, window;
  int H, H_kv, group;     // query heads, K/V heads per batch entry; group = H / H_kv
  Strides dk_st, dv_st;   // element strides of dK and dV
  float scale_log2;       // scale * log2(e)
  float scale;
  unsigned long long wait_limit_ns;
};

template <int D>
struct BwdSmem {
  static constexpr int kChunks = D / 64;
  static constexpr uint32_t kTileBytes = 128 * D * 2;      // K, V, Q or dO tile
  alignas(1024) uint8_t k[kTileBytes];
  alignas(1024) uint8_t v[kTileBytes];
  alignas(1024) uint8_t q[kBwdQStages][kTileBytes];
  alignas(1024) uint8_t dout[kTileBytes];                  // one stage: see the producer
  alignas(1024) uint8_t ds[kBwdKeys * kBwdRows * 2];       // dS^T: [key][query], 64-query chunks
  alignas(1024) uint8_t stage[8][32 * 32 * 4];             // dQ staging: 32 rows x 32 fp32, two per readout warp
                                                           // (1 KB aligned: the 128-byte swizzle's atoms)
  alignas(16) float lp[kBwdQStages][kBwdRows];
  alignas(16) float dd[kBwdQStages][kBwdRows];
  alignas(8) uint64_t kv_full;
  uint64_t q_full[kBwdQStages], q_empty[kBwdQStages], do_full, do_empty;
  uint64_t s_full, dp_full, pa_full, ds_full, dq_full, dq_free, mma_final, mma_drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

// query tiles (of 128 rows) that can see some key of the tile [kv0, kv0 + 128)
__device__ __forceinline__ void q_tile_range(int kv0, int N, int causal, int window, int& i_begin, int& i_end) {
  const int n_q = (N + kBwdRows - 1) / kBwdRows;
  // causal: from the diagonal; a two-sided window: from the first query whose band reaches kv0
  i_begin = causal ? kv0 / kBwdRows : (window > 0 ? max(0, kv0 - window + 1) / kBwdRows : 0);
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
                                                   int H, Strides o_st, Strides do_st, long long total_rows) {
  constexpr int G = D / 8;                      // threads per row
  // the last heads' rows first: the first heads' zeroed accumulator rows, which the main
  // kernel's first chunk adds into, are then the most recently written (still in L2)
  const long long g = (long long)(gridDim.x - 1 - blockIdx.x) * (256 / G) + threadIdx.x / G;
  const int c = threadIdx.x % G;
  if (g >= total_rows) return;
  const long long bh = g / Np;
  const int n = int(g % Np);
  float dot = 0.f;
  if (n < N) {
    const int b_idx = int(bh / H), h = int(bh % H);
    const uint4 a = *reinterpret_cast<const uint4*>(o + o_st.at(b_idx, h, n) + c * 8);
    const uint4 b = *reinterpret_cast<const uint4*>(dout + do_st.at(b_idx, h, n) + c * 8);
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
                                                       int H, Strides dq_st, long long total_rows) {
  constexpr int G = D / 8;
  // the last heads' rows first: the main kernel's last chunk added into them last, so they are
  // the accumulator rows most likely still in L2
  const long long g = (long long)(gridDim.x - 1 - blockIdx.x) * (256 / G) + threadIdx.x / G;   // row of [BH, N]
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
  *reinterpret_cast<uint4*>(dq + dq_st.at(int(bh / H), int(bh % H), n) + c * 8) = out;
}

// ----------------------------------------------------------------------------- main kernel
// tm_dq: the fp32 accumulator [BH, Np, D] as the 4-D tensor (D, Np, BH, 1), 32 x 32 boxes with
// the 128-byte swizzle (the layout of a compute warp's staging slot).  tm_dk, tm_dv: dK and dV
// as (D, N, H_kv, B), boxes of 64 columns x 32 rows (one compute warp's key rows).
// kDkSmem: dK += dS^T Q_i reads dS from shared memory and is issued after dQ_i = dS_i K, so that
// the readout of dQ_i runs under it; otherwise dK reads dS^T from TMEM (written there by phase B)
// and is issued first.  The host takes the first form when K/V heads are shared: a CTA then
// adds into the accumulators of every query head of its group, the L2 holds more of them at
// once, and the readout is slower; with one query head per K/V head the second is faster.
template <int D, bool kDkSmem>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ CUtensorMap tm_dk,
                  const __grid_constant__ CUtensorMap tm_dv, const BwdParams prm) {
  using Smem = BwdSmem<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the layout fills almost all 227 KB, so no slack is left for realigning the base
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicOr(&g_status, FA_DEVICE_SMEM_ALIGN);
    return;
  }
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // this CTA's K/V head; with shared K/V heads it runs the query tiles of every query head of
  // its group in turn (dK and dV accumulate over all of them)
  // chunks of K/V heads, key tile 0 (the longest under a causal mask) of every head first
  int bh, kv_tile;
  grid_item(int(blockIdx.x), prm.BH / prm.group, prm.n_kv_tiles, kBwdChunkHeads, bh, kv_tile);
  const int kv0 = kv_tile * kBwdKeys;
  int i_begin, i_end;
  q_tile_range(kv0, prm.N, prm.causal, prm.window, i_begin, i_end);
  const int n_i = i_end - i_begin;                         // query tiles per query head, >= 1
  const int n_it = n_i * prm.group;
  const int bh_q0 = (bh / prm.H_kv) * prm.H + (bh % prm.H_kv) * prm.group;   // first query head
  // (no division when every K/V head serves one query head)
  const int b_idx = bh / prm.H_kv, h_kv = bh % prm.H_kv;   // batch entry and K/V head
  auto q_tile = [&](int it) { return prm.group == 1 ? i_begin + it : i_begin + it % n_i; };
  auto q_head = [&](int it) { return prm.group == 1 ? bh_q0 : bh_q0 + it / n_i; };
  volatile int* abort = &sm.abort;
  const uint64_t lim = prm.wait_limit_ns;

  if (threadIdx.x == 0) {
    sm.abort = 0;
    mbar_init(smem_u32(&sm.kv_full), 1);
    for (int s = 0; s < kBwdQStages; ++s) {
      mbar_init(smem_u32(&sm.q_full[s]), 1);
      mbar_init(smem_u32(&sm.q_empty[s]), 1);
    }
    mbar_init(smem_u32(&sm.s_full), 1);
    mbar_init(smem_u32(&sm.dp_full), 1);
    mbar_init(smem_u32(&sm.pa_full), 256);
    mbar_init(smem_u32(&sm.ds_full), 256);
    mbar_init(smem_u32(&sm.dq_full), 1);
    mbar_init(smem_u32(&sm.dq_free), 128);   // the four readout warps
    mbar_init(smem_u32(&sm.mma_final), 1);
    mbar_init(smem_u32(&sm.mma_drain), 1);
    mbar_init(smem_u32(&sm.do_full), 1);
    mbar_init(smem_u32(&sm.do_empty), 1);
    fence_mbar_init();
  }
  if (warp == kBwdWarpTma && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
    tma_prefetch_desc(&tm_dq);
    tma_prefetch_desc(&tm_dk);
    tma_prefetch_desc(&tm_dv);
  }
  if (warp == kBwdWarpMma) {
    tmem_alloc(smem_u32(&sm.tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp >= kBwdWarpTma) {
  regs_lower<kBwdRegsOther>();
  if (warp == kBwdWarpTma) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint32_t kvb = smem_u32(&sm.kv_full);
      mbar_expect_tx(kvb, 2 * Smem::kTileBytes);
      for (int c = 0; c < Smem::kChunks; ++c) {
        tma_load_rows(smem_u32(sm.k) + c * 16384, &tm_k, kvb, c * 64, kv0, h_kv, b_idx);
        tma_load_rows(smem_u32(sm.v) + c * 16384, &tm_v, kvb, c * 64, kv0, h_kv, b_idx);
      }
      int issued = 0;
      // Q_i (with its L and D rows) through two stages; dO_i through one: its last reader,
      // dV_i, comes first in tile i and its next reader, dP_{i+1}, last, so one stage leaves
      // the load of dO_{i+1} most of a tile to land
      int issued_do = 0;
      for (int it = 0; it < n_it; ++it) {
        const int qs = it % kBwdQStages;
        const uint32_t ph = (it / kBwdQStages) & 1;
        const int q0 = q_tile(it) * kBwdRows;
        const int bq = q_head(it);
        if (!mbar_wait_inl(smem_u32(&sm.q_empty[qs]), ph ^ 1, abort, lim)) break;
        const uint32_t qb = smem_u32(&sm.q_full[qs]);
        mbar_expect_tx(qb, Smem::kTileBytes + 2 * kBwdRows * 4);
        for (int c = 0; c < Smem::kChunks; ++c)
          tma_load_rows(smem_u32(sm.q[qs]) + c * 16384, &tm_q, qb, c * 64, q0, bq - b_idx * prm.H, b_idx);
        const size_t row = size_t(bq) * prm.Np + q0;
        bulk_load(smem_u32(sm.lp[qs]), prm.lp + row, kBwdRows * 4, qb);
        bulk_load(smem_u32(sm.dd[qs]), prm.dd + row, kBwdRows * 4, qb);
        issued = it + 1;
        if (!mbar_wait_inl(smem_u32(&sm.do_empty), (it & 1) ^ 1, abort, lim)) break;
        const uint32_t db = smem_u32(&sm.do_full);
        mbar_expect_tx(db, Smem::kTileBytes);
        for (int c = 0; c < Smem::kChunks; ++c)
          tma_load_rows(smem_u32(sm.dout) + c * 16384, &tm_do, db, c * 64, q0, bq - b_idx * prm.H, b_idx);
        issued_do = it + 1;
      }
      mbar_wait_drain_inl(kvb, 0, lim);
      for (int it = max(0, issued - kBwdQStages); it < issued; ++it)
        mbar_wait_drain_inl(smem_u32(&sm.q_full[it % kBwdQStages]), (it / kBwdQStages) & 1, lim);
      if (issued_do > 0) mbar_wait_drain_inl(smem_u32(&sm.do_full), (issued_do - 1) & 1, lim);
    }
  } else if (warp == kBwdWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    // the whole warp runs this loop (uniformly); each tcgen05 op is issued by one elected lane
    {
      auto wait = [&](uint32_t bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait_inl(bar, parity, abort, lim));
      };
      constexpr uint32_t idesc_t = idesc_bf16_f32(128, kBwdRows, false, false);   // S^T, dP^T
      constexpr uint32_t idesc_kv = idesc_bf16_f32(128, D, false, true);          // dV, dK (A in TMEM)
      constexpr uint32_t idesc_q = idesc_bf16_f32(kBwdRows, D, true, true);       // dQ
      const uint64_t dk_kmaj = sw128_desc(smem_u32(sm.k), 16, 1024);
      const uint64_t dv_kmaj = sw128_desc(smem_u32(sm.v), 16, 1024);
      const uint64_t dk_mn = sw128_desc(smem_u32(sm.k), 16384, 1024);
      const uint64_t dds_mn = sw128_desc(smem_u32(sm.ds), 16384, 1024);
      // the dS buffer holds one 128-byte row of 64 queries per key: MN-major dS for dQ, K-major
      // dS^T for dK
      const uint64_t dds_kmaj = sw128_desc(smem_u32(sm.ds), 16, 1024);
      constexpr uint32_t idesc_dk = idesc_bf16_f32(128, D, false, true);            // dK (A = dS^T)
      // X^T = M_tile N_i^T with both operands K-major over the head dim (S^T and dP^T)
      auto issue_t = [&](uint64_t a, const uint8_t* b_tile, uint32_t d_col) {
        const uint64_t b = sw128_desc(smem_u32(b_tile), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_bf16_ss_w(tmem + d_col, desc_advance(a, off), desc_advance(b, off), idesc_t, kk > 0);
        }
      };
      // dV, dK += A(TMEM, 128 x 128 queries) * B (MN-major dO_i or Q_i: 16 queries = 2 KB per
      // k-step); A (P^T or dS^T) sits in TMEM as two 32-column halves, one per query half, at
      // a_col and a_col + 64; each 16-query k-step takes 8 of those columns
      auto issue_kv = [&](uint32_t a_col, const uint8_t* b_tile, uint32_t d_col, bool first) {
        const uint64_t b = sw128_desc(smem_u32(b_tile), 16384, 1024);
#pragma unroll
        for (int kk = 0; kk < kBwdRows / 16; ++kk)
          mma_bf16_ts_w(tmem + d_col, tmem + a_col + (kk >> 2) * 64 + (kk & 3) * 8, desc_advance(b, kk * 2048),
                        idesc_kv, (first && kk == 0) ? 0u : 1u);
      };
      bool ok = wait(smem_u32(&sm.kv_full), 0) && wait(smem_u32(&sm.q_full[0]), 0);
      if (ok) {
        tc_fence_after();
        issue_t(dk_kmaj, sm.q[0], kTS);
        mma_commit_w(smem_u32(&sm.s_full));
        ok = wait(smem_u32(&sm.do_full), 0);
      }
      if (ok) {
        tc_fence_after();
        issue_t(dv_kmaj, sm.dout, kTdP);
        mma_commit_w(smem_u32(&sm.dp_full));
      }
      for (int it = 0; ok && it < n_it; ++it) {
        const int qs = it % kBwdQStages;
        const bool has_next = it + 1 < n_it;
        const int qn = (it + 1) % kBwdQStages;
        // dV += P^T dO_i
        if (!wait(smem_u32(&sm.pa_full), it & 1)) break;
        tc_fence_after();
        issue_kv(kTP, sm.dout, kTdV, it == 0);
        mma_commit_w(smem_u32(&sm.do_empty));   // dV_i was dO_i's last reader
        // S^T of the next tile (overwrites P^T only after dV above has read it)
        if (has_next) {
          if (!wait(smem_u32(&sm.q_full[qn]), ((it + 1) / kBwdQStages) & 1)) break;
          issue_t(dk_kmaj, sm.q[qn], kTS);
          mma_commit_w(smem_u32(&sm.s_full));
        }
        if (!wait(smem_u32(&sm.ds_full), it & 1)) break;
        if constexpr (kDkSmem) {
          // dQ_i = dS_i K first, so that its readout runs under dK += dS^T Q_i; both read dS
          // from shared memory (dQ_i overwrites the dP^T columns, which phase B has read)
          if (!wait(smem_u32(&sm.dq_free), (it & 1) ^ 1)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kBwdKeys / 16; ++kk)
            mma_bf16_ss_w(tmem + kTdQ, desc_advance(dds_mn, kk * 2048), desc_advance(dk_mn, kk * 2048), idesc_q,
                          kk > 0);
          mma_commit_w(smem_u32(&sm.dq_full));
          const uint64_t bq = sw128_desc(smem_u32(sm.q[qs]), 16384, 1024);
#pragma unroll
          for (int kk = 0; kk < kBwdRows / 16; ++kk)
            mma_bf16_ss_w(tmem + kTdK, desc_advance(dds_kmaj, (kk >> 2) * 16384 + (kk & 3) * 32),
                          desc_advance(bq, kk * 2048), idesc_dk, (it == 0 && kk == 0) ? 0u : 1u);
        } else {
          // dK += dS^T Q_i with A = dS^T from TMEM, then dQ_i = dS_i K into the same columns
          tc_fence_after();
          issue_kv(kTdS, sm.q[qs], kTdK, it == 0);
          if (!wait(smem_u32(&sm.dq_free), (it & 1) ^ 1)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kBwdKeys / 16; ++kk)
            mma_bf16_ss_w(tmem + kTdQ, desc_advance(dds_mn, kk * 2048), desc_advance(dk_mn, kk * 2048), idesc_q,
                          kk > 0);
          mma_commit_w(smem_u32(&sm.dq_full));
        }
        mma_commit_w(smem_u32(&sm.q_empty[qs]));
        // dP^T of the next tile once dQ_i has been read out of the same columns
        if (has_next) {
          if (!wait(smem_u32(&sm.dq_free), it & 1)) break;
          if (!wait(smem_u32(&sm.do_full), (it + 1) & 1)) break;
          tc_fence_after();
          issue_t(dv_kmaj, sm.dout, kTdP);
          mma_commit_w(smem_u32(&sm.dp_full));
        }
      }
      mma_commit_w(smem_u32(&sm.mma_final));
      mma_commit_w(smem_u32(&sm.mma_drain));
      mbar_wait_drain_inl(smem_u32(&sm.mma_drain), 0, lim);
    }
  }
  } else if (warp >= kBwdWarpRead) {
    regs_lower<kBwdRegsRead>();
    // ------------------------------------------------------------------ dQ readout warps
    // One warp per TMEM lane quadrant (query rows 32 q .. of a tile): its rows of dQ_i from TMEM
    // into registers as soon as the product completes, then 32 columns at a time through its
    // two 4 KB staging slots, in the 128-byte swizzled layout, into the fp32 accumulator, one
    // TMA tensor reduction per block.
    const int quad = warp & 3;
    const uint32_t lane_base = uint32_t(quad * 32) << 16;
    const uint32_t slot0 = smem_u32(sm.stage[2 * quad]), slot1 = smem_u32(sm.stage[2 * quad + 1]);
    for (int it = 0; it < n_it; ++it) {
      if (!__all_sync(0xffffffffu, mbar_wait_inl(smem_u32(&sm.dq_full), it & 1, abort, lim))) break;
      tc_fence_after();
      const int q_row = q_tile(it) * kBwdRows + quad * 32;   // my first query row of the tile
      const int q_hd = q_head(it);
      // 64 columns at a time (the registers the readout warpgroup has); the columns are free
      // for dP_{i+1} once the last 64 are in registers
#pragma unroll
      for (int h = 0; h < D / 64; ++h) {
        uint32_t v[64];
        tmem_ld32_async(tmem + lane_base + kTdQ + h * 64, v);
        tmem_ld32_async(tmem + lane_base + kTdQ + h * 64 + 32, v + 32);
        tmem_ld_wait();
        reg_fence<64>(v);
        if (h == D / 64 - 1) {
          tc_fence_before();
          mbar_arrive(smem_u32(&sm.dq_free));
        }
#pragma unroll
        for (int p2 = 0; p2 < 2; ++p2) {
          const uint32_t slot = p2 ? slot1 : slot0;
          if (lane == 0) bulk_wait_group_read<1>();   // the block before the previous one has left this slot
          __syncwarp();
          // row `lane`, 16-byte chunk c at lane * 128 + (c ^ (lane & 7)) * 16: the 128-byte swizzle
#pragma unroll
          for (int c16 = 0; c16 < 8; ++c16)
            st_shared_v4(slot + lane * 128 + ((c16 ^ (lane & 7)) << 4), v[32 * p2 + 4 * c16],
                         v[32 * p2 + 4 * c16 + 1], v[32 * p2 + 4 * c16 + 2], v[32 * p2 + 4 * c16 + 3]);
          fence_proxy_async_smem();   // the tensor reduction reads the slot through the async proxy
          __syncwarp();
          if (lane == 0) {
            tma_reduce_add_rows(&tm_dq, slot, 64 * h + 32 * p2, q_row, q_hd, 0);
            bulk_commit_group();
          }
        }
      }
    }
    // every reduction this warp issued has read its slot before the CTA's shared memory is
    // released (the adds complete with the grid, before the finalise kernel runs)
    if (lane == 0) bulk_wait_group_read<0>();
    __syncwarp();
  } else {
    regs_raise<kBwdRegsCompute>();
    // ------------------------------------------------------------------ compute warps
    // Two warps per TMEM lane quadrant: warp w owns lanes 32 (w % 4) .. (keys for S^T, dP^T;
    // queries for dQ) and query half hq = w / 4 (queries 64 hq .. 64 hq + 63 of each tile).
    const int quad = warp & 3;
    const int hq = warp >> 2;
    const int r = quad * 32 + lane;            // key row of S^T / dP^T, query row of dQ
    const int key = kv0 + r;
    const uint32_t lane_base = uint32_t(quad * 32) << 16;
    const float c = prm.scale_log2;
    const uint32_t col_s = kTS + hq * 64;      // my S^T columns; P^T goes to the first 32 of them
    const uint32_t col_dp = kTdP + hq * 64;    // my dP^T columns
    const uint32_t ds_row = smem_u32(sm.ds) + hq * 16384 + r * 128;   // 64 queries = one 128-byte row
    const uint32_t sw = r & 7;
    uint32_t pk[32];                           // packed P^T of the current tile (phase A -> phase B)
    bool ok = true;

    // phase A: P^T = 2^(S^T c - L) for my 64 queries -> TMEM (bf16) and pk
    // The masked and the unmasked form of phase A are separate instantiations: folded into one
    // body, the masking code is predicated rather than branched around and costs issue slots on
    // every tile.
    auto phase_a = [&](int it, auto masked) -> bool {
      const int qs = it % kBwdQStages;
      const int q0 = q_tile(it) * kBwdRows;
      bool w_ok = mbar_wait_inl(smem_u32(&sm.q_full[qs]), (it / kBwdQStages) & 1, abort, lim);
      w_ok = w_ok && mbar_wait_inl(smem_u32(&sm.s_full), it & 1, abort, lim);
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
        // the queries that may attend to this key form one range: [key, key + W - 1] (causal;
        // W unbounded without a window), [key - W + 1, key + W - 1] (two-sided window), or all;
        // none for a padded key.  As columns, [a, b)
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
    // phase B: dS^T = P^T o (dP^T - D) for my 64 queries -> shared memory and, unless dK reads
    // it from there, TMEM (bf16)
    auto phase_b = [&](int it) -> bool {
      const int qs = it % kBwdQStages;
      // my rows of the dS buffer are free: dP of this tile completing means every earlier MMA
      // has, the products that read the previous tile's dS among them
      const bool w_ok = mbar_wait_inl(smem_u32(&sm.dp_full), it & 1, abort, lim);
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
        // (dP - D) * P on pairs; P comes back from its packed bf16 form (a shift per half)
        const float2 d2 = *reinterpret_cast<const float2*>(ddp + 2 * j2);
        const uint32_t w = pk[j2];
        const uint64_t p2 = f2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
        const uint64_t t2 = f2_add(f2(__uint_as_float(dr[2 * j2]), __uint_as_float(dr[2 * j2 + 1])), f2(-d2.x, -d2.y));
        float s0, s1;
        f2_split(f2_mul(t2, p2), s0, s1);
        pd[j2] = pack_bf16x2(s0, s1);
      }
      if constexpr (!kDkSmem) {   // dS^T into my dP^T columns, the A operand of dK
        tmem_st16(tmem + lane_base + col_dp, pd);
        tmem_st16(tmem + lane_base + col_dp + 16, pd + 16);
      }
#pragma unroll
      for (int c16 = 0; c16 < 8; ++c16)
        st_shared_v4(ds_row + ((c16 ^ sw) << 4), pd[4 * c16], pd[4 * c16 + 1], pd[4 * c16 + 2], pd[4 * c16 + 3]);
      if constexpr (!kDkSmem) tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(smem_u32(&sm.ds_full));
      return true;
    };
    // order: B(i), A(i+1); the readout warps take dQ_i out of TMEM meanwhile
    // phase A masks only on the diagonal, the window's far edge and the tail key tile
    auto run_a = [&](int it) -> bool {
      const int qbase = q_tile(it) * kBwdRows + hq * 64;
      const bool need_mask = (prm.causal && kv0 + kBwdKeys - 1 > qbase) ||
                             (prm.window > 0 && kv0 < qbase + 64 - prm.window) || (kv0 + kBwdKeys > prm.N) ||
                             (!prm.causal && prm.window > 0 && qbase + prm.window - 1 < kv0 + kBwdKeys - 1);
      return need_mask ? phase_a(it, std::true_type{}) : phase_a(it, std::false_type{});
    };
    ok = run_a(0);
    for (int it = 0; ok && it < n_it; ++it) {
      if (!phase_b(it)) { ok = false; break; }
      if (it + 1 < n_it && !run_a(it + 1)) { ok = false; break; }
    }
    // epilogue: warps of query half 0 write dK = scale * acc, those of half 1 write dV = acc.
    // My 32 key rows, as bf16, go to the Q buffers (idle once every MMA has completed) in the
    // layout of 32-row TMA boxes (64 columns of 128-byte swizzled rows each), and lane 0 writes
    // them with TMA tensor stores, which skip the rows past N.
    if (ok && __all_sync(0xffffffffu, mbar_wait_inl(smem_u32(&sm.mma_final), 0, abort, lim))) {
      tc_fence_after();
      const float mul = hq == 0 ? prm.scale : 1.f;
      const uint32_t col0 = hq == 0 ? kTdK : kTdV;
      const uint32_t out = smem_u32(sm.q[warp >> 2]) + uint32_t(warp & 3) * (D / 64) * 4096;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t rr[32];
        tmem_ld32(tmem + lane_base + col0 + ch * 32, rr);
        uint32_t w[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          w[j] = pack_bf16x2(__uint_as_float(rr[2 * j]) * mul, __uint_as_float(rr[2 * j + 1]) * mul);
        // columns 32 ch .. : 16-byte pieces 4 (ch & 1) .. of row `lane` in box ch / 2
        const uint32_t row = out + uint32_t(ch >> 1) * 4096 + uint32_t(lane) * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          st_shared_v4(row + ((((ch & 1) * 4 + j) ^ (lane & 7)) << 4), w[4 * j], w[4 * j + 1], w[4 * j + 2],
                       w[4 * j + 3]);
      }
      fence_proxy_async_smem();   // the tensor stores read the boxes through the async proxy
      __syncwarp();
      if (lane == 0) {
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx)
          tma_store_rows(hq == 0 ? &tm_dk : &tm_dv, out + bx * 4096, bx * 64, kv0 + quad * 32, h_kv, b_idx);
        bulk_commit_group();
      }
    }
    // every reduction and store this warp issued has read its shared memory before the CTA's
    // shared memory is released (the writes complete with the grid, before the finalise kernel)
    if (lane == 0) bulk_wait_group_read<0>();
    __syncwarp();
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
