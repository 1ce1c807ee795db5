// Split-key forward for a few new query rows over a long key sequence (a generation step
// over a key/value cache).
//
// Query row i stands at key position N_k - N_q + i, and the causal and window masks apply
// there.  The rows that read one K/V head (its group of query heads times the N_q new
// positions, "rows" in all) are cut into blocks of 16, the M of an m16n8k16 warp MMA, so one
// pass over the head's keys serves all of them.  The keys are cut into chunks ("splits"),
// one CTA per (split, row block, K/V head).  Each of a CTA's four warps streams its own
// 16-key steps through a private three-stage ring, filled by TMA tensor loads that its lane 0
// issues and that complete on one mbarrier per stage, and keeps its own running max m, sum l
// and unnormalised output; the CTA merges its warps, and when there is more than one
// split a second kernel merges the splits by their logsumexps:
//   L = M + ln sum_s exp(L_s - M),  O = sum_s exp(L_s - L) O_s   (M = max_s L_s).
// Every split's O_s is already normalised by its own l; a split with no allowed key has
// L_s = -inf and weight 0.  The work is bound by reading K and V from HBM once.
//
// With an FP8 K/V cache (kFp8) K and V arrive as E4M3 codes with one scale per tensor
// (K = s_k K8, V = s_v V8).  The ring then holds the raw codes; before each step the warp
// converts its 16 keys to f16 (exactly: every E4M3 value is an f16 value) into one padded
// tile, and the MMAs run on f16 operands (Q rounded to f16, clamped to its finite range).
// s_k is folded into the softmax scale and s_v into the final division.
#pragma once

#include <climits>
#include <cstdint>

#include "sm100.cuh"

namespace fa {

constexpr int kDecWarps = 4;
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kDecRows = 16;        // query rows per CTA: the M of the MMA
constexpr int kDecKeys = 16;        // keys per warp step
constexpr int kDecStages = 3;       // depth of each warp's copy ring
constexpr int kDecMergeWarps = 8;   // warps (one output row each) per CTA of the split merge
// CTAs resident at once on a B200 (148 SMs): two per SM, one at d = 256 (its rings take 198 KB)
__host__ __device__ constexpr int dec_slots(int d) { return d == 256 ? 148 : 148 * 2; }
constexpr int kDecCtaOverheadKeys = 128;   // a CTA's fixed cost (Q load, ring fill, merge), in keys

template <int D, bool kFp8 = false>
struct DecLayout {
  // A ring stage holds one step's K tile, then its V tile, as their TMA loads leave them: boxes
  // of 16 key rows, 128-byte swizzled (16-byte piece c of row r at c ^ (r % 8)).  bf16: D / 64
  // boxes of 64 elements a tile, read by the MMAs in place.  FP8: the raw E4M3 codes, D / 128
  // boxes of 128 a tile (at d = 64 one unswizzled box of 64-byte rows), which the warp converts
  // into the f16 K, V tile pair that follows its ring.
  static constexpr int kBoxX = kFp8 && D >= 128 ? 128 : 64;   // elements of a box row
  static constexpr bool kSwizzled = !kFp8 || D >= 128;
  static constexpr int kBoxBytes = kDecKeys * kBoxX * (kFp8 ? 1 : 2);
  static constexpr int kKvTileBytes = kDecKeys * D * (kFp8 ? 1 : 2);
  static constexpr int kBoxes = kKvTileBytes / kBoxBytes;     // TMA loads per tile
  static constexpr int kStageBytes = 2 * kKvTileBytes;        // K, then V
  // a converted f16 row, padded by 16 bytes so that the eight rows an 8x8 matrix load reads
  // start in eight different 16-byte bank groups
  static constexpr int kRowBytes = 2 * D + 16;
  static constexpr int kConvTileBytes = kDecKeys * kRowBytes;
  static constexpr int kConvBytes = kFp8 ? 2 * kConvTileBytes : 0;
  // each warp's ring starts on a 1 KB boundary (the swizzle's atom)
  static constexpr int kWarpBytes = (kDecStages * kStageBytes + kConvBytes + 1023) / 1024 * 1024;
  static constexpr int kRingBytes = kDecWarps * kWarpBytes;
  // after the key loop the rings hold each warp's O [16][D], m [16] and l [16] (fp32)
  static constexpr int kMergeFloats = kDecRows * D + 2 * kDecRows;
  static constexpr int kMergeBytes = kDecWarps * kMergeFloats * 4;
  static constexpr int kDataBytes = kRingBytes > kMergeBytes ? kRingBytes : kMergeBytes;
  // then one mbarrier per (warp, stage) and one abort flag per warp
  static constexpr int kBarOffset = kDataBytes;
  static constexpr int kAbortOffset = kBarOffset + kDecWarps * kDecStages * 8;
  // the dynamic shared memory is rounded up to 1 KB inside the kernel: 1 KB of slack
  static constexpr int kSmemBytes = 1024 + kAbortOffset + kDecWarps * 4;
  static_assert(kStageBytes % 1024 == 0 && kBoxBytes % 1024 == 0, "ring stages and boxes on 1 KB boundaries");
  static_assert(kSmemBytes <= 232448, "decode shared memory exceeds 227 KB");
};

// K and V ([B, H_kv, N_k, d], bf16 or E4M3 codes) reach the kernel as tensor maps.
struct DecParams {
  const __nv_bfloat16* q;   // [B, H, N_q, d]
  float v_scale;            // FP8: s_v (s_k is in scale_log2)
  __nv_bfloat16* o;         // [B, H, N_q, d]
  float* lse;               // [B, H, N_q] contiguous
  float* o_part;            // [n_splits][total_rows][d]; only when n_splits > 1
  float* l_part;            // [n_splits][total_rows]
  Strides q_st, k_st, v_st, o_st;
  long long total_rows;     // B * H * N_q
  int H, H_kv, group, Nq, Nk;
  int rows, row_blocks;     // rows per K/V head (group * N_q), blocks of 16 of them
  int n_splits, chunk, key_begin;   // split s covers keys [key_begin + s chunk, + chunk)
  int causal, window;
  float scale_log2;         // scale * log2(e)
  unsigned long long wait_limit_ns;   // bound on each wait for a ring stage
};

// Closed interval [lo, hi] of the keys a query at position pos may attend.
__host__ __device__ inline void dec_band(int pos, int Nk, int causal, int window, int& lo, int& hi) {
  if (causal) {
    hi = pos;
    lo = window > 0 ? pos - window + 1 : 0;
  } else if (window > 0) {
    lo = pos - window + 1;
    hi = pos + window - 1;
  } else {
    lo = 0;
    hi = Nk - 1;
  }
  if (lo < 0) lo = 0;
  if (hi > Nk - 1) hi = Nk - 1;
}

// How a decode problem is cut: a pure function of the shapes, so that the workspace size
// can be asked before the call.  window must already be clamped to N_k.
struct DecPlan {
  int rows, row_blocks, n_splits, chunk, key_begin;
  long long total_rows, ctas;
  size_t ws_bytes;
};

inline DecPlan dec_plan(int B, int H, int H_kv, int Nq, int Nk, int d, int causal, int window) {
  DecPlan pl;
  pl.rows = (H / H_kv) * Nq;
  pl.row_blocks = (pl.rows + kDecRows - 1) / kDecRows;
  pl.total_rows = (long long)B * H * Nq;
  // keys any row may attend: the bands move right with the position, so they run from the
  // first row's lowest key to the last row's highest
  int lo_first, hi_first, lo_last, hi_last;
  dec_band(Nk - Nq, Nk, causal, window, lo_first, hi_first);
  dec_band(Nk - 1, Nk, causal, window, lo_last, hi_last);
  pl.key_begin = lo_first & ~(kDecKeys - 1);
  const int steps = (hi_last + 1 - pl.key_begin + kDecKeys - 1) / kDecKeys;
  const long long base = (long long)B * H_kv * pl.row_blocks;
  // pick the split count that minimises (waves of resident CTAs) x (keys per CTA + its fixed
  // cost); at least two steps per warp in a split
  int max_splits = steps / (2 * kDecWarps);
  if (max_splits < 1) max_splits = 1;
  if (max_splits > 512) max_splits = 512;
  long long best_cost = -1;
  int best_steps = steps;
  for (int ns = 1; ns <= max_splits; ++ns) {
    const int per = (steps + ns - 1) / ns;
    const int used = (steps + per - 1) / per;
    const long long waves = (base * used + dec_slots(d) - 1) / dec_slots(d);
    const long long cost = waves * ((long long)per * kDecKeys + kDecCtaOverheadKeys);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_steps = per;
    }
  }
  pl.chunk = best_steps * kDecKeys;
  pl.n_splits = (steps + best_steps - 1) / best_steps;
  pl.ctas = base * pl.n_splits;
  pl.ws_bytes = pl.n_splits > 1 ? size_t(pl.n_splits) * size_t(pl.total_rows) * size_t(d + 1) * 4 : 0;
  return pl;
}

// The MMA and the P packing in the operand type: bf16, or f16 for the FP8 K/V path.
template <bool kF16>
__device__ __forceinline__ void dec_mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if constexpr (kF16)
    mma_16816_f16(d, a, b0, b1);
  else
    mma_16816(d, a, b0, b1);
}
template <bool kF16>
__device__ __forceinline__ uint32_t dec_pack(float lo, float hi) {
  if constexpr (kF16)
    return pack_f16x2(lo, hi);
  else
    return pack_bf16x2(lo, hi);
}

// Bounded wait for a ring stage, inline (no call in the key loop, whose registers would then
// have to survive one): the same limit and status as mbar_wait.
__device__ __forceinline__ bool dec_wait(uint32_t bar, uint32_t parity, volatile int* abort, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t n = 1;; ++n) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((n & 63u) == 0 && (*abort || global_timer_ns() - t0 > limit_ns)) {
      if (!*abort) atomicOr(&g_status, FA_DEVICE_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
}

// tm_k, tm_v: K and V (bf16, or the E4M3 codes) as the 4-D tensors (d, N_k, H_kv, B), boxes of
// DecLayout::kBoxX elements x 16 keys.
template <int D, bool kFp8>
__global__ void __launch_bounds__(kDecThreads, 2)
    fa_decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const DecParams p) {
  using Lay = DecLayout<D, kFp8>;
  constexpr int KS = D / 16;   // k-steps of S = Q K^T
  constexpr int NT = D / 8;    // 8-column n-tiles of O
  constexpr float kLn2 = 0.6931471805599453f;
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(dec_dyn_smem()) + 1023) &
                                                         ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBarOffset) + warp * kDecStages;   // my ring's
  volatile int* abort = reinterpret_cast<volatile int*>(smem + Lay::kAbortOffset) + warp;
  if (lane == 0) {
    *abort = 0;
    for (int st = 0; st < kDecStages; ++st) mbar_init(smem_u32(&bars[st]), 1);
    fence_mbar_init();
    fence_proxy_async_smem();   // the ring's copies complete on these barriers through the async proxy
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  __syncwarp();
  const int g = lane >> 2, t = lane & 3;   // MMA fragment row group and column pair
  // the merge grid may be scheduled once every CTA of this one has started: its CTAs then wait
  // (grid_dep_wait) on SMs this grid's last wave frees, instead of a launch after it
  grid_dep_launch_dependents();

  int bid = blockIdx.x;
  const int rb = bid % p.row_blocks;
  bid /= p.row_blocks;
  const int split = bid % p.n_splits;
  bid /= p.n_splits;
  const int hkv = bid % p.H_kv, b = bid / p.H_kv;
  const int row0 = rb * kDecRows;
  const int pos0 = p.Nk - p.Nq;   // key position of query row 0

  // bands of the block's rows: the union bounds the keys to visit, the intersection says
  // which 16-key steps need no mask
  int lo_min = INT_MAX, hi_max = -1, lo_max = 0, hi_min = INT_MAX;
  for (int lr = 0; lr < kDecRows && row0 + lr < p.rows; ++lr) {
    int lo, hi;
    dec_band(pos0 + (row0 + lr) % p.Nq, p.Nk, p.causal, p.window, lo, hi);
    lo_min = min(lo_min, lo);
    hi_max = max(hi_max, hi);
    lo_max = max(lo_max, lo);
    hi_min = min(hi_min, hi);
  }

  // this lane's rows g and g + 8 of the block (rows past the end stay unmasked, read zero Q
  // and are never written)
  int band_lo[2], band_hi[2];
  const __nv_bfloat16* qrow[2];
  for (int hf = 0; hf < 2; ++hf) {
    const int r = row0 + g + 8 * hf;
    if (r < p.rows) {
      const int hq = hkv * p.group + r / p.Nq, i = r % p.Nq;
      dec_band(pos0 + i, p.Nk, p.causal, p.window, band_lo[hf], band_hi[hf]);
      qrow[hf] = p.q + p.q_st.at(b, hq, i);
    } else {
      band_lo[hf] = INT_MIN;
      band_hi[hf] = INT_MAX;
      qrow[hf] = nullptr;
    }
  }
  // Q as the A operand of every k-step: rows g, g + 8; columns 2t, 2t + 1 (+ 8)
  auto qword = [&](const __nv_bfloat16* row, int c) -> uint32_t {
    if (!row) return 0u;
    const uint32_t w = ld_global_u32(row + c);
    if constexpr (kFp8)
      return bf16x2_to_f16x2_sat(w);
    else
      return w;
  };
  uint32_t qa[KS][4];
#pragma unroll
  for (int kk = 0; kk < KS; ++kk) {
    const int c = 16 * kk + 2 * t;
    qa[kk][0] = qword(qrow[0], c);
    qa[kk][1] = qword(qrow[1], c);
    qa[kk][2] = qword(qrow[0], c + 8);
    qa[kk][3] = qword(qrow[1], c + 8);
  }

  // this CTA's keys, in 16-key steps dealt round-robin to the warps
  const int k_begin = p.key_begin + split * p.chunk;
  const int k_end = min(p.Nk, k_begin + p.chunk);
  const int kb = max(k_begin, lo_min), ke = min(k_end - 1, hi_max);
  const int s0 = kb & ~(kDecKeys - 1);
  const int n_steps = kb <= ke ? (ke - s0) / kDecKeys + 1 : 0;
  const int my_steps = n_steps > warp ? (n_steps - warp + kDecWarps - 1) / kDecWarps : 0;

  unsigned char* ring = smem + warp * Lay::kWarpBytes;
  // lane 0: step it's K and V tiles into stage it % kDecStages; keys past N_k read as zero
  auto issue = [&](int it) {
    const int key0 = s0 + kDecKeys * (warp + kDecWarps * it);
    const uint32_t stage = smem_u32(ring + (it % kDecStages) * Lay::kStageBytes);
    const uint32_t bar = smem_u32(&bars[it % kDecStages]);
    mbar_expect_tx(bar, Lay::kStageBytes);
#pragma unroll
    for (int c = 0; c < Lay::kBoxes; ++c) {
      tma_load_rows(stage + c * Lay::kBoxBytes, &tm_k, bar, c * Lay::kBoxX, key0, hkv, b);
      tma_load_rows(stage + Lay::kKvTileBytes + c * Lay::kBoxBytes, &tm_v, bar, c * Lay::kBoxX, key0, hkv, b);
    }
  };
  // byte offset of the 16-byte piece holding elements col .. col + 7 of key row kr of a tile in a
  // stage (128-byte swizzled boxes of 64 elements), or of a converted f16 tile (padded rows)
  auto piece = [&](int kr, int col) -> int {
    if constexpr (kFp8)
      return kr * Lay::kRowBytes + col * 2;
    else
      return (col >> 6) * Lay::kBoxBytes + kr * 128 + ((((col & 63) >> 3) ^ (kr & 7)) << 4);
  };

  float acc[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};

  int issued = 0;   // lane 0's loads; every lane tracks the same count
  if (lane == 0)
    for (int it = 0; it < min(my_steps, kDecStages - 1); ++it) issue(it);
  issued = min(my_steps, kDecStages - 1);
  bool ok = true;
  int it = 0;
  for (; it < my_steps; ++it) {
    // step it has landed; the vote also puts every lane past step it - 1, whose stage the next
    // load (issued at the end of this step) overwrites
    if (!__all_sync(0xffffffffu, dec_wait(smem_u32(&bars[it % kDecStages]), (it / kDecStages) & 1, abort,
                                          p.wait_limit_ns))) {
      ok = false;
      break;
    }
    const unsigned char* ks = ring + (it % kDecStages) * Lay::kStageBytes;
    if constexpr (kFp8) {
      // E4M3 -> f16 into the converted tiles: 16 codes (one 16-byte piece) per lane at a time
      constexpr int kPieces = D / 16;
      constexpr int kPerTensor = kDecKeys * kPieces;
      unsigned char* conv = ring + kDecStages * Lay::kStageBytes;
#pragma unroll
      for (int x = 0; x < 2 * kPerTensor / 32; ++x) {
        const int c = lane + 32 * x;
        const int tensor = c / kPerTensor, rem = c % kPerTensor;
        const int row = rem / kPieces, col = rem % kPieces;
        const int src = Lay::kSwizzled ? (col >> 3) * Lay::kBoxBytes + row * 128 + (((col & 7) ^ (row & 7)) << 4)
                                       : row * D + col * 16;
        const uint4 w = *reinterpret_cast<const uint4*>(ks + tensor * Lay::kKvTileBytes + src);
        uint4 lo, hi;
        lo.x = e4m3x2_to_f16x2(w.x);
        lo.y = e4m3x2_to_f16x2(w.x >> 16);
        lo.z = e4m3x2_to_f16x2(w.y);
        lo.w = e4m3x2_to_f16x2(w.y >> 16);
        hi.x = e4m3x2_to_f16x2(w.z);
        hi.y = e4m3x2_to_f16x2(w.z >> 16);
        hi.z = e4m3x2_to_f16x2(w.w);
        hi.w = e4m3x2_to_f16x2(w.w >> 16);
        unsigned char* dst = conv + tensor * Lay::kConvTileBytes + row * Lay::kRowBytes + col * 32;
        *reinterpret_cast<uint4*>(dst) = lo;
        *reinterpret_cast<uint4*>(dst + 16) = hi;
      }
      __syncwarp();   // the converted tiles are complete for every lane
      ks = conv;
    }
    const unsigned char* vs = ks + (kFp8 ? Lay::kConvTileBytes : Lay::kKvTileBytes);
    const int key0 = s0 + kDecKeys * (warp + kDecWarps * it);

    // S = Q K^T for 16 keys: n-tiles of keys 0-7 and 8-15
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      uint32_t kf[4];   // matrices: keys 0-7 | 8-15  x  columns 16kk + 0-7 | 8-15
      ldmatrix_x4(kf, ks + piece(((lane >> 4) << 3) + (lane & 7), 16 * kk + ((lane >> 3) & 1) * 8));
      dec_mma<kFp8>(s[0], qa[kk], kf[0], kf[1]);
      dec_mma<kFp8>(s[1], qa[kk], kf[2], kf[3]);
    }
    // scale into the log2 domain; mask keys outside a row's band (and past N_k)
    const bool need_mask = key0 < lo_max || key0 + kDecKeys - 1 > hi_min;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        s[nt][c] *= p.scale_log2;
        if (need_mask) {
          const int key = key0 + 8 * nt + 2 * t + (c & 1);
          if (key < band_lo[c >> 1] || key > band_hi[c >> 1]) s[nt][c] = -INFINITY;
        }
      }
    // online softmax per row: the four lanes of a row group share it
    float alpha[2];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      float mx = fmaxf(fmaxf(s[0][2 * hf], s[0][2 * hf + 1]), fmaxf(s[1][2 * hf], s[1][2 * hf + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_run[hf], mx);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;   // a row with no key yet stays at 0
      alpha[hf] = ex2_approx(m_run[hf] - m_use);
      m_run[hf] = m_new;
      float sum = 0.f;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          s[nt][2 * hf + e] = ex2_approx(s[nt][2 * hf + e] - m_use);
          sum += s[nt][2 * hf + e];
        }
      l_run[hf] = l_run[hf] * alpha[hf] + sum;   // this lane's share; summed over the group at the end
    }
    // O = alpha O + P V; P (bf16, or f16) is the A operand straight from the S fragments
    const uint32_t pa[4] = {dec_pack<kFp8>(s[0][0], s[0][1]), dec_pack<kFp8>(s[0][2], s[0][3]),
                            dec_pack<kFp8>(s[1][0], s[1][1]), dec_pack<kFp8>(s[1][2], s[1][3])};
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      acc[j][0] *= alpha[0];
      acc[j][1] *= alpha[0];
      acc[j][2] *= alpha[1];
      acc[j][3] *= alpha[1];
    }
#pragma unroll
    for (int j = 0; j < D / 16; ++j) {
      uint32_t vf[4];   // transposed matrices: keys 0-7 | 8-15  x  columns 16j + 0-7 | 8-15
      ldmatrix_x4_trans(vf, vs + piece(((lane >> 3) & 1) * 8 + (lane & 7), 16 * j + (lane >> 4) * 8));
      dec_mma<kFp8>(acc[2 * j], pa, vf[0], vf[1]);
      dec_mma<kFp8>(acc[2 * j + 1], pa, vf[2], vf[3]);
    }
    // the next load goes into stage it - 1's slot, which every lane has left (the vote above)
    if (issued < my_steps) {
      if (lane == 0) issue(issued);
      ++issued;
    }
  }
  // after an abort, the loads still in flight land before the ring is reused or released
  if (lane == 0)
    for (int j = it; j < issued; ++j) mbar_wait_drain(smem_u32(&bars[j % kDecStages]), (j / kDecStages) & 1, p.wait_limit_ns);
  __syncwarp();
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    l_run[hf] += __shfl_xor_sync(0xffffffffu, l_run[hf], 1);
    l_run[hf] += __shfl_xor_sync(0xffffffffu, l_run[hf], 2);
  }

  // merge the four warps through shared memory (the rings are free once all warps are here)
  __syncthreads();
  float* mw = reinterpret_cast<float*>(smem) + warp * Lay::kMergeFloats;
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    *reinterpret_cast<float2*>(mw + g * D + 8 * j + 2 * t) = make_float2(acc[j][0], acc[j][1]);
    *reinterpret_cast<float2*>(mw + (g + 8) * D + 8 * j + 2 * t) = make_float2(acc[j][2], acc[j][3]);
  }
  if (t == 0) {
    mw[kDecRows * D + g] = m_run[0];
    mw[kDecRows * D + g + 8] = m_run[1];
    mw[kDecRows * D + kDecRows + g] = l_run[0];
    mw[kDecRows * D + kDecRows + g + 8] = l_run[1];
  }
  __syncthreads();

  constexpr int kPairs = D / 2;                    // column pairs per row
  constexpr int kRowSets = kDecThreads / kPairs;   // rows handled side by side
  const int cp = threadIdx.x % kPairs;
  const float* all = reinterpret_cast<const float*>(smem);
  for (int lr = threadIdx.x / kPairs; lr < kDecRows; lr += kRowSets) {
    const int r = row0 + lr;
    if (r >= p.rows) break;
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) mx = fmaxf(mx, all[w * Lay::kMergeFloats + kDecRows * D + lr]);
    float l = 0.f, o0 = 0.f, o1 = 0.f;
    if (mx != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) {
        const float* src = all + w * Lay::kMergeFloats;
        const float wt = ex2_approx(src[kDecRows * D + lr] - mx);
        l += wt * src[kDecRows * D + kDecRows + lr];
        o0 += wt * src[lr * D + 2 * cp];
        o1 += wt * src[lr * D + 2 * cp + 1];
      }
    }
    float inv = l > 0.f ? 1.f / l : 0.f;
    if constexpr (kFp8) inv *= p.v_scale;   // V = s_v V8
    const float lse = l > 0.f ? (mx + lg2_approx(l)) * kLn2 : -INFINITY;
    const int hq = hkv * p.group + r / p.Nq, i = r % p.Nq;
    const long long grow = ((long long)b * p.H + hq) * p.Nq + i;
    if (p.n_splits == 1) {
      *reinterpret_cast<uint32_t*>(p.o + p.o_st.at(b, hq, i) + 2 * cp) = pack_bf16x2(o0 * inv, o1 * inv);
      if (cp == 0) p.lse[grow] = lse;
    } else {
      const long long prow = (long long)split * p.total_rows + grow;
      *reinterpret_cast<float2*>(p.o_part + prow * D + 2 * cp) = make_float2(o0 * inv, o1 * inv);
      if (cp == 0) p.l_part[prow] = lse;
    }
  }
}

// Merge the splits of every output row: one warp per row, D / 32 (2, 4 or 8) columns per lane.  The
// lanes first read up to 32 splits' L_s at once (lane s holds split s); the O_s loads of
// eight splits are then in flight together, so the row costs a few memory latencies rather
// than one per split.
template <int D>
__global__ void __launch_bounds__(32 * kDecMergeWarps) fa_decode_merge_kernel(const DecParams p) {
  constexpr float kLn2 = 0.6931471805599453f, kLog2e = 1.4426950408889634f;
  constexpr int C = D / 32;
  grid_dep_wait();   // the splits' partial results are complete and visible
  const long long grow = (long long)blockIdx.x * kDecMergeWarps + (threadIdx.x >> 5);
  if (grow >= p.total_rows) return;   // whole warps leave together
  const int lane = threadIdx.x & 31;
  float mx = -INFINITY;
  for (int s0 = 0; s0 < p.n_splits; s0 += 32)
    if (s0 + lane < p.n_splits) mx = fmaxf(mx, p.l_part[(long long)(s0 + lane) * p.total_rows + grow]);
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
  float acc[C];
#pragma unroll
  for (int c = 0; c < C; ++c) acc[c] = 0.f;
  float sum = 0.f;
  if (mx != -INFINITY) {
    for (int s0 = 0; s0 < p.n_splits; s0 += 32) {
      const int s = s0 + lane;
      const float wt = s < p.n_splits ? ex2_approx((p.l_part[(long long)s * p.total_rows + grow] - mx) * kLog2e) : 0.f;
      sum += wt;
      const int cnt = min(32, p.n_splits - s0);
#pragma unroll 8
      for (int j = 0; j < cnt; ++j) {
        const float w = __shfl_sync(0xffffffffu, wt, j);
        const float* src = p.o_part + ((long long)(s0 + j) * p.total_rows + grow) * D + lane * C;
        if constexpr (C % 4 == 0) {
#pragma unroll
          for (int c = 0; c < C; c += 4) {
            const float4 x = *reinterpret_cast<const float4*>(src + c);
            acc[c] += w * x.x;
            acc[c + 1] += w * x.y;
            acc[c + 2] += w * x.z;
            acc[c + 3] += w * x.w;
          }
        } else {
          const float2 x = *reinterpret_cast<const float2*>(src);
          acc[0] += w * x.x;
          acc[1] += w * x.y;
        }
      }
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, m);
  }
  const float inv = sum > 0.f ? 1.f / sum : 0.f;
  const int i = int(grow % p.Nq);
  const long long bh = grow / p.Nq;
  const int b = int(bh / p.H), hq = int(bh % p.H);
  __nv_bfloat16* dst = p.o + p.o_st.at(b, hq, i) + lane * C;
  if constexpr (C % 4 == 0) {
#pragma unroll
    for (int c = 0; c < C; c += 4) {
      uint2 w;
      w.x = pack_bf16x2(acc[c] * inv, acc[c + 1] * inv);
      w.y = pack_bf16x2(acc[c + 2] * inv, acc[c + 3] * inv);
      *reinterpret_cast<uint2*>(dst + c) = w;
    }
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  }
  if (lane == 0) p.lse[grow] = sum > 0.f ? mx + lg2_approx(sum) * kLn2 : -INFINITY;
}

}  // namespace fa
