// TEST INFRASTRUCTURE ONLY: the persistent kernels' work-item schedules (persist_item, and
// fwd_item of fwd_persist_kernel.cuh / bwd_item of bwd_persist_kernel.cuh, compiled from the
// kernels' own source) evaluated on the host for many shapes, grid sizes and both item orders.
//
// For each case it checks that the CTAs' item lists together hold every (head, query-tile pair)
// exactly once, that a CTA's list ends at its first -1 (no later round yields an item), and that
// every item's K/V tile ranges are the ones kv_tile_range gives its two query tiles.  It prints
// one line per case: BH N causal window order grid, the largest CTA load and the mean load, in
// K/V tile steps plus one per item.  Then the same coverage check for the backward's items
// (K/V head, key tile) with q_tile_range's query tiles, for 1, 2 and 4 query heads per K/V
// head, printing "bwd" lines with the loads in query iterations plus one per item; and for the
// d = 256 forward's items (head, 128-row query tile) with kv_tile_range256's 64-key tiles,
// printing "f256" lines.
// usage: emu_sched_main   (exit 1 at the first violation)
#include "emu.h"
#include "fwd_persist_kernel.cuh"
#include "bwd_persist_kernel.cuh"
#include "fwd256_persist_kernel.cuh"

#include <algorithm>
#include <cstdio>
#include <vector>

namespace fa {
// the shared memory the (never launched) d = 256 kernels refer to; this program only walks schedules
alignas(1024) uint8_t smem_raw[1024];
}  // namespace fa

using namespace fa;

int main() {
  struct Shape {
    int BH, N, causal, window;
  };
  const Shape shapes[] = {{1, 1, 1, 0},       {1, 128, 0, 0},     {1, 300, 1, 0},        {3, 700, 1, 0},
                          {4, 520, 1, 100},   {4, 400, 0, 50},    {5, 1000, 1, 1},       {2, 257, 0, 0},
                          {64, 4096, 1, 0},   {64, 4096, 0, 0},   {16, 32768, 1, 4096},  {16, 32768, 0, 4096},
                          {128, 1024, 1, 0},  {7, 3000, 1, 600}};
  const unsigned grids[] = {1, 2, 3, 5, 7, 64, 148, 1000};
  for (const Shape& sh : shapes) {
    FwdParams prm{};
    prm.N = sh.N;
    prm.BH = sh.BH;
    prm.H = sh.BH;
    prm.group = 1;
    prm.causal = sh.causal;
    prm.window = std::min(sh.window, sh.N);
    prm.n_pairs = ((sh.N + kBlockM - 1) / kBlockM + kQTiles - 1) / kQTiles;
    const int n_items = prm.n_pairs * prm.BH;
    for (int order : {int(kOrderHeadMajor), int(kOrderPairMajor)}) {
      for (unsigned G : grids) {
        const unsigned g = std::min<unsigned>(G, unsigned(n_items));   // the launch's clamp
        gridDim = dim3s{g, 1, 1};
        std::vector<int> seen(n_items, 0);
        long long max_load = 0, total = 0;
        for (unsigned cta = 0; cta < g; ++cta) {
          blockIdx = dim3s{cta, 0, 0};
          long long load = 0;
          int r = 0;
          for (;; ++r) {
            const int pos = persist_item(n_items, r);
            if (pos < 0) break;
            if (pos >= n_items) {
              std::printf("FAIL position %d out of range\n", pos);
              return 1;
            }
            const FwdItem it = fwd_item(prm, order, pos);
            const int pair = it.q0 / (kQTiles * kBlockM);
            if (it.bh < 0 || it.bh >= prm.BH || pair < 0 || pair >= prm.n_pairs ||
                it.q0 != pair * kQTiles * kBlockM || it.b_idx != it.bh / prm.H || it.h_q != it.bh % prm.H) {
              std::printf("FAIL bad item at position %d\n", pos);
              return 1;
            }
            int b0, e0, b1, e1;
            kv_tile_range(it.q0, prm.N, prm.causal, prm.window, b0, e0);
            kv_tile_range(it.q0 + kBlockM, prm.N, prm.causal, prm.window, b1, e1);
            if (e1 == 0) b1 = e1 = b0;
            if (it.b0 != b0 || it.e0 != e0 || it.b1 != b1 || it.e1 != e1 || it.t_begin != b0 ||
                it.t_end != std::max(e0, e1)) {
              std::printf("FAIL tile ranges of item (%d, %d)\n", it.bh, pair);
              return 1;
            }
            ++seen[it.bh * prm.n_pairs + pair];
            load += (it.t_end - it.t_begin) + 1;
          }
          for (int rr = r + 1; rr < r + 4; ++rr)
            if (persist_item(n_items, rr) >= 0) {
              std::printf("FAIL CTA %u has an item after its list ended\n", cta);
              return 1;
            }
          max_load = std::max(max_load, load);
          total += load;
        }
        for (int i = 0; i < n_items; ++i)
          if (seen[i] != 1) {
            std::printf("FAIL item %d taken %d times (BH %d N %d order %d grid %u)\n", i, seen[i], sh.BH, sh.N,
                        order, g);
            return 1;
          }
        std::printf("%d %d %d %d %d %u %lld %.3f\n", sh.BH, sh.N, sh.causal, sh.window, order, g, max_load,
                    double(total) / g);
      }
    }
  }
  // the backward: BH here counts query heads; the items are (K/V head, key tile)
  for (const Shape& sh : shapes) {
    for (int group : {1, 2, 4}) {
      if (sh.BH % group) continue;
      BwdParams prm{};
      prm.N = sh.N;
      prm.BH = sh.BH;
      prm.H = sh.BH;   // one batch entry
      prm.H_kv = sh.BH / group;
      prm.group = group;
      prm.causal = sh.causal;
      prm.window = std::min(sh.window, sh.N);
      prm.n_kv_tiles = (sh.N + kBwdKeys - 1) / kBwdKeys;
      const int n_items = prm.n_kv_tiles * prm.H_kv;
      for (int order : {int(kOrderHeadMajor), int(kOrderPairMajor)}) {
        for (unsigned G : grids) {
          const unsigned g = std::min<unsigned>(G, unsigned(n_items));
          gridDim = dim3s{g, 1, 1};
          std::vector<int> seen(n_items, 0);
          long long max_load = 0, total = 0;
          for (unsigned cta = 0; cta < g; ++cta) {
            blockIdx = dim3s{cta, 0, 0};
            long long load = 0;
            for (int r = 0;; ++r) {
              const int pos = persist_item(n_items, r);
              if (pos < 0) break;
              const BwdItem it = bwd_item(prm, order, pos);
              const int tile = it.kv0 / kBwdKeys;
              int ib, ie;
              q_tile_range(it.kv0, prm.N, prm.causal, prm.window, ib, ie);
              if (it.b_idx != 0 || it.h_kv < 0 || it.h_kv >= prm.H_kv || tile < 0 || tile >= prm.n_kv_tiles ||
                  it.kv0 != tile * kBwdKeys || it.i_begin != ib || it.n_i != ie - ib || it.n_i < 1 ||
                  it.n_it != it.n_i * group || it.bh_q0 != it.h_kv * group ||
                  bwd_q_head(it, group, it.n_it - 1) != it.bh_q0 + group - 1 ||
                  bwd_q_tile(it, group, it.n_it - 1) != ie - 1) {
                std::printf("FAIL bwd item at position %d\n", pos);
                return 1;
              }
              ++seen[it.h_kv * prm.n_kv_tiles + tile];
              load += it.n_it + 1;
            }
            max_load = std::max(max_load, load);
            total += load;
          }
          for (int i = 0; i < n_items; ++i)
            if (seen[i] != 1) {
              std::printf("FAIL bwd item %d taken %d times\n", i, seen[i]);
              return 1;
            }
          std::printf("bwd %d %d %d %d %d %d %u %lld %.3f\n", sh.BH, group, sh.N, sh.causal, sh.window, order, g,
                      max_load, double(total) / g);
        }
      }
    }
  }
  // the d = 256 forward: one 128-row query tile per item
  for (const Shape& sh : shapes) {
    FwdParams prm{};
    prm.N = sh.N;
    prm.BH = sh.BH;
    prm.H = sh.BH;
    prm.group = 1;
    prm.causal = sh.causal;
    prm.window = std::min(sh.window, sh.N);
    prm.n_pairs = (sh.N + k256BlockM - 1) / k256BlockM;
    const int n_items = prm.n_pairs * prm.BH;
    for (int order : {int(kOrderHeadMajor), int(kOrderPairMajor)}) {
      for (unsigned G : grids) {
        const unsigned g = std::min<unsigned>(G, unsigned(n_items));
        gridDim = dim3s{g, 1, 1};
        std::vector<int> seen(n_items, 0);
        long long max_load = 0, total = 0;
        for (unsigned cta = 0; cta < g; ++cta) {
          blockIdx = dim3s{cta, 0, 0};
          long long load = 0;
          for (int r = 0;; ++r) {
            const int pos = persist_item(n_items, r);
            if (pos < 0) break;
            const Fwd256Item it = fwd256_item(prm, order, pos);
            const int tile = it.q0 / k256BlockM;
            int tb, te;
            kv_tile_range256(it.q0, prm.N, prm.causal, prm.window, tb, te);
            if (it.bh < 0 || it.bh >= prm.BH || tile < 0 || tile >= prm.n_pairs || it.q0 != tile * k256BlockM ||
                it.t_begin != tb || it.t_end != te || te <= tb) {
              std::printf("FAIL f256 item at position %d\n", pos);
              return 1;
            }
            ++seen[it.bh * prm.n_pairs + tile];
            load += (te - tb) + 1;
          }
          max_load = std::max(max_load, load);
          total += load;
        }
        for (int i = 0; i < n_items; ++i)
          if (seen[i] != 1) {
            std::printf("FAIL f256 item %d taken %d times\n", i, seen[i]);
            return 1;
          }
        std::printf("f256 %d %d %d %d %d %u %lld %.3f\n", sh.BH, sh.N, sh.causal, sh.window, order, g, max_load,
                    double(total) / g);
      }
    }
  }
  // The one-item-per-CTA grids (grid_item): every CTA index maps to a distinct (head, pos) in
  // range for head counts that are and are not multiples of the chunk.  For the causal forward's
  // pair costs (query tiles' K/V steps plus one), print the makespan of CTAs started in index
  // order on 148 SMs, each SM taking the next CTA when its previous one ends: "grid heads n_pos
  // chunk makespan_chunked makespan_head_major mean".
  {
    struct GridCase {
      int heads, n_pos, chunk;
    };
    const GridCase gcs[] = {{1, 1, 16}, {1, 16, 16}, {5, 3, 16}, {16, 16, 16}, {17, 4, 16}, {64, 16, 16},
                            {33, 7, 8},  {16, 32, 8}, {64, 32, 8}, {100, 2, 8}, {16, 128, 16}};
    for (const GridCase& gc : gcs) {
      const int n = gc.heads * gc.n_pos;
      std::vector<int> seen(n, 0);
      std::vector<long long> cost_chunked(n), cost_head(n);
      for (int blk = 0; blk < n; ++blk) {
        int head = -1, pos = -1;
        grid_item(blk, gc.heads, gc.n_pos, gc.chunk, head, pos);
        if (head < 0 || head >= gc.heads || pos < 0 || pos >= gc.n_pos) {
          std::printf("FAIL grid item of CTA %d: head %d pos %d\n", blk, head, pos);
          return 1;
        }
        ++seen[head * gc.n_pos + pos];
        const int pair = gc.n_pos - 1 - pos;   // forward: pos 0 is the last (longest) causal pair
        cost_chunked[blk] = 2 * pair + 2 + 1;
        const int hm_pair = gc.n_pos - 1 - blk % gc.n_pos;
        cost_head[blk] = 2 * hm_pair + 2 + 1;
      }
      for (int i = 0; i < n; ++i)
        if (seen[i] != 1) {
          std::printf("FAIL grid item %d taken %d times\n", i, seen[i]);
          return 1;
        }
      auto makespan = [](const std::vector<long long>& cost) {
        std::vector<long long> sm(148, 0);
        long long end = 0;
        for (long long c : cost) {
          auto it = std::min_element(sm.begin(), sm.end());
          *it += c;
          end = std::max(end, *it);
        }
        return end;
      };
      long long total = 0;
      for (long long c : cost_chunked) total += c;
      std::printf("grid %d %d %d %lld %lld %.3f\n", gc.heads, gc.n_pos, gc.chunk, makespan(cost_chunked),
                  makespan(cost_head), double(total) / 148);
    }
  }
  return 0;
}
