// TEST INFRASTRUCTURE ONLY: the one-item-per-CTA kernels' work-item schedule (grid_item of
// grid_sched.cuh, compiled from the library's own source) evaluated on the host.
//
// For several head counts, items per head and chunk sizes it checks that every CTA index maps to
// a distinct (head, position) in range, and prints one line per case with the makespan of the
// causal forward's pair costs under the hardware's in-order dispatch, for the chunked order and
// for the head-major one.
// usage: emu_sched_main   (exit 1 at the first violation)
#include "emu.h"
#include "sm100.cuh"
#include "grid_sched.cuh"

#include <algorithm>
#include <cstdio>
#include <vector>

using namespace fa;

int main() {
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
                            {33, 7, 8},  {64, 16, 8}, {64, 32, 8}, {100, 2, 8}, {16, 128, 8}};
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
