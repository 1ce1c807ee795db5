// Work-item schedule of the one-item-per-CTA kernels: which CTA of a grid takes which item.
#pragma once

namespace fa {

// Heads per chunk of the one-item-per-CTA grids (grid_item): the forward's chunks are query
// heads, the backward's K/V heads.  Large enough that the costliest items of a chunk fill most
// of the 148 SMs' first wave; small enough that the chunk's K/V (forward) or Q, dO and dQ
// accumulator (backward) stay well inside the 126 MB L2.  Measured on a B200 (causal N4096 and
// the N32768 causal band): 8 forward heads beat 16 and 32 by 1-1.5 %; 8 and 16 K/V heads tie
// in the backward.
constexpr int kFwdChunkHeads = 8;
constexpr int kBwdChunkHeads = 8;

// Item (head, pos) of CTA `blk` in a grid of n_heads * n_pos CTAs, where pos 0 is a head's
// costliest item and costs fall with pos (causal masks, band edges).  The hardware starts CTAs
// in index order, so the index order is the run order.  Heads are taken in chunks of `chunk`,
// and inside a chunk position-major: pos 0 of every head of the chunk, then pos 1, and so on.
// The costly items then start first across the chunk, and the cheap ones fill the gaps at its
// end, instead of every head's costly item starting just behind the previous head's cheap ones
// (which leaves the last heads' costly items to run alone after everything else).  With every
// cost alike the order only regroups heads.  The last chunk may hold fewer heads.
__device__ __forceinline__ void grid_item(int blk, int n_heads, int n_pos, int chunk, int& head,
                                          int& pos) {
  const int per_chunk = chunk * n_pos;
  const int c = blk / per_chunk;
  const int r = blk - c * per_chunk;
  const int in_chunk = min(chunk, n_heads - c * chunk);
  pos = r / in_chunk;
  head = c * chunk + (r - pos * in_chunk);
}

}  // namespace fa
