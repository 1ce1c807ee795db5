// Work-item schedules: which CTA of a grid takes which work item, for the one-item-per-CTA
// kernels (grid_item) and for the persistent kernels (persist_item).
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

// Orders of the work items.  Head-major keeps the items that run at the same time on few heads
// (their K/V, or Q/dO, stay in L2); the cost-major order puts the longest item of every head
// first, so that items come in decreasing cost when the mask makes the cost depend on the
// position (causal, or a band whose edge tiles are short).
enum : int { kOrderHeadMajor = 0, kOrderPairMajor = 1 };

// The r-th item of this CTA, as a position in the item order, or -1 when it has no r-th item.
// Rounds of gridDim.x items are dealt out in a snake (round 0 to CTAs 0, 1, ..., round 1 to
// CTAs G-1, G-2, ...), so that in a cost-decreasing order a CTA that took a costly item in one
// round takes a cheap one in the next.  Positions grow with r, so the first -1 ends the list.
__device__ __forceinline__ int persist_item(int n_items, int r) {
  const long long g = gridDim.x;
  const long long pos = (long long)r * g + ((r & 1) ? g - 1 - blockIdx.x : blockIdx.x);
  return pos < n_items ? int(pos) : -1;
}

}  // namespace fa
