// Work-item schedule of the persistent kernels: which CTA of the grid takes which item.
#pragma once

namespace fa {

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
