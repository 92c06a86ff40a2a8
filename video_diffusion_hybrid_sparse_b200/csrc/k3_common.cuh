// k3_common.cuh - pieces shared by the two softmax-branch kernels (bf16 and
// e4m3 operands): work-item decoding of the persistent grid and the barrier
// slots.
#pragma once

#include "kernels.h"

namespace vdn {
namespace k3 {

struct Item {
  int b, h, c, pair, ntiles;
  int row0;   // first query row of the item within the batch
  int nrows;  // rows of the item's query segment from row0 on (the tiles mask rows past it)
};

// Work items come in blocks of query segments, each block ordered (batch,
// head, segment, pair); the host chooses the blocks (plan_items in api.cu).
__device__ __forceinline__ Item decode_item(int item, const K3Params& p) {
  const Geom& g = p.g;
  int blk = 0;
  {
    int lo = 0, hi = p.n_blocks - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.blk_item0[mid] <= item) lo = mid;
      else hi = mid - 1;
    }
    blk = lo;
  }
  const int r = item - p.blk_item0[blk];
  const int s_lo = p.blk_seg0[blk], s_hi = p.blk_seg0[blk + 1];
  const int per_bh = p.seg_pair0[s_hi] - p.seg_pair0[s_lo];
  const int bh = r / per_bh;
  const int target = p.seg_pair0[s_lo] + (r - bh * per_bh);
  // segment k of the block with seg_pair0[k] <= target < seg_pair0[k + 1]
  int lo = s_lo, hi = s_hi - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.seg_pair0[mid] <= target) lo = mid;
    else hi = mid - 1;
  }
  const QSeg sg = p.segs[lo];
  Item it;
  it.b = bh / g.H;
  it.h = bh - it.b * g.H;
  it.pair = target - p.seg_pair0[lo];
  it.c = sg.c;
  it.row0 = sg.row0 + it.pair * 2 * kBlockM;
  it.nrows = sg.nrows - it.pair * 2 * kBlockM;
  it.ntiles = it.nrows > kBlockM ? 2 : 1;
  return it;
}

// Barrier slots.  kPFull + t: the first half of P_t (keys 0-63) is in TMEM;
// kPFull2 + t: the second half (both softmax kernels hand P over in halves).
enum {
  kQFull = 0, kQEmpty = 1, kKFull = 2, kKEmpty = 4, kVFull = 6, kVEmpty = 8,
  kSFull = 10, kPFull = 12, kOFull = 14, kDone = 16, kPFull2 = 17, kNumBars = 19
};

}  // namespace k3
}  // namespace vdn
