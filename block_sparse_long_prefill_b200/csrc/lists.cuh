// lists.cuh -- exclusive prefix sums of the block-major dispatch list counts.
//
// [MoBA] = "MoBA: 어텐션에 전문가 혼합을 적용해 긴 문맥을 효율적으로 처리하는 블록 어텐션
// (feat. MoonshotAI)", §"MoBA의 구현", step 2: the queries that picked a block are
// regrouped by block; the lists are laid out one after another, so each list's first
// entry is the exclusive prefix sum of the counts before it.
#pragma once

#include <stdint.h>

#include "params.h"

namespace moba {

// Run by all NT threads of one CTA.  For every list L in (chunk, batch, kv-head,
// block) order: listoff[L] = cursor[L] = entries of the lists before L, tileoff[L] =
// their 256-entry units; listoff[nlists] and tileoff[nlists] are the totals.  Thread
// t takes a contiguous run of lists (its loads of the counts are independent), then
// the runs' totals are scanned across the CTA.  `sh` holds 2 * NT / 32 ints.  The
// counts are read through L2 (they were produced by other CTAs' atomics).
template <int NT>
__device__ __forceinline__ void scan_lists(const int *counts, int *cursor, int *listoff,
                                           int *tileoff, int nlists, int *sh) {
  static_assert(NT % 32 == 0 && NT <= 1024, "whole warps");
  constexpr int NW = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (nlists + NT - 1) / NT;
  const int l0 = min(nlists, tid * per), l1 = min(nlists, l0 + per);
  int se = 0, st = 0;
  for (int L = l0; L < l1; ++L) {
    const int c = __ldcg(counts + L);
    se += c;
    st += (c + kUnitRows - 1) / kUnitRows;
  }
  int ie = se, it = st;  // inclusive within the warp
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int ye = __shfl_up_sync(0xffffffffu, ie, off);
    const int yt = __shfl_up_sync(0xffffffffu, it, off);
    if (lane >= off) { ie += ye; it += yt; }
  }
  int *we = sh, *wt = sh + NW;
  if (lane == 31) { we[warp] = ie; wt[warp] = it; }
  __syncthreads();
  if (warp == 0) {
    int xe = lane < NW ? we[lane] : 0, xt = lane < NW ? wt[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int ye = __shfl_up_sync(0xffffffffu, xe, off);
      const int yt = __shfl_up_sync(0xffffffffu, xt, off);
      if (lane >= off) { xe += ye; xt += yt; }
    }
    if (lane < NW) { we[lane] = xe; wt[lane] = xt; }  // inclusive warp totals
  }
  __syncthreads();
  int pe = (warp ? we[warp - 1] : 0) + ie - se;
  int pt = (warp ? wt[warp - 1] : 0) + it - st;
  for (int L = l0; L < l1; ++L) {
    const int c = __ldcg(counts + L);
    listoff[L] = pe;
    cursor[L] = pe;
    tileoff[L] = pt;
    pe += c;
    pt += (c + kUnitRows - 1) / kUnitRows;
  }
  if (tid == NT - 1) {
    listoff[nlists] = pe;
    tileoff[nlists] = pt;
  }
}

}  // namespace moba
