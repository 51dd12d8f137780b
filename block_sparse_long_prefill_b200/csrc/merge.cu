// merge.cu -- step 5 of the MoBA implementation ([MoBA] = "MoBA: 어텐션에 전문가 혼합을
// 적용해 긴 문맥을 효율적으로 처리하는 블록 어텐션 (feat. MoonshotAI)", §"MoBA의 구현"):
// a query attends to its own block and to several past blocks at once, so the partial
// results are combined by online softmax.  Each partial is a normalised output o_s and
// its log-sum-exp l_s; the merged row is
//     lse = log sum_s exp(l_s),   out = sum_s exp(l_s - lse) o_s.
//
// A streaming kernel: LPR = d/8 lanes cover one row with 16-byte vectors, so every
// partial row (slots contiguous per row) and the output row move in coalesced
// 16-byte accesses; the per-row weights are computed redundantly by those lanes.
// Warps walk the rows grid-stride.
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "params.h"

namespace moba {

constexpr int kMergeThreads = 256;
// Past slots whose loads are issued before the weights: 4, or 12 for long lists (all of
// a row's partial loads in flight at once, for fewer resident warps).

__device__ __forceinline__ void add_scaled(float (&acc)[8], float w, uint4 v) {
  const uint32_t x[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    acc[2 * e] = fmaf(w, __uint_as_float(x[e] << 16), acc[2 * e]);
    acc[2 * e + 1] = fmaf(w, __uint_as_float(x[e] & 0xFFFF0000u), acc[2 * e + 1]);
  }
}

// One row: LPR lanes (a sub-group) own 16 bytes of the row each.  Lane v of the
// sub-group also loads block choice v and partial log-sum-exp v of the row (v < topk,
// for topk <= LPR), so that every load of the row is in flight at once.  Lane v then
// computes the weight of slot v alone (one exponential), and the sub-group shares the
// maximum, the sum and the weights with shuffles.  Row indices fit 32 bits: the host
// bounds batch * hq * N below 2^31 whenever partials exist.
template <int D, int kMergeEager>
__device__ __forceinline__ void merge_row(const MergeParams &p, int row, int nrows, int v,
                                          unsigned gmask, int gbase) {
  constexpr int LPR = D / 8;
  const int bh = row / nrows, il = row - bh * nrows;
  const int h = bh % p.hq, b = bh / p.hq;
  const int i = p.row_begin + il;
  const int c = (p.q_off + i) / p.block;  // own block of the row's key position
  const int npast = p.topk - 1;
  // Chunk-local row: the pass covers rows [row_begin, row_end) of one chunk.
  const int64_t pbase = ((int64_t)bh * p.chunk_rows + il) * p.topk;
  const uint4 *po = reinterpret_cast<const uint4 *>(p.opart) + pbase * LPR + v;
  const int32_t *irow = p.idx + ((int64_t)bh * p.N + i) * p.topk;
  const bool spread = p.topk <= LPR;
  int my_blk = -1;
  float my_l = 0.f;
  if (spread && v < p.topk) {
    my_blk = __ldg(irow + v);
    my_l = p.lpart[pbase + v];
  }
  const uint4 own = po[(int64_t)npast * LPR];
  uint4 early[kMergeEager];
#pragma unroll
  for (int s = 0; s < kMergeEager; ++s)
    if (s < npast) early[s] = po[(int64_t)s * LPR];
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  float lse;
  if (spread) {
    // Valid past slots: the leading choices below the own block; slot npast is the
    // own block.
    const bool bad = v < npast && (my_blk < 0 || my_blk >= c);
    const unsigned badm = (__ballot_sync(gmask, bad) >> gbase) & ((1u << LPR) - 1u);
    const int np = badm ? (__ffs(badm) - 1) : npast;
    float mx = -INFINITY;
    for (int s = 0; s < p.topk; ++s) {
      const float ls = __shfl_sync(gmask, my_l, gbase + s);
      if (s < np || s == npast) mx = fmaxf(mx, ls);
    }
    const float e_mine = (v < np || v == npast) ? __expf(my_l - mx) : 0.f;
    float tot = 0.f;
    for (int s = 0; s < p.topk; ++s) tot += __shfl_sync(gmask, e_mine, gbase + s);
    const float inv = 1.f / tot;
    lse = mx + __logf(tot);
    add_scaled(acc, __shfl_sync(gmask, e_mine, gbase + npast) * inv, own);
#pragma unroll
    for (int s = 0; s < kMergeEager; ++s) {
      if (s < npast) {
        const float w = __shfl_sync(gmask, e_mine, gbase + s) * inv;
        if (s < np) add_scaled(acc, w, early[s]);
      }
    }
    for (int s = kMergeEager; s < npast; ++s) {
      const float w = __shfl_sync(gmask, e_mine, gbase + s) * inv;
      if (s < np) add_scaled(acc, w, po[(int64_t)s * LPR]);
    }
  } else {
    int np = 0;
    for (int s = 0; s < npast; ++s) {
      const int blk = __ldg(irow + s);
      if (blk < 0 || blk >= c) break;
      ++np;
    }
    const float l_own = p.lpart[pbase + npast];
    float mx = l_own;
    for (int s = 0; s < np; ++s) mx = fmaxf(mx, p.lpart[pbase + s]);
    float tot = __expf(l_own - mx);
    for (int s = 0; s < np; ++s) tot += __expf(p.lpart[pbase + s] - mx);
    lse = mx + __logf(tot);
    add_scaled(acc, __expf(l_own - lse), own);
#pragma unroll
    for (int s = 0; s < kMergeEager; ++s)
      if (s < np) add_scaled(acc, __expf(p.lpart[pbase + s] - lse), early[s]);
    for (int s = kMergeEager; s < np; ++s)
      add_scaled(acc, __expf(p.lpart[pbase + s] - lse), po[(int64_t)s * LPR]);
  }
  uint4 w;
  w.x = pack_bf16x2(acc[0], acc[1]);
  w.y = pack_bf16x2(acc[2], acc[3]);
  w.z = pack_bf16x2(acc[4], acc[5]);
  w.w = pack_bf16x2(acc[6], acc[7]);
  uint16_t *dst = p.out + b * p.o_sb + (int64_t)h * p.o_sh + (int64_t)i * p.o_sn + v * 8;
  *reinterpret_cast<uint4 *>(dst) = w;
  if (v == 0) p.lse[(int64_t)bh * p.N + i] = lse;
}

template <int D, int EAGER>
__global__ void __launch_bounds__(kMergeThreads)
merge_partials_kernel(const MergeParams p) {
  constexpr int LPR = D / 8;       // lanes per row
  constexpr int RPW = 32 / LPR;    // rows per warp
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPR, v = lane % LPR;
  if (sub >= RPW) return;          // D = 80: the last two lanes idle
  const int gbase = sub * LPR;
  const unsigned gmask = (LPR == 32 ? 0xffffffffu : ((1u << LPR) - 1u)) << gbase;
  const int nwarps = (int)((gridDim.x * kMergeThreads) >> 5);
  const int warp_id = (int)((blockIdx.x * kMergeThreads + threadIdx.x) >> 5);
  const int nrows = p.row_end - p.row_begin;
  const int total = p.batch * p.hq * nrows;
  // Rows warp_id * RPW + sub, then a grid-stride walk.
  for (int row = warp_id * RPW + sub; row < total; row += nwarps * RPW)
    merge_row<D, EAGER>(p, row, nrows, v, gmask, gbase);
}

cudaError_t launch_merge(const MergeParams &p, cudaStream_t st) {
  const int64_t rows = (int64_t)p.batch * p.hq * (p.row_end - p.row_begin);
  const int rpw = 32 / (p.d / 8);
  const int64_t warps = (rows + rpw - 1) / rpw;
  int64_t blocks = (warps * 32 + kMergeThreads - 1) / kMergeThreads;
  // Enough CTAs to fill every SM several times over; each warp then walks rows.
  int dev = 0, nsm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int64_t cap = (int64_t)nsm * 8 * 4;
  if (blocks > cap) blocks = cap;
  if (blocks <= 0) return cudaSuccess;
  const bool long_list = p.topk - 1 > 4;
  switch (p.d) {
    case 64:
      if (long_list) merge_partials_kernel<64, 12><<<(unsigned)blocks, kMergeThreads, 0, st>>>(p);
      else merge_partials_kernel<64, 4><<<(unsigned)blocks, kMergeThreads, 0, st>>>(p);
      break;
    case 80:
      if (long_list) merge_partials_kernel<80, 12><<<(unsigned)blocks, kMergeThreads, 0, st>>>(p);
      else merge_partials_kernel<80, 4><<<(unsigned)blocks, kMergeThreads, 0, st>>>(p);
      break;
    case 128:
      if (long_list) merge_partials_kernel<128, 12><<<(unsigned)blocks, kMergeThreads, 0, st>>>(p);
      else merge_partials_kernel<128, 4><<<(unsigned)blocks, kMergeThreads, 0, st>>>(p);
      break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace moba
