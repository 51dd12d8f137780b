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
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "params.h"

namespace moba {

constexpr int kMergeThreads = 256;
constexpr int kMergeEager = 4;  // past slots whose loads are issued before the weights

__device__ __forceinline__ void add_scaled(float (&acc)[8], float w, uint4 v) {
  const uint32_t x[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    acc[2 * e] = fmaf(w, __uint_as_float(x[e] << 16), acc[2 * e]);
    acc[2 * e + 1] = fmaf(w, __uint_as_float(x[e] & 0xFFFF0000u), acc[2 * e + 1]);
  }
}

template <int D>
__global__ void __launch_bounds__(kMergeThreads)
merge_partials_kernel(const MergeParams p) {
  constexpr int LPR = D / 8;       // lanes per row
  constexpr int RPW = 32 / LPR;    // rows per warp
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPR, v = lane % LPR;
  const int64_t warp_id = ((int64_t)blockIdx.x * kMergeThreads + threadIdx.x) >> 5;
  const int nrows = p.row_end - p.row_begin;
  const int64_t total = (int64_t)p.batch * p.hq * nrows;
  const int64_t row = warp_id * RPW + sub;
  if (sub >= RPW || row >= total) return;
  const int il = (int)(row % nrows);
  const int64_t bh = row / nrows;
  const int h = (int)(bh % p.hq), b = (int)(bh / p.hq);
  const int i = p.row_begin + il;
  const int c = i / p.block;
  const int npast = p.topk - 1;
  // Chunk-local row: the pass covers rows [row_begin, row_end) of one chunk.
  const int64_t pbase = (bh * p.chunk_rows + il) * p.topk;
  const uint4 *po = reinterpret_cast<const uint4 *>(p.opart) + pbase * LPR + v;
  // Issue the row's loads before any of them is needed.
  const int32_t *irow = p.idx + (bh * p.N + i) * p.topk;
  uint4 own = po[(int64_t)npast * LPR];
  uint4 early[kMergeEager];
#pragma unroll
  for (int s = 0; s < kMergeEager; ++s)
    if (s < npast) early[s] = po[(int64_t)s * LPR];
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
  const float lse = mx + __logf(tot);
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  add_scaled(acc, __expf(l_own - lse), own);
#pragma unroll
  for (int s = 0; s < kMergeEager; ++s)
    if (s < np) add_scaled(acc, __expf(p.lpart[pbase + s] - lse), early[s]);
  for (int s = kMergeEager; s < np; ++s)
    add_scaled(acc, __expf(p.lpart[pbase + s] - lse), po[(int64_t)s * LPR]);
  uint4 w;
  w.x = pack_bf16x2(acc[0], acc[1]);
  w.y = pack_bf16x2(acc[2], acc[3]);
  w.z = pack_bf16x2(acc[4], acc[5]);
  w.w = pack_bf16x2(acc[6], acc[7]);
  uint16_t *dst = p.out + b * p.o_sb + (int64_t)h * p.o_sh + (int64_t)i * p.o_sn + v * 8;
  *reinterpret_cast<uint4 *>(dst) = w;
  if (v == 0) p.lse[bh * p.N + i] = lse;
}

cudaError_t launch_merge(const MergeParams &p, cudaStream_t st) {
  const int64_t rows = (int64_t)p.batch * p.hq * (p.row_end - p.row_begin);
  const int rpw = 32 / (p.d / 8);
  const int64_t warps = (rows + rpw - 1) / rpw;
  const int64_t blocks = (warps * 32 + kMergeThreads - 1) / kMergeThreads;
  if (blocks <= 0) return cudaSuccess;
  switch (p.d) {
    case 64: merge_partials_kernel<64><<<(unsigned)blocks, kMergeThreads, 0, st>>>(p); break;
    case 80: merge_partials_kernel<80><<<(unsigned)blocks, kMergeThreads, 0, st>>>(p); break;
    case 128: merge_partials_kernel<128><<<(unsigned)blocks, kMergeThreads, 0, st>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace moba
