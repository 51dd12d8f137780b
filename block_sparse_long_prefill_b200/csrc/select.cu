// select.cu -- MoBA selection stage on sm_100a: key mean-pooling, gate scores with
// causal block masking, per-row top-k, and the block-major dispatch lists.
//
// [MoBA] = "MoBA: 어텐션에 전문가 혼합을 적용해 긴 문맥을 효율적으로 처리하는 블록 어텐션
//          (feat. MoonshotAI)", PyTorch KR forum summary of the MoBA paper.
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "lists.cuh"
#include "params.h"

namespace moba {

// ------------------------------------------------------------------ pooling
//
// [MoBA] §"블록 분할과 top-k 게이팅": MeanPool(K[I_j]) over the keys of block j
// (positions [j*block, min((j+1)*block, N)): a partial last block when block does
// not divide N).  One CTA per (block, kv-head, batch).  Threads read 16-byte vectors along d
// (coalesced rows), accumulate in fp32, and reduce across row groups in a fixed
// order (deterministic).  Also writes the split hi = bf16(mean), lo = bf16(mean - hi)
// that the gate multiplies with on the tensor cores.
constexpr int kPoolThreads = 256;

__global__ void __launch_bounds__(kPoolThreads)
pool_keys_kernel(const uint16_t *__restrict__ k, int64_t sb, int64_t sh, int64_t sn, int hkv,
                 int d, int block, int N, int nblk, float *__restrict__ kbar,
                 uint16_t *__restrict__ split) {
  extern __shared__ float red[];  // [ngroups][d]
  const int j = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int vpr = d >> 3;                   // 16-byte vectors per key row
  const int ngroups = kPoolThreads / vpr;   // rows read concurrently
  const int t = threadIdx.x;
  const int vec = t % vpr, grp = t / vpr;
  const int len = min(block, N - j * block);  // keys in this block
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  if (grp < ngroups) {
    const uint16_t *base = k + b * sb + hk * sh + (int64_t)j * block * sn + vec * 8;
    int r = grp;
    for (; r + 7 * ngroups < len; r += 8 * ngroups) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        v[u] = __ldg(reinterpret_cast<const uint4 *>(base + (int64_t)(r + u * ngroups) * sn));
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[2 * e] += __uint_as_float(w[e] << 16);
          acc[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
        }
      }
    }
    for (; r < len; r += ngroups) {
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(base + (int64_t)r * sn));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] += __uint_as_float(w[e] << 16);
        acc[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[grp * d + vec * 8 + e] = acc[e];
  }
  __syncthreads();
  const int64_t bh = (int64_t)b * hkv + hk;
  for (int c = t; c < d; c += kPoolThreads) {
    float s = 0.f;
    for (int g = 0; g < ngroups; ++g) s += red[g * d + c];
    const float mean = s / (float)len;
    kbar[(bh * nblk + j) * d + c] = mean;
    const __nv_bfloat16 hi = __float2bfloat16_rn(mean);
    const __nv_bfloat16 lo = __float2bfloat16_rn(mean - __bfloat162float(hi));
    uint16_t *sp = split + bh * 2 * (int64_t)nblk * d;
    sp[(int64_t)j * d + c] = __bfloat16_as_ushort(hi);
    sp[((int64_t)nblk + j) * d + c] = __bfloat16_as_ushort(lo);
  }
}

// Min/max pooling (the MoBA page: Quest is MoBA with smaller blocks and a min/max
// pooled block representation): kmax_j and kmin_j, the element-wise maximum and minimum
// of the keys of block j, written as bf16 planes [batch, hkv, 2, nblk, d] (plane 0 the
// maxima, plane 1 the minima; exact, the keys are bf16).  Same CTA layout as the mean.
__global__ void __launch_bounds__(kPoolThreads)
pool_minmax_kernel(const uint16_t *__restrict__ k, int64_t sb, int64_t sh, int64_t sn, int hkv,
                   int d, int block, int N, int nblk, uint16_t *__restrict__ planes) {
  extern __shared__ float red[];  // [2][ngroups][d]
  const int j = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int vpr = d >> 3;
  const int ngroups = kPoolThreads / vpr;
  const int t = threadIdx.x;
  const int vec = t % vpr, grp = t / vpr;
  const int len = min(block, N - j * block);
  float mx[8], mn[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) { mx[e] = -INFINITY; mn[e] = INFINITY; }
  if (grp < ngroups) {
    const uint16_t *base = k + b * sb + hk * sh + (int64_t)j * block * sn + vec * 8;
    for (int r = grp; r < len; r += ngroups) {
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(base + (int64_t)r * sn));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float lo = __uint_as_float(w[e] << 16), hi = __uint_as_float(w[e] & 0xFFFF0000u);
        mx[2 * e] = fmaxf(mx[2 * e], lo);
        mn[2 * e] = fminf(mn[2 * e], lo);
        mx[2 * e + 1] = fmaxf(mx[2 * e + 1], hi);
        mn[2 * e + 1] = fminf(mn[2 * e + 1], hi);
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      red[grp * d + vec * 8 + e] = mx[e];
      red[(ngroups + grp) * d + vec * 8 + e] = mn[e];
    }
  }
  __syncthreads();
  const int64_t bh = (int64_t)b * hkv + hk;
  uint16_t *pl = planes + bh * 2 * (int64_t)nblk * d;
  for (int c = t; c < d; c += kPoolThreads) {
    float a = -INFINITY, z = INFINITY;
    for (int g = 0; g < ngroups; ++g) {
      a = fmaxf(a, red[g * d + c]);
      z = fminf(z, red[(ngroups + g) * d + c]);
    }
    // Exact: a and z are bf16 values.
    pl[(int64_t)j * d + c] = (uint16_t)(__float_as_uint(a) >> 16);
    pl[((int64_t)nblk + j) * d + c] = (uint16_t)(__float_as_uint(z) >> 16);
  }
}

// ------------------------------------------------------------ gate + top-k
//
// [MoBA] §"블록 분할과 top-k 게이팅": s_j = <q, MeanPool(K[I_j])>, unscaled;
// §"인과성 보존": only blocks j < c = i / block compete, block c is always kept.
// One CTA = 64 query rows of one (batch, q-head); 4 warps of 16 rows.
//
// Scores come from bf16 tensor-core MMAs (mma.sync m16n8k16, fp32 accumulate):
// q is exactly bf16, and kbar = hi + lo to about 2^-17 relative, so
// s = q.hi + q.lo is fp32-accurate -- far inside the 1e-3 gate-gap tolerance.
// The selection is k-1 rounds of a quad-wide arg-max over the row's scores in
// shared memory (ties to the lower block), then a rank placement into ascending
// order.  Each CTA also counts its picks per past block (shared-memory histogram,
// one global atomic per non-empty block) for the dispatch lists.
constexpr int kGateRows = 64;
constexpr int kGateThreads = 128;
constexpr int kGateChunk = 32;  // pooled blocks staged per pass

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t &r0, uint32_t &r1,
                                            uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int D>
__global__ void __launch_bounds__(kGateThreads)
gate_topk_kernel(const SelectParams p) {
  constexpr int KS = D / 16;           // k-steps
  constexpr int LDK = D + 8;           // padded row stride (elements): conflict-free ldmatrix
  extern __shared__ __align__(128) unsigned char smem[];
  uint16_t *ks = reinterpret_cast<uint16_t *>(smem);                       // [2][32][LDK]
  float *ss = reinterpret_cast<float *>(ks + 2 * kGateChunk * LDK);        // [64][lds]
  const int i0 = blockIdx.x * kGateRows;
  const int h = blockIdx.y, b = blockIdx.z;
  const int hk = h / p.G;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rows = min(kGateRows, p.N - i0);
  // Past blocks any row of this tile may score (query row i sits at key position
  // q_off + i).
  const int nb = min(p.nblk, (p.q_off + i0 + rows - 1) / p.block);
  const int lds = ((nb + 31) & ~31) + 4;
  int *hist = reinterpret_cast<int *>(ss + kGateRows * lds);               // [nblk]
  const int wr0 = warp * 16;  // this warp's first row in the tile
  const int g = lane >> 2, t4 = lane & 3;

  // Query fragments straight from global memory (every load in flight at once):
  // A of m16n8k16 holds rows g, g+8 and columns 2*t4 (+1), (+8) of each 16-wide step.
  uint32_t afrag[KS][4];
  {
    const uint16_t *qg = p.q + b * p.q_sb + h * p.q_sh;
    const int ra = i0 + wr0 + g, rb = ra + 8;
    const bool va = ra < p.N, vb = rb < p.N;
    const uint32_t *qa = reinterpret_cast<const uint32_t *>(qg + (int64_t)(va ? ra : 0) * p.q_sn);
    const uint32_t *qb = reinterpret_cast<const uint32_t *>(qg + (int64_t)(vb ? rb : 0) * p.q_sn);
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      const int w0 = s * 8 + t4;  // 32-bit word of column s*16 + 2*t4
      afrag[s][0] = va ? __ldg(qa + w0) : 0u;
      afrag[s][1] = vb ? __ldg(qb + w0) : 0u;
      afrag[s][2] = va ? __ldg(qa + w0 + 4) : 0u;
      afrag[s][3] = vb ? __ldg(qb + w0 + 4) : 0u;
    }
  }
  for (int j = tid; j < p.nblk; j += kGateThreads) hist[j] = 0;

  const uint16_t *kb = p.kbar_split + ((int64_t)b * p.hkv + hk) * 2 * p.nblk * D;
  // Largest own-block index among this warp's rows: n-tiles at or past it are skipped.
  const int wlast = min(i0 + wr0 + 15, p.N - 1);
  const int cw = (wr0 < rows) ? (p.q_off + wlast) / p.block : 0;
  const int nchunk = (nb + kGateChunk - 1) / kGateChunk;
  for (int ch = 0; ch < nchunk; ++ch) {
    const int j0 = ch * kGateChunk;
    if (ch > 0) __syncthreads();  // previous chunk's ldmatrix reads are done
    for (int e = tid; e < 2 * kGateChunk * (D / 8); e += kGateThreads) {
      const int part = e / (kGateChunk * (D / 8));
      const int rem = e % (kGateChunk * (D / 8));
      const int jj = rem / (D / 8), c = rem % (D / 8);
      const bool ok = j0 + jj < nb;
      const uint16_t *src = kb + ((int64_t)part * p.nblk + (ok ? j0 + jj : 0)) * D + c * 8;
      cp_async_16_zfill(smem_u32(ks + (part * kGateChunk + jj) * LDK + c * 8), src, ok);
    }
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();
    // n-tiles of 8 blocks this warp needs in this chunk (warp-uniform).
    const int ntc = min(kGateChunk / 8, max(0, (cw - j0 + 7) / 8));
    float acc_hi[kGateChunk / 8][4], acc_lo[kGateChunk / 8][4];
#pragma unroll
    for (int nt = 0; nt < kGateChunk / 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) { acc_hi[nt][e] = 0.f; acc_lo[nt][e] = 0.f; }
#pragma unroll
    for (int s = 0; s < KS; ++s) {
#pragma unroll
      for (int nt = 0; nt < kGateChunk / 8; ++nt) {
        if (nt < ntc) {
          // Matrices: (hi, k0..7), (hi, k8..15), (lo, k0..7), (lo, k8..15) for 8 blocks.
          const int part = (lane >> 4) & 1;
          const int jj = nt * 8 + (lane & 7);
          const int c = s * 16 + 8 * ((lane >> 3) & 1);
          uint32_t h0, h1, l0, l1;
          ldmatrix_x4(smem_u32(ks + (part * kGateChunk + jj) * LDK + c), h0, h1, l0, l1);
          if (p.minmax) {
            // max(q_d kmax_d, q_d kmin_d) = q+_d kmax_d + q-_d kmin_d: the positive part
            // of q against the maxima, the negative part against the minima (exact).
            uint32_t ap[4], an[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162 *>(&afrag[s][e]);
              const __nv_bfloat162 z = __float2bfloat162_rn(0.f);
              const __nv_bfloat162 xp = __hmax2(x, z), xn = __hmin2(x, z);
              ap[e] = *reinterpret_cast<const uint32_t *>(&xp);
              an[e] = *reinterpret_cast<const uint32_t *>(&xn);
            }
            mma_bf16_16816(acc_hi[nt], ap, h0, h1);
            mma_bf16_16816(acc_lo[nt], an, l0, l1);
          } else {
            mma_bf16_16816(acc_hi[nt], afrag[s], h0, h1);
            mma_bf16_16816(acc_lo[nt], afrag[s], l0, l1);
          }
        }
      }
    }
#pragma unroll
    for (int nt = 0; nt < kGateChunk / 8; ++nt) {
      if (nt < ntc) {
        const int col = j0 + nt * 8 + 2 * t4;
        ss[(wr0 + g) * lds + col] = acc_hi[nt][0] + acc_lo[nt][0];
        ss[(wr0 + g) * lds + col + 1] = acc_hi[nt][1] + acc_lo[nt][1];
        ss[(wr0 + g + 8) * lds + col] = acc_hi[nt][2] + acc_lo[nt][2];
        ss[(wr0 + g + 8) * lds + col + 1] = acc_hi[nt][3] + acc_lo[nt][3];
      }
    }
  }
  cp_async_wait_all();
  __syncthreads();

  // Top-(k-1) over past blocks; one quad of lanes per row, two passes of 8 rows.
  // Every lane runs the warp's largest round count so the shuffles stay converged.
  const int npick_max = p.topk - 1;
  int *sel_base = reinterpret_cast<int *>(ks);  // reuses the key staging: [64][32]
  for (int pass = 0; pass < 2; ++pass) {
    const int r = wr0 + pass * 8 + g;
    const int i = i0 + r;
    const bool live = r < rows;
    const int c = live ? (p.q_off + i) / p.block : 0;
    float *srow = ss + r * lds;
    int *sel = sel_base + r * 32;
    const int npick = min(npick_max, c);
    const int rounds = (live && c > npick_max) ? npick : 0;
    const int wrounds = __reduce_max_sync(0xffffffffu, rounds);
    for (int round = 0; round < wrounds; ++round) {
      float best = -INFINITY;
      int bj = 0x7fffffff;
      if (round < rounds) {
        for (int j = t4; j < c; j += 4) {
          const float v = srow[j];
          if (v > best) { best = v; bj = j; }
        }
      }
#pragma unroll
      for (int off = 1; off <= 2; off <<= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, off);
        const int oj = __shfl_xor_sync(0xffffffffu, bj, off);
        if (ob > best || (ob == best && oj < bj)) { best = ob; bj = oj; }
      }
      if (round < rounds) {
        if (bj != 0x7fffffff && (bj & 3) == t4) srow[bj] = -INFINITY;
        if (t4 == 0) sel[round] = bj;
      }
      __syncwarp();
    }
    __syncwarp();
    if (live) {
      int32_t *orow = p.idx + (((int64_t)b * p.hq + h) * p.N + i) * p.topk;
      if (c <= npick_max) {
        for (int s = t4; s < p.topk; s += 4) orow[s] = (s < c) ? s : (s == c ? c : -1);
        for (int j = t4; j < c; j += 4) atomicAdd(&hist[j], 1);
      } else {
        for (int s = t4; s < npick; s += 4) {
          const int v = sel[s];
          int rank = 0;
          for (int u = 0; u < npick; ++u) rank += sel[u] < v;
          orow[rank] = v;
          atomicAdd(&hist[v], 1);
        }
        if (t4 == 0) orow[npick] = c;
        for (int s = npick + 1 + t4; s < p.topk; s += 4) orow[s] = -1;
      }
    }
  }
  __syncthreads();
  // One global atomic per (list, CTA).
  const int chunk = i0 / p.chunk_rows;
  int *cnt = p.counts + (((int64_t)chunk * p.batch + b) * p.hkv + hk) * p.nblk;
  for (int j = tid; j < nb; j += kGateThreads)
    if (hist[j]) atomicAdd(&cnt[j], hist[j]);
}

// ------------------------------------------------------------- list offsets
//
// Exclusive prefix sums of the list counts (entries) and of their 256-entry units,
// over all lists in (chunk, batch, kv-head, block) order; resets the scatter
// cursors.  One CTA.  (The unit table that these offsets index is written by the
// scatter kernel's grid.)
constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads)
list_scan_kernel(const int *__restrict__ counts, int *__restrict__ cursor, int *__restrict__ listoff,
                 int *__restrict__ tileoff, int nlists) {
  __shared__ int sh[2 * kScanThreads / 32];
  scan_lists<kScanThreads>(counts, cursor, listoff, tileoff, nlists, sh);
}

// ----------------------------------------------------------------- scatter
//
// [MoBA] §"MoBA의 구현", steps 1-2: assign each (query, q-head) to the KV blocks it
// picked and regroup the queries by block.  One CTA = 128 rows x all G q-heads of one
// kv-head.  Entries of one CTA reserve their places with one atomic per block.
// The order of entries inside a list is not fixed; no result depends on it (each
// row's attention is computed independently of the rows sharing its tile).
//
// The CTA's block choices are read once into shared memory when they fit.
// The grid also writes the unit table: one {list, first entry, rows} record per unit
// of up to 256 entries (two 128-row tiles over the same block), so the attention
// kernel reads a unit's description with a single load.
constexpr int kScatterThreads = 256;
constexpr size_t kScatterCacheBytes = 96 * 1024;

__global__ void __launch_bounds__(kScatterThreads)
scatter_kernel(const ScatterParams p) {
  extern __shared__ int sh[];
  int *hist = sh;             // [nblk]
  int *base = sh + p.nblk;    // [nblk]
  int *picks = sh + 2 * p.nblk;  // [G][128][ps] when p.cache_rows (ps = topk | 1: rows of a
                                 // warp start in distinct banks)
  const int ps = p.topk | 1;
  const int i0 = blockIdx.x * kTileRows;
  const int hk = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const int npast = p.topk - 1;
  const int rows = min(kTileRows, p.N - i0);
  const int nb = min(p.nblk, (p.q_off + i0 + rows - 1) / p.block);

  {
    // Unit table, grid-stride over the lists.
    const long long nthreads = (long long)gridDim.x * gridDim.y * gridDim.z * kScatterThreads;
    const long long gtid =
        (((long long)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x) * kScatterThreads + tid;
    for (long long L = gtid; L < p.nlists; L += nthreads) {
      const int first = p.listoff[L], cnt = p.counts[L], t0 = p.tileoff[L];
      for (int k = 0; k * kUnitRows < cnt; ++k)
        p.tiles[t0 + k] = make_int4((int)L, first + k * kUnitRows, min(kUnitRows, cnt - k * kUnitRows), 0);
    }
  }

  for (int j = tid; j < nb; j += kScatterThreads) hist[j] = 0;
  const int64_t head0 = ((int64_t)b * p.hq + (int64_t)hk * p.G) * p.N + i0;  // row (b, hk*G, i0)
  if (p.cache_rows) {
    // Each head's rows i0 .. i0 + rows - 1 are one contiguous run of rows * topk words.
    const int run = rows * p.topk;
    for (int g = 0; g < p.G; ++g) {
      const int32_t *src = p.idx + (head0 + (int64_t)g * p.N) * p.topk;
      for (int e = tid; e < run; e += kScatterThreads) {
        const int r = e / p.topk;
        picks[(g * kTileRows + r) * ps + (e - r * p.topk)] = src[e];
      }
    }
  }
  __syncthreads();
  // Pair e = (g, r) of the tile; a warp holds 32 rows of one head (128 % 32 == 0).
  const int pairs = p.G * kTileRows;
  auto pick = [&](int g, int r, int s) -> int {
    return p.cache_rows ? picks[(g * kTileRows + r) * ps + s]
                        : p.idx[(head0 + (int64_t)g * p.N + r) * p.topk + s];
  };
  for (int e = tid; e < pairs; e += kScatterThreads) {
    const int g = e / kTileRows, r = e % kTileRows;
    const bool row_ok = r < rows;
    const int c = (p.q_off + i0 + r) / p.block;
    for (int s = 0; s < npast; ++s) {
      const int j = row_ok ? pick(g, r, s) : -1;
      // Past picks come first; the own block and the -1 padding end them.
      if (j < 0 || j >= c) break;
      atomicAdd(&hist[j], 1);
    }
  }
  __syncthreads();
  const int chunk = i0 / p.chunk_rows;
  int *cur = p.cursor + (((int64_t)chunk * p.batch + b) * p.hkv + hk) * p.nblk;
  for (int j = tid; j < nb; j += kScatterThreads) {
    base[j] = hist[j] ? atomicAdd(&cur[j], hist[j]) : 0;
    hist[j] = 0;
  }
  __syncthreads();
  for (int e = tid; e < pairs; e += kScatterThreads) {
    const int g = e / kTileRows, r = e % kTileRows;
    const bool row_ok = r < rows;
    const int i = i0 + r;
    const int c = (p.q_off + i) / p.block;
    for (int s = 0; s < npast; ++s) {
      const int j = row_ok ? pick(g, r, s) : -1;
      if (j < 0 || j >= c) break;
      const int pos = base[j] + atomicAdd(&hist[j], 1);
      p.entries[pos] = (uint32_t)(((int64_t)i * p.G + g) * npast + s);
    }
  }
}

// ------------------------------------------------------------ static gates
//
// [MoBA] §"MoBA의 구현" preamble: sliding-window attention is MoBA whose gate always
// picks the most recent blocks; an attention sink is MoBA whose gate picks the first
// block together with the most recent ones.  Row i (own block c) keeps block c, the
// first `sink` blocks and the k-1-sink most recent blocks before c (all past blocks
// when c <= k-1).  The choice depends on c alone.  One CTA = one 128-row tile of one
// (batch, kv-head): the tile's rows have own block c0 = (q_off + i0) / block, or c0 + 1
// past a block boundary inside the tile (block >= 128); it writes the tile's G * 128
// idx rows and adds, per own block, its rows times G to the list count of every past
// pick.
constexpr int kStaticThreads = 256;

// Entry s of the choice list of a row whose own block is c.
__device__ __forceinline__ int static_pick(int c, int s, int npast, int sink) {
  const int recent = npast - sink;
  if (c <= npast) return s < c ? s : (s == c ? c : -1);
  if (s < sink) return s;
  if (s < npast) return c - recent + (s - sink);
  return s == npast ? c : -1;
}

__global__ void __launch_bounds__(kStaticThreads)
static_select_kernel(int32_t *__restrict__ idx, int *__restrict__ counts, int batch, int hq,
                     int hkv, int N, int q_off, int block, int topk, int sink, int nblk,
                     int chunk_rows) {
  const int i0 = blockIdx.x * kTileRows;
  const int hk = blockIdx.y, b = blockIdx.z;
  const int G = hq / hkv;
  const int rows = min(kTileRows, N - i0);
  const int c0 = (q_off + i0) / block;
  // Rows [0, rows0) of the tile sit in block c0, the rest in c0 + 1.
  const int rows0 = min(rows, (c0 + 1) * block - (q_off + i0));
  const int npast = topk - 1;
  // Each head's rows i0 .. i0 + rows - 1 are one contiguous run of rows * topk words.
  const int run = rows * topk;
  for (int g = 0; g < G; ++g) {
    int32_t *dst = idx + (((int64_t)b * hq + (int64_t)hk * G + g) * N + i0) * topk;
    for (int e = threadIdx.x; e < run; e += kStaticThreads) {
      const int r = e / topk;
      dst[e] = static_pick(r < rows0 ? c0 : c0 + 1, e - r * topk, npast, sink);
    }
  }
  const int chunk = i0 / chunk_rows;
  int *cnt = counts + (((int64_t)chunk * batch + b) * hkv + hk) * nblk;
  for (int part = 0; part < 2; ++part) {
    const int c = c0 + part;
    const int nr = part ? rows - rows0 : rows0;
    if (nr <= 0 || (int)threadIdx.x >= npast) continue;
    const int j = static_pick(c, threadIdx.x, npast, sink);
    if (j >= 0 && j < c) atomicAdd(&cnt[j], nr * G);
  }
}

cudaError_t launch_static_select(int32_t *idx, int *counts, int batch, int hq, int hkv, int N,
                                 int q_off, int block, int topk, int sink, int nblk, int chunk_rows,
                                 cudaStream_t st) {
  dim3 grid((N + kTileRows - 1) / kTileRows, hkv, batch);
  static_select_kernel<<<grid, kStaticThreads, 0, st>>>(idx, counts, batch, hq, hkv, N, q_off,
                                                        block, topk, sink, nblk, chunk_rows);
  return cudaGetLastError();
}

// Host-side launchers (called by the ABI layer).
cudaError_t launch_pool(const uint16_t *k, int64_t sb, int64_t sh, int64_t sn, int batch, int hkv,
                        int N, int d, int block, float *kbar, uint16_t *split, cudaStream_t st) {
  const int nblk = (N + block - 1) / block;
  const int ngroups = kPoolThreads / (d / 8);
  const size_t smem = sizeof(float) * ngroups * d;
  dim3 grid(nblk, hkv, batch);
  pool_keys_kernel<<<grid, kPoolThreads, smem, st>>>(k, sb, sh, sn, hkv, d, block, N, nblk, kbar,
                                                      split);
  return cudaGetLastError();
}

cudaError_t launch_pool_minmax(const uint16_t *k, int64_t sb, int64_t sh, int64_t sn, int batch,
                               int hkv, int N, int d, int block, uint16_t *planes, cudaStream_t st) {
  const int nblk = (N + block - 1) / block;
  const int ngroups = kPoolThreads / (d / 8);
  const size_t smem = sizeof(float) * 2 * ngroups * d;
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(pool_minmax_kernel,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(nblk, hkv, batch);
  pool_minmax_kernel<<<grid, kPoolThreads, smem, st>>>(k, sb, sh, sn, hkv, d, block, N, nblk, planes);
  return cudaGetLastError();
}

size_t gate_smem_bytes(int d, int nblk) {
  const int ldk = d + 8;
  const int lds = ((nblk + 31) & ~31) + 4;
  // Key staging (also holds the 64 x 32 selection scratch afterwards), scores, counts.
  const size_t stage = sizeof(uint16_t) * 2 * kGateChunk * ldk;
  const size_t sel = sizeof(int) * kGateRows * 32;
  return (stage > sel ? stage : sel) + sizeof(float) * kGateRows * lds + sizeof(int) * nblk;
}

template <int D>
static cudaError_t launch_gate_d(const SelectParams &p, cudaStream_t st) {
  const size_t smem = gate_smem_bytes(D, p.nblk);
  cudaError_t e = cudaFuncSetAttribute(gate_topk_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((p.N + kGateRows - 1) / kGateRows, p.hq, p.batch);
  gate_topk_kernel<D><<<grid, kGateThreads, smem, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gate(const SelectParams &p, cudaStream_t st) {
  switch (p.d) {
    case 64: return launch_gate_d<64>(p, st);
    case 80: return launch_gate_d<80>(p, st);
    case 128: return launch_gate_d<128>(p, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_scan(const int *counts, int *cursor, int *listoff, int *tileoff, int nlists,
                        cudaStream_t st) {
  list_scan_kernel<<<1, kScanThreads, 0, st>>>(counts, cursor, listoff, tileoff, nlists);
  return cudaGetLastError();
}

cudaError_t launch_scatter(ScatterParams p, cudaStream_t st) {
  dim3 grid((p.N + kTileRows - 1) / kTileRows, p.hkv, p.batch);
  const size_t cache = sizeof(int) * (size_t)p.G * kTileRows * (p.topk | 1);
  // Staging pays for itself when a row has several picks to read twice.
  p.cache_rows = (p.topk - 1 >= 4 && cache <= kScatterCacheBytes) ? 1 : 0;
  const size_t smem = sizeof(int) * 2 * p.nblk + (p.cache_rows ? cache : 0);
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem);
    if (e != cudaSuccess) return e;
  }
  scatter_kernel<<<grid, kScatterThreads, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace moba
