// bwd.cu -- backward of MoBA attention on sm_100a tensor cores (tcgen05 + TMEM).
//
// [MoBA] = "MoBA: 어텐션에 전문가 혼합을 적용해 긴 문맥을 효율적으로 처리하는 블록 어텐션
//          (feat. MoonshotAI)", PyTorch KR forum summary of the MoBA paper.
//
// §"MoBA와 전체 어텐션의 하이브리드" trains models whose layers are MoBA attention, so
// gradients flow through it.  The gate is a parameter-free top-k and passes no
// gradient: for the block choice the forward made, the layer is softmax attention over
// each row's key set J_i.  With z_ij = scale q_i.k_j, p_ij = exp(z_ij - lse_i) and the
// upstream gradient dO:
//     D_i = dO_i . o_i,  dp_ij = dO_i . v_j,  dz_ij = p_ij (dp_ij - D_i)
//     dQ_i = scale sum_j dz_ij k_j,  dK_j = scale sum_i dz_ij q_i,  dV_j = sum_i p_ij dO_i
// The work follows the forward's decomposition (§"MoBA의 구현"): the past blocks a row
// picked are whole blocks reached through the block-major dispatch lists of the
// selection step, and the own block is causal.
//
// Four kernels, no atomics:
//   bwd_prep_kernel   per row: lse in log2 units and D_i = dO_i . o_i (from the bf16 o)
//   bwd_dq_kernel     query-stationary: a 128-row tile (128 entries of a block list
//                     against their past block, or 128 contiguous rows against their
//                     own block, causal) walks the block's 128-key chunks:
//                     S = Q K^T, dP = dO V^T (tensor cores, TMEM), dS = P (dP - D) on
//                     the CUDA cores (thread r = row r), dQ += dS K (tensor cores);
//                     the row's dQ over that block is an fp32 partial, one slot per block
//   bwd_dkdv_kernel   key-stationary: a unit is one 128-key tile of one block and one KV
//                     head; it walks every 128-row query tile that attends the tile (the
//                     block's lists over all query chunks, then the block's own rows of
//                     every q-head of the group, causal on the diagonal tile):
//                     S^T = K Q^T, dP^T = V dO^T, P^T and dS^T (thread r = key r),
//                     dV += P^T dO, dK += dS^T Q, accumulated in TMEM over the whole walk
//                     and written once
//   bwd_dq_merge_kernel  dQ_i = scale * (sum of the row's slots)
// Roles in both tile kernels: warp 0 TMA loads of K/V, warp 1 the tcgen05 issuer and
// TMEM owner, warps 2-3 the cp.async gather of the query-side rows (Q, dO, row
// statistics) into the 128-byte-swizzled tile layout, warps 4-11 the elementwise work
// (two warp groups over the same TMEM lanes, one per half of the 128 columns: the
// backward needs no reduction along a row, so the columns split freely).
// Every wait is bounded (2 s), as in the forward.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "params.h"

namespace moba {

constexpr int kBwdThreads = 384;

// Tile geometry: a 128-row bf16 tile of D columns is stored as 64-column regions of
// 128-byte rows with the 128-byte swizzle (the TMA layout the forward uses).
template <int D>
struct BwdTile {
  static constexpr int R0 = 128 * 128;              // bytes of one 64-column region
  static constexpr int TILE = 128 * D * 2;          // bytes of a 128 x D tile
  static constexpr uint32_t BYTES = 128u * D * 2u;
};

// K-major operand (rows = M or N, K = the D columns): k-step ks of 16 columns.
template <int D>
__device__ __forceinline__ uint64_t bwd_kmajor_desc(uint32_t tile, int ks) {
  if (ks < 4) return smem_desc(tile + ks * 32, 16, 1024, kSwizzle128);
  return smem_desc(tile + BwdTile<D>::R0 + (ks - 4) * 32, 16, 1024, kSwizzle128);
}

// MN-major B operand over the tile's rows (the K dimension of the product): rows
// [16 kk, 16 kk + 16), all D columns (for D = 128 the second 64-column region is one
// leading-byte offset away).
template <int D>
__device__ __forceinline__ uint64_t bwd_mn_desc(uint32_t tile, int kk) {
  if (D == 128) return smem_desc(tile + kk * 2048, BwdTile<D>::R0, 1024, kSwizzle128);
  return smem_desc(tile + kk * 2048, 16, 1024, kSwizzle128);
}

// ------------------------------------------------------------------ prep

// rowstat[(b * hq + h) * N + i] = (lse_i * log2(e), D_i = dO_i . o_i), one warp per row
// group: D / 8 lanes per row with 16-byte loads.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwdParams p) {
  constexpr int LPR = D / 8, RPW = 32 / LPR;
  const int lane = threadIdx.x & 31, sub = lane / LPR, v = lane % LPR;
  const int gw = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int nw = (int)((gridDim.x * blockDim.x) >> 5);
  const long long total = (long long)p.batch * p.hq * p.N;
  for (long long row = (long long)gw * RPW + sub; row - sub < total; row += (long long)nw * RPW) {
    const bool ok = row < total;
    float acc = 0.f;
    long long bh = 0;
    int i = 0;
    if (ok) {
      bh = row / p.N;
      i = (int)(row - bh * p.N);
      const int b = (int)(bh / p.hq), h = (int)(bh % p.hq);
      const uint4 o = *reinterpret_cast<const uint4 *>(p.out + b * p.o_sb + h * p.o_sh +
                                                       (int64_t)i * p.o_sn + v * 8);
      const uint4 g = *reinterpret_cast<const uint4 *>(p.dout + b * p.do_sb + h * p.do_sh +
                                                       (int64_t)i * p.do_sn + v * 8);
      const uint32_t ov[4] = {o.x, o.y, o.z, o.w}, gv[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc = fmaf(__uint_as_float(ov[e] << 16), __uint_as_float(gv[e] << 16), acc);
        acc = fmaf(__uint_as_float(ov[e] & 0xFFFF0000u), __uint_as_float(gv[e] & 0xFFFF0000u), acc);
      }
    }
#pragma unroll
    for (int off = 1; off < LPR; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (ok && v == 0)
      p.rowstat[row] = make_float2(p.lse[row] * 1.4426950408889634f, acc);
  }
}

// ------------------------------------------------------------------ shared state

struct BwdBars {
  uint64_t q_full[2], q_empty[2];   // query-side tile (Q, dO, row statistics) per stage
  uint64_t k_full[3], k_empty[3], v_full[3], v_empty[3];
  uint64_t s_full[2], ds_full[2];   // per half: S / dP ready; dS (and P) written back
  uint64_t acc_full, acc_empty;     // accumulators final / read out
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

// One query tile of a work item: gathered entries of a block list, or contiguous rows.
struct BwdRows {
  int gathered;   // 1: entries [ent0, ent0 + rows) of the list storage
  int ent0;
  int b, h, row0; // contiguous rows row0 .. row0 + rows - 1 of (b, h)
  int rows;
};

// Row r of a query tile: (b, h, i) and the partial slot of the block (gathered: the
// entry's slot; contiguous: the own-block slot npast).
__device__ __forceinline__ void tile_row(const BwdParams &p, const BwdRows &t, int hk, int r,
                                         int &h, int &i, int &slot) {
  if (t.gathered) {
    const uint32_t ent = __ldg(p.entries + t.ent0 + r);
    slot = (int)(ent % (uint32_t)p.npast);
    const uint32_t ig = ent / (uint32_t)p.npast;
    h = hk * p.G + (int)(ig % (uint32_t)p.G);
    i = (int)(ig / (uint32_t)p.G);
  } else {
    h = t.h;
    i = t.row0 + r;
    slot = p.npast;
  }
}

// Gather of a query tile by the 64 threads of warps 2-3: warp w (0 or 1) copies tile
// rows [64 w, 64 w + 64).  Lane l decodes rows 64 w + 2 l and 64 w + 2 l + 1 (the list
// entries of a gathered tile are global loads, so the next tile's rows are decoded while
// the gather waits for a free stage) and leaves their source rows in the warp's table in
// shared memory; the copies then go eight lanes to a row, each lane 16 bytes of a 128-byte
// row segment, so that one warp instruction moves four whole segments (coalesced).
struct GatherRows {
  const float2 *st[2];
  bool valid[2];
};

struct RowSrc {
  const uint16_t *q, *g;   // source rows of Q and dO, or null (a row past the tile's end)
};

__device__ __forceinline__ void decode_rows(const BwdParams &p, const BwdRows &t, int b, int hk,
                                            int gt, RowSrc *tab, GatherRows &gr, bool prefetch = false) {
  const int w = gt >> 5, l = gt & 31;
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    const int r = 64 * w + 2 * l + x;
    gr.valid[x] = r < t.rows;
    int h = 0, i = 0, slot = 0;
    if (gr.valid[x]) tile_row(p, t, hk, r, h, i, slot);
    const int bb = t.gathered ? b : t.b;
    RowSrc src;
    src.q = gr.valid[x] ? p.q + bb * p.q_sb + (int64_t)h * p.q_sh + (int64_t)i * p.q_sn : nullptr;
    src.g = gr.valid[x] ? p.dout + bb * p.do_sb + (int64_t)h * p.do_sh + (int64_t)i * p.do_sn : nullptr;
    // (dQ pass) The rows go into L2 now: their copies wait for the current tile to
    // release the buffer, and then read L2 instead of DRAM.
    if (prefetch && gr.valid[x]) {
      prefetch_l2_bulk(src.q, (uint32_t)p.d * 2u);
      prefetch_l2_bulk(src.g, (uint32_t)p.d * 2u);
    }
    tab[r] = src;
    gr.st[x] = p.rowstat + ((int64_t)bb * p.hq + h) * p.N + i;
  }
  __syncwarp();
}

__device__ __forceinline__ void cp_async_8(uint32_t dst_smem, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst_smem), "l"(src) : "memory");
}

// Issues the copies of the warp's 64 decoded rows into a query tile: Q and dO rows into
// the swizzled tiles, the row statistics into `stats` (rows past the tile's end: zero
// rows and lse = +inf, so that p = 0 there), as one cp.async group; land_tile then waits
// for the group and arrives once on `full` (64 arrivals complete it).
template <int D>
__device__ __forceinline__ void issue_rows(const BwdParams &p, const GatherRows &gr,
                                           const RowSrc *tab, uint32_t qt, uint32_t dot,
                                           float2 *stats, int gt) {
  const int w = gt >> 5, l = gt & 31;
  const int cc = l & 7;                      // 16-byte chunk of a 128-byte row segment
#pragma unroll 4
  for (int s4 = 0; s4 < 16; ++s4) {
    const int r = 64 * w + 4 * s4 + (l >> 3);
    const RowSrc src = tab[r];
    const bool valid = src.q != nullptr;
#pragma unroll
    for (int rg = 0; rg < D / 64; ++rg) {
      const uint32_t off = rg * BwdTile<D>::R0 + r * 128 + ((cc ^ (r & 7)) << 4);
      cp_async_16_zfill(qt + off, valid ? src.q + rg * 64 + cc * 8 : p.q, valid);
      cp_async_16_zfill(dot + off, valid ? src.g + rg * 64 + cc * 8 : p.dout, valid);
    }
  }
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    const int r = 64 * w + 2 * l + x;
    if (gr.valid[x]) cp_async_8(smem_u32(stats + r), gr.st[x]);
    else stats[r] = make_float2(INFINITY, 0.f);
  }
  cp_async_commit();
  __syncwarp();   // the table is read; the next decode may overwrite it
}

__device__ __forceinline__ void land_tile(uint64_t *full) {
  cp_async_wait_all();
  fence_proxy_async_smem();
  mbar_arrive(full);
}

// ------------------------------------------------------------------ dQ

// Work item u of the dQ pass: u < 2 * units -> half (u & 1) of gathered unit u / 2 of the
// forward's unit table (entries of one block list, one past block); else a contiguous
// 128-row tile of one (b, h) against its own block.
struct DqItem {
  BwdRows t;
  int b, hk;
  int key0, nc;   // keys [key0, key0 + 128 nc)
  int causal;     // own block: mask keys after the row
};

__device__ __forceinline__ bool dq_item(const BwdParams &p, int u, int ngath, DqItem &it) {
  if (u < 2 * ngath) {
    const int4 rec = __ldg(p.tiles + (u >> 1));
    const int x = u & 1;
    const int L = rec.x;
    const int j = L % p.nblk;
    it.hk = (L / p.nblk) % p.hkv;
    it.b = (L / (p.nblk * p.hkv)) % p.batch;
    it.t.gathered = 1;
    it.t.ent0 = rec.y + x * 128;
    it.t.rows = min(128, rec.z - x * 128);
    it.t.b = it.b;
    it.t.h = 0;
    it.t.row0 = 0;
    it.key0 = j * p.block;
    it.nc = p.block / kTileKeys;
    it.causal = 0;
    return it.t.rows > 0;
  }
  u -= 2 * ngath;
  const int nrt = (p.N + 127) / 128;
  const int rt = nrt - 1 - u % nrt;            // later (heavier) tiles first
  const int bh = u / nrt;
  it.b = bh / p.hq;
  const int h = bh % p.hq;
  it.hk = h / p.G;
  it.t.gathered = 0;
  it.t.ent0 = 0;
  it.t.b = it.b;
  it.t.h = h;
  it.t.row0 = rt * 128;
  it.t.rows = min(128, p.N - rt * 128);
  it.key0 = (it.t.row0 / p.block) * p.block;
  it.nc = (it.t.row0 + it.t.rows - 1 - it.key0) / kTileKeys + 1;
  it.causal = 1;
  return true;
}

template <int D>
struct DqCfg {
  static constexpr int ST = (D == 128) ? 2 : 3;
  static constexpr int Q_OFF = 0;
  static constexpr int DO_OFF = BwdTile<D>::TILE;
  static constexpr int K_OFF = 2 * BwdTile<D>::TILE;
  static constexpr int V_OFF = K_OFF + ST * BwdTile<D>::TILE;
  static constexpr int ST_OFF = V_OFF + ST * BwdTile<D>::TILE;   // float2 stats [128]
  static constexpr int TAB_OFF = ST_OFF + 128 * 8;                 // RowSrc [128]
  static constexpr int STG_OFF = TAB_OFF + 128 * 16;              // 8 warps x 32 rows x 64 B
  static constexpr int BAR_OFF = STG_OFF + 8 * 2048;
  static constexpr int SMEM = BAR_OFF + 1024 + 1024;
};

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_dq_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
              const BwdParams p) {
  using C = DqCfg<D>;
  using T = BwdTile<D>;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char *sbase = smem_raw + (base - raw);
  BwdBars &bar = *reinterpret_cast<BwdBars *>(sbase + C::BAR_OFF);
  float2 *stats = reinterpret_cast<float2 *>(sbase + C::ST_OFF);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int site0 = (8 * 16 + (D == 64 ? 0 : 2)) * 256;
  constexpr uint32_t FULL = 0xffffffffu;
  const int ngath = (p.npast > 0) ? __ldg(p.tileoff + p.nlists) : 0;
  const int nitems = 2 * ngath + p.batch * p.hq * ((p.N + 127) / 128);

  if (tid == 0) {
    mbar_init(&bar.q_full[0], 64);
    mbar_init(&bar.q_empty[0], 1);
    for (int s = 0; s < 3; ++s) {
      mbar_init(&bar.k_full[s], 1);
      mbar_init(&bar.k_empty[s], 1);
      mbar_init(&bar.v_full[s], 1);
      mbar_init(&bar.v_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bar.s_full[x], 1);
      mbar_init(&bar.ds_full[x], 128);
    }
    mbar_init(&bar.acc_full, 1);
    mbar_init(&bar.acc_empty, 256);
    mbar_init(&bar.mma_done, 1);
    bar.abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(&bar.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;
  volatile int *abort = &bar.abort;
  // TMEM: S [0, 128), dP [128, 256), dQ [256, 256 + D).

  if (warp == 0) {
    // ------------------------------------------------------------ K / V loads
    if (lane < 2) {
      const bool kside = lane == 0;
      uint64_t *full = kside ? bar.k_full : bar.v_full;
      uint64_t *empty = kside ? bar.k_empty : bar.v_empty;
      const CUtensorMap *m = kside ? &tmK : &tmV;
      const int off = kside ? C::K_OFF : C::V_OFF;
      uint32_t cnt = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < nitems; u += gridDim.x) {
        DqItem it;
        if (!dq_item(p, u, ngath, it)) continue;
        for (int m2 = 0; m2 < it.nc; ++m2, ++cnt) {
          const int st = cnt % C::ST;
          if (!(ok = mbar_wait(&empty[st], ((cnt / C::ST) & 1) ^ 1, abort, p.status, site0 + 1))) break;
          unsigned char *dst = sbase + off + st * T::TILE;
          mbar_arrive_expect_tx(&full[st], T::BYTES);
          const int key = it.key0 + m2 * kTileKeys;
          tma_load_4d(dst, m, &full[st], 0, key, it.hk, it.b);
          if (D == 128) tma_load_4d(dst + T::R0, m, &full[st], 64, key, it.hk, it.b);
        }
      }
      if (*abort) {
        for (uint32_t u = (cnt > (uint32_t)C::ST ? cnt - C::ST : 0); u < cnt; ++u) {
          const unsigned long long t0 = global_timer_ns();
          while (!mbar_try_wait(&full[u % C::ST], (u / C::ST) & 1) && global_timer_ns() - t0 < wait_limit_ns(p.status)) {}
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // Each 128-key chunk is taken as two 64-key halves x, one per elementwise warp
      // group, each with its own TMEM buffer: S_x at 128 x, dP_x at 128 x + 64; dQ at
      // 256.  While one group works on its half, the tensor core computes the other's.
      constexpr uint32_t idS = idesc_bf16(128, 64, 0, 0);
      constexpr uint32_t idQ = idesc_bf16(128, D, 0, 1);
      const uint32_t tQ = tmem + 256;
      const uint32_t qt = base + C::Q_OFF, dot = base + C::DO_OFF;
      uint32_t kvc = 0, qn = 0, an = 0;
      uint32_t sc[2] = {0u, 0u};
      bool ok = true;
      for (int u = blockIdx.x; ok && u < nitems; u += gridDim.x) {
        DqItem it;
        if (!dq_item(p, u, ngath, it)) continue;
        if (!(ok = mbar_wait(&bar.q_full[0], qn & 1, abort, p.status, site0 + 2))) break;
        ++qn;
        // The previous item's dQ must have been read out before this one accumulates.
        if (!(ok = mbar_wait(&bar.acc_empty, (an & 1) ^ 1, abort, p.status, site0 + 3))) break;
        ++an;
        tc_fence_after();
        for (int m2 = 0; m2 <= it.nc && ok; ++m2) {
          const uint32_t sm = kvc + m2, sp = kvc + m2 - 1;
          const int st = sm % C::ST;
          if (m2 < it.nc) {
            if (!(ok = mbar_wait(&bar.k_full[st], (sm / C::ST) & 1, abort, p.status, site0 + 5))) break;
            if (!(ok = mbar_wait(&bar.v_full[st], (sm / C::ST) & 1, abort, p.status, site0 + 6))) break;
            tc_fence_after();
          }
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            const uint32_t tS = tmem + 128 * x, tP = tmem + 128 * x + 64;
            if (m2 > 0) {
              // dQ += dS_x(m-1) K_x(m-1), once group x wrote dS back.
              if (!(ok = mbar_wait(&bar.ds_full[x], sc[x] & 1, abort, p.status, site0 + 4))) break;
              ++sc[x];
              tc_fence_after();
              const uint32_t kt = base + C::K_OFF + (sp % C::ST) * T::TILE;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                umma_ts(tQ, tS + kk * 8, bwd_mn_desc<D>(kt, 4 * x + kk), idQ,
                        (m2 == 1 && x == 0 && kk == 0) ? 0u : 1u);
              if (x == 1) umma_commit(&bar.k_empty[sp % C::ST]);
            }
            if (m2 < it.nc) {
              const uint32_t kt = base + C::K_OFF + st * T::TILE + x * 8192;
              const uint32_t vt = base + C::V_OFF + st * T::TILE + x * 8192;
#pragma unroll
              for (int ks = 0; ks < D / 16; ++ks)
                umma_ss(tS, bwd_kmajor_desc<D>(qt, ks), bwd_kmajor_desc<D>(kt, ks), idS, ks > 0 ? 1u : 0u);
#pragma unroll
              for (int ks = 0; ks < D / 16; ++ks)
                umma_ss(tP, bwd_kmajor_desc<D>(dot, ks), bwd_kmajor_desc<D>(vt, ks), idS, ks > 0 ? 1u : 0u);
              umma_commit(&bar.s_full[x]);
              if (x == 1) umma_commit(&bar.v_empty[st]);
            }
          }
        }
        if (!ok) break;
        umma_commit(&bar.acc_full);
        umma_commit(&bar.q_empty[0]);
        kvc += it.nc;
      }
      umma_commit(&bar.mma_done);
      const unsigned long long t0 = global_timer_ns();
      while (!mbar_try_wait(&bar.mma_done, 0) && global_timer_ns() - t0 < wait_limit_ns(p.status)) {}
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ row gather
    const int gt = tid - 64;
    uint32_t qn = 0;
    bool ok = true;
    // The next item's rows are decoded after the current item's copies have landed and
    // been handed on (their arrive is what the MMA issuer waits for), while the gather
    // waits for the buffer to come free again.
    auto next_item = [&](int u, DqItem &it) -> int {
      for (; u < nitems; u += gridDim.x)
        if (dq_item(p, u, ngath, it)) return u;
      return nitems;
    };
    DqItem it;
    GatherRows gr;
    RowSrc *tab = reinterpret_cast<RowSrc *>(sbase + C::TAB_OFF);
    int u = next_item(blockIdx.x, it);
    if (u < nitems) decode_rows(p, it.t, it.b, it.hk, gt, tab, gr);
    while (ok && u < nitems) {
      ok = mbar_wait(&bar.q_empty[0], (qn & 1) ^ 1, abort, p.status, site0 + 7);
      if (!(ok = __all_sync(FULL, ok))) break;
      ++qn;
      issue_rows<D>(p, gr, tab, base + C::Q_OFF, base + C::DO_OFF, stats, gt);
      land_tile(&bar.q_full[0]);
      u = next_item(u + gridDim.x, it);
      if (u < nitems) decode_rows(p, it.t, it.b, it.hk, gt, tab, gr, true);
    }
    cp_async_wait_all();
  } else {
    // ------------------------------------------------------------ dS and dQ out
    // Two warp groups share the rows: group grp (warps 4-7 or 8-11) takes the columns
    // [64 grp, 64 grp + 64) of S and dP and half of dQ's columns, so that two warps per
    // sub-partition hide each other's TMEM and exponential latencies.
    const int r = (tid - 128) & 127;               // row == TMEM lane
    const int grp = (warp - 4) >> 2;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tS = tmem + lane_off + 128 * grp, tP = tS + 64, tQ = tmem + lane_off + 256;
    const float sl2 = p.scale_log2;
    uint32_t sc = 0, an = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < nitems; u += gridDim.x) {
      DqItem it;
      if (!dq_item(p, u, ngath, it)) continue;
      const bool live = r < it.t.rows;
      int h = 0, i = 0, slot = 0;
      if (live) tile_row(p, it.t, it.hk, r, h, i, slot);
      // The row's statistics (rows past the tile's end: p = 0).
      float lse2 = INFINITY, Dr = 0.f;
      if (live) {
        const float2 st2 = p.rowstat[((int64_t)it.b * p.hq + h) * p.N + i];
        lse2 = st2.x;
        Dr = st2.y;
      }
      for (int m2 = 0; m2 < it.nc; ++m2, ++sc) {
        ok = mbar_wait(&bar.s_full[grp], sc & 1, abort, p.status, site0 + 8);
        if (!(ok = __all_sync(FULL, ok))) break;
        tc_fence_after();
        const int key0 = it.key0 + m2 * kTileKeys + 64 * grp;
        {
          uint32_t sv[64], pv[64];
          tmem_ld64(tS, sv);
          tmem_ld64(tP, pv);
          tmem_wait_ld();
          uint32_t ds[32];
#pragma unroll
          for (int e = 0; e < 64; e += 2) {
            float d2[2];
#pragma unroll
            for (int f = 0; f < 2; ++f) {
              const int key = key0 + e + f;
              float pr = ex2_approx(fmaf(__uint_as_float(sv[e + f]), sl2, -lse2));
              if (it.causal && key > i) pr = 0.f;
              d2[f] = pr * (__uint_as_float(pv[e + f]) - Dr);
            }
            ds[e / 2] = pack_bf16x2(d2[0], d2[1]);
          }
          tmem_st32(tS, ds);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar.ds_full[grp]);
      }
      if (!ok) break;
      ok = mbar_wait(&bar.acc_full, an & 1, abort, p.status, site0 + 9);
      if (!(ok = __all_sync(FULL, ok))) break;
      ++an;
      tc_fence_after();
      float *dst = p.dqp + ((((int64_t)it.b * p.hq + h) * p.N + i) * p.topk + slot) * D;
      // The fp32 partials go out through a per-warp staging buffer (32 rows x 16 columns,
      // 16-byte chunks XOR-swizzled by row pair): lane r writes its row's 64 bytes, then
      // each store instruction writes eight whole 64-byte row segments (coalesced).
      unsigned char *stg = sbase + C::STG_OFF + (warp - 4) * 2048;
      float *rdst[4];
      bool rlive[4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int src = jj * 8 + (lane >> 2);
        rdst[jj] = reinterpret_cast<float *>(__shfl_sync(FULL, reinterpret_cast<uintptr_t>(dst), src));
        rlive[jj] = __shfl_sync(FULL, live ? 1 : 0, src) != 0;
      }
#pragma unroll
      for (int c0 = grp * (D / 2); c0 < (grp + 1) * (D / 2); c0 += 16) {
        uint32_t o[16];
        tmem_ld16(tQ + c0, o);
        tmem_wait_ld();
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4)
          *reinterpret_cast<uint4 *>(stg + lane * 64 + ((v4 ^ ((lane >> 1) & 3)) << 4)) =
              make_uint4(o[4 * v4], o[4 * v4 + 1], o[4 * v4 + 2], o[4 * v4 + 3]);
        __syncwarp();
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int row = jj * 8 + (lane >> 2), ch = lane & 3;
          if (rlive[jj]) {
            const uint4 q = *reinterpret_cast<const uint4 *>(stg + row * 64 + ((ch ^ ((row >> 1) & 3)) << 4));
            *reinterpret_cast<uint4 *>(rdst[jj] + c0 + ch * 4) = q;
          }
        }
        __syncwarp();
      }
      tc_fence_before();
      mbar_arrive(&bar.acc_empty);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ dK / dV

template <int D>
struct DkvCfg {
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = BwdTile<D>::TILE;
  static constexpr int Q_OFF = 2 * BwdTile<D>::TILE;                  // 2 stages of Q
  static constexpr int DO_OFF = Q_OFF + 2 * BwdTile<D>::TILE;         // 2 stages of dO
  static constexpr int ST_OFF = DO_OFF + 2 * BwdTile<D>::TILE;        // 2 x float2 [128]
  static constexpr int TAB_OFF = ST_OFF + 2 * 128 * 8;                 // RowSrc [128]
  static constexpr int BAR_OFF = TAB_OFF + 128 * 16;
  static constexpr int SMEM = BAR_OFF + 1024 + 1024;
};

// The query tiles of a key-tile unit, in the order every role walks them: the 128-entry
// tiles of the block's list in each query chunk, then, for every q-head of the group,
// the 128-row tiles of the block's own rows from the key tile on (the first one, on the
// diagonal, is causal).
struct DkvWalk {
  int b, hk, j, kt0;    // unit: key tile [kt0, kt0 + 128) of block j
  int blk_end;          // min((j + 1) block, N)
  int ch, e, e_end;     // list phase
  int g, r0;            // own phase
  int phase;            // 0 lists, 1 own rows, 2 done
};

// Unit u of CTA blockIdx.x (u = blockIdx.x + k gridDim.x) -> the k-th unit of the CTA
// in cost order.  Units are ranked with the block index slowest (early blocks are past
// blocks of the most rows, so their lists are the longest: roughly longest first), and
// CTA x takes rank x of even stripes of gridDim.x ranks and rank gridDim.x - 1 - x of odd
// ones (a snake), so that every CTA gets a similar mix of long and short walks.
// Returns false when the rank is past the last unit.
__device__ __forceinline__ bool dkv_walk_begin(const BwdParams &p, int u, DkvWalk &w) {
  const int tpb = p.block / kTileKeys;
  const int nunits = p.batch * p.hkv * p.nblk * tpb;
  const int stripe = u / (int)gridDim.x, pos = u - stripe * (int)gridDim.x;
  const int rank = stripe * (int)gridDim.x + ((stripe & 1) ? (int)gridDim.x - 1 - pos : pos);
  if (rank >= nunits) return false;
  const int t = rank % tpb;
  int rest = rank / tpb;
  w.hk = rest % p.hkv;
  rest /= p.hkv;
  w.b = rest % p.batch;
  w.j = rest / p.batch;
  w.kt0 = w.j * p.block + t * kTileKeys;
  w.blk_end = min((w.j + 1) * p.block, p.N);
  w.ch = 0;
  w.e = w.e_end = 0;
  w.g = 0;
  w.r0 = w.kt0;
  w.phase = (p.npast > 0) ? 0 : 1;
  if (w.phase == 0) {
    const int L = (w.b * p.hkv + w.hk) * p.nblk + w.j;
    w.e = __ldg(p.listoff + L);
    w.e_end = __ldg(p.listoff + L + 1);
  }
  return w.kt0 < p.N;
}

// The next query tile (returns false when the walk is over).
__device__ __forceinline__ bool dkv_walk_next(const BwdParams &p, DkvWalk &w, BwdRows &t,
                                              int &diag) {
  while (w.phase == 0) {
    if (w.e < w.e_end) {
      t.gathered = 1;
      t.ent0 = w.e;
      t.rows = min(128, w.e_end - w.e);
      t.b = w.b;
      t.h = 0;
      t.row0 = 0;
      diag = 0;
      w.e += 128;
      return true;
    }
    if (++w.ch >= p.nchunks) {
      w.phase = 1;
      break;
    }
    const int L = ((w.ch * p.batch + w.b) * p.hkv + w.hk) * p.nblk + w.j;
    w.e = __ldg(p.listoff + L);
    w.e_end = __ldg(p.listoff + L + 1);
  }
  if (w.phase == 1) {
    if (w.r0 >= w.blk_end) {
      w.r0 = w.kt0;
      if (++w.g >= p.G) {
        w.phase = 2;
        return false;
      }
    }
    t.gathered = 0;
    t.ent0 = 0;
    t.b = w.b;
    t.h = w.hk * p.G + w.g;
    t.row0 = w.r0;
    t.rows = min(128, w.blk_end - w.r0);
    diag = (w.r0 == w.kt0);
    w.r0 += 128;
    return true;
  }
  return false;
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                const BwdParams p) {
  using C = DkvCfg<D>;
  using T = BwdTile<D>;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char *sbase = smem_raw + (base - raw);
  BwdBars &bar = *reinterpret_cast<BwdBars *>(sbase + C::BAR_OFF);
  float2 *stats_all = reinterpret_cast<float2 *>(sbase + C::ST_OFF);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int site0 = (9 * 16 + (D == 64 ? 0 : 2)) * 256;
  constexpr uint32_t FULL = 0xffffffffu;
  // Loop bound over whole stripes of gridDim.x units (the snake order of dkv_walk_begin
  // maps the last, partial stripe onto ranks in reverse; ranks past the last unit skip).
  const int nunits0 = p.batch * p.hkv * p.nblk * (p.block / kTileKeys);
  const int nunits = (nunits0 + (int)gridDim.x - 1) / (int)gridDim.x * (int)gridDim.x;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.q_full[s], 64);
      mbar_init(&bar.q_empty[s], 1);
    }
    mbar_init(&bar.k_full[0], 1);
    mbar_init(&bar.k_empty[0], 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bar.s_full[x], 1);
      mbar_init(&bar.ds_full[x], 128);
    }
    mbar_init(&bar.acc_full, 1);
    mbar_init(&bar.acc_empty, 256);
    mbar_init(&bar.mma_done, 1);
    bar.abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(&bar.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;
  volatile int *abort = &bar.abort;
  // TMEM: S^T [0, 128), dP^T [128, 256), dK [256, 256 + D), dV [256 + D, 256 + 2 D).

  if (warp == 0) {
    // ------------------------------------------------------------ K / V tiles
    if (lane == 0) {
      uint32_t kn = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
        DkvWalk w;
        if (!dkv_walk_begin(p, u, w)) continue;
        if (!(ok = mbar_wait(&bar.k_empty[0], (kn & 1) ^ 1, abort, p.status, site0 + 1))) break;
        ++kn;
        mbar_arrive_expect_tx(&bar.k_full[0], 2 * T::BYTES);
        unsigned char *kd = sbase + C::K_OFF, *vd = sbase + C::V_OFF;
        tma_load_4d(kd, &tmK, &bar.k_full[0], 0, w.kt0, w.hk, w.b);
        tma_load_4d(vd, &tmV, &bar.k_full[0], 0, w.kt0, w.hk, w.b);
        if (D == 128) {
          tma_load_4d(kd + T::R0, &tmK, &bar.k_full[0], 64, w.kt0, w.hk, w.b);
          tma_load_4d(vd + T::R0, &tmV, &bar.k_full[0], 64, w.kt0, w.hk, w.b);
        }
      }
      if (*abort && kn > 0) {
        const unsigned long long t0 = global_timer_ns();
        while (!mbar_try_wait(&bar.k_full[0], (kn - 1) & 1) && global_timer_ns() - t0 < wait_limit_ns(p.status)) {}
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // Each 128-row query tile is taken as two 64-row halves x, one per elementwise
      // warp group, each with its own TMEM buffer: S^T_x at 128 x, dP^T_x at 128 x + 64;
      // dK at 256, dV at 256 + D.  While one group works on its half, the tensor core
      // computes the other's products.
      constexpr uint32_t idS = idesc_bf16(128, 64, 0, 0);
      constexpr uint32_t idG = idesc_bf16(128, D, 0, 1);
      const uint32_t tK = tmem + 256, tV = tmem + 256 + D;
      const uint32_t kt = base + C::K_OFF, vt = base + C::V_OFF;
      uint32_t kn = 0, qn = 0, an = 0;
      uint32_t sc[2] = {0u, 0u};
      bool ok = true;
      for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
        DkvWalk w;
        if (!dkv_walk_begin(p, u, w)) continue;
        if (!(ok = mbar_wait(&bar.k_full[0], kn & 1, abort, p.status, site0 + 2))) break;
        ++kn;
        if (!(ok = mbar_wait(&bar.acc_empty, (an & 1) ^ 1, abort, p.status, site0 + 3))) break;
        ++an;
        tc_fence_after();
        BwdRows t;
        int diag;
        bool more = dkv_walk_next(p, w, t, diag);
        int n = 0;
        uint32_t prev_stage = 0;
        while (ok) {
          const uint32_t st = qn % 2;
          if (more) {
            if (!(ok = mbar_wait(&bar.q_full[st], (qn / 2) & 1, abort, p.status, site0 + 4))) break;
            tc_fence_after();
          }
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            const uint32_t tS = tmem + 128 * x, tP = tmem + 128 * x + 64;
            if (n > 0) {
              // dV += P^T_x dO_x and dK += dS^T_x Q_x of the previous query tile.
              if (!(ok = mbar_wait(&bar.ds_full[x], sc[x] & 1, abort, p.status, site0 + 5))) break;
              ++sc[x];
              tc_fence_after();
              const uint32_t qp = base + C::Q_OFF + prev_stage * T::TILE;
              const uint32_t dp = base + C::DO_OFF + prev_stage * T::TILE;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint32_t acc = (n == 1 && x == 0 && kk == 0) ? 0u : 1u;
                umma_ts(tV, tS + kk * 8, bwd_mn_desc<D>(dp, 4 * x + kk), idG, acc);
                umma_ts(tK, tP + kk * 8, bwd_mn_desc<D>(qp, 4 * x + kk), idG, acc);
              }
              if (x == 1) umma_commit(&bar.q_empty[prev_stage]);
            }
            if (more) {
              const uint32_t qt = base + C::Q_OFF + st * T::TILE + x * 8192;
              const uint32_t dot = base + C::DO_OFF + st * T::TILE + x * 8192;
#pragma unroll
              for (int ks = 0; ks < D / 16; ++ks)
                umma_ss(tS, bwd_kmajor_desc<D>(kt, ks), bwd_kmajor_desc<D>(qt, ks), idS, ks > 0 ? 1u : 0u);
#pragma unroll
              for (int ks = 0; ks < D / 16; ++ks)
                umma_ss(tP, bwd_kmajor_desc<D>(vt, ks), bwd_kmajor_desc<D>(dot, ks), idS, ks > 0 ? 1u : 0u);
              umma_commit(&bar.s_full[x]);
            }
          }
          if (!ok || !more) break;
          prev_stage = st;
          ++qn;
          ++n;
          more = dkv_walk_next(p, w, t, diag);
        }
        if (!ok) break;
        umma_commit(&bar.acc_full);
        umma_commit(&bar.k_empty[0]);
      }
      umma_commit(&bar.mma_done);
      const unsigned long long t0 = global_timer_ns();
      while (!mbar_try_wait(&bar.mma_done, 0) && global_timer_ns() - t0 < wait_limit_ns(p.status)) {}
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ query-side gather
    const int gt = tid - 64;
    uint32_t qn = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
      DkvWalk w;
      if (!dkv_walk_begin(p, u, w)) continue;
      BwdRows t;
      int diag;
      GatherRows gr;
      RowSrc *tab = reinterpret_cast<RowSrc *>(sbase + C::TAB_OFF);
      // The next tile's rows are decoded after the current tile's copies have landed and
      // been handed on, while the gather waits for the next stage to come free.
      bool have = dkv_walk_next(p, w, t, diag);
      if (have) decode_rows(p, t, w.b, w.hk, gt, tab, gr);
      while (ok && have) {
        const uint32_t st = qn % 2;
        ok = mbar_wait(&bar.q_empty[st], ((qn / 2) & 1) ^ 1, abort, p.status, site0 + 6);
        if (!(ok = __all_sync(FULL, ok))) break;
        ++qn;
        issue_rows<D>(p, gr, tab, base + C::Q_OFF + st * T::TILE, base + C::DO_OFF + st * T::TILE,
                      stats_all + st * 128, gt);
        land_tile(&bar.q_full[st]);
        have = dkv_walk_next(p, w, t, diag);
        if (have) decode_rows(p, t, w.b, w.hk, gt, tab, gr);
      }
    }
    cp_async_wait_all();
  } else {
    // ------------------------------------------------------------ P^T, dS^T; dK, dV out
    // Two warp groups share the keys: group grp takes the query columns
    // [64 grp, 64 grp + 64) of S^T and dP^T and half of dK's and dV's columns.
    const int r = (tid - 128) & 127;               // key within the tile == TMEM lane
    const int grp = (warp - 4) >> 2;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tS = tmem + lane_off + 128 * grp, tP = tS + 64;
    const uint32_t tK = tmem + lane_off + 256, tV = tmem + lane_off + 256 + D;
    const float sl2 = p.scale_log2;
    uint32_t sc = 0, an = 0, qn = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
      DkvWalk w;
      if (!dkv_walk_begin(p, u, w)) continue;
      const int key = w.kt0 + r;
      BwdRows t;
      int diag;
      while (ok && dkv_walk_next(p, w, t, diag)) {
        // The tile's row statistics were written by the gather warps before they arrived
        // on the stage's q_full barrier (whose phase cannot move on before this tile's
        // products are done, which needs this warp group's P and dS).
        const uint32_t st = qn % 2;
        ok = mbar_wait(&bar.q_full[st], (qn / 2) & 1, abort, p.status, site0 + 9);
        if (!(ok = __all_sync(FULL, ok))) break;
        const float2 *stats = stats_all + st * 128;
        ++qn;
        ok = mbar_wait(&bar.s_full[grp], sc & 1, abort, p.status, site0 + 7);
        if (!(ok = __all_sync(FULL, ok))) break;
        ++sc;
        tc_fence_after();
        {
          const int half = grp;
          uint32_t sv[64], pv[64];
          tmem_ld64(tS, sv);
          tmem_ld64(tP, pv);
          tmem_wait_ld();
          uint32_t pp[32], dd[32];
#pragma unroll
          for (int e = 0; e < 64; e += 2) {
            float pr[2], d2[2];
#pragma unroll
            for (int f = 0; f < 2; ++f) {
              const int col = half * 64 + e + f;          // query row of the tile
              const float2 st2 = stats[col];
              pr[f] = ex2_approx(fmaf(__uint_as_float(sv[e + f]), sl2, -st2.x));
              if (diag && key > t.row0 + col) pr[f] = 0.f;
              d2[f] = pr[f] * (__uint_as_float(pv[e + f]) - st2.y);
            }
            pp[e / 2] = pack_bf16x2(pr[0], pr[1]);
            dd[e / 2] = pack_bf16x2(d2[0], d2[1]);
          }
          tmem_st32(tS, pp);
          tmem_st32(tP, dd);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar.ds_full[grp]);
      }
      if (!ok) break;
      ok = mbar_wait(&bar.acc_full, an & 1, abort, p.status, site0 + 8);
      if (!(ok = __all_sync(FULL, ok))) break;
      ++an;
      tc_fence_after();
      const bool live = key < p.N;
      uint16_t *dkr = p.dk + w.b * p.dk_sb + (int64_t)w.hk * p.dk_sh + (int64_t)key * p.dk_sn;
      uint16_t *dvr = p.dv + w.b * p.dv_sb + (int64_t)w.hk * p.dv_sh + (int64_t)key * p.dv_sn;
      const float sc_k = p.scale;
#pragma unroll
      for (int c0 = grp * (D / 2); c0 < (grp + 1) * (D / 2); c0 += 32) {
        uint32_t a[32], bv[32];
        tmem_ld32(tK + c0, a);
        tmem_ld32(tV + c0, bv);
        tmem_wait_ld();
        if (live) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 x, y;
            x.x = pack_bf16x2(__uint_as_float(a[e]) * sc_k, __uint_as_float(a[e + 1]) * sc_k);
            x.y = pack_bf16x2(__uint_as_float(a[e + 2]) * sc_k, __uint_as_float(a[e + 3]) * sc_k);
            x.z = pack_bf16x2(__uint_as_float(a[e + 4]) * sc_k, __uint_as_float(a[e + 5]) * sc_k);
            x.w = pack_bf16x2(__uint_as_float(a[e + 6]) * sc_k, __uint_as_float(a[e + 7]) * sc_k);
            y.x = pack_bf16x2(__uint_as_float(bv[e]), __uint_as_float(bv[e + 1]));
            y.y = pack_bf16x2(__uint_as_float(bv[e + 2]), __uint_as_float(bv[e + 3]));
            y.z = pack_bf16x2(__uint_as_float(bv[e + 4]), __uint_as_float(bv[e + 5]));
            y.w = pack_bf16x2(__uint_as_float(bv[e + 6]), __uint_as_float(bv[e + 7]));
            *reinterpret_cast<uint4 *>(dkr + c0 + e) = x;
            *reinterpret_cast<uint4 *>(dvr + c0 + e) = y;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bar.acc_empty);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ dQ merge

// dq_i = scale * (the row's own-block slot + its valid past slots): D / 8 lanes per row
// with 16-byte stores; the partial slots are fp32.
template <int D>
__global__ void __launch_bounds__(256) bwd_dq_merge_kernel(const BwdParams p) {
  constexpr int LPR = D / 8, RPW = 32 / LPR;
  const int lane = threadIdx.x & 31, sub = lane / LPR, v = lane % LPR;
  const int gw = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int nw = (int)((gridDim.x * blockDim.x) >> 5);
  const long long total = (long long)p.batch * p.hq * p.N;
  for (long long row = (long long)gw * RPW + sub; row < total; row += (long long)nw * RPW) {
    const long long bh = row / p.N;
    const int i = (int)(row - bh * p.N);
    const int b = (int)(bh / p.hq), h = (int)(bh % p.hq);
    const int c = i / p.block;
    const int np = min(c, p.npast);             // the row's past slots are the first np
    const float *src = p.dqp + row * p.topk * D + v * 8;
    float acc[8];
    {
      const float4 a = *reinterpret_cast<const float4 *>(src + (int64_t)p.npast * D);
      const float4 bq = *reinterpret_cast<const float4 *>(src + (int64_t)p.npast * D + 4);
      acc[0] = a.x; acc[1] = a.y; acc[2] = a.z; acc[3] = a.w;
      acc[4] = bq.x; acc[5] = bq.y; acc[6] = bq.z; acc[7] = bq.w;
    }
    for (int s = 0; s < np; ++s) {
      const float4 a = *reinterpret_cast<const float4 *>(src + (int64_t)s * D);
      const float4 bq = *reinterpret_cast<const float4 *>(src + (int64_t)s * D + 4);
      acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
      acc[4] += bq.x; acc[5] += bq.y; acc[6] += bq.z; acc[7] += bq.w;
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0] * p.scale, acc[1] * p.scale);
    o.y = pack_bf16x2(acc[2] * p.scale, acc[3] * p.scale);
    o.z = pack_bf16x2(acc[4] * p.scale, acc[5] * p.scale);
    o.w = pack_bf16x2(acc[6] * p.scale, acc[7] * p.scale);
    *reinterpret_cast<uint4 *>(p.dq + b * p.dq_sb + (int64_t)h * p.dq_sh + (int64_t)i * p.dq_sn + v * 8) = o;
  }
}

// ------------------------------------------------------------------ launch

template <int D>
static cudaError_t launch_bwd_d(const CUtensorMap *maps, const BwdParams &p, int nsm, cudaStream_t st) {
  const long long rows = (long long)p.batch * p.hq * p.N;
  const int rpw = 32 / (D / 8);
  long long blocks = (rows / rpw + 8) / 8;
  if (blocks > (long long)nsm * 16) blocks = (long long)nsm * 16;
  if (blocks < 1) blocks = 1;
  bwd_prep_kernel<D><<<(unsigned)blocks, 256, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  e = cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, DqCfg<D>::SMEM);
  if (e != cudaSuccess) return e;
  bwd_dq_kernel<D><<<nsm, kBwdThreads, DqCfg<D>::SMEM, st>>>(maps[0], maps[1], p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  e = cudaFuncSetAttribute(bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, DkvCfg<D>::SMEM);
  if (e != cudaSuccess) return e;
  const long long nunits = (long long)p.batch * p.hkv * p.nblk * (p.block / kTileKeys);
  const int grid = (int)(nunits < nsm ? nunits : nsm);
  bwd_dkdv_kernel<D><<<grid, kBwdThreads, DkvCfg<D>::SMEM, st>>>(maps[0], maps[1], p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  bwd_dq_merge_kernel<D><<<(unsigned)blocks, 256, 0, st>>>(p);
  return cudaGetLastError();
}

// maps: K and V (64-column boxes of 128 rows, 128-byte swizzle).
cudaError_t launch_bwd(const CUtensorMap *maps, const BwdParams &p, int nsm, cudaStream_t st) {
  switch (p.d) {
    case 64: return launch_bwd_d<64>(maps, p, nsm, st);
    case 128: return launch_bwd_d<128>(maps, p, nsm, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace moba
