// attn.cu -- block-sparse / sliding-window attention forward on sm_100a tensor cores.
//
// [MoBA] = "MoBA: 어텐션에 전문가 혼합을 적용해 긴 문맥을 효율적으로 처리하는 블록 어텐션
//          (feat. MoonshotAI)", PyTorch KR forum summary of the MoBA paper.
// [SWA]  = "SWA + MoE: 어텐션과 희소 전문가", Bit-Axon architecture page.
//
// One persistent kernel, two tile kinds:
//   kQueryMajor  128 contiguous query rows of one (batch, q-head).  MoBA: the causal own
//                block (§"MoBA의 구현": current block with causal=True), the window
//                tail into earlier unselected blocks, and the merge of the past-block
//                partials by log-sum-exp (step 5).  SWA: the causal band of [SWA]
//                §"슬라이딩 윈도우 마스크".
//   kGathered    up to 128 (row, q-head) pairs of one block-major list against the
//                whole past block they picked (steps 3-4, causal=False); writes a
//                normalised partial output and its log-sum-exp per (row, slot).
//
// Per CTA (512 threads, one CTA per SM, 512 TMEM columns):
//   warp 0       TMA producers: lane 0 the query tile (query-major) and K chunks of 128
//                keys, lane 1 the V chunks (separate K and V rings)
//   warp 1       tcgen05 MMA issuer (one thread) and TMEM owner
//   warps 2-3    query-row gather with cp.async (gathered tiles)
//   warps 4-11   softmax, two warpgroups: thread r of group h owns row r (TMEM lane r)
//                and keys [64 h, 64 h + 64) of each chunk; the two halves of a row
//                exchange their maxima through shared memory; S -> P in place; O is
//                rescaled only when the running maximum grows by more than 2^8
//   warps 12-15  epilogue: normalises O and stores it (a partial or the output),
//                then frees the O buffer
// TMEM: S/P double buffer at columns [0,128) and [128,256); O double buffer at
// [256,384) and [384,512), so a tile's epilogue overlaps the next tile's MMAs.
// S = Q K^T is an SS MMA; P (bf16) overwrites its own S columns and is the A operand
// (from TMEM) of O += P V.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "params.h"

namespace moba {

constexpr int kAttnThreads = 512;
constexpr int kRescaleThreshold = 8;  // log2 units
// Of every 16 probabilities, this many take the FMA-pipe 2^x (exp2_fma) instead of
// the MUFU unit, whose 16 results per clock and SM bound the softmax otherwise.
#ifndef MOBA_EXP_EMU_PER16
#define MOBA_EXP_EMU_PER16 0
#endif
constexpr int kExpEmuPer16 = MOBA_EXP_EMU_PER16;
// Registers per thread after the re-split: producer/MMA/gather, softmax, epilogue.
constexpr int kRegsWG0 = 64, kRegsSoftmax = 160, kRegsEpilogue = 128;
constexpr int kRegSplitTotal = 128 * (kRegsWG0 + 2 * kRegsSoftmax + kRegsEpilogue);
static_assert(kRegSplitTotal <= 65536, "register split exceeds the register file");
static_assert(kRegsEpilogue * kAttnThreads == 65536, "the epilogue keeps the launch budget");

template <int D>
struct AttnCfg {
  static constexpr int ST = (D == 128) ? 2 : 3;            // K/V pipeline stages
  static constexpr int R0 = 128 * 128;                     // bytes of the 64-column region
  static constexpr int R1 = (D == 128) ? 128 * 128 : (D == 80 ? 128 * 32 : 0);
  static constexpr int TILE = R0 + ((R1 + 1023) / 1024) * 1024;  // one 128 x D operand tile
  static constexpr int Q_OFF = 0;                          // 2 query buffers
  static constexpr int K_OFF = 2 * TILE;                   // ST key stages
  static constexpr int V_OFF = K_OFF + ST * TILE;          // ST value stages
  static constexpr int BAR_OFF = V_OFF + ST * TILE;
  static constexpr int SMEM = BAR_OFF + 8192 + 1024;       // + barriers/stats + alignment slack
  static constexpr uint32_t BYTES = 128u * D * 2u;         // bytes one full tile load moves
};

struct Bars {
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[3], v_full[3], k_empty[3], v_empty[3];
  uint64_t s_full[2];
  uint64_t p_full, o_done[2], mma_done;
  uint64_t o_full[2], o_free[2], stat_full[2];
  uint32_t tmem_base;
  int abort;
  float2 stat[2][2][128];  // per O buffer, key half and row: running max (log2), row sum
  float xmax[2][2][128];   // per S buffer, key half and row: the half-row maximum
};

// What one tile covers.  All roles derive it independently from the tile index.
struct TileInfo {
  int b, h, hk;
  int i0;          // query-major: first row
  int rows;        // valid rows
  int nc;          // key chunks
  int key0;        // query-major MoBA: first key of the tail (window) range
  int ntail;       // query-major MoBA: chunks before the own block
  int cB;          // query-major MoBA: first key of the own block
  // gathered
  int list;        // list id
  int ent0;        // first entry of this tile in the entry array
  int j;           // past block
};

__device__ __forceinline__ void query_major_tile(const AttnParams &p, int t, TileInfo &ti) {
  const int HB = p.hq * p.batch;
  const int nq = (p.row_end - p.row_begin + kTileRows - 1) / kTileRows;
  const int qt = nq - 1 - t / HB;  // later (heavier) tiles first
  const int hb = t % HB;
  ti.h = hb % p.hq;
  ti.b = hb / p.hq;
  ti.hk = ti.h / p.G;
  ti.i0 = p.row_begin + qt * kTileRows;
  ti.rows = min(kTileRows, p.row_end - ti.i0);
  const int ilast = ti.i0 + ti.rows - 1;
  if (p.is_moba) {
    ti.cB = (ti.i0 / p.block) * p.block;
    int tl = ti.cB;
    if (p.window > 0) {
      const int lo = max(0, ti.i0 - p.window + 1);
      tl = min(ti.cB, (lo / kTileKeys) * kTileKeys);
    }
    ti.key0 = tl;
    ti.ntail = (ti.cB - tl) / kTileKeys;
    ti.nc = ti.ntail + (ti.i0 - ti.cB) / kTileKeys + 1;
  } else {
    const int lo = max(0, ti.i0 - p.window + 1);
    ti.key0 = (lo / kTileKeys) * kTileKeys;
    ti.ntail = 0;
    ti.cB = 0;
    ti.nc = (ilast - ti.key0) / kTileKeys + 1;
  }
}

__device__ __forceinline__ void gathered_tile(const AttnParams &p, int4 rec, TileInfo &ti) {
  const int L = rec.x;
  ti.list = L;
  ti.ent0 = rec.y;
  ti.rows = rec.z;
  ti.j = L % p.nblk;
  ti.hk = (L / p.nblk) % p.hkv;
  ti.b = (L / (p.nblk * p.hkv)) % p.batch;
  ti.h = -1;
  ti.i0 = 0;
  ti.nc = p.block / kTileKeys;
}

// Walks this CTA's tiles t = t_begin + blockIdx.x, t += gridDim.x.  Gathered tiles
// come from the tile table; the next record is loaded one tile ahead.
template <int MODE>
struct TileIter {
  int t, t_end;
  int4 nxt;
  __device__ __forceinline__ TileIter(const AttnParams &p, int t_begin, int t_end_) {
    t = t_begin + (int)blockIdx.x;
    t_end = t_end_;
    if (MODE == kGathered && t < t_end) nxt = __ldg(p.tiles + t);
  }
  __device__ __forceinline__ bool valid() const { return t < t_end; }
  __device__ __forceinline__ void get(const AttnParams &p, TileInfo &ti) {
    if (MODE == kGathered) {
      const int4 cur = nxt;
      if (t + (int)gridDim.x < t_end) nxt = __ldg(p.tiles + t + gridDim.x);
      gathered_tile(p, cur, ti);
    } else {
      query_major_tile(p, t, ti);
    }
  }
  __device__ __forceinline__ void next() { t += gridDim.x; }
};

// Key of chunk m of a tile.
template <int MODE>
__device__ __forceinline__ int chunk_key(const AttnParams &p, const TileInfo &ti, int m) {
  if (MODE == kGathered) return ti.j * p.block + m * kTileKeys;
  return ti.key0 + m * kTileKeys;
}

// Operand descriptors.  Region 0 holds columns [0, 64) of a 128-row tile (128-byte
// rows, 128-byte swizzle); region 1 holds columns [64, 128) the same way (D = 128) or
// columns [64, 80) with 32-byte rows and 32-byte swizzle (D = 80).
template <int D>
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile, int ks) {
  if (ks < 4) return smem_desc(tile + ks * 32, 16, 1024, kSwizzle128);
  if (D == 128) return smem_desc(tile + AttnCfg<D>::R0 + (ks - 4) * 32, 16, 1024, kSwizzle128);
  return smem_desc(tile + AttnCfg<D>::R0, 16, 256, kSwizzle32);
}

// V as the MN-major B operand of O += P V, keys [16 kk, 16 kk + 16).  rg = 0: the 64
// columns of region 0 (128-byte swizzle; 8-key groups 1024 bytes apart).  rg = 1: the
// 16 columns of the D = 80 tail region (32-byte swizzle, groups 256 bytes apart).
// rg = 2 (D = 128): all 128 columns in one operand, the second 64-column atom a
// leading-byte-offset of one region away.
template <int D>
__device__ __forceinline__ uint64_t v_desc(uint32_t tile, int kk, int rg) {
  if (rg == 0) return smem_desc(tile + kk * 2048, 16, 1024, kSwizzle128);
  if (rg == 2) return smem_desc(tile + kk * 2048, AttnCfg<D>::R0, 1024, kSwizzle128);
  return smem_desc(tile + AttnCfg<D>::R0 + kk * 512, 16, 256, kSwizzle32);
}

template <int D, int MODE>
__global__ void __launch_bounds__(kAttnThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQ1,
                const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmK1,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmV1,
                const AttnParams p) {
  using C = AttnCfg<D>;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char *sbase = smem_raw + (base - raw);
  Bars &bar = *reinterpret_cast<Bars *>(sbase + C::BAR_OFF);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int site0 = (MODE * 16 + (D == 64 ? 0 : (D == 80 ? 1 : 2))) * 256;
  constexpr uint32_t FULL = 0xffffffffu;

  // Tile range.
  int t_begin = 0, t_end = p.ntiles;
  if (MODE == kGathered) {
    t_begin = __ldg(p.tileoff + p.chunk * p.lists_per_chunk);
    t_end = __ldg(p.tileoff + (p.chunk + 1) * p.lists_per_chunk);
  }

  if (tid == 0) {
    mbar_init(&bar.q_full[0], MODE == kGathered ? 64 : 1);
    mbar_init(&bar.q_full[1], MODE == kGathered ? 64 : 1);
    mbar_init(&bar.q_empty[0], 1);
    mbar_init(&bar.q_empty[1], 1);
    for (int s = 0; s < 3; ++s) {
      mbar_init(&bar.k_full[s], 1);
      mbar_init(&bar.v_full[s], 1);
      mbar_init(&bar.k_empty[s], 1);
      mbar_init(&bar.v_empty[s], 1);
    }
    mbar_init(&bar.s_full[0], 1);
    mbar_init(&bar.s_full[1], 1);
    mbar_init(&bar.p_full, 256);
    mbar_init(&bar.o_done[0], 1);
    mbar_init(&bar.o_done[1], 1);
    mbar_init(&bar.mma_done, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar.o_full[b], 1);
      mbar_init(&bar.o_free[b], 128);
      mbar_init(&bar.stat_full[b], 256);
    }
    bar.abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    if (MODE == kQueryMajor) tma_prefetch_desc(&tmQ);
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

  // Register split (launch: 512 threads x 128): see kRegSplitTotal.
  if (warp < 4) {
    setmaxnreg_dec<kRegsWG0>();
    if (warp == 0) {
      // ---------------------------------------------------------- producers
      // Lane 0 loads query tiles (query-major) and K chunks; lane 1 loads V chunks.
      // K and V have separate rings: a K slot frees once its S = Q K^T is done, long
      // before the V slot of the same chunk (freed by P V).
      if (lane < 2) {
        const bool kside = lane == 0;
        uint64_t *full = kside ? bar.k_full : bar.v_full;
        uint64_t *empty = kside ? bar.k_empty : bar.v_empty;
        const CUtensorMap *m0 = kside ? &tmK : &tmV;
        const CUtensorMap *m1 = kside ? &tmK1 : &tmV1;
        const int off = kside ? C::K_OFF : C::V_OFF;
        uint32_t cnt = 0;
        int lt = 0;
        bool ok = true;
        for (TileIter<MODE> it(p, t_begin, t_end); ok && it.valid(); it.next(), ++lt) {
          TileInfo ti;
          it.get(p, ti);
          if (MODE == kQueryMajor && kside) {
            const int qb = lt & 1;
            if (!(ok = mbar_wait(&bar.q_empty[qb], ((lt >> 1) & 1) ^ 1, abort, p.status, site0 + 1))) break;
            unsigned char *qd = sbase + C::Q_OFF + qb * C::TILE;
            mbar_arrive_expect_tx(&bar.q_full[qb], C::BYTES);
            tma_load_4d(qd, &tmQ, &bar.q_full[qb], 0, ti.i0, ti.h, ti.b);
            if (D != 64) tma_load_4d(qd + C::R0, &tmQ1, &bar.q_full[qb], 64, ti.i0, ti.h, ti.b);
          }
          for (int m = 0; m < ti.nc; ++m, ++cnt) {
            const int st = cnt % C::ST;
            if (!(ok = mbar_wait(&empty[st], ((cnt / C::ST) & 1) ^ 1, abort, p.status, site0 + 2))) break;
            const int key = chunk_key<MODE>(p, ti, m);
            unsigned char *dst = sbase + off + st * C::TILE;
            mbar_arrive_expect_tx(&full[st], C::BYTES);
            tma_load_4d(dst, m0, &full[st], 0, key, ti.hk, ti.b);
            if (D != 64) tma_load_4d(dst + C::R0, m1, &full[st], 64, key, ti.hk, ti.b);
          }
        }
        // Let every load issued so far land before the CTA can retire.
        if (*abort) {
          for (uint32_t u = (cnt > (uint32_t)C::ST ? cnt - C::ST : 0); u < cnt; ++u) {
            const unsigned long long t0 = global_timer_ns();
            while (!mbar_try_wait(&full[u % C::ST], (u / C::ST) & 1) && global_timer_ns() - t0 < kWaitTimeoutNs) {}
          }
        }
      }
    } else if (warp == 1) {
      // -------------------------------------------------------- MMA issuer
      if (lane == 0) {
        constexpr uint32_t idS = idesc_bf16(128, 128, 0, 0);
        constexpr uint32_t idO64 = idesc_bf16(128, 64, 0, 1);
        constexpr uint32_t idO128 = idesc_bf16(128, 128, 0, 1);
        constexpr uint32_t idO16 = idesc_bf16(128, 16, 0, 1);
        uint32_t kvc = 0, scnt = 0, pcnt = 0;
        uint32_t ofree_uses[2] = {0u, 0u};  // tiles started per O buffer
        auto ofree_parity = [&](int b) -> uint32_t { return ((ofree_uses[b]++) & 1) ^ 1; };
        int lt = 0;
        bool ok = true;
        auto issue_pv = [&](uint32_t tO, int first, uint32_t sbuf, int st) {
          const uint32_t vt = base + C::V_OFF + st * C::TILE;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t acc = (first && kk == 0) ? 0u : 1u;
            const uint32_t a = sbuf + kk * 8;
            if (D == 128) {
              umma_ts(tO, a, v_desc<D>(vt, kk, 2), idO128, acc);
            } else {
              umma_ts(tO, a, v_desc<D>(vt, kk, 0), idO64, acc);
              if (D == 80) umma_ts(tO + 64, a, v_desc<D>(vt, kk, 1), idO16, acc);
            }
          }
        };
        // Chunks of consecutive tiles form one stream: S of chunk g is issued before
        // P V of chunk g-1, also across a tile boundary, so the next tile's first
        // S = Q K^T overlaps the current tile's last softmax.
        struct Pending { bool valid, first, last; uint32_t sbuf, tO; int st, ob; };
        Pending pend = {false, false, false, 0u, 0u, 0, 0};
        uint32_t pv_slot = 0;  // pipeline slot of the pending P V
        auto issue_pending = [&]() -> bool {
          if (!mbar_wait(&bar.p_full, pcnt & 1, abort, p.status, site0 + 5)) return false;
          ++pcnt;
          if (!mbar_wait(&bar.v_full[pend.st], (pv_slot / C::ST) & 1, abort, p.status, site0 + 6)) return false;
          if (pend.first) {
            if (!mbar_wait(&bar.o_free[pend.ob], ofree_parity(pend.ob), abort, p.status, site0 + 7)) return false;
          }
          tc_fence_after();
          issue_pv(pend.tO, pend.first, pend.sbuf, pend.st);
          // Every P V completes a phase of o_done[its index & 1] (the softmax tracks
          // them in order); a tile's last one also hands the O buffer to the epilogue.
          umma_commit(&bar.o_done[pv_slot & 1]);
          if (pend.last) umma_commit(&bar.o_full[pend.ob]);
          umma_commit(&bar.v_empty[pend.st]);
          pend.valid = false;
          return true;
        };
        for (TileIter<MODE> it(p, t_begin, t_end); ok && it.valid(); it.next(), ++lt) {
          TileInfo ti;
          it.get(p, ti);
          const int qb = lt & 1, ob = lt & 1;
          const uint32_t tO = tmem + 256 + 128 * ob;
          if (!(ok = mbar_wait(&bar.q_full[qb], (lt >> 1) & 1, abort, p.status, site0 + 3))) break;
          tc_fence_after();
          const uint32_t qt = base + C::Q_OFF + qb * C::TILE;
          for (int m = 0; m < ti.nc; ++m) {
            const int st = kvc % C::ST;
            if (!(ok = mbar_wait(&bar.k_full[st], (kvc / C::ST) & 1, abort, p.status, site0 + 4))) break;
            tc_fence_after();
            const uint32_t kt = base + C::K_OFF + st * C::TILE;
            const uint32_t sb = tmem + 128 * (scnt & 1);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)
              umma_ss(sb, kmajor_desc<D>(qt, ks), kmajor_desc<D>(kt, ks), idS, ks > 0 ? 1u : 0u);
            umma_commit(&bar.s_full[scnt & 1]);
            umma_commit(&bar.k_empty[st]);
            if (m == ti.nc - 1) umma_commit(&bar.q_empty[qb]);
            if (pend.valid && !(ok = issue_pending())) break;
            pend = {true, m == 0, m == ti.nc - 1, sb, tO, st, ob};
            pv_slot = kvc;
            ++scnt;
            ++kvc;
          }
        }
        if (ok && pend.valid) ok = issue_pending();
        // Every MMA issued so far completes before TMEM is released.
        umma_commit(&bar.mma_done);
        const unsigned long long t0 = global_timer_ns();
        while (!mbar_try_wait(&bar.mma_done, 0) && global_timer_ns() - t0 < kWaitTimeoutNs) {}
      }
    } else if (MODE == kGathered) {
      // -------------------------------------------------------- row gather
      // Thread u owns rows u and u + 64 of the tile: it reads their list entries
      // first, then issues all of their 16-byte copies (no dependent loads between).
      const int u = tid - 64;  // 0..63
      constexpr int VPR = D / 8;  // 16-byte vectors per row
      const int npast = p.npast;
      int lt = 0;
      for (TileIter<MODE> it(p, t_begin, t_end); it.valid(); it.next(), ++lt) {
        TileInfo ti;
        it.get(p, ti);
        const int qb = lt & 1;
        uint32_t ent[2] = {0u, 0u};
#pragma unroll
        for (int k2 = 0; k2 < 2; ++k2)
          if (u + 64 * k2 < ti.rows) ent[k2] = __ldg(p.entries + ti.ent0 + u + 64 * k2);
        if (!mbar_wait(&bar.q_empty[qb], ((lt >> 1) & 1) ^ 1, abort, p.status, site0 + 11)) break;
        const uint32_t qt = base + C::Q_OFF + qb * C::TILE;
#pragma unroll
        for (int k2 = 0; k2 < 2; ++k2) {
          const int r = u + 64 * k2;
          const bool valid = r < ti.rows;
          const uint16_t *row = p.q;
          if (valid) {
            const uint32_t ig = ent[k2] / (uint32_t)npast;
            const int g = (int)(ig % (uint32_t)p.G);
            const int i = (int)(ig / (uint32_t)p.G);
            row = p.q + ti.b * p.q_sb + (int64_t)(ti.hk * p.G + g) * p.q_sh + (int64_t)i * p.q_sn;
          }
#pragma unroll
          for (int c = 0; c < VPR; ++c) {
            uint32_t dst;
            if (c < 8) {
              dst = qt + r * 128 + ((c ^ (r & 7)) << 4);
            } else if (D == 128) {
              dst = qt + C::R0 + r * 128 + (((c - 8) ^ (r & 7)) << 4);
            } else {
              dst = qt + C::R0 + r * 32 + (((c - 8) ^ ((r >> 2) & 1)) << 4);
            }
            cp_async_16_zfill(dst, valid ? row + c * 8 : p.q, valid);
          }
        }
        cp_async_commit();
        cp_async_wait_all();
        fence_proxy_async_smem();
        mbar_arrive(&bar.q_full[qb]);
      }
    }
  } else if (warp < 12) {
    // ------------------------------------------------------------ softmax
    // tcgen05.ld / st are warp-collective (.sync.aligned): every wait is made
    // warp-uniform with __all_sync, and no TMEM access sits under a per-row branch.
    setmaxnreg_inc<kRegsSoftmax>();
    const int half = (warp - 4) >> 2;       // key half of each chunk
    const int r = (tid - 128) & 127;        // row within the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    // O columns this half rescales: [oc0, oc1).
    constexpr int OH = ((D / 2 + 15) / 16) * 16;
    const int oc0 = half ? OH : 0, oc1 = half ? D : OH;
    const float sl2 = p.scale_log2;
    uint32_t scnt = 0;
    // P V number k (counted over all chunks of this CTA, like scnt) completes phase
    // k >> 1 of o_done[k & 1].  pv_seen: P Vs whose completion was already awaited.
    uint32_t pv_seen = 0;
    int lt = 0;
    bool ok = true;
    for (TileIter<MODE> it(p, t_begin, t_end); ok && it.valid(); it.next(), ++lt) {
      TileInfo ti;
      it.get(p, ti);
      const int ob = lt & 1;
      const uint32_t tO = tmem + lane_off + 256 + 128 * ob;
      const bool live = r < ti.rows;
      const int i = ti.i0 + r;  // query-major row
      const int32_t *irow = (MODE == kQueryMajor && p.is_moba && live)
                                ? p.idx + (((int64_t)ti.b * p.hq + ti.h) * p.N + i) * p.topk
                                : nullptr;
      float m_run = -INFINITY, l_run = 0.f;
      for (int m = 0; m < ti.nc; ++m, ++scnt) {
        const int sbi = scnt & 1;
        const uint32_t tS = tmem + lane_off + 128 * sbi;
        // The two halves must take every decision together (they meet at named
        // barriers), so each wait's outcome is AND-ed over both warpgroups.
        ok = mbar_wait(&bar.s_full[sbi], (scnt >> 1) & 1, abort, p.status, site0 + 12);
        if (!(ok = named_barrier_and(1, 256, ok))) break;
        tc_fence_after();
        uint32_t sv[64];
        tmem_ld32(tS + 64 * half, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld32(tS + 64 * half + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        tmem_wait_ld();
        float *s = reinterpret_cast<float *>(sv);
        // Masks.
        const int key0 = chunk_key<MODE>(p, ti, m) + 64 * half;
        if (MODE == kQueryMajor) {
          if (p.is_moba) {
            if (m < ti.ntail) {
              // Window tail into an earlier block: keys i - j < window that the row's
              // own selection does not already cover.
              bool covered = false;
              if (irow) {
                const int blk = key0 / p.block;
                for (int u2 = 0; u2 < p.topk; ++u2) covered |= (__ldg(irow + u2) == blk);
              }
#pragma unroll
              for (int e = 0; e < 64; ++e)
                if (covered || !live || i - (key0 + e) >= p.window) s[e] = -INFINITY;
            } else if (key0 + 64 > ti.i0) {
#pragma unroll
              for (int e = 0; e < 64; ++e)
                if (key0 + e > i) s[e] = -INFINITY;
            }
          } else {
            const bool full = (key0 + 63 <= ti.i0) && (key0 >= ti.i0 + ti.rows - 1 - p.window + 1);
            if (!full) {
#pragma unroll
              for (int e = 0; e < 64; ++e) {
                const int j = key0 + e;
                if (j > i || i - j >= p.window) s[e] = -INFINITY;
              }
            }
          }
        }
        float mx4[8];
#pragma unroll
        for (int u2 = 0; u2 < 8; ++u2) mx4[u2] = s[u2];
#pragma unroll
        for (int e = 8; e < 64; ++e) mx4[e & 7] = fmaxf(mx4[e & 7], s[e]);
        // The row maximum over both halves of the chunk.
        bar.xmax[sbi][half][r] = fmaxf(fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])),
                                       fmaxf(fmaxf(mx4[4], mx4[5]), fmaxf(mx4[6], mx4[7])));
        named_barrier_sync(1, 256);
        const float mx = fmaxf(bar.xmax[sbi][0][r], bar.xmax[sbi][1][r]);
        const float m_new = fmaxf(m_run, mx * sl2);
        // Raise the running maximum only when it grows by more than 2^8 (or from
        // -inf); rows that keep theirs multiply O by 1 when the warp rescales.  Both
        // halves of a row take the same decision from the same numbers.
        const bool raise = (m == 0) || (m_new > m_run + (float)kRescaleThreshold);
        const bool scale_o = raise && m > 0 && m_run != -INFINITY;
        const float alpha = scale_o ? ex2_approx(m_run - m_new) : 1.f;
        if (raise) {
          l_run *= alpha;
          m_run = m_new;
        }
        const float mu = (m_run == -INFINITY) ? 0.f : m_run;
        float ls[8];
#pragma unroll
        for (int u2 = 0; u2 < 8; ++u2) ls[u2] = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float x0 = fmaf(s[2 * e], sl2, -mu), x1 = fmaf(s[2 * e + 1], sl2, -mu);
          const float p0 = ((2 * e) % 16 >= 16 - kExpEmuPer16) ? exp2_fma(x0) : ex2_approx(x0);
          const float p1 = ((2 * e + 1) % 16 >= 16 - kExpEmuPer16) ? exp2_fma(x1) : ex2_approx(x1);
          ls[e & 7] += p0 + p1;
          sv[e] = pack_bf16x2(p0, p1);
        }
        // P of keys [64 half, 64 half + 64) -> TMEM columns [32 half, 32 half + 32).
        tmem_st16(tS + 32 * half, *reinterpret_cast<uint32_t(*)[16]>(&sv[0]));
        tmem_st16(tS + 32 * half + 16, *reinterpret_cast<uint32_t(*)[16]>(&sv[16]));
        l_run += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
        // Before P V number scnt may be issued, the P V two back must be complete
        // (o_done[scnt & 1] is reused by it); if this chunk rescales O, the previous
        // one too.  The pair of warpgroups decides together.
        const bool rescale = (m > 0) && named_barrier_and(2, 256, !__any_sync(FULL, scale_o)) == false;
        const uint32_t need = rescale ? scnt : (scnt >= 1 ? scnt - 1 : 0);
        while (pv_seen < need) {
          ok = mbar_wait(&bar.o_done[pv_seen & 1], (pv_seen >> 1) & 1, abort, p.status, site0 + 13);
          if (!(ok = named_barrier_and(1, 256, ok))) break;
          ++pv_seen;
        }
        if (!ok) break;
        if (rescale) {
          // O holds chunks 0..m-1 now; rescale this half's columns where a row of the
          // warp raised its maximum.
          tc_fence_after();
          if (__any_sync(FULL, scale_o)) {
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 16) {
              if (c0 < oc0 || c0 >= oc1) continue;
              uint32_t o[16];
              tmem_ld16(tO + c0, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st16(tO + c0, o);
            }
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar.p_full);
      }
      if (!ok) break;
      // Hand the row statistics to the epilogue once it has drained this O buffer's
      // previous tile (that also orders every earlier P V before this point).
      ok = mbar_wait(&bar.o_free[ob], ((lt >> 1) & 1) ^ 1, abort, p.status, site0 + 14);
      if (!(ok = named_barrier_and(1, 256, ok))) break;
      bar.stat[ob][half][r] = make_float2(m_run, l_run);
      mbar_arrive(&bar.stat_full[ob]);
    }
  } else {
    // ----------------------------------------------------------- epilogue
    // Keeps the registers it was launched with (kRegsEpilogue).
    const int r = tid - 384;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    int lt = 0;
    bool ok = true;
    for (TileIter<MODE> it(p, t_begin, t_end); ok && it.valid(); it.next(), ++lt) {
      TileInfo ti;
      it.get(p, ti);
      const int ob = lt & 1;
      const uint32_t tO = tmem + lane_off + 256 + 128 * ob;
      const bool live = r < ti.rows;
      int i = ti.i0 + r, h = ti.h, slot = 0;
      if (MODE == kGathered && live) {
        const uint32_t ent = __ldg(p.entries + ti.ent0 + r);
        slot = (int)(ent % (uint32_t)p.npast);
        const uint32_t ig = ent / (uint32_t)p.npast;
        h = ti.hk * p.G + (int)(ig % (uint32_t)p.G);
        i = (int)(ig / (uint32_t)p.G);
      }
      ok = mbar_wait(&bar.stat_full[ob], (lt >> 1) & 1, abort, p.status, site0 + 15);
      ok = ok && mbar_wait(&bar.o_full[ob], (lt >> 1) & 1, abort, p.status, site0 + 16);
      if (!(ok = __all_sync(FULL, ok))) break;
      tc_fence_after();
      const float2 st0 = bar.stat[ob][0][r], st1 = bar.stat[ob][1][r];
      const float m_run = st0.x, l_run = st0.y + st1.y;
      const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
      const float own_lse = (m_run + log2f(l_run)) * 0.69314718055994530942f;  // natural log
      // Destination: a partial slot (gathered tiles: the row's past-block slot; MoBA
      // query-major tiles: the own-block slot topk-1, merged afterwards), or the
      // output itself when nothing needs merging (SWA, or topk = 1).
      uint16_t *dst;
      float *ldst;
      if (MODE == kGathered || (p.is_moba && p.npast > 0)) {
        const int sl = (MODE == kGathered) ? slot : p.npast;
        const int64_t pidx = (((int64_t)ti.b * p.hq + h) * p.chunk_rows + (i - p.chunk * p.chunk_rows)) * p.topk + sl;
        dst = p.opart + pidx * D;
        ldst = p.lpart + pidx;
      } else {
        dst = p.out + ti.b * p.o_sb + (int64_t)h * p.o_sh + (int64_t)i * p.o_sn;
        ldst = p.lse + ((int64_t)ti.b * p.hq + h) * p.N + i;
      }
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        const int cols = (D - c0) < 32 ? (D - c0) : 32;  // D = 80 ends with 16
        uint32_t o[32];
        __syncwarp();
        if (cols == 32) tmem_ld32(tO + c0, o);
        else tmem_ld16(tO + c0, *reinterpret_cast<uint32_t(*)[16]>(&o[0]));
        tmem_wait_ld();
        if (live) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            if (v4 * 8 >= cols) break;
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[8 * v4 + 0]) * inv_l, __uint_as_float(o[8 * v4 + 1]) * inv_l);
            w.y = pack_bf16x2(__uint_as_float(o[8 * v4 + 2]) * inv_l, __uint_as_float(o[8 * v4 + 3]) * inv_l);
            w.z = pack_bf16x2(__uint_as_float(o[8 * v4 + 4]) * inv_l, __uint_as_float(o[8 * v4 + 5]) * inv_l);
            w.w = pack_bf16x2(__uint_as_float(o[8 * v4 + 6]) * inv_l, __uint_as_float(o[8 * v4 + 7]) * inv_l);
            *reinterpret_cast<uint4 *>(dst + c0 + 8 * v4) = w;
          }
        }
      }
      if (live) *ldst = own_lse;
      tc_fence_before();
      mbar_arrive(&bar.o_free[ob]);
    }
  }

  // Roles ran on single lanes or with per-thread waits: reconverge every warp before
  // the CTA barrier (bar.sync is warp-aligned) and before the warp-wide dealloc.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ launch

template <int D, int MODE>
static cudaError_t launch_attn_dm(const CUtensorMap *maps, const AttnParams &p, int grid,
                                  cudaStream_t st) {
  using C = AttnCfg<D>;
  auto kern = attn_fwd_kernel<D, MODE>;
  // The warpgroups re-split the registers the CTA is launched with (setmaxnreg); a
  // build that launched with fewer than 168 per thread would leave an increase
  // waiting forever, so refuse to launch it.
  static int regs = 0;
  if (regs == 0) {
    cudaFuncAttributes fa;
    cudaError_t e0 = cudaFuncGetAttributes(&fa, kern);
    if (e0 != cudaSuccess) return e0;
    regs = fa.numRegs;
  }
  if (regs * kAttnThreads < kRegSplitTotal) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<grid, kAttnThreads, C::SMEM, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], p);
  return cudaGetLastError();
}

// maps: Q (64-col box), Q tail, K, K tail, V, V tail.
cudaError_t launch_attn(const CUtensorMap *maps, const AttnParams &p, int mode, int grid,
                        cudaStream_t st) {
  if (mode == kQueryMajor) {
    switch (p.d) {
      case 64: return launch_attn_dm<64, kQueryMajor>(maps, p, grid, st);
      case 80: return launch_attn_dm<80, kQueryMajor>(maps, p, grid, st);
      case 128: return launch_attn_dm<128, kQueryMajor>(maps, p, grid, st);
    }
  } else {
    switch (p.d) {
      case 64: return launch_attn_dm<64, kGathered>(maps, p, grid, st);
      case 80: return launch_attn_dm<80, kGathered>(maps, p, grid, st);
      case 128: return launch_attn_dm<128, kGathered>(maps, p, grid, st);
    }
  }
  return cudaErrorInvalidValue;
}

int attn_smem_bytes(int d) {
  switch (d) {
    case 64: return AttnCfg<64>::SMEM;
    case 80: return AttnCfg<80>::SMEM;
    case 128: return AttnCfg<128>::SMEM;
  }
  return 0;
}

}  // namespace moba
