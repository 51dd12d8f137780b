// attn.cu -- block-sparse / sliding-window attention forward on sm_100a tensor cores.
//
// [MoBA] = "MoBA: 어텐션에 전문가 혼합을 적용해 긴 문맥을 효율적으로 처리하는 블록 어텐션
//          (feat. MoonshotAI)", PyTorch KR forum summary of the MoBA paper.
// [SWA]  = "SWA + MoE: 어텐션과 희소 전문가", Bit-Axon architecture page.
//
// One persistent kernel, two work kinds:
//   kQueryMajor  contiguous 128-row query tiles of one (batch, q-head).  MoBA: the causal
//                own block (§"MoBA의 구현": current block with causal=True) plus the
//                window tail into earlier blocks the row did not select; the result is
//                the own-block partial that the merge pass combines with the past-block
//                partials (step 5).  SWA: the causal band of [SWA] §"슬라이딩 윈도우
//                마스크", written straight to the output.
//   kGathered    gathered (row, q-head) pairs of one block-major list against the whole
//                past block they picked (steps 3-4, causal=False); writes a normalised
//                partial output and its log-sum-exp per (row, slot).
//
// Each CTA runs two tile streams, A and B, over a shared K/V chunk sequence: a work
// unit is a pair of 128-row tiles that attend to the same keys (two q-heads of one KV
// head, two row tiles of one head, or 256 entries of one block list).  While one
// stream's softmax runs, the tensor core works on the other stream's S = Q K^T and
// O += P V, so the exponentials and the MMAs overlap (the FA4 ping-pong).
//   warp 0       TMA producers: lane 0 the query tiles (query-major) and K chunks of 128
//                keys, lane 1 the V chunks (separate K and V rings)
//   warp 1       tcgen05 MMA issuer (one thread) and TMEM owner
//   warps 2-3    query-row gather (gathered work): TMA gather4 of four rows per
//                instruction, or cp.async when q's strides admit no 2-D row view
//   warps 4-7    stream A softmax + epilogue; thread r owns row r (TMEM lane r)
//   warps 8-11   stream B softmax + epilogue
// TMEM: S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512).  P (bf16) overwrites
// its own S columns and is the A operand (from TMEM) of O += P V.  A stream's S of
// chunk m is issued after its P V of chunk m-1, so when the softmax sees S(m) complete
// (commit semantics: every earlier MMA is complete) it may rescale O at once.  The
// running maximum is raised lazily: O and l are rescaled only when it grows by more
// than 2^8.  The gathered pass skips the row maximum once a row has one: a chunk is
// computed against the running maximum and redone with its exact maximum only when its
// row sum exceeds 2^60.  MoBA launches let the two streams' exponentials overlap;
// sliding-window launches alternate them per sub-partition.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "params.h"

namespace moba {

constexpr int kAttnThreads = 384;

// Packed f32x2 arithmetic (two lanes of fp32 per instruction, each rounded as the
// scalar instruction would be): d = a * b + c and d += a on pairs.
__device__ __forceinline__ void fma_f32x2(float &d0, float &d1, float a0, float a1, float b,
                                          float c) {
  asm("{.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %4};\n\tmov.b64 rc, {%5, %5};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b), "f"(c));
}
// 2^x on the exponential unit, kept in program order (volatile): the compiler may not
// hoist the softmax's exponentials above the barrier waits before them, where they
// would issue while the other stream's exponentials are running (measured 2% slower
// at 1M tokens).
__device__ __forceinline__ float ex2_in_order(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void add_f32x2(float &d0, float &d1, float a0, float a1) {
  asm("{.reg .b64 ra, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rd, {%0, %1};\n\t"
      "add.rn.f32x2 rd, rd, ra;\n\tmov.b64 {%0, %1}, rd;}"
      : "+f"(d0), "+f"(d1)
      : "f"(a0), "f"(a1));
}
constexpr int kRescaleThreshold = 8;  // log2 units
// A gathered chunk computed against a stale running maximum is kept while its row sum is
// at most 2^60: every probability is then below 2^60, so P (bf16), l and O (fp32) stay
// finite.
constexpr float kSumBound = 1.152921504606846976e18f;
// Of every 16 probabilities, this many take the FMA-pipe 2^x (exp2_fma) instead of
// the MUFU unit.
#ifndef MOBA_EXP_EMU_PER16
#define MOBA_EXP_EMU_PER16 0
#endif
constexpr int kExpEmuPer16 = MOBA_EXP_EMU_PER16;
// Registers per thread after the re-split: producer/MMA/gather, each softmax stream.
constexpr int kRegsWG0 = 72, kRegsSoftmax = 216;
constexpr int kRegSplitTotal = 128 * (kRegsWG0 + 2 * kRegsSoftmax);
static_assert(kRegSplitTotal <= 65536, "register split exceeds the register file");

template <int D>
struct AttnCfg {
  static constexpr int ST = (D == 128) ? 2 : 3;            // K and V ring stages each
  static constexpr int R0 = 128 * 128;                     // bytes of the 64-column region
  static constexpr int R1 = (D == 128) ? 128 * 128 : (D == 80 ? 128 * 32 : 0);
  static constexpr int TILE = R0 + ((R1 + 1023) / 1024) * 1024;  // one 128 x D operand tile
  static constexpr int Q_OFF = 0;                          // Q_A, Q_B
  static constexpr int K_OFF = 2 * TILE;                   // K ring
  static constexpr int V_OFF = K_OFF + ST * TILE;          // V ring
  static constexpr int EPI_OFF = V_OFF + ST * TILE;       // 8 softmax warps x 32 rows x 64 B
  static constexpr int BAR_OFF = EPI_OFF + 8 * 2048;
  static constexpr int SMEM = BAR_OFF + 1024 + 1024;       // + barriers + alignment slack
  static constexpr uint32_t BYTES = 128u * D * 2u;         // bytes one full tile load moves
};

struct Bars {
  uint64_t q_full[2], q_empty[2];                          // per stream
  uint64_t k_full[3], v_full[3], k_empty[3], v_empty[3];
  uint64_t s_full[2], p_full[2], o_full[2];                // per stream
  uint64_t turn[2][4];   // exponential-phase token of stream x, per sub-partition pair
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

// One stream's tile of a work unit.
struct Tile {
  int b, h, hk;
  int i0;      // query-major: first query row (at key position q_off + i0)
  int rows;    // valid rows (0: the stream is idle in this unit)
  int ent0;    // gathered: first list entry
  int cB;      // query-major MoBA: first key (position) of the own block of the tile's
               // first row (the tile's later rows may sit in the next block)
};

// A work unit: two tiles over one key-chunk sequence.
struct Unit {
  Tile t[2];
  int b, hk;
  int key0;    // first key of chunk 0
  int nc;      // chunks
  int j;       // gathered: the past block
};

// Query-major units.  With GQA (G >= 2) a unit is two q-heads of one KV head at the
// same rows; otherwise two consecutive row tiles of one head (MoBA: of one block),
// attending to the union of their key ranges with per-row masks.
__device__ __forceinline__ void query_major_unit(const AttnParams &p, int u, Unit &w) {
  const int nq = (p.row_end - p.row_begin + kTileRows - 1) / kTileRows;
  int qt0, qt1, g0, g1, hb;
  if (p.G >= 2) {
    const int per_hk = (p.G + 1) / 2;                      // head pairs per KV head
    const int HB = p.batch * p.hkv * per_hk;
    const int slot = nq - 1 - u / HB;                      // later (heavier) rows first
    hb = u % HB;
    qt0 = qt1 = slot;
    const int ph = hb % per_hk;
    g0 = 2 * ph;
    g1 = (2 * ph + 1 < p.G) ? 2 * ph + 1 : -1;
    hb /= per_hk;                                          // (b, hk)
  } else {
    // Row-tile pairs, grouped by tpb tiles from the pass's first row: for MoBA a pair
    // stays inside one block when that row starts a block; otherwise (a chunk that
    // starts mid-block) a pair may span two blocks, which the union key range and the
    // per-row masks below handle.
    const int tpb = p.is_moba ? p.block / kTileRows : nq;   // tiles per pairing group
    const int ppg = (tpb + 1) / 2;                         // pairs per group
    const int ngroups = (nq + tpb - 1) / tpb;
    const int HB = p.batch * p.hkv;
    const int pr = ngroups * ppg - 1 - u / HB;             // later rows first
    hb = u % HB;
    const int grp = pr / ppg, k = pr % ppg;
    qt0 = grp * tpb + 2 * k;
    const int lim = min(nq, (grp + 1) * tpb);
    qt1 = (qt0 + 1 < lim) ? qt0 + 1 : -1;
    g0 = 0;
    g1 = (qt1 >= 0) ? 0 : -1;
    if (qt1 < 0) qt1 = qt0;
  }
  w.b = hb / p.hkv;
  w.hk = hb % p.hkv;
  w.j = 0;
  int lo = 0x7fffffff, hi = -1;
  for (int x = 0; x < 2; ++x) {
    Tile &t = w.t[x];
    const int g = x ? g1 : g0;
    const int qt = x ? qt1 : qt0;
    t.b = w.b;
    t.hk = w.hk;
    t.h = w.hk * p.G + (g < 0 ? 0 : g);
    t.i0 = p.row_begin + qt * kTileRows;
    t.rows = (g < 0) ? 0 : min(kTileRows, p.row_end - t.i0);
    t.ent0 = 0;
    t.cB = 0;
    if (t.rows == 0) continue;
    // Key positions: row i0 of q sits at position q_off + i0.
    const int a0 = p.q_off + t.i0;
    const int ilast = a0 + t.rows - 1;
    int first;
    if (p.is_moba) {
      t.cB = (a0 / p.block) * p.block;
      first = t.cB;
      if (p.window > 0) first = min(t.cB, (max(0, a0 - p.window + 1) / kTileKeys) * kTileKeys);
    } else {
      first = (max(0, a0 - p.window + 1) / kTileKeys) * kTileKeys;
    }
    lo = min(lo, first);
    hi = max(hi, ilast);
  }
  w.key0 = lo;
  w.nc = (hi - lo) / kTileKeys + 1;
}

__device__ __forceinline__ void gathered_unit(const AttnParams &p, int4 rec, Unit &w) {
  const int L = rec.x;
  w.j = L % p.nblk;
  w.hk = (L / p.nblk) % p.hkv;
  w.b = (L / (p.nblk * p.hkv)) % p.batch;
  w.key0 = w.j * p.block;
  w.nc = p.block / kTileKeys;
  for (int x = 0; x < 2; ++x) {
    Tile &t = w.t[x];
    t.b = w.b;
    t.hk = w.hk;
    t.h = -1;
    t.i0 = 0;
    t.cB = 0;
    t.ent0 = rec.y + x * kTileRows;
    t.rows = max(0, min(kTileRows, rec.z - x * kTileRows));
  }
}

// Walks this CTA's units u = u_begin + blockIdx.x, u += gridDim.x.  Gathered units
// come from the unit table; the next record is loaded one unit ahead.
template <int MODE>
struct UnitIter {
  int u, u_end;
  int4 nxt;
  __device__ __forceinline__ UnitIter(const AttnParams &p, int u_begin, int u_end_) {
    u = u_begin + (int)blockIdx.x;
    u_end = u_end_;
    if (MODE == kGathered && u < u_end) nxt = __ldg(p.tiles + u);
  }
  __device__ __forceinline__ bool valid() const { return u < u_end; }
  __device__ __forceinline__ void get(const AttnParams &p, Unit &w) {
    if (MODE == kGathered) {
      const int4 cur = nxt;
      if (u + (int)gridDim.x < u_end) nxt = __ldg(p.tiles + u + gridDim.x);
      gathered_unit(p, cur, w);
    } else {
      query_major_unit(p, u, w);
    }
  }
  __device__ __forceinline__ void next() { u += gridDim.x; }
};

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

  // Unit range.
  int u_begin = 0, u_end = p.ntiles;
  if (MODE == kGathered) {
    u_begin = __ldg(p.tileoff + p.chunk * p.lists_per_chunk);
    u_end = __ldg(p.tileoff + (p.chunk + 1) * p.lists_per_chunk);
  }

  if (tid == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bar.q_full[x], (MODE == kGathered && !p.q_gather_tma) ? 32 : 1);
      mbar_init(&bar.q_empty[x], 1);
      mbar_init(&bar.s_full[x], 1);
      mbar_init(&bar.p_full[x], 128);
      mbar_init(&bar.o_full[x], 1);
    }
    for (int s = 0; s < 3; ++s) {
      mbar_init(&bar.k_full[s], 1);
      mbar_init(&bar.v_full[s], 1);
      mbar_init(&bar.k_empty[s], 1);
      mbar_init(&bar.v_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x)
      for (int q = 0; q < 4; ++q) mbar_init(&bar.turn[x][q], 1);
    mbar_init(&bar.mma_done, 1);
    bar.abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    if (MODE == kQueryMajor || p.q_gather_tma) tma_prefetch_desc(&tmQ);
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

  // Register split (launch: 384 threads x 168): see kRegSplitTotal.
  if (warp < 4) {
    setmaxnreg_dec<kRegsWG0>();
    if (warp == 0) {
      // ---------------------------------------------------------- producers
      // Lane 0 loads the query tiles (query-major) and K chunks; lane 1 the V chunks.
      if (lane < 2) {
        const bool kside = lane == 0;
        uint64_t *full = kside ? bar.k_full : bar.v_full;
        uint64_t *empty = kside ? bar.k_empty : bar.v_empty;
        const CUtensorMap *m0 = kside ? &tmK : &tmV;
        const CUtensorMap *m1 = kside ? &tmK1 : &tmV1;
        const int off = kside ? C::K_OFF : C::V_OFF;
        uint32_t cnt = 0;
        uint32_t quse[2] = {0u, 0u};
        bool ok = true;
        // Test hook (moba_debug_fault_next_launch): the V loader of CTA 0 of the launch
        // that finds the one-shot flag set takes it and leaves its first V chunk unloaded,
        // so that the MMA issuer's wait for it runs out and the launch ends through the
        // bounded-wait path with MOBA_ERR_DEVICE.
        bool skip_first = false;
        if (!kside && blockIdx.x == 0 && atomicExch(&p.status[3], 0) == 1) skip_first = true;
        for (UnitIter<MODE> it(p, u_begin, u_end); ok && it.valid(); it.next()) {
          Unit w;
          it.get(p, w);
          if (MODE == kQueryMajor && kside) {
#pragma unroll
            for (int x = 0; x < 2; ++x) {
              if (!ok) break;
              const Tile &t = w.t[x];
              if (t.rows == 0) continue;
              ok = mbar_wait(&bar.q_empty[x], (quse[x] & 1) ^ 1, abort, p.status, site0 + 1);
              if (!ok) break;
              ++quse[x];
              unsigned char *qd = sbase + C::Q_OFF + x * C::TILE;
              mbar_arrive_expect_tx(&bar.q_full[x], C::BYTES);
              tma_load_4d(qd, &tmQ, &bar.q_full[x], 0, t.i0, t.h, t.b);
              if (D != 64) tma_load_4d(qd + C::R0, &tmQ1, &bar.q_full[x], 64, t.i0, t.h, t.b);
            }
            if (!ok) break;
          }
          for (int m = 0; m < w.nc; ++m, ++cnt) {
            const int st = cnt % C::ST;
            if (!(ok = mbar_wait(&empty[st], ((cnt / C::ST) & 1) ^ 1, abort, p.status, site0 + 2))) break;
            const int key = w.key0 + m * kTileKeys;
            unsigned char *dst = sbase + off + st * C::TILE;
            if (skip_first && cnt == 0) continue;   // nothing issued, nothing to drain
            mbar_arrive_expect_tx(&full[st], C::BYTES);
            tma_load_4d(dst, m0, &full[st], 0, key, w.hk, w.b);
            if (D != 64) tma_load_4d(dst + C::R0, m1, &full[st], 64, key, w.hk, w.b);
          }
        }
        // Let every load issued so far land before the CTA can retire.
        if (*abort) {
          for (uint32_t u = (cnt > (uint32_t)C::ST ? cnt - C::ST : 0); u < cnt; ++u) {
            const unsigned long long t0 = global_timer_ns();
            while (!mbar_try_wait(&full[u % C::ST], (u / C::ST) & 1) && global_timer_ns() - t0 < wait_limit_ns(p.status)) {}
          }
          for (int x = 0; x < 2; ++x) {
            if (quse[x] == 0) continue;
            const unsigned long long t0 = global_timer_ns();
            while (!mbar_try_wait(&bar.q_full[x], (quse[x] - 1) & 1) && global_timer_ns() - t0 < wait_limit_ns(p.status)) {}
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
        uint32_t kvc = 0;                      // pipeline slot of chunk 0 of this unit
        uint32_t quse[2] = {0u, 0u}, pcnt[2] = {0u, 0u};
        bool ok = true;
        for (UnitIter<MODE> it(p, u_begin, u_end); ok && it.valid(); it.next()) {
          Unit w;
          it.get(p, w);
          const bool act[2] = {w.t[0].rows > 0, w.t[1].rows > 0};
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            if (!act[x] || !ok) continue;
            ok = mbar_wait(&bar.q_full[x], quse[x] & 1, abort, p.status, site0 + 3);
            ++quse[x];
          }
          if (!ok) break;
          tc_fence_after();
          // Per chunk m, for each active stream: O += P V of chunk m-1, then S = Q K^T
          // of chunk m (the stream's S buffer is free once its P was consumed).
          for (int m = 0; m <= w.nc && ok; ++m) {
            const uint32_t slot_m = kvc + m, slot_p = kvc + m - 1;
            const int st_m = slot_m % C::ST, st_p = slot_p % C::ST;
            if (m < w.nc) {
              if (!(ok = mbar_wait(&bar.k_full[st_m], (slot_m / C::ST) & 1, abort, p.status, site0 + 4))) break;
            }
            if (m > 0) {
              if (!(ok = mbar_wait(&bar.v_full[st_p], (slot_p / C::ST) & 1, abort, p.status, site0 + 6))) break;
            }
#pragma unroll
            for (int x = 0; x < 2; ++x) {
              if (!act[x] || !ok) continue;
              const uint32_t sb = tmem + 128 * x;
              const uint32_t tO = tmem + 256 + 128 * x;
              if (m > 0) {
                if (!(ok = mbar_wait(&bar.p_full[x], pcnt[x] & 1, abort, p.status, site0 + 5))) break;
                ++pcnt[x];
                tc_fence_after();
                const uint32_t vt = base + C::V_OFF + st_p * C::TILE;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                  const uint32_t acc = (m == 1 && kk == 0) ? 0u : 1u;
                  const uint32_t a = sb + kk * 8;
                  if (D == 128) {
                    umma_ts(tO, a, v_desc<D>(vt, kk, 2), idO128, acc);
                  } else {
                    umma_ts(tO, a, v_desc<D>(vt, kk, 0), idO64, acc);
                    if (D == 80) umma_ts(tO + 64, a, v_desc<D>(vt, kk, 1), idO16, acc);
                  }
                }
                if (m == w.nc) umma_commit(&bar.o_full[x]);
              }
              if (m < w.nc) {
                const uint32_t qt = base + C::Q_OFF + x * C::TILE;
                const uint32_t kt = base + C::K_OFF + st_m * C::TILE;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks)
                  umma_ss(sb, kmajor_desc<D>(qt, ks), kmajor_desc<D>(kt, ks), idS, ks > 0 ? 1u : 0u);
                umma_commit(&bar.s_full[x]);
                if (m == w.nc - 1) umma_commit(&bar.q_empty[x]);
              }
            }
            if (!ok) break;
            if (m < w.nc) umma_commit(&bar.k_empty[st_m]);
            if (m > 0) umma_commit(&bar.v_empty[st_p]);
          }
          kvc += w.nc;
        }
        // Every MMA issued so far completes before TMEM is released.
        umma_commit(&bar.mma_done);
        const unsigned long long t0 = global_timer_ns();
        while (!mbar_try_wait(&bar.mma_done, 0) && global_timer_ns() - t0 < wait_limit_ns(p.status)) {}
      }
    } else if (MODE == kGathered) {
      // -------------------------------------------------------- row gather
      // Warp 2 fills stream A's query tile, warp 3 stream B's.
      const int x = warp - 2;
      const int npast = p.npast;
      const uint32_t qt = base + C::Q_OFF + x * C::TILE;
      uint32_t quse = 0;
      bool ok = true;
      if (p.q_gather_tma) {
        // TMA gather4: lane l owns tile rows 4l .. 4l+3 and fetches them, 64 columns
        // (and the 16-column tail for D = 80) per instruction, into the swizzled tile
        // layout; rows past the unit's end repeat a valid row and are never stored.
        // While a unit's copies are in flight the warp decodes the next unit's rows.
        auto rows_of = [&](const Tile &t, int (&rr)[4], bool pf) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int r = 4 * lane + e;
            const uint32_t ent = __ldg(p.entries + t.ent0 + (r < t.rows ? r : 0));
            const uint32_t ig = ent / (uint32_t)npast;
            const int g = (int)(ig % (uint32_t)p.G);
            const int i = (int)(ig / (uint32_t)p.G);
            rr[e] = ((t.b * p.hq + t.hk * p.G + g) * p.N) + i;
            // The next unit's rows go into L2 while the current unit runs, so that its
            // gather reads L2 instead of DRAM.
            if (pf && r < t.rows)
              prefetch_l2_bulk(p.q + t.b * p.q_sb + (int64_t)(t.hk * p.G + g) * p.q_sh + (int64_t)i * p.q_sn, D * 2);
          }
        };
        int u = u_begin + (int)blockIdx.x;
        int rr[4];
        Unit w;
        Tile tx;
        tx.rows = 0;
        if (u < u_end) {
          gathered_unit(p, __ldg(p.tiles + u), w);
          tx = x ? w.t[1] : w.t[0];
          if (tx.rows > 0) rows_of(tx, rr, false);
        }
        for (; ok && u < u_end; u += gridDim.x) {
          if (tx.rows > 0) {
            if (!(ok = mbar_wait(&bar.q_empty[x], (quse & 1) ^ 1, abort, p.status, site0 + 11))) break;
            ++quse;
            if (lane == 0) mbar_arrive_expect_tx(&bar.q_full[x], C::BYTES);
            __syncwarp();
            tma_gather4_2d(qt + lane * 512, &tmQ, &bar.q_full[x], 0, rr[0], rr[1], rr[2], rr[3]);
            if (D == 128)
              tma_gather4_2d(qt + C::R0 + lane * 512, &tmQ, &bar.q_full[x], 64, rr[0], rr[1], rr[2], rr[3]);
            if (D == 80)
              tma_gather4_2d(qt + C::R0 + lane * 128, &tmQ1, &bar.q_full[x], 64, rr[0], rr[1], rr[2], rr[3]);
          }
          const int un = u + (int)gridDim.x;
          tx.rows = 0;
          if (un < u_end) {
            gathered_unit(p, __ldg(p.tiles + un), w);
            tx = x ? w.t[1] : w.t[0];
            if (tx.rows > 0) rows_of(tx, rr, true);
          }
        }
        // After an abort, let the last gather land before the CTA can retire.
        if (*abort && quse > 0) {
          const unsigned long long t0 = global_timer_ns();
          while (!mbar_try_wait(&bar.q_full[x], (quse - 1) & 1) && global_timer_ns() - t0 < wait_limit_ns(p.status)) {}
        }
      } else {
        // cp.async: lane l owns rows l, l + 32, l + 64, l + 96; it reads their list
        // entries first, then issues all of their 16-byte copies.
        const int l = lane;
        constexpr int VPR = D / 8;  // 16-byte vectors per row
        for (UnitIter<MODE> it(p, u_begin, u_end); ok && it.valid(); it.next()) {
          Unit w;
          it.get(p, w);
          const Tile t = x ? w.t[1] : w.t[0];
          if (t.rows == 0) continue;
          uint32_t ent[4];
#pragma unroll
          for (int k2 = 0; k2 < 4; ++k2)
            ent[k2] = (l + 32 * k2 < t.rows) ? __ldg(p.entries + t.ent0 + l + 32 * k2) : 0u;
          if (!(ok = mbar_wait(&bar.q_empty[x], (quse & 1) ^ 1, abort, p.status, site0 + 11))) break;
          ++quse;
#pragma unroll
          for (int k2 = 0; k2 < 4; ++k2) {
            const int r = l + 32 * k2;
            const bool valid = r < t.rows;
            const uint16_t *row = p.q;
            if (valid) {
              const uint32_t ig = ent[k2] / (uint32_t)npast;
              const int g = (int)(ig % (uint32_t)p.G);
              const int i = (int)(ig / (uint32_t)p.G);
              row = p.q + t.b * p.q_sb + (int64_t)(t.hk * p.G + g) * p.q_sh + (int64_t)i * p.q_sn;
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
          mbar_arrive(&bar.q_full[x]);
        }
      }
    }
  } else {
    // ------------------------------------------------- softmax + epilogue
    // tcgen05.ld / st are warp-collective (.sync.aligned): every wait is made
    // warp-uniform with __all_sync, and no TMEM access sits under a per-row branch.
    setmaxnreg_inc<kRegsSoftmax>();
    const int x = (warp - 4) >> 2;          // stream
    const int r = (tid - 128) & 127;        // row within the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tS = tmem + lane_off + 128 * x;
    const uint32_t tO = tmem + lane_off + 256 + 128 * x;
    const float sl2 = p.scale_log2;
    uint32_t scnt = 0, ocnt = 0;
    // Ping-pong of the exponential phases (sliding-window launches): the softmax warps
    // of streams A and B that share a sub-partition (warps w and w + 4) take turns, so
    // that one stream's exponentials run while the tensor core works on the other
    // stream's MMAs instead of both streams contending for the same exponential units
    // at once.  Stream x waits on turn[x][q] before its exponentials and passes
    // turn[x ^ 1][q] after them; stream B hands stream A the first turn.  Both streams
    // take one turn per chunk of every unit (an idle stream passes its turns on at
    // once), so the turns stay paired.  MoBA launches run without turns: there the two
    // warps' exponentials overlapping keep the exponential unit at its full rate (a lone
    // warp issues its instructions at about 10 cycles each, two warps at 8), which ran
    // the gathered pass 12% faster at 1M tokens; the band pass at d = 80 is 1% faster
    // with the turns.
    const bool turns = !p.is_moba;
    const int q4 = warp & 3;
    uint64_t *my_turn = &bar.turn[x][q4];
    uint64_t *other_turn = &bar.turn[x ^ 1][q4];
    uint32_t tcnt = 0;
    if (turns && x == 1 && lane == 0) mbar_arrive(other_turn);
    bool ok = true;
    for (UnitIter<MODE> it(p, u_begin, u_end); ok && it.valid(); it.next()) {
      Unit w;
      it.get(p, w);
      const Tile t = x ? w.t[1] : w.t[0];   // (a select: w stays in registers)
      if (t.rows == 0) {
        for (int m = 0; turns && m < w.nc && ok; ++m, ++tcnt) {
          ok = mbar_wait(my_turn, tcnt & 1, abort, p.status, site0 + 15);
          ok = __all_sync(FULL, ok);
          __syncwarp();
          if (ok && lane == 0) mbar_arrive(other_turn);
        }
        continue;
      }
      const bool live = r < t.rows;
      // Row identity.
      int i = t.i0 + r, h = t.h, slot = 0;
      if (MODE == kGathered && live) {
        const uint32_t ent = __ldg(p.entries + t.ent0 + r);
        slot = (int)(ent % (uint32_t)p.npast);
        const uint32_t ig = ent / (uint32_t)p.npast;
        h = t.hk * p.G + (int)(ig % (uint32_t)p.G);
        i = (int)(ig / (uint32_t)p.G);
      }
      const int32_t *irow = (MODE == kQueryMajor && p.is_moba && live)
                                ? p.idx + (((int64_t)t.b * p.hq + h) * p.N + i) * p.topk
                                : nullptr;
      const int pos = p.q_off + i;        // the row's key position (masks)
      const int a0 = p.q_off + t.i0;      // query-major: the tile's first key position
      // Query-major MoBA: the first key of the row's own block (a tile's rows may span
      // two blocks when its first row does not start at a multiple of 128).
      const int cBr = (MODE == kQueryMajor && p.is_moba) ? (pos / p.block) * p.block : 0;
      float m_run = -INFINITY, l_run = 0.f;
      for (int m = 0; m < w.nc; ++m, ++scnt) {
        ok = mbar_wait(&bar.s_full[x], scnt & 1, abort, p.status, site0 + 12);
        if (!(ok = __all_sync(FULL, ok))) break;
        tc_fence_after();
        uint32_t sv[128];
        float *s = reinterpret_cast<float *>(sv);
        const int key0 = w.key0 + m * kTileKeys;
        float lsum;
        if constexpr (MODE == kGathered) {
          // S of the chunk into registers (the gathered pass has no masks).
          auto load_s = [&]() {
            tmem_ld64(tS, *reinterpret_cast<uint32_t(*)[64]>(&sv[0]));
            tmem_ld64(tS + 64, *reinterpret_cast<uint32_t(*)[64]>(&sv[64]));
            tmem_wait_ld();
          };
          // The chunk's exact row maximum raises the running maximum when it grows by
          // more than thr (always from -inf); l and O are rescaled by the same factor.
          // S(m) complete implies P V of chunk m-1 complete: O is final for now.
          auto raise_max = [&](float thr) {
            float mx8[8];
  #pragma unroll
            for (int u2 = 0; u2 < 8; ++u2) mx8[u2] = s[u2];
  #pragma unroll
            for (int e = 8; e < 128; ++e) mx8[e & 7] = fmaxf(mx8[e & 7], s[e]);
            const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                   fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
            const float m_new = fmaxf(m_run, mx * sl2);
            const bool raise = (m_run == -INFINITY) || (m_new > m_run + thr);
            const bool scale_o = raise && m_run != -INFINITY;
            const float alpha = scale_o ? ex2_approx(m_run - m_new) : 1.f;
            if (raise) {
              l_run *= alpha;
              m_run = m_new;
            }
            if (__any_sync(FULL, scale_o)) {
  #pragma unroll
              for (int c0 = 0; c0 < D; c0 += 16) {
                uint32_t o[16];
                tmem_ld16(tO + c0, o);
                tmem_wait_ld();
  #pragma unroll
                for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                tmem_st16(tO + c0, o);
              }
            }
          };
          // P = 2^(s * scale * log2 e - mu) packed to bf16 over the first 64 words of sv;
          // returns the chunk's row sum.  Scale and sums in packed pairs (eight running
          // sums: four pairs).
          auto exps = [&]() -> float {
            const float mu = (m_run == -INFINITY) ? 0.f : m_run;
            float ls[8];
  #pragma unroll
            for (int u2 = 0; u2 < 8; ++u2) ls[u2] = 0.f;
  #pragma unroll
            for (int e = 0; e < 64; ++e) {
              float x0, x1;
              fma_f32x2(x0, x1, s[2 * e], s[2 * e + 1], sl2, -mu);
              const float p0 = ((2 * e) % 16 >= 16 - kExpEmuPer16) ? exp2_fma(x0) : ex2_in_order(x0);
              const float p1 = ((2 * e + 1) % 16 >= 16 - kExpEmuPer16) ? exp2_fma(x1) : ex2_in_order(x1);
              add_f32x2(ls[2 * (e & 3)], ls[2 * (e & 3) + 1], p0, p1);
              sv[e] = pack_bf16x2(p0, p1);
            }
            return ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
          };
          load_s();
          // The exact maximum is taken while some row of the warp has none yet; after
          // that a chunk reuses the running maximum.  Its probabilities are then bounded
          // by their sum, and the chunk is redone with its exact maximum only when that
          // sum leaves the range that keeps P, l and O finite in fp32 and bf16 (S is
          // still in TMEM: P is not stored yet).  This takes the row maximum off the
          // chunk's critical path (measured 4-5% on the 1M-token pass).
          if (__any_sync(FULL, m_run == -INFINITY)) raise_max((float)kRescaleThreshold);
          if (turns) {
            ok = mbar_wait(my_turn, tcnt & 1, abort, p.status, site0 + 15);
            ++tcnt;
            if (!(ok = __all_sync(FULL, ok))) break;
          }
          lsum = exps();
          if (__any_sync(FULL, !(lsum <= kSumBound))) {
            load_s();
            raise_max(0.f);
            lsum = exps();
          }
        } else {
          // Query-major passes (own block, sliding window): the exact maximum of every
          // chunk, raised lazily.
          tmem_ld64(tS, *reinterpret_cast<uint32_t(*)[64]>(&sv[0]));
          tmem_ld64(tS + 64, *reinterpret_cast<uint32_t(*)[64]>(&sv[64]));
          tmem_wait_ld();
          // Masks.
          if (MODE == kQueryMajor) {
            if (p.is_moba) {
              if (key0 < cBr) {
                // Window tail into an earlier block: keys i - j < window that the row's
                // own selection does not already cover.  (block is a multiple of 128, so
                // the chunk's keys all lie in one block.)
                bool covered = false;
                if (irow) {
                  const int blk = key0 / p.block;
                  for (int u2 = 0; u2 < p.topk; ++u2) covered |= (__ldg(irow + u2) == blk);
                }
                const bool none = covered || !live || p.window <= 0;
  #pragma unroll
                for (int e = 0; e < 128; ++e)
                  if (none || pos - (key0 + e) >= p.window) s[e] = -INFINITY;
              } else if (key0 + kTileKeys - 1 > pos) {
  #pragma unroll
                for (int e = 0; e < 128; ++e)
                  if (key0 + e > pos) s[e] = -INFINITY;
              }
            } else {
              const bool full = (key0 + kTileKeys - 1 <= a0) &&
                                (key0 >= a0 + t.rows - 1 - p.window + 1);
              if (!full) {
  #pragma unroll
                for (int e = 0; e < 128; ++e) {
                  const int j = key0 + e;
                  if (j > pos || pos - j >= p.window) s[e] = -INFINITY;
                }
              }
            }
          }
          float mx8[8];
  #pragma unroll
          for (int u2 = 0; u2 < 8; ++u2) mx8[u2] = s[u2];
  #pragma unroll
          for (int e = 8; e < 128; ++e) mx8[e & 7] = fmaxf(mx8[e & 7], s[e]);
          const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                 fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
          const float m_new = fmaxf(m_run, mx * sl2);
          // Raise the running maximum only when it grows by more than 2^8 (or from
          // -inf); rows that keep theirs multiply O by 1 when the warp rescales.
          const bool raise = (m == 0) || (m_new > m_run + (float)kRescaleThreshold);
          const bool scale_o = raise && m > 0 && m_run != -INFINITY;
          const float alpha = scale_o ? ex2_approx(m_run - m_new) : 1.f;
          if (raise) {
            l_run *= alpha;
            m_run = m_new;
          }
          if (__any_sync(FULL, scale_o)) {
            // S(m) complete implies P V of chunk m-1 complete: O is final for now.
  #pragma unroll
            for (int c0 = 0; c0 < D; c0 += 16) {
              uint32_t o[16];
              tmem_ld16(tO + c0, o);
              tmem_wait_ld();
  #pragma unroll
              for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st16(tO + c0, o);
            }
          }
          if (turns) {
            ok = mbar_wait(my_turn, tcnt & 1, abort, p.status, site0 + 15);
            ++tcnt;
            if (!(ok = __all_sync(FULL, ok))) break;
          }
          const float mu = (m_run == -INFINITY) ? 0.f : m_run;
          // Scale and row sums in packed pairs (eight running sums: four pairs).
          float ls[8];
  #pragma unroll
          for (int u2 = 0; u2 < 8; ++u2) ls[u2] = 0.f;
  #pragma unroll
          for (int e = 0; e < 64; ++e) {
            float x0, x1;
            fma_f32x2(x0, x1, s[2 * e], s[2 * e + 1], sl2, -mu);
            const float p0 = ((2 * e) % 16 >= 16 - kExpEmuPer16) ? exp2_fma(x0) : ex2_in_order(x0);
            const float p1 = ((2 * e + 1) % 16 >= 16 - kExpEmuPer16) ? exp2_fma(x1) : ex2_in_order(x1);
            add_f32x2(ls[2 * (e & 3)], ls[2 * (e & 3) + 1], p0, p1);
            sv[e] = pack_bf16x2(p0, p1);
          }
          lsum = ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
        }
        __syncwarp();
        if (turns && lane == 0) mbar_arrive(other_turn);
        tmem_st32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_st32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        l_run += lsum;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar.p_full[x]);
      }
      if (!ok) break;
      // ------------------------------------------------------------ epilogue
      ok = mbar_wait(&bar.o_full[x], ocnt & 1, abort, p.status, site0 + 14);
      if (!(ok = __all_sync(FULL, ok))) break;
      ++ocnt;
      tc_fence_after();
      const float inv_l = (l_run > 0.f) ? 1.f / l_run : 0.f;
      const float own_lse = (m_run + log2f(l_run)) * 0.69314718055994530942f;  // natural log
      // Destination: a partial slot (gathered: the row's past-block slot; MoBA
      // query-major: the own-block slot topk-1, merged afterwards), or the output
      // itself when nothing needs merging (SWA, or topk = 1).
      uint16_t *dst;
      float *ldst;
      if (MODE == kGathered || (p.is_moba && p.npast > 0)) {
        const int sl = (MODE == kGathered) ? slot : p.npast;
        const int64_t pidx = (((int64_t)t.b * p.hq + h) * p.chunk_rows + (i - p.chunk * p.chunk_rows)) * p.topk + sl;
        dst = p.opart + pidx * D;
        ldst = p.lpart + pidx;
      } else {
        dst = p.out + t.b * p.o_sb + (int64_t)h * p.o_sh + (int64_t)i * p.o_sn;
        ldst = p.lse + ((int64_t)t.b * p.hq + h) * p.N + i;
      }
      // Stores go through a per-warp staging buffer (32 rows x 64 bytes, chunk index
      // XOR-swizzled by row pair): lane r writes its row's piece, then each lane stores
      // 16 bytes of eight whole 64-byte row segments per instruction (coalesced).
      unsigned char *stg = sbase + C::EPI_OFF + (warp - 4) * 2048;
      const int wl = r & 31;                  // this lane's row within the warp
      uint16_t *rdst[4];
      bool rlive[4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int src = jj * 8 + (lane >> 2);
        rdst[jj] = reinterpret_cast<uint16_t *>(__shfl_sync(FULL, reinterpret_cast<uintptr_t>(dst), src));
        rlive[jj] = __shfl_sync(FULL, live ? 1 : 0, src) != 0;
      }
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        const int cols = (D - c0) < 32 ? (D - c0) : 32;  // D = 80 ends with 16
        uint32_t o[32];
        __syncwarp();
        if (cols == 32) tmem_ld32(tO + c0, o);
        else tmem_ld16(tO + c0, *reinterpret_cast<uint32_t(*)[16]>(&o[0]));
        tmem_wait_ld();
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          if (v4 * 8 >= cols) break;
          uint4 q4;
          q4.x = pack_bf16x2(__uint_as_float(o[8 * v4 + 0]) * inv_l, __uint_as_float(o[8 * v4 + 1]) * inv_l);
          q4.y = pack_bf16x2(__uint_as_float(o[8 * v4 + 2]) * inv_l, __uint_as_float(o[8 * v4 + 3]) * inv_l);
          q4.z = pack_bf16x2(__uint_as_float(o[8 * v4 + 4]) * inv_l, __uint_as_float(o[8 * v4 + 5]) * inv_l);
          q4.w = pack_bf16x2(__uint_as_float(o[8 * v4 + 6]) * inv_l, __uint_as_float(o[8 * v4 + 7]) * inv_l);
          *reinterpret_cast<uint4 *>(stg + wl * 64 + ((v4 ^ ((wl >> 1) & 3)) << 4)) = q4;
        }
        __syncwarp();
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int row = jj * 8 + (lane >> 2), ch = lane & 3;
          if (ch * 8 < cols && rlive[jj]) {
            const uint4 q4 = *reinterpret_cast<const uint4 *>(stg + row * 64 + ((ch ^ ((row >> 1) & 3)) << 4));
            *reinterpret_cast<uint4 *>(rdst[jj] + c0 + ch * 8) = q4;
          }
        }
      }
      if (live) *ldst = own_lse;
      // The O reads are done before this stream's next P lets a P V overwrite O.
      __syncwarp();
      tc_fence_before();
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
  // build that launched with fewer than the split needs would leave an increase
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

// Query-major work units for rows [row_begin, row_end) (see query_major_unit).
int query_major_units(int batch, int hq, int hkv, int block, int is_moba, int row_begin,
                      int row_end) {
  const int nq = (row_end - row_begin + kTileRows - 1) / kTileRows;
  const int G = hq / hkv;
  if (G >= 2) return nq * batch * hkv * ((G + 1) / 2);
  const int tpb = is_moba ? block / kTileRows : nq;
  const int ngroups = (nq + tpb - 1) / tpb;
  return ngroups * ((tpb + 1) / 2) * batch * hkv;
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
