// gate.cu -- MoBA gate scores and top-k on the sm_100a tensor cores (tcgen05 + TMA).
//
// [MoBA] = "MoBA: 어텐션에 전문가 혼합을 적용해 긴 문맥을 효율적으로 처리하는 블록 어텐션
//          (feat. MoonshotAI)", PyTorch KR forum summary of the MoBA paper.
//
// §"블록 분할과 top-k 게이팅": the gate score of query i for block j is the unscaled
// inner product s_j = <q_i, MeanPool(K[I_j])>; each query keeps the k blocks with the
// highest scores.  §"인과성 보존": only blocks wholly before the query's own block
// c = (q_off + i) / block compete (j < c), block c is always kept, later blocks never.
//
// It takes problems of at most 256 blocks with k - 1 <= 31; the general gate of
// select.cu takes the others (and the min/max pooled variant).
// One persistent CTA per SM takes chunks of consecutive 128-row query tiles, ordered
// (batch, kv-head, row tile, q-head), from a global counter (the cost of a tile grows
// with its row position, so a static split would leave SMs idle); the pooled keys of a
// kv-head stay staged in shared memory while the CTA's tiles stay in that kv-head.
// A tile's 128 rows span at most two blocks (block >= 128): rows before the boundary
// have own block c, the others c + 1, and the tile needs the scores of blocks [0, c_hi)
// for its last row's own block c_hi.  The last tile of a head may hold fewer than 128
// rows (its missing rows load as zeros and are never written).
//   warp 0     TMA producer: query tiles (a ring of up to eight) and, per kv-head, the
//              pooled keys kbar = hi + lo (two bf16 matrices of up to 256 rows; two
//              slots when they fit, so the next kv-head's keys load early); it also
//              takes the tile chunks from the counter and hands them on
//   warp 1     tcgen05 MMA issuer and TMEM owner: S = Q hi^T + Q lo^T in fp32, into
//              one of 2-4 TMEM accumulators (N = c rounded up to 16 columns)
//   warps 2-9  top-k, two groups of four warps taking the tiles (and accumulators) in
//              turn: thread r owns row r (TMEM lane r) and ranks its c scores --
//              k - 1 <= 4: a float register list without branches (a strictly greater
//              score displaces; ties keep the lower block); longer lists: 32-bit packed
//              keys merged by sorting networks (lists of 8, 16) or inserted (24, 32),
//              with an exact 64-bit rescan of rows whose boundary keys tie in their
//              score bits -- then stages the row's choices in ascending order, the own
//              block and -1 padding (stored coalesced per warp), and counts the picks
//              per past block for the dispatch lists.
// The last CTA to finish turns the list counts into list offsets.
// q is exactly bf16 and kbar = hi + lo to about 2^-17 relative, so the fp32 scores
// match an fp32 inner product with the pooled keys far inside the ranking tolerance.
#include <cuda.h>
#include <stdint.h>

#include <algorithm>

#include "common.cuh"
#include "lists.cuh"
#include "params.h"

namespace moba {

constexpr int kGateTcThreads = 320;
constexpr int kGateMaxBlocks = 256;   // pooled keys staged at once (MMA N <= 256)
constexpr int kGateMaxPicks = 4;      // past blocks per row kept in the float list
constexpr int kGateMaxList = 32;      // packed-key list length limit: k - 1 <= 31

constexpr int kGateMaxStages = 8;     // query tile ring depth limit
constexpr int kGateSmemLimit = 227 * 1024;

// Shared memory: a ring of qst query tiles, the pooled keys hi and lo (kc16 rows each),
// eight per-warp pick histograms, eight per-warp output staging areas (32 rows of str
// words, str = topk | 1 so that the rows start in distinct banks), barriers.  qst is
// chosen on the host to fill the shared memory the staged pooled keys leave.
template <int D>
struct GateCfg {
  static constexpr int QR0 = 128 * 128;                                // query region 0 bytes
  static constexpr int QR1 = (D == 128) ? 128 * 128 : (D == 80 ? 128 * 32 : 0);
  static constexpr int QTILE = QR0 + ((QR1 + 1023) / 1024) * 1024;
  static constexpr uint32_t QBYTES = 128u * D * 2u;
  static constexpr int R1ROW = (D == 128) ? 128 : (D == 80 ? 32 : 0);  // region 1 bytes per row
  __host__ __device__ static constexpr int kmat(int kc16) {           // one of hi / lo
    return kc16 * 128 + ((kc16 * R1ROW + 1023) / 1024) * 1024;
  }
  __host__ __device__ static constexpr int k_off(int qst) { return qst * QTILE; }
  // ks staging slots for the pooled keys, each holding hi and lo.
  __host__ __device__ static constexpr int hist_off(int qst, int kc16, int ks) {
    return k_off(qst) + ks * 2 * kmat(kc16);
  }
  __host__ __device__ static constexpr int stg_off(int qst, int kc16, int ks) {
    return hist_off(qst, kc16, ks) + 8 * 4 * kGateMaxBlocks;
  }
  __host__ __device__ static constexpr int bar_off(int qst, int kc16, int ks, int str) {
    return stg_off(qst, kc16, ks) + ((8 * 32 * str * 4 + 15) & ~15);
  }
  __host__ __device__ static constexpr int smem(int qst, int kc16, int ks, int str) {
    return bar_off(qst, kc16, ks, str) + 512 + 1024;
  }
};

constexpr int kGateSchedRing = 4;     // tile chunks handed from the producer to the others
constexpr int kGateMaxAcc = 4;        // TMEM accumulators (score tiles in flight)

struct GateBars {
  uint64_t q_full[kGateMaxStages], q_empty[kGateMaxStages];
  uint64_t k_full[2], k_empty[2];
  uint64_t acc_full[kGateMaxAcc], acc_empty[kGateMaxAcc];
  uint64_t sched_full[kGateSchedRing], sched_empty[kGateSchedRing];
  uint64_t mma_done;
  int sched[kGateSchedRing];   // first tile of each handed-out chunk, -1 at the end
  uint32_t tmem_base;
  int abort;
};

// K-major operand descriptor for k-step ks of a tile whose region 0 holds columns
// [0, 64) of `rows` rows (128-byte rows, 128-byte swizzle) and whose region 1 holds
// the remaining columns (D = 128: 64 more, same layout; D = 80: 16, 32-byte rows and
// 32-byte swizzle).
template <int D>
__device__ __forceinline__ uint64_t gate_desc(uint32_t tile, int ks, int rows) {
  if (ks < 4) return smem_desc(tile + ks * 32, 16, 1024, kSwizzle128);
  if (D == 128) return smem_desc(tile + rows * 128 + (ks - 4) * 32, 16, 1024, kSwizzle128);
  return smem_desc(tile + rows * 128, 16, 256, kSwizzle32);
}

// Tile t of the range -> (b, hk, row tile, g): rows [128 rt, 128 rt + 128) of q-head
// hk * G + g.  Ordered so that consecutive tiles share the kv-head.
struct GateTile {
  int b, hk, g, rt;
  int c;        // own block of the tile's first row: (q_off + 128 rt) / block
  int c_hi;     // own block of the tile's last row (c or c + 1)
  int chunk;    // query chunk of the tile's rows: 128 rt / chunk_rows
};
__device__ __forceinline__ void gate_tile_last(const GateParams &p, GateTile &r) {
  const int last = p.q_off + min(r.rt * 128 + 127, p.N - 1);
  r.c_hi = r.c + (last >= (r.c + 1) * p.block ? 1 : 0);
}
__device__ __forceinline__ GateTile gate_tile(const GateParams &p, int t) {
  GateTile r;
  r.g = t % p.G;
  t /= p.G;
  const int nrt = (p.N + 127) / 128;
  r.rt = t % nrt;
  t /= nrt;
  r.hk = t % p.hkv;
  r.b = t / p.hkv;
  r.c = (p.q_off + r.rt * 128) / p.block;
  r.chunk = (r.rt * 128) / p.chunk_rows;
  gate_tile_last(p, r);
  return r;
}

// The next tile in that order, without divisions (one decode per range, then steps;
// the first row moves by 128 <= block positions, so its block grows by at most one).
__device__ __forceinline__ void gate_tile_next(const GateParams &p, GateTile &r) {
  if (++r.g < p.G) return;
  r.g = 0;
  ++r.rt;
  if (p.q_off + r.rt * 128 >= (r.c + 1) * p.block) ++r.c;
  if (r.rt * 128 == (r.chunk + 1) * p.chunk_rows) ++r.chunk;
  if (r.rt < (p.N + 127) / 128) {
    gate_tile_last(p, r);
    return;
  }
  r.rt = 0;
  r.c = p.q_off / p.block;
  r.chunk = 0;
  gate_tile_last(p, r);
  if (++r.hk < p.hkv) return;
  r.hk = 0;
  ++r.b;
}

// Insertion of (v, j) into the descending list val / idx.  Entries past the npick in
// use hold +inf and are never displaced, so the element carried past the last used
// entry falls off; an entry is displaced only by a strictly greater score, so ties
// keep the block that came first, the lower one.
template <int KM>
__device__ __forceinline__ void topk_insert(float (&val)[KM], int (&idx)[KM], float v, int j) {
#pragma unroll
  for (int e = 0; e < KM; ++e) {
    const bool take = v > val[e];
    const float tv = val[e];
    const int tj = idx[e];
    val[e] = take ? v : tv;
    idx[e] = take ? j : tj;
    v = take ? tv : v;
    j = take ? tj : j;
  }
}

// The k-1 best (score, block) pairs of one row over blocks [0, c), from the TMEM
// accumulator row at `acc`, in the float list above.  cw (>= c, the same on every
// lane of the warp) bounds the warp-collective TMEM loads.
template <int KM>
__device__ __forceinline__ void topk_scan(uint32_t acc, int c, int cw, int npick, float (&val)[KM],
                                          int (&idx)[KM]) {
#pragma unroll
  for (int e = 0; e < KM; ++e) {
    val[e] = (e < npick) ? -INFINITY : INFINITY;
    idx[e] = -1;
  }
  for (int j0 = 0; j0 < cw; j0 += 32) {
    uint32_t sc[32];
    tmem_ld32(acc + j0, sc);
    tmem_wait_ld();
    // Every score goes through the short list, with no branch.
#pragma unroll
    for (int e = 0; e < 32; ++e)
      topk_insert<KM>(val, idx, (j0 + e < c) ? __uint_as_float(sc[e]) : -INFINITY, j0 + e);
  }
}

// Insertion of key v into the descending list L of packed keys: two unsigned min / max
// per entry.  Entries past the npick + 1 in use hold all ones and are never displaced.
template <int KM, typename K>
__device__ __forceinline__ void packed_insert(K (&L)[KM], K v) {
#pragma unroll
  for (int e = 0; e < KM; ++e) {
    const K hi = max(L[e], v);
    v = min(L[e], v);
    L[e] = hi;
  }
}

// Sorting networks on packed keys (one unsigned min and max per comparator).
// Batcher's odd-even merge sort of W keys, as a comparator list built at compile time
// (so that every index is a constant once the loop over it is unrolled).
template <int W>
struct SortNet {
  int lo[W * W], hi[W * W];
  int n;
  constexpr SortNet() : lo(), hi(), n(0) {
    for (int p = 1; p < W; p *= 2)
      for (int k = p; k >= 1; k /= 2)
        for (int j = k % p; j + k < W; j += 2 * k)
          for (int i = 0; i < k; ++i)
            if (i + j + k < W && (i + j) / (2 * p) == (i + j + k) / (2 * p)) {
              lo[n] = i + j;
              hi[n] = i + j + k;
              ++n;
            }
  }
};

// B := B in ascending order.
template <int W>
__device__ __forceinline__ void sort_asc(uint32_t (&B)[W]) {
  constexpr SortNet<W> net;
#pragma unroll
  for (int t = 0; t < net.n; ++t) {
    const uint32_t a = B[net.lo[t]], b = B[net.hi[t]];
    B[net.lo[t]] = min(a, b);
    B[net.hi[t]] = max(a, b);
  }
}

// L (W keys, descending) := the W greatest of L and the batch B (W keys, ascending):
// the element-wise maximum of a descending and an ascending sequence is bitonic and
// holds the W greatest; half-cleaners then sort it descending.
template <int W>
__device__ __forceinline__ void merge_top(uint32_t (&L)[W], const uint32_t (&B)[W]) {
#pragma unroll
  for (int e = 0; e < W; ++e) L[e] = max(L[e], B[e]);
#pragma unroll
  for (int k = W / 2; k >= 1; k /= 2) {
#pragma unroll
    for (int i = 0; i < W; ++i) {
      if ((i & k) == 0) {
        const uint32_t a = L[i], b = L[i + k];
        L[i] = max(a, b);
        L[i + k] = min(a, b);
      }
    }
  }
}

// The scores of blocks j0 .. j0 + 15 (raw fp32 bits in s) into the list L, KM at a time:
// packed keys (blocks at or after c: key 0, never kept), a sort, a merge.
template <int KM>
__device__ __forceinline__ void net_batches(uint32_t (&L)[KM], const uint32_t (&s)[16], int j0,
                                            int c, uint32_t imask) {
  const uint32_t jb = imask - (uint32_t)j0;
#pragma unroll
  for (int h = 0; h < 16; h += KM) {
    if (j0 + h < c) {
      uint32_t B[KM];
#pragma unroll
      for (int e = 0; e < KM; ++e) {
        const uint32_t b = s[h + e];
        const uint32_t ord = b ^ ((uint32_t)((int32_t)b >> 31) | 0x80000000u);
        B[e] = (j0 + h + e < c) ? ((ord & ~imask) | (jb - (uint32_t)(h + e))) : 0u;
      }
      sort_asc<KM>(B);
      merge_top<KM>(L, B);
    }
  }
}

template <int D, int KM>
__global__ void __launch_bounds__(kGateTcThreads, 1)
gate_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQ1,
               const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmK1,
               const GateParams p) {
  using C = GateCfg<D>;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char *sbase = smem_raw + (base - raw);
  // Pooled-key rows staged per kv-head: every past block of the last row tile.
  const int kc16 = (min(p.nblk, kGateMaxBlocks) + 15) & ~15;
  const int qst = p.qstages;
  const int kmat = C::kmat(kc16);
  const int k_off = C::k_off(qst);
  const int str = p.topk | 1;
  // TMEM accumulators of accw columns (a power of two >= kc16) share the 512 columns:
  // tile u of the CTA uses accumulator u % nacc (nacc even, so a group's tiles never
  // use the other group's accumulators).
  const int accw = kc16 <= 32 ? 32 : (kc16 <= 64 ? 64 : (kc16 <= 128 ? 128 : 256));
  const int nacc = min(kGateMaxAcc, 512 / accw);
  const int ks = p.kslots;
  GateBars &bar = *reinterpret_cast<GateBars *>(sbase + C::bar_off(qst, kc16, ks, str));
  int *hist = reinterpret_cast<int *>(sbase + C::hist_off(qst, kc16, ks));
  int *stg_all = reinterpret_cast<int *>(sbase + C::stg_off(qst, kc16, ks));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int site0 = (3 * 16 + (D == 64 ? 0 : (D == 80 ? 1 : 2))) * 256;
  constexpr uint32_t FULL = 0xffffffffu;

  // Tiles are handed out in chunks of p.chunk_tiles consecutive tiles from a global
  // counter: the producer takes a chunk and passes its first tile through the sched
  // ring to the MMA issuer and the top-k warps, which walk the same tiles in order.
  const int ntiles = p.batch * p.hkv * ((p.N + 127) / 128) * p.G;

  if (tid == 0) {
    for (int s = 0; s < qst; ++s) {
      mbar_init(&bar.q_full[s], 1);
      mbar_init(&bar.q_empty[s], 1);
    }
    for (int s = 0; s < kGateMaxAcc; ++s) {
      mbar_init(&bar.acc_full[s], 1);
      mbar_init(&bar.acc_empty[s], 4);
    }
    for (int s = 0; s < kGateSchedRing; ++s) {
      mbar_init(&bar.sched_full[s], 1);
      mbar_init(&bar.sched_empty[s], 9);   // the MMA issuer and the eight top-k warps
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.k_full[s], 1);
      mbar_init(&bar.k_empty[s], 1);
    }
    mbar_init(&bar.mma_done, 1);
    bar.abort = 0;
    fence_barrier_init();
  }
  for (int j = tid; j < 8 * kGateMaxBlocks; j += kGateTcThreads) hist[j] = 0;
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
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
  // The first tile of chunk kq of this CTA (-1: no more tiles), or -1 with ok = false
  // when the wait gave up.
  auto take_chunk = [&](uint32_t kq, int site, bool &ok) -> int {
    const int slot = kq % kGateSchedRing;
    ok = mbar_wait(&bar.sched_full[slot], (kq / kGateSchedRing) & 1, abort, p.status, site);
    return ok ? *reinterpret_cast<volatile int *>(&bar.sched[slot]) : -1;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      bool ok = true;
      int cur = -1;
      uint32_t kuse = 0, quse = 0;
      // The counter is read one chunk ahead, so its latency overlaps a chunk's loads.
      int next = atomicAdd(p.sched, p.chunk_tiles);
      for (uint32_t kq = 0; ok; ++kq) {
        // Hand on the chunk taken last time, take the following one.
        int start = next;
        if (start >= ntiles) start = -1;
        else next = atomicAdd(p.sched, p.chunk_tiles);
        const int slot = kq % kGateSchedRing;
        if (!(ok = mbar_wait(&bar.sched_empty[slot], ((kq / kGateSchedRing) & 1) ^ 1, abort, p.status,
                             site0 + 7))) break;
        *reinterpret_cast<volatile int *>(&bar.sched[slot]) = start;
        mbar_arrive(&bar.sched_full[slot]);
        if (start < 0) break;
        const int end = min(start + p.chunk_tiles, ntiles);
        GateTile gt = gate_tile(p, start);
      for (int t = start; ok && t < end; ++t, gate_tile_next(p, gt)) {
        const int grp = gt.b * p.hkv + gt.hk;
        if (grp != cur) {
          cur = grp;
          // Slot kuse % ks; with two slots the next kv-head's keys load while the
          // MMAs of the current one still run.
          const int ksl = kuse % ks;
          if (!(ok = mbar_wait(&bar.k_empty[ksl], ((kuse / ks) & 1) ^ 1, abort, p.status, site0 + 1)))
            break;
          ++kuse;
          const uint32_t kbytes = 2u * (uint32_t)kc16 * (uint32_t)D * 2u;
          mbar_arrive_expect_tx(&bar.k_full[ksl], kbytes);
          for (int part = 0; part < 2; ++part) {
            unsigned char *kd = sbase + k_off + (ksl * 2 + part) * kmat;
            const int plane = grp * 2 + part;
            tma_load_3d(kd, &tmK, &bar.k_full[ksl], 0, 0, plane);
            if (D != 64) tma_load_3d(kd + kc16 * 128, &tmK1, &bar.k_full[ksl], 64, 0, plane);
          }
        }
        const int s = quse % qst;
        if (!(ok = mbar_wait(&bar.q_empty[s], ((quse / qst) & 1) ^ 1, abort, p.status, site0 + 2))) break;
        unsigned char *qd = sbase + s * C::QTILE;
        const int h = gt.hk * p.G + gt.g;
        mbar_arrive_expect_tx(&bar.q_full[s], C::QBYTES);
        tma_load_4d(qd, &tmQ, &bar.q_full[s], 0, gt.rt * 128, h, gt.b);
        if (D != 64) tma_load_4d(qd + C::QR0, &tmQ1, &bar.q_full[s], 64, gt.rt * 128, h, gt.b);
        ++quse;
      }
      }
      if (*abort) {
        // Let issued loads land before the CTA can retire.
        const unsigned long long t0 = global_timer_ns();
        for (uint32_t u = (quse > (uint32_t)qst ? quse - qst : 0u); u < quse; ++u)
          while (!mbar_try_wait(&bar.q_full[u % qst], (u / qst) & 1) && global_timer_ns() - t0 < wait_limit_ns(p.status)) {}
        for (uint32_t u = (kuse > (uint32_t)ks ? kuse - ks : 0u); u < kuse; ++u)
          while (!mbar_try_wait(&bar.k_full[u % ks], (u / ks) & 1) && global_timer_ns() - t0 < wait_limit_ns(p.status)) {}
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      int cur = -1;
      uint32_t kuse = 0, quse = 0, ause = 0;
      uint32_t kslot = base + k_off;                        // staged keys in use
      for (uint32_t kq = 0; ok; ++kq) {
        const int start = take_chunk(kq, site0 + 8, ok);
        if (ok) mbar_arrive(&bar.sched_empty[kq % kGateSchedRing]);
        if (!ok || start < 0) break;
        const int end = min(start + p.chunk_tiles, ntiles);
        GateTile gt = gate_tile(p, start);
      for (int t = start; ok && t < end; ++t, gate_tile_next(p, gt)) {
        const int grp = gt.b * p.hkv + gt.hk;
        if (grp != cur) {
          // The slot in use may be refilled once the MMAs issued so far are done.
          if (cur >= 0) umma_commit(&bar.k_empty[(kuse - 1) % ks]);
          cur = grp;
          const int ksl = kuse % ks;
          if (!(ok = mbar_wait(&bar.k_full[ksl], (kuse / ks) & 1, abort, p.status, site0 + 3))) break;
          ++kuse;
          kslot = base + k_off + ksl * 2 * kmat;
        }
        const int s = quse % qst, a = ause % nacc;
        if (!(ok = mbar_wait(&bar.q_full[s], (quse / qst) & 1, abort, p.status, site0 + 4))) break;
        if (!(ok = mbar_wait(&bar.acc_empty[a], ((ause / nacc) & 1) ^ 1, abort, p.status, site0 + 5)))
          break;
        tc_fence_after();
        const int c = gt.c_hi;                              // own block of the last row
        // Score columns needed (none when every row keeps all its past blocks).
        const int nn = (c > p.topk - 1) ? min((c + 15) & ~15, kc16) : 0;
        if (nn > 0) {
          const uint32_t idesc = idesc_bf16(128, nn, 0, 0);
          const uint32_t qt = base + s * C::QTILE;
          const uint32_t acc = tmem + accw * a;
#pragma unroll
          for (int part = 0; part < 2; ++part) {
            const uint32_t kt = kslot + part * kmat;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)
              umma_ss(acc, gate_desc<D>(qt, ks, 128), gate_desc<D>(kt, ks, kc16), idesc,
                      (part > 0 || ks > 0) ? 1u : 0u);
          }
        }
        umma_commit(&bar.acc_full[a]);
        umma_commit(&bar.q_empty[s]);
        ++quse;
        ++ause;
      }
      }
      umma_commit(&bar.mma_done);
      const unsigned long long t0 = global_timer_ns();
      while (!mbar_try_wait(&bar.mma_done, 0) && global_timer_ns() - t0 < wait_limit_ns(p.status)) {}
    }
  } else {
    // ------------------------------------------------------------ top-k
    // Each warp counts its rows' picks in its own shared histogram and adds it to the
    // list counts when its rows move to another (chunk, batch, kv-head) list, so no
    // barrier across warps is needed.
    // Two groups of four warps take the tiles in turn: group gi (warps 2-5 or 6-9)
    // handles the CTA's tiles u = gi, gi + 2, ... (accumulator u % nacc).
    const int gi = (warp - 2) >> 2;
    const int r = 32 * (warp & 3) + lane;                  // row within the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    int *whist = hist + (warp - 2) * kGateMaxBlocks;
    // The warp's 32 output rows are staged here, then written as one contiguous run of
    // 32 * topk words with coalesced stores.
    int *stg = stg_all + (warp - 2) * 32 * str;
    int *orow = stg + lane * str;
    const int r0 = lane / p.topk, s0 = lane - r0 * p.topk;
    const int dq = 32 / p.topk, dr = 32 - dq * p.topk;
    const int npast = p.topk - 1;
    // Low key bits that carry the block index of a packed key.
    const uint32_t imask = (1u << (32 - __clz(max(p.nblk - 1, 1)))) - 1u;
    bool ok = true;
    int cur_list = -1;
    auto flush = [&](int list) {
      __syncwarp();
      for (int j = lane; j < p.nblk; j += 32) {
        const int v = whist[j];
        if (v) {
          atomicAdd(&p.counts[(int64_t)list * p.nblk + j], v);
          whist[j] = 0;
        }
      }
      __syncwarp();
    };
    uint32_t u = 0;                                        // tile number within this CTA
    for (uint32_t kq = 0; ok; ++kq) {
      const int start = take_chunk(kq, site0 + 9, ok);
      ok = __all_sync(FULL, ok);
      if (ok && lane == 0) mbar_arrive(&bar.sched_empty[kq % kGateSchedRing]);
      if (!ok || start < 0) break;
      const int end = min(start + p.chunk_tiles, ntiles);
      GateTile gt = gate_tile(p, start);
    for (int t = start; ok && t < end; ++t, ++u, gate_tile_next(p, gt)) {
      if ((int)(u & 1) != gi) continue;                    // the other group's tile
      const int i = gt.rt * 128 + r;
      const bool valid = i < p.N;                         // the last tile may be partial
      // The row's own block: the tile's first row's, or the next one past a boundary.
      const int c = gt.c + ((p.q_off + i >= (gt.c + 1) * p.block) ? 1 : 0);
      const int h = gt.hk * p.G + gt.g;
      const int a = u % nacc;
      const int list = (gt.chunk * p.batch + gt.b) * p.hkv + gt.hk;
      if (list != cur_list) {
        if (cur_list >= 0) flush(cur_list);
        cur_list = list;
      }
      ok = mbar_wait(&bar.acc_full[a], (u / nacc) & 1, abort, p.status, site0 + 6);
      if (!(ok = __all_sync(FULL, ok))) break;
      tc_fence_after();
      const int i0w = i - lane;                            // the warp's first row
      int32_t *gout = p.idx + (((int64_t)gt.b * p.hq + h) * p.N + i0w) * p.topk;
      // Rows that keep every past block (c <= npast) need no scores; the warp scans the
      // accumulator when any of its rows needs one, up to its largest own block.
      const bool scored = valid && npast > 0 && c > npast;
      const int cw = __reduce_max_sync(FULL, scored ? c : 0);
      if (cw == 0) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.acc_empty[a]);
        const int nk = min(c, npast);
        for (int s = 0; s < p.topk; ++s) orow[s] = (s < nk) ? s : (s == nk ? c : -1);
        if (valid)
          for (int j = 0; j < nk; ++j) atomicAdd(&whist[j], 1);
      } else {
        const int npick = npast;
        const uint32_t acc = tmem + lane_off + accw * a;
        int pk[KM];                                         // the row's picks, any order
        if constexpr (KM <= kGateMaxPicks) {
          float val[KM];
          int idx[KM];
          topk_scan<KM>(acc, c, cw, npick, val, idx);
#pragma unroll
          for (int e = 0; e < KM; ++e) pk[e] = idx[e];
        } else {
          // Packed keys: the order-preserving integer image of the score with its low
          // index bits replaced by (imask - j), so that one unsigned comparison ranks a
          // greater score first and, between equal truncated scores, the lower block.
          uint32_t L[KM];
          if constexpr (KM == 8 || KM == 16) {
            // Batches of KM keys, sorted by a network and merged into the list; scores
            // come in 16-column TMEM loads, the next one in flight during the sort.
#pragma unroll
            for (int e = 0; e < KM; ++e) L[e] = 0u;
            uint32_t s0[16], s1[16];
            tmem_ld16(acc, s0);
            tmem_wait_ld();
            for (int j0 = 0; j0 < cw; j0 += 32) {
              if (j0 + 16 < cw) tmem_ld16(acc + j0 + 16, s1);
              net_batches<KM>(L, s0, j0, c, imask);
              tmem_wait_ld();
              if (j0 + 16 < cw) {
                if (j0 + 32 < cw) tmem_ld16(acc + j0 + 32, s0);
                net_batches<KM>(L, s1, j0 + 16, c, imask);
                tmem_wait_ld();
              }
            }
          } else {
#pragma unroll
            for (int e = 0; e < KM; ++e) L[e] = (e <= npick) ? 0u : 0xFFFFFFFFu;
            for (int j0 = 0; j0 < cw; j0 += 32) {
              uint32_t sc[32];
              tmem_ld32(acc + j0, sc);
              tmem_wait_ld();
              const uint32_t jb = imask - (uint32_t)j0;
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                const uint32_t b = sc[e];
                const uint32_t ord = b ^ ((uint32_t)((int32_t)b >> 31) | 0x80000000u);
                packed_insert<KM>(L, (j0 + e < c) ? ((ord & ~imask) | (jb - (uint32_t)e)) : 0u);
              }
            }
          }
          // L[0..npick] holds the npick + 1 greatest keys in descending order.  When the last
          // kept and the first dropped key differ in their score bits, every kept score
          // exceeds every dropped one and the choice is the exact one; otherwise the
          // row is decided again on the full fp32 scores.
          // (Written as a reduction over adjacent pairs: a select of L[npick] would
          // index L at run time and move it to local memory.)
          bool near_tie = false;
#pragma unroll
          for (int e = 0; e + 1 < KM; ++e)
            near_tie |= (e + 1 == npick) & (((L[e] ^ L[e + 1]) & ~imask) == 0u);
          near_tie &= scored;
#pragma unroll
          for (int e = 0; e < KM; ++e) pk[e] = (int)(imask - (L[e] & imask));
          if (__any_sync(FULL, near_tie)) {
            // The same scan on 64-bit keys: the full 32-bit score image above the block
            // index, i.e. the exact rule (greater score first, then the lower block).
            unsigned long long X[KM];
#pragma unroll
            for (int e = 0; e < KM; ++e) X[e] = (e < npick) ? 0ull : ~0ull;
            for (int j0 = 0; j0 < cw; j0 += 32) {
              uint32_t sc[32];
              tmem_ld32(acc + j0, sc);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                const uint32_t b = sc[e];
                const uint32_t ord = b ^ ((uint32_t)((int32_t)b >> 31) | 0x80000000u);
                const unsigned long long key =
                    ((unsigned long long)ord << 32) | (0xFFFFFFFFu - (uint32_t)(j0 + e));
                packed_insert<KM>(X, (j0 + e < c) ? key : 0ull);
              }
            }
            if (near_tie) {
#pragma unroll
              for (int e = 0; e < KM; ++e) pk[e] = (int)(0xFFFFFFFFu - (uint32_t)X[e]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.acc_empty[a]);
        if (!scored) {
          // A row of a scoring warp that keeps all of its past blocks.
          const int nk = min(c, npast);
          for (int s = 0; s < p.topk; ++s) orow[s] = (s < nk) ? s : (s == nk ? c : -1);
          if (valid)
            for (int j = 0; j < nk; ++j) atomicAdd(&whist[j], 1);
        } else {
          // Ascending block order.
          if (c <= 64) {
            unsigned long long m = 0;
#pragma unroll
            for (int e = 0; e < KM; ++e)
              if (e < npick) m |= 1ull << pk[e];
            for (int s = 0; s < npick; ++s) {
              orow[s] = __ffsll((long long)m) - 1;
              m &= m - 1;
            }
          } else {
#pragma unroll
            for (int e = 0; e < KM; ++e) {
              if (e < npick) {
                int rank = 0;
#pragma unroll
                for (int f = 0; f < KM; ++f)
                  if (f < npick) rank += pk[f] < pk[e];
                orow[rank] = pk[e];
              }
            }
          }
#pragma unroll
          for (int e = 0; e < KM; ++e)
            if (e < npick && pk[e] >= 0) atomicAdd(&whist[pk[e]], 1);  // < 0 only for NaN scores
          orow[npick] = c;
          for (int s = npick + 1; s < p.topk; ++s) orow[s] = -1;
        }
      }
      // Staged rows -> idx: word w = 32 m + lane of the run is entry (r, s) of the warp;
      // only the warp's rows below N are written.
      __syncwarp();
      {
        const int nw = max(0, min(32, p.N - i0w)) * p.topk;
        int rr = r0, ss = s0;
        for (int w = lane; w < nw; w += 32) {
          gout[w] = stg[rr * str + ss];
          rr += dq;
          ss += dr;
          if (ss >= p.topk) { ss -= p.topk; ++rr; }
        }
      }
      __syncwarp();
    }
    }
    if (cur_list >= 0) flush(cur_list);
  }

  __syncwarp();
  tc_fence_before();
  __threadfence();  // this thread's count atomics, before the CTA's ticket below
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
  if (p.done != nullptr) {
    // The last CTA to finish turns the list counts into list offsets.
    int *ticket = hist + 64;  // the histograms are flushed and free
    if (tid == 0) ticket[0] = atomicAdd(p.done, 1);
    __syncthreads();
    if (ticket[0] == (int)gridDim.x - 1) {
      __threadfence();
      scan_lists<kGateTcThreads>(p.counts, p.cursor, p.listoff, p.tileoff, p.nlists, hist);
    }
  }
}

template <int D, int KM>
static cudaError_t launch_gate_tc_dk(const CUtensorMap *maps, GateParams p, int grid,
                                     cudaStream_t st) {
  using C = GateCfg<D>;
  // About eight chunks per CTA.
  const long long ntiles = (long long)p.batch * p.hkv * ((p.N + 127) / 128) * p.G;
  p.chunk_tiles = (int)std::max(1LL, std::min(32LL, ntiles / (8LL * grid)));
  auto kern = gate_tc_kernel<D, KM>;
  const int kc16 = (min(p.nblk, kGateMaxBlocks) + 15) & ~15;
  const int str = p.topk | 1;
  // Two pooled-key slots when they leave room for three query stages; then as many
  // query stages as the shared memory holds.
  const int ks = C::smem(3, kc16, 2, str) <= kGateSmemLimit ? 2 : 1;
  int qst = kGateMaxStages;
  while (qst > 2 && C::smem(qst, kc16, ks, str) > kGateSmemLimit) --qst;
  if (C::smem(qst, kc16, ks, str) > kGateSmemLimit) return cudaErrorInvalidConfiguration;
  p.qstages = qst;
  p.kslots = ks;
  const int bytes = C::smem(qst, kc16, ks, str);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  kern<<<grid, kGateTcThreads, bytes, st>>>(maps[0], maps[1], maps[2], maps[3], p);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_gate_tc_d(const CUtensorMap *maps, const GateParams &p, int grid,
                                    cudaStream_t st) {
  const int npast = p.topk - 1;
  if (npast <= 2) return launch_gate_tc_dk<D, 2>(maps, p, grid, st);
  if (npast <= kGateMaxPicks) return launch_gate_tc_dk<D, kGateMaxPicks>(maps, p, grid, st);
  // Packed lists hold npast + 1 keys.
  if (npast + 1 <= 8) return launch_gate_tc_dk<D, 8>(maps, p, grid, st);
  if (npast + 1 <= 16) return launch_gate_tc_dk<D, 16>(maps, p, grid, st);
  if (npast + 1 <= 24) return launch_gate_tc_dk<D, 24>(maps, p, grid, st);
  if (npast + 1 <= kGateMaxList) return launch_gate_tc_dk<D, kGateMaxList>(maps, p, grid, st);
  return cudaErrorInvalidValue;
}

// maps: Q (64-column box of 128 rows), Q tail, kbar planes (64-column box of
// min(nblk, 256) rounded to 16 rows), kbar tail.
cudaError_t launch_gate_tc(const CUtensorMap *maps, const GateParams &p, int grid, cudaStream_t st) {
  switch (p.d) {
    case 64: return launch_gate_tc_d<64>(maps, p, grid, st);
    case 80: return launch_gate_tc_d<80>(maps, p, grid, st);
    case 128: return launch_gate_tc_d<128>(maps, p, grid, st);
  }
  return cudaErrorInvalidValue;
}

// Whether this kernel takes the problem: at most 256 pooled blocks (all staged at once)
// and at most 31 past picks per row (a register list scanned without branches).
bool gate_tc_supports(int nblk, int topk) {
  return nblk <= kGateMaxBlocks && topk - 1 < kGateMaxList;
}

}  // namespace moba
