// params.h -- problem description, workspace layout and kernel parameter blocks
// shared by the host-side ABI and the kernels.
#pragma once

#include <stddef.h>
#include <stdint.h>
#include <vector_types.h>

namespace moba {

constexpr int kTileRows = 128;   // query rows per attention tile (tcgen05 M)
constexpr int kUnitRows = 256;   // list entries per gathered work unit (two tiles)
constexpr int kTileKeys = 128;   // keys per attention chunk (tcgen05 N of S = QK^T)
constexpr size_t kPartialCapBytes = size_t(4) << 30;  // partial outputs kept per pass

// Block-major dispatch lists and partial outputs, carved out of the caller's workspace.
// List L = ((chunk * batch + b) * hkv + hk) * nblk + j holds the (row, q-head, slot)
// triples of the rows of query chunk `chunk` that picked past block j.
struct WorkspaceLayout {
  int nblk;         // ceil((q_off + N) / block): a partial last block when block does not
                    // divide the key count
  int G;            // hq / hkv
  int npast;        // topk - 1: partial slots per row
  int chunk_rows;   // query rows per pass (multiple of 128)
  int nchunks;
  int nlists;       // nchunks * batch * hkv * nblk
  size_t off_counts;   // int32 [nlists + 2]   entries per list (atomic counts), then the
                       //                      gate's tile counter and finished-CTA count
  size_t off_cursor;   // int32 [nlists]       scatter cursors
  size_t off_listoff;  // int32 [nlists + 1]   exclusive prefix of counts
  size_t off_tileoff;  // int32 [nlists + 1]   exclusive prefix of ceil(count / 256)
  size_t off_entries;  // uint32 [max_entries] entry = (i * G + g) * npast + slot
  size_t off_tiles;    // int4 [max_tiles]      per 256-entry unit: list, first entry, rows
  size_t off_opart;    // bf16 [batch, hq, chunk_rows, topk, d]: slots 0..npast-1 past
                       //      blocks, slot npast the own block
  size_t off_lpart;    // f32  [batch, hq, chunk_rows, topk]
  size_t total;
  long long max_entries;
  long long max_tiles;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// N query rows; the keys run over q_off + N positions (q_off > 0: a chunk of a longer
// prefill whose queries are the last N positions).
inline WorkspaceLayout make_layout(int batch, int hq, int hkv, int N, int d, int block,
                                   int topk, int q_off = 0) {
  WorkspaceLayout w{};
  w.nblk = (q_off + N + block - 1) / block;
  w.G = hq / hkv;
  w.npast = topk - 1;
  // Partials exist only when a row can attend past blocks: topk slots per row then.
  const size_t nslots = w.npast > 0 ? size_t(topk) : 0;
  const size_t per_row = nslots * (size_t(d) * 2 + 4) * size_t(batch) * size_t(hq);
  long long rows = N;
  if (per_row > 0 && per_row * size_t(N) > kPartialCapBytes) {
    rows = static_cast<long long>(kPartialCapBytes / per_row) / kTileRows * kTileRows;
    if (rows < kTileRows) rows = kTileRows;
  }
  w.chunk_rows = static_cast<int>(rows);
  w.nchunks = static_cast<int>((N + w.chunk_rows - 1) / w.chunk_rows);
  w.nlists = w.nchunks * batch * hkv * w.nblk;
  w.max_entries = static_cast<long long>(batch) * hq * N * w.npast;
  w.max_tiles = w.max_entries / kUnitRows + w.nlists + 1;
  size_t off = 0;
  w.off_counts = off;  off = align_up(off + sizeof(int) * size_t(w.nlists + 2), 256);
  w.off_cursor = off;  off = align_up(off + sizeof(int) * size_t(w.nlists), 256);
  w.off_listoff = off; off = align_up(off + sizeof(int) * size_t(w.nlists + 1), 256);
  w.off_tileoff = off; off = align_up(off + sizeof(int) * size_t(w.nlists + 1), 256);
  w.off_entries = off; off = align_up(off + sizeof(uint32_t) * size_t(w.max_entries), 256);
  w.off_tiles = off;   off = align_up(off + 16 * size_t(w.max_tiles), 256);
  const size_t prow = size_t(batch) * hq * size_t(w.chunk_rows) * nslots;
  w.off_opart = off;   off = align_up(off + prow * size_t(d) * 2, 256);
  w.off_lpart = off;   off = align_up(off + prow * sizeof(float), 256);
  w.total = off;
  return w;
}

// Parameters of the gate / top-k kernel.
struct SelectParams {
  const uint16_t *q;     // bf16 bits
  int64_t q_sb, q_sh, q_sn;
  const uint16_t *kbar_split;  // [batch, hkv, 2, nblk, d]
  int32_t *idx;          // [batch, hq, N, topk]
  int *counts;           // workspace list counts
  int batch, hq, hkv, N, d, block, topk, nblk, G, chunk_rows;
  int q_off;             // position of query row 0 among the keys
  int minmax;            // 1: the planes are block maxima and minima (min/max pooling), and
                         // the score is q+ . kmax + q- . kmin; 0: hi + lo of the means
};

// Parameters of the tensor-core gate / top-k kernel (q and the pooled keys arrive
// through TMA maps).
struct GateParams {
  int *status;           // device status words
  int32_t *idx;          // [batch, hq, N, topk]
  int *counts;           // workspace list counts
  int batch, hq, hkv, N, d, block, topk, nblk, G, chunk_rows;
  int q_off;             // position of query row 0 among the keys
  int qstages;           // query tile ring depth (set by the launcher)
  int kslots;            // pooled-key staging slots, 1 or 2 (set by the launcher)
  int *sched;            // tile counter, zero at launch (the word after the list counts)
  int chunk_tiles;       // tiles per chunk taken from it (set by the launcher)
  // When done is set (zero at launch, the second word after the counts), the last
  // CTA to finish writes the list offsets (cursor, listoff, tileoff over nlists).
  int *done;
  int *cursor, *listoff, *tileoff;
  int nlists;
};

struct ScatterParams {
  const int32_t *idx;
  int *cursor;
  uint32_t *entries;
  int batch, hq, hkv, N, block, topk, nblk, G, chunk_rows;
  int q_off;               // position of query row 0 among the keys
  // Unit table (written by the scatter grid from the scanned offsets).
  const int *counts;
  const int *listoff;
  const int *tileoff;
  int4 *tiles;
  int nlists;
  int cache_rows;          // 1: the CTA's block choices are staged in shared memory
};

// Attention kernel modes.
enum AttnMode : int {
  kQueryMajor = 0,  // contiguous 128-row query tiles: own block (MoBA) or band (SWA)
  kGathered = 1,    // gathered rows of one block-major list against one whole block
};

struct AttnParams {
  int *status;             // device status words (see common.cuh)
  // Tensors (bf16 bits) and strides in elements.
  const uint16_t *q;
  int64_t q_sb, q_sh, q_sn;
  uint16_t *out;
  int64_t o_sb, o_sh, o_sn;
  float *lse;              // [batch, hq, N]
  const int32_t *idx;      // [batch, hq, N, topk] (MoBA) or null (SWA)
  // Problem: N query rows; keys and values run over q_off + N positions, query row i
  // sits at position q_off + i.
  int batch, hq, hkv, N, d, block, topk, window, G;
  int q_off;
  float scale_log2;        // scale * log2(e)
  int is_moba;             // 0: sliding window only (swa_attn_fwd)
  // Gathered pass: 1 when the query rows are fetched by TMA gather4 through a 2-D map
  // over q (row ((b * hq + h) * N + i)); 0 when by cp.async (q's strides admit no
  // single row stride, or the row count exceeds int32).
  int q_gather_tma;
  // Query-major pass: row range of this pass.
  int row_begin, row_end;  // multiples of 128 except row_end == N (any N)
  int ntiles;              // query-major work units in this pass
  // Block-major lists and partials (MoBA).
  const int *listoff;
  const int *tileoff;
  const int4 *tiles;       // per gathered unit: list, first entry, rows (<= 256)
  const uint32_t *entries;
  uint16_t *opart;         // [batch, hq, chunk_rows, topk, d]
  float *lpart;            // [batch, hq, chunk_rows, topk]
  int chunk, chunk_rows, npast, nblk, lists_per_chunk;
};

// Parameters of the merge pass (one query chunk).
struct MergeParams {
  const uint16_t *opart;   // [batch, hq, chunk_rows, topk, d]
  const float *lpart;      // [batch, hq, chunk_rows, topk]
  const int32_t *idx;      // [batch, hq, N, topk]
  uint16_t *out;
  int64_t o_sb, o_sh, o_sn;
  float *lse;              // [batch, hq, N]
  int batch, hq, N, d, block, topk, chunk_rows, row_begin, row_end;
  int q_off;               // position of query row 0 among the keys
};

// Parameters of the backward kernels (bwd.cu).
struct BwdParams {
  int *status;             // device status words
  const uint16_t *q, *out, *dout;
  int64_t q_sb, q_sh, q_sn, o_sb, o_sh, o_sn, do_sb, do_sh, do_sn;
  const float *lse;        // [batch, hq, N] (natural log)
  uint16_t *dq, *dk, *dv;
  int64_t dq_sb, dq_sh, dq_sn, dk_sb, dk_sh, dk_sn, dv_sb, dv_sh, dv_sn;
  float2 *rowstat;         // [batch, hq, N]: lse * log2(e), D = dO . o
  float *dqp;              // [batch, hq, N, topk, d] fp32 partial dQ per block slot
  int batch, hq, hkv, N, d, block, topk, npast, nblk, G, nchunks, nlists;
  float scale, scale_log2;
  // Dispatch lists of the forward's selection step (its workspace).
  const uint32_t *entries;
  const int4 *tiles;
  const int *tileoff, *listoff;
};

// Bytes of the backward's own workspace: the row statistics, then the dQ partials.
inline size_t bwd_workspace_bytes(int batch, int hq, int N, int d, int topk, size_t *off_dqp) {
  const size_t rows = size_t(batch) * hq * size_t(N);
  const size_t a = align_up(rows * 8, 256);
  if (off_dqp) *off_dqp = a;
  return a + align_up(rows * size_t(topk) * size_t(d) * 4, 256);
}

}  // namespace moba
