// api.cu -- the C ABI of libmoba (declared in include/moba.h): argument checks,
// workspace carving, TMA descriptors and kernel launches.  Every step of the
// computation runs in the kernels of select.cu and attn.cu.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "common.cuh"
#include "moba.h"
#include "params.h"

namespace moba {

__device__ int g_device_status[kStatusWords] = {MOBA_OK, 0, 0, 0};

cudaError_t launch_pool(const uint16_t *k, int64_t sb, int64_t sh, int64_t sn, int batch, int hkv,
                        int N, int d, int block, float *kbar, uint16_t *split, cudaStream_t st);
cudaError_t launch_gate(const SelectParams &p, cudaStream_t st);
cudaError_t launch_scan(const int *counts, int *cursor, int *listoff, int *tileoff, int nlists,
                        cudaStream_t st);
cudaError_t launch_scatter(ScatterParams p, cudaStream_t st);
cudaError_t launch_pool_minmax(const uint16_t *k, int64_t sb, int64_t sh, int64_t sn, int batch,
                               int hkv, int N, int d, int block, uint16_t *planes, cudaStream_t st);
cudaError_t launch_static_select(int32_t *idx, int *counts, int batch, int hq, int hkv, int N,
                                 int q_off, int block, int topk, int sink, int nblk, int chunk_rows,
                                 cudaStream_t st);
cudaError_t launch_gate_tc(const CUtensorMap *maps, const GateParams &p, int grid, cudaStream_t st);
bool gate_tc_supports(int nblk, int topk);
cudaError_t launch_attn(const CUtensorMap *maps, const AttnParams &p, int mode, int grid,
                        cudaStream_t st);
cudaError_t launch_merge(const MergeParams &p, cudaStream_t st);
int query_major_units(int batch, int hq, int hkv, int block, int is_moba, int row_begin,
                      int row_end);
cudaError_t launch_bwd(const CUtensorMap *maps, const BwdParams &p, int nsm, cudaStream_t st);

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_tensor(const moba_tensor &t) {
  if (!t.ptr) return MOBA_ERR_ARG;
  if (!aligned16(t.ptr)) return MOBA_ERR_ALIGN;
  // bf16 strides in elements: 16-byte multiples.
  if ((t.sb % 8) || (t.sh % 8) || (t.sn % 8) || t.sb < 0 || t.sh < 0 || t.sn < 0)
    return MOBA_ERR_ALIGN;
  return MOBA_OK;
}

int check_device(int *num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOBA_ERR_NODEVICE;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return MOBA_ERR_NODEVICE;
  if (major != 10) return MOBA_ERR_NODEVICE;
  if (num_sms && cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MOBA_ERR_NODEVICE;
  return MOBA_OK;
}

int check_attn_dim(int d) { return (d == 64 || d == 80 || d == 128) ? MOBA_OK : MOBA_ERR_DIM; }

// N query rows at key positions q_off .. q_off + N - 1 (q_off = 0: a whole prefill).
int check_moba_shape(int batch, int hq, int hkv, int N, int d, int block, int topk, int q_off = 0) {
  if (batch < 1 || hq < 1 || hkv < 1 || N < 1 || block < 1) return MOBA_ERR_SHAPE;
  if (hq % hkv) return MOBA_ERR_SHAPE;
  // Any N and q_off (the last query tile may be partial and a tile may span two blocks);
  // block a multiple of the kernels' 128-key chunks, so that a chunk never holds keys of
  // two blocks (block need not divide the key count: the last block is then partial).
  if (block % kTileKeys) return MOBA_ERR_SHAPE;
  if (q_off < 0 || (long long)q_off + N >= (1ll << 31)) return MOBA_ERR_SHAPE;
  if (topk < 1 || topk > 32) return MOBA_ERR_ARG;
  const long long G = hq / hkv;
  if ((long long)N * G * (topk - 1) >= (1ll << 31)) return MOBA_ERR_SHAPE;
  if ((long long)batch * hq * N * (topk - 1) >= (1ll << 31)) return MOBA_ERR_SHAPE;
  if ((long long)batch * hq * N * topk >= (1ll << 40)) return MOBA_ERR_SHAPE;
  if (check_attn_dim(d) != MOBA_OK) return MOBA_ERR_DIM;
  return MOBA_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 4-D map over a bf16 [batch, heads, N, d] tensor (dims innermost first: d, N, heads,
// batch) whose box is `cols` columns x 128 rows, with the given swizzle.
int make_map(CUtensorMap *map, const moba_tensor &t, int batch, int heads, int N, int d, int cols,
             CUtensorMapSwizzle swz) {
  auto enc = get_encode();
  if (!enc) return MOBA_ERR_LAUNCH;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)heads, (cuuint64_t)batch};
  cuuint64_t strides[3] = {(cuuint64_t)t.sn * 2, (cuuint64_t)t.sh * 2, (cuuint64_t)t.sb * 2};
  // A size-1 dimension may carry any stride; give TMA a legal one.
  if (heads == 1) strides[1] = strides[0] * (cuuint64_t)N;
  if (batch == 1) strides[2] = strides[1] * (cuuint64_t)heads;
  cuuint32_t box[4] = {(cuuint32_t)cols, 128u, 1u, 1u};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, t.ptr, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MOBA_OK : MOBA_ERR_LAUNCH;
}

// Q, Q tail, K, K tail, V, V tail.
// q has Nq rows, k and v Nk rows.
int make_attn_maps(CUtensorMap *maps, const moba_tensor &q, const moba_tensor &k,
                   const moba_tensor &v, int batch, int hq, int hkv, int Nq, int Nk, int d) {
  const moba_tensor *ts[3] = {&q, &k, &v};
  const int heads[3] = {hq, hkv, hkv};
  const int rows[3] = {Nq, Nk, Nk};
  for (int a = 0; a < 3; ++a) {
    int rc = make_map(&maps[2 * a], *ts[a], batch, heads[a], rows[a], d, 64, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    if (d == 80)
      rc = make_map(&maps[2 * a + 1], *ts[a], batch, heads[a], rows[a], d, 16, CU_TENSOR_MAP_SWIZZLE_32B);
    else
      maps[2 * a + 1] = maps[2 * a];
    if (rc) return rc;
  }
  return MOBA_OK;
}

// 2-D maps over q viewed as rows ((b * hq + h) * N + i) of d columns, one row high, for
// the TMA gather of the gathered pass: a 64-column box (128-byte swizzle) and, for d = 80,
// a 16-column tail box (32-byte swizzle).  Returns false when q's strides give no such
// uniform row view or the row count does not fit the gather's int32 coordinates.
bool make_gather_maps(CUtensorMap *maps, const moba_tensor &q, int batch, int hq, int N, int d) {
  const long long rows = (long long)batch * hq * N;
  if (rows >= (1ll << 31)) return false;
  if (hq > 1 && q.sh != (int64_t)N * q.sn) return false;
  if (batch > 1 && q.sb != (int64_t)hq * N * q.sn) return false;
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)q.sn * 2};
  cuuint32_t estr[2] = {1u, 1u};
  cuuint32_t box0[2] = {64u, 1u};
  if (enc(&maps[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q.ptr, dims, strides, box0, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  maps[1] = maps[0];
  if (d == 80) {
    cuuint32_t box1[2] = {16u, 1u};
    if (enc(&maps[1], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q.ptr, dims, strides, box1, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  return true;
}

// 3-D maps over the pooled-key split [batch, hkv, 2, nblk, d] viewed as planes
// (b * hkv + hk) * 2 + part of nblk rows: a 64-column box of `rows` rows (128-byte
// swizzle) and, for d = 80, a 16-column tail box (32-byte swizzle).  Rows past nblk
// read as zero.
int make_kbar_maps(CUtensorMap *maps, const void *split, int batch, int hkv, int nblk, int d,
                   int rows) {
  auto enc = get_encode();
  if (!enc) return MOBA_ERR_LAUNCH;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)nblk, (cuuint64_t)batch * hkv * 2};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)nblk * d * 2};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  cuuint32_t box0[3] = {64u, (cuuint32_t)rows, 1u};
  void *ptr = const_cast<void *>(split);
  if (enc(&maps[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, ptr, dims, strides, box0, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return MOBA_ERR_LAUNCH;
  maps[1] = maps[0];
  if (d == 80) {
    cuuint32_t box1[3] = {16u, (cuuint32_t)rows, 1u};
    if (enc(&maps[1], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, ptr, dims, strides, box1, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MOBA_ERR_LAUNCH;
  }
  return MOBA_OK;
}

int launch_status(cudaError_t e) { return e == cudaSuccess ? MOBA_OK : MOBA_ERR_LAUNCH; }

// Per-pass timing events of moba_attn_fwd (diagnostics; see moba_set_pass_events).
constexpr int kMaxPassEvents = 1024;
cudaEvent_t g_pass_events[kMaxPassEvents];
int g_pass_nevents = 0;

void record_pass_event(int k, cudaStream_t st) {
  if (k < g_pass_nevents && g_pass_events[k]) cudaEventRecord(g_pass_events[k], st);
}

// Device address of the status words on the current device.
int status_words(int **ptr) {
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return MOBA_ERR_LAUNCH;
  *ptr = static_cast<int *>(p);
  return MOBA_OK;
}

}  // namespace
}  // namespace moba

using namespace moba;

extern "C" {

int moba_workspace_size_chunk(int batch, int hq, int hkv, int Nq, int Nk, int d, int block,
                              int topk, size_t *bytes) {
  if (!bytes) return MOBA_ERR_ARG;
  const int rc = check_moba_shape(batch, hq, hkv, Nq, d, block, topk, Nk - Nq);
  if (rc) return rc;
  *bytes = make_layout(batch, hq, hkv, Nq, d, block, topk, Nk - Nq).total;
  return MOBA_OK;
}

int moba_workspace_size(int batch, int hq, int hkv, int N, int d, int block, int topk,
                        size_t *bytes) {
  return moba_workspace_size_chunk(batch, hq, hkv, N, N, d, block, topk, bytes);
}

int moba_pool_keys(moba_tensor k, int batch, int hkv, int N, int d, int block, float *kbar,
                   void *kbar_split, void *stream) {
  if (batch < 1 || hkv < 1 || N < 1 || block < 1) return MOBA_ERR_SHAPE;
  if (d < 8 || d > 256 || d % 8) return MOBA_ERR_DIM;
  int rc = check_tensor(k);
  if (rc) return rc;
  if (!kbar || !kbar_split) return MOBA_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(kbar) & 3u) || (reinterpret_cast<uintptr_t>(kbar_split) & 1u))
    return MOBA_ERR_ALIGN;
  if ((rc = check_device(nullptr))) return rc;
  return launch_status(launch_pool(static_cast<const uint16_t *>(k.ptr), k.sb, k.sh, k.sn, batch,
                                   hkv, N, d, block, kbar, static_cast<uint16_t *>(kbar_split),
                                   static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

// Selection over the block representation in `kbar_split`: the hi / lo split of the
// means (minmax = 0; the tensor-core gate when it takes the problem) or the maxima /
// minima planes of min/max pooling (minmax = 1; the general gate).
static int select_topk_impl(moba_tensor q, const void *kbar_split, int batch, int hq, int hkv,
                            int N, int Nk, int d, int block, int topk, int32_t *idx,
                            void *workspace, size_t workspace_bytes, void *stream, int minmax) {
  const int q_off = Nk - N;
  int rc = check_moba_shape(batch, hq, hkv, N, d, block, topk, q_off);
  if (rc) return rc;
  if ((rc = check_tensor(q))) return rc;
  if (!kbar_split || !idx) return MOBA_ERR_ARG;
  if (!aligned16(kbar_split) || (reinterpret_cast<uintptr_t>(idx) & 3u)) return MOBA_ERR_ALIGN;
  const WorkspaceLayout w = make_layout(batch, hq, hkv, N, d, block, topk, q_off);
  if (!workspace || workspace_bytes < w.total) return MOBA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MOBA_ERR_ALIGN;
  if ((rc = check_device(nullptr))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char *ws = static_cast<char *>(workspace);
  int *counts = reinterpret_cast<int *>(ws + w.off_counts);
  // The list counts and the tensor-core gate's two counters after them.
  if (cudaMemsetAsync(counts, 0, sizeof(int) * (size_t)(w.nlists + 2), st) != cudaSuccess)
    return MOBA_ERR_LAUNCH;
  int *cursor = reinterpret_cast<int *>(ws + w.off_cursor);
  int *listoff = reinterpret_cast<int *>(ws + w.off_listoff);
  int *tileoff = reinterpret_cast<int *>(ws + w.off_tileoff);
  int4 *tiles = reinterpret_cast<int4 *>(ws + w.off_tiles);
  bool scanned = false;  // list offsets already written by the gate kernel
  if (!minmax && gate_tc_supports(w.nblk, topk)) {
    // Tensor-core gate: q tiles and the pooled keys through TMA.
    int nsm = 0;
    if ((rc = check_device(&nsm))) return rc;
    CUtensorMap maps[4];
    if ((rc = make_map(&maps[0], q, batch, hq, N, d, 64, CU_TENSOR_MAP_SWIZZLE_128B))) return rc;
    if (d == 80) {
      if ((rc = make_map(&maps[1], q, batch, hq, N, d, 16, CU_TENSOR_MAP_SWIZZLE_32B))) return rc;
    } else {
      maps[1] = maps[0];
    }
    const int rows = (w.nblk + 15) & ~15;
    if ((rc = make_kbar_maps(&maps[2], kbar_split, batch, hkv, w.nblk, d, rows))) return rc;
    GateParams gp{};
    if ((rc = status_words(&gp.status))) return rc;
    gp.idx = idx;
    gp.counts = counts;
    gp.sched = counts + w.nlists;
    if (w.npast > 0) {
      gp.done = counts + w.nlists + 1;
      gp.cursor = cursor; gp.listoff = listoff; gp.tileoff = tileoff; gp.nlists = w.nlists;
      scanned = true;
    }
    gp.batch = batch; gp.hq = hq; gp.hkv = hkv; gp.N = N; gp.d = d; gp.block = block;
    gp.topk = topk; gp.nblk = w.nblk; gp.G = w.G; gp.chunk_rows = w.chunk_rows;
    gp.q_off = q_off;
    const long long ntiles = (long long)batch * hkv * ((N + kTileRows - 1) / kTileRows) * w.G;
    const int grid = (int)(ntiles < nsm ? ntiles : nsm);
    if ((rc = launch_status(launch_gate_tc(maps, gp, grid, st)))) return rc;
  } else {
    SelectParams sp{};
    sp.q = static_cast<const uint16_t *>(q.ptr);
    sp.q_sb = q.sb; sp.q_sh = q.sh; sp.q_sn = q.sn;
    sp.kbar_split = static_cast<const uint16_t *>(kbar_split);
    sp.idx = idx;
    sp.counts = counts;
    sp.batch = batch; sp.hq = hq; sp.hkv = hkv; sp.N = N; sp.d = d; sp.block = block;
    sp.topk = topk; sp.nblk = w.nblk; sp.G = w.G; sp.chunk_rows = w.chunk_rows;
    sp.q_off = q_off;
    sp.minmax = minmax;
    if ((rc = launch_status(launch_gate(sp, st)))) return rc;
  }
  if (w.npast == 0) return MOBA_OK;
  if (!scanned && (rc = launch_status(launch_scan(counts, cursor, listoff, tileoff, w.nlists, st))))
    return rc;
  ScatterParams cp{};
  cp.idx = idx;
  cp.counts = counts;
  cp.listoff = listoff;
  cp.tileoff = tileoff;
  cp.tiles = tiles;
  cp.nlists = w.nlists;
  cp.cursor = cursor;
  cp.entries = reinterpret_cast<uint32_t *>(ws + w.off_entries);
  cp.batch = batch; cp.hq = hq; cp.hkv = hkv; cp.N = N; cp.block = block; cp.topk = topk;
  cp.nblk = w.nblk; cp.G = w.G; cp.chunk_rows = w.chunk_rows;
  cp.q_off = q_off;
  return launch_status(launch_scatter(cp, st));
}

extern "C" {

int moba_select_topk_chunk(moba_tensor q, const void *kbar_split, int batch, int hq, int hkv,
                           int N, int Nk, int d, int block, int topk, int32_t *idx,
                           void *workspace, size_t workspace_bytes, void *stream) {
  return select_topk_impl(q, kbar_split, batch, hq, hkv, N, Nk, d, block, topk, idx, workspace,
                          workspace_bytes, stream, 0);
}

int moba_pool_keys_minmax(moba_tensor k, int batch, int hkv, int N, int d, int block,
                          void *kminmax, void *stream) {
  if (batch < 1 || hkv < 1 || N < 1 || block < 1) return MOBA_ERR_SHAPE;
  if (d < 8 || d > 256 || d % 8) return MOBA_ERR_DIM;
  int rc = check_tensor(k);
  if (rc) return rc;
  if (!kminmax) return MOBA_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(kminmax) & 1u) return MOBA_ERR_ALIGN;
  if ((rc = check_device(nullptr))) return rc;
  return launch_status(launch_pool_minmax(static_cast<const uint16_t *>(k.ptr), k.sb, k.sh, k.sn,
                                          batch, hkv, N, d, block,
                                          static_cast<uint16_t *>(kminmax),
                                          static_cast<cudaStream_t>(stream)));
}

int moba_select_topk_minmax(moba_tensor q, const void *kminmax, int batch, int hq, int hkv, int N,
                            int Nk, int d, int block, int topk, int32_t *idx, void *workspace,
                            size_t workspace_bytes, void *stream) {
  return select_topk_impl(q, kminmax, batch, hq, hkv, N, Nk, d, block, topk, idx, workspace,
                          workspace_bytes, stream, 1);
}

int moba_select_static(int batch, int hq, int hkv, int N, int Nk, int d, int block, int topk,
                       int sink, int32_t *idx, void *workspace, size_t workspace_bytes,
                       void *stream) {
  const int q_off = Nk - N;
  int rc = check_moba_shape(batch, hq, hkv, N, d, block, topk, q_off);
  if (rc) return rc;
  if (sink < 0 || sink > topk - 1) return MOBA_ERR_ARG;
  if (!idx) return MOBA_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(idx) & 3u) return MOBA_ERR_ALIGN;
  const WorkspaceLayout w = make_layout(batch, hq, hkv, N, d, block, topk, q_off);
  if (!workspace || workspace_bytes < w.total) return MOBA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MOBA_ERR_ALIGN;
  if ((rc = check_device(nullptr))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char *ws = static_cast<char *>(workspace);
  int *counts = reinterpret_cast<int *>(ws + w.off_counts);
  if (cudaMemsetAsync(counts, 0, sizeof(int) * (size_t)(w.nlists + 2), st) != cudaSuccess)
    return MOBA_ERR_LAUNCH;
  if ((rc = launch_status(launch_static_select(idx, counts, batch, hq, hkv, N, q_off, block, topk,
                                               sink, w.nblk, w.chunk_rows, st))))
    return rc;
  if (w.npast == 0) return MOBA_OK;
  int *cursor = reinterpret_cast<int *>(ws + w.off_cursor);
  int *listoff = reinterpret_cast<int *>(ws + w.off_listoff);
  int *tileoff = reinterpret_cast<int *>(ws + w.off_tileoff);
  if ((rc = launch_status(launch_scan(counts, cursor, listoff, tileoff, w.nlists, st)))) return rc;
  ScatterParams cp{};
  cp.idx = idx;
  cp.counts = counts;
  cp.listoff = listoff;
  cp.tileoff = tileoff;
  cp.tiles = reinterpret_cast<int4 *>(ws + w.off_tiles);
  cp.nlists = w.nlists;
  cp.cursor = cursor;
  cp.entries = reinterpret_cast<uint32_t *>(ws + w.off_entries);
  cp.batch = batch; cp.hq = hq; cp.hkv = hkv; cp.N = N; cp.block = block; cp.topk = topk;
  cp.nblk = w.nblk; cp.G = w.G; cp.chunk_rows = w.chunk_rows;
  cp.q_off = q_off;
  return launch_status(launch_scatter(cp, st));
}

int moba_select_topk(moba_tensor q, const void *kbar_split, int batch, int hq, int hkv, int N,
                     int d, int block, int topk, int32_t *idx, void *workspace,
                     size_t workspace_bytes, void *stream) {
  return moba_select_topk_chunk(q, kbar_split, batch, hq, hkv, N, N, d, block, topk, idx,
                                workspace, workspace_bytes, stream);
}

int moba_attn_fwd_chunk(moba_tensor q, moba_tensor k, moba_tensor v, const int32_t *idx,
                        int batch, int hq, int hkv, int N, int Nk, int d, int block, int topk,
                        int window, float scale, moba_tensor out, float *lse, void *workspace,
                        size_t workspace_bytes, void *stream) {
  const int q_off = Nk - N;
  int rc = check_moba_shape(batch, hq, hkv, N, d, block, topk, q_off);
  if (rc) return rc;
  if (window < 0) return MOBA_ERR_ARG;
  if ((rc = check_tensor(q)) || (rc = check_tensor(k)) || (rc = check_tensor(v)) ||
      (rc = check_tensor(out)))
    return rc;
  if (!idx || !lse) return MOBA_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(idx) & 3u) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return MOBA_ERR_ALIGN;
  const WorkspaceLayout w = make_layout(batch, hq, hkv, N, d, block, topk, q_off);
  if (!workspace || workspace_bytes < w.total) return MOBA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MOBA_ERR_ALIGN;
  int nsm = 0;
  if ((rc = check_device(&nsm))) return rc;
  CUtensorMap maps[6];
  if ((rc = make_attn_maps(maps, q, k, v, batch, hq, hkv, N, Nk, d))) return rc;
  // The gathered pass reads q through 2-D row maps in place of the 4-D tile maps.
  CUtensorMap gmaps[6];
  for (int a = 0; a < 6; ++a) gmaps[a] = maps[a];
  const int q_gather_tma = make_gather_maps(gmaps, q, batch, hq, N, d) ? 1 : 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char *ws = static_cast<char *>(workspace);
  AttnParams p{};
  if ((rc = status_words(&p.status))) return rc;
  p.q = static_cast<const uint16_t *>(q.ptr);
  p.q_sb = q.sb; p.q_sh = q.sh; p.q_sn = q.sn;
  p.out = static_cast<uint16_t *>(out.ptr);
  p.o_sb = out.sb; p.o_sh = out.sh; p.o_sn = out.sn;
  p.lse = lse;
  p.idx = idx;
  p.batch = batch; p.hq = hq; p.hkv = hkv; p.N = N; p.d = d; p.block = block; p.topk = topk;
  p.window = window; p.G = w.G;
  p.q_off = q_off;
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)d);
  p.scale_log2 = sc * 1.4426950408889634f;
  p.is_moba = 1;
  p.listoff = reinterpret_cast<const int *>(ws + w.off_listoff);
  p.tileoff = reinterpret_cast<const int *>(ws + w.off_tileoff);
  p.tiles = reinterpret_cast<const int4 *>(ws + w.off_tiles);
  p.entries = reinterpret_cast<const uint32_t *>(ws + w.off_entries);
  p.opart = reinterpret_cast<uint16_t *>(ws + w.off_opart);
  p.lpart = reinterpret_cast<float *>(ws + w.off_lpart);
  p.chunk_rows = w.chunk_rows;
  p.npast = w.npast;
  p.nblk = w.nblk;
  p.lists_per_chunk = batch * hkv * w.nblk;
  int ev = 0;
  record_pass_event(ev++, st);
  for (int c = 0; c < w.nchunks; ++c) {
    p.chunk = c;
    p.row_begin = c * w.chunk_rows;
    p.row_end = (c + 1) * w.chunk_rows < N ? (c + 1) * w.chunk_rows : N;
    if (w.npast > 0) {
      p.ntiles = 0;  // read from the workspace by the kernel
      p.q_gather_tma = q_gather_tma;
      if ((rc = launch_status(launch_attn(gmaps, p, kGathered, nsm, st)))) return rc;
      p.q_gather_tma = 0;
      record_pass_event(ev++, st);
    }
    p.ntiles = query_major_units(batch, hq, hkv, block, 1, p.row_begin, p.row_end);
    const int grid = p.ntiles < nsm ? p.ntiles : nsm;
    if ((rc = launch_status(launch_attn(maps, p, kQueryMajor, grid, st)))) return rc;
    record_pass_event(ev++, st);
    if (w.npast > 0) {
      MergeParams mp{};
      mp.opart = p.opart;
      mp.lpart = p.lpart;
      mp.idx = idx;
      mp.out = p.out;
      mp.o_sb = out.sb; mp.o_sh = out.sh; mp.o_sn = out.sn;
      mp.lse = lse;
      mp.batch = batch; mp.hq = hq; mp.N = N; mp.d = d; mp.block = block; mp.topk = topk;
      mp.chunk_rows = w.chunk_rows;
      mp.row_begin = p.row_begin;
      mp.row_end = p.row_end;
      mp.q_off = q_off;
      if ((rc = launch_status(launch_merge(mp, st)))) return rc;
      record_pass_event(ev++, st);
    }
  }
  return MOBA_OK;
}

int moba_attn_fwd(moba_tensor q, moba_tensor k, moba_tensor v, const int32_t *idx, int batch,
                  int hq, int hkv, int N, int d, int block, int topk, int window, float scale,
                  moba_tensor out, float *lse, void *workspace, size_t workspace_bytes,
                  void *stream) {
  return moba_attn_fwd_chunk(q, k, v, idx, batch, hq, hkv, N, N, d, block, topk, window, scale,
                             out, lse, workspace, workspace_bytes, stream);
}

int moba_set_pass_events(void *const *events, int count) {
  if (count < 0 || count > kMaxPassEvents) return MOBA_ERR_ARG;
  if (!events) count = 0;
  for (int k = 0; k < kMaxPassEvents; ++k)
    g_pass_events[k] = (k < count) ? static_cast<cudaEvent_t>(events[k]) : nullptr;
  g_pass_nevents = count;
  return MOBA_OK;
}

int swa_attn_fwd_chunk(moba_tensor q, moba_tensor k, moba_tensor v, int batch, int hq, int hkv,
                       int N, int Nk, int d, int window, float scale, moba_tensor out, float *lse,
                       void *stream) {
  if (batch < 1 || hq < 1 || hkv < 1 || N < 1 || hq % hkv) return MOBA_ERR_SHAPE;
  // Query row i sits at key position Nk - N + i (any offset).
  const int q_off = Nk - N;
  if (q_off < 0 || (long long)Nk >= (1ll << 31)) return MOBA_ERR_SHAPE;
  if (window < 1) return MOBA_ERR_ARG;
  int rc = check_attn_dim(d);
  if (rc) return rc;
  if ((rc = check_tensor(q)) || (rc = check_tensor(k)) || (rc = check_tensor(v)) ||
      (rc = check_tensor(out)))
    return rc;
  if (!lse) return MOBA_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return MOBA_ERR_ALIGN;
  int nsm = 0;
  if ((rc = check_device(&nsm))) return rc;
  CUtensorMap maps[6];
  if ((rc = make_attn_maps(maps, q, k, v, batch, hq, hkv, N, Nk, d))) return rc;
  AttnParams p{};
  if ((rc = status_words(&p.status))) return rc;
  p.q = static_cast<const uint16_t *>(q.ptr);
  p.q_sb = q.sb; p.q_sh = q.sh; p.q_sn = q.sn;
  p.out = static_cast<uint16_t *>(out.ptr);
  p.o_sb = out.sb; p.o_sh = out.sh; p.o_sn = out.sn;
  p.lse = lse;
  p.idx = nullptr;
  p.batch = batch; p.hq = hq; p.hkv = hkv; p.N = N; p.d = d; p.block = 0; p.topk = 0;
  p.window = window < Nk ? window : Nk;
  p.q_off = q_off;
  p.G = hq / hkv;
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)d);
  p.scale_log2 = sc * 1.4426950408889634f;
  p.is_moba = 0;
  p.row_begin = 0;
  p.row_end = N;
  p.ntiles = query_major_units(batch, hq, hkv, 0, 0, 0, N);
  p.npast = 0;
  const int grid = p.ntiles < nsm ? p.ntiles : nsm;
  return launch_status(launch_attn(maps, p, kQueryMajor, grid, static_cast<cudaStream_t>(stream)));
}

int swa_attn_fwd(moba_tensor q, moba_tensor k, moba_tensor v, int batch, int hq, int hkv, int N,
                 int d, int window, float scale, moba_tensor out, float *lse, void *stream) {
  return swa_attn_fwd_chunk(q, k, v, batch, hq, hkv, N, N, d, window, scale, out, lse, stream);
}

int moba_bwd_workspace_size(int batch, int hq, int hkv, int N, int d, int block, int topk,
                            size_t *bytes) {
  if (!bytes) return MOBA_ERR_ARG;
  const int rc = check_moba_shape(batch, hq, hkv, N, d, block, topk, 0);
  if (rc) return rc;
  if (d != 64 && d != 128) return MOBA_ERR_DIM;
  *bytes = bwd_workspace_bytes(batch, hq, N, d, topk, nullptr);
  return MOBA_OK;
}

int moba_attn_bwd(moba_tensor q, moba_tensor k, moba_tensor v, moba_tensor out, moba_tensor dout,
                  const float *lse, const int32_t *idx, const void *workspace,
                  size_t workspace_bytes, int batch, int hq, int hkv, int N, int d, int block,
                  int topk, int window, float scale, moba_tensor dq, moba_tensor dk,
                  moba_tensor dv, void *bwd_workspace, size_t bwd_workspace_bytes_, void *stream) {
  int rc = check_moba_shape(batch, hq, hkv, N, d, block, topk, 0);
  if (rc) return rc;
  if (d != 64 && d != 128) return MOBA_ERR_DIM;
  if (window != 0) return MOBA_ERR_ARG;
  const moba_tensor ts[8] = {q, k, v, out, dout, dq, dk, dv};
  for (const moba_tensor &t : ts)
    if ((rc = check_tensor(t))) return rc;
  if (!lse || !idx) return MOBA_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(idx) & 3u))
    return MOBA_ERR_ALIGN;
  const WorkspaceLayout w = make_layout(batch, hq, hkv, N, d, block, topk, 0);
  if (!workspace || workspace_bytes < w.total) return MOBA_ERR_WORKSPACE;
  size_t off_dqp = 0;
  const size_t need = bwd_workspace_bytes(batch, hq, N, d, topk, &off_dqp);
  if (!bwd_workspace || bwd_workspace_bytes_ < need) return MOBA_ERR_WORKSPACE;
  if (!aligned16(workspace) || !aligned16(bwd_workspace)) return MOBA_ERR_ALIGN;
  int nsm = 0;
  if ((rc = check_device(&nsm))) return rc;
  CUtensorMap maps[6];
  if ((rc = make_attn_maps(maps, q, k, v, batch, hq, hkv, N, N, d))) return rc;
  const CUtensorMap kv[2] = {maps[2], maps[4]};
  const char *ws = static_cast<const char *>(workspace);
  char *bws = static_cast<char *>(bwd_workspace);
  BwdParams p{};
  if ((rc = status_words(&p.status))) return rc;
  p.q = static_cast<const uint16_t *>(q.ptr);
  p.q_sb = q.sb; p.q_sh = q.sh; p.q_sn = q.sn;
  p.out = static_cast<const uint16_t *>(out.ptr);
  p.o_sb = out.sb; p.o_sh = out.sh; p.o_sn = out.sn;
  p.dout = static_cast<const uint16_t *>(dout.ptr);
  p.do_sb = dout.sb; p.do_sh = dout.sh; p.do_sn = dout.sn;
  p.lse = lse;
  p.dq = static_cast<uint16_t *>(dq.ptr);
  p.dq_sb = dq.sb; p.dq_sh = dq.sh; p.dq_sn = dq.sn;
  p.dk = static_cast<uint16_t *>(dk.ptr);
  p.dk_sb = dk.sb; p.dk_sh = dk.sh; p.dk_sn = dk.sn;
  p.dv = static_cast<uint16_t *>(dv.ptr);
  p.dv_sb = dv.sb; p.dv_sh = dv.sh; p.dv_sn = dv.sn;
  p.rowstat = reinterpret_cast<float2 *>(bws);
  p.dqp = reinterpret_cast<float *>(bws + off_dqp);
  p.batch = batch; p.hq = hq; p.hkv = hkv; p.N = N; p.d = d; p.block = block; p.topk = topk;
  p.npast = topk - 1; p.nblk = w.nblk; p.G = w.G; p.nchunks = w.nchunks; p.nlists = w.nlists;
  const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)d);
  p.scale = sc;
  p.scale_log2 = sc * 1.4426950408889634f;
  p.entries = reinterpret_cast<const uint32_t *>(ws + w.off_entries);
  p.tiles = reinterpret_cast<const int4 *>(ws + w.off_tiles);
  p.tileoff = reinterpret_cast<const int *>(ws + w.off_tileoff);
  p.listoff = reinterpret_cast<const int *>(ws + w.off_listoff);
  return launch_status(launch_bwd(kv, p, nsm, static_cast<cudaStream_t>(stream)));
}

int moba_device_status(void) {
  int v[2] = {MOBA_OK, 0};
  if (cudaDeviceSynchronize() != cudaSuccess) return MOBA_ERR_LAUNCH;
  if (cudaMemcpyFromSymbol(v, g_device_status, sizeof(v)) != cudaSuccess) return MOBA_ERR_LAUNCH;
  const int zero[2] = {MOBA_OK, 0};
  if (cudaMemcpyToSymbol(g_device_status, zero, sizeof(zero)) != cudaSuccess) return MOBA_ERR_LAUNCH;
  return v[0];
}

int moba_debug_set_wait_limit_us(int microseconds) {
  if (microseconds < 0) return MOBA_ERR_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return MOBA_ERR_LAUNCH;
  if (cudaMemcpyToSymbol(g_device_status, &microseconds, sizeof(int), 2 * sizeof(int)) != cudaSuccess)
    return MOBA_ERR_LAUNCH;
  return MOBA_OK;
}

int moba_debug_fault_next_launch(int kind) {
  if (kind < 0 || kind > 1) return MOBA_ERR_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return MOBA_ERR_LAUNCH;
  if (cudaMemcpyToSymbol(g_device_status, &kind, sizeof(int), 3 * sizeof(int)) != cudaSuccess)
    return MOBA_ERR_LAUNCH;
  return MOBA_OK;
}

const char *moba_status_string(int status) {
  switch (status) {
    case MOBA_OK: return "ok";
    case MOBA_ERR_SHAPE: return "unsupported shape (hq % hkv, block % 128, size limits)";
    case MOBA_ERR_DIM: return "unsupported head dimension";
    case MOBA_ERR_ALIGN: return "pointer or stride not 16-byte aligned";
    case MOBA_ERR_ARG: return "invalid argument";
    case MOBA_ERR_WORKSPACE: return "workspace missing or too small";
    case MOBA_ERR_LAUNCH: return "CUDA launch or driver call failed";
    case MOBA_ERR_DEVICE: return "a kernel wait timed out on the device";
    case MOBA_ERR_NODEVICE: return "no sm_100 device is current";
    case MOBA_ERR_TOO_LARGE: return "problem exceeds the 32 MiB static scratch of moba_prefill_static";
  }
  return "unknown status";
}

}  // extern "C"
