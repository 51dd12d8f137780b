// noalloc.cu -- MoBA prefill for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all: code that runs inside a CUDA-graph
// capture where allocation is forbidden, plugins whose host framework owns every
// allocation, or embedded runtimes with a fixed memory budget decided up front.  For
// them this entry point keeps all of its scratch (pooled keys, block choices, dispatch
// lists, partial outputs) in one file-scope device array of fixed size instead of a
// caller-provided workspace; the caller passes only q, k, v, out and lse.
//
// The array is part of this library's device module: a GPU that runs this entry point
// holds it (kStaticScratchBytes) until the process exits.  In host code its name is
// only a host-side stand-in, never a device address, so the first call on each device
// looks the device address up with cudaGetSymbolAddress (that device current) and
// caches it; make that first call before any stream capture.  Every call shares the
// array and leaves its contents behind; the list counters that must start at zero are
// cleared by the selection step on each call.  Calls whose work overlaps on the GPU
// (different streams, or concurrent host threads) race on the array.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "moba.h"
#include "params.h"

namespace moba {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
int static_scratch(void **ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOBA_ERR_NODEVICE;
  if (dev < 0 || dev >= kMaxDevices) return MOBA_ERR_NODEVICE;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return MOBA_ERR_LAUNCH;
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  return MOBA_OK;
}

}  // namespace
}  // namespace moba

using namespace moba;

extern "C" {

int moba_prefill_static(moba_tensor q, moba_tensor k, moba_tensor v, int batch, int hq, int hkv,
                        int N, int d, int block, int topk, int window, float scale,
                        moba_tensor out, float *lse, void *stream) {
  size_t ws = 0;
  int rc = moba_workspace_size(batch, hq, hkv, N, d, block, topk, &ws);
  if (rc) return rc;
  // Carve: pooled keys (f32), their bf16 split, block choices, workspace.
  const size_t nblk = size_t((N + block - 1) / block);
  const size_t kbar_bytes = align_up(size_t(batch) * hkv * nblk * d * 4, 256);
  const size_t split_bytes = align_up(size_t(batch) * hkv * 2 * nblk * d * 2, 256);
  const size_t idx_bytes = align_up(size_t(batch) * hq * size_t(N) * topk * 4, 256);
  const size_t need = kbar_bytes + split_bytes + idx_bytes + align_up(ws, 256);
  if (need > kStaticScratchBytes) return MOBA_ERR_TOO_LARGE;
  void *base = nullptr;
  if ((rc = static_scratch(&base))) return rc;
  unsigned char *sp = static_cast<unsigned char *>(base);
  float *kbar = reinterpret_cast<float *>(sp);
  void *split = sp + kbar_bytes;
  int32_t *idx = reinterpret_cast<int32_t *>(sp + kbar_bytes + split_bytes);
  void *work = sp + kbar_bytes + split_bytes + idx_bytes;
  if ((rc = moba_pool_keys(k, batch, hkv, N, d, block, kbar, split, stream))) return rc;
  if ((rc = moba_select_topk(q, split, batch, hq, hkv, N, d, block, topk, idx, work, ws, stream)))
    return rc;
  return moba_attn_fwd(q, k, v, idx, batch, hq, hkv, N, d, block, topk, window, scale, out, lse,
                       work, ws, stream);
}

}  // extern "C"
