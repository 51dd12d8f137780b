// noalloc.cu -- MoBA prefill for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all: plugins whose host framework owns every
// device allocation and hands the plugin only its inputs and outputs, or embedded
// runtimes whose memory budget is fixed and fully assigned before the first request.
// For them this entry point keeps all of its scratch (pooled keys, block choices,
// dispatch lists, partial outputs) in one file-scope device array of fixed size
// instead of a caller-provided workspace; the caller passes only q, k, v, out and lse.
//
// The array is part of this library's device module: a GPU that runs this entry point
// holds it (kStaticScratchBytes) until the process exits.  In host code its name is
// only a host-side stand-in, never a device address, so the first call on each device
// (with that device current) looks the device address up with cudaGetSymbolAddress
// and caches it, keyed by the device and its current CUDA context; make that first
// call before any stream capture.  After a cudaDeviceReset the primary context is a
// new one, and the next call looks the address up again.  Every call shares the array
// and leaves its contents behind; the list counters that must start at zero are
// cleared by the selection step on each call.  Calls whose work overlaps on the GPU
// (different streams, or concurrent host threads) race on the array.
#include <cuda.h>
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
CUcontext g_scratch_ctx[kMaxDevices] = {};

// The current CUDA context (through the driver entry point the runtime exposes), or
// null when it cannot be read.
CUcontext current_context() {
  using GetCurrent = CUresult (*)(CUcontext *);
  static GetCurrent fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<GetCurrent>(p);
  }
  CUcontext ctx = nullptr;
  if (fn && fn(&ctx) != CUDA_SUCCESS) ctx = nullptr;
  return ctx;
}

// Device address of the scratch array on the current device: looked up once per
// device and context (a device reset makes a new context, and the lookup is redone).
int static_scratch(void **ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOBA_ERR_NODEVICE;
  if (dev < 0 || dev >= kMaxDevices) return MOBA_ERR_NODEVICE;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  const CUcontext ctx = current_context();
  if (!g_scratch_ptr[dev] || ctx != g_scratch_ctx[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return MOBA_ERR_LAUNCH;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
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
  // Every argument the three steps check is checked here first, so that a bad call
  // returns before any kernel is enqueued (and before the shared array is touched).
  if (window < 0) return MOBA_ERR_ARG;
  if (!q.ptr || !k.ptr || !v.ptr || !out.ptr || !lse) return MOBA_ERR_ARG;
  const moba_tensor ts[4] = {q, k, v, out};
  for (const moba_tensor &t : ts) {
    if (reinterpret_cast<uintptr_t>(t.ptr) & 15u) return MOBA_ERR_ALIGN;
    if ((t.sb % 8) || (t.sh % 8) || (t.sn % 8) || t.sb < 0 || t.sh < 0 || t.sn < 0)
      return MOBA_ERR_ALIGN;
  }
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return MOBA_ERR_ALIGN;
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
