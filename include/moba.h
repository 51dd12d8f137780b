/*
 * moba.h -- C ABI of libmoba: MoBA block-sparse attention prefill and sliding-window
 * attention prefill on NVIDIA B200 (sm_100a).
 *
 * The method (cited by page title and section):
 *   [MoBA] "MoBA: 어텐션에 전문가 혼합을 적용해 긴 문맥을 효율적으로 처리하는 블록 어텐션
 *          (feat. MoonshotAI)", PyTorch KR forum summary of the MoBA paper.
 *   [SWA]  "SWA + MoE: 어텐션과 희소 전문가", Bit-Axon architecture page.
 *
 * A MoBA prefill is three calls on one stream, in this order:
 *   moba_pool_keys   -> pooled block keys
 *   moba_select_topk -> per-row block choices (idx) + block-major dispatch lists in
 *                       the workspace
 *   moba_attn_fwd    -> out and per-row log-sum-exp, reading the dispatch lists
 * swa_attn_fwd is independent (the window-only special case).
 *
 * Conventions shared by every call:
 *   - Tensors are device pointers described by moba_tensor: element (b, h, n, 0) sits
 *     at ptr + b*sb + h*sh + n*sn (strides in elements); the head dimension d is
 *     contiguous.  ptr and every stride times the element size must be multiples of
 *     16 bytes.  q is [batch, hq, N, d]; k, v are [batch, hkv, N, d]; out is
 *     [batch, hq, N, d]; all bf16.
 *   - GQA: query head h reads KV head h / (hq / hkv).
 *   - Block j covers key positions [j*block, min((j+1)*block, N)) (0-based; the MoBA
 *     page numbers blocks from 1); there are n = ceil(N / block) blocks.  When block
 *     does not divide N the last block is partial: it holds the N mod block remaining
 *     positions and is pooled over those keys.  block must be a multiple of 128 (the
 *     attention kernels walk keys in chunks of 128, and a chunk must not hold keys of
 *     two blocks); N is free (moba_pool_keys alone takes any block >= 1).
 *   - d must be 64, 80 or 128 (moba_pool_keys alone takes any multiple of 8 up to
 *     256).
 *   - Ownership: the caller allocates every buffer (inputs, outputs, workspace); the
 *     library allocates no device memory and keeps no state between calls (except the
 *     fixed scratch array of moba_prefill_static, below).
 *   - Execution: every call only enqueues kernels on `stream` (a cudaStream_t, 0 for
 *     the legacy default stream) and returns; nothing synchronises.
 *   - Errors: calls return MOBA_OK (0) or a negative MOBA_ERR_* code.  Argument
 *     errors are detected on the host before anything is launched.  Kernel waits are
 *     bounded: a wait that runs out records MOBA_ERR_DEVICE in a device-side status
 *     word that moba_device_status() reads.
 */
#ifndef MOBA_H
#define MOBA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOBA_OK 0
#define MOBA_ERR_SHAPE -1     /* hq % hkv, block % 128, sizes out of range */
#define MOBA_ERR_DIM -2       /* unsupported head dimension */
#define MOBA_ERR_ALIGN -3     /* pointer or stride not 16-byte aligned */
#define MOBA_ERR_ARG -4       /* topk < 1, window < 0, null pointer, ... */
#define MOBA_ERR_WORKSPACE -5 /* workspace missing or too small */
#define MOBA_ERR_LAUNCH -6    /* a CUDA launch or driver call failed */
#define MOBA_ERR_DEVICE -7    /* a kernel wait ran out (see moba_device_status) */
#define MOBA_ERR_NODEVICE -8  /* no sm_100 device is current */
#define MOBA_ERR_TOO_LARGE -9 /* problem needs more than moba_prefill_static's scratch */

typedef struct {
    void *ptr;
    int64_t sb, sh, sn; /* strides in elements for batch, head and position */
} moba_tensor;

/*
 * Bytes of workspace that moba_select_topk and moba_attn_fwd need for this problem.
 * The workspace holds the block-major dispatch lists that moba_select_topk writes
 * and moba_attn_fwd reads, and the per-(row, past block) partial outputs that
 * moba_attn_fwd merges.  Host-only; launches nothing.
 */
int moba_workspace_size(int batch, int hq, int hkv, int N, int d, int block, int topk,
                        size_t *bytes);

/*
 * [MoBA] §"블록 분할과 top-k 게이팅": MeanPool(K[I_j]) for every block j.
 *   k          : bf16 keys [batch, hkv, N, d]
 *   kbar       : float32 out [batch, hkv, n, d], contiguous: the block means
 *                (n = ceil(N / block); a partial last block: the mean of its keys)
 *   kbar_split : bf16 out [batch, hkv, 2, n, d], contiguous: hi = bf16(kbar)
 *                and lo = bf16(kbar - hi), the two bf16 terms the gate multiplies by
 */
int moba_pool_keys(moba_tensor k, int batch, int hkv, int N, int d, int block, float *kbar,
                   void *kbar_split, void *stream);

/*
 * [MoBA] §"블록 분할과 top-k 게이팅" and §"인과성 보존": for every query row i (block
 * c = i / block) score the past blocks j < c with s_j = <q_i, kbar_j> (no scale),
 * keep the own block c and the topk-1 best past blocks (ties to the lower j; all
 * past blocks when c <= topk-1), then build the block-major dispatch lists of
 * §"MoBA의 구현" (steps 1-2: assign queries to KV blocks, regroup by block).
 *   q          : bf16 queries [batch, hq, N, d]
 *   kbar_split : as written by moba_pool_keys
 *   idx        : int32 out [batch, hq, N, topk], contiguous: the kept blocks in
 *                ascending order (the own block last), -1 padded
 *   workspace  : device buffer of at least moba_workspace_size() bytes; receives
 *                the dispatch lists
 */
int moba_select_topk(moba_tensor q, const void *kbar_split, int batch, int hq, int hkv, int N,
                     int d, int block, int topk, int32_t *idx, void *workspace,
                     size_t workspace_bytes, void *stream);

/*
 * [MoBA] §"표준 어텐션에서 블록 어텐션으로" and §"MoBA의 구현": out_i =
 * Softmax(scale q_i K[J_i]^T) V[J_i] with J_i = { j <= i : j / block in idx[i] },
 * unioned with the causal window { j : 0 <= i - j < window } when window > 0.
 * Past blocks are attended block-major (steps 3-4) into partial results that the
 * own-block pass merges by log-sum-exp (step 5).
 *   q, k, v    : bf16 [batch, hq|hkv, N, d], d in {64, 80, 128}
 *   idx        : as written by moba_select_topk for the same q and shapes
 *   workspace  : the same buffer moba_select_topk filled (read, then partly reused)
 *   window     : 0 for none
 *   scale      : logit scale; <= 0 selects 1/sqrt(d)
 *   out        : bf16 out [batch, hq, N, d]
 *   lse        : float32 out [batch, hq, N], contiguous: natural log of the sum of
 *                exp(scale q_i . k_j) over J_i
 */
int moba_attn_fwd(moba_tensor q, moba_tensor k, moba_tensor v, const int32_t *idx, int batch,
                  int hq, int hkv, int N, int d, int block, int topk, int window, float scale,
                  moba_tensor out, float *lse, void *workspace, size_t workspace_bytes,
                  void *stream);

/*
 * [SWA] §"어텐션 공식" and §"슬라이딩 윈도우 마스크": softmax(scale QK^T + M) V with
 * M_ij = 0 iff j <= i and i - j < window, else -inf.  window >= N gives dense causal
 * attention.  Any N >= 1 (no block constraint).
 *   q, k, v, out : bf16 [batch, hq|hkv, N, d], d in {64, 80, 128}
 *   lse          : float32 out [batch, hq, N], contiguous
 */
int swa_attn_fwd(moba_tensor q, moba_tensor k, moba_tensor v, int batch, int hq, int hkv, int N,
                 int d, int window, float scale, moba_tensor out, float *lse, void *stream);

/*
 * Chunked prefill: N query rows that are the last N of Nk positions (query row i sits
 * at position Nk - N + i, as when a long prompt is prefilled chunk by chunk against
 * the keys and values cached so far).  Each row's block choice and attention are those
 * of the same row in a whole prefill of the Nk positions ([MoBA] §"인과성 보존": a row
 * sees only keys at or before its own position, so it does not depend on the other
 * rows).  k and v hold the Nk positions ([batch, hkv, Nk, d]); pool them with
 * moba_pool_keys(k, ..., Nk, ...).  q, idx, out and lse hold the N query rows.
 * Any N and Nk >= N (block as for the whole prefill); Nk = N is the whole prefill, and
 * the calls without _chunk are exactly that.  The workspace is sized by
 * moba_workspace_size_chunk for the same (N, Nk).  swa_attn_fwd_chunk takes any N,
 * Nk >= N and window >= 1.
 */
int moba_workspace_size_chunk(int batch, int hq, int hkv, int N, int Nk, int d, int block,
                              int topk, size_t *bytes);
int moba_select_topk_chunk(moba_tensor q, const void *kbar_split, int batch, int hq, int hkv,
                           int N, int Nk, int d, int block, int topk, int32_t *idx,
                           void *workspace, size_t workspace_bytes, void *stream);
int moba_attn_fwd_chunk(moba_tensor q, moba_tensor k, moba_tensor v, const int32_t *idx,
                        int batch, int hq, int hkv, int N, int Nk, int d, int block, int topk,
                        int window, float scale, moba_tensor out, float *lse, void *workspace,
                        size_t workspace_bytes, void *stream);
int swa_attn_fwd_chunk(moba_tensor q, moba_tensor k, moba_tensor v, int batch, int hq, int hkv,
                       int N, int Nk, int d, int window, float scale, moba_tensor out, float *lse,
                       void *stream);

/*
 * Min/max pooling (the MoBA page: Quest is MoBA with smaller blocks and a min/max
 * pooled block representation).  moba_pool_keys_minmax writes, per block, the
 * element-wise maximum and minimum of its keys as bf16 planes [batch, hkv, 2, n, d]
 * (plane 0 maxima, plane 1 minima; n = ceil(N / block); exact).  N is the key count.
 * moba_select_topk_minmax then scores the past blocks of each query row with
 * s_j = sum_d max(q_d kmax_jd, q_d kmin_jd) -- the largest inner product q can have
 * with a key inside block j's min/max box, computed as q+ . kmax_j + q- . kmin_j -- and
 * keeps the own block and the topk-1 best past blocks like moba_select_topk_chunk
 * (same idx, lists and workspace; N query rows, the last N of Nk positions).
 */
int moba_pool_keys_minmax(moba_tensor k, int batch, int hkv, int N, int d, int block,
                          void *kminmax, void *stream);
int moba_select_topk_minmax(moba_tensor q, const void *kminmax, int batch, int hq, int hkv, int N,
                            int Nk, int d, int block, int topk, int32_t *idx, void *workspace,
                            size_t workspace_bytes, void *stream);

/*
 * Static gates ([MoBA] §"MoBA의 구현" preamble: sliding-window attention is MoBA whose
 * gate always picks the most recent blocks; an attention sink is MoBA whose gate picks
 * the first block together with the most recent ones): in place of moba_select_topk,
 * row i (own block c, at position Nk - N + i) keeps block c, the first `sink` blocks and
 * the topk-1-sink most recent blocks before c (all past blocks when c <= topk-1).  No
 * score, no pooled keys.  Writes idx and the dispatch lists exactly as
 * moba_select_topk_chunk does, for moba_attn_fwd_chunk (Nk = N: the whole prefill).
 *   sink : 0 <= sink <= topk-1 (MOBA_ERR_ARG otherwise)
 */
int moba_select_static(int batch, int hq, int hkv, int N, int Nk, int d, int block, int topk,
                       int sink, int32_t *idx, void *workspace, size_t workspace_bytes,
                       void *stream);

/*
 * The whole MoBA prefill (moba_pool_keys, moba_select_topk, moba_attn_fwd) without any
 * caller-provided workspace, for callers that cannot allocate device memory: plugins
 * whose host framework owns every device allocation and hands them only their inputs
 * and outputs, and runtimes whose memory budget is fixed and fully assigned up front.
 * The paper has no counterpart; it is a deployment convenience.
 *   Arguments as for moba_attn_fwd; out and lse are written, nothing else is.  Every
 *   argument is checked before anything is enqueued.
 *   Scratch: one 32 MiB device array inside the library (held, on each GPU that runs
 *   this call, until the process exits).  Problems whose pooled keys, block choices
 *   and workspace (moba_workspace_size) need more return MOBA_ERR_TOO_LARGE.
 *   Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 *   The first call on a device (that device current) looks up the array's device
 *   address and caches it per device and CUDA context, so a call after a
 *   cudaDeviceReset looks it up again; make that first call before any stream
 *   capture.  All calls share the array and it keeps the last call's contents (the
 *   counters that must start at zero are cleared by every call): calls that overlap
 *   on the GPU (other streams, other host threads) race and must be serialised by the
 *   caller.
 */
int moba_prefill_static(moba_tensor q, moba_tensor k, moba_tensor v, int batch, int hq, int hkv,
                        int N, int d, int block, int topk, int window, float scale,
                        moba_tensor out, float *lse, void *stream);

/*
 * Backward of MoBA attention (training: [MoBA] §"MoBA와 전체 어텐션의 하이브리드" trains
 * models whose layers are MoBA attention).  The gate is a parameter-free top-k and passes
 * no gradient, so for the block choice idx of the forward the layer is softmax attention
 * over each row's key set J_i, and with z_ij = scale q_i.k_j, p_ij = exp(z_ij - lse_i):
 *     D_i = dO_i . o_i,  dz_ij = p_ij (dO_i . v_j - D_i),
 *     dQ_i = scale sum_j dz_ij k_j,  dK_j = scale sum_i dz_ij q_i,  dV_j = sum_i p_ij dO_i
 * (a KV head's dK and dV sum over the q-heads that read it).  Whole prefills (Nk = N)
 * without a window; d in {64, 128}; any N (block a multiple of 128).
 *   q, k, v, out, lse, idx : as given to / returned by moba_attn_fwd (out bf16, lse the
 *                            natural-log row statistic)
 *   workspace   : the buffer moba_select_topk filled for this idx (its dispatch lists
 *                 are read; moba_attn_fwd leaves them intact)
 *   dout        : bf16 upstream gradient [batch, hq, N, d]
 *   dq          : bf16 out [batch, hq, N, d];  dk, dv : bf16 out [batch, hkv, N, d]
 *   bwd_workspace : device buffer of at least moba_bwd_workspace_size() bytes (row
 *                 statistics and fp32 dQ partials, one per row and block slot)
 * Errors: MOBA_ERR_ARG for window != 0, MOBA_ERR_DIM for d = 80, MOBA_ERR_WORKSPACE for a
 * missing or short buffer; the rest as for moba_attn_fwd.  Four kernels, no atomics:
 * results are deterministic.
 */
int moba_bwd_workspace_size(int batch, int hq, int hkv, int N, int d, int block, int topk,
                            size_t *bytes);
int moba_attn_bwd(moba_tensor q, moba_tensor k, moba_tensor v, moba_tensor out, moba_tensor dout,
                  const float *lse, const int32_t *idx, const void *workspace,
                  size_t workspace_bytes, int batch, int hq, int hkv, int N, int d, int block,
                  int topk, int window, float scale, moba_tensor dq, moba_tensor dk,
                  moba_tensor dv, void *bwd_workspace, size_t bwd_workspace_bytes, void *stream);

/*
 * Reads and clears the device-side status word that bounded kernel waits write
 * (MOBA_OK or MOBA_ERR_DEVICE) on the current device.  Synchronises the device.
 */
int moba_device_status(void);

/*
 * Test hooks for the bounded waits (they change nothing unless called; both
 * synchronise the current device first).
 * moba_debug_set_wait_limit_us: every kernel wait that has not completed after this
 *   many microseconds gives up (MOBA_ERR_DEVICE); 0 restores the default of 2 s.
 * moba_debug_fault_next_launch(1): the next attention launch (moba_attn_fwd's passes or
 *   swa_attn_fwd) leaves the first V chunk of its first CTA unloaded, so that a wait
 *   runs out on purpose: the launch ends through the bounded-wait path (its roles stop,
 *   copies in flight are drained, TMEM is freed) and moba_device_status() then reports
 *   MOBA_ERR_DEVICE.  One shot: the launch that takes the flag clears it; 0 clears it.
 *   Nothing faults or traps, and the context stays usable.
 * Return MOBA_OK, MOBA_ERR_ARG for a value out of range, MOBA_ERR_LAUNCH when a CUDA call
 * fails.  The paper has no counterpart; these exist to test failure handling.
 */
int moba_debug_set_wait_limit_us(int microseconds);
int moba_debug_fault_next_launch(int kind);

/* Static description of a status code. */
const char *moba_status_string(int status);

/* Diagnostics for benchmarks: per-pass timing of moba_attn_fwd.  `events` holds
 * `count` cudaEvent_t handles created by the caller (count 0 or events NULL switches
 * this off).  While set, every moba_attn_fwd call records, on its stream, events[0]
 * before its first kernel and events[k] after its k-th kernel, as far as count
 * allows.  The kernels run per query chunk, in launch order: the past-block pass, the
 * own-block pass and the merge pass of chunk 0, then those of chunk 1, and so on (with
 * topk = 1 only the own-block pass runs).  The library keeps the handles, not the
 * events: they must outlive their use.  A process-wide setting, not synchronised
 * between host threads.
 * Returns MOBA_OK, or MOBA_ERR_ARG when count is outside [0, 1024]. */
int moba_set_pass_events(void *const *events, int count);

#ifdef __cplusplus
}
#endif

#endif /* MOBA_H */
