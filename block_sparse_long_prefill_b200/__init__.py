"""MoBA block-sparse attention prefill and sliding-window attention prefill on B200.

A thin ctypes binding over ``libmoba.so`` (declared in ``include/moba.h``).  The
functions here only turn torch tensors into pointers, strides and a stream and pass
them through the C ABI: every step of the computation runs in the library's sm_100a
kernels.  There is no CPU fallback; importing fails loudly when the library is
missing.

Method sources (by page title and section):
  [MoBA] "MoBA: 어텐션에 전문가 혼합을 적용해 긴 문맥을 효율적으로 처리하는 블록 어텐션
         (feat. MoonshotAI)", PyTorch KR forum summary of the MoBA paper.
  [SWA]  "SWA + MoE: 어텐션과 희소 전문가", Bit-Axon architecture page.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoba.so")

MOBA_OK = 0
_STATUS = {
    -1: "MOBA_ERR_SHAPE", -2: "MOBA_ERR_DIM", -3: "MOBA_ERR_ALIGN", -4: "MOBA_ERR_ARG",
    -5: "MOBA_ERR_WORKSPACE", -6: "MOBA_ERR_LAUNCH", -7: "MOBA_ERR_DEVICE", -8: "MOBA_ERR_NODEVICE",
    -9: "MOBA_ERR_TOO_LARGE",
}

# Entry points declared in include/moba.h.
ABI_FUNCTIONS = ("moba_workspace_size", "moba_pool_keys", "moba_select_topk", "moba_attn_fwd",
                 "swa_attn_fwd", "moba_workspace_size_chunk", "moba_select_topk_chunk",
                 "moba_attn_fwd_chunk", "swa_attn_fwd_chunk", "moba_select_static",
                 "moba_pool_keys_minmax", "moba_select_topk_minmax",
                 "moba_prefill_static", "moba_bwd_workspace_size", "moba_attn_bwd",
                 "moba_device_status", "moba_debug_set_wait_limit_us",
                 "moba_debug_fault_next_launch", "moba_set_pass_events", "moba_status_string")


class MobaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn}: {_STATUS.get(code, code)} ({status_string(code)})")


class MobaTensor(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("sb", ctypes.c_int64), ("sh", ctypes.c_int64),
                ("sn", ctypes.c_int64)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m block_sparse_long_prefill_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    I, P, S = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
    T = MobaTensor
    lib.moba_workspace_size.argtypes = [I, I, I, I, I, I, I, ctypes.POINTER(S)]
    lib.moba_pool_keys.argtypes = [T, I, I, I, I, I, P, P, P]
    lib.moba_select_topk.argtypes = [T, P, I, I, I, I, I, I, I, P, P, S, P]
    lib.moba_attn_fwd.argtypes = [T, T, T, P, I, I, I, I, I, I, I, I, ctypes.c_float, T, P, P, S, P]
    lib.swa_attn_fwd.argtypes = [T, T, T, I, I, I, I, I, I, ctypes.c_float, T, P, P]
    lib.moba_workspace_size_chunk.argtypes = [I, I, I, I, I, I, I, I, ctypes.POINTER(S)]
    lib.moba_select_topk_chunk.argtypes = [T, P, I, I, I, I, I, I, I, I, P, P, S, P]
    lib.moba_attn_fwd_chunk.argtypes = [T, T, T, P, I, I, I, I, I, I, I, I, I, ctypes.c_float, T, P,
                                        P, S, P]
    lib.swa_attn_fwd_chunk.argtypes = [T, T, T, I, I, I, I, I, I, I, ctypes.c_float, T, P, P]
    lib.moba_select_static.argtypes = [I, I, I, I, I, I, I, I, I, P, P, S, P]
    lib.moba_pool_keys_minmax.argtypes = [T, I, I, I, I, I, P, P]
    lib.moba_select_topk_minmax.argtypes = [T, P, I, I, I, I, I, I, I, I, P, P, S, P]
    lib.moba_prefill_static.argtypes = [T, T, T, I, I, I, I, I, I, I, I, ctypes.c_float, T, P, P]
    lib.moba_bwd_workspace_size.argtypes = [I, I, I, I, I, I, I, ctypes.POINTER(S)]
    lib.moba_attn_bwd.argtypes = [T, T, T, T, T, P, P, P, S, I, I, I, I, I, I, I, I,
                                  ctypes.c_float, T, T, T, P, S, P]
    lib.moba_device_status.argtypes = []
    lib.moba_debug_set_wait_limit_us.argtypes = [I]
    lib.moba_debug_fault_next_launch.argtypes = [I]
    lib.moba_set_pass_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), I]
    lib.moba_status_string.argtypes = [I]
    lib.moba_status_string.restype = ctypes.c_char_p
    for name in ABI_FUNCTIONS[:-1]:
        getattr(lib, name).restype = I
    return lib


_lib = _load()


def library() -> ctypes.CDLL:
    return _lib


def status_string(code: int) -> str:
    return _lib.moba_status_string(int(code)).decode()


def _check(fn: str, rc: int) -> None:
    if rc != MOBA_OK:
        raise MobaError(fn, rc)


def _t(x: torch.Tensor) -> MobaTensor:
    """[b, h, n, d] tensor with a contiguous last dimension -> moba_tensor."""
    if x.dim() != 4:
        raise ValueError("expected a [batch, heads, N, d] tensor")
    if x.stride(3) != 1:
        raise ValueError("the head dimension must be contiguous")
    return MobaTensor(x.data_ptr(), x.stride(0), x.stride(1), x.stride(2))


_BF16, _F32, _I32 = torch.bfloat16, torch.float32, torch.int32


def _device(fn: str, *specs):
    """Checks the tensors a call passes to the library and returns their device.

    Each spec is (name, tensor, dtype, must_be_contiguous, shape or None); None tensors
    are skipped.  Every tensor must be a CUDA tensor of the given dtype, and all of them
    must sit on one device: the library launches on the current device, which the
    wrappers make that device."""
    dev = None
    for name, t, dt, contig, shape in specs:
        if t is None:
            continue
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise ValueError(f"{fn}: {name} must be a CUDA tensor")
        if dt is not None and t.dtype != dt:
            raise ValueError(f"{fn}: {name} must be {dt}, not {t.dtype}")
        if contig and not t.is_contiguous():
            raise ValueError(f"{fn}: {name} must be contiguous")
        if shape is not None and tuple(t.shape) != tuple(shape):
            raise ValueError(f"{fn}: {name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{fn}: every tensor must be on {dev}; {name} is on {t.device}")
    return dev


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def workspace_size(batch, hq, hkv, N, d, block, topk) -> int:
    out = ctypes.c_size_t(0)
    _check("moba_workspace_size",
           _lib.moba_workspace_size(batch, hq, hkv, N, d, block, topk, ctypes.byref(out)))
    return out.value


def moba_pool_keys(k: torch.Tensor, block: int, kbar=None, kbar_split=None, stream=None):
    """[MoBA] §블록 분할과 top-k 게이팅: block means of the keys.  Returns (kbar float32
    [b, hkv, n, d], kbar_split bf16 [b, hkv, 2, n, d])."""
    b, hkv, N, d = k.shape
    n = -(-N // block)  # a partial last block when block does not divide N
    dev = _device("moba_pool_keys", ("k", k, _BF16, False, None),
                  ("kbar", kbar, _F32, True, (b, hkv, n, d)),
                  ("kbar_split", kbar_split, _BF16, True, (b, hkv, 2, n, d)))
    with torch.cuda.device(dev):
        if kbar is None:
            kbar = torch.empty(b, hkv, n, d, dtype=torch.float32, device=dev)
        if kbar_split is None:
            kbar_split = torch.empty(b, hkv, 2, n, d, dtype=torch.bfloat16, device=dev)
        _check("moba_pool_keys", _lib.moba_pool_keys(_t(k), b, hkv, N, d, block, kbar.data_ptr(),
                                                     kbar_split.data_ptr(), _stream(stream)))
    return kbar, kbar_split


def moba_select_topk(q: torch.Tensor, kbar_split: torch.Tensor, block: int, topk: int,
                     workspace: torch.Tensor, idx=None, stream=None):
    """[MoBA] §블록 분할과 top-k 게이팅 + §인과성 보존: per-row block choices (int32
    [b, hq, N, topk], ascending, -1 padded) and the dispatch lists in ``workspace``."""
    b, hq, N, d = q.shape
    return moba_select_topk_chunk(q, kbar_split, block, topk, N, workspace, idx, stream)


def moba_attn_fwd(q, k, v, idx, block: int, topk: int, workspace: torch.Tensor, window: int = 0,
                  scale: float = 0.0, out=None, lse=None, stream=None):
    """[MoBA] §MoBA의 구현: attention over the selected blocks (unioned with the causal
    window).  Returns (out bf16 [b, hq, N, d], lse float32 [b, hq, N])."""
    return moba_attn_fwd_chunk(q, k, v, idx, block, topk, workspace, window, scale, out, lse,
                               stream)


def swa_attn_fwd(q, k, v, window: int, scale: float = 0.0, out=None, lse=None, stream=None):
    """[SWA] §슬라이딩 윈도우 마스크: causal band attention (window >= N is dense causal)."""
    return swa_attn_fwd_chunk(q, k, v, window, scale, out, lse, stream)


def workspace_size_chunk(batch, hq, hkv, N, Nk, d, block, topk) -> int:
    out = ctypes.c_size_t(0)
    _check("moba_workspace_size_chunk",
           _lib.moba_workspace_size_chunk(batch, hq, hkv, N, Nk, d, block, topk, ctypes.byref(out)))
    return out.value


def moba_select_topk_chunk(q, kbar_split: torch.Tensor, block: int, topk: int, kv_len: int,
                           workspace: torch.Tensor, idx=None, stream=None):
    """Block choices for the N query rows of ``q``, which are the last N of ``kv_len``
    positions (pooled keys of all kv_len positions in ``kbar_split``)."""
    b, hq, N, d = q.shape
    hkv = kbar_split.shape[1]
    dev = _device("moba_select_topk", ("q", q, _BF16, False, None),
                  ("kbar_split", kbar_split, _BF16, True, None),
                  ("workspace", workspace, None, True, None),
                  ("idx", idx, _I32, True, (b, hq, N, topk)))
    with torch.cuda.device(dev):
        if idx is None:
            idx = torch.empty(b, hq, N, topk, dtype=torch.int32, device=dev)
        _check("moba_select_topk",
               _lib.moba_select_topk_chunk(_t(q), kbar_split.data_ptr(), b, hq, hkv, N, kv_len, d,
                                           block, topk, idx.data_ptr(), workspace.data_ptr(),
                                           workspace.numel() * workspace.element_size(),
                                           _stream(stream)))
    return idx


def moba_attn_fwd_chunk(q, k, v, idx, block: int, topk: int, workspace: torch.Tensor,
                        window: int = 0, scale: float = 0.0, out=None, lse=None, stream=None):
    """Attention of the N query rows of ``q`` (the last N positions) over the keys and
    values of all k.shape[2] positions.  Returns (out, lse) for the N rows."""
    b, hq, N, d = q.shape
    hkv, Nk = k.shape[1], k.shape[2]
    dev = _device("moba_attn_fwd", ("q", q, _BF16, False, None), ("k", k, _BF16, False, None),
                  ("v", v, _BF16, False, tuple(k.shape)),
                  ("idx", idx, _I32, True, (b, hq, N, topk)),
                  ("workspace", workspace, None, True, None),
                  ("out", out, _BF16, False, tuple(q.shape)),
                  ("lse", lse, _F32, True, (b, hq, N)))
    with torch.cuda.device(dev):
        if out is None:
            out = torch.empty_like(q)
        if lse is None:
            lse = torch.empty(b, hq, N, dtype=torch.float32, device=dev)
        _check("moba_attn_fwd",
               _lib.moba_attn_fwd_chunk(_t(q), _t(k), _t(v), idx.data_ptr(), b, hq, hkv, N, Nk, d,
                                        block, topk, window, float(scale), _t(out), lse.data_ptr(),
                                        workspace.data_ptr(),
                                        workspace.numel() * workspace.element_size(),
                                        _stream(stream)))
    return out, lse


def swa_attn_fwd_chunk(q, k, v, window: int, scale: float = 0.0, out=None, lse=None, stream=None):
    """Sliding-window attention of the last N positions (q) over k.shape[2] positions."""
    b, hq, N, d = q.shape
    hkv, Nk = k.shape[1], k.shape[2]
    dev = _device("swa_attn_fwd", ("q", q, _BF16, False, None), ("k", k, _BF16, False, None),
                  ("v", v, _BF16, False, tuple(k.shape)),
                  ("out", out, _BF16, False, tuple(q.shape)),
                  ("lse", lse, _F32, True, (b, hq, N)))
    with torch.cuda.device(dev):
        if out is None:
            out = torch.empty_like(q)
        if lse is None:
            lse = torch.empty(b, hq, N, dtype=torch.float32, device=dev)
        _check("swa_attn_fwd",
               _lib.swa_attn_fwd_chunk(_t(q), _t(k), _t(v), b, hq, hkv, N, Nk, d, window,
                                       float(scale), _t(out), lse.data_ptr(), _stream(stream)))
    return out, lse


def moba_select_static(batch: int, hq: int, hkv: int, N: int, d: int, block: int, topk: int,
                       sink: int, workspace: torch.Tensor, kv_len=None, idx=None, stream=None,
                       device=None):
    """Static gate in place of moba_select_topk: own block, the first ``sink`` blocks and
    the most recent past blocks (sink = 0: sliding window at block granularity; sink = 1:
    an attention sink).  N query rows, the last N of ``kv_len`` (default N) positions."""
    kv = kv_len or N
    dev = _device("moba_select_static", ("workspace", workspace, None, True, None),
                  ("idx", idx, _I32, True, (batch, hq, N, topk)))
    if device is not None and torch.device(device) != dev and torch.device(device).index is not None:
        raise ValueError(f"moba_select_static: device {device} differs from the workspace's {dev}")
    with torch.cuda.device(dev):
        if idx is None:
            idx = torch.empty(batch, hq, N, topk, dtype=torch.int32, device=dev)
        _check("moba_select_static",
               _lib.moba_select_static(batch, hq, hkv, N, kv, d, block, topk, sink, idx.data_ptr(),
                                       workspace.data_ptr(),
                                       workspace.numel() * workspace.element_size(),
                                       _stream(stream)))
    return idx


def moba_pool_keys_minmax(k: torch.Tensor, block: int, out=None, stream=None):
    """Min/max pooling: bf16 [b, hkv, 2, n, d] with the block maxima (plane 0) and minima
    (plane 1) of the keys."""
    b, hkv, N, d = k.shape
    n = -(-N // block)
    dev = _device("moba_pool_keys_minmax", ("k", k, _BF16, False, None),
                  ("out", out, _BF16, True, (b, hkv, 2, n, d)))
    with torch.cuda.device(dev):
        if out is None:
            out = torch.empty(b, hkv, 2, n, d, dtype=torch.bfloat16, device=dev)
        _check("moba_pool_keys_minmax",
               _lib.moba_pool_keys_minmax(_t(k), b, hkv, N, d, block, out.data_ptr(),
                                          _stream(stream)))
    return out


def moba_select_topk_minmax(q, kminmax: torch.Tensor, block: int, topk: int, kv_len: int,
                            workspace: torch.Tensor, idx=None, stream=None):
    """Selection on min/max pooled blocks (score q+ . kmax + q- . kmin); N query rows,
    the last N of ``kv_len`` positions."""
    b, hq, N, d = q.shape
    hkv = kminmax.shape[1]
    dev = _device("moba_select_topk_minmax", ("q", q, _BF16, False, None),
                  ("kminmax", kminmax, _BF16, True, None),
                  ("workspace", workspace, None, True, None),
                  ("idx", idx, _I32, True, (b, hq, N, topk)))
    with torch.cuda.device(dev):
        if idx is None:
            idx = torch.empty(b, hq, N, topk, dtype=torch.int32, device=dev)
        _check("moba_select_topk_minmax",
               _lib.moba_select_topk_minmax(_t(q), kminmax.data_ptr(), b, hq, hkv, N, kv_len, d,
                                            block, topk, idx.data_ptr(), workspace.data_ptr(),
                                            workspace.numel() * workspace.element_size(),
                                            _stream(stream)))
    return idx


def moba_prefill_chunk(q, k, v, block: int, topk: int, window: int = 0, stream=None):
    """Chunked prefill: q holds the last N of the k.shape[2] positions.  Pools all keys,
    selects and attends for the N rows; returns (out, lse, idx)."""
    b, hq, N, d = q.shape
    hkv, Nk = k.shape[1], k.shape[2]
    dev = _device("moba_prefill_chunk", ("q", q, _BF16, False, None), ("k", k, _BF16, False, None))
    with torch.cuda.device(dev):
        _, ks = moba_pool_keys(k, block, stream=stream)
        ws = torch.empty(workspace_size_chunk(b, hq, hkv, N, Nk, d, block, topk),
                         dtype=torch.uint8, device=dev)
        idx = moba_select_topk_chunk(q, ks, block, topk, Nk, ws, stream=stream)
        out, lse = moba_attn_fwd_chunk(q, k, v, idx, block, topk, ws, window, stream=stream)
    return out, lse, idx


def moba_prefill_static(q, k, v, block: int, topk: int, window: int = 0, scale: float = 0.0,
                        out=None, lse=None, stream=None):
    """The whole prefill with the library's own fixed scratch (no workspace): for
    callers that cannot allocate device memory.  Returns (out, lse)."""
    b, hq, N, d = q.shape
    hkv = k.shape[1]
    dev = _device("moba_prefill_static", ("q", q, _BF16, False, None),
                  ("k", k, _BF16, False, None), ("v", v, _BF16, False, tuple(k.shape)),
                  ("out", out, _BF16, False, tuple(q.shape)),
                  ("lse", lse, _F32, True, (b, hq, N)))
    with torch.cuda.device(dev):
        if out is None:
            out = torch.empty_like(q)
        if lse is None:
            lse = torch.empty(b, hq, N, dtype=torch.float32, device=dev)
        _check("moba_prefill_static",
               _lib.moba_prefill_static(_t(q), _t(k), _t(v), b, hq, hkv, N, d, block, topk,
                                        window, float(scale), _t(out), lse.data_ptr(),
                                        _stream(stream)))
    return out, lse


def bwd_workspace_size(batch, hq, hkv, N, d, block, topk) -> int:
    out = ctypes.c_size_t(0)
    _check("moba_bwd_workspace_size",
           _lib.moba_bwd_workspace_size(batch, hq, hkv, N, d, block, topk, ctypes.byref(out)))
    return out.value


def moba_attn_bwd(q, k, v, out, lse, dout, idx, block: int, topk: int, workspace: torch.Tensor,
                  scale: float = 0.0, dq=None, dk=None, dv=None, bwd_workspace=None, stream=None):
    """[MoBA] §MoBA와 전체 어텐션의 하이브리드 (training through MoBA layers): gradients of
    MoBA attention for the block choice ``idx`` of the forward.  ``workspace`` is the
    one moba_select_topk filled (its dispatch lists are read).  Returns (dq, dk, dv)."""
    b, hq, N, d = q.shape
    hkv = k.shape[1]
    dev = _device("moba_attn_bwd", ("q", q, _BF16, False, None), ("k", k, _BF16, False, None),
                  ("v", v, _BF16, False, tuple(k.shape)), ("out", out, _BF16, False, tuple(q.shape)),
                  ("dout", dout, _BF16, False, tuple(q.shape)),
                  ("lse", lse, _F32, True, (b, hq, N)), ("idx", idx, _I32, True, (b, hq, N, topk)),
                  ("workspace", workspace, None, True, None),
                  ("dq", dq, _BF16, False, tuple(q.shape)), ("dk", dk, _BF16, False, tuple(k.shape)),
                  ("dv", dv, _BF16, False, tuple(k.shape)),
                  ("bwd_workspace", bwd_workspace, None, True, None))
    with torch.cuda.device(dev):
        dq = torch.empty_like(q) if dq is None else dq
        dk = torch.empty_like(k) if dk is None else dk
        dv = torch.empty_like(v) if dv is None else dv
        if bwd_workspace is None:
            bwd_workspace = torch.empty(bwd_workspace_size(b, hq, hkv, N, d, block, topk),
                                        dtype=torch.uint8, device=dev)
        _check("moba_attn_bwd",
               _lib.moba_attn_bwd(_t(q), _t(k), _t(v), _t(out), _t(dout), lse.data_ptr(),
                                  idx.data_ptr(), workspace.data_ptr(),
                                  workspace.numel() * workspace.element_size(), b, hq, hkv, N, d,
                                  block, topk, 0, float(scale), _t(dq), _t(dk), _t(dv),
                                  bwd_workspace.data_ptr(),
                                  bwd_workspace.numel() * bwd_workspace.element_size(),
                                  _stream(stream)))
    return dq, dk, dv


def set_pass_events(events) -> None:
    """Diagnostics: moba_attn_fwd records these torch.cuda.Event objects before its
    first kernel and after each pass (past blocks, own block, merge) of its first query
    chunk; None or [] switches it off.  Each event is recorded once here first so that
    its CUDA handle exists."""
    events = list(events or [])
    for e in events:
        if not e.cuda_event:
            e.record()
    arr = (ctypes.c_void_p * max(1, len(events)))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check("moba_set_pass_events", _lib.moba_set_pass_events(arr, len(events)))


def debug_set_wait_limit_us(microseconds: int) -> None:
    """Test hook: kernel waits give up after this many microseconds (0: the default)."""
    _check("moba_debug_set_wait_limit_us", _lib.moba_debug_set_wait_limit_us(int(microseconds)))


def debug_fault_next_launch(kind: int = 1) -> None:
    """Test hook: the next attention launch leaves one load undone so that a bounded wait
    runs out (MOBA_ERR_DEVICE from device_status()); 0 clears a pending request."""
    _check("moba_debug_fault_next_launch", _lib.moba_debug_fault_next_launch(int(kind)))


def device_status() -> int:
    """Reads and clears the device-side wait-timeout status (synchronises)."""
    return int(_lib.moba_device_status())


class MobaPrefill:
    """The three MoBA calls with their buffers allocated once for a fixed shape.  N query
    rows; with ``kv_len`` (> N) they are the last N of kv_len positions (chunked
    prefill: k and v hold all kv_len positions)."""

    def __init__(self, batch, hq, hkv, N, d, block, topk, window=0, device="cuda", kv_len=None):
        kv = kv_len or N
        self.shape = (batch, hq, hkv, N, d)
        self.kv_len = kv
        self.block, self.topk, self.window = block, topk, window
        n = -(-kv // block)  # a partial last block when block does not divide kv_len
        self.workspace = torch.empty(workspace_size_chunk(batch, hq, hkv, N, kv, d, block, topk),
                                     dtype=torch.uint8, device=device)
        self.kbar = torch.empty(batch, hkv, n, d, dtype=torch.float32, device=device)
        self.kbar_split = torch.empty(batch, hkv, 2, n, d, dtype=torch.bfloat16, device=device)
        self.idx = torch.empty(batch, hq, N, topk, dtype=torch.int32, device=device)
        self.out = torch.empty(batch, hq, N, d, dtype=torch.bfloat16, device=device)
        self.lse = torch.empty(batch, hq, N, dtype=torch.float32, device=device)

    def __call__(self, q, k, v, stream=None):
        moba_pool_keys(k, self.block, self.kbar, self.kbar_split, stream)
        moba_select_topk_chunk(q, self.kbar_split, self.block, self.topk, self.kv_len,
                               self.workspace, self.idx, stream)
        moba_attn_fwd_chunk(q, k, v, self.idx, self.block, self.topk, self.workspace, self.window,
                            out=self.out, lse=self.lse, stream=stream)
        return self.out, self.lse


def moba_prefill(q, k, v, block: int, topk: int, window: int = 0, stream=None):
    """Pool, select and attend in one call; returns (out, lse, idx)."""
    b, hq, N, d = q.shape
    runner = MobaPrefill(b, hq, k.shape[1], N, d, block, topk, window, device=q.device)
    out, lse = runner(q, k, v, stream)
    return out, lse, runner.idx


class MobaPrefillHost:
    """The whole MoBA prefill from pinned host buffers to pinned host buffers, pipelined
    over KV-head groups.  The path needs no exchange between KV heads (a q-head reads its
    own KV head only), so the heads split into ``groups`` independent sub-problems: the
    upload of group g+1, the kernels of group g and the download of group g-1 run on
    three streams at once, through two sets of device buffers.  The results are those of
    MobaPrefill on the whole problem.

    q_h: [batch, hq, N, d], k_h, v_h: [batch, hkv, N, d] bf16, pinned; out_h like q_h and
    lse_h [batch, hq, N] float32, pinned.  Per batch item and group the head range is
    contiguous in host memory."""

    def __init__(self, batch, hq, hkv, N, d, block, topk, window=0, device="cuda", groups=None):
        G = hq // hkv
        if groups is None:
            groups = max(g for g in (1, 2, 4, 8) if hkv % g == 0)
        if hkv % groups:
            raise ValueError("groups must divide hkv")
        self.batch, self.hq, self.hkv, self.N, self.d = batch, hq, hkv, N, d
        self.groups, self.G = groups, G
        self.hkv_g, self.hq_g = hkv // groups, hq // groups
        self.device = torch.device(device)
        self.runners = [MobaPrefill(1, self.hq_g, self.hkv_g, N, d, block, topk, window, device=device)
                        for _ in range(2)]
        self.qd = [torch.empty(1, self.hq_g, N, d, dtype=torch.bfloat16, device=device) for _ in range(2)]
        self.kd = [torch.empty(1, self.hkv_g, N, d, dtype=torch.bfloat16, device=device) for _ in range(2)]
        self.vd = [torch.empty(1, self.hkv_g, N, d, dtype=torch.bfloat16, device=device) for _ in range(2)]
        self.s_h2d = torch.cuda.Stream(device)
        self.s_run = torch.cuda.Stream(device)
        self.s_d2h = torch.cuda.Stream(device)

    def __call__(self, q_h, k_h, v_h, out_h, lse_h):
        cur = torch.cuda.current_stream(self.device)
        for s in (self.s_h2d, self.s_run, self.s_d2h):
            s.wait_stream(cur)
        inputs_free = [None, None]   # the kernels of the slot's last use have read its inputs
        outputs_free = [None, None]  # the download of the slot's last output is done
        units = [(b, g) for b in range(self.batch) for g in range(self.groups)]
        for u, (b, g) in enumerate(units):
            slot = u % 2
            hq0, hk0 = g * self.hq_g, g * self.hkv_g
            with torch.cuda.stream(self.s_h2d):
                if inputs_free[slot] is not None:
                    self.s_h2d.wait_event(inputs_free[slot])
                self.qd[slot].copy_(q_h[b:b + 1, hq0:hq0 + self.hq_g], non_blocking=True)
                self.kd[slot].copy_(k_h[b:b + 1, hk0:hk0 + self.hkv_g], non_blocking=True)
                self.vd[slot].copy_(v_h[b:b + 1, hk0:hk0 + self.hkv_g], non_blocking=True)
                loaded = torch.cuda.Event()
                loaded.record(self.s_h2d)
            with torch.cuda.stream(self.s_run):
                self.s_run.wait_event(loaded)
                if outputs_free[slot] is not None:
                    self.s_run.wait_event(outputs_free[slot])
                self.runners[slot](self.qd[slot], self.kd[slot], self.vd[slot], self.s_run)
                done = torch.cuda.Event()
                done.record(self.s_run)
                inputs_free[slot] = done
            with torch.cuda.stream(self.s_d2h):
                self.s_d2h.wait_event(done)
                r = self.runners[slot]
                out_h[b:b + 1, hq0:hq0 + self.hq_g].copy_(r.out, non_blocking=True)
                lse_h[b:b + 1, hq0:hq0 + self.hq_g].copy_(r.lse, non_blocking=True)
                fetched = torch.cuda.Event()
                fetched.record(self.s_d2h)
                outputs_free[slot] = fetched
        for s in (self.s_h2d, self.s_run, self.s_d2h):
            cur.wait_stream(s)
        return out_h, lse_h


def moba_prefill_varlen(q, k, v, cu_seqlens, block: int, topk: int, window: int = 0,
                        stream=None):
    """MoBA prefill of a batch of sequences of different lengths, packed along the token
    axis (FlashAttention's varlen layout): q [total, hq, d], k, v [total, hkv, d] bf16,
    ``cu_seqlens`` the prefix offsets (batch + 1 ints from 0 to total; a list or a CPU
    tensor).  Sequence s is positions cu_seqlens[s] .. cu_seqlens[s+1] - 1 and is its own
    prefill: its own blocks, its own causal order.  Any lengths (its last block may be
    partial).  Each sequence goes
    through the library's calls as a [1, heads, N_s, d] strided view of the packed
    tensors (no copy); the pooled keys, block choices and workspace are sized for the
    longest sequence and reused in stream order.  Returns (out [total, hq, d] bf16, lse
    [hq, total] float32)."""
    T, hq, d = q.shape
    hkv = k.shape[1]
    offs = [int(x) for x in (cu_seqlens.tolist() if torch.is_tensor(cu_seqlens) else cu_seqlens)]
    if len(offs) < 2 or offs[0] != 0 or offs[-1] != T or any(b < a for a, b in zip(offs, offs[1:])):
        raise ValueError("cu_seqlens must rise from 0 to the token count")
    lens = [b - a for a, b in zip(offs, offs[1:])]
    nmax = max(lens)
    out = torch.empty_like(q)
    lse = torch.empty(hq, T, dtype=torch.float32, device=q.device)
    if nmax == 0:
        return out, lse
    nb = -(-nmax // block)
    dev = q.device
    ws = torch.empty(workspace_size(1, hq, hkv, nmax, d, block, topk), dtype=torch.uint8, device=dev)
    kbar_f = torch.empty(hkv * nb * d, dtype=torch.float32, device=dev)
    ks_f = torch.empty(hkv * 2 * nb * d, dtype=torch.bfloat16, device=dev)
    idx_f = torch.empty(hq * nmax * topk, dtype=torch.int32, device=dev)
    lse_f = torch.empty(hq * nmax, dtype=torch.float32, device=dev)

    def view(t, a, n):  # packed [total, heads, d] -> [1, heads, n, d] over positions a .. a+n-1
        return t[a:a + n].permute(1, 0, 2).unsqueeze(0)

    cur = torch.cuda.current_stream(dev) if stream is None else stream
    for a, n in zip(offs, lens):
        if n == 0:
            continue
        nbs = -(-n // block)
        kbar = kbar_f[:hkv * nbs * d].view(1, hkv, nbs, d)
        ks = ks_f[:hkv * 2 * nbs * d].view(1, hkv, 2, nbs, d)
        idx = idx_f[:hq * n * topk].view(1, hq, n, topk)
        lse_s = lse_f[:hq * n].view(1, hq, n)
        qs, kk, vv, os_ = view(q, a, n), view(k, a, n), view(v, a, n), view(out, a, n)
        moba_pool_keys(kk, block, kbar, ks, stream)
        moba_select_topk(qs, ks, block, topk, ws, idx, stream)
        moba_attn_fwd(qs, kk, vv, idx, block, topk, ws, window, out=os_, lse=lse_s, stream=stream)
        with torch.cuda.stream(cur):
            lse[:, a:a + n].copy_(lse_s[0], non_blocking=True)
    return out, lse
