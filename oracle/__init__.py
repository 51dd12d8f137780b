"""fp64 CPU oracle for MoBA block-sparse attention prefill and sliding-window attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg import this package; the CUDA library never does, and
the two share no code.

``moba_oracle.c`` holds the arithmetic (plain loops in double precision); this module
only marshals arrays into it.  ``naive.py`` holds an independent dense-mask
formulation used to pin the gathered one on small inputs.

Sources, cited by page title and section:
  [MoBA] "MoBA: 어텐션에 전문가 혼합을 적용해 긴 문맥을 효율적으로 처리하는 블록 어텐션
         (feat. MoonshotAI)", PyTorch KR forum summary of the MoBA paper.
  [SWA]  "SWA + MoE: 어텐션과 희소 전문가", Bit-Axon architecture page.

Parity pins: every function here is pinned by a ``-m "not gpu"`` test (closed forms,
library special cases, brute force, invariants); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import math

import numpy as np

from . import build as _build

MODE_MOBA = 0
MODE_SWA = 1
MODE_DENSE = 2

_ERRORS = {-1: "bad argument", -2: "idx names a block the row may not see", -3: "out of memory"}

_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(_build.build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.orc_num_threads.restype = I
        lib.orc_pool_keys.argtypes = [P, I, I, I, I, I, P]
        lib.orc_gate_scores.argtypes = [P, P, I, I, I, I, I, I, P, I, P]
        lib.orc_select_topk.argtypes = [P, I, I, I, I, I, P, I, P, P]
        lib.orc_attention.argtypes = [P, P, P, I, I, I, I, I, I, I, I, P, I,
                                      ctypes.c_double, P, I, P, P]
        lib.orc_attention_bwd.argtypes = [P, P, P, P, I, I, I, I, I, I, I, P, I, ctypes.c_double,
                                          P, I, P, P, I, P, P]
        for f in (lib.orc_pool_keys, lib.orc_gate_scores, lib.orc_select_topk, lib.orc_attention,
                  lib.orc_attention_bwd):
            f.restype = I
        _lib = lib
    return _lib


def _check(rc: int) -> None:
    if rc != 0:
        raise ValueError(f"oracle: {_ERRORS.get(rc, rc)}")


def bf16_bits(x) -> np.ndarray:
    """Raw bf16 bit patterns (uint16, C-contiguous) of a torch bf16 tensor or a
    uint16 array."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch
    assert x.dtype == torch.bfloat16, x.dtype
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def bf16_to_f64(x) -> np.ndarray:
    """Exact widening of bf16 values to float64."""
    bits = bf16_bits(x).astype(np.uint32) << 16
    return bits.view(np.float32).astype(np.float64)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _rows(rows, N: int) -> np.ndarray:
    if rows is None:
        return np.arange(N, dtype=np.int32)
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int32))


def num_threads() -> int:
    """OpenMP threads the oracle runs with."""
    return int(_load().orc_num_threads())


def n_blocks(N: int, block: int) -> int:
    """ceil(N / block): when block does not divide N the last block is partial."""
    return -(-N // block)


def pool_keys(k, block: int) -> np.ndarray:
    """[MoBA] §블록 분할과 top-k 게이팅: kbar[b,hk,j] = mean of K[b,hk,j*B:min((j+1)*B,N)]
    (a partial last block: the mean of the keys it holds).
    ``k``: bf16 [b, hkv, N, d].  Returns float64 [b, hkv, ceil(N/B), d]."""
    kb = bf16_bits(k)
    b, hkv, N, d = kb.shape
    if block < 1:
        raise ValueError("block must be positive")
    out = np.empty((b, hkv, n_blocks(N, block), d), dtype=np.float64)
    _check(_load().orc_pool_keys(_ptr(kb), b, hkv, N, d, block, _ptr(out)))
    return out


def gate_scores(q, kbar: np.ndarray, block: int, rows=None) -> np.ndarray:
    """[MoBA] §블록 분할과 top-k 게이팅 and §인과성 보존: unscaled s_j = <q_i, kbar_j> for
    past blocks j < i/B, -inf elsewhere.  Returns float64 [b, hq, len(rows), n]."""
    qb = bf16_bits(q)
    b, hq, N, d = qb.shape
    kbar = np.ascontiguousarray(kbar, dtype=np.float64)
    hkv, n = kbar.shape[1], kbar.shape[2]
    assert kbar.shape == (b, hkv, n_blocks(N, block), d)
    r = _rows(rows, N)
    out = np.empty((b, hq, len(r), n), dtype=np.float64)
    _check(_load().orc_gate_scores(_ptr(qb), _ptr(kbar), b, hq, hkv, N, d, block,
                                   _ptr(r), len(r), _ptr(out)))
    return out


def select_topk(scores: np.ndarray, N: int, block: int, topk: int, rows=None):
    """[MoBA] §블록 분할과 top-k 게이팅 + §인과성 보존: own block forced, k-1 best past
    blocks (ties to the lower index).  Returns (idx int32 [b,hq,R,topk] ascending and
    -1 padded, gap float64 [b,hq,R])."""
    scores = np.ascontiguousarray(scores, dtype=np.float64)
    b, hq, R, n = scores.shape
    r = _rows(rows, N)
    assert len(r) == R and n == n_blocks(N, block)
    idx = np.empty((b, hq, R, topk), dtype=np.int32)
    gap = np.empty((b, hq, R), dtype=np.float64)
    _check(_load().orc_select_topk(_ptr(scores), b, hq, N, block, topk, _ptr(r), R,
                                   _ptr(idx), _ptr(gap)))
    return idx, gap


def pool_minmax(k, block: int):
    """The MoBA page: Quest is MoBA with smaller blocks and a min/max pooled block
    representation.  Element-wise maximum and minimum of the keys of each block
    (positions [j*B, min((j+1)*B, N))).  Returns (kmax, kmin) float64
    [b, hkv, ceil(N/B), d]."""
    kd = bf16_to_f64(k)
    b, hkv, N, d = kd.shape
    n = n_blocks(N, block)
    kmax = np.empty((b, hkv, n, d))
    kmin = np.empty((b, hkv, n, d))
    for j in range(n):
        blk = kd[:, :, j * block:min((j + 1) * block, N)]
        kmax[:, :, j] = blk.max(axis=2)
        kmin[:, :, j] = blk.min(axis=2)
    return kmax, kmin


def minmax_scores(q, kmax: np.ndarray, kmin: np.ndarray, block: int, rows=None) -> np.ndarray:
    """Score of past block j for query row i: the largest inner product q_i can have
    with a key inside block j's min/max box, sum_d max(q_d kmax_jd, q_d kmin_jd) (the
    reading taken of the page's min/max pooled representation); -inf for j >= c, as in
    gate_scores.  Returns float64 [b, hq, len(rows), n]."""
    qd = bf16_to_f64(q)
    b, hq, N, d = qd.shape
    hkv, n = kmax.shape[1], kmax.shape[2]
    G = hq // hkv
    r = _rows(rows, N)
    out = np.full((b, hq, len(r), n), -np.inf)
    for h in range(hq):
        qi = qd[:, h, r]                                     # [b, R, d]
        hi = qi[:, :, None, :] * kmax[:, h // G][:, None]    # [b, R, n, d]
        lo = qi[:, :, None, :] * kmin[:, h // G][:, None]
        s = np.maximum(hi, lo).sum(-1)                       # [b, R, n]
        c = (r // block)[None, :, None]
        out[:, h] = np.where(np.arange(n)[None, None, :] < c, s, -np.inf)
    return out


def select_static(N: int, block: int, topk: int, sink: int, rows=None, batch: int = 1,
                  hq: int = 1) -> np.ndarray:
    """[MoBA] §"MoBA의 구현" preamble on static sparse attention as special cases of MoBA:
    sliding-window attention is MoBA whose gate always picks the most recent blocks, and
    an attention sink is MoBA whose gate always picks the first block together with the
    most recent ones.  Row i (own block c = i / block) keeps its own block and k-1 past
    blocks: the first ``sink`` blocks and the k-1-sink most recent blocks before c (all
    past blocks when c <= k-1).  No score is involved.  Returns int32
    [batch, hq, len(rows), topk], ascending, -1 padded (the same for every batch and
    head)."""
    if not 0 <= sink <= topk - 1:
        raise ValueError("need 0 <= sink <= topk - 1")
    r = _rows(rows, N)
    out = np.full((len(r), topk), -1, dtype=np.int32)
    for t, i in enumerate(r):
        c = int(i) // block
        if c <= topk - 1:
            keep = list(range(c + 1))
        else:
            recent = topk - 1 - sink
            keep = list(range(sink)) + list(range(c - recent, c)) + [c]
        out[t, :len(keep)] = keep
    return np.broadcast_to(out, (batch, hq, len(r), topk)).copy()


def attention(q, k, v, *, mode: int, block: int = 1, topk: int = 1, idx=None,
              window: int = 0, scale: float | None = None, rows=None):
    """Softmax attention over each row's key set (see ``orc_attention``).

    ``q`` bf16 [b,hq,N,d]; ``k``, ``v`` bf16 [b,hkv,N,d]; ``idx`` int32
    [b,hq,len(rows),topk] for MODE_MOBA.  Returns (out float64 [b,hq,R,d],
    lse float64 [b,hq,R])."""
    qb, kb, vb = bf16_bits(q), bf16_bits(k), bf16_bits(v)
    b, hq, N, d = qb.shape
    hkv = kb.shape[1]
    assert kb.shape == (b, hkv, N, d) and vb.shape == kb.shape
    r = _rows(rows, N)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if mode == MODE_MOBA:
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        assert idx.shape == (b, hq, len(r), topk), idx.shape
        idx_p = _ptr(idx)
    else:
        idx_p = None
    out = np.empty((b, hq, len(r), d), dtype=np.float64)
    lse = np.empty((b, hq, len(r)), dtype=np.float64)
    _check(_load().orc_attention(_ptr(qb), _ptr(kb), _ptr(vb), b, hq, hkv, N, d, mode,
                                 block, topk, idx_p, window, float(scale), _ptr(r), len(r),
                                 _ptr(out), _ptr(lse)))
    return out, lse


def moba(q, k, v, *, block: int, topk: int, window: int = 0, scale=None, rows=None):
    """The whole MoBA prefill path ([MoBA] §MoBA의 구현, steps in the page's order):
    pool the keys, score the past blocks, select the top-k, attend over the selected
    keys (unioned with the optional causal window).  Returns a dict with kbar,
    scores, idx, gap, out and lse."""
    kbar = pool_keys(k, block)
    N = bf16_bits(q).shape[2]
    s = gate_scores(q, kbar, block, rows)
    idx, gap = select_topk(s, N, block, topk, rows)
    out, lse = attention(q, k, v, mode=MODE_MOBA, block=block, topk=topk, idx=idx,
                         window=window, scale=scale, rows=rows)
    return {"kbar": kbar, "scores": s, "idx": idx, "gap": gap, "out": out, "lse": lse}


def swa(q, k, v, *, window: int, scale=None, rows=None):
    """[SWA] §어텐션 공식 + §슬라이딩 윈도우 마스크: causal band of width ``window``."""
    return attention(q, k, v, mode=MODE_SWA, window=window, scale=scale, rows=rows)


def dense_causal(q, k, v, *, scale=None, rows=None):
    """[MoBA] §표준 어텐션에서 블록 어텐션으로: full causal attention."""
    return attention(q, k, v, mode=MODE_DENSE, scale=scale, rows=rows)
