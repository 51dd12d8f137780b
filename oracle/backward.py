"""Backward of MoBA attention for a fixed block choice (small inputs only).

TEST INFRASTRUCTURE ONLY: the reference that a backward kernel will be checked
against.  Nothing in the product path imports it.

[MoBA] §"MoBA와 전체 어텐션의 하이브리드" trains models with MoBA layers, so gradients
flow through MoBA attention.  The gate is parameter-free: it picks blocks by a top-k,
which passes no gradient, so for a given choice MoBA attention is plain softmax
attention over each row's key set J_i (§"MoBA의 구현": the selected blocks' keys up to
the row, unioned with the optional causal window).  With z_ij = scale q_i . k_j on J_i,
p_ij = exp(z_ij - lse_i), o_i = sum_j p_ij v_j and an upstream gradient dO:

    dV_j = sum_i p_ij dO_i
    dp_ij = dO_i . v_j
    D_i  = sum_j p_ij dp_ij  (= dO_i . o_i)
    dz_ij = p_ij (dp_ij - D_i)
    dQ_i = scale sum_j dz_ij k_j
    dK_j = scale sum_i dz_ij q_i

in float64, per (batch, q-head); a KV head's dK and dV sum over the q-heads that
share it (GQA).  Written row by row from those formulas (no dense matrix products
over masked pairs), so that it is independent of the dense-mask formulation it is
pinned against.
"""
from __future__ import annotations

import math

import numpy as np

from . import _check, _load, _ptr, bf16_bits, bf16_to_f64, n_blocks


def key_set(i: int, idx_row, block: int, window: int) -> np.ndarray:
    """J_i: keys j <= i whose block is in idx_row, unioned with i - window < j <= i."""
    keep = set(int(x) for x in idx_row if x >= 0)
    js = [j for j in range(i + 1) if (j // block) in keep or (window > 0 and i - j < window)]
    return np.asarray(js, dtype=np.int64)


def moba_backward(q, k, v, idx: np.ndarray, dout: np.ndarray, *, block: int, window: int = 0,
                  scale: float | None = None):
    """q [b, hq, N, d], k, v [b, hkv, N, d] (bf16 tensors or float arrays), idx int32
    [b, hq, N, topk] (the block choice, -1 padded), dout float [b, hq, N, d].
    Returns (out, lse, dq, dk, dv) in float64."""
    qd = q if isinstance(q, np.ndarray) else bf16_to_f64(q)
    kd = k if isinstance(k, np.ndarray) else bf16_to_f64(k)
    vd = v if isinstance(v, np.ndarray) else bf16_to_f64(v)
    do = np.asarray(dout, dtype=np.float64)
    b, hq, N, d = qd.shape
    hkv = kd.shape[1]
    G = hq // hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    assert idx.shape[:3] == (b, hq, N) and n_blocks(N, block) >= 1
    out = np.zeros((b, hq, N, d))
    lse = np.zeros((b, hq, N))
    dq = np.zeros_like(qd)
    dk = np.zeros_like(kd)
    dv = np.zeros_like(vd)
    for bb in range(b):
        for h in range(hq):
            hk = h // G
            for i in range(N):
                J = key_set(i, idx[bb, h, i], block, window)
                z = scale * (kd[bb, hk, J] @ qd[bb, h, i])
                m = z.max()
                e = np.exp(z - m)
                l = e.sum()
                p = e / l
                lse[bb, h, i] = m + math.log(l)
                o = p @ vd[bb, hk, J]
                out[bb, h, i] = o
                dp = vd[bb, hk, J] @ do[bb, h, i]
                Di = float(do[bb, h, i] @ o)
                dz = p * (dp - Di)
                dq[bb, h, i] = scale * (dz @ kd[bb, hk, J])
                dk[bb, hk, J] += scale * np.outer(dz, qd[bb, h, i])
                dv[bb, hk, J] += np.outer(p, do[bb, h, i])
    return out, lse, dq, dk, dv


def moba_backward_sampled(q, k, v, idx: np.ndarray, dout, *, block: int, rows, keys,
                          window: int = 0, scale: float | None = None):
    """The same gradients from the C oracle (``orc_attention_bwd``, float64, OpenMP) at
    a sample: dQ at the row positions ``rows`` of every q-head, dK and dV at the key
    positions ``keys`` of every KV head (each key's sums run over every row of its
    group that attends it).  ``idx`` int32 [b, hq, N, topk] is the choice of every
    row; q, k, v, dout bf16 tensors.  Returns (dq [b, hq, R, d], dk, dv [b, hkv, K, d])
    in float64."""
    qb, kb, vb, ob = bf16_bits(q), bf16_bits(k), bf16_bits(v), bf16_bits(dout)
    b, hq, N, d = qb.shape
    hkv = kb.shape[1]
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    topk = idx.shape[-1]
    assert idx.shape == (b, hq, N, topk) and ob.shape == qb.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
    kk = np.ascontiguousarray(np.asarray(keys, dtype=np.int32))
    dq = np.empty((b, hq, len(r), d))
    dk = np.empty((b, hkv, len(kk), d))
    dv = np.empty((b, hkv, len(kk), d))
    _check(_load().orc_attention_bwd(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(ob), b, hq, hkv, N, d,
                                     block, topk, _ptr(idx), window, float(scale), _ptr(r), len(r),
                                     _ptr(dq), _ptr(kk), len(kk), _ptr(dk), _ptr(dv)))
    return dq, dk, dv
