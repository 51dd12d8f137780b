"""Dense-mask formulation of MoBA / SWA attention (small inputs only).

TEST INFRASTRUCTURE ONLY.  This is the "naive" reading of the method: build the full
N x N additive mask (0 where a key is visible, -inf elsewhere) from each row's block
set and run one dense masked softmax in float64, as the MoBA page describes its
attention-mask based reference implementation (§"MoBA 설치 및 사용법" / the
``moba_naive`` paragraph of §"효율성과 확장성").  It is written independently of the
gathered C oracle, with numpy only, and pins it on small inputs.
"""
from __future__ import annotations

import math

import numpy as np


def block_mask(N: int, block: int, block_sets, window: int = 0) -> np.ndarray:
    """Boolean visibility mask [N, N] for one (batch, head).

    ``block_sets[i]`` is the set of blocks row i attends (its own block included).
    A key j is visible iff j <= i and (j's block is in the set, or 0 <= i-j < window).
    """
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    causal = j <= i
    member = np.zeros((N, N), dtype=bool)
    for row in range(N):
        for blk in block_sets[row]:
            member[row, blk * block:(blk + 1) * block] = True
    if window > 0:
        member |= (i - j) < window
    return causal & member


def masked_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, mask: np.ndarray,
                     scale: float | None = None):
    """Dense masked softmax attention for one head: q, k, v float64 [N, d], mask bool
    [N, N].  Returns (out [N, d], lse [N])."""
    d = q.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    z = scale * (q @ k.T)
    z = np.where(mask, z, -np.inf)
    m = z.max(axis=1, keepdims=True)
    p = np.exp(z - m)
    l = p.sum(axis=1, keepdims=True)
    return (p @ v) / l, (m + np.log(l))[:, 0]


def block_sets_from_idx(idx_row_major: np.ndarray):
    """Turn idx [N, topk] (-1 padded) into a list of block sets."""
    return [set(int(x) for x in row if x >= 0) for row in idx_row_major]
