"""Parity checks of the CUDA path against the fp64 oracle (test helpers).

Tolerances (bf16 inputs, fp32 accumulation):
  - selected blocks: bit-exact wherever the oracle's gap between the (k-1)-th and
    k-th best past score exceeds 1e-3; below that, the two sets may differ only by
    blocks whose oracle scores lie within 1e-3 of the oracle's boundary score;
  - out: max-abs 2e-2 and relative L2 1e-2; lse: max-abs 1e-3 -- both against the
    oracle re-run with the GPU's own block choices, so near-tie rows are checked too.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

GAP_TOL = 1e-3
OUT_ABS = 2e-2
OUT_REL_L2 = 1e-2
LSE_ABS = 1e-3


def check_idx(idx_gpu: np.ndarray, idx_orc: np.ndarray, gap: np.ndarray, scores: np.ndarray,
              rows: np.ndarray, block: int):
    """idx arrays [b, h, R, k]; gap [b, h, R]; scores [b, h, R, n].  Returns the count
    of near-tie rows where the sets differ (allowed)."""
    assert idx_gpu.shape == idx_orc.shape, (idx_gpu.shape, idx_orc.shape)
    b, h, R, k = idx_gpu.shape
    # Structure: ascending, own block last among the valid entries, -1 padding.
    c = (rows // block)[None, None, :]
    valid = idx_gpu >= 0
    nvalid = valid.sum(-1)
    want_n = np.minimum(k, c + 1)
    assert np.array_equal(nvalid, np.broadcast_to(want_n, nvalid.shape)), "wrong number of blocks"
    last = np.take_along_axis(idx_gpu, (nvalid - 1)[..., None], axis=-1)[..., 0]
    assert np.array_equal(last, np.broadcast_to(c, last.shape)), "own block is not kept"
    assert np.all(valid[..., 1:] <= valid[..., :-1]), "padding before a valid entry"
    both = valid[..., 1:] & valid[..., :-1]
    assert np.all(np.diff(idx_gpu, axis=-1)[both] > 0), "not ascending / duplicate"
    same = np.all(idx_gpu == idx_orc, axis=-1)
    clear = gap > GAP_TOL
    bad = clear & ~same
    assert not bad.any(), f"{bad.sum()} rows with a clear gap differ, first at {np.argwhere(bad)[0]}"
    loose = 0
    for pos in np.argwhere(~same):
        bb, hh, rr = pos
        a = set(int(x) for x in idx_gpu[bb, hh, rr] if x >= 0)
        o = set(int(x) for x in idx_orc[bb, hh, rr] if x >= 0)
        cc = int(rows[rr]) // block
        past_o = sorted((x for x in o if x != cc), key=lambda j: -scores[bb, hh, rr, j])
        boundary = scores[bb, hh, rr, past_o[-1]]
        for x in a ^ o:
            assert abs(scores[bb, hh, rr, x] - boundary) <= GAP_TOL + 1e-9, (pos, a, o)
        loose += 1
    return loose


def check_out(out_gpu: np.ndarray, lse_gpu: np.ndarray, out_orc: np.ndarray, lse_orc: np.ndarray):
    out_gpu = out_gpu.astype(np.float64)
    err = np.abs(out_gpu - out_orc)
    max_abs = float(err.max()) if err.size else 0.0
    rel_l2 = float(np.linalg.norm(out_gpu - out_orc) / max(np.linalg.norm(out_orc), 1e-30))
    lse_err = float(np.abs(lse_gpu.astype(np.float64) - lse_orc).max()) if lse_orc.size else 0.0
    assert np.all(np.isfinite(out_gpu)), "non-finite output"
    assert max_abs <= OUT_ABS, f"out max-abs {max_abs}"
    assert rel_l2 <= OUT_REL_L2, f"out rel-L2 {rel_l2}"
    assert lse_err <= LSE_ABS, f"lse max-abs {lse_err}"
    return {"max_abs": max_abs, "rel_l2": rel_l2, "lse_abs": lse_err}


def rows_of(t: torch.Tensor, rows) -> np.ndarray:
    """Rows [b, h, rows, ...] of a device tensor as a host array (bf16 -> float32)."""
    sel = t[:, :, torch.as_tensor(rows, dtype=torch.long, device=t.device)]
    if sel.dtype == torch.bfloat16:
        sel = sel.float()
    return sel.cpu().numpy()
