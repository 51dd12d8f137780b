"""The parity checks themselves reject the mistakes they are meant to catch (CPU)."""
import numpy as np
import pytest

from tests.parity import check_idx, check_out


def _case():
    rows = np.arange(8, dtype=np.int32) * 64 + 63       # rows of blocks 0..7 (B = 64)
    k = 3
    scores = np.full((1, 1, 8, 8), -np.inf)
    rng = np.random.default_rng(0)
    for r in range(8):
        scores[0, 0, r, :r] = rng.normal(size=r) * 10
    idx = np.full((1, 1, 8, k), -1, dtype=np.int32)
    gap = np.full((1, 1, 8), np.inf)
    for r in range(8):
        past = sorted(range(r), key=lambda j: -scores[0, 0, r, j])[:k - 1]
        sel = sorted(past) + [r]
        idx[0, 0, r, :len(sel)] = sel
        if r > k - 1:
            d = np.sort(scores[0, 0, r, :r])[::-1]
            gap[0, 0, r] = d[k - 2] - d[k - 1]
    return idx, gap, scores, rows


def test_check_idx_accepts_the_oracle_itself():
    idx, gap, scores, rows = _case()
    assert check_idx(idx.copy(), idx, gap, scores, rows, 64) == 0


@pytest.mark.parametrize("mutate", ["swap_block", "drop_own", "unsorted", "pad_inside"])
def test_check_idx_rejects_planted_mistakes(mutate):
    idx, gap, scores, rows = _case()
    bad = idx.copy()
    if mutate == "swap_block":
        r = 7
        others = [j for j in range(7) if j not in bad[0, 0, r]]
        bad[0, 0, r, 0] = others[0]
        bad[0, 0, r, :2] = np.sort(bad[0, 0, r, :2])
    elif mutate == "drop_own":
        bad[0, 0, 5, 2] = -1
    elif mutate == "unsorted":
        bad[0, 0, 6, :2] = bad[0, 0, 6, :2][::-1]
    else:
        bad[0, 0, 1, :] = [-1, 0, 1]
    with pytest.raises(AssertionError):
        check_idx(bad, idx, gap, scores, rows, 64)


def test_check_out_tolerances():
    ref = np.random.default_rng(1).normal(size=(1, 2, 16, 8))
    lse = np.zeros((1, 2, 16))
    check_out(ref + 1e-3, lse + 1e-4, ref, lse)
    with pytest.raises(AssertionError):
        check_out(ref + 3e-2, lse, ref, lse)
    with pytest.raises(AssertionError):
        check_out(ref, lse + 2e-3, ref, lse)
