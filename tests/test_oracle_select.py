"""Pins for the oracle's pooling and block selection (CPU only).

Each test checks the oracle against something other than itself: a library routine,
brute-force enumeration, a closed form or an invariant the pages fix.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (scale * torch.randn(shape, generator=g)).to(torch.bfloat16)


# --------------------------------------------------------------------------- pool

def test_pool_constant_block_is_exact():
    b, hkv, N, d, B = 1, 2, 64, 8, 16
    vals = torch.tensor([0.5, -1.25, 3.0, 0.0078125], dtype=torch.float32)
    k = torch.empty(b, hkv, N, d)
    for j in range(N // B):
        k[:, :, j * B:(j + 1) * B, :] = vals[j]
    kbar = oracle.pool_keys(k.to(torch.bfloat16), B)
    for j in range(N // B):
        assert np.all(kbar[:, :, j, :] == float(vals[j]))


@pytest.mark.parametrize("B", [1, 2, 8, 128])
def test_pool_matches_numpy_mean(B):
    k = _bf16((2, 3, 256, 16), seed=1)
    kbar = oracle.pool_keys(k, B)
    ref = oracle.bf16_to_f64(k).reshape(2, 3, 256 // B, B, 16).mean(axis=3)
    np.testing.assert_allclose(kbar, ref, rtol=0, atol=1e-15)


def test_pool_partial_last_block_is_the_mean_of_its_keys():
    """N = 100, B = 64: block 1 holds positions 64..99 and is pooled over those 36
    keys only (numpy mean of the slice); a constant partial block pools exactly."""
    k = _bf16((2, 2, 100, 16), seed=2)
    kbar = oracle.pool_keys(k, 64)
    assert kbar.shape == (2, 2, 2, 16)
    kd = oracle.bf16_to_f64(k)
    np.testing.assert_allclose(kbar[:, :, 0], kd[:, :, :64].mean(axis=2), rtol=0, atol=1e-15)
    np.testing.assert_allclose(kbar[:, :, 1], kd[:, :, 64:].mean(axis=2), rtol=0, atol=1e-15)
    kc = torch.zeros(1, 1, 100, 8)
    kc[:, :, 64:] = 0.375
    assert np.all(oracle.pool_keys(kc.to(torch.bfloat16), 64)[0, 0, 1] == 0.375)


# ---------------------------------------------------------------------- selection

def _brute_force_sets(s_row, c, k):
    """Own block plus the (k-1)-subset of past blocks with the largest score sum."""
    past = list(range(c))
    if c <= k - 1:
        return set(past) | {c}
    best, best_sum = None, -math.inf
    for comb in itertools.combinations(past, k - 1):
        tot = sum(s_row[j] for j in comb)
        if tot > best_sum:
            best, best_sum = comb, tot
    return set(best) | {c}


@pytest.mark.parametrize("B", [1, 2, 8, 128])
def test_select_matches_brute_force(B):
    n = 8 if B < 128 else 6
    N = n * B
    d = 8
    q = _bf16((1, 2, N, d), seed=10 + B)
    k = _bf16((1, 1, N, d), seed=20 + B)
    kbar = oracle.pool_keys(k, B)
    # Every row of every block, all k in 1..n.
    rows = np.arange(N, dtype=np.int32)
    s = oracle.gate_scores(q, kbar, B, rows)
    # Independent check of the scores: numpy inner products with the pooled keys.
    qd = oracle.bf16_to_f64(q)
    for h in range(2):
        full = qd[0, h] @ kbar[0, 0].T
        for i in range(0, N, max(1, N // 37)):
            c = i // B
            np.testing.assert_allclose(s[0, h, i, :c], full[i, :c], rtol=1e-13, atol=1e-13)
            assert np.all(np.isneginf(s[0, h, i, c:]))
    for k_ in range(1, n + 1):
        idx, gap = oracle.select_topk(s, N, B, k_, rows)
        for h in range(2):
            for i in rows:
                c = i // B
                got = [x for x in idx[0, h, i] if x >= 0]
                assert got == sorted(got)
                assert len(got) == min(k_, c + 1)
                assert list(idx[0, h, i, len(got):]) == [-1] * (k_ - len(got))
                assert set(got) == _brute_force_sets(s[0, h, i], c, k_), (B, k_, h, i)


def test_select_token_level_when_block_is_one():
    """B = 1: the gate score of block j is <q_i, k_j> itself; the row keeps its own
    token and the k-1 past tokens with the largest raw inner products."""
    N, d, k_ = 64, 16, 5
    q = _bf16((1, 1, N, d), 3)
    k = _bf16((1, 1, N, d), 4)
    s = oracle.gate_scores(q, oracle.pool_keys(k, 1), 1)
    idx, _ = oracle.select_topk(s, N, 1, k_)
    qd, kd = oracle.bf16_to_f64(q)[0, 0], oracle.bf16_to_f64(k)[0, 0]
    for i in range(N):
        raw = qd[i] @ kd[:i].T
        order = sorted(range(i), key=lambda j: (-raw[j], j))
        want = sorted(order[:k_ - 1] + [i])
        assert [x for x in idx[0, 0, i] if x >= 0] == want


def test_future_blocks_never_chosen_and_own_block_forced():
    """A future block with a huge pooled key is never selected; the own block is
    kept even when its pooled key scores lowest (MoBA §인과성 보존)."""
    N, B, d = 512, 64, 4
    n = N // B
    q = torch.ones(1, 1, N, d)
    k = torch.zeros(1, 1, N, d)
    for j in range(n):
        k[0, 0, j * B:(j + 1) * B, :] = float(j % 3) - 1.0
    k[0, 0, 7 * B:, :] = 50.0   # last block scores highest of all
    k[0, 0, 3 * B:4 * B, :] = -50.0  # block 3 scores lowest
    q, k = q.to(torch.bfloat16), k.to(torch.bfloat16)
    s = oracle.gate_scores(q, oracle.pool_keys(k, B), B)
    idx, _ = oracle.select_topk(s, N, B, 2)
    for i in range(N):
        c = i // B
        got = [x for x in idx[0, 0, i] if x >= 0]
        assert c in got
        assert all(x <= c for x in got)
    rows_in_3 = range(3 * B, 4 * B)
    for i in rows_in_3:
        assert 3 in idx[0, 0, i]


def test_ties_go_to_the_lower_block():
    N, B, d = 256, 32, 4
    q = torch.ones(1, 1, N, d, dtype=torch.bfloat16)
    k = torch.ones(1, 1, N, d, dtype=torch.bfloat16)  # every pooled key identical
    s = oracle.gate_scores(q, oracle.pool_keys(k, B), B)
    idx, gap = oracle.select_topk(s, N, B, 3)
    for i in range(2 * B, N):
        c = i // B
        assert list(idx[0, 0, i]) == [0, 1, c]
        # With c <= k-1 every past block is kept and no choice is made.
        assert gap[0, 0, i] == (0.0 if c > 2 else np.inf)


def test_gap_is_kth_minus_k_plus_first_past_score():
    N, B, d = 1024, 64, 16
    q = _bf16((1, 1, N, d), 7)
    k = _bf16((1, 1, N, d), 8)
    s = oracle.gate_scores(q, oracle.pool_keys(k, B), B)
    for k_ in (1, 2, 4):
        _, gap = oracle.select_topk(s, N, B, k_)
        for i in range(0, N, 13):
            c = i // B
            if c <= k_ - 1 or k_ == 1:
                assert gap[0, 0, i] == math.inf
            else:
                desc = np.sort(s[0, 0, i, :c])[::-1]
                assert gap[0, 0, i] == desc[k_ - 2] - desc[k_ - 1]


def test_attended_key_count_closed_form():
    """|J_i| = (i mod B) + 1 + min(k-1, c) * B (q = 0 makes lse = ln|J|)."""
    N, B, d, k_ = 1024, 64, 8, 4
    q = _bf16((1, 1, N, d), 11)
    k = _bf16((1, 1, N, d), 12)
    v = _bf16((1, 1, N, d), 13)
    s = oracle.gate_scores(q, oracle.pool_keys(k, B), B)
    idx, _ = oracle.select_topk(s, N, B, k_)
    zero_q = torch.zeros_like(q)
    _, lse = oracle.attention(zero_q, k, v, mode=oracle.MODE_MOBA, block=B, topk=k_, idx=idx)
    i = np.arange(N)
    want = (i % B) + 1 + np.minimum(k_ - 1, i // B) * B
    np.testing.assert_allclose(lse[0, 0], np.log(want), rtol=0, atol=1e-12)


def test_sparsity_matches_the_pages_arithmetic():
    with open(os.path.join(GOLDEN, "sparsity.json")) as f:
        cases = json.load(f)["cases"]
    d = 2
    for case in cases:
        N, B, k_ = case["N"], case["B"], case["k"]
        q = _bf16((1, 1, N, d), 5)
        k = _bf16((1, 1, N, d), 6)
        v = torch.zeros_like(k)
        last = np.array([N - 1], dtype=np.int32)
        s = oracle.gate_scores(q, oracle.pool_keys(k, B), B, last)
        idx, _ = oracle.select_topk(s, N, B, k_, last)
        _, lse = oracle.attention(torch.zeros_like(q), k, v, mode=oracle.MODE_MOBA, block=B,
                                  topk=k_, idx=idx, rows=last)
        nkeys = round(math.exp(lse[0, 0, 0]))
        assert nkeys == k_ * B
        assert 1.0 - nkeys / N == pytest.approx(case["sparsity"], abs=0)


def test_selection_invariant_under_a_common_key_shift():
    """Adding one vector u to every key shifts every gate score of a row by <q, u>:
    the chosen blocks do not change.  Values on a coarse grid keep k + u exact in
    bf16."""
    N, B, d = 512, 32, 8
    g = torch.Generator().manual_seed(9)
    q = (torch.randint(-16, 17, (1, 2, N, d), generator=g) / 8.0).to(torch.bfloat16)
    k = (torch.randint(-16, 17, (1, 1, N, d), generator=g) / 8.0).to(torch.bfloat16)
    u = (torch.randint(-8, 9, (d,), generator=g) / 2.0)
    k2 = (k.float() + u).to(torch.bfloat16)
    assert torch.equal(k2.float(), k.float() + u)
    s1 = oracle.gate_scores(q, oracle.pool_keys(k, B), B)
    s2 = oracle.gate_scores(q, oracle.pool_keys(k2, B), B)
    i1, g1 = oracle.select_topk(s1, N, B, 4)
    i2, g2 = oracle.select_topk(s2, N, B, 4)
    assert np.array_equal(i1, i2)
    finite = np.isfinite(g1)
    np.testing.assert_allclose(g1[finite], g2[finite], atol=1e-12)


# ------------------------------------------------------------- partial last block

@pytest.mark.parametrize("B", [2, 8, 128])
def test_select_with_partial_last_block_matches_brute_force(B):
    """N = 6B + B/2: the last block is partial.  It is only ever a row's own block, so
    every past block is full, and the choice equals brute force for all k."""
    n_full = 6
    N = n_full * B + B // 2
    d = 8
    q = _bf16((1, 2, N, d), seed=40 + B)
    k = _bf16((1, 1, N, d), seed=50 + B)
    kbar = oracle.pool_keys(k, B)
    assert kbar.shape[2] == n_full + 1
    rows = np.arange(N, dtype=np.int32)
    s = oracle.gate_scores(q, kbar, B, rows)
    for k_ in range(1, n_full + 2):
        idx, _ = oracle.select_topk(s, N, B, k_, rows)
        for h in range(2):
            for i in rows:
                c = i // B
                got = [x for x in idx[0, h, i] if x >= 0]
                assert len(got) == min(k_, c + 1)
                assert set(got) == _brute_force_sets(s[0, h, i], c, k_), (B, k_, h, i)


def test_rows_before_a_partial_block_ignore_it():
    """Causality: rows in the full blocks of an N = 5B + 40 problem choose exactly as
    in the problem cut at 5B (they never see the partial block)."""
    B, d, k_ = 64, 16, 3
    N = 5 * B + 40
    q = _bf16((1, 2, N, d), seed=61)
    k = _bf16((1, 1, N, d), seed=62)
    full = oracle.select_topk(oracle.gate_scores(q, oracle.pool_keys(k, B), B), N, B, k_)
    Nc = 5 * B
    cut = oracle.select_topk(oracle.gate_scores(q[:, :, :Nc], oracle.pool_keys(k[:, :, :Nc], B), B),
                             Nc, B, k_)
    assert np.array_equal(full[0][:, :, :Nc], cut[0])
    assert np.array_equal(full[1][:, :, :Nc], cut[1])


# ------------------------------------------------------------------- static gates

@pytest.mark.parametrize("sink", [0, 1, 2])
def test_static_gate_is_moba_top_k_on_scores_that_rank_those_blocks(sink):
    """The MoBA page: sliding-window attention is MoBA whose gate always picks the most
    recent blocks, an attention sink MoBA whose gate also picks the first block.  With
    pooled keys whose scores rise with the block index (and the first `sink` blocks
    above all of them), the score-based top-k picks exactly the static rule's blocks."""
    B, n, d, k_ = 16, 12, 4, 5
    N = n * B
    q = torch.ones(1, 1, N, d)
    k = torch.zeros(1, 1, N, d)
    for j in range(n):
        k[0, 0, j * B:(j + 1) * B, :] = 100.0 + 4.0 * j if j >= sink else 1000.0 + j
    q, k = q.to(torch.bfloat16), k.to(torch.bfloat16)
    s = oracle.gate_scores(q, oracle.pool_keys(k, B), B)
    idx, _ = oracle.select_topk(s, N, B, k_)
    assert np.array_equal(idx, oracle.select_static(N, B, k_, sink))


def test_static_gate_definition():
    """Closed form of a few rows: B = 4, k = 4, sink = 1."""
    idx = oracle.select_static(40, 4, 4, 1, rows=[0, 5, 9, 13, 39])
    assert idx[0, 0].tolist() == [[0, -1, -1, -1], [0, 1, -1, -1], [0, 1, 2, -1], [0, 1, 2, 3],
                                  [0, 7, 8, 9]]
    with pytest.raises(ValueError):
        oracle.select_static(40, 4, 4, 4)


# ----------------------------------------------------------------- min/max pooling

def test_minmax_pool_and_scores_bound_every_key():
    """The min/max block score is an upper bound of q . k for every key k of the block,
    reached when one key holds every coordinate's extreme of q's sign pattern; with one
    key per block it is q . k itself (B = 1: token-level, like the mean)."""
    B, N, d = 8, 64, 16
    q = _bf16((1, 2, N, d), seed=71)
    k = _bf16((1, 1, N, d), seed=72)
    kmax, kmin = oracle.pool_minmax(k, B)
    kd = oracle.bf16_to_f64(k)[0, 0]
    np.testing.assert_array_equal(kmax[0, 0], kd.reshape(N // B, B, d).max(axis=1))
    np.testing.assert_array_equal(kmin[0, 0], kd.reshape(N // B, B, d).min(axis=1))
    s = oracle.minmax_scores(q, kmax, kmin, B)
    qd = oracle.bf16_to_f64(q)[0]
    for h in range(2):
        for i in range(0, N, 5):
            c = i // B
            for j in range(c):
                dots = qd[h, i] @ kd[j * B:(j + 1) * B].T
                assert s[0, h, i, j] >= dots.max() - 1e-12
                # the box corner that matches q's signs attains the score
                corner = np.where(qd[h, i] >= 0, kmax[0, 0, j], kmin[0, 0, j])
                assert abs(s[0, h, i, j] - qd[h, i] @ corner) <= 1e-12
            assert np.all(np.isneginf(s[0, h, i, c:]))
    s1 = oracle.minmax_scores(q, *oracle.pool_minmax(k, 1), 1)
    ref = oracle.gate_scores(q, oracle.pool_keys(k, 1), 1)
    np.testing.assert_allclose(s1, ref, rtol=0, atol=1e-12)


def test_minmax_pool_partial_block():
    k = _bf16((1, 1, 100, 8), seed=73)
    kmax, kmin = oracle.pool_minmax(k, 64)
    kd = oracle.bf16_to_f64(k)[0, 0]
    np.testing.assert_array_equal(kmax[0, 0, 1], kd[64:].max(axis=0))
    np.testing.assert_array_equal(kmin[0, 0, 1], kd[64:].min(axis=0))
