"""The benchmark's work accounting (CPU): the attended-pair counts that every TFLOP/s
figure divides by must equal a brute-force count of the key sets the oracle's dense-mask
formulation attends, for whole prefills, chunks (queries that are the last positions),
windows and partial last blocks; the per-pass split must add up to the whole."""
import dataclasses

import numpy as np
import pytest
import torch

import bench
import oracle
import workloads
from oracle import naive


def _brute_pairs(w, idx_rows):
    """Sum over rows (positions q_off .. seqlen-1), heads and batch of |J_i| from the
    dense N x N visibility mask built from each row's block set."""
    N = w.seqlen
    total = 0
    for b in range(w.batch):
        for h in range(w.hq):
            sets = [set()] * w.q_off + [set(int(x) for x in r if x >= 0) for r in idx_rows[b, h]]
            mask = naive.block_mask(N, w.block, sets, w.window)
            total += int(mask[w.q_off:].sum())
    return total


@pytest.mark.parametrize("kw", [
    dict(seqlen=1024, block=128, topk=3),
    dict(seqlen=1024, block=128, topk=3, window=200),
    dict(seqlen=1152, block=256, topk=2, window=300),      # a partial last block
    dict(seqlen=2048, block=256, topk=4, q_len=640),       # a chunk starting mid-block
    dict(seqlen=1024, block=128, topk=20),                 # k >= n: dense causal
])
def test_attended_pairs_equal_the_dense_mask_count(kw):
    w = workloads.small_moba(batch=1, hq=2, hkv=1, d=64, **{k: v for k, v in kw.items() if k != "q_len"})
    if "q_len" in kw:
        w = dataclasses.replace(w, q_len=kw["q_len"])
    q, k, v = workloads.make_inputs(w, 3)
    rows = np.arange(w.q_off, w.seqlen, dtype=np.int32)
    s = oracle.gate_scores(q, oracle.pool_keys(k, w.block), w.block, rows)
    idx, _ = oracle.select_topk(s, w.seqlen, w.block, w.topk, rows)
    got = bench.attended_pairs_moba(torch.from_numpy(idx), w)
    assert got == _brute_pairs(w, idx)
    if w.topk >= w.nblocks and w.window == 0:
        assert got == bench.dense_pairs(w)
    # The per-pass split (summed over all query chunks) covers the same work.
    work = bench.pass_work_moba(torch.from_numpy(idx), w)
    assert work["past_block_pass"] + work["own_block_pass"] == 4.0 * w.d * got


def test_swa_pairs_closed_form():
    w = workloads.small_swa(batch=1, hq=3, hkv=3, seqlen=777, d=80, window=100)
    i = np.arange(777)
    j = np.arange(777)
    band = (j[None, :] <= i[:, None]) & (i[:, None] - j[None, :] < 100)
    assert bench.attended_pairs_swa(w) == int(band.sum()) * 3


def test_layout_chunks_and_launch_counts_follow_the_workspace_rule():
    """The benchmark's launch count per step: the selection launches plus three passes
    per query chunk, with the chunk count of the 4 GiB partials rule."""
    w = workloads.WORKLOADS["moba1m"]
    per_row = w.topk * (w.d * 2 + 4) * w.batch * w.hq
    rows = ((4 << 30) // per_row) // 128 * 128
    assert bench.layout_chunks(w) == -(-w.nq // rows) > 1
    assert bench.launches_per_step(w) == 3 + 3 * bench.layout_chunks(w)
    assert bench.layout_chunks(workloads.WORKLOADS["gqa32k"]) == 1
    assert bench.launches_per_step(workloads.WORKLOADS["gqa32k"]) == 6
    assert bench.launches_per_step(workloads.WORKLOADS["swa16k"]) == 1
