"""GPU parity of the MoBA path (pool -> select -> attention) against the fp64 oracle,
through the C ABI, on seeded synthetic inputs."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.parity import check_idx, check_out, rows_of

pytestmark = pytest.mark.gpu


def _moba():
    import block_sparse_long_prefill_b200 as moba
    return moba


def run_and_check(w: workloads.Workload, seed=0, rows=None, check_pool=True):
    moba = _moba()
    q, k, v = workloads.make_inputs(w, seed)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    runner = moba.MobaPrefill(w.batch, w.hq, w.hkv, w.seqlen, w.d, w.block, w.topk, w.window)
    out, lse = runner(qd, kd, vd)
    torch.cuda.synchronize()
    assert moba.device_status() == 0
    if rows is None:
        rows = np.arange(w.seqlen, dtype=np.int32)
    kbar_o = oracle.pool_keys(k, w.block)
    if check_pool:
        kb = runner.kbar.cpu().numpy().astype(np.float64)
        scale = np.abs(kbar_o).max()
        assert np.abs(kb - kbar_o).max() <= 1e-5 * scale + 1e-7
        split = runner.kbar_split.float().cpu().numpy().astype(np.float64)
        recon = split[:, :, 0] + split[:, :, 1]
        assert np.abs(recon - kbar_o).max() <= 2e-5 * scale + 1e-7
    scores = oracle.gate_scores(q, kbar_o, w.block, rows)
    idx_o, gap = oracle.select_topk(scores, w.seqlen, w.block, w.topk, rows)
    idx_g = rows_of(runner.idx, rows)
    loose = check_idx(idx_g, idx_o, gap, scores, rows, w.block)
    out_o, lse_o = oracle.attention(q, k, v, mode=oracle.MODE_MOBA, block=w.block, topk=w.topk,
                                    idx=idx_g, window=w.window, rows=rows)
    stats = check_out(rows_of(out, rows), rows_of(lse, rows), out_o, lse_o)
    stats["loose_rows"] = loose
    return stats, runner


@pytest.mark.parametrize("name,kw", [
    ("tiny", dict()),
    ("gqa_small", dict(batch=1, hq=4, hkv=2, seqlen=2048, d=128, block=256, topk=3)),
    ("d80", dict(batch=1, hq=2, hkv=1, seqlen=1024, d=80, block=128, topk=4)),
    ("batch2_g4", dict(batch=2, hq=8, hkv=2, seqlen=1024, d=64, block=128, topk=2)),
    ("k1", dict(batch=1, hq=2, hkv=2, seqlen=1024, d=128, block=128, topk=1)),
    ("k_all", dict(batch=1, hq=2, hkv=1, seqlen=1024, d=64, block=128, topk=8)),
    ("k_over", dict(batch=1, hq=1, hkv=1, seqlen=768, d=64, block=128, topk=20)),
    ("one_block", dict(batch=1, hq=2, hkv=1, seqlen=512, d=128, block=512, topk=3)),
    ("window", dict(batch=1, hq=4, hkv=2, seqlen=2048, d=128, block=512, topk=2, window=300)),
    ("window_wide", dict(batch=1, hq=2, hkv=1, seqlen=1024, d=64, block=128, topk=2, window=700)),
    ("window_dense", dict(batch=1, hq=2, hkv=1, seqlen=1024, d=128, block=256, topk=2, window=4096)),
    ("big_k", dict(batch=1, hq=2, hkv=1, seqlen=4096, d=128, block=128, topk=16)),
    # block does not divide N: the last block is partial (its rows' own block)
    ("partial_block", dict(batch=1, hq=4, hkv=2, seqlen=1280, d=128, block=512, topk=2)),
    ("partial_d80_k3", dict(batch=1, hq=2, hkv=1, seqlen=1664, d=80, block=256, topk=3)),
    ("partial_window", dict(batch=1, hq=2, hkv=1, seqlen=2432, d=64, block=512, topk=2, window=300)),
    ("partial_long_list", dict(batch=1, hq=2, hkv=2, seqlen=4224, d=128, block=256, topk=12)),
    ("partial_k_all", dict(batch=2, hq=2, hkv=1, seqlen=1152, d=64, block=256, topk=8)),
    # N not a multiple of 128: a partial last query tile (and a partial last block)
    ("any_n_1000", dict(batch=1, hq=4, hkv=2, seqlen=1000, d=128, block=256, topk=3)),
    ("any_n_4097_window", dict(batch=1, hq=2, hkv=1, seqlen=4097, d=64, block=512, topk=4,
                               window=300)),
    ("any_n_d80_long_list", dict(batch=1, hq=2, hkv=2, seqlen=3001, d=80, block=128, topk=12)),
    ("any_n_below_one_tile", dict(batch=2, hq=2, hkv=1, seqlen=77, d=64, block=128, topk=2)),
    ("any_n_k1", dict(batch=1, hq=2, hkv=1, seqlen=700, d=128, block=128, topk=1)),
])
def test_moba_small_full_rows(name, kw):
    w = workloads.WORKLOADS["tiny"] if name == "tiny" else workloads.small_moba(name=name, **kw)
    stats, _ = run_and_check(w)
    print(name, stats)


def test_moba_deterministic():
    moba = _moba()
    w = workloads.small_moba(batch=1, hq=4, hkv=2, seqlen=2048, d=128, block=256, topk=3)
    q, k, v = (t.cuda() for t in workloads.make_inputs(w, 3))
    r = moba.MobaPrefill(w.batch, w.hq, w.hkv, w.seqlen, w.d, w.block, w.topk)
    o1, l1 = (t.clone() for t in r(q, k, v))
    i1 = r.idx.clone()
    o2, l2 = r(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(i1, r.idx)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_moba_strided_inputs():
    """q/k/v as [b, N, h, d] storage viewed as [b, h, N, d] (non-contiguous heads)."""
    moba = _moba()
    w = workloads.small_moba(batch=1, hq=4, hkv=2, seqlen=1024, d=128, block=128, topk=3)
    q, k, v = workloads.make_inputs(w, 5)
    qs = q.transpose(1, 2).contiguous().cuda().transpose(1, 2)
    ks = k.transpose(1, 2).contiguous().cuda().transpose(1, 2)
    vs = v.transpose(1, 2).contiguous().cuda().transpose(1, 2)
    out, lse, idx = moba.moba_prefill(qs, ks, vs, w.block, w.topk)
    out2, lse2, idx2 = moba.moba_prefill(q.cuda(), k.cuda(), v.cuda(), w.block, w.topk)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx2)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


@pytest.mark.parametrize("name,kw", [
    # 512 blocks: more pooled keys than the tensor-core gate stages at once, so the
    # selection takes the general (mma.sync) gate kernel (as do rows with > 4 picks).
    ("many_blocks", dict(batch=1, hq=2, hkv=1, seqlen=65536, d=64, block=128, topk=4)),
    # exactly the tensor-core gate's block limit (256 blocks), d = 80, GQA.
    ("blocks256_d80", dict(batch=1, hq=4, hkv=2, seqlen=32768, d=80, block=128, topk=5)),
    # long top-k lists (k - 1 > 4: packed-key lists), 128 / 256 / 64 blocks.
    ("k9_blocks128", dict(batch=1, hq=2, hkv=1, seqlen=16384, d=64, block=128, topk=9)),
    ("k13_blocks256", dict(batch=1, hq=2, hkv=2, seqlen=32768, d=128, block=128, topk=13)),
    ("k32_blocks64", dict(batch=1, hq=2, hkv=1, seqlen=8192, d=128, block=128, topk=32)),
    # packed-key lists of 8 (k - 1 = 5) and 24 (k - 1 = 19) entries
    ("k6_blocks64", dict(batch=1, hq=2, hkv=1, seqlen=8192, d=64, block=128, topk=6)),
    ("k20_blocks64", dict(batch=1, hq=2, hkv=1, seqlen=8192, d=128, block=128, topk=20)),
    # N not a multiple of 128 at 65 and 129 blocks (tensor-core gate, float and packed lists)
    ("any_n_33000", dict(batch=1, hq=4, hkv=1, seqlen=33000, d=128, block=512, topk=3)),
    ("any_n_33000_k13", dict(batch=1, hq=2, hkv=1, seqlen=33000, d=128, block=256, topk=13)),
])
def test_moba_block_count_limits_sampled_rows(name, kw):
    w = workloads.small_moba(name=name, **kw)
    rows = workloads.sampled_rows(w, seed=2)
    stats, _ = run_and_check(w, rows=rows)
    print(name, stats)


@pytest.mark.parametrize("name", ["gqa32k", "hybrid64k", "moba1m"])
def test_moba_full_size_sampled_rows(name):
    """The full-size workloads in the launch configuration the benchmark times
    (moba1m: 1M tokens, 25 query chunks of partials), checked on sampled rows."""
    w = workloads.WORKLOADS[name]
    rows = workloads.sampled_rows(w, seed=0)
    stats, _ = run_and_check(w, rows=rows)
    print(name, stats)


def test_pass_events_time_each_pass():
    """moba_set_pass_events: the events recorded between the passes of moba_attn_fwd
    bracket the passes in order, and recording them changes no result."""
    moba = _moba()
    w = workloads.small_moba(batch=1, hq=4, hkv=2, seqlen=4096, d=128, block=256, topk=3)
    q, k, v = (t.cuda() for t in workloads.make_inputs(w, 4))
    r = moba.MobaPrefill(w.batch, w.hq, w.hkv, w.seqlen, w.d, w.block, w.topk)
    o1, l1 = (t.clone() for t in r(q, k, v))
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    moba.set_pass_events(evs)
    try:
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record()
        o2, l2 = r(q, k, v)
        end.record()
        torch.cuda.synchronize()
    finally:
        moba.set_pass_events(None)
    assert moba.device_status() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    passes = [a.elapsed_time(b) for a, b in zip(evs[:-1], evs[1:])]
    assert all(t > 0 for t in passes), passes
    assert start.elapsed_time(evs[0]) >= 0 and evs[-1].elapsed_time(end) >= 0
    assert sum(passes) <= start.elapsed_time(end) + 1e-3


@pytest.mark.parametrize("name,kw", [
    ("float_list", dict(batch=1, hq=2, hkv=1, seqlen=8192, d=128, block=128, topk=4)),
    ("packed12", dict(batch=1, hq=2, hkv=1, seqlen=8192, d=128, block=128, topk=10)),
    ("packed16_d64", dict(batch=1, hq=2, hkv=2, seqlen=16384, d=64, block=128, topk=14)),
])
def test_moba_tied_blocks_keep_the_lower_block(name, kw):
    """Blocks 2m and 2m+1 hold identical keys, so their gate scores are equal in every
    precision and the top-k boundary often splits a pair.  The choice is then decided
    by the lower block alone: it must equal the oracle's on every row whose boundary
    score is clear (by 1e-3) of every score it does not equal."""
    moba = _moba()
    w = workloads.small_moba(name=name, **kw)
    q, k, v = workloads.make_inputs(w, 7)
    kb = k.view(w.batch, w.hkv, w.seqlen // w.block, w.block, w.d)
    kb[:, :, 1::2] = kb[:, :, 0::2]
    runner = moba.MobaPrefill(w.batch, w.hq, w.hkv, w.seqlen, w.d, w.block, w.topk, w.window)
    runner(q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    assert moba.device_status() == 0
    rows = np.arange(w.seqlen, dtype=np.int32)
    kbar_o = oracle.pool_keys(k, w.block)
    scores = oracle.gate_scores(q, kbar_o, w.block, rows)
    idx_o, _ = oracle.select_topk(scores, w.seqlen, w.block, w.topk, rows)
    idx_g = rows_of(runner.idx, rows)
    npast = w.topk - 1
    checked = split = 0
    for bb in range(w.batch):
        for hh in range(w.hq):
            for r in rows:
                c = int(r) // w.block
                if c <= npast:
                    assert np.array_equal(idx_g[bb, hh, r], idx_o[bb, hh, r])
                    continue
                s = scores[bb, hh, r, :c]
                past = [int(x) for x in idx_o[bb, hh, r] if 0 <= x < c]
                vb = min(s[j] for j in past)
                others = s[s != vb]
                if others.size and np.abs(others - vb).min() <= 1e-3:
                    continue
                checked += 1
                split += int(np.sum(s == vb) > sum(1 for j in past if s[j] == vb))
                assert np.array_equal(idx_g[bb, hh, r], idx_o[bb, hh, r]), (bb, hh, r)
    assert checked > 0.9 * w.batch * w.hq * (w.seqlen - (npast + 1) * w.block)
    assert split > 100  # the boundary splits a tied pair on many rows
    print(name, "checked", checked, "split pairs", split)


def test_moba_score_jump_after_the_first_chunk():
    """Past block 0's first 128 keys score about 0 against every later query row and its
    other keys about 600 (raw dot product): in the gathered pass the first chunk sets the
    row's running maximum, and the next chunk's probabilities against it would be about
    2^76.  That chunk must be redone with its exact maximum (its row sum leaves the bound
    the pass accepts), so the output and lse still match the fp64 oracle."""
    moba = _moba()
    w = workloads.small_moba(name="score_jump", batch=1, hq=2, hkv=1, seqlen=2048, d=128,
                             block=512, topk=2)
    q, k, v = workloads.make_inputs(w, 11)
    u = torch.ones(w.d) / w.d ** 0.5
    kf = 0.05 * k.float()
    kf[0, 0, 128:512] += 24.0 * u
    qf = 0.05 * q.float()
    qf[0, :, 512:] += 25.0 * u
    q, k = qf.to(torch.bfloat16), kf.to(torch.bfloat16)
    runner = moba.MobaPrefill(w.batch, w.hq, w.hkv, w.seqlen, w.d, w.block, w.topk, w.window)
    out, lse = runner(q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    assert moba.device_status() == 0
    rows = np.arange(w.seqlen, dtype=np.int32)
    idx_g = rows_of(runner.idx, rows)
    assert np.all(idx_g[0, :, 512:, 0] == 0)   # every later row picks block 0
    out_o, lse_o = oracle.attention(q, k, v, mode=oracle.MODE_MOBA, block=w.block, topk=w.topk,
                                    idx=idx_g, window=w.window, rows=rows)
    assert lse_o[0, :, 512:].min() > 40.0     # the jump really dominates those rows
    stats = check_out(rows_of(out, rows), rows_of(lse, rows), out_o, lse_o)
    print("score jump", stats)


@pytest.mark.parametrize("batch,hq,hkv,groups", [(1, 8, 4, 4), (2, 4, 2, 2), (1, 2, 1, 1)])
def test_host_pipeline_equals_device_path(batch, hq, hkv, groups):
    """MobaPrefillHost (pinned host buffers, KV-head groups pipelined over three streams)
    gives exactly the device path's results."""
    moba = _moba()
    w = workloads.small_moba(batch=batch, hq=hq, hkv=hkv, seqlen=2048, d=128, block=256, topk=3,
                             window=100)
    q, k, v = workloads.make_inputs(w, 9)
    ref = moba.MobaPrefill(w.batch, w.hq, w.hkv, w.seqlen, w.d, w.block, w.topk, w.window)
    o_ref, l_ref = (t.cpu() for t in ref(q.cuda(), k.cuda(), v.cuda()))
    host = moba.MobaPrefillHost(w.batch, w.hq, w.hkv, w.seqlen, w.d, w.block, w.topk, w.window,
                                groups=groups)
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    out_h = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    lse_h = torch.empty(w.batch, w.hq, w.seqlen, dtype=torch.float32).pin_memory()
    for _ in range(2):
        out_h.zero_()
        host(qh, kh, vh, out_h, lse_h)
        torch.cuda.synchronize()
        assert moba.device_status() == 0
        assert torch.equal(out_h, o_ref) and torch.equal(lse_h, l_ref)
