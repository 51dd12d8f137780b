"""GPU parity of chunked prefill: the N query rows are the last N of Nk positions
(q_off = Nk - N), attending to keys and values of all Nk positions.  A row's block
choice and attention depend only on keys at or before its own position ([MoBA]
§"인과성 보존"), so the reference is the fp64 oracle run on the whole Nk-position
sequence at rows q_off .. Nk - 1."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.parity import check_idx, check_out

pytestmark = pytest.mark.gpu


def _moba():
    import block_sparse_long_prefill_b200 as moba
    return moba


@pytest.mark.parametrize("name,kw,N", [
    ("chunk_gqa", dict(batch=1, hq=4, hkv=2, seqlen=4096, d=128, block=512, topk=3), 1024),
    # the chunk starts mid-block (q_off = 2432 = 4 blocks + 384 rows), no GQA
    ("chunk_mid_block", dict(batch=1, hq=2, hkv=1, seqlen=3072, d=64, block=512, topk=2), 640),
    ("chunk_window_d80", dict(batch=2, hq=2, hkv=1, seqlen=2560, d=80, block=256, topk=3,
                              window=300), 1024),
    ("chunk_long_list", dict(batch=1, hq=2, hkv=2, seqlen=8192, d=128, block=256, topk=12), 2048),
    # a partial last block (Nk = 8.5 blocks) and an offset
    ("chunk_partial_block", dict(batch=1, hq=4, hkv=1, seqlen=2176, d=64, block=256, topk=3), 896),
    # one row tile
    ("chunk_one_tile", dict(batch=1, hq=2, hkv=1, seqlen=2048, d=128, block=128, topk=4), 128),
    # offsets that are not multiples of 128: query tiles span two blocks
    ("chunk_offset_2500", dict(batch=1, hq=4, hkv=2, seqlen=6000, d=128, block=512, topk=3), 3500),
    ("chunk_offset_window", dict(batch=1, hq=2, hkv=1, seqlen=3333, d=64, block=256, topk=4,
                                 window=300), 1111),
    ("chunk_offset_long_list_d80", dict(batch=1, hq=2, hkv=2, seqlen=5000, d=80, block=128,
                                        topk=10), 2345),
])
def test_moba_chunk_matches_whole_sequence_rows(name, kw, N):
    moba = _moba()
    w = workloads.small_moba(name=name, **kw)
    Nk = w.seqlen
    q_off = Nk - N
    q, k, v = workloads.make_inputs(w, 11)
    qc = q[:, :, q_off:].contiguous()
    out, lse, idx = moba.moba_prefill_chunk(qc.cuda(), k.cuda(), v.cuda(), w.block, w.topk, w.window)
    torch.cuda.synchronize()
    assert moba.device_status() == 0
    rows = np.arange(q_off, Nk, dtype=np.int32)
    kbar_o = oracle.pool_keys(k, w.block)
    scores = oracle.gate_scores(q, kbar_o, w.block, rows)
    idx_o, gap = oracle.select_topk(scores, Nk, w.block, w.topk, rows)
    idx_g = idx.cpu().numpy()
    loose = check_idx(idx_g, idx_o, gap, scores, rows, w.block)
    out_o, lse_o = oracle.attention(q, k, v, mode=oracle.MODE_MOBA, block=w.block, topk=w.topk,
                                    idx=idx_g, window=w.window, rows=rows)
    stats = check_out(out.float().cpu().numpy(), lse.cpu().numpy(), out_o, lse_o)
    stats["loose_rows"] = loose
    print(name, stats)


def test_moba_chunk_of_the_whole_sequence_equals_the_whole_prefill():
    """Nk = N: the chunk entry points are the whole prefill (bit for bit)."""
    moba = _moba()
    w = workloads.small_moba(batch=1, hq=4, hkv=2, seqlen=2048, d=128, block=256, topk=3)
    q, k, v = (t.cuda() for t in workloads.make_inputs(w, 12))
    o1, l1, i1 = moba.moba_prefill_chunk(q, k, v, w.block, w.topk)
    o2, l2, i2 = moba.moba_prefill(q, k, v, w.block, w.topk)
    torch.cuda.synchronize()
    assert torch.equal(i1, i2) and torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("Nk,N,window,d", [(3000, 1080, 500, 80), (4096, 1024, 4096, 128),
                                           (2304, 256, 64, 64), (3000, 1100, 700, 80),
                                           (2049, 1000, 300, 64)])
def test_swa_chunk_matches_whole_sequence_rows(Nk, N, window, d):
    moba = _moba()
    w = workloads.small_swa(batch=1, hq=4, hkv=2, seqlen=Nk, d=d, window=window)
    q, k, v = workloads.make_inputs(w, 13)
    q_off = Nk - N
    out, lse = moba.swa_attn_fwd_chunk(q[:, :, q_off:].contiguous().cuda(), k.cuda(), v.cuda(), window)
    torch.cuda.synchronize()
    assert moba.device_status() == 0
    rows = np.arange(q_off, Nk, dtype=np.int32)
    out_o, lse_o = oracle.swa(q, k, v, window=window, rows=rows)
    stats = check_out(out.float().cpu().numpy(), lse.cpu().numpy(), out_o, lse_o)
    print("swa_chunk", Nk, N, window, stats)
