"""GPU parity of min/max pooled selection (the MoBA page: Quest is MoBA with smaller
blocks and min/max pooling): the pooled planes bit-exact, block choices against the
oracle's min/max scores (exact where the boundary gap exceeds 1e-3), and attention
over the GPU's choices against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.parity import check_idx, check_out

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,kw,N", [
    ("small_blocks", dict(batch=1, hq=4, hkv=2, seqlen=2048, d=128, block=128, topk=4), None),
    ("d64_window", dict(batch=2, hq=2, hkv=1, seqlen=1536, d=64, block=128, topk=3, window=200), None),
    ("d80_chunk_partial", dict(batch=1, hq=2, hkv=1, seqlen=2176, d=80, block=256, topk=3), 1024),
    ("chunk_offset_any_n", dict(batch=1, hq=2, hkv=1, seqlen=2500, d=128, block=256, topk=3), 1003),
])
def test_minmax_selection_matches_oracle(name, kw, N):
    import block_sparse_long_prefill_b200 as moba
    w = workloads.small_moba(name=name, **kw)
    Nk = w.seqlen
    N = N or Nk
    q_off = Nk - N
    q, k, v = workloads.make_inputs(w, 31)
    qc = q[:, :, q_off:].contiguous().cuda()
    kd, vd = k.cuda(), v.cuda()
    planes = moba.moba_pool_keys_minmax(kd, w.block)
    ws = torch.empty(moba.workspace_size_chunk(w.batch, w.hq, w.hkv, N, Nk, w.d, w.block, w.topk),
                     dtype=torch.uint8, device="cuda")
    idx = moba.moba_select_topk_minmax(qc, planes, w.block, w.topk, Nk, ws)
    out, lse = moba.moba_attn_fwd_chunk(qc, kd, vd, idx, w.block, w.topk, ws, w.window)
    torch.cuda.synchronize()
    assert moba.device_status() == 0
    kmax, kmin = oracle.pool_minmax(k, w.block)
    pl = planes.float().cpu().numpy().astype(np.float64)
    assert np.array_equal(pl[:, :, 0], kmax) and np.array_equal(pl[:, :, 1], kmin)
    rows = np.arange(q_off, Nk, dtype=np.int32)
    scores = oracle.minmax_scores(q, kmax, kmin, w.block, rows)
    idx_o, gap = oracle.select_topk(scores, Nk, w.block, w.topk, rows)
    idx_g = idx.cpu().numpy()
    loose = check_idx(idx_g, idx_o, gap, scores, rows, w.block)
    out_o, lse_o = oracle.attention(q, k, v, mode=oracle.MODE_MOBA, block=w.block, topk=w.topk,
                                    idx=idx_g, window=w.window, rows=rows)
    stats = check_out(out.float().cpu().numpy(), lse.cpu().numpy(), out_o, lse_o)
    stats["loose_rows"] = loose
    print(name, stats)
