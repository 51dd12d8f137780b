"""GPU parity of the static gates (attention sink / sliding window as MoBA with a fixed
gate, [MoBA] §"MoBA의 구현" preamble): block choices bit-exact against the oracle's
definition, attention against the oracle over the same choices."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.parity import check_out

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,kw,sink,N", [
    ("recent_blocks", dict(batch=1, hq=4, hkv=2, seqlen=2048, d=128, block=256, topk=3), 0, None),
    ("sink_window_d80", dict(batch=2, hq=2, hkv=1, seqlen=2560, d=80, block=256, topk=4,
                             window=200), 1, None),
    ("sink2_chunk", dict(batch=1, hq=2, hkv=2, seqlen=4096, d=64, block=128, topk=5), 2, 1024),
    ("own_block_only", dict(batch=1, hq=2, hkv=1, seqlen=1024, d=128, block=128, topk=1), 0, None),
    ("sink_partial_block", dict(batch=1, hq=2, hkv=1, seqlen=1664, d=128, block=256, topk=3), 1, None),
    # a chunk at offset 1223: query tiles span two blocks
    ("sink_chunk_offset", dict(batch=1, hq=2, hkv=1, seqlen=3000, d=128, block=256, topk=4), 1, 1777),
])
def test_static_gate_matches_oracle(name, kw, sink, N):
    import block_sparse_long_prefill_b200 as moba
    w = workloads.small_moba(name=name, **kw)
    Nk = w.seqlen
    N = N or Nk
    q_off = Nk - N
    q, k, v = workloads.make_inputs(w, 21)
    qc = q[:, :, q_off:].contiguous().cuda()
    kd, vd = k.cuda(), v.cuda()
    ws = torch.empty(moba.workspace_size_chunk(w.batch, w.hq, w.hkv, N, Nk, w.d, w.block, w.topk),
                     dtype=torch.uint8, device="cuda")
    idx = moba.moba_select_static(w.batch, w.hq, w.hkv, N, w.d, w.block, w.topk, sink, ws, kv_len=Nk)
    out, lse = moba.moba_attn_fwd_chunk(qc, kd, vd, idx, w.block, w.topk, ws, w.window)
    torch.cuda.synchronize()
    assert moba.device_status() == 0
    rows = np.arange(q_off, Nk, dtype=np.int32)
    idx_o = oracle.select_static(Nk, w.block, w.topk, sink, rows, w.batch, w.hq)
    assert np.array_equal(idx.cpu().numpy(), idx_o)
    out_o, lse_o = oracle.attention(q, k, v, mode=oracle.MODE_MOBA, block=w.block, topk=w.topk,
                                    idx=idx_o, window=w.window, rows=rows)
    stats = check_out(out.float().cpu().numpy(), lse.cpu().numpy(), out_o, lse_o)
    print(name, stats)
