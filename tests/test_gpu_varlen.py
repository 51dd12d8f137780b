"""Varlen batches: sequences of different lengths packed along the token axis, each its
own MoBA prefill.  The packed call must give, for every sequence, exactly what the
sequence gives on its own (bit for bit), and that agrees with the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.parity import check_idx, check_out

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("lens,hq,hkv,d,block,topk,window", [
    ([1024, 384, 2176], 4, 2, 128, 256, 3, 0),     # 2176: a partial last block
    ([640, 128, 1536, 896], 2, 1, 64, 128, 4, 200),
    ([1280], 2, 2, 80, 512, 2, 0),
    # lengths that are not multiples of 128, a one-token sequence among them
    ([1000, 1, 2049], 4, 2, 128, 256, 3, 0),
    ([333, 1500, 77], 2, 1, 64, 128, 4, 100),
])
def test_varlen_equals_each_sequence_alone(lens, hq, hkv, d, block, topk, window):
    import block_sparse_long_prefill_b200 as moba
    offs = np.concatenate([[0], np.cumsum(lens)]).tolist()
    T = offs[-1]
    g = torch.Generator().manual_seed(5)
    q = torch.randn(T, hq, d, generator=g).to(torch.bfloat16)
    nb = -(-T // 128)
    k = (torch.randn(T, hkv, d, generator=g)
         + 0.5 * torch.randn(nb, 1, d, generator=g).repeat_interleave(128, 0)[:T]).to(torch.bfloat16)
    v = torch.randn(T, hkv, d, generator=g).to(torch.bfloat16)
    out, lse = moba.moba_prefill_varlen(q.cuda(), k.cuda(), v.cuda(), offs, block, topk, window)
    torch.cuda.synchronize()
    assert moba.device_status() == 0
    for a, n in zip(offs, lens):
        qs, ks, vs = (t[a:a + n].permute(1, 0, 2).unsqueeze(0).contiguous() for t in (q, k, v))
        o1, l1, i1 = moba.moba_prefill(qs.cuda(), ks.cuda(), vs.cuda(), block, topk, window)
        torch.cuda.synchronize()
        assert torch.equal(out[a:a + n].permute(1, 0, 2).unsqueeze(0), o1)
        assert torch.equal(lse[:, a:a + n].unsqueeze(0), l1)
        rows = np.arange(n, dtype=np.int32)
        scores = oracle.gate_scores(qs, oracle.pool_keys(ks, block), block, rows)
        idx_o, gap = oracle.select_topk(scores, n, block, topk, rows)
        idx_g = i1.cpu().numpy()
        check_idx(idx_g, idx_o, gap, scores, rows, block)
        out_o, lse_o = oracle.attention(qs, ks, vs, mode=oracle.MODE_MOBA, block=block, topk=topk,
                                        idx=idx_g, window=window, rows=rows)
        print(n, check_out(o1.float().cpu().numpy(), l1.cpu().numpy(), out_o, lse_o))
