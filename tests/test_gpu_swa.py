"""GPU parity of sliding-window (and dense causal) attention against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.parity import check_out, rows_of

pytestmark = pytest.mark.gpu


def _run(w, seed=0, rows=None):
    import block_sparse_long_prefill_b200 as moba
    q, k, v = workloads.make_inputs(w, seed)
    out, lse = moba.swa_attn_fwd(q.cuda(), k.cuda(), v.cuda(), w.window)
    torch.cuda.synchronize()
    assert moba.device_status() == 0
    if rows is None:
        rows = np.arange(w.seqlen, dtype=np.int32)
    out_o, lse_o = oracle.swa(q, k, v, window=w.window, rows=rows)
    return check_out(rows_of(out, rows), rows_of(lse, rows), out_o, lse_o)


@pytest.mark.parametrize("d", [64, 80, 128])
@pytest.mark.parametrize("N,window", [(1000, 300), (1024, 128), (777, 1), (640, 5000), (2048, 513)])
def test_swa_small(d, N, window):
    w = workloads.small_swa(batch=1, hq=2, hkv=2, seqlen=N, d=d, window=window)
    print(d, N, window, _run(w))


def test_swa_gqa_batch():
    w = workloads.Workload("swa_gqa", 2, 4, 2, 900, 128, window=200)
    print(_run(w))


def test_swa16k_sampled_rows():
    w = workloads.WORKLOADS["swa16k"]
    rows = workloads.sampled_rows(w, 0)
    print(_run(w, rows=rows))


def test_dense_causal_via_full_window():
    w = workloads.small_swa(batch=1, hq=2, hkv=2, seqlen=1536, d=128, window=1536)
    print(_run(w))
