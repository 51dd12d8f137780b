"""Failure handling of the bounded kernel waits, made to happen on purpose without any
fault: with a short wait limit set, the next attention launch leaves one of its loads
undone (moba_debug_fault_next_launch), so the wait for it runs out.  The launch must
end (its roles stop, drain their copies, free TMEM), moba_device_status() must report
MOBA_ERR_DEVICE, and the next normal call in the same process must give the right
answer."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.parity import check_out

pytestmark = pytest.mark.gpu

MOBA_ERR_DEVICE = -7


def test_a_wait_that_runs_out_reports_an_error_and_the_context_stays_usable():
    import block_sparse_long_prefill_b200 as moba
    w = workloads.small_swa(batch=1, hq=2, hkv=2, seqlen=1024, d=64, window=256)
    q, k, v = workloads.make_inputs(w, 17)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    ref, ref_lse = moba.swa_attn_fwd(qd, kd, vd, w.window)
    torch.cuda.synchronize()
    assert moba.device_status() == 0
    try:
        moba.debug_set_wait_limit_us(2000)           # 2 ms
        moba.debug_fault_next_launch(1)
        out, lse = moba.swa_attn_fwd(qd, kd, vd, w.window)
        assert moba.device_status() == MOBA_ERR_DEVICE
    finally:
        moba.debug_fault_next_launch(0)
        moba.debug_set_wait_limit_us(0)
    assert moba.device_status() == 0                  # read and cleared
    out2, lse2 = moba.swa_attn_fwd(qd, kd, vd, w.window)
    torch.cuda.synchronize()
    assert moba.device_status() == 0
    assert torch.equal(out2, ref) and torch.equal(lse2, ref_lse)
    rows = np.arange(w.seqlen, dtype=np.int32)
    out_o, lse_o = oracle.swa(q, k, v, window=w.window, rows=rows)
    check_out(out2.float().cpu().numpy(), lse2.cpu().numpy(), out_o, lse_o)
