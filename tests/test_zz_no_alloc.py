"""moba_prefill_static: the whole MoBA prefill for callers that cannot allocate device
memory (plugins whose host framework owns every device allocation, runtimes whose
memory budget is fixed and fully assigned up front).  It keeps its scratch in one fixed
device array inside the library, so the caller passes only q, k, v and the outputs.
Its results must equal the allocating entry points' (moba_pool_keys ->
moba_select_topk -> moba_attn_fwd) within the parity tolerance, on consecutive calls
(the shared array keeps the previous call's contents, and the selection step must
clear what has to start at zero)."""
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

OUT_ABS = 2e-2
LSE_ABS = 1e-3


def _case(seed, **kw):
    w = workloads.small_moba(**kw)
    q, k, v = (t.cuda() for t in workloads.make_inputs(w, seed))
    return w, q, k, v


def test_static_scratch_matches_the_allocating_path_twice():
    import block_sparse_long_prefill_b200 as moba
    torch.cuda.set_device(0)
    cases = [
        _case(0, batch=1, hq=4, hkv=2, seqlen=2048, d=128, block=256, topk=3),
        _case(1, batch=2, hq=2, hkv=1, seqlen=1024, d=64, block=128, topk=4, window=200),
        # a partial last block (block does not divide N)
        _case(3, batch=1, hq=2, hkv=1, seqlen=1408, d=128, block=512, topk=2),
    ]
    for w, q, k, v in cases:
        ref = moba.MobaPrefill(w.batch, w.hq, w.hkv, w.seqlen, w.d, w.block, w.topk, w.window)
        out_ref, lse_ref = (t.clone() for t in ref(q, k, v))
        for _ in range(2):
            out, lse = moba.moba_prefill_static(q, k, v, w.block, w.topk, w.window)
            torch.cuda.synchronize()
            assert moba.device_status() == 0
            assert (out.float() - out_ref.float()).abs().max().item() <= OUT_ABS
            assert (lse - lse_ref).abs().max().item() <= LSE_ABS


def test_static_scratch_rejects_problems_beyond_its_size():
    import block_sparse_long_prefill_b200 as moba
    w, q, k, v = _case(2, batch=1, hq=32, hkv=8, seqlen=8192, d=128, block=512, topk=8)
    with pytest.raises(moba.MobaError) as e:
        moba.moba_prefill_static(q, k, v, w.block, w.topk)
    assert e.value.code == -9
