"""GPU parity of the MoBA backward (moba_attn_bwd) against the fp64 oracle, through the
C ABI, on seeded synthetic inputs and upstream gradients.

For the block choice the forward made, the gradients are those of softmax attention
over each row's key set ([MoBA] §"MoBA와 전체 어텐션의 하이브리드": models are trained
through MoBA layers; the top-k gate passes no gradient).  The oracle is run with the
GPU's own block choices (checked against the oracle's selection first), like the
forward's parity tests.

Tolerance, from the arithmetic: the kernels multiply bf16 operands (q, k, v, dO, and
the probabilities and dz rounded to bf16 before the products that use them) with fp32
accumulation, and write bf16 results, so each element carries a relative rounding of a
few 2^-9 and sums of many terms average it down.  Each of dQ, dK, dV must be within
relative L2 1e-2 of the oracle and within 2e-2 of it element-wise, measured against the
largest magnitude of that gradient (a popular key sums thousands of rows)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from oracle import backward
from tests.parity import check_idx, rows_of

pytestmark = pytest.mark.gpu

REL_L2 = 1e-2
MAX_REL = 2e-2


def _check_grad(name, got, want):
    got = got.astype(np.float64)
    err = np.abs(got - want)
    scale = max(float(np.abs(want).max()), 1e-30)
    rel_l2 = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30))
    assert np.all(np.isfinite(got)), name
    assert rel_l2 <= REL_L2, (name, rel_l2)
    assert float(err.max()) <= MAX_REL * scale, (name, float(err.max()), scale)
    return {"rel_l2": rel_l2, "max_rel": float(err.max()) / scale}


def run_bwd(w, seed, rows=None, keys=None):
    import block_sparse_long_prefill_b200 as moba
    q, k, v = workloads.make_inputs(w, seed)
    do = workloads.make_grad(w, seed)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    r = moba.MobaPrefill(w.batch, w.hq, w.hkv, w.seqlen, w.d, w.block, w.topk)
    out, lse = r(qd, kd, vd)
    dq, dk, dv = moba.moba_attn_bwd(qd, kd, vd, out, lse, dod, r.idx, w.block, w.topk, r.workspace)
    torch.cuda.synchronize()
    assert moba.device_status() == 0
    N = w.seqlen
    rows = np.arange(N, dtype=np.int32) if rows is None else rows
    keys = np.arange(N, dtype=np.int32) if keys is None else keys
    # The GPU's block choices, checked against the oracle's selection at the rows.
    kbar = oracle.pool_keys(k, w.block)
    scores = oracle.gate_scores(q, kbar, w.block, rows)
    idx_o, gap = oracle.select_topk(scores, N, w.block, w.topk, rows)
    check_idx(rows_of(r.idx, rows), idx_o, gap, scores, rows, w.block)
    idx_g = r.idx.cpu().numpy()
    gq, gk, gv = backward.moba_backward_sampled(q, k, v, idx_g, do, block=w.block, rows=rows,
                                                keys=keys)
    stats = {"dq": _check_grad("dq", rows_of(dq, rows), gq),
             "dk": _check_grad("dk", rows_of(dk, keys), gk),
             "dv": _check_grad("dv", rows_of(dv, keys), gv)}
    return stats, (q, k, v, do), (dq, dk, dv, out)


@pytest.mark.parametrize("name,kw", [
    ("tiny", dict(batch=1, hq=1, hkv=1, seqlen=1024, d=64, block=128, topk=3)),
    ("gqa_d128", dict(batch=1, hq=4, hkv=2, seqlen=2048, d=128, block=256, topk=3)),
    ("any_n_batch2", dict(batch=2, hq=2, hkv=2, seqlen=1000, d=128, block=256, topk=2)),
    ("own_block_only", dict(batch=1, hq=2, hkv=1, seqlen=768, d=64, block=128, topk=1)),
    ("long_list", dict(batch=1, hq=2, hkv=1, seqlen=2048, d=128, block=128, topk=12)),
    ("partial_block_g4", dict(batch=1, hq=4, hkv=1, seqlen=1280, d=64, block=512, topk=2)),
])
def test_moba_backward_every_row_and_key(name, kw):
    w = workloads.small_moba(name=name, **kw)
    stats, _, _ = run_bwd(w, seed=41)
    print(name, stats)


def test_moba_backward_full_size_sampled():
    """The 32K workload (32 / 8 heads, block 512, top-3): dQ at the sampled rows, dK and
    dV at keys of four blocks (first, last and two inner; tile edges included), and the
    softmax sum identities over every key of every KV head."""
    w = workloads.WORKLOADS["gqa32k"]
    rows = workloads.sampled_rows(w, seed=0)
    B = w.block
    keys = []
    for j in (0, 17, 40, w.seqlen // B - 1):
        keys += [j * B, j * B + 1, j * B + 127, j * B + 128, j * B + B - 1]
    keys = np.asarray(sorted(keys), dtype=np.int32)
    stats, (q, k, v, do), (dq, dk, dv, out) = run_bwd(w, seed=0, rows=rows, keys=keys)
    print("gqa32k", stats)
    # sum_j dV_j = sum over the group's rows of dO_i;  sum_j dK_j = 0.
    G = w.hq // w.hkv
    dod = do.cuda().double()
    sdv = dv.double().sum(2)                                        # [b, hkv, d]
    sdo = dod.view(w.batch, w.hkv, G, w.seqlen, w.d).sum((2, 3))
    assert torch.linalg.norm(sdv - sdo) <= 1e-2 * torch.linalg.norm(sdo)
    sdk = dk.double().sum(2)
    assert torch.linalg.norm(sdk) <= 1e-2 * dk.double().abs().sum(2).norm()


def test_moba_backward_is_deterministic():
    import block_sparse_long_prefill_b200 as moba
    w = workloads.small_moba(batch=1, hq=4, hkv=2, seqlen=2048, d=128, block=256, topk=3)
    q, k, v = (t.cuda() for t in workloads.make_inputs(w, 3))
    do = workloads.make_grad(w, 3).cuda()
    r = moba.MobaPrefill(w.batch, w.hq, w.hkv, w.seqlen, w.d, w.block, w.topk)
    out, lse = r(q, k, v)
    g1 = [t.clone() for t in moba.moba_attn_bwd(q, k, v, out, lse, do, r.idx, w.block, w.topk,
                                                r.workspace)]
    g2 = moba.moba_attn_bwd(q, k, v, out, lse, do, r.idx, w.block, w.topk, r.workspace)
    torch.cuda.synchronize()
    assert moba.device_status() == 0
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)
