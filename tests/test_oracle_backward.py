"""Pins for the MoBA backward oracle (CPU): torch autograd in float64 through the
independent dense-mask formulation, central finite differences, and the forward it
returns against the forward oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import backward, naive


def _inputs(b, hq, hkv, N, d, seed):
    g = torch.Generator().manual_seed(seed)
    mk = lambda h: torch.randn(b, h, N, d, generator=g).to(torch.bfloat16)
    return mk(hq), mk(hkv), mk(hkv), torch.randn(b, hq, N, d, generator=g, dtype=torch.float64)


def _autograd(qd, kd, vd, do, idx, block, window):
    """Dense masked softmax in torch float64 (mask from the same block sets), GQA by
    repeating KV heads; gradients by autograd."""
    b, hq, N, d = qd.shape
    G = hq // kd.shape[1]
    q = torch.tensor(qd, requires_grad=True)
    k = torch.tensor(kd, requires_grad=True)
    v = torch.tensor(vd, requires_grad=True)
    masks = torch.stack([torch.stack([torch.from_numpy(naive.block_mask(
        N, block, naive.block_sets_from_idx(idx[bb, h]), window)) for h in range(hq)])
        for bb in range(b)])
    kr, vr = k.repeat_interleave(G, 1), v.repeat_interleave(G, 1)
    z = (q @ kr.transpose(-1, -2)) / math.sqrt(d)
    z = z.masked_fill(~masks, -math.inf)
    out = torch.softmax(z, -1) @ vr
    out.backward(torch.from_numpy(do))
    return out.detach().numpy(), q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


@pytest.mark.parametrize("b,hq,hkv,N,d,block,topk,window", [
    (1, 2, 1, 96, 8, 16, 3, 0),
    (2, 4, 2, 80, 8, 16, 2, 10),     # GQA, a window, a partial last block
    (1, 1, 1, 64, 4, 8, 20, 0),      # k >= n: dense causal
])
def test_backward_matches_autograd_of_the_dense_mask(b, hq, hkv, N, d, block, topk, window):
    q, k, v, do = _inputs(b, hq, hkv, N, d, seed=N + hq)
    r = oracle.moba(q, k, v, block=block, topk=topk, window=window)
    out, lse, dq, dk, dv = backward.moba_backward(q, k, v, r["idx"], do.numpy(), block=block,
                                                  window=window)
    np.testing.assert_allclose(out, r["out"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, r["lse"], rtol=0, atol=1e-12)
    qd, kd, vd = (oracle.bf16_to_f64(t) for t in (q, k, v))
    ao, adq, adk, adv = _autograd(qd, kd, vd, do.numpy(), r["idx"], block, window)
    np.testing.assert_allclose(out, ao, rtol=0, atol=1e-12)
    for got, want in ((dq, adq), (dk, adk), (dv, adv)):
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-11)


def test_backward_matches_finite_differences():
    """d/dx of sum(dO * out) by central differences on a few coordinates of q, k, v."""
    b, hq, hkv, N, d, block, topk = 1, 2, 1, 40, 4, 8, 2
    q, k, v, do = _inputs(b, hq, hkv, N, d, seed=7)
    idx = oracle.moba(q, k, v, block=block, topk=topk)["idx"]
    qd, kd, vd = (oracle.bf16_to_f64(t) for t in (q, k, v))
    _, _, dq, dk, dv = backward.moba_backward(qd, kd, vd, idx, do.numpy(), block=block)

    def loss(qx, kx, vx):
        o = backward.moba_backward(qx, kx, vx, idx, do.numpy(), block=block)[0]
        return float((o * do.numpy()).sum())

    eps = 1e-6
    rng = np.random.default_rng(0)
    for name, arr, grad in (("q", qd, dq), ("k", kd, dk), ("v", vd, dv)):
        for _ in range(4):
            pos = tuple(int(rng.integers(0, s)) for s in arr.shape)
            plus, minus = arr.copy(), arr.copy()
            plus[pos] += eps
            minus[pos] -= eps
            args = {"q": (qd, kd, vd), "k": (qd, kd, vd), "v": (qd, kd, vd)}[name]
            xp = [plus if a is arr else a for a in args]
            xm = [minus if a is arr else a for a in args]
            fd = (loss(*xp) - loss(*xm)) / (2 * eps)
            assert abs(fd - grad[pos]) <= 1e-6 * max(1.0, abs(fd)), (name, pos, fd, grad[pos])


def _bf16(x):
    return torch.as_tensor(x).to(torch.bfloat16)


@pytest.mark.parametrize("b,hq,hkv,N,d,block,topk,window", [
    (1, 2, 1, 96, 8, 16, 3, 0),
    (2, 4, 2, 80, 8, 16, 2, 10),     # GQA, a window, a partial last block
    (1, 1, 1, 64, 4, 8, 20, 0),      # k >= n: dense causal
    (1, 4, 1, 130, 16, 32, 2, 0),    # G = 4, N not a multiple of the block
])
def test_sampled_backward_equals_the_row_by_row_oracle(b, hq, hkv, N, d, block, topk, window):
    """The C oracle's sampled gradients (dQ at listed rows, dK / dV at listed keys, each
    key summed over every row of its group that attends it) equal the row-by-row
    numpy oracle, which autograd and finite differences pin, at every row and key."""
    q, k, v, _ = _inputs(b, hq, hkv, N, d, seed=3 * N + hq)
    do = _bf16(torch.randn(b, hq, N, d, generator=torch.Generator().manual_seed(N)))
    idx = oracle.moba(q, k, v, block=block, topk=topk, window=window)["idx"]
    _, _, dq, dk, dv = backward.moba_backward(q, k, v, idx, oracle.bf16_to_f64(do), block=block,
                                              window=window)
    allr = np.arange(N, dtype=np.int32)
    sq, sk, sv = backward.moba_backward_sampled(q, k, v, idx, do, block=block, rows=allr,
                                                keys=allr, window=window)
    for got, want in ((sq, dq), (sk, dk), (sv, dv)):
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-10)
    # A sample is the matching slice of the whole.
    rows, keys = np.array([N - 1, 0, N // 2], dtype=np.int32), np.array([3, N - 2], dtype=np.int32)
    tq, tk, tv = backward.moba_backward_sampled(q, k, v, idx, do, block=block, rows=rows, keys=keys,
                                                window=window)
    np.testing.assert_allclose(tq, dq[:, :, rows], rtol=0, atol=1e-10)
    np.testing.assert_allclose(tk, dk[:, :, keys], rtol=0, atol=1e-10)
    np.testing.assert_allclose(tv, dv[:, :, keys], rtol=0, atol=1e-10)


def test_backward_sum_identities():
    """Identities of softmax attention that hold for any key sets, per KV head:
    sum_j dV_j = sum over its q-heads' rows of dO_i (the weights of a row sum to one);
    sum_j dK_j = 0 (the dz of a row sum to zero); sum_j k_j . dK_j = sum_i q_i . dQ_i
    (both are sum_ij dz_ij z_ij); sum_j v_j . dV_j = sum_i dO_i . o_i."""
    b, hq, hkv, N, d, block, topk, window = 1, 4, 2, 72, 8, 16, 2, 12
    q, k, v, do = _inputs(b, hq, hkv, N, d, seed=11)
    idx = oracle.moba(q, k, v, block=block, topk=topk, window=window)["idx"]
    out, _, dq, dk, dv = backward.moba_backward(q, k, v, idx, do.numpy(), block=block, window=window)
    qd, kd, vd = (oracle.bf16_to_f64(t) for t in (q, k, v))
    G = hq // hkv
    dod = do.numpy()
    for hk in range(hkv):
        hs = slice(hk * G, (hk + 1) * G)
        np.testing.assert_allclose(dv[0, hk].sum(0), dod[0, hs].sum((0, 1)), atol=1e-10)
        np.testing.assert_allclose(dk[0, hk].sum(0), 0.0, atol=1e-10)
        np.testing.assert_allclose((kd[0, hk] * dk[0, hk]).sum(), (qd[0, hs] * dq[0, hs]).sum(),
                                   atol=1e-10)
        np.testing.assert_allclose((vd[0, hk] * dv[0, hk]).sum(), (dod[0, hs] * out[0, hs]).sum(),
                                   atol=1e-10)
