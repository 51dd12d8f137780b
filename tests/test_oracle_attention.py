"""Pins for the oracle's attention (CPU only): library special cases (torch SDPA in
float64), closed forms, an independent dense-mask formulation, and invariants."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import naive


def _bf16(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


def _qkv(b, hq, hkv, N, d, seed=0):
    return _bf16((b, hq, N, d), seed), _bf16((b, hkv, N, d), seed + 1), _bf16((b, hkv, N, d), seed + 2)


def _sdpa(q, k, v, mask=None, causal=False):
    """torch's scaled_dot_product_attention in float64 on the CPU, GQA by repeating
    KV heads.  Returns (out, lse) with lse from the same masked logits."""
    qd, kd, vd = (torch.from_numpy(oracle.bf16_to_f64(t)) for t in (q, k, v))
    G = qd.shape[1] // kd.shape[1]
    kd, vd = kd.repeat_interleave(G, dim=1), vd.repeat_interleave(G, dim=1)
    out = F.scaled_dot_product_attention(qd, kd, vd, attn_mask=mask, is_causal=causal)
    z = (qd @ kd.transpose(-1, -2)) / math.sqrt(qd.shape[-1])
    N = qd.shape[2]
    if causal:
        z = z.masked_fill(~torch.ones(N, N, dtype=torch.bool).tril(), -math.inf)
    if mask is not None:
        z = z.masked_fill(~mask, -math.inf)
    return out.numpy(), torch.logsumexp(z, dim=-1).numpy()


def _moba(q, k, v, B, topk, window=0):
    return oracle.moba(q, k, v, block=B, topk=topk, window=window)


TOL = dict(rtol=0, atol=1e-12)


def test_dense_mode_matches_sdpa_causal():
    q, k, v = _qkv(2, 4, 2, 300, 32)
    out, lse = oracle.dense_causal(q, k, v)
    ref, rlse = _sdpa(q, k, v, causal=True)
    np.testing.assert_allclose(out, ref, **TOL)
    np.testing.assert_allclose(lse, rlse, **TOL)


@pytest.mark.parametrize("B,topk,window", [(64, 8, 0), (64, 100, 0), (512, 1, 0), (64, 1, 512),
                                           (64, 2, 10_000)])
def test_moba_reduces_to_dense_causal(B, topk, window):
    """top-k >= n, or B = N, or a window >= N: every causal key is attended."""
    q, k, v = _qkv(1, 2, 1, 512, 16, seed=3)
    r = _moba(q, k, v, B, topk, window)
    ref, rlse = _sdpa(q, k, v, causal=True)
    np.testing.assert_allclose(r["out"], ref, **TOL)
    np.testing.assert_allclose(r["lse"], rlse, **TOL)


def test_topk_one_is_block_diagonal_causal():
    q, k, v = _qkv(1, 2, 2, 256, 16, seed=5)
    B = 64
    r = _moba(q, k, v, B, 1)
    for j in range(256 // B):
        sl = slice(j * B, (j + 1) * B)
        ref, rlse = _sdpa(q[:, :, sl], k[:, :, sl], v[:, :, sl], causal=True)
        np.testing.assert_allclose(r["out"][:, :, sl], ref, **TOL)
        np.testing.assert_allclose(r["lse"][:, :, sl], rlse, **TOL)


def test_window_one_closed_form():
    """w = 1 and no block: each row sees only itself, out_i = v_i, lse_i = scale q_i.k_i."""
    q, k, v = _qkv(1, 1, 1, 100, 8, seed=6)
    out, lse = oracle.swa(q, k, v, window=1)
    qd, kd, vd = (oracle.bf16_to_f64(t)[0, 0] for t in (q, k, v))
    np.testing.assert_allclose(out[0, 0], vd, **TOL)
    np.testing.assert_allclose(lse[0, 0], (qd * kd).sum(-1) / math.sqrt(8), **TOL)


@pytest.mark.parametrize("N,w", [(300, 64), (256, 256), (200, 1000)])
def test_swa_matches_sdpa_with_band_mask(N, w):
    q, k, v = _qkv(1, 3, 3, N, 80, seed=7)
    out, lse = oracle.swa(q, k, v, window=w)
    i = torch.arange(N)[:, None]
    j = torch.arange(N)[None, :]
    band = (j <= i) & (i - j < w)
    ref, rlse = _sdpa(q, k, v, mask=band)
    np.testing.assert_allclose(out, ref, **TOL)
    np.testing.assert_allclose(lse, rlse, **TOL)


@pytest.mark.parametrize("B,topk,window", [(32, 3, 0), (16, 4, 24), (64, 2, 0), (8, 5, 3)])
def test_gathered_matches_naive_mask(B, topk, window):
    """The C oracle's gathered key walk equals a dense masked softmax built from the
    same block sets (independent numpy formulation)."""
    N, d = 256, 16
    q, k, v = _qkv(1, 2, 1, N, d, seed=8)
    r = _moba(q, k, v, B, topk, window)
    qd, kd, vd = (oracle.bf16_to_f64(t)[0] for t in (q, k, v))
    for h in range(2):
        mask = naive.block_mask(N, B, naive.block_sets_from_idx(r["idx"][0, h]), window)
        out, lse = naive.masked_attention(qd[h], kd[0], vd[0], mask)
        np.testing.assert_allclose(r["out"][0, h], out, **TOL)
        np.testing.assert_allclose(r["lse"][0, h], lse, **TOL)


def test_gqa_equals_repeated_kv_heads():
    q, k, v = _qkv(2, 6, 2, 256, 16, seed=9)
    B, topk = 32, 3
    r = _moba(q, k, v, B, topk, 16)
    kr, vr = k.repeat_interleave(3, dim=1), v.repeat_interleave(3, dim=1)
    r2 = _moba(q, kr, vr, B, topk, 16)
    assert np.array_equal(r["idx"], r2["idx"])
    np.testing.assert_allclose(r["out"], r2["out"], rtol=0, atol=0)
    np.testing.assert_allclose(r["lse"], r2["lse"], rtol=0, atol=0)


def test_current_and_past_merge_by_lse_equals_one_softmax():
    """MoBA §MoBA의 구현: the causal current block and the non-causal past blocks,
    computed apart and merged through their log-sum-exp, give the single softmax."""
    N, d, B, topk = 512, 16, 64, 3
    q, k, v = _qkv(1, 2, 1, N, d, seed=10)
    r = _moba(q, k, v, B, topk)
    idx = r["idx"]
    c = (np.arange(N) // B)[None, None, :, None]
    cur = np.where(idx == c, idx, -1).astype(np.int32)
    past = np.where((idx >= 0) & (idx != c), idx, -1).astype(np.int32)
    o_c, l_c = oracle.attention(q, k, v, mode=oracle.MODE_MOBA, block=B, topk=topk, idx=cur)
    has_past = (past >= 0).any(-1)
    # Rows of block 0 have no past blocks; give them a dummy set and ignore it.
    past_safe = np.where(has_past[..., None], past, cur).astype(np.int32)
    o_p, l_p = oracle.attention(q, k, v, mode=oracle.MODE_MOBA, block=B, topk=topk, idx=past_safe)
    l_p = np.where(has_past, l_p, -np.inf)
    lse = np.logaddexp(l_c, l_p)
    out = np.exp(l_c - lse)[..., None] * o_c + np.where(has_past, np.exp(l_p - lse), 0)[..., None] * o_p
    np.testing.assert_allclose(out, r["out"], **TOL)
    np.testing.assert_allclose(lse, r["lse"], **TOL)


def test_output_invariants():
    """out_i lies in the coordinatewise range of the attended values, and
    max z <= lse <= max z + ln|J|."""
    N, d, B, topk, w = 384, 16, 32, 3, 20
    q, k, v = _qkv(1, 1, 1, N, d, seed=11)
    r = _moba(q, k, v, B, topk, w)
    qd, kd, vd = (oracle.bf16_to_f64(t)[0, 0] for t in (q, k, v))
    sets = naive.block_sets_from_idx(r["idx"][0, 0])
    mask = naive.block_mask(N, B, sets, w)
    for i in range(N):
        J = np.nonzero(mask[i])[0]
        o = r["out"][0, 0, i]
        assert np.all(o >= vd[J].min(0) - 1e-12) and np.all(o <= vd[J].max(0) + 1e-12)
        z = (kd[J] @ qd[i]) / math.sqrt(d)
        assert z.max() - 1e-12 <= r["lse"][0, 0, i] <= z.max() + math.log(len(J)) + 1e-12


def test_rejects_idx_naming_a_future_block():
    q, k, v = _qkv(1, 1, 1, 128, 8)
    idx = np.full((1, 1, 128, 2), -1, dtype=np.int32)
    idx[..., 0] = 1  # block 1 is in the future for rows of block 0
    with pytest.raises(ValueError):
        oracle.attention(q, k, v, mode=oracle.MODE_MOBA, block=64, topk=2, idx=idx)


def test_sampled_rows_equal_full_rows():
    q, k, v = _qkv(1, 2, 1, 512, 16, seed=12)
    full = _moba(q, k, v, 64, 3, 40)
    rows = np.array([0, 5, 63, 64, 200, 511], dtype=np.int32)
    part = oracle.moba(q, k, v, block=64, topk=3, window=40, rows=rows)
    assert np.array_equal(part["idx"], full["idx"][:, :, rows])
    np.testing.assert_allclose(part["out"], full["out"][:, :, rows], rtol=0, atol=0)


# ------------------------------------------------------------- partial last block

@pytest.mark.parametrize("N,B,topk,window", [(500, 64, 100, 0), (300, 128, 3, 0), (200, 64, 1, 10_000)])
def test_moba_with_partial_block_reduces_to_dense_causal(N, B, topk, window):
    """B does not divide N: top-k >= n (or a window >= N) still attends every causal
    key, the partial last block included (torch SDPA, float64)."""
    q, k, v = _qkv(1, 2, 1, N, 16, seed=13)
    r = _moba(q, k, v, B, topk, window)
    ref, rlse = _sdpa(q, k, v, causal=True)
    np.testing.assert_allclose(r["out"], ref, **TOL)
    np.testing.assert_allclose(r["lse"], rlse, **TOL)


@pytest.mark.parametrize("N,B,topk,window", [(250, 32, 3, 0), (230, 16, 4, 24), (100, 64, 2, 0)])
def test_gathered_with_partial_block_matches_naive_mask(N, B, topk, window):
    d = 16
    q, k, v = _qkv(1, 2, 1, N, d, seed=14)
    r = _moba(q, k, v, B, topk, window)
    qd, kd, vd = (oracle.bf16_to_f64(t)[0] for t in (q, k, v))
    for h in range(2):
        mask = naive.block_mask(N, B, naive.block_sets_from_idx(r["idx"][0, h]), window)
        out, lse = naive.masked_attention(qd[h], kd[0], vd[0], mask)
        np.testing.assert_allclose(r["out"][0, h], out, **TOL)
        np.testing.assert_allclose(r["lse"][0, h], lse, **TOL)


def test_topk_one_with_partial_block_is_block_diagonal_causal():
    """k = 1: each row attends its own block causally, the partial last block as a
    shorter causal block (SDPA per block)."""
    N, B = 200, 64
    q, k, v = _qkv(1, 2, 2, N, 16, seed=15)
    r = _moba(q, k, v, B, 1)
    for j in range(-(-N // B)):
        sl = slice(j * B, min((j + 1) * B, N))
        ref, rlse = _sdpa(q[:, :, sl], k[:, :, sl], v[:, :, sl], causal=True)
        np.testing.assert_allclose(r["out"][:, :, sl], ref, **TOL)
        np.testing.assert_allclose(r["lse"][:, :, sl], rlse, **TOL)
