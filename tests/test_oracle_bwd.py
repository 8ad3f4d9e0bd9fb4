"""Pins of the oracle's backward (article section "Le passage arrière fait deux
fois le travail du passage avant": dO, D = rowsum(dO*O), dP, dS, dQ/dK/dV; and
section "Un budget sur la masse de gradient ...": kept blocks reweighted).

* torch fp64 autograd of sum_t <w_b(t) dO_t, O_t> (a library routine);
* central finite differences of the oracle's own forward (no torch);
* the gradient is linear in the block weights: bwd(w) = sum_b w_b G_b, where
  G_b is the gradient with only block b's dO;
* all-ones weights reproduce the unweighted (dense) path bit for bit.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle


def _rand(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return scale * torch.randn(*shape, generator=g, dtype=torch.float64)


def _torch_grads(cu, q, k, v, do, scale, block, wblk, causal):
    q = q.clone().requires_grad_(True)
    k = k.clone().requires_grad_(True)
    v = v.clone().requires_grad_(True)
    T, hq, d = q.shape
    G = hq // k.shape[1]
    loss = 0.0
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        if b == a:
            continue
        qs = q[a:b].permute(1, 0, 2)
        ks = k[a:b].permute(1, 0, 2).repeat_interleave(G, dim=0)
        vs = v[a:b].permute(1, 0, 2).repeat_interleave(G, dim=0)
        o = F.scaled_dot_product_attention(qs, ks, vs, is_causal=causal, scale=scale)
        dos = do[a:b].permute(1, 0, 2).clone()
        if wblk is not None:
            rows = torch.arange(b - a) // block
            dos = dos * torch.as_tensor(wblk[s])[:, rows][:, :, None]
        loss = loss + (dos * o).sum()
    loss.backward()
    return q.grad, k.grad, v.grad


@pytest.mark.parametrize("weighted", [False, True])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("seqlens,hq,hkv,d,block", [
    ((96,), 4, 2, 16, 32),
    ((1, 50, 77), 4, 1, 8, 16),
])
def test_bwd_matches_autograd(seqlens, hq, hkv, d, block, causal, weighted):
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    T = int(cu[-1])
    q, k, v = _rand((T, hq, d), 11), _rand((T, hkv, d), 12), _rand((T, hkv, d), 13)
    do = _rand((T, hq, d), 14)
    nbmax = int(oracle.nblocks(cu, block).max())
    wblk = None
    if weighted:
        rng = np.random.default_rng(3)
        wblk = rng.uniform(0.0, 4.0, size=(len(seqlens), hq, nbmax))
        wblk[rng.uniform(size=wblk.shape) < 0.3] = 0.0
    scale = 1.0 / math.sqrt(d)
    dq, dk, dv = oracle.attn_bwd(cu, q, k, v, do, scale, block, wblk, causal)
    tq, tk, tv = _torch_grads(cu, q, k, v, do, scale, block, wblk, causal)
    for got, ref in ((dq, tq), (dk, tk), (dv, tv)):
        ref = ref.numpy()
        err = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
        assert err < 1e-12, err


def _loss(cu, q, k, v, do, scale, wrow, causal):
    o, _ = oracle.attn_fwd(cu, q, k, v, scale, causal)
    return float((wrow[:, :, None] * do.numpy() * o).sum())


def test_bwd_central_finite_differences():
    # Tiny case: N <= 32, d = 8, Hq = 2, Hkv = 1, block 4, random weights.
    cu = np.array([0, 13, 32], dtype=np.int32)
    T, hq, hkv, d, block = 32, 2, 1, 8, 4
    q, k, v = _rand((T, hq, d), 21), _rand((T, hkv, d), 22), _rand((T, hkv, d), 23)
    do = _rand((T, hq, d), 24)
    nbmax = int(oracle.nblocks(cu, block).max())
    wblk = np.random.default_rng(5).uniform(0.5, 3.0, size=(2, hq, nbmax))
    wrow = np.zeros((T, hq))
    for s in range(2):
        for t in range(cu[s], cu[s + 1]):
            wrow[t] = wblk[s, :, (t - cu[s]) // block]
    scale = 0.4
    dq, dk, dv = oracle.attn_bwd(cu, q, k, v, do, scale, block, wblk, True)
    h = 1e-6
    rng = np.random.default_rng(9)
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for trial in range(4):
            e = torch.from_numpy(rng.standard_normal(x.shape))
            args = {"q": q, "k": k, "v": v}
            args[name] = x + h * e
            lp = _loss(cu, args["q"], args["k"], args["v"], do, scale, wrow, True)
            args[name] = x - h * e
            lm = _loss(cu, args["q"], args["k"], args["v"], do, scale, wrow, True)
            fd = (lp - lm) / (2 * h)
            an = float((g * e.numpy()).sum())
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_bwd_linear_in_block_weights():
    cu = np.array([0, 70, 128], dtype=np.int32)
    T, hq, hkv, d, block = 128, 2, 1, 8, 16
    q, k, v = _rand((T, hq, d), 31), _rand((T, hkv, d), 32), _rand((T, hkv, d), 33)
    do = _rand((T, hq, d), 34)
    nb = oracle.nblocks(cu, block)
    nbmax = int(nb.max())
    scale = 1.0 / math.sqrt(d)
    w = np.random.default_rng(1).uniform(0.0, 5.0, size=(2, hq, nbmax))
    acc = [np.zeros_like(q.numpy()), np.zeros_like(k.numpy()), np.zeros_like(v.numpy())]
    dense_sum = [np.zeros_like(a) for a in acc]
    for s in range(2):
        for h in range(hq):
            for b in range(int(nb[s])):
                onehot = np.zeros((2, hq, nbmax))
                onehot[s, h, b] = 1.0
                Gb = oracle.attn_bwd(cu, q, k, v, do, scale, block, onehot, True)
                for i in range(3):
                    acc[i] += w[s, h, b] * Gb[i]
                    dense_sum[i] += Gb[i]
    got = oracle.attn_bwd(cu, q, k, v, do, scale, block, w, True)
    dense = oracle.attn_bwd(cu, q, k, v, do, scale, block, None, True)
    for i in range(3):
        assert np.linalg.norm(got[i] - acc[i]) <= 1e-12 * np.linalg.norm(acc[i])
        assert np.linalg.norm(dense[i] - dense_sum[i]) <= 1e-12 * np.linalg.norm(dense[i])


def test_all_ones_weights_bit_identical_to_dense():
    cu = np.array([0, 100], dtype=np.int32)
    q, k, v = _rand((100, 2, 8), 41), _rand((100, 2, 8), 42), _rand((100, 2, 8), 43)
    do = _rand((100, 2, 8), 44)
    ones = np.ones((1, 2, 4))
    a = oracle.attn_bwd(cu, q, k, v, do, 0.3, 32, ones, True)
    b = oracle.attn_bwd(cu, q, k, v, do, 0.3, 32, None, True)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_zero_weight_rows_contribute_nothing_to_dq():
    cu = np.array([0, 64], dtype=np.int32)
    q, k, v = _rand((64, 1, 8), 51), _rand((64, 1, 8), 52), _rand((64, 1, 8), 53)
    do = _rand((64, 1, 8), 54)
    w = np.array([[[1.0, 0.0, 2.0, 0.0]]])
    dq, _, _ = oracle.attn_bwd(cu, q, k, v, do, 0.3, 16, w, True)
    assert np.all(dq[16:32] == 0.0) and np.all(dq[48:64] == 0.0)
    assert np.abs(dq[0:16]).max() > 0 and np.abs(dq[32:48]).max() > 0


def test_block_norms_and_rowdot_match_numpy():
    cu = np.array([0, 70, 70, 200], dtype=np.int32)   # includes an empty segment
    do = _rand((200, 3, 8), 61)
    o = _rand((200, 3, 8), 62)
    block = 32
    m = oracle.block_norms(cu, do, block)
    nb = oracle.nblocks(cu, block)
    assert m.shape == (3, 3, int(nb.max()))
    d = do.numpy()
    for s in range(3):
        for h in range(3):
            for i in range(m.shape[2]):
                r0 = cu[s] + i * block
                r1 = min(cu[s] + (i + 1) * block, cu[s + 1])
                ref = np.linalg.norm(d[r0:r1, h, :]) if i < nb[s] else 0.0
                assert abs(m[s, h, i] - ref) <= 1e-13 * max(ref, 1.0)
    D = oracle.rowdot(do, o)
    np.testing.assert_allclose(D, np.einsum("thd,thd->ht", d, o.numpy()), rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("causal", [True, False])
def test_row_sampled_oracle_equals_full_oracle(causal):
    # The row-sampled evaluation (used for parity at full size) must agree with
    # the full oracle at those rows, including empty segments and GQA.
    cu = np.array([0, 40, 40, 131, 200], dtype=np.int32)
    T, hq, hkv, d, block = 200, 4, 2, 8, 16
    q, k, v = _rand((T, hq, d), 71), _rand((T, hkv, d), 72), _rand((T, hkv, d), 73)
    do = _rand((T, hq, d), 74)
    nbmax = int(oracle.nblocks(cu, block).max())
    w = np.random.default_rng(2).uniform(0.0, 3.0, size=(4, hq, nbmax))
    w[:, :, 1] = 0.0
    scale = 0.35
    o, lse = oracle.attn_fwd(cu, q, k, v, scale, causal)
    dq, dk, dv = oracle.attn_bwd(cu, q, k, v, do, scale, block, w, causal)
    rng = np.random.default_rng(4)
    rows = rng.integers(0, T, size=25)
    heads = rng.integers(0, hq, size=25)
    o_r, lse_r = oracle.attn_fwd_rows(cu, q, k, v, scale, rows, heads, causal)
    np.testing.assert_allclose(o_r, o[rows, heads], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse_r, lse[heads, rows], rtol=1e-12, atol=1e-13)
    kvr = rng.integers(0, T, size=20)
    kvh = rng.integers(0, hkv, size=20)
    dq_r, dk_r, dv_r = oracle.attn_bwd_rows(cu, q, k, v, do, scale, block, w, rows, heads,
                                            kvr, kvh, causal)
    np.testing.assert_allclose(dq_r, dq[rows, heads], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk_r, dk[kvr, kvh], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv_r, dv[kvr, kvh], rtol=1e-10, atol=1e-12)
