"""Pins of the oracle's selection (article section "Un budget sur la masse de
gradient, et un tirage qui garde le gradient non biaisé"): a budget delta bounds
the discarded share of gradient mass, each block is kept with probability
proportional to its gradient norm, and kept blocks are reweighted so that the
gradient is unbiased in expectation.

Reading: p_b = min(1, m_b / tau), tau the largest threshold with expected
discarded mass sum_b (1 - p_b) m_b <= delta * sum_b m_b.
"""
import math

import numpy as np
import pytest

import oracle
import synthetic


def _tau_closed_form(m, delta):
    """Piecewise solution: on (m_(k), m_(k+1)] the discarded mass is
    S1_k - S2_k / tau with S1_k, S2_k the sum and the sum of squares of the k
    smallest norms; solve S1_k - S2_k / tau = delta * M on the first piece whose
    right end already exceeds the budget."""
    m = np.sort(np.asarray(m, dtype=np.float64))
    M = math.fsum(m)
    B = delta * M
    n = len(m)
    for kk in range(1, n + 1):
        S1 = math.fsum(m[:kk])
        S2 = math.fsum(m[:kk] ** 2)
        right = m[kk] if kk < n else math.inf
        if right == math.inf:
            f_right = S1
        elif right == 0.0:
            f_right = 0.0
        else:
            f_right = S1 - S2 / right
        if f_right > B:
            if S1 - B <= 0:
                continue
            return S2 / (S1 - B)
    raise AssertionError("no crossing")


@pytest.mark.parametrize("seed", range(12))
@pytest.mark.parametrize("delta", [0.01, 0.1, 0.3, 0.7])
def test_tau_matches_closed_form(seed, delta):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 300))
    m = rng.lognormal(0.0, 2.0, size=n)
    if seed % 3 == 0:
        m[rng.uniform(size=n) < 0.2] = 0.0            # zero-norm blocks
    if m.sum() == 0:
        m[0] = 1.0
    t = oracle.tau(m, delta)
    ref = _tau_closed_form(m, delta)
    assert abs(t - ref) <= 1e-12 * ref, (t, ref)


@pytest.mark.parametrize("seed", range(8))
def test_budget_and_maximality(seed):
    rng = np.random.default_rng(100 + seed)
    m = rng.lognormal(0.0, 1.5, size=int(rng.integers(2, 512)))
    delta = float(rng.uniform(0.01, 0.9))
    t = oracle.tau(m, delta)
    M = math.fsum(m)
    p = np.minimum(1.0, m / t)
    disc = math.fsum((1.0 - p) * m)
    assert disc <= delta * M * (1 + 1e-12)
    p2 = np.minimum(1.0, m / (t * (1 + 1e-9)))
    assert math.fsum((1.0 - p2) * m) > delta * M


def test_pinned_sum_is_a_sum():
    rng = np.random.default_rng(7)
    for n in (0, 1, 31, 32, 33, 500):
        x = rng.lognormal(0, 2, size=n)
        ref = math.fsum(x)
        assert abs(oracle.pinned_sum(x) - ref) <= 64 * 2.0 ** -52 * max(ref, 1e-300)


def test_single_block_and_equal_norms():
    # one block: the budget can only be met by keeping it with p = 1 - delta
    for delta in (0.1, 0.5):
        t = oracle.tau([2.0], delta)
        assert abs(2.0 / t - (1 - delta)) < 1e-13
    # equal norms: p = 1 - delta for every block
    t = oracle.tau(np.full(40, 3.0), 0.25)
    assert abs(3.0 / t - 0.75) < 1e-13


def _select_all(m, nb, delta, seed, step):
    return oracle.select(m, nb, delta, seed, step)


def test_select_outputs_consistent():
    w = synthetic.VARLEN
    nb = oracle.nblocks(w.cu_seqlens(), w.block)
    m = synthetic.random_norms(w.nseq, 4, w.nbmax, nb, 1.5, seed=3)
    m[0, 1, :5] = 0.0
    r = _select_all(m, nb, 0.2, seed=11, step=4)
    for s in range(w.nseq):
        for h in range(4):
            n = int(nb[s])
            t = r["tau"][s, h]
            keep = r["keep"][s, h]
            assert keep[n:].sum() == 0 and np.all(r["w"][s, h, n:] == 0)
            idx = np.nonzero(keep[:n])[0]
            assert r["kept_cnt"][s, h] == len(idx)
            np.testing.assert_array_equal(r["kept_idx"][s, h, :len(idx)], idx)
            assert np.all(r["kept_idx"][s, h, len(idx):] == -1)
            mm = m[s, h, :n].astype(np.float64)
            p = np.minimum(1.0, mm / t)
            np.testing.assert_array_equal(r["p"][s, h, :n], p)
            for i in range(n):
                u = oracle.block_u24(11, 4, s, h, i)
                want = p[i] >= 1.0 or u < p[i] * 2.0 ** 24
                assert bool(keep[i]) == want
                if want:
                    assert r["w"][s, h, i] == np.float32(1.0 / p[i])
            # zero-norm blocks are never kept (their contribution is zero anyway)
            assert not np.any(keep[:n][mm == 0.0])
            assert math.fsum((1 - p) * mm) <= 0.2 * math.fsum(mm) * (1 + 1e-12)


def test_delta_zero_keeps_everything_with_unit_weight():
    nb = np.array([8, 3], dtype=np.int32)
    m = synthetic.random_norms(2, 3, 8, nb, 2.0, seed=1)
    r = oracle.select(m, nb, 0.0, seed=0, step=0)
    assert np.all(r["tau"] == 0.0)
    for s in range(2):
        assert np.all(r["keep"][s, :, :nb[s]] == 1) and np.all(r["w"][s, :, :nb[s]] == 1.0)
        assert np.all(r["kept_cnt"][s] == nb[s])


def test_all_zero_norms_keep_all():
    nb = np.array([4], dtype=np.int32)
    r = oracle.select(np.zeros((1, 2, 4)), nb, 0.3, 0, 0)
    assert np.all(r["keep"] == 1) and np.all(r["w"] == 1.0)


def test_delta_out_of_range_rejected():
    nb = np.array([4], dtype=np.int32)
    with pytest.raises(ValueError):
        oracle.select(np.ones((1, 1, 4)), nb, 1.0, 0, 0)
    with pytest.raises(ValueError):
        oracle.select(np.ones((1, 1, 4)), nb, -0.1, 0, 0)


def test_masks_change_across_steps_and_heads():
    # The skipped set adapts per head and per step (article, same section).
    nb = np.array([256], dtype=np.int32)
    m = synthetic.random_norms(1, 4, 256, nb, 2.0, seed=2)
    a = oracle.select(m, nb, 0.1, 0, 0)["keep"]
    b = oracle.select(m, nb, 0.1, 0, 1)["keep"]
    assert (a != b).sum() > 10
    m2 = m.copy()
    m2[0, 1] = m2[0, 0]
    c = oracle.select(m2, nb, 0.1, 0, 0)["keep"]
    assert (c[0, 0] != c[0, 1]).sum() > 0


def test_keep_frequency_matches_probability():
    nb = np.array([16], dtype=np.int32)
    m = synthetic.random_norms(1, 1, 16, nb, 1.5, seed=4)
    n_steps = 4000
    cnt = np.zeros(16)
    for st in range(n_steps):
        r = oracle.select(m, nb, 0.3, 9, st)
        cnt += r["keep"][0, 0]
    p = r["p"][0, 0]
    for i in range(16):
        if p[i] >= 1.0:
            assert cnt[i] == n_steps
            continue
        sd = math.sqrt(n_steps * p[i] * (1 - p[i]))
        assert abs(cnt[i] - n_steps * p[i]) < 4.5 * sd + 1, (i, cnt[i], n_steps * p[i])


def test_sampled_gradient_unbiased_tiny():
    """Mean of the reweighted sparse gradient over 10^4 draws equals the dense
    gradient within its Monte-Carlo interval (Tiny workload).  Uses linearity:
    the weighted gradient is sum_b w_b G_b with G_b the oracle's per-block
    gradient, so each draw costs only a selection."""
    w = synthetic.TINY
    inp = synthetic.make_inputs(w)
    cu = w.cu_seqlens()
    nb = oracle.nblocks(cu, w.block)
    norms = oracle.block_norms(cu, inp["dout"], w.block)
    nbmax = norms.shape[2]
    rng = np.random.default_rng(17)
    # 8 fixed random projections of the concatenated (dq, dk, dv)
    shapes = [tuple(inp["q"].shape), tuple(inp["k"].shape), tuple(inp["v"].shape)]
    R = [[rng.standard_normal(sh) for sh in shapes] for _ in range(8)]
    blocks = [(0, h, b) for h in range(w.hq) for b in range(int(nb[0]))]
    C = np.zeros((8, len(blocks)))
    for j, (s, h, b) in enumerate(blocks):
        onehot = np.zeros((1, w.hq, nbmax))
        onehot[s, h, b] = 1.0
        G = oracle.attn_bwd(cu, inp["q"], inp["k"], inp["v"], inp["dout"], w.scale, w.block, onehot)
        for r in range(8):
            C[r, j] = sum(float((R[r][i] * G[i]).sum()) for i in range(3))
    dense = C.sum(axis=1)
    n_draw = 10000
    est = np.zeros((n_draw, 8))
    p_b = None
    for st in range(n_draw):
        sel = oracle.select(norms, nb, w.delta, seed=0, step=st)
        wv = np.array([sel["w"][s, h, b] for (s, h, b) in blocks], dtype=np.float64)
        est[st] = C @ wv
        p_b = np.array([sel["p"][s, h, b] for (s, h, b) in blocks])
    var = ((1 - p_b) / p_b * C ** 2).sum(axis=1)      # exact per-draw variance
    mean = est.mean(axis=0)
    z = (mean - dense) / np.sqrt(var / n_draw + 1e-300)
    assert np.all(np.abs(z) < 4.0), z
    # and the empirical variance agrees with the exact one
    np.testing.assert_allclose(est.var(axis=0), var, rtol=0.15)


# ---------------------------------------------------------------------------
# Alternative rules (article section "Le choix des blocs pèse plus que la
# quantité sautée"): fixed fraction and top-k.
# ---------------------------------------------------------------------------
def _tau_fixed_closed_form(m, f):
    """On (m_(j+1), m_(j)] of the descending order the expected kept count is
    j + S/tau, S the sum of the smaller norms: solve j + S/tau = f n on the
    piece where the count crosses f n."""
    m = np.sort(np.asarray(m, dtype=np.float64))[::-1]
    n = len(m)
    target = f * n
    for j in range(0, n):
        S = math.fsum(m[j:])
        hi = m[j - 1] if j > 0 else math.inf     # tau <= hi keeps the j largest outright
        lo = m[j]
        if target - j <= 0:
            continue
        t = S / (target - j)
        if lo <= t <= hi:
            return t
    raise AssertionError("no crossing")


@pytest.mark.parametrize("seed", range(10))
@pytest.mark.parametrize("f", [0.05, 0.2, 0.5, 0.9])
def test_fixed_fraction_tau_matches_closed_form(seed, f):
    rng = np.random.default_rng(200 + seed)
    m = rng.lognormal(0.0, 2.0, size=int(rng.integers(2, 400)))
    t = oracle.tau_fixed_fraction(m, f)
    ref = _tau_fixed_closed_form(m, f)
    assert abs(t - ref) <= 1e-12 * ref, (t, ref)
    # expected kept count hits the target; a slightly larger tau falls short
    p = np.minimum(1.0, m / t)
    assert abs(math.fsum(p) - f * len(m)) <= 1e-9 * f * len(m)
    assert math.fsum(np.minimum(1.0, m / (t * (1 + 1e-9)))) < f * len(m)


def test_fixed_fraction_selection_outputs():
    nb = np.array([100, 37], dtype=np.int32)
    m = synthetic.random_norms(2, 3, 100, nb, 1.5, seed=8)
    r = oracle.select_rule(oracle.RULE_FIXED_FRACTION, m, nb, 0.25, seed=4, step=6)
    for s in range(2):
        for h in range(3):
            n = int(nb[s])
            t = r["tau"][s, h]
            p = np.minimum(1.0, m[s, h, :n].astype(np.float64) / t)
            np.testing.assert_array_equal(r["p"][s, h, :n], p)
            for i in range(n):
                u = oracle.block_u24(4, 6, s, h, i)
                assert bool(r["keep"][s, h, i]) == (p[i] >= 1.0 or u < p[i] * 2.0 ** 24)
            kept = np.nonzero(r["keep"][s, h, :n])[0]
            np.testing.assert_array_equal(r["kept_idx"][s, h, :len(kept)], kept)
            np.testing.assert_array_equal(r["w"][s, h, kept], (1.0 / p[kept]).astype(np.float32))


@pytest.mark.parametrize("f", [0.01, 0.1, 0.33, 1.0])
def test_topk_matches_library_sort(f):
    nb = np.array([256, 57], dtype=np.int32)
    m = synthetic.random_norms(2, 4, 256, nb, 2.0, seed=9)
    m[1, 2, 10:20] = m[1, 2, 5]                  # ties: the lower index wins
    r = oracle.select_rule(oracle.RULE_TOPK, m, nb, f, seed=0, step=0)
    for s in range(2):
        for h in range(4):
            n = int(nb[s])
            k = min(n, math.ceil(f * n))
            order = np.lexsort((np.arange(n), -m[s, h, :n].astype(np.float64)))
            want = np.sort(order[:k])
            kept = np.nonzero(r["keep"][s, h, :n])[0]
            np.testing.assert_array_equal(kept, want)
            assert r["kept_cnt"][s, h] == k
            assert np.all(r["w"][s, h, kept] == 1.0)
            if k:
                assert r["tau"][s, h] == m[s, h, order[k - 1]]
    # top-k is the same at every step (deterministic)
    r2 = oracle.select_rule(oracle.RULE_TOPK, m, nb, f, seed=5, step=77)
    np.testing.assert_array_equal(r["keep"], r2["keep"])


def test_rule_zero_is_the_budget_rule():
    nb = np.array([64], dtype=np.int32)
    m = synthetic.random_norms(1, 2, 64, nb, 1.5, seed=1)
    a = oracle.select_rule(oracle.RULE_BUDGET, m, nb, 0.1, 3, 4)
    b = oracle.select(m, nb, 0.1, 3, 4)
    for k_ in a:
        np.testing.assert_array_equal(a[k_], b[k_])
