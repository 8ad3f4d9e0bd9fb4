"""Pins of the oracle's dense forward: it must be exactly softmax attention
(the article keeps the FlashAttention forward unchanged, standfirst and section
"Le passage arrière fait deux fois le travail du passage avant"; FlashAttention
is exact, voce.life course, section "Le mécanisme").  Pinned against torch's
fp64 scaled_dot_product_attention, a library routine, per segment."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float64)


def _sdpa_ref(cu, q, k, v, scale, causal):
    T, hq, d = q.shape
    hkv = k.shape[1]
    G = hq // hkv
    o = torch.zeros_like(q)
    lse = torch.zeros(hq, T, dtype=torch.float64)
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        if b == a:
            continue
        qs = q[a:b].permute(1, 0, 2)                                  # [hq, n, d]
        ks = k[a:b].permute(1, 0, 2).repeat_interleave(G, dim=0)      # head h -> kv h//G
        vs = v[a:b].permute(1, 0, 2).repeat_interleave(G, dim=0)
        o[a:b] = F.scaled_dot_product_attention(qs, ks, vs, is_causal=causal, scale=scale).permute(1, 0, 2)
        sc = scale * qs @ ks.transpose(1, 2)
        if causal:
            n = b - a
            sc = sc.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), -math.inf)
        lse[:, a:b] = torch.logsumexp(sc, dim=-1)
    return o, lse


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("seqlens,hq,hkv,d", [
    ((200,), 4, 2, 16),
    ((1, 37, 130, 64), 6, 3, 8),
    ((129,), 2, 2, 32),
])
def test_fwd_matches_sdpa(seqlens, hq, hkv, d, causal):
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    T = int(cu[-1])
    q, k, v = _rand((T, hq, d), 1), _rand((T, hkv, d), 2), _rand((T, hkv, d), 3)
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle.attn_fwd(cu, q, k, v, scale, causal)
    o_ref, lse_ref = _sdpa_ref(cu, q, k, v, scale, causal)
    np.testing.assert_allclose(o, o_ref.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref.numpy(), rtol=1e-12, atol=1e-12)


def test_first_causal_row_copies_v():
    # Row 0 of a causal segment sees only key 0: O = v_0, LSE = scale <q0,k0>.
    cu = np.array([0, 5, 9], dtype=np.int32)
    q, k, v = _rand((9, 2, 4), 4), _rand((9, 1, 4), 5), _rand((9, 1, 4), 6)
    o, lse = oracle.attn_fwd(cu, q, k, v, 0.5, True)
    for a in (0, 5):
        for h in range(2):
            np.testing.assert_allclose(o[a, h], v[a, 0].numpy(), rtol=0, atol=1e-15)
            assert abs(lse[h, a] - 0.5 * float(q[a, h] @ k[a, 0])) < 1e-14


def test_gqa_mapping_is_consecutive_groups():
    # With Hq=4, Hkv=2, heads 0,1 read KV head 0 and heads 2,3 read KV head 1.
    cu = np.array([0, 16], dtype=np.int32)
    q = _rand((16, 1, 8), 7).repeat(1, 4, 1)
    k, v = _rand((16, 2, 8), 8), _rand((16, 2, 8), 9)
    o, _ = oracle.attn_fwd(cu, q, k, v, 0.3, True)
    np.testing.assert_array_equal(o[:, 0], o[:, 1])
    np.testing.assert_array_equal(o[:, 2], o[:, 3])
    assert np.abs(o[:, 0] - o[:, 2]).max() > 1e-3


def test_synthetic_prefix_equals_full_draw():
    import synthetic
    w = synthetic.TINY.with_(seqlens=(300,))
    full = synthetic.make_inputs(w)
    pre = synthetic.make_inputs(w, rows=130)
    for k in ("q", "k", "v", "dout"):
        assert torch.equal(full[k][:130], pre[k])
    assert list(pre["cu_seqlens"]) == [0, 130]
