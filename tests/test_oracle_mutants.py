"""Mutation check of the oracle's pins: a plausible mistake planted in the
oracle (compiled in with -DLFO_MUTANT=k, on the CPU) must make at least one
pin fail, and the oracle as written must pass all of them.

Planted mistakes: 1 scores without the softmax scale; 2 KV head h % hkv instead
of h / (hq/hkv); 3 D from the unweighted dO; 4 dK without the scale; 5 dS with
the sign flipped; 6 discarded mass p*m instead of (1-p)*m; 7 Philox with nine
rounds; 8 weight p instead of 1/p; 9 causal mask one key short; 10 block norm
squared."""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")


def _rand(shape, seed):
    return torch.randn(*shape, generator=torch.Generator().manual_seed(seed), dtype=torch.float64)


def pin_philox_kat():
    for line in open(GOLD):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        w = [int(x, 16) for x in line.split()]
        if [int(x) for x in oracle.philox4x32_10(w[0:4], w[4:6])] != w[6:10]:
            return False
    return True


def _sdpa(q, k, v, G):
    qs = q.transpose(0, 1)
    ks = k.transpose(0, 1).repeat_interleave(G, 0)
    vs = v.transpose(0, 1).repeat_interleave(G, 0)
    return F.scaled_dot_product_attention(qs, ks, vs, is_causal=True, scale=0.3).transpose(0, 1)


def pin_forward_sdpa():
    cu = np.array([0, 40], dtype=np.int32)
    q, k, v = _rand((40, 4, 8), 1), _rand((40, 2, 8), 2), _rand((40, 2, 8), 3)
    o, _ = oracle.attn_fwd(cu, q, k, v, 0.3, True)
    return np.allclose(o, _sdpa(q, k, v, 2).numpy(), rtol=1e-10, atol=1e-12)


def pin_backward_autograd():
    cu = np.array([0, 48], dtype=np.int32)
    q, k, v, do = _rand((48, 4, 8), 4), _rand((48, 2, 8), 5), _rand((48, 2, 8), 6), _rand((48, 4, 8), 7)
    w = np.array([[[2.0, 0.5, 3.0]] * 4]).reshape(1, 4, 3)
    dq, dk, dv = oracle.attn_bwd(cu, q, k, v, do, 0.3, 16, w, True)
    qg, kg, vg = (t.clone().requires_grad_(True) for t in (q, k, v))
    rows = torch.arange(48) // 16
    wrow = torch.as_tensor(w[0])[:, rows].transpose(0, 1)[:, :, None]
    (_sdpa(qg, kg, vg, 2) * do * wrow).sum().backward()
    return all(np.allclose(a, b.numpy(), rtol=1e-9, atol=1e-11)
               for a, b in ((dq, qg.grad), (dk, kg.grad), (dv, vg.grad)))


def pin_tau_closed_form():
    m = np.random.default_rng(3).lognormal(0.0, 2.0, size=80)
    delta = 0.2
    t = oracle.tau(m, delta)
    ms = np.sort(m)
    B = delta * math.fsum(ms)
    for kk in range(1, len(ms) + 1):
        S1, S2 = math.fsum(ms[:kk]), math.fsum(ms[:kk] ** 2)
        right = ms[kk] if kk < len(ms) else math.inf
        f_right = S1 - S2 / right if right < math.inf else S1
        if f_right > B and S1 - B > 0:
            return abs(t - S2 / (S1 - B)) <= 1e-12 * t
    return False


def pin_weights_unbiased():
    """E[keep_b * w_b] = 1 for every block (z-test over 3000 draws)."""
    nb = np.array([8], dtype=np.int32)
    m = np.random.default_rng(5).lognormal(0.0, 1.5, size=(1, 1, 8))
    acc = np.zeros(8)
    n = 3000
    for st in range(n):
        r = oracle.select(m, nb, 0.4, 1, st)
        acc += r["w"][0, 0].astype(np.float64)
    p = r["p"][0, 0]
    sd = np.sqrt((1 - p) / p / n)
    return bool(np.all(np.abs(acc / n - 1.0) < 5 * sd + 1e-12))


def pin_norms_numpy():
    cu = np.array([0, 70], dtype=np.int32)
    do = _rand((70, 2, 8), 9)
    m = oracle.block_norms(cu, do, 32)
    d = do.numpy()
    ref = [[np.linalg.norm(d[i * 32:min(70, (i + 1) * 32), h]) for i in range(3)] for h in range(2)]
    return np.allclose(m[0], np.array(ref), rtol=1e-12)


PINS = [pin_philox_kat, pin_forward_sdpa, pin_backward_autograd, pin_tau_closed_form,
        pin_weights_unbiased, pin_norms_numpy]


def _run_pins():
    return {p.__name__: bool(p()) for p in PINS}


def test_oracle_as_written_passes_every_pin():
    assert all(_run_pins().values())


@pytest.mark.parametrize("mutant", range(1, 11))
def test_planted_mistake_is_caught(mutant, tmp_path):
    path = oracle.build_variant(mutant, str(tmp_path / ("liblfo_m%d.so" % mutant)))
    prev = oracle.use_library(path)
    try:
        res = _run_pins()
    finally:
        oracle.restore_library(prev)
    assert not all(res.values()), (mutant, res)
