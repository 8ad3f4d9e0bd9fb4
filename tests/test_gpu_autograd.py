"""The autograd wrapper returns exactly what the C-ABI calls return, and at
delta = 0 the dense gradient of torch's own attention (fp32 reference)."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import block_sparse_attention_dense_b200 as lf
from block_sparse_attention_dense_b200.autograd import lazyflash_attention
import synthetic
from _helpers import rel_fro, run_step

pytestmark = pytest.mark.gpu


def _reference(q, k, v, cu, dout):
    """fp32 torch attention per segment (the reference the survey names)."""
    q = q.float().detach().requires_grad_(True)
    k = k.float().detach().requires_grad_(True)
    v = v.float().detach().requires_grad_(True)
    G = q.shape[1] // k.shape[1]
    outs = []
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        qs = q[a:b].transpose(0, 1)
        ks = k[a:b].transpose(0, 1).repeat_interleave(G, 0)
        vs = v[a:b].transpose(0, 1).repeat_interleave(G, 0)
        outs.append(F.scaled_dot_product_attention(qs, ks, vs, is_causal=True).transpose(0, 1))
    o = torch.cat(outs, 0)
    (o * dout.float()).sum().backward()
    return o.detach(), q.grad, k.grad, v.grad


def test_autograd_matches_c_abi_and_dense_reference():
    w = synthetic.Workload("ag", (300, 200), hq=4, hkv=2, d=128, block=128, sigma=1.5, delta=0.0)
    inp = synthetic.make_inputs(w)
    dev = {k_: t.cuda() for k_, t in inp.items()}
    q = dev["q"].clone().requires_grad_(True)
    k = dev["k"].clone().requires_grad_(True)
    v = dev["v"].clone().requires_grad_(True)
    o = lazyflash_attention(q, k, v, dev["cu_seqlens"], w.max_seqlen, delta=0.0, seed=1, step=2)
    o.backward(dev["dout"])
    _, _, bufs = run_step(w, inp, seed=1, step=2, delta=0.0)
    assert torch.equal(o.detach(), bufs.o)
    for got, ref in ((q.grad, bufs.dq), (k.grad, bufs.dk), (v.grad, bufs.dv)):
        assert rel_fro(got.float().cpu(), ref.float().cpu()) < 1e-5
    o_ref, dq_ref, dk_ref, dv_ref = _reference(dev["q"], dev["k"], dev["v"], w.cu_seqlens(), dev["dout"])
    assert (o.detach().float() - o_ref).abs().max().item() < 1e-2
    for got, ref in ((q.grad, dq_ref), (k.grad, dk_ref), (v.grad, dv_ref)):
        assert rel_fro(got.float().cpu(), ref.cpu()) < 1e-2


def test_autograd_steps_draw_fresh_masks():
    w = synthetic.GQA_MID.with_(seqlens=(1024,), delta=0.3)
    inp = synthetic.make_inputs(w)
    dev = {k_: t.cuda() for k_, t in inp.items()}
    grads = []
    for _ in range(2):
        q = dev["q"].clone().requires_grad_(True)
        o = lazyflash_attention(q, dev["k"], dev["v"], dev["cu_seqlens"], w.max_seqlen, delta=0.3)
        o.backward(dev["dout"])
        grads.append(q.grad.clone())
    assert not torch.equal(grads[0], grads[1])
