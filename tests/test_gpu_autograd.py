"""The autograd wrapper returns exactly what the C-ABI calls return, and at
delta = 0 the dense gradient of torch's own attention (fp32 reference)."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import block_sparse_attention_dense_b200 as lf
import oracle
from block_sparse_attention_dense_b200.autograd import lazyflash_attention
import synthetic
from _helpers import nb_per_seq, rel_fro, run_step

pytestmark = pytest.mark.gpu


def _reference(q, k, v, cu, dout):
    """fp32 torch attention per segment: the plain PyTorch reference of the dense
    attention gradient."""
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


def test_autograd_at_positive_delta_matches_the_oracle():
    """delta > 0 through the autograd wrapper: the selection it drew equals the
    oracle's on the GPU's block norms (bit-exact), and the gradients equal the
    oracle's reweighted gradient for that draw (article section "Un budget sur la
    masse de gradient, et un tirage qui garde le gradient non biaisé": the estimate
    is the dense gradient of the kept blocks' output gradients times 1/p)."""
    w = synthetic.Workload("ag_delta", (700, 300), hq=4, hkv=2, d=128, block=128, sigma=2.0,
                           delta=0.2)
    inp = synthetic.make_inputs(w)
    dev = {k_: t.cuda() for k_, t in inp.items()}
    q = dev["q"].clone().requires_grad_(True)
    k = dev["k"].clone().requires_grad_(True)
    v = dev["v"].clone().requires_grad_(True)
    sel_gpu = {}
    o = lazyflash_attention(q, k, v, dev["cu_seqlens"], w.max_seqlen, delta=w.delta, seed=9,
                            step=4, selection_out=sel_gpu)
    o.backward(dev["dout"])
    lf.lf_check_device_error()
    assert sel_gpu["step"] == 4
    nb = nb_per_seq(w)
    sel = oracle.select(sel_gpu["norm"].cpu().numpy(), nb, w.delta, 9, 4)
    np.testing.assert_array_equal(sel_gpu["keep"].cpu().numpy(), sel["keep"])
    np.testing.assert_array_equal(sel_gpu["weight"].cpu().numpy().view(np.uint32),
                                  sel["w"].view(np.uint32))
    np.testing.assert_array_equal(sel_gpu["tau"].cpu().numpy().view(np.uint64),
                                  sel["tau"].view(np.uint64))
    kept = sel["keep"][:, :, : int(nb.max())]
    assert 0 < kept.sum() < kept.size        # a real sparse draw
    dq_ref, dk_ref, dv_ref = oracle.attn_bwd(w.cu_seqlens(), inp["q"], inp["k"], inp["v"],
                                             inp["dout"], w.scale, w.block,
                                             sel["w"].astype(np.float64), True)
    for got, ref in ((q.grad, dq_ref), (k.grad, dk_ref), (v.grad, dv_ref)):
        assert rel_fro(got.float().cpu().numpy(), ref) < 1e-2
