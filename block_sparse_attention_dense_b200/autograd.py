"""LazyFlash as a torch.autograd.Function (argument marshalling only).

The forward is the exact dense attention (lf_attn_fwd); the backward selects
query blocks from the incoming output gradient (lf_block_select: budget delta,
Philox draw keyed on (seed, step)) and runs the block-sparse backward over the
kept blocks (lf_attn_bwd).  The returned gradients are the reweighted estimate:
unbiased in expectation, exactly the dense gradient at delta = 0 (LazyFlash
article, section "Un budget sur la masse de gradient, et un tirage qui garde le
gradient non biaisé").

Tensors use the THD layout of include/lazyflash.h: q [T, hq, d], k and v
[T, hkv, d] (bf16, CUDA, contiguous); cu_seqlens int32 CUDA [nseq + 1].
"""
from __future__ import annotations

import itertools
import math

import torch

from . import (Buffers, lf_attn_bwd, lf_attn_fwd, lf_block_select, make_desc)

_step_counter = itertools.count()


class LazyFlashAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, cu_seqlens, max_seqlen, delta, seed, step, causal, block_q,
                softmax_scale, selection_out):
        for t in (q, k, v):
            if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
                raise ValueError("q, k, v must be contiguous bf16 CUDA tensors")
        T, hq, d = q.shape
        hkv = k.shape[1]
        scale = softmax_scale if softmax_scale is not None else 1.0 / math.sqrt(d)
        desc = make_desc(cu_seqlens, max_seqlen, T, hq, hkv, d, scale, causal, block_q)
        o = torch.empty_like(q)
        lse = torch.empty(hq, T, dtype=torch.float32, device=q.device)
        lf_attn_fwd(desc, q, k, v, o, lse)
        ctx.save_for_backward(q, k, v, o, lse, cu_seqlens)
        ctx.desc = desc
        ctx.delta = float(delta)
        ctx.seed = int(seed)
        ctx.step = int(next(_step_counter) if step is None else step)
        ctx.selection_out = selection_out
        return o

    @staticmethod
    def backward(ctx, grad_o):
        q, k, v, o, lse, cu_seqlens = ctx.saved_tensors
        desc = ctx.desc
        dout = grad_o.to(torch.bfloat16).contiguous()
        # the backward's own buffers only: o and lse are the forward's saved tensors
        bufs = Buffers(desc, device=q.device, forward=False)
        lf_block_select(desc, dout, o, ctx.delta, ctx.seed, ctx.step, 0, bufs.norm, bufs.D,
                        bufs.tau, bufs.w, bufs.keep, bufs.kept_idx, bufs.kept_cnt)
        lf_attn_bwd(desc, q, k, v, o, lse, dout, bufs.D, bufs.w, bufs.kept_idx, bufs.kept_cnt,
                    bufs.dq, bufs.dk, bufs.dv, bufs.ws)
        if ctx.selection_out is not None:
            ctx.selection_out.update(norm=bufs.norm, tau=bufs.tau, keep=bufs.keep,
                                     weight=bufs.w, kept_cnt=bufs.kept_cnt, step=ctx.step)
        return bufs.dq, bufs.dk, bufs.dv, None, None, None, None, None, None, None, None, None


def lazyflash_attention(q, k, v, cu_seqlens, max_seqlen, delta=0.1, seed=0, step=None,
                        causal=True, block_q=128, softmax_scale=None, selection_out=None):
    """Dense attention forward, LazyFlash block-sparse backward.

    ``step`` defaults to a process-wide counter, so every backward draws a
    fresh mask; pass it explicitly to replay a draw.  If ``selection_out`` is a
    dict, the backward stores in it the selection it drew: block norms ``norm``,
    thresholds ``tau``, ``keep``, block weights ``weight`` ([nseq, hq, nbmax]
    device tensors), ``kept_cnt`` and the Philox ``step`` used."""
    return LazyFlashAttention.apply(q, k, v, cu_seqlens, max_seqlen, delta, seed, step, causal,
                                    block_q, softmax_scale, selection_out)
