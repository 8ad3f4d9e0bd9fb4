"""Shared test plumbing: move synthetic workloads to the GPU and run the
LazyFlash step through the C ABI.  No method arithmetic lives here."""
import numpy as np
import torch

import block_sparse_attention_dense_b200 as lf
import synthetic


def to_dev(inp):
    return {k: v.cuda() for k, v in inp.items()}


def desc_for(w: synthetic.Workload, cu_dev):
    return lf.make_desc(cu_dev, w.max_seqlen, w.total_tokens, w.hq, w.hkv, w.d, w.scale,
                        w.causal, w.block)


def run_step(w: synthetic.Workload, inp=None, seed=0, step=0, delta=None, flags=0, norms=None):
    """Runs fwd + select + bwd on the GPU; returns (desc, dev inputs, Buffers)."""
    if inp is None:
        inp = synthetic.make_inputs(w)
    dev = to_dev(inp)
    desc = desc_for(w, dev["cu_seqlens"])
    bufs = lf.Buffers(desc)
    if norms is not None:
        bufs.norm.copy_(torch.as_tensor(norms, dtype=torch.float32))
        flags |= lf.LF_SELECT_NORMS_GIVEN
    lf.lazyflash_step(desc, dev["q"], dev["k"], dev["v"], dev["dout"],
                      w.delta if delta is None else delta, seed, step, bufs, flags=flags)
    lf.lf_check_device_error()
    torch.cuda.synchronize()
    return desc, dev, bufs


def rel_fro(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / max(nb, 1e-30))


def nb_per_seq(w):
    cu = w.cu_seqlens()
    return ((np.diff(cu) + w.block - 1) // w.block).astype(np.int32)


def bf16_half_ulp(x):
    """Half the spacing of bf16 numbers at |x| (8 significant bits): the largest
    error the rounding of an exact value to the bf16 output format can add."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.exp2(e - 8)


def o_within(o, o_ref, tol):
    """O is stored in bf16: the kernel's value may differ from the exact one by `tol`
    (the stated max-abs tolerance) before its rounding to bf16, plus that rounding.
    Returns (ok, worst excess, |o_ref| at the worst element) for the message."""
    o = np.asarray(o, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    excess = np.abs(o - o_ref) - (tol + bf16_half_ulp(o_ref))
    i = int(np.argmax(excess))
    return bool(excess.flat[i] <= 0), float(excess.flat[i]), float(np.abs(o_ref).flat[i])
