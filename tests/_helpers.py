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
