"""lf_attn_bwd_static_ws: the sparse backward for callers that cannot allocate
device memory (plugin interfaces that pass an operator only its inputs and
outputs, and runtimes that forbid cudaMalloc/cudaFree while they run or
capture).  Its scratch is the library's own static device array; its results
must match lf_attn_bwd with a caller workspace, call after call.

This file is collected last on purpose: if it fails, every other test has
already run.
"""
import ctypes

import pytest
import torch

import block_sparse_attention_dense_b200 as lf
import synthetic
from _helpers import rel_fro, run_step

GRAD_TOL = 1e-2   # the backward parity tolerance of the other GPU tests


# two query heads per KV head (dK/dV stored by the backward's CTAs) and forty (dK/dV through
# fp32 accumulators in the static array), each with the selection's D and with D computed
# by the call itself
@pytest.mark.gpu
@pytest.mark.parametrize("D_given", [True, False], ids=["D_given", "D_computed"])
@pytest.mark.parametrize("hq,lens", [(4, (700, 300)), (80, (300, 200))],
                         ids=["group2", "group40"])
def test_static_scratch_backward_matches_workspace_backward_twice(hq, lens, D_given):
    w = synthetic.Workload("no_alloc", lens, hq=hq, hkv=2, d=128, block=128, sigma=1.5,
                           delta=0.1)
    # one full step through the ordinary entry points (caller workspace)
    desc, dev, bufs = run_step(w, synthetic.make_inputs(w), seed=2, step=3)
    ref = {k: getattr(bufs, k).float().cpu() for k in ("dq", "dk", "dv")}
    need = lf.lf_workspace_size(desc, lf.LF_WS_BWD)
    assert need <= 32 << 20
    for call in range(2):
        out = {k: torch.full_like(getattr(bufs, k), float("nan")) for k in ("dq", "dk", "dv")}
        # without D, the call computes it from o and dout in the static array too
        lf.lf_attn_bwd_static_ws(desc, dev["q"], dev["k"], dev["v"], bufs.o, bufs.lse,
                                 dev["dout"], bufs.D if D_given else None, bufs.w, bufs.kept_idx,
                                 bufs.kept_cnt, out["dq"], out["dk"], out["dv"])
        lf.lf_check_device_error()
        torch.cuda.synchronize()
        for k in ("dq", "dk", "dv"):
            got = out[k].float().cpu()
            assert torch.isfinite(got).all(), (call, k)
            assert rel_fro(got, ref[k]) < GRAD_TOL, (call, k)


def test_static_scratch_rejects_oversize_problem_before_launch():
    L = lf.lib()
    fn = L.lf_attn_bwd_static_ws
    fn.argtypes = [ctypes.POINTER(lf.lf_attn_desc)] + [ctypes.c_void_p] * 14
    fn.restype = ctypes.c_int
    # 32768 tokens x 32 heads x 128 x 4 B = 512 MiB of accumulator > 32 MiB
    d = lf.lf_attn_desc(1, 0x1000, 32768, 32768, 32, 8, 128, 0.088, 1, 128)
    p = 0x10000
    assert fn(ctypes.byref(d), *([p] * 13), None) == lf.LF_ERR_WORKSPACE
