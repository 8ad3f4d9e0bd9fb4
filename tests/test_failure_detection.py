"""Failure detection without a GPU fault: every wait in the
kernels is bounded; when one runs out the kernel records it in a device flag
and returns, and the host reads LF_ERR_TIMEOUT.  The self-test makes a wait run
out (a barrier phase that nothing completes) and checks that the status comes
back and that the context still works afterwards."""
import ctypes

import pytest
import torch

import block_sparse_attention_dense_b200 as lf
import synthetic
from _helpers import run_step


def test_selftest_rejects_bad_limits_on_host():
    L = lf.lib()
    L.lf_watchdog_selftest.argtypes = [ctypes.c_uint32, ctypes.c_void_p]
    L.lf_watchdog_selftest.restype = ctypes.c_int
    assert L.lf_watchdog_selftest(5, None) == lf.LF_ERR_INVALID_ARG
    assert L.lf_watchdog_selftest(40, None) == lf.LF_ERR_INVALID_ARG


@pytest.mark.gpu
def test_expired_wait_is_reported_and_context_survives():
    lf.lf_check_device_error()                  # start from a clean flag
    lf.lf_watchdog_selftest(22)                 # ~2 ms at 2 GHz
    with pytest.raises(lf.LfError) as ei:
        lf.lf_check_device_error()
    assert ei.value.code == lf.LF_ERR_TIMEOUT
    lf.lf_check_device_error()                  # the flag was cleared
    # the context still runs the real path correctly
    w = synthetic.TINY
    _, _, bufs = run_step(w)
    assert torch.isfinite(bufs.dq.float()).all() and torch.isfinite(bufs.o.float()).all()


@pytest.mark.gpu
def test_next_call_reports_the_expired_wait_without_a_sync():
    """An expired wait is reported by the next call of any entry point (which then
    launches nothing) until lf_sync_status clears it."""
    lf.lf_sync_status()
    w = synthetic.TINY
    inp = synthetic.make_inputs(w)
    desc, dev, bufs = run_step(w, inp)
    lf.lf_watchdog_selftest(22)
    torch.cuda.synchronize()                    # the failing kernel has finished
    marker = torch.full_like(bufs.o, 7.0)
    for _ in range(2):                          # every call until cleared
        with pytest.raises(lf.LfError) as ei:
            lf.lf_attn_fwd(desc, dev["q"], dev["k"], dev["v"], marker, bufs.lse)
        assert ei.value.code == lf.LF_ERR_TIMEOUT
    torch.cuda.synchronize()
    assert torch.all(marker == 7.0)             # nothing was launched
    with pytest.raises(lf.LfError) as ei:
        lf.lf_attn_bwd(desc, dev["q"], dev["k"], dev["v"], bufs.o, bufs.lse, dev["dout"], bufs.D,
                       bufs.w, bufs.kept_idx, bufs.kept_cnt, bufs.dq, bufs.dk, bufs.dv, bufs.ws)
    assert ei.value.code == lf.LF_ERR_TIMEOUT
    with pytest.raises(lf.LfError) as ei:
        lf.lf_sync_status()
    assert ei.value.code == lf.LF_ERR_TIMEOUT
    lf.lf_sync_status()                         # cleared
    lf.lf_attn_fwd(desc, dev["q"], dev["k"], dev["v"], marker, bufs.lse)
    lf.lf_sync_status()
    assert torch.equal(marker, bufs.o)


@pytest.mark.gpu
def test_bad_segment_table_is_reported_by_the_next_call():
    """cu_seqlens that disagree with total_tokens (a segment ending past T) are found on
    the device: the kernels skip that segment without touching its rows, and the next
    call returns LF_ERR_INVALID_ARG until lf_sync_status clears it."""
    lf.lf_sync_status()
    w = synthetic.TINY
    inp = synthetic.make_inputs(w)
    desc, dev, bufs = run_step(w, inp)
    bad_cu = torch.tensor([0, w.total_tokens + 64], dtype=torch.int32, device="cuda")
    bad = lf.make_desc(bad_cu, w.total_tokens + 64, w.total_tokens, w.hq, w.hkv, w.d, w.scale,
                       w.causal, w.block)
    lf.lf_attn_fwd(bad, dev["q"], dev["k"], dev["v"], bufs.o, bufs.lse)
    torch.cuda.synchronize()
    with pytest.raises(lf.LfError) as ei:
        lf.lf_attn_fwd(desc, dev["q"], dev["k"], dev["v"], bufs.o, bufs.lse)
    assert ei.value.code == lf.LF_ERR_INVALID_ARG
    with pytest.raises(lf.LfError) as ei:
        lf.lf_sync_status()
    assert ei.value.code == lf.LF_ERR_INVALID_ARG
    lf.lf_sync_status()
    _, _, again = run_step(w, inp)
    assert torch.equal(again.o, bufs.o)
