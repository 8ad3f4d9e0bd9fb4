"""Python binding of the LazyFlash C ABI (include/lazyflash.h).

Argument marshalling only: every step of the path runs in the CUDA kernels of
liblazyflash.so.  PyTorch provides device memory and streams.  There is no CPU
fallback: importing the binding without the built library raises.

Functions keep the C names: lf_attn_fwd, lf_block_select, lf_attn_bwd,
lf_workspace_size, lf_sync_status (alias lf_check_device_error),
lf_status_string.  Tensors are torch
CUDA tensors in the layouts the header states; the stream defaults to torch's
current stream.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblazyflash.so")

LF_OK, LF_ERR_INVALID_ARG, LF_ERR_UNSUPPORTED, LF_ERR_WORKSPACE, LF_ERR_CUDA, LF_ERR_TIMEOUT = range(6)
LF_WS_FWD, LF_WS_SELECT, LF_WS_BWD = 0, 1, 2
LF_SELECT_NORMS_GIVEN = 0x1
LF_RULE_BUDGET, LF_RULE_FIXED_FRACTION, LF_RULE_TOPK = 0, 1, 2

EXPORTED = ("lf_workspace_size", "lf_attn_fwd", "lf_block_select", "lf_attn_bwd",
            "lf_sync_status", "lf_check_device_error", "lf_status_string")


class LfError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__("%s: %s" % (what, lf_status_string(code)))
        self.code = code


class lf_attn_desc(ctypes.Structure):
    _fields_ = [
        ("nseq", ctypes.c_int32),
        ("cu_seqlens", ctypes.c_void_p),
        ("max_seqlen", ctypes.c_int32),
        ("total_tokens", ctypes.c_int32),
        ("hq", ctypes.c_int32),
        ("hkv", ctypes.c_int32),
        ("d", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float),
        ("causal", ctypes.c_int32),
        ("block_q", ctypes.c_int32),
    ]


_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError("liblazyflash.so is not built (run __graft_entry__.build()); "
                          "there is no fallback path")
    L = ctypes.CDLL(LIB_PATH)
    vp, sz, i32, u32, u64, dbl = (ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_uint32,
                                  ctypes.c_uint64, ctypes.c_double)
    dptr = ctypes.POINTER(lf_attn_desc)
    L.lf_status_string.argtypes = [i32]
    L.lf_status_string.restype = ctypes.c_char_p
    L.lf_workspace_size.argtypes = [dptr, i32, ctypes.POINTER(sz)]
    L.lf_workspace_size.restype = i32
    L.lf_attn_fwd.argtypes = [dptr, vp, vp, vp, vp, vp, vp, sz, vp]
    L.lf_attn_fwd.restype = i32
    L.lf_block_select.argtypes = [dptr, vp, vp, dbl, u64, u64, u32, vp, vp, vp, vp, vp, vp, vp,
                                  vp, sz, vp]
    L.lf_block_select.restype = i32
    L.lf_attn_bwd.argtypes = [dptr, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.lf_attn_bwd.restype = i32
    L.lf_check_device_error.argtypes = [vp]
    L.lf_check_device_error.restype = i32
    L.lf_sync_status.argtypes = [vp]
    L.lf_sync_status.restype = i32
    _lib = L
    return L


def lib():
    return _load()


def lf_status_string(code: int) -> str:
    return _load().lf_status_string(int(code)).decode()


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(code: int, what: str):
    if code != LF_OK:
        raise LfError(code, what)


def make_desc(cu_seqlens: torch.Tensor, max_seqlen: int, total_tokens: int, hq: int, hkv: int,
              d: int, softmax_scale: float, causal: bool = True, block_q: int = 128) -> lf_attn_desc:
    """cu_seqlens must be an int32 CUDA tensor that outlives every call using the desc."""
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda:
        raise ValueError("cu_seqlens must be an int32 CUDA tensor")
    desc = lf_attn_desc(cu_seqlens.numel() - 1, cu_seqlens.data_ptr(), int(max_seqlen),
                        int(total_tokens), hq, hkv, d, float(softmax_scale), int(bool(causal)),
                        block_q)
    desc._keepalive = cu_seqlens
    return desc


def lf_workspace_size(desc: lf_attn_desc, which: int) -> int:
    n = ctypes.c_size_t(0)
    _check(_load().lf_workspace_size(ctypes.byref(desc), which, ctypes.byref(n)), "lf_workspace_size")
    return n.value


def lf_attn_fwd(desc, q, k, v, o, lse, ws=None, stream=None):
    _check(_load().lf_attn_fwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                               _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                               _stream(stream)), "lf_attn_fwd")


def lf_block_select(desc, dout, o, delta, seed, step, flags, block_norm, D, tau, block_weight,
                    keep, kept_idx, kept_cnt, ws=None, stream=None):
    _check(_load().lf_block_select(ctypes.byref(desc), _ptr(dout), _ptr(o), float(delta),
                                   int(seed) & (2**64 - 1), int(step) & (2**64 - 1), int(flags),
                                   _ptr(block_norm), _ptr(D), _ptr(tau), _ptr(block_weight),
                                   _ptr(keep), _ptr(kept_idx), _ptr(kept_cnt), _ptr(ws),
                                   0 if ws is None else ws.numel() * ws.element_size(),
                                   _stream(stream)), "lf_block_select")


def lf_block_select_rule(desc, dout, o, rule, param, seed, step, flags, block_norm, D, tau,
                         block_weight, keep, kept_idx, kept_cnt, ws=None, stream=None):
    L = _load()
    fn = L.lf_block_select_rule
    fn.argtypes = [ctypes.POINTER(lf_attn_desc), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                   ctypes.c_double, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint32] + \
        [ctypes.c_void_p] * 8 + [ctypes.c_size_t, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    _check(fn(ctypes.byref(desc), _ptr(dout), _ptr(o), int(rule), float(param),
              int(seed) & (2**64 - 1), int(step) & (2**64 - 1), int(flags), _ptr(block_norm),
              _ptr(D), _ptr(tau), _ptr(block_weight), _ptr(keep), _ptr(kept_idx), _ptr(kept_cnt),
              _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)),
           "lf_block_select_rule")


def lf_attn_bwd(desc, q, k, v, o, lse, dout, D, block_weight, kept_idx, kept_cnt, dq, dk, dv,
                ws, stream=None):
    _check(_load().lf_attn_bwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                               _ptr(dout), _ptr(D), _ptr(block_weight), _ptr(kept_idx),
                               _ptr(kept_cnt), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws),
                               0 if ws is None else ws.numel() * ws.element_size(),
                               _stream(stream)), "lf_attn_bwd")


def lf_watchdog_selftest(limit_log2=24, stream=None):
    L = _load()
    L.lf_watchdog_selftest.argtypes = [ctypes.c_uint32, ctypes.c_void_p]
    L.lf_watchdog_selftest.restype = ctypes.c_int
    _check(L.lf_watchdog_selftest(int(limit_log2), _stream(stream)), "lf_watchdog_selftest")


def lf_sync_status(stream=None):
    """Synchronizes the stream; raises LfError for a device-side failure of an
    earlier call (and clears it)."""
    _check(_load().lf_sync_status(_stream(stream)), "lf_sync_status")


def lf_check_device_error(stream=None):
    _check(_load().lf_check_device_error(_stream(stream)), "lf_check_device_error")


class Buffers:
    """Device buffers of one attention layer for one LazyFlash step (torch
    allocations: plumbing only).  With forward=False the forward's outputs (o, lse)
    are not allocated: the caller already holds them."""

    def __init__(self, desc: lf_attn_desc, device="cuda", forward: bool = True):
        T, hq, hkv, d = desc.total_tokens, desc.hq, desc.hkv, desc.d
        nbmax = (desc.max_seqlen + desc.block_q - 1) // desc.block_q
        bf = dict(dtype=torch.bfloat16, device=device)
        f32 = dict(dtype=torch.float32, device=device)
        self.o = torch.empty(T, hq, d, **bf) if forward else None
        self.lse = torch.empty(hq, T, **f32) if forward else None
        self.norm = torch.empty(desc.nseq, hq, nbmax, **f32)
        self.D = torch.empty(hq, T, **f32)
        self.tau = torch.empty(desc.nseq, hq, dtype=torch.float64, device=device)
        self.w = torch.empty(desc.nseq, hq, nbmax, **f32)
        self.keep = torch.empty(desc.nseq, hq, nbmax, dtype=torch.uint8, device=device)
        self.kept_idx = torch.empty(desc.nseq, hq, nbmax, dtype=torch.int32, device=device)
        self.kept_cnt = torch.empty(desc.nseq, hq, dtype=torch.int32, device=device)
        self.dq = torch.empty(T, hq, d, **bf)
        self.dk = torch.empty(T, hkv, d, **bf)
        self.dv = torch.empty(T, hkv, d, **bf)
        nws = lf_workspace_size(desc, LF_WS_BWD)
        self.ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=device)


def lazyflash_step(desc, q, k, v, dout, delta, seed, step, bufs: Buffers, flags=0, stream=None):
    """Forward, selection and sparse backward of one layer (three C-ABI calls)."""
    lf_attn_fwd(desc, q, k, v, bufs.o, bufs.lse, stream=stream)
    lf_block_select(desc, dout, bufs.o, delta, seed, step, flags, bufs.norm, bufs.D, bufs.tau,
                    bufs.w, bufs.keep, bufs.kept_idx, bufs.kept_cnt, stream=stream)
    lf_attn_bwd(desc, q, k, v, bufs.o, bufs.lse, dout, bufs.D, bufs.w, bufs.kept_idx,
                bufs.kept_cnt, bufs.dq, bufs.dk, bufs.dv, bufs.ws, stream=stream)


def lf_attn_bwd_static_ws(desc, q, k, v, o, lse, dout, D, block_weight, kept_idx, kept_cnt, dq,
                          dk, dv, stream=None):
    """lf_attn_bwd with the library's static scratch array instead of a caller
    workspace (for callers that cannot allocate; see include/lazyflash.h)."""
    L = _load()
    fn = L.lf_attn_bwd_static_ws
    fn.argtypes = [ctypes.POINTER(lf_attn_desc)] + [ctypes.c_void_p] * 14
    fn.restype = ctypes.c_int
    _check(fn(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
              _ptr(D), _ptr(block_weight), _ptr(kept_idx), _ptr(kept_cnt), _ptr(dq), _ptr(dk),
              _ptr(dv), _stream(stream)), "lf_attn_bwd_static_ws")
