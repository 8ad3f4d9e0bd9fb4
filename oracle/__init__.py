"""CPU oracle for the LazyFlash hot path -- test infrastructure only.

A plain fp64 C implementation (``lazyflash_oracle.c``) of what the path
computes, wrapped with ctypes.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline arm of ``bench.py`` may import this package.  The CUDA product
path (``block_sparse_attention_dense_b200``) never imports it and shares no
code, header, table or helper with it.

Every function takes and returns numpy arrays; floating-point inputs are
upcast to float64 (bf16 values upcast exactly).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lazyflash_oracle.c")
_LIB = os.path.join(_HERE, "liblfo.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle (gcc, -O2, OpenMP, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
            "-fno-fast-math", "-Wall", "-o", tmp, _SRC, "-lm",
        ])
        os.replace(tmp, _LIB)
    return _LIB


def build_variant(mutant: int, out_path: str) -> str:
    """Compile the oracle with planted mistake number ``mutant`` (tests only)."""
    subprocess.check_call([
        "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
        "-fno-fast-math", "-DLFO_MUTANT=%d" % int(mutant), "-o", out_path, _SRC, "-lm",
    ])
    return out_path


def use_library(path):
    """Point this module at another build of the oracle (None: the default).
    Returns the previous handle so that the caller can restore it."""
    global _lib
    with _lock:
        prev = _lib
        _lib = None if path is None else _declare(ctypes.CDLL(path))
    return prev


def restore_library(prev):
    global _lib
    with _lock:
        _lib = prev


def lib():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _declare(ctypes.CDLL(build()))
    return _lib


def _declare(L):
    """Declares the C signatures on a loaded oracle library."""
    dp = ctypes.POINTER(ctypes.c_double)
    i32p = ctypes.POINTER(ctypes.c_int32)
    u32p = ctypes.POINTER(ctypes.c_uint32)
    c_int, c_dbl = ctypes.c_int, ctypes.c_double
    L.lfo_philox4x32_10.argtypes = [u32p, u32p, u32p]
    L.lfo_philox4x32_10.restype = None
    L.lfo_block_u24.argtypes = [ctypes.c_uint64, ctypes.c_uint64, c_int, c_int, c_int]
    L.lfo_block_u24.restype = ctypes.c_uint32
    L.lfo_attn_fwd.argtypes = [c_int, i32p, c_int, c_int, c_int, c_int, c_dbl, c_int,
                               dp, dp, dp, dp, dp]
    L.lfo_block_norms.argtypes = [c_int, i32p, c_int, c_int, c_int, c_int, c_int, dp, dp]
    L.lfo_rowdot.argtypes = [c_int, c_int, c_int, dp, dp, dp]
    L.lfo_pinned_sum.argtypes = [dp, c_int]
    L.lfo_pinned_sum.restype = c_dbl
    L.lfo_tau.argtypes = [dp, c_int, c_dbl]
    L.lfo_tau.restype = c_dbl
    L.lfo_discarded_mass.argtypes = [dp, c_int, c_dbl, dp]
    L.lfo_discarded_mass.restype = c_dbl
    L.lfo_select.argtypes = [c_int, i32p, c_int, c_int, dp, c_dbl, ctypes.c_uint64,
                             ctypes.c_uint64, dp, dp, ctypes.POINTER(ctypes.c_float),
                             ctypes.POINTER(ctypes.c_uint8), i32p, i32p]
    L.lfo_attn_bwd.argtypes = [c_int, i32p, c_int, c_int, c_int, c_int, c_dbl, c_int,
                               c_int, c_int, dp, dp, dp, dp, dp, dp, dp, dp]
    L.lfo_select_rule.argtypes = [c_int, c_int, i32p, c_int, c_int, dp, c_dbl,
                                  ctypes.c_uint64, ctypes.c_uint64, dp, dp,
                                  ctypes.POINTER(ctypes.c_float),
                                  ctypes.POINTER(ctypes.c_uint8), i32p, i32p]
    L.lfo_tau_fixed_fraction.argtypes = [dp, c_int, c_dbl]
    L.lfo_tau_fixed_fraction.restype = c_dbl
    L.lfo_expected_kept.argtypes = [dp, c_int, c_dbl, dp]
    L.lfo_expected_kept.restype = c_dbl
    L.lfo_attn_fwd_rows.argtypes = [c_int, i32p, c_int, c_int, c_int, c_int, c_dbl, c_int,
                                    dp, dp, dp, c_int, i32p, i32p, dp, dp]
    L.lfo_attn_bwd_rows.argtypes = [c_int, i32p, c_int, c_int, c_int, c_int, c_dbl, c_int,
                                    c_int, c_int, dp, dp, dp, dp, dp,
                                    c_int, i32p, i32p, dp, c_int, i32p, i32p, dp, dp]
    return L


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").numpy()
    return np.ascontiguousarray(a, dtype=np.int32)


def _p(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def _check(rc, what):
    if rc != 0:
        raise ValueError("oracle %s rejected its arguments (code %d)" % (what, rc))


def philox4x32_10(ctr, key) -> np.ndarray:
    c = np.ascontiguousarray(ctr, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.zeros(4, dtype=np.uint32)
    lib().lfo_philox4x32_10(_p(c, ctypes.c_uint32), _p(k, ctypes.c_uint32), _p(out, ctypes.c_uint32))
    return out


def block_u24(seed: int, step: int, s: int, h: int, i: int) -> int:
    return int(lib().lfo_block_u24(seed, step, s, h, i))


def attn_fwd(cu_seqlens, q, k, v, scale: float, causal: bool = True):
    """Dense attention: returns (o [T,Hq,d] f64, lse [Hq,T] f64)."""
    cu = _i32(cu_seqlens)
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, hq, d = q.shape
    hkv = k.shape[1]
    o = np.zeros_like(q)
    lse = np.zeros((hq, T), dtype=np.float64)
    dp = ctypes.c_double
    _check(lib().lfo_attn_fwd(len(cu) - 1, _p(cu, ctypes.c_int32), T, hq, hkv, d, scale, int(causal),
                              _p(q, dp), _p(k, dp), _p(v, dp), _p(o, dp), _p(lse, dp)), "attn_fwd")
    return o, lse


def nblocks(cu_seqlens, block: int) -> np.ndarray:
    cu = _i32(cu_seqlens)
    lens = np.diff(cu.astype(np.int64))
    return ((lens + block - 1) // block).astype(np.int32)


def block_norms(cu_seqlens, dout, block: int, nbmax: int | None = None) -> np.ndarray:
    cu = _i32(cu_seqlens)
    do = _f64(dout)
    T, hq, d = do.shape
    nb = nblocks(cu, block)
    nbmax = int(nb.max()) if nbmax is None else nbmax
    out = np.zeros((len(cu) - 1, hq, nbmax), dtype=np.float64)
    dp = ctypes.c_double
    _check(lib().lfo_block_norms(len(cu) - 1, _p(cu, ctypes.c_int32), T, hq, d, block, nbmax,
                                 _p(do, dp), _p(out, dp)), "block_norms")
    return out


def rowdot(dout, o) -> np.ndarray:
    do, o = _f64(dout), _f64(o)
    T, hq, d = do.shape
    D = np.zeros((hq, T), dtype=np.float64)
    dp = ctypes.c_double
    lib().lfo_rowdot(T, hq, d, _p(do, dp), _p(o, dp), _p(D, dp))
    return D


def pinned_sum(x) -> float:
    x = _f64(x)
    return float(lib().lfo_pinned_sum(_p(x, ctypes.c_double), len(x)))


def tau(m, delta: float) -> float:
    m = _f64(m)
    return float(lib().lfo_tau(_p(m, ctypes.c_double), len(m), delta))


def discarded_mass(m, tau_: float) -> float:
    m = _f64(m)
    scratch = np.zeros(max(1, len(m)), dtype=np.float64)
    return float(lib().lfo_discarded_mass(_p(m, ctypes.c_double), len(m), tau_,
                                          _p(scratch, ctypes.c_double)))


def select(norms, nb, delta: float, seed: int, step: int) -> dict:
    """Budgeted proportional selection for norms [nseq, hq, nbmax]."""
    m = _f64(norms)
    nseq, hq, nbmax = m.shape
    nb = _i32(nb)
    out = {
        "tau": np.zeros((nseq, hq), dtype=np.float64),
        "p": np.zeros((nseq, hq, nbmax), dtype=np.float64),
        "w": np.zeros((nseq, hq, nbmax), dtype=np.float32),
        "keep": np.zeros((nseq, hq, nbmax), dtype=np.uint8),
        "kept_idx": np.zeros((nseq, hq, nbmax), dtype=np.int32),
        "kept_cnt": np.zeros((nseq, hq), dtype=np.int32),
    }
    dp = ctypes.c_double
    _check(lib().lfo_select(nseq, _p(nb, ctypes.c_int32), hq, nbmax, _p(m, dp), float(delta),
                            int(seed) & (2**64 - 1), int(step) & (2**64 - 1),
                            _p(out["tau"], dp), _p(out["p"], dp), _p(out["w"], ctypes.c_float),
                            _p(out["keep"], ctypes.c_uint8), _p(out["kept_idx"], ctypes.c_int32),
                            _p(out["kept_cnt"], ctypes.c_int32)), "select")
    return out


def attn_bwd(cu_seqlens, q, k, v, dout, scale: float, block: int, wblk=None,
             causal: bool = True):
    """Gradient of sum_t <w_b(t) dO_t, O_t>: returns (dq, dk, dv) in f64.

    ``wblk`` is [nseq, hq, nbmax] (None = all ones, the dense backward)."""
    cu = _i32(cu_seqlens)
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(dout)
    T, hq, d = q.shape
    hkv = k.shape[1]
    nb = nblocks(cu, block)
    if wblk is not None:
        wb = _f64(wblk)
        nbmax = wb.shape[2]
        wptr = _p(wb, ctypes.c_double)
    else:
        nbmax = int(nb.max())
        wptr = None
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dp = ctypes.c_double
    _check(lib().lfo_attn_bwd(len(cu) - 1, _p(cu, ctypes.c_int32), T, hq, hkv, d, scale, int(causal),
                              block, nbmax, _p(q, dp), _p(k, dp), _p(v, dp), _p(do, dp), wptr,
                              _p(dq, dp), _p(dk, dp), _p(dv, dp)), "attn_bwd")
    return dq, dk, dv


def attn_fwd_rows(cu_seqlens, q, k, v, scale: float, rows, heads, causal: bool = True):
    """O [n, d] and LSE [n] of query rows (rows[i], heads[i]) only."""
    cu = _i32(cu_seqlens)
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, hq, d = q.shape
    hkv = k.shape[1]
    rows, heads = _i32(rows), _i32(heads)
    n = len(rows)
    o = np.zeros((n, d), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    dp, ip = ctypes.c_double, ctypes.c_int32
    _check(lib().lfo_attn_fwd_rows(len(cu) - 1, _p(cu, ip), T, hq, hkv, d, scale, int(causal),
                                   _p(q, dp), _p(k, dp), _p(v, dp), n, _p(rows, ip), _p(heads, ip),
                                   _p(o, dp), _p(lse, dp)), "attn_fwd_rows")
    return o, lse


def attn_bwd_rows(cu_seqlens, q, k, v, dout, scale: float, block: int, wblk, qrows, qheads,
                  kvrows, kvheads, causal: bool = True):
    """dQ at query rows (qrows, qheads) and dK, dV at KV rows (kvrows, kvheads)."""
    cu = _i32(cu_seqlens)
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(dout)
    T, hq, d = q.shape
    hkv = k.shape[1]
    nb = nblocks(cu, block)
    if wblk is not None:
        wb = _f64(wblk)
        nbmax = wb.shape[2]
        wptr = _p(wb, ctypes.c_double)
    else:
        nbmax = int(nb.max())
        wptr = None
    qrows, qheads, kvrows, kvheads = _i32(qrows), _i32(qheads), _i32(kvrows), _i32(kvheads)
    dq = np.zeros((len(qrows), d))
    dk = np.zeros((len(kvrows), d))
    dv = np.zeros((len(kvrows), d))
    dp, ip = ctypes.c_double, ctypes.c_int32
    _check(lib().lfo_attn_bwd_rows(len(cu) - 1, _p(cu, ip), T, hq, hkv, d, scale, int(causal),
                                   block, nbmax, _p(q, dp), _p(k, dp), _p(v, dp), _p(do, dp), wptr,
                                   len(qrows), _p(qrows, ip), _p(qheads, ip), _p(dq, dp),
                                   len(kvrows), _p(kvrows, ip), _p(kvheads, ip), _p(dk, dp),
                                   _p(dv, dp)), "attn_bwd_rows")
    return dq, dk, dv


RULE_BUDGET, RULE_FIXED_FRACTION, RULE_TOPK = 0, 1, 2


def select_rule(rule: int, norms, nb, param: float, seed: int, step: int) -> dict:
    """Selection by rule 0 (budget delta = param), 1 (fixed fraction f = param)
    or 2 (top-k with k = ceil(param * n)); same outputs as select()."""
    m = _f64(norms)
    nseq, hq, nbmax = m.shape
    nb = _i32(nb)
    out = {
        "tau": np.zeros((nseq, hq), dtype=np.float64),
        "p": np.zeros((nseq, hq, nbmax), dtype=np.float64),
        "w": np.zeros((nseq, hq, nbmax), dtype=np.float32),
        "keep": np.zeros((nseq, hq, nbmax), dtype=np.uint8),
        "kept_idx": np.zeros((nseq, hq, nbmax), dtype=np.int32),
        "kept_cnt": np.zeros((nseq, hq), dtype=np.int32),
    }
    dp = ctypes.c_double
    _check(lib().lfo_select_rule(int(rule), nseq, _p(nb, ctypes.c_int32), hq, nbmax, _p(m, dp),
                                 float(param), int(seed) & (2**64 - 1), int(step) & (2**64 - 1),
                                 _p(out["tau"], dp), _p(out["p"], dp), _p(out["w"], ctypes.c_float),
                                 _p(out["keep"], ctypes.c_uint8), _p(out["kept_idx"], ctypes.c_int32),
                                 _p(out["kept_cnt"], ctypes.c_int32)), "select_rule")
    return out


def tau_fixed_fraction(m, f: float) -> float:
    m = _f64(m)
    return float(lib().lfo_tau_fixed_fraction(_p(m, ctypes.c_double), len(m), f))
