"""Seeded synthetic workloads shared by the tests, the bench and the oracle runs.

This module only draws numbers and lays them out. It holds none of the
method's arithmetic: no attention, no norms, no budget, no random keep draw.
Both the CUDA path and the CPU oracle receive the arrays built here.

Recipe (the article's LongAlign/Qwen3-8B training data is not available, so
seeded tensors with the same attention shapes stand in for it):

* ``numpy.random.SeedSequence(seed)`` spawns five independent PCG64 streams:
  Q, K, V and a base dO as float32 standard normals (row-major, so the first
  rows of a tensor never depend on how many rows follow), and one
  LogNormal(0, sigma) scale per (segment, query head, block of ``block``
  rows); every dO row of a block is multiplied by that block's scale.  The skewed per-block scale reproduces the
  uneven spread of output-gradient mass across query blocks that the LazyFlash
  article builds on ("Le passage arrière fait deux fois le travail du passage
  avant").
* All four tensors are rounded to bfloat16 (round to nearest even, by torch).
  The same bf16 values go to the GPU and, upcast exactly to float64, to the
  oracle.
* Packed variable-length batches draw their segment lengths from a separate
  ``PCG64(seed)`` generator as uniform integers in ``[lo, hi]`` until the
  total is reached; the last segment is clipped.

Layout ("THD"): every token tensor is ``[T, H, d]`` row-major; segments are
delimited by ``cu_seqlens`` (int32, ``nseq + 1`` entries).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seqlens: tuple            # lengths of the packed segments
    hq: int
    hkv: int
    d: int
    block: int                # selection block (query rows per block)
    sigma: float              # LogNormal sigma of the per-block dO scale
    delta: float              # gradient-mass budget
    causal: bool = True
    seed: int = 0

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens))

    @property
    def nseq(self) -> int:
        return len(self.seqlens)

    @property
    def max_seqlen(self) -> int:
        return int(max(self.seqlens))

    @property
    def nbmax(self) -> int:
        return (self.max_seqlen + self.block - 1) // self.block

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def cu_seqlens(self) -> np.ndarray:
        cu = np.zeros(self.nseq + 1, dtype=np.int32)
        cu[1:] = np.cumsum(np.asarray(self.seqlens, dtype=np.int64))
        return cu

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def varlen_lengths(total: int, lo: int, hi: int, seed: int = 0) -> tuple:
    """Segment lengths ~ Uniform{lo..hi} drawn until ``total``; last one clipped."""
    rng = np.random.Generator(np.random.PCG64(seed))
    out: List[int] = []
    acc = 0
    while acc < total:
        n = int(rng.integers(lo, hi, endpoint=True))
        n = min(n, total - acc)
        out.append(n)
        acc += n
    return tuple(out)


# The five workloads of the measurement plan.  Only their attention shapes come
# from the article's Qwen3-8B setting (32 query heads, 8 KV heads, head dim 128).
TINY = Workload("tiny", (512,), hq=2, hkv=2, d=64, block=64, sigma=1.5, delta=0.1)
GQA_MID = Workload("gqa_mid", (4096,), hq=32, hkv=8, d=128, block=128, sigma=1.5, delta=0.05)
LONG = Workload("long", (16384,), hq=32, hkv=8, d=128, block=128, sigma=1.5, delta=0.05)
HEADLINE = Workload("headline", (32768,), hq=32, hkv=8, d=128, block=128, sigma=2.0, delta=0.1)
VARLEN = Workload("varlen", varlen_lengths(65536, 2048, 16384, seed=0), hq=32, hkv=8, d=128,
                  block=128, sigma=1.5, delta=0.2)
LONG_DELTAS = (0.0, 0.05, 0.2)

WORKLOADS = {w.name: w for w in (TINY, GQA_MID, LONG, HEADLINE, VARLEN)}


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(a).to(torch.bfloat16)


def make_inputs(w: Workload, seed: Optional[int] = None, rows: Optional[int] = None) -> dict:
    """Host bf16 tensors q, k, v, dout (THD) plus cu_seqlens for workload ``w``.

    ``rows`` < T returns only the first ``rows`` tokens (identical to the same
    rows of the full draw) with a single segment; it requires ``w`` to have one
    segment, so that a causal prefix is itself a complete problem."""
    seed = w.seed if seed is None else seed
    streams = [np.random.Generator(np.random.PCG64(c))
               for c in np.random.SeedSequence(seed).spawn(5)]
    T = w.total_tokens if rows is None else int(rows)
    if rows is not None and (w.nseq != 1 or not 0 < T <= w.total_tokens):
        raise ValueError("a prefix needs a single-segment workload and 0 < rows <= T")
    q = streams[0].standard_normal((T, w.hq, w.d), dtype=np.float32)
    k = streams[1].standard_normal((T, w.hkv, w.d), dtype=np.float32)
    v = streams[2].standard_normal((T, w.hkv, w.d), dtype=np.float32)
    do = streams[3].standard_normal((T, w.hq, w.d), dtype=np.float32)
    scales = streams[4].lognormal(0.0, w.sigma, size=(w.nseq, w.hq, w.nbmax)).astype(np.float32)
    cu = w.cu_seqlens() if rows is None else np.array([0, T], dtype=np.int32)
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        nb = (b - a + w.block - 1) // w.block
        for i in range(nb):
            r0, r1 = a + i * w.block, min(a + (i + 1) * w.block, b)
            do[r0:r1] *= scales[s, :, i][None, :, None]
    return {
        "q": _bf16(q), "k": _bf16(k), "v": _bf16(v), "dout": _bf16(do),
        "cu_seqlens": torch.from_numpy(cu),
    }


def random_norms(nseq: int, hq: int, nbmax: int, nb_per_seq, sigma: float, seed: int) -> np.ndarray:
    """A float32 block-norm array [nseq, hq, nbmax] (zeros past each segment's
    block count), for tests that feed the same norms to both sides."""
    rng = np.random.Generator(np.random.PCG64(seed))
    m = rng.lognormal(0.0, sigma, size=(nseq, hq, nbmax)).astype(np.float32)
    for s, nb in enumerate(nb_per_seq):
        m[s, :, nb:] = 0.0
    return m


def make_layer_step_inputs(w: Workload, layers: int, device, seed: int = 0) -> dict:
    """Inputs of the synthetic layer-stack step (random weights, no data set), drawn on
    ``device`` from a seeded torch generator: activations x [T, hq*d] ~ N(0, 1); per layer
    W_qkv [hq*d, (hq + 2 hkv) d] and W_o [hq*d, hq*d] ~ N(0, 1/(hq*d)); and the loss
    gradient g [T, hq*d] ~ N(0, 1) times a LogNormal(0, sigma) scale per token block,
    shared by all heads (a per-head scale would be averaged away by the output
    projection, which mixes the heads, before the gradient reaches the attention)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    T, hidden = w.total_tokens, w.hq * w.d
    nqkv = (w.hq + 2 * w.hkv) * w.d

    def normal(shape, std):
        return (torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * std).to(torch.bfloat16)

    x = normal((T, hidden), 1.0)
    wqkv = [normal((hidden, nqkv), hidden ** -0.5) for _ in range(layers)]
    wo = [normal((hidden, hidden), hidden ** -0.5) for _ in range(layers)]
    g = torch.randn((T, w.hq, w.d), generator=gen, device=device, dtype=torch.float32)
    nb = (T + w.block - 1) // w.block
    scales = torch.empty((nb,), device=device, dtype=torch.float32).log_normal_(0.0, w.sigma, generator=gen)
    g *= scales.repeat_interleave(w.block)[:T, None, None]
    cu = torch.tensor([0, T], dtype=torch.int32, device=device)
    return {"x": x, "wqkv": wqkv, "wo": wo, "g": g.reshape(T, hidden).to(torch.bfloat16), "cu_seqlens": cu}
