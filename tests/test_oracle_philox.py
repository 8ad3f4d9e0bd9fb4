"""Pins of the oracle's Philox4x32-10 draw (the random keep decision of the
LazyFlash selection, article section "Un budget sur la masse de gradient, et un
tirage qui garde le gradient non biaisé")."""
import os

import numpy as np

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")


def _kat():
    rows = []
    for line in open(GOLD):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        w = [int(x, 16) for x in line.split()]
        rows.append((w[0:4], w[4:6], w[6:10]))
    return rows


def test_known_answer_vectors():
    rows = _kat()
    assert len(rows) == 3
    for ctr, key, want in rows:
        got = oracle.philox4x32_10(ctr, key)
        assert [int(x) for x in got] == want


def test_block_u24_is_word0_shifted():
    # counter = (block, head, segment, step mod 2^32), key = (seed lo, seed hi)
    seed, step = 0x0123456789ABCDEF, (1 << 32) + 7
    for (s, h, i) in [(0, 0, 0), (3, 17, 255), (9, 31, 111)]:
        w = oracle.philox4x32_10([i, h, s, step & 0xFFFFFFFF], [seed & 0xFFFFFFFF, seed >> 32])
        assert oracle.block_u24(seed, step, s, h, i) == int(w[0]) >> 8


def test_u24_uniformity_chi2():
    # 64 equal bins over 2^24; 32768 draws over varying block/head/step.
    n, bins = 32768, 64
    counts = np.zeros(bins, dtype=np.int64)
    for j in range(n):
        u = oracle.block_u24(0, j // 256, 0, (j // 16) % 16, j % 16)
        counts[u >> 18] += 1
    e = n / bins
    chi2 = float(((counts - e) ** 2 / e).sum())
    # 63 degrees of freedom: mean 63, sd ~11.2; 130 is far in the tail (p < 1e-6)
    assert chi2 < 130.0, chi2


def test_streams_differ_across_step_head_segment():
    a = [oracle.block_u24(5, 0, 0, 0, i) for i in range(64)]
    b = [oracle.block_u24(5, 1, 0, 0, i) for i in range(64)]
    c = [oracle.block_u24(5, 0, 0, 1, i) for i in range(64)]
    d = [oracle.block_u24(5, 0, 1, 0, i) for i in range(64)]
    e = [oracle.block_u24(6, 0, 0, 0, i) for i in range(64)]
    for other in (b, c, d, e):
        assert sum(x == y for x, y in zip(a, other)) <= 1
