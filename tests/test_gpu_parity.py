"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded bf16 inputs.

Tolerances (fp32 accumulation of bf16 inputs on the GPU, fp64 in the oracle):
keep masks, weights, tau and kept lists bit-exact given the same norm vector;
block norms 1e-5 relative; O 1e-2 max-abs before its rounding to the bf16 output
(so 1e-2 plus half a bf16 ulp of the exact value: for |O| >= 4 the rounding alone
can exceed 1e-2); LSE 1e-3 abs; dQ/dK/dV 1e-2 relative Frobenius.
"""
import math

import numpy as np
import pytest
import torch

import block_sparse_attention_dense_b200 as lf
import oracle
import synthetic
from _helpers import desc_for, nb_per_seq, o_within, rel_fro, run_step, to_dev

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL, GRAD_TOL, NORM_TOL = 1e-2, 1e-3, 1e-2, 1e-5

# Small workloads the full oracle finishes in seconds; they span several tiles
# and ragged tails.
SMALL = [
    synthetic.TINY,
    synthetic.Workload("ragged_gqa", (700,), hq=4, hkv=2, d=128, block=128, sigma=1.5, delta=0.1),
    synthetic.Workload("varlen_small", (1, 130, 0, 257, 64), hq=4, hkv=1, d=64, block=64,
                       sigma=1.5, delta=0.2),
    synthetic.Workload("mha_noncausal", (300, 200), hq=2, hkv=2, d=128, block=128, sigma=1.0,
                       delta=0.05, causal=False),
    synthetic.Workload("blk64_d128", (520,), hq=4, hkv=1, d=128, block=64, sigma=2.0, delta=0.3),
    # group of 8 query heads per KV head, d = 64 with 128-row blocks, ragged tail
    synthetic.Workload("mqa_g8_d64", (600,), hq=8, hkv=1, d=64, block=128, sigma=1.5, delta=0.15),
    # GQA without the causal mask, two segments, 64-row blocks
    synthetic.Workload("gqa_noncausal", (384, 129), hq=4, hkv=2, d=64, block=64, sigma=1.5,
                       delta=0.1, causal=False),
    # three query heads per KV head: an odd group in one backward CTA; the forward's
    # head-in-group index with an odd group
    synthetic.Workload("gqa3_d128", (333, 200), hq=6, hkv=2, d=128, block=128, sigma=1.5,
                       delta=0.1),
    # exactly 32 query heads per KV head: the largest group one backward CTA walks
    # whole (every head's start search and shared-memory slot in use, dK/dV stored
    # directly as bf16), d = 128, two segments
    synthetic.Workload("mqa_g32_d128", (300, 170), hq=32, hkv=1, d=128, block=128, sigma=1.5,
                       delta=0.15),
    # 40 query heads per KV head: beyond the 32 heads one backward CTA walks, so two
    # CTAs share each KV tile and dK/dV meet in the fp32 accumulators
    synthetic.Workload("mqa_g40_d64", (300, 170), hq=40, hkv=1, d=64, block=128, sigma=1.5,
                       delta=0.2),
    # the same split group with 64-row blocks: the half-skipping backward on the
    # accumulator path
    synthetic.Workload("mqa_g40_blk64", (200, 90), hq=40, hkv=1, d=64, block=64, sigma=2.0,
                       delta=0.3),
    # 60 segments: the forward's segment search takes its multi-round path (more than 32
    # segment starts) and meets empty, one-token and tile-edge lengths (127, 128, 129, 256)
    synthetic.Workload("many_segments", (0, 1, 127, 128, 129, 256, 300, 5, 64, 200) * 6, hq=2,
                       hkv=1, d=64, block=64, sigma=1.5, delta=0.2),
]


def _cpu(t):
    return t.detach().float().cpu().numpy()


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_forward_matches_oracle(w):
    inp = synthetic.make_inputs(w)
    desc, dev, bufs = run_step(w, inp)
    o_ref, lse_ref = oracle.attn_fwd(w.cu_seqlens(), inp["q"], inp["k"], inp["v"], w.scale, w.causal)
    o = _cpu(bufs.o)
    lse = _cpu(bufs.lse)
    assert o_within(o, o_ref, O_TOL)[0], o_within(o, o_ref, O_TOL)
    assert np.abs(lse - lse_ref).max() < LSE_TOL


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_norms_and_rowdot_match_oracle(w):
    inp = synthetic.make_inputs(w)
    desc, dev, bufs = run_step(w, inp)
    cu = w.cu_seqlens()
    m_ref = oracle.block_norms(cu, inp["dout"], w.block, w.nbmax)
    m = _cpu(bufs.norm)
    assert np.all(np.abs(m - m_ref) <= NORM_TOL * np.maximum(m_ref, 1e-30))
    # D from the same bf16 O the GPU stored
    D_ref = oracle.rowdot(inp["dout"], bufs.o.cpu())
    D = _cpu(bufs.D)
    scale = np.sqrt(oracle.rowdot(inp["dout"], inp["dout"]) * oracle.rowdot(bufs.o.cpu(), bufs.o.cpu()))
    assert np.all(np.abs(D - D_ref) <= 1e-5 * scale + 1e-30)


@pytest.mark.parametrize("w", [SMALL[2], SMALL[7]], ids=lambda w: w.name)
def test_max_seqlen_above_the_longest_segment(w):
    """max_seqlen is an upper bound on the segment lengths: three times the longest
    (more KV-tile CTAs, forward work units and per-block slots than any segment uses)
    gives the oracle's results, with the slots past each segment's blocks empty."""
    inp = synthetic.make_inputs(w)
    dev = to_dev(inp)
    big = 3 * w.max_seqlen + 5
    desc = lf.make_desc(dev["cu_seqlens"], big, w.total_tokens, w.hq, w.hkv, w.d, w.scale,
                        w.causal, w.block)
    bufs = lf.Buffers(desc)
    lf.lazyflash_step(desc, dev["q"], dev["k"], dev["v"], dev["dout"], w.delta, 3, 1, bufs)
    lf.lf_check_device_error()
    torch.cuda.synchronize()
    cu, nb = w.cu_seqlens(), nb_per_seq(w)
    assert bufs.norm.shape[2] == (big + w.block - 1) // w.block
    o_ref, lse_ref = oracle.attn_fwd(cu, inp["q"], inp["k"], inp["v"], w.scale, w.causal)
    assert o_within(_cpu(bufs.o), o_ref, O_TOL)[0], o_within(_cpu(bufs.o), o_ref, O_TOL)
    assert np.abs(_cpu(bufs.lse) - lse_ref).max() < LSE_TOL
    m = _cpu(bufs.norm)
    m_ref = oracle.block_norms(cu, inp["dout"], w.block, m.shape[2])
    assert np.all(np.abs(m - m_ref) <= NORM_TOL * np.maximum(m_ref, 1e-30))
    sel = oracle.select(m, nb, w.delta, 3, 1)
    np.testing.assert_array_equal(bufs.keep.cpu().numpy(), sel["keep"])
    np.testing.assert_array_equal(bufs.w.cpu().numpy(), sel["w"])
    np.testing.assert_array_equal(bufs.kept_cnt.cpu().numpy(), sel["kept_cnt"])
    dq_ref, dk_ref, dv_ref = oracle.attn_bwd(cu, inp["q"], inp["k"], inp["v"], inp["dout"],
                                             w.scale, w.block, sel["w"].astype(np.float64),
                                             w.causal)
    assert rel_fro(_cpu(bufs.dq), dq_ref) < GRAD_TOL
    assert rel_fro(_cpu(bufs.dk), dk_ref) < GRAD_TOL
    assert rel_fro(_cpu(bufs.dv), dv_ref) < GRAD_TOL


def _select_case(nseq_lens, hq, block, sigma, seed):
    w = synthetic.Workload("sel", tuple(nseq_lens), hq=hq, hkv=1 if hq % 2 else 2, d=64,
                           block=block, sigma=sigma, delta=0.1)
    nb = nb_per_seq(w)
    m = synthetic.random_norms(w.nseq, hq, w.nbmax, nb, sigma, seed)
    return w, nb, m


@pytest.mark.parametrize("case", [
    ((512,), 2, 64, 1.5),
    ((32768,), 32, 128, 2.0),
    (synthetic.VARLEN.seqlens, 32, 128, 1.5),
    ((65536,), 4, 64, 2.0),
    ((1, 100, 0, 5000), 8, 128, 0.5),
], ids=["tiny", "headline", "varlen", "blk64_1024", "odd"])
@pytest.mark.parametrize("delta", [0.0, 0.05, 0.1, 0.4, 0.95])
def test_selection_bit_exact_given_norms(case, delta):
    lens, hq, block, sigma = case
    w, nb, m = _select_case(lens, hq, block, sigma, seed=hq + len(lens))
    if sum(lens) == 0:
        pytest.skip("empty")
    m[0, 0, : min(3, nb[0])] = 0.0          # zero-norm blocks
    desc = desc_for(w, torch.as_tensor(w.cu_seqlens()).cuda())
    nbmax = w.nbmax
    dummy = torch.zeros(w.total_tokens, hq, 64, dtype=torch.bfloat16, device="cuda")
    norm = torch.as_tensor(m, device="cuda")
    D = torch.empty(hq, w.total_tokens, device="cuda")
    tau = torch.empty(w.nseq, hq, dtype=torch.float64, device="cuda")
    wt = torch.empty(w.nseq, hq, nbmax, device="cuda")
    keep = torch.empty(w.nseq, hq, nbmax, dtype=torch.uint8, device="cuda")
    kidx = torch.empty(w.nseq, hq, nbmax, dtype=torch.int32, device="cuda")
    kcnt = torch.empty(w.nseq, hq, dtype=torch.int32, device="cuda")
    for seed, step in [(0, 0), (0x9E3779B97F4A7C15, 12345), (7, 2**32 + 3)]:
        lf.lf_block_select(desc, dummy, dummy, delta, seed, step, lf.LF_SELECT_NORMS_GIVEN, norm, D,
                           tau, wt, keep, kidx, kcnt)
        lf.lf_check_device_error()
        ref = oracle.select(m, nb, delta, seed, step)
        np.testing.assert_array_equal(tau.cpu().numpy().view(np.uint64), ref["tau"].view(np.uint64))
        np.testing.assert_array_equal(keep.cpu().numpy(), ref["keep"])
        np.testing.assert_array_equal(wt.cpu().numpy().view(np.uint32), ref["w"].view(np.uint32))
        np.testing.assert_array_equal(kcnt.cpu().numpy(), ref["kept_cnt"])
        np.testing.assert_array_equal(kidx.cpu().numpy(), ref["kept_idx"])


def test_selection_at_the_largest_block_count():
    """The selection holds one segment's norms in shared memory as fp64 (200 KB):
    25,600 blocks is the largest count it takes, bit-exact there; one block more
    is refused before any launch."""
    nbig = 200 * 1024 // 8
    w = synthetic.Workload("sel_max", (nbig * 128,), hq=1, hkv=1, d=64, block=128, sigma=2.0,
                           delta=0.1)
    nb = nb_per_seq(w)
    m = synthetic.random_norms(1, 1, w.nbmax, nb, 2.0, seed=11)
    cu = torch.as_tensor(w.cu_seqlens()).cuda()
    desc = desc_for(w, cu)
    dummy = torch.zeros(w.total_tokens, 1, 64, dtype=torch.bfloat16, device="cuda")
    norm = torch.as_tensor(m, device="cuda")
    D = torch.empty(1, w.total_tokens, device="cuda")
    tau = torch.empty(1, 1, dtype=torch.float64, device="cuda")
    wt = torch.empty(1, 1, w.nbmax, device="cuda")
    keep = torch.empty(1, 1, w.nbmax, dtype=torch.uint8, device="cuda")
    kidx = torch.empty(1, 1, w.nbmax, dtype=torch.int32, device="cuda")
    kcnt = torch.empty(1, 1, dtype=torch.int32, device="cuda")
    lf.lf_block_select(desc, dummy, dummy, w.delta, 5, 6, lf.LF_SELECT_NORMS_GIVEN, norm, D, tau, wt,
                       keep, kidx, kcnt)
    lf.lf_check_device_error()
    ref = oracle.select(m, nb, w.delta, 5, 6)
    np.testing.assert_array_equal(tau.cpu().numpy().view(np.uint64), ref["tau"].view(np.uint64))
    np.testing.assert_array_equal(keep.cpu().numpy(), ref["keep"])
    np.testing.assert_array_equal(wt.cpu().numpy().view(np.uint32), ref["w"].view(np.uint32))
    np.testing.assert_array_equal(kcnt.cpu().numpy(), ref["kept_cnt"])
    np.testing.assert_array_equal(kidx.cpu().numpy(), ref["kept_idx"])
    w2 = w.with_(seqlens=(nbig * 128 + 1,))
    cu2 = torch.as_tensor(w2.cu_seqlens()).cuda()
    with pytest.raises(lf.LfError) as err:
        lf.lf_block_select(desc_for(w2, cu2), dummy, dummy, w.delta, 5, 6, lf.LF_SELECT_NORMS_GIVEN,
                           norm, D, tau, wt, keep, kidx, kcnt)
    assert err.value.code == lf.LF_ERR_UNSUPPORTED


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_backward_matches_oracle(w):
    inp = synthetic.make_inputs(w)
    desc, dev, bufs = run_step(w, inp, seed=3, step=1)
    cu = w.cu_seqlens()
    nb = nb_per_seq(w)
    # the GPU's keep decisions equal the oracle's on the GPU's norms
    sel = oracle.select(_cpu(bufs.norm), nb, w.delta, 3, 1)
    np.testing.assert_array_equal(bufs.keep.cpu().numpy(), sel["keep"])
    np.testing.assert_array_equal(bufs.w.cpu().numpy(), sel["w"])
    dq_ref, dk_ref, dv_ref = oracle.attn_bwd(cu, inp["q"], inp["k"], inp["v"], inp["dout"],
                                             w.scale, w.block, sel["w"].astype(np.float64),
                                             w.causal)
    assert rel_fro(_cpu(bufs.dq), dq_ref) < GRAD_TOL
    assert rel_fro(_cpu(bufs.dk), dk_ref) < GRAD_TOL
    assert rel_fro(_cpu(bufs.dv), dv_ref) < GRAD_TOL
    # rows of dropped blocks get exactly zero dQ
    dq = bufs.dq.cpu()
    for s in range(w.nseq):
        for h in range(w.hq):
            for b in range(int(nb[s])):
                if sel["keep"][s, h, b] == 0:
                    r0 = cu[s] + b * w.block
                    r1 = min(cu[s] + (b + 1) * w.block, cu[s + 1])
                    assert torch.all(dq[r0:r1, h] == 0)


@pytest.mark.parametrize("w", SMALL[:2], ids=lambda w: w.name)
def test_delta_zero_is_the_dense_backward(w):
    inp = synthetic.make_inputs(w)
    desc, dev, bufs = run_step(w, inp, delta=0.0)
    assert torch.all(bufs.keep.cpu()[:, :, : int(nb_per_seq(w).max())] == 1)
    dq_ref, dk_ref, dv_ref = oracle.attn_bwd(w.cu_seqlens(), inp["q"], inp["k"], inp["v"],
                                             inp["dout"], w.scale, w.block, None, w.causal)
    assert rel_fro(_cpu(bufs.dq), dq_ref) < GRAD_TOL
    assert rel_fro(_cpu(bufs.dk), dk_ref) < GRAD_TOL
    assert rel_fro(_cpu(bufs.dv), dv_ref) < GRAD_TOL


def test_heavy_budget_leaves_unreached_kv_tiles_zero():
    w = synthetic.Workload("heavy", (1024,), hq=2, hkv=1, d=128, block=128, sigma=3.0, delta=0.95)
    inp = synthetic.make_inputs(w)
    desc, dev, bufs = run_step(w, inp, seed=1)
    sel = oracle.select(_cpu(bufs.norm), nb_per_seq(w), w.delta, 1, 0)
    dq_ref, dk_ref, dv_ref = oracle.attn_bwd(w.cu_seqlens(), inp["q"], inp["k"], inp["v"],
                                             inp["dout"], w.scale, w.block,
                                             sel["w"].astype(np.float64), True)
    assert rel_fro(_cpu(bufs.dk), dk_ref) < GRAD_TOL
    assert rel_fro(_cpu(bufs.dv), dv_ref) < GRAD_TOL
    assert rel_fro(_cpu(bufs.dq), dq_ref) < GRAD_TOL
    # a KV tile is reached only by kept blocks at or after it (causal)
    kept = sel["keep"][0, :, :]
    for j in range(8):
        if not kept[:, j:].any():
            assert torch.all(bufs.dk[j * 128:(j + 1) * 128] == 0)
            assert torch.all(bufs.dv[j * 128:(j + 1) * 128] == 0)


@pytest.mark.parametrize("block", [64, 128])
def test_noncausal_keys_of_the_next_segment_stay_out(block):
    """Without the causal mask, the last KV tile of a segment also holds the next
    segment's keys.  Here half of those keys share a large first coordinate with
    this segment's queries, so their scores (about 450) lie far above this segment's
    LSE and exp() of them overflows fp32; they must contribute nothing (the
    article's attention is per sequence: a key of another segment has P = 0)."""
    w = synthetic.Workload("segment_edge", (200, 150), hq=2, hkv=1, d=64, block=block, sigma=1.0,
                           delta=0.0, causal=False)
    inp = synthetic.make_inputs(w)
    q, k = inp["q"].clone(), inp["k"].clone()
    # segment 0's queries against segment 1's keys: +-60 * 60 / sqrt(64) = +-450 (the
    # sign alternates so that no coordinate of segment 1's keys is a common offset,
    # which would leave dQ's bf16 rounding noise on a sum that is exactly zero)
    q[:200, :, 0] = 60.0
    k[200:, :, 0] = torch.tensor([60.0, -60.0]).repeat(75)[:, None].to(k.dtype)
    k[:200, :, 0] = 0.0      # the scores within each segment stay ordinary
    q[200:, :, 0] = 0.0
    inp = dict(inp, q=q, k=k)
    desc, dev, bufs = run_step(w, inp)
    cu = w.cu_seqlens()
    o_ref, lse_ref = oracle.attn_fwd(cu, inp["q"], inp["k"], inp["v"], w.scale, w.causal)
    assert o_within(_cpu(bufs.o), o_ref, O_TOL)[0], o_within(_cpu(bufs.o), o_ref, O_TOL)
    dq_ref, dk_ref, dv_ref = oracle.attn_bwd(cu, inp["q"], inp["k"], inp["v"], inp["dout"],
                                             w.scale, w.block, None, w.causal)
    for got, ref in ((bufs.dq, dq_ref), (bufs.dk, dk_ref), (bufs.dv, dv_ref)):
        assert torch.isfinite(got).all()
        assert rel_fro(_cpu(got), ref) < GRAD_TOL


def test_same_seed_step_reproduces_and_steps_differ():
    w = synthetic.GQA_MID.with_(seqlens=(2048,))
    inp = synthetic.make_inputs(w)
    _, _, b1 = run_step(w, inp, seed=5, step=9)
    _, _, b2 = run_step(w, inp, seed=5, step=9)
    _, _, b3 = run_step(w, inp, seed=5, step=10)
    # masks, weights and the forward are bit-reproducible; dQ, dK and dV sum
    # per-tile / per-head partials with float reductions in arrival order, so
    # only their values are reproducible
    assert torch.equal(b1.keep, b2.keep) and torch.equal(b1.w, b2.w) and torch.equal(b1.o, b2.o)
    for a, b in ((b1.dq, b2.dq), (b1.dk, b2.dk), (b1.dv, b2.dv)):
        assert rel_fro(a.float().cpu(), b.float().cpu()) < 1e-5
    assert not torch.equal(b1.keep, b3.keep)


def test_empty_batch_is_a_noop():
    cu = torch.zeros(2, dtype=torch.int32, device="cuda")
    desc = lf.make_desc(cu, 0, 0, 2, 2, 64, 0.125, True, 64)
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    f = torch.zeros(16, dtype=torch.float32, device="cuda")
    lf.lf_attn_fwd(desc, x, x, x, x, f)
    lf.lf_check_device_error()


# ---------------------------------------------------------------------------
# Full-size workloads, in the launch configuration the bench times: outputs the
# oracle can compute one by one (sampled rows) plus properties at any size.
# ---------------------------------------------------------------------------
# one 256K-token segment with d = 64 and 64-row blocks: 4096 blocks per head in the
# selection and in the backward's kept lists
LONG_D64 = synthetic.Workload("long_d64", (262144,), hq=2, hkv=1, d=64, block=64, sigma=2.0,
                              delta=0.1)


def _kv_tile_rows(w, cu, kv_tile):
    """Sampled KV rows of one KV tile for the dK/dV check: "first" is KV tile 0 of
    the longest segment, whose walk is the longest of the launch (under the causal
    mask every kept query tile of the segment reaches it: many work-list ring and
    pipeline-phase wraps, and the longest accumulation in tensor memory); "last" is
    the segment-final tile of the last segment (the shortest walk).  Returns (rows,
    kv heads)."""
    lens = np.diff(cu)
    if kv_tile == "first":
        s = int(np.argmax(lens))
        u0, u1 = int(cu[s]), int(cu[s]) + 128
        rows = np.arange(u0, u1, 8, dtype=np.int32)
        heads = np.zeros(len(rows), dtype=np.int32)     # one KV head: one LSE pass
    else:
        s = w.nseq - 1
        u0 = max(int(cu[s + 1]) - 128, int(cu[s]))
        rows = np.arange(u0, int(cu[s + 1]), 8, dtype=np.int32)
        heads = (np.arange(len(rows)) % w.hkv).astype(np.int32)
    return rows, heads


@pytest.mark.parametrize("w,kv_tile", [
    (synthetic.HEADLINE, "first"), (synthetic.LONG, "first"), (synthetic.VARLEN, "first"),
    (LONG_D64, "last"),
], ids=["headline", "long", "varlen", "long_d64"])
def test_full_size_sampled_parity(w, kv_tile):
    inp = synthetic.make_inputs(w)
    desc, dev, bufs = run_step(w, inp)
    cu = w.cu_seqlens()
    nb = nb_per_seq(w)
    rng = np.random.default_rng(1)
    # selection: bit-exact against the oracle on the GPU's norms
    norms = _cpu(bufs.norm)
    sel = oracle.select(norms, nb, w.delta, 0, 0)
    np.testing.assert_array_equal(bufs.keep.cpu().numpy(), sel["keep"])
    np.testing.assert_array_equal(bufs.kept_idx.cpu().numpy(), sel["kept_idx"])
    np.testing.assert_array_equal(bufs.w.cpu().numpy().view(np.uint32), sel["w"].view(np.uint32))
    # norms of sampled blocks
    dout = inp["dout"]
    for _ in range(16):
        s = int(rng.integers(0, w.nseq))
        h = int(rng.integers(0, w.hq))
        b = int(rng.integers(0, nb[s]))
        r0, r1 = cu[s] + b * w.block, min(cu[s] + (b + 1) * w.block, cu[s + 1])
        ref = math.sqrt(float((dout[r0:r1, h].double() ** 2).sum()))
        assert abs(norms[s, h, b] - ref) <= NORM_TOL * ref
    # forward: sampled rows, including segment starts/ends and the last row
    rows = list(rng.integers(0, w.total_tokens, size=24)) + [0, w.total_tokens - 1]
    rows += [int(c) for c in cu[1:-1]] + [int(c) - 1 for c in cu[1:-1]]
    rows = np.array(rows[:40], dtype=np.int32)
    heads = rng.integers(0, w.hq, size=len(rows)).astype(np.int32)
    o_ref, lse_ref = oracle.attn_fwd_rows(cu, inp["q"], inp["k"], inp["v"], w.scale, rows, heads)
    o = _cpu(bufs.o)[rows, heads]
    lse = _cpu(bufs.lse)[heads, rows]
    assert o_within(o, o_ref, O_TOL)[0], o_within(o, o_ref, O_TOL)
    assert np.abs(lse - lse_ref).max() < LSE_TOL
    # backward: dQ at sampled rows of kept blocks, zero at dropped blocks; dK/dV at
    # sampled rows of one KV tile (see _kv_tile_rows)
    wb = sel["w"].astype(np.float64)
    kept_rows, kept_heads = [], []
    dq = bufs.dq.cpu()
    for _ in range(200):
        s = int(rng.integers(0, w.nseq))
        h = int(rng.integers(0, w.hq))
        b = int(rng.integers(0, nb[s]))
        t = int(cu[s] + b * w.block + rng.integers(0, min(w.block, cu[s + 1] - cu[s] - b * w.block)))
        if sel["keep"][s, h, b]:
            if len(kept_rows) < 24:
                kept_rows.append(t)
                kept_heads.append(h)
        else:
            assert torch.all(dq[t, h] == 0)
    kv_rows, kv_heads = _kv_tile_rows(w, cu, kv_tile)
    if kv_tile == "first":
        # the walk checked is long: count the kept (head, query tile) pairs it visits
        s0 = int(np.searchsorted(cu, kv_rows[0], side="right") - 1)
        G = w.hq // w.hkv
        per = 128 // w.block
        kept_tiles = sel["keep"][s0, :G, : nb[s0]]
        ntile = (nb[s0] + per - 1) // per
        walked = sum(int(kept_tiles[h, i * per:(i + 1) * per].any()) for h in range(G)
                     for i in range(ntile))
        assert walked >= 40, walked
    dq_ref, dk_ref, dv_ref = oracle.attn_bwd_rows(cu, inp["q"], inp["k"], inp["v"], dout, w.scale,
                                                  w.block, wb, kept_rows, kept_heads, kv_rows,
                                                  kv_heads)
    assert rel_fro(_cpu(bufs.dq)[kept_rows, kept_heads], dq_ref) < GRAD_TOL
    dk = _cpu(bufs.dk)[kv_rows, kv_heads]
    dv = _cpu(bufs.dv)[kv_rows, kv_heads]
    if np.linalg.norm(dk_ref) > 0:
        assert rel_fro(dk, dk_ref) < GRAD_TOL
        assert rel_fro(dv, dv_ref) < GRAD_TOL
    else:
        assert np.all(dk == 0) and np.all(dv == 0)


def test_gqa_mid_full_oracle():
    """The GQA-mid workload (4096 tokens, 32 query heads over 8 KV heads, d = 128,
    delta = 0.05) against the full oracle: every output element."""
    w = synthetic.GQA_MID
    inp = synthetic.make_inputs(w)
    desc, dev, bufs = run_step(w, inp, seed=4, step=7)
    cu = w.cu_seqlens()
    nb = nb_per_seq(w)
    o_ref, lse_ref = oracle.attn_fwd(cu, inp["q"], inp["k"], inp["v"], w.scale, w.causal)
    assert o_within(_cpu(bufs.o), o_ref, O_TOL)[0], o_within(_cpu(bufs.o), o_ref, O_TOL)
    assert np.abs(_cpu(bufs.lse) - lse_ref).max() < LSE_TOL
    m_ref = oracle.block_norms(cu, inp["dout"], w.block, w.nbmax)
    m = _cpu(bufs.norm)
    assert np.all(np.abs(m - m_ref) <= NORM_TOL * np.maximum(m_ref, 1e-30))
    D_ref = oracle.rowdot(inp["dout"], bufs.o.cpu())
    scale = np.sqrt(oracle.rowdot(inp["dout"], inp["dout"]) * oracle.rowdot(bufs.o.cpu(), bufs.o.cpu()))
    assert np.all(np.abs(_cpu(bufs.D) - D_ref) <= 1e-5 * scale + 1e-30)
    sel = oracle.select(m, nb, w.delta, 4, 7)
    np.testing.assert_array_equal(bufs.tau.cpu().numpy().view(np.uint64), sel["tau"].view(np.uint64))
    np.testing.assert_array_equal(bufs.keep.cpu().numpy(), sel["keep"])
    np.testing.assert_array_equal(bufs.w.cpu().numpy().view(np.uint32), sel["w"].view(np.uint32))
    np.testing.assert_array_equal(bufs.kept_idx.cpu().numpy(), sel["kept_idx"])
    np.testing.assert_array_equal(bufs.kept_cnt.cpu().numpy(), sel["kept_cnt"])
    assert 0 < sel["keep"].mean() < 1
    dq_ref, dk_ref, dv_ref = oracle.attn_bwd(cu, inp["q"], inp["k"], inp["v"], inp["dout"], w.scale,
                                             w.block, sel["w"].astype(np.float64), w.causal)
    assert rel_fro(_cpu(bufs.dq), dq_ref) < GRAD_TOL
    assert rel_fro(_cpu(bufs.dk), dk_ref) < GRAD_TOL
    assert rel_fro(_cpu(bufs.dv), dv_ref) < GRAD_TOL


@pytest.mark.parametrize("w", [SMALL[1], SMALL[4]], ids=lambda w: w.name)
def test_backward_computes_D_itself(w):
    """lf_attn_bwd with D = NULL computes D = rowsum(dO * O) from o and dout in its
    workspace; the gradients match those computed with the selection's D."""
    inp = synthetic.make_inputs(w)
    desc, dev, bufs = run_step(w, inp, seed=3, step=1)
    ref = {k: getattr(bufs, k).float().cpu() for k in ("dq", "dk", "dv")}
    out = {k: torch.full_like(getattr(bufs, k), float("nan")) for k in ("dq", "dk", "dv")}
    lf.lf_attn_bwd(desc, dev["q"], dev["k"], dev["v"], bufs.o, bufs.lse, dev["dout"], None, bufs.w,
                   bufs.kept_idx, bufs.kept_cnt, out["dq"], out["dk"], out["dv"], bufs.ws)
    lf.lf_check_device_error()
    sel = oracle.select(_cpu(bufs.norm), nb_per_seq(w), w.delta, 3, 1)
    dq_ref, dk_ref, dv_ref = oracle.attn_bwd(w.cu_seqlens(), inp["q"], inp["k"], inp["v"],
                                             inp["dout"], w.scale, w.block,
                                             sel["w"].astype(np.float64), w.causal)
    for k, oref in (("dq", dq_ref), ("dk", dk_ref), ("dv", dv_ref)):
        got = out[k].float().cpu()
        assert torch.isfinite(got).all(), k
        assert rel_fro(got, oref) < GRAD_TOL, k
        # the same gradients as with the selection's D, up to the rounding of the sums
        assert rel_fro(got, ref[k]) < 1e-3, k


@pytest.mark.parametrize("case", [
    ((512,), 2, 64, 1.5),
    ((32768,), 32, 128, 2.0),
    ((1, 100, 0, 5000), 8, 128, 0.5),
    ((65536,), 4, 64, 2.0),
], ids=["tiny", "headline", "odd", "blk64_1024"])
@pytest.mark.parametrize("rule,param", [
    (lf.LF_RULE_FIXED_FRACTION, 0.1), (lf.LF_RULE_FIXED_FRACTION, 0.5),
    (lf.LF_RULE_FIXED_FRACTION, 1.0), (lf.LF_RULE_TOPK, 0.1), (lf.LF_RULE_TOPK, 0.37),
    (lf.LF_RULE_TOPK, 1.0), (lf.LF_RULE_BUDGET, 0.2),
])
def test_selection_rules_bit_exact_given_norms(case, rule, param):
    """The fixed-fraction and top-k rules (article section "Le choix des blocs
    pèse plus que la quantité sautée") in the same selection kernel."""
    lens, hq, block, sigma = case
    w, nb, m = _select_case(lens, hq, block, sigma, seed=7 * hq + len(lens))
    m[0, 0, : min(3, nb[0])] = 0.0
    m[0, 1 % hq, 5:9] = m[0, 1 % hq, 4]               # ties for top-k
    desc = desc_for(w, torch.as_tensor(w.cu_seqlens()).cuda())
    nbmax = w.nbmax
    dummy = torch.zeros(w.total_tokens, hq, 64, dtype=torch.bfloat16, device="cuda")
    norm = torch.as_tensor(m, device="cuda")
    D = torch.empty(hq, w.total_tokens, device="cuda")
    tau = torch.empty(w.nseq, hq, dtype=torch.float64, device="cuda")
    wt = torch.empty(w.nseq, hq, nbmax, device="cuda")
    keep = torch.empty(w.nseq, hq, nbmax, dtype=torch.uint8, device="cuda")
    kidx = torch.empty(w.nseq, hq, nbmax, dtype=torch.int32, device="cuda")
    kcnt = torch.empty(w.nseq, hq, dtype=torch.int32, device="cuda")
    for seed, step in [(0, 0), (123, 2**33 + 5)]:
        lf.lf_block_select_rule(desc, dummy, dummy, rule, param, seed, step, lf.LF_SELECT_NORMS_GIVEN,
                                norm, D, tau, wt, keep, kidx, kcnt)
        lf.lf_check_device_error()
        ref = oracle.select_rule(rule, m, nb, param, seed, step)
        np.testing.assert_array_equal(tau.cpu().numpy().view(np.uint64), ref["tau"].view(np.uint64))
        np.testing.assert_array_equal(keep.cpu().numpy(), ref["keep"])
        np.testing.assert_array_equal(wt.cpu().numpy().view(np.uint32), ref["w"].view(np.uint32))
        np.testing.assert_array_equal(kcnt.cpu().numpy(), ref["kept_cnt"])
        np.testing.assert_array_equal(kidx.cpu().numpy(), ref["kept_idx"])


def test_backward_with_topk_and_fixed_fraction_weights():
    w = synthetic.Workload("rules_bwd", (700,), hq=4, hkv=2, d=128, block=128, sigma=1.5, delta=0.1)
    inp = synthetic.make_inputs(w)
    dev = to_dev(inp)
    desc = desc_for(w, dev["cu_seqlens"])
    cu = w.cu_seqlens()
    nb = nb_per_seq(w)
    for rule, param in ((lf.LF_RULE_TOPK, 0.3), (lf.LF_RULE_FIXED_FRACTION, 0.4)):
        bufs = lf.Buffers(desc)
        lf.lf_attn_fwd(desc, dev["q"], dev["k"], dev["v"], bufs.o, bufs.lse)
        lf.lf_block_select_rule(desc, dev["dout"], bufs.o, rule, param, 3, 1, 0, bufs.norm, bufs.D,
                                bufs.tau, bufs.w, bufs.keep, bufs.kept_idx, bufs.kept_cnt)
        lf.lf_attn_bwd(desc, dev["q"], dev["k"], dev["v"], bufs.o, bufs.lse, dev["dout"], bufs.D,
                       bufs.w, bufs.kept_idx, bufs.kept_cnt, bufs.dq, bufs.dk, bufs.dv, bufs.ws)
        lf.lf_check_device_error()
        sel = oracle.select_rule(rule, _cpu(bufs.norm), nb, param, 3, 1)
        np.testing.assert_array_equal(bufs.keep.cpu().numpy(), sel["keep"])
        dq_ref, dk_ref, dv_ref = oracle.attn_bwd(cu, inp["q"], inp["k"], inp["v"], inp["dout"], w.scale,
                                                 w.block, sel["w"].astype(np.float64), True)
        assert rel_fro(_cpu(bufs.dq), dq_ref) < GRAD_TOL
        assert rel_fro(_cpu(bufs.dk), dk_ref) < GRAD_TOL
        assert rel_fro(_cpu(bufs.dv), dv_ref) < GRAD_TOL


@pytest.mark.parametrize("w", [SMALL[0], SMALL[4], SMALL[1]], ids=lambda w: w.name)
def test_dropped_blocks_are_never_read(w):
    """Dropped tiles are never loaded or computed (article section "Un budget sur la
    masse de gradient ..."): after the selection, the Q and dO rows of every dropped
    block are overwritten with NaN; a backward that loaded or multiplied any of them
    (even by a zero weight) would return NaN.  With 64-row blocks this covers the
    dropped half of a 128-row tile whose other half is kept."""
    inp = synthetic.make_inputs(w)
    desc, dev, bufs = run_step(w, inp, seed=3, step=1)
    cu = w.cu_seqlens()
    nb = nb_per_seq(w)
    keep = bufs.keep.cpu().numpy()
    q_bad, do_bad = dev["q"].clone(), dev["dout"].clone()
    dropped = 0
    for s in range(w.nseq):
        for h in range(w.hq):
            for b in range(int(nb[s])):
                if keep[s, h, b] == 0:
                    r0 = int(cu[s]) + b * w.block
                    r1 = min(r0 + w.block, int(cu[s + 1]))
                    q_bad[r0:r1, h] = float("nan")
                    do_bad[r0:r1, h] = float("nan")
                    dropped += 1
    assert dropped > 0
    out = {k: torch.empty_like(getattr(bufs, k)) for k in ("dq", "dk", "dv")}
    lf.lf_attn_bwd(desc, q_bad, dev["k"], dev["v"], bufs.o, bufs.lse, do_bad, bufs.D, bufs.w,
                   bufs.kept_idx, bufs.kept_cnt, out["dq"], out["dk"], out["dv"], bufs.ws)
    lf.lf_sync_status()
    for k in ("dq", "dk", "dv"):
        got = out[k].float().cpu()
        assert torch.isfinite(got).all(), k
        assert rel_fro(got, getattr(bufs, k).float().cpu()) < 1e-5, k
