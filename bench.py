"""LazyFlash attention step benchmark (forward + selection + sparse backward).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lazyflash|reference]
                    [--workload headline|varlen|long|gqa_mid|tiny] [--delta D]

One step = the whole hot path over one batch: lf_attn_fwd, lf_block_select and
lf_attn_bwd on the workload's synthetic bf16 inputs (a Qwen3-8B-shaped layer:
Hq=32, Hkv=8, d=128; N=32768 tokens, delta=0.1 by default).  Inputs stay
resident in HBM for `value`; `e2e` repeats the step through the same API with
host (pinned) inputs copied in and the results (O, LSE, dQ, dK, dV) copied out
inside the timed region; the copies run on two side streams into and out of
double-buffered device tensors, overlapping the kernels of neighbouring steps
as a data-fed training loop would.  One headline step touches ~2.4 GB, far more than
the 126 MB L2, so no explicit flush is needed between its steps; the smaller workloads
reported beside it are timed with a 256 MB write before every step.

Under torchrun each rank runs an independent replica (the path has no data
exchange): `value` = all ranks' FLOPs / the slowest rank's time.

`--impl reference` times the CPU oracle (fp64 C, OpenMP) on a bounded sample of
the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

TILE = 128


def _load_json(path):
    try:
        with open(path) as f:
            return json.load(f)
    except Exception:
        return None


def tile_flops(w: synthetic.Workload, keep=None):
    """Tile-level FLOPs: forward (all tiles), backward dense-equivalent and
    backward executed (query tiles holding a kept block).  ntile(i) = KV tiles
    a 128-row query tile i meets: i + 1 causal, all tiles of the segment
    otherwise.  Forward: 4*128*128*d per (query tile, KV tile); backward: 10*."""
    unit = TILE * TILE * w.d
    fwd = bwd_dense = bwd_exec = 0
    per = TILE // w.block
    for s, L in enumerate(w.seqlens):
        nt = (L + TILE - 1) // TILE
        for i in range(nt):
            n_kv = (i + 1) if w.causal else nt
            fwd += w.hq * n_kv * 4 * unit
            bwd_dense += w.hq * n_kv * 10 * unit
            if keep is not None:
                b0 = i * per
                kept_heads = keep[s, :, b0:b0 + per].any(axis=1).sum()
                bwd_exec += int(kept_heads) * n_kv * 10 * unit
    return fwd, bwd_dense, bwd_exec


def selection_telemetry(w: synthetic.Workload, norm, tau, keep, bwd_exec_fl, bwd_dense_fl):
    """What the selection did, per (segment, head), from the GPU's outputs: the
    kept fraction of blocks, tau, and the expected discarded share
    sum_b (1 - p_b) m_b / sum_b m_b with p_b = min(1, m_b / tau), which the budget
    bounds by delta (article sections "Un budget sur la masse de gradient ..." and
    "Le choix des blocs pèse plus que la quantité sautée")."""
    kept_frac, taus, shares = [], [], []
    n_kept = n_all = 0
    for s, L in enumerate(w.seqlens):
        nb = (L + w.block - 1) // w.block
        if nb == 0:
            continue
        for h in range(w.hq):
            m = norm[s, h, :nb].astype(np.float64)
            k = keep[s, h, :nb]
            n_kept += int(k.sum())
            n_all += nb
            kept_frac.append(float(k.mean()))
            t = float(tau[s, h])
            taus.append(t)
            tot = m.sum()
            if t > 0 and tot > 0:
                p = np.minimum(1.0, m / t)
                shares.append(float(((1.0 - p) * m).sum() / tot))
            else:
                shares.append(0.0)

    def mmm(x):
        return {"min": float(np.min(x)), "median": float(np.median(x)), "max": float(np.max(x))}

    return {"kept_fraction": n_kept / max(1, n_all),
            "kept_fraction_per_head": mmm(kept_frac),
            "tau": mmm(taus),
            "expected_discarded_share": {"max": float(np.max(shares)),
                                         "median": float(np.median(shares)),
                                         "bound_delta": w.delta,
                                         "within_bound": bool(np.max(shares) <= w.delta + 1e-12)},
            "executed_vs_dense_flops": bwd_exec_fl / bwd_dense_fl,
            "heads": len(kept_frac)}


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
_CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


_REASON_NAMES = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
                 ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
                 ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
                 ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))


def _summarise(sm, mx, reasons, source):
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
            "reasons": sorted(reasons), "samples": len(sm), "source": source}


class _NvmlSampler:
    """SM clock and clock-event reasons every 5 ms from a thread of this process
    (read-only NVML queries), so that even a short timed region is covered."""

    def __init__(self, device_index: int):
        import threading
        import pynvml
        self.nv = pynvml
        pynvml.nvmlInit()
        uuid = str(torch.cuda.get_device_properties(device_index).uuid)
        if not uuid.startswith("GPU-"):
            uuid = "GPU-" + uuid
        self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode() if isinstance(uuid, str) else uuid)
        self.mx = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        self.bits = [(name, getattr(pynvml, attr)) for name, attr in _REASON_NAMES]
        self.sm, self.reasons = [], set()
        self.stop_ev = threading.Event()
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()
        t0 = time.time()
        while not self.sm and time.time() - t0 < 2.0:   # first sample before timing starts
            time.sleep(0.001)

    def _run(self):
        nv = self.nv
        while not self.stop_ev.is_set():
            try:
                self.sm.append(float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.bits:
                    if bits & bit:
                        self.reasons.add(name)
            except Exception:
                return
            self.stop_ev.wait(0.005)

    def stop(self):
        self.stop_ev.set()
        self.t.join(timeout=5)
        try:
            self.nv.nvmlShutdown()
        except Exception:
            pass
        return _summarise(self.sm, self.mx, self.reasons, "nvml, 5 ms")


class _SmiSampler:
    """Fallback: nvidia-smi in a subprocess (first sample after ~0.1-0.5 s)."""

    def __init__(self, device_index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        uuid = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
        except Exception:
            pass
        sel = ["-i", uuid] if uuid else []
        try:
            self.p = subprocess.Popen(["nvidia-smi", "--query-gpu=" + _CLOCK_FIELDS,
                                       "--format=csv,noheader,nounits", "-lms", "100", *sel],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return _summarise(sm, mx, reasons, "nvidia-smi, 100 ms")


def ClockSampler(device_index: int):
    """Starts sampling now; .stop() returns the summary for the JSON line."""
    try:
        return _NvmlSampler(device_index)
    except Exception:
        return _SmiSampler(device_index)


# ---------------------------------------------------------------------------
# CPU oracle sample (the cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------
def kernels_per_step(w: synthetic.Workload) -> int:
    """This library's kernels in one step: forward; norms and selection; the
    backward's prologue (dQ accumulator rows, D), the backward and the dQ
    conversion; the one-thread kernel that ends each of the three calls (it copies
    the device failure flag to the host-mapped page); plus the dK/dV conversions
    when one backward CTA cannot hold the whole query group (more than 32 query
    heads per KV head)."""
    group = w.hq // w.hkv
    return 9 + (0 if group <= 32 else 2)


def oracle_sample(w: synthetic.Workload, inp, prefix: int, seed=0, step=0):
    """The oracle's forward, selection and weighted backward on the first
    `prefix` tokens of segment 0 (a causal prefix is itself a complete problem),
    all heads.  Returns a dict: seconds of the backward and of the whole step,
    the sample's executed backward tile FLOPs and step FLOPs, and the threads."""
    import oracle
    ws = w.with_(seqlens=(prefix,))
    sl = slice(0, prefix)
    q, k, v, do = inp["q"][sl], inp["k"][sl], inp["v"][sl], inp["dout"][sl]
    cu = ws.cu_seqlens()
    oracle.lib()
    t0 = time.perf_counter()
    o, lse = oracle.attn_fwd(cu, q, k, v, ws.scale, ws.causal)
    m = oracle.block_norms(cu, do, ws.block)
    sel = oracle.select(m, oracle.nblocks(cu, ws.block), ws.delta, seed, step)
    t1 = time.perf_counter()
    oracle.attn_bwd(cu, q, k, v, do, ws.scale, ws.block, sel["w"].astype(np.float64), ws.causal)
    t2 = time.perf_counter()
    f, _, b = tile_flops(ws, sel["keep"])
    threads = int(os.environ.get("OMP_NUM_THREADS", len(os.sched_getaffinity(0))))
    return {"bwd_s": t2 - t1, "step_s": t2 - t0, "bwd_flops": b, "step_flops": f + b,
            "threads": threads}


def max_over_ranks(values, dist=None, device=None):
    """Element-wise maximum of every rank's `values` (the job is as slow as its slowest
    rank); a single process returns them unchanged."""
    if dist is None:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def whole_job_tflops(n_ranks, steps, flops_per_step, ms):
    """Throughput of the whole job: each of `n_ranks` ranks ran `steps` steps of
    `flops_per_step` (weak scaling) within `ms`, the maximum over ranks."""
    return n_ranks * steps * flops_per_step / (ms * 1e-3) / 1e12


def run_reference(args, w, rank):
    if rank != 0:
        return
    prefix = min(args.ref_prefix, w.seqlens[0])
    inp = synthetic.make_inputs(w, rows=prefix) if w.nseq == 1 else synthetic.make_inputs(w)
    for _ in range(args.warmup):
        oracle_sample(w, inp, prefix)
    tot_b = tot_s = tot_f = 0.0
    threads = 1
    for _ in range(args.steps):
        r = oracle_sample(w, inp, prefix)
        tot_b += r["bwd_s"]
        tot_s += r["step_s"]
        tot_f += r["bwd_flops"]
        threads = r["threads"]
    val = tot_f / tot_b / 1e12
    sample = ("oracle backward (its executed tile FLOPs over its own time; the forward and "
              "selection that feed it run untimed) on the first %d tokens of the %s workload, "
              "all %d heads (a causal prefix is a complete sub-problem)" % (prefix, w.name, w.hq))
    line = {
        "impl": "reference", "metric": args.metric, "value": val, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot_s / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, args),
        "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(w, args):
    return {"workload": w.name, "seqlens": list(w.seqlens) if w.nseq <= 16 else "%d segments" % w.nseq,
            "total_tokens": w.total_tokens, "hq": w.hq, "hkv": w.hkv, "d": w.d, "block": w.block,
            "causal": w.causal, "delta": w.delta, "dO_block_scale": "LogNormal(0,%g)" % w.sigma,
            "seed": 0, "step": 0, "rule": args.rule if hasattr(args, "rule") else "budget",
            "rule_param": getattr(args, "rule_param", None),
            "l2": "no flush: one step touches ~2.4 GB (Q, dO, O, dQ 256 MiB each, K, V, dK, dV "
                  "64 MiB each, the 512 MiB dQ accumulator), far more than the 126 MB L2, so "
                  "each step reads its inputs from HBM",
            "parallelism": "replicas" if args.gpus > 1 else "single"}


# ---------------------------------------------------------------------------
# LazyFlash arm
# ---------------------------------------------------------------------------
def run_layers(args, w):
    """Synthetic layer-stack step: per layer a QKV projection, LazyFlash attention
    (the autograd wrapper: exact forward, block-sparse backward), an output projection
    and a residual add; loss <x_L, g> with a block-skewed g; backward and a plain SGD
    update (lr 1e-9) of the random weights; every step's loss must be finite.  Timed at
    the workload's delta against delta = 0 (the dense backward through the same
    kernels), plus the attention's own fwd+bwd."""
    from block_sparse_attention_dense_b200.autograd import lazyflash_attention
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    L, T, hq, hkv, d = args.layers, w.total_tokens, w.hq, w.hkv, w.d
    inp = synthetic.make_layer_step_inputs(w, L, dev)
    params = [p.clone().requires_grad_(True) for p in inp["wqkv"] + inp["wo"]]
    wqkv, wo = params[:L], params[L:]
    x0, g, cu = inp["x"], inp["g"], inp["cu_seqlens"]

    def layer_step(delta):
        x = x0
        for l in range(L):
            qkv = x @ wqkv[l]
            q = qkv[:, :hq * d].reshape(T, hq, d).contiguous()
            k = qkv[:, hq * d:(hq + hkv) * d].reshape(T, hkv, d).contiguous()
            v = qkv[:, (hq + hkv) * d:].reshape(T, hkv, d).contiguous()
            o = lazyflash_attention(q, k, v, cu, T, delta=delta, causal=w.causal, block_q=w.block)
            x = x + o.reshape(T, hq * d) @ wo[l]
        loss = (x.float() * g.float()).sum()
        grads = torch.autograd.grad(loss, params)
        finite.append(torch.isfinite(loss))
        with torch.no_grad():
            # the update runs every step; lr 1e-9 keeps the random weights (and so every
            # later step's inputs) in range: the skewed loss gradient summed over T rows
            # is large, and a diverging stack would time non-finite data
            for p, gr in zip(params, grads):
                p.sub_(gr, alpha=1e-9)

    att = synthetic.make_inputs(w)
    aq, ak, av, adout = (att[n].to(dev) for n in ("q", "k", "v", "dout"))
    aq.requires_grad_(True)
    ak.requires_grad_(True)
    av.requires_grad_(True)

    def attn_step(delta):
        o = lazyflash_attention(aq, ak, av, cu, T, delta=delta, causal=w.causal, block_q=w.block)
        torch.autograd.grad(o, (aq, ak, av), adout)

    finite = []

    def timed(fn, delta):
        for _ in range(args.warmup):
            fn(delta)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            fn(delta)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / args.steps

    ms = {"step": {}, "attention": {}}
    for name, delta in (("lazyflash", w.delta), ("dense", 0.0)):
        ms["step"][name] = timed(layer_step, delta)
        ms["attention"][name] = timed(attn_step, delta)
    if not bool(torch.stack(finite).all()):
        raise SystemExit("the synthetic layer stack produced a non-finite loss")
    line = {
        "metric": "synthetic %d-layer step (QKV proj, LazyFlash attention, out proj, residual; "
                  "fwd + bwd + SGD) speed-up over the dense backward (delta = 0)" % L,
        "value": ms["step"]["dense"] / ms["step"]["lazyflash"],
        "unit": "x",
        "higher_is_better": True,
        "ms_per_step": ms["step"],
        "attention_fwd_bwd": {"ms": ms["attention"],
                              "speedup": ms["attention"]["dense"] / ms["attention"]["lazyflash"]},
        "steps": args.steps, "warmup": args.warmup, "n_gpus": 1,
        "dtype": "bf16", "data": "synthetic (random weights, no data set)",
        "config": {"workload": w.name, "layers": L, "total_tokens": T, "hq": hq, "hkv": hkv, "d": d,
                   "hidden": hq * d, "delta": w.delta, "dO_block_scale": "LogNormal(0,%g)" % w.sigma},
    }
    print(json.dumps(line), flush=True)


def measure_workload(lf, w, dev, steps=5, warmup=2):
    """fwd / select / bwd ms (CUDA events on the launching stream, inputs resident) of
    one synthetic workload at its own delta, with its executed and dense-equivalent
    backward FLOPs: the other configurations of the measurement plan, reported beside
    the headline line."""
    stream = torch.cuda.current_stream()
    inp = synthetic.make_inputs(w)
    d_in = {k: v.to(dev) for k, v in inp.items() if k != "cu_seqlens"}
    cu = inp["cu_seqlens"].to(dev)
    desc = lf.make_desc(cu, w.max_seqlen, w.total_tokens, w.hq, w.hkv, w.d, w.scale, w.causal,
                        w.block)
    b = lf.Buffers(desc, device=dev)

    def run(record=None):
        ev = record or [None] * 4
        if ev[0]: ev[0].record(stream)
        lf.lf_attn_fwd(desc, d_in["q"], d_in["k"], d_in["v"], b.o, b.lse)
        if ev[1]: ev[1].record(stream)
        lf.lf_block_select(desc, d_in["dout"], b.o, w.delta, 0, 0, 0, b.norm, b.D, b.tau, b.w,
                           b.keep, b.kept_idx, b.kept_cnt)
        if ev[2]: ev[2].record(stream)
        lf.lf_attn_bwd(desc, d_in["q"], d_in["k"], d_in["v"], b.o, b.lse, d_in["dout"], b.D, b.w,
                       b.kept_idx, b.kept_cnt, b.dq, b.dk, b.dv, b.ws)
        if ev[3]: ev[3].record(stream)

    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    # smaller workloads fit in L2: a 256 MB write before every timed step (outside the
    # phase events) leaves each step to start from HBM
    flush = torch.empty(64 << 20, dtype=torch.float32, device=dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for e in evs:
        flush.zero_()
        run(e)
    torch.cuda.synchronize()
    del flush
    lf.lf_sync_status()
    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / steps
    sel_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / steps
    bwd_ms = sum(e[2].elapsed_time(e[3]) for e in evs) / steps
    keep = b.keep.cpu().numpy()
    fwd_fl, bwd_dense_fl, bwd_exec_fl = tile_flops(w, keep)
    out = {"tokens": w.total_tokens, "segments": w.nseq, "delta": w.delta,
           "fwd_ms": fwd_ms, "select_ms": sel_ms, "bwd_ms": bwd_ms,
           "fwd_tflops": fwd_fl / (fwd_ms * 1e-3) / 1e12,
           "bwd_tflops_executed": bwd_exec_fl / (bwd_ms * 1e-3) / 1e12,
           "bwd_executed_fraction": bwd_exec_fl / bwd_dense_fl, "steps": steps,
           "l2": "256 MB written before every timed step"}
    del b, d_in
    torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="lazyflash", choices=["lazyflash", "reference"])
    ap.add_argument("--workload", default="headline", choices=sorted(synthetic.WORKLOADS))
    ap.add_argument("--delta", type=float, default=None)
    ap.add_argument("--rule", default="budget", choices=["budget", "fixed", "topk"],
                    help="selection rule (budget = LazyFlash; fixed fraction and top-k are the "
                         "article's comparison rules); --rule-param is f for the latter two")
    ap.add_argument("--rule-param", type=float, default=None)
    ap.add_argument("--seqlen", type=int, default=None, help="override the workload's length "
                    "(single-segment workloads)")
    ap.add_argument("--cpu-prefix", type=int, default=3072,
                    help="tokens of the oracle sample timed for cpu_baseline")
    ap.add_argument("--ref-prefix", type=int, default=1024,
                    help="tokens of the oracle sample timed per step by --impl reference")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense-arm", action="store_true",
                    help="skip the delta = 0 comparison run after the timed region")
    ap.add_argument("--layers", type=int, default=0,
                    help="time the synthetic layer-stack step instead (its own JSON line)")
    args = ap.parse_args()
    args.metric = "LazyFlash attn bwd ms & executed TFLOP/s at N=32K, Hq32/Hkv8 d128, delta=0.1"
    w = synthetic.WORKLOADS[args.workload]
    if args.delta is not None:
        w = w.with_(delta=args.delta)
    if args.seqlen is not None:
        if w.nseq != 1:
            raise SystemExit("--seqlen applies to single-segment workloads")
        w = w.with_(seqlens=(args.seqlen,))
    if args.layers > 0:
        run_layers(args, w)
        return
    rule_id = {"budget": 0, "fixed": 1, "topk": 2}[args.rule]
    rule_param = w.delta if rule_id == 0 else args.rule_param
    if rule_id != 0 and rule_param is None:
        raise SystemExit("--rule fixed/topk needs --rule-param f")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    if args.impl == "reference":
        run_reference(args, w, rank)
        if dist is not None:
            dist.destroy_process_group()
        return

    import block_sparse_attention_dense_b200 as lf
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()

    inp = synthetic.make_inputs(w)
    host = {k: v.pin_memory() for k, v in inp.items() if k != "cu_seqlens"}
    d_in = {k: v.to(dev) for k, v in host.items()}
    cu = inp["cu_seqlens"].to(dev)
    desc = lf.make_desc(cu, w.max_seqlen, w.total_tokens, w.hq, w.hkv, w.d, w.scale, w.causal,
                        w.block)
    bufs = lf.Buffers(desc, device=dev)

    def select(param):
        lf.lf_block_select_rule(desc, d_in["dout"], bufs.o, rule_id, param, 0, 0, 0, bufs.norm,
                                bufs.D, bufs.tau, bufs.w, bufs.keep, bufs.kept_idx, bufs.kept_cnt)

    def step(param):
        lf.lf_attn_fwd(desc, d_in["q"], d_in["k"], d_in["v"], bufs.o, bufs.lse)
        select(param)
        lf.lf_attn_bwd(desc, d_in["q"], d_in["k"], d_in["v"], bufs.o, bufs.lse, d_in["dout"],
                       bufs.D, bufs.w, bufs.kept_idx, bufs.kept_cnt, bufs.dq, bufs.dk, bufs.dv,
                       bufs.ws)

    def timed_region(K, param):
        """K steps back to back on `stream`, CUDA events around the region and around
        each phase; returns (region ms, summed fwd, select and bwd ms)."""
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for i in range(K):
            e = ev[i]
            e[0].record(stream)
            lf.lf_attn_fwd(desc, d_in["q"], d_in["k"], d_in["v"], bufs.o, bufs.lse)
            e[1].record(stream)
            select(param)
            e[2].record(stream)
            lf.lf_attn_bwd(desc, d_in["q"], d_in["k"], d_in["v"], bufs.o, bufs.lse, d_in["dout"],
                           bufs.D, bufs.w, bufs.kept_idx, bufs.kept_cnt, bufs.dq, bufs.dk, bufs.dv,
                           bufs.ws)
            e[3].record(stream)
        end.record(stream)
        torch.cuda.synchronize()
        return (start.elapsed_time(end), sum(e[0].elapsed_time(e[1]) for e in ev),
                sum(e[1].elapsed_time(e[2]) for e in ev), sum(e[2].elapsed_time(e[3]) for e in ev))

    for _ in range(max(3, args.warmup)):
        step(rule_param)
    lf.lf_sync_status()
    torch.cuda.synchronize()
    keep = bufs.keep.cpu().numpy()
    fwd_fl, bwd_dense_fl, bwd_exec_fl = tile_flops(w, keep)
    telemetry = selection_telemetry(w, bufs.norm.cpu().numpy(), bufs.tau.cpu().numpy(), keep,
                                    bwd_exec_fl, bwd_dense_fl)

    # ---- device-timed steps, inputs resident; per-phase events on the launching stream
    K = args.steps
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    total_ms, fwd_sum, sel_sum, bwd_sum = timed_region(K, rule_param)
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    fwd_ms, sel_ms, bwd_ms = fwd_sum / K, sel_sum / K, bwd_sum / K
    lf.lf_sync_status()

    # ---- the dense backward (delta = 0) through the same kernels: does the backward's
    # time follow the executed fraction?  (article section "A 32 000 tokens, 5,72 fois")
    # ---- selection telemetry beyond the workload's own delta (outside the timed regions):
    # the speech setting's delta = 0.4 on the same gradients, and the kept fraction at
    # causal prefixes of the sequence (a prefix is itself a complete problem, with the
    # same per-block gradient scales), article sections "Un budget qui ne se transpose
    # pas du texte à la parole" and "Le choix des blocs pèse plus que la quantité sautée"
    if rule_id == 0 and w.nseq == 1 and not args.no_dense_arm:
        extra = {}

        def sel_bufs(dsc):
            nbm = (dsc.max_seqlen + dsc.block_q - 1) // dsc.block_q
            f32 = dict(dtype=torch.float32, device=dev)
            return dict(norm=torch.empty(dsc.nseq, w.hq, nbm, **f32),
                        D=torch.empty(w.hq, dsc.total_tokens, **f32),
                        tau=torch.empty(dsc.nseq, w.hq, dtype=torch.float64, device=dev),
                        w=torch.empty(dsc.nseq, w.hq, nbm, **f32),
                        keep=torch.empty(dsc.nseq, w.hq, nbm, dtype=torch.uint8, device=dev),
                        kept_idx=torch.empty(dsc.nseq, w.hq, nbm, dtype=torch.int32, device=dev),
                        kept_cnt=torch.empty(dsc.nseq, w.hq, dtype=torch.int32, device=dev))

        def run_select(dsc, dout, o, delta):
            b = sel_bufs(dsc)
            lf.lf_block_select(dsc, dout, o, delta, 0, 0, 0, b["norm"], b["D"], b["tau"], b["w"],
                               b["keep"], b["kept_idx"], b["kept_cnt"])
            nb = (dsc.total_tokens + w.block - 1) // w.block
            return float(b["keep"][:, :, :nb].float().mean())

        extra["delta_0.4_kept_fraction"] = run_select(desc, d_in["dout"], bufs.o, 0.4)
        by_len = {}
        for n_tok in (8192, 16384, 32768, 65536):
            if n_tok > w.total_tokens:
                continue
            cu_p = torch.tensor([0, n_tok], dtype=torch.int32, device=dev)
            dp = lf.make_desc(cu_p, n_tok, n_tok, w.hq, w.hkv, w.d, w.scale, w.causal, w.block)
            by_len[str(n_tok)] = run_select(dp, d_in["dout"][:n_tok], bufs.o[:n_tok], w.delta)
        extra["kept_fraction_by_length_at_delta"] = by_len
        lf.lf_sync_status()
        telemetry.update(extra)

    dense_arm = None
    if rule_id == 0 and w.delta > 0 and not args.no_dense_arm:
        K0 = max(3, K // 2)
        for _ in range(2):
            step(0.0)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        _, _, _, bwd0_sum = timed_region(K0, 0.0)
        lf.lf_sync_status()
        bwd0_ms = max_over_ranks([bwd0_sum / K0], dist, dev)[0]
        dense_arm = {"delta": 0.0, "steps": K0, "bwd_ms": bwd0_ms,
                     "bwd_tflops": bwd_dense_fl / (bwd0_ms * 1e-3) / 1e12}
        step(rule_param)          # leave the workload's own selection in the buffers
        torch.cuda.synchronize()

    # ---- end to end through the API: host inputs in, results out, every step.  The
    # copies run on two side streams with double-buffered device inputs and outputs,
    # so step i+1's upload and step i's download overlap the kernels of the steps
    # around them; every step's copies lie inside the timed region.
    out_keys = ("o", "lse", "dq", "dk", "dv")
    h_out = [{k_: torch.empty_like(getattr(bufs, k_), device="cpu").pin_memory() for k_ in out_keys}
             for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in h_out[0].values())
    sets_in = [d_in, {k_: torch.empty_like(t) for k_, t in d_in.items()}]
    sets_buf = [bufs, lf.Buffers(desc, device=dev)]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    Ke = max(3, K)   # as many steps as the device-timed region
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e2s = torch.cuda.Event(enable_timing=True)
    e2e = torch.cuda.Event(enable_timing=True)
    e2s.record(stream)
    up.wait_event(e2s)
    # per set: q/k/v uploaded, dout uploaded, forward done, backward done, results out
    up_qkv, up_do, fwd_done, computed, downloaded = ([None, None] for _ in range(5))

    def upload(i):
        # the forward needs only q, k, v: dout follows, under the forward
        s_ = i % 2
        if computed[s_] is not None:          # step i-2 has finished reading this set
            up.wait_event(computed[s_])
        with torch.cuda.stream(up):
            for k_ in ("q", "k", "v"):
                sets_in[s_][k_].copy_(host[k_], non_blocking=True)
            up_qkv[s_] = torch.cuda.Event()
            up_qkv[s_].record(up)
            sets_in[s_]["dout"].copy_(host["dout"], non_blocking=True)
            up_do[s_] = torch.cuda.Event()
            up_do[s_].record(up)

    def download(s_, keys, after):
        down.wait_event(after)
        with torch.cuda.stream(down):
            for k_ in keys:
                h_out[s_][k_].copy_(getattr(sets_buf[s_], k_), non_blocking=True)

    upload(0)
    for i in range(Ke):
        s_ = i % 2
        din, b = sets_in[s_], sets_buf[s_]
        if downloaded[s_] is not None:        # step i-2's results have left this set
            stream.wait_event(downloaded[s_])
        stream.wait_event(up_qkv[s_])
        lf.lf_attn_fwd(desc, din["q"], din["k"], din["v"], b.o, b.lse)
        fwd_done[s_] = torch.cuda.Event()
        fwd_done[s_].record(stream)
        stream.wait_event(up_do[s_])
        lf.lf_block_select_rule(desc, din["dout"], b.o, rule_id, rule_param, 0, 0, 0, b.norm, b.D,
                                b.tau, b.w, b.keep, b.kept_idx, b.kept_cnt)
        lf.lf_attn_bwd(desc, din["q"], din["k"], din["v"], b.o, b.lse, din["dout"], b.D, b.w,
                       b.kept_idx, b.kept_cnt, b.dq, b.dk, b.dv, b.ws)
        computed[s_] = torch.cuda.Event()
        computed[s_].record(stream)
        if i + 1 < Ke:
            upload(i + 1)
        # O and LSE leave under the selection and the backward; the gradients after it
        download(s_, ("o", "lse"), fwd_done[s_])
        download(s_, ("dq", "dk", "dv"), computed[s_])
        downloaded[s_] = torch.cuda.Event()
        downloaded[s_].record(down)
    stream.wait_event(downloaded[(Ke - 1) % 2])
    e2e.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e2s.elapsed_time(e2e)
    lf.lf_check_device_error()

    # ---- max over ranks (the job is as slow as its slowest rank)
    total_ms, bwd_sum, e2e_ms = max_over_ranks([total_ms, bwd_sum, e2e_ms], dist, dev)
    bwd_ms = bwd_sum / K

    n = world
    step_fl = fwd_fl + bwd_exec_fl
    # the metric: the LazyFlash backward's executed FLOPs per second, whole job
    value = whole_job_tflops(n, K, bwd_exec_fl, bwd_sum)
    # end to end: the same backward FLOPs per second of data-fed step time (fwd, select,
    # bwd, host copies in and out)
    e2e_val = whole_job_tflops(n, Ke, bwd_exec_fl, e2e_ms)
    peaks = _load_json(os.path.join(ROOT, "MEASURED_PEAKS.json"))
    if peaks:
        peak, peak_burst, peak_src = (float(peaks["bf16_tflops_sustained"]),
                                      float(peaks["bf16_tflops"]), "measured")
    else:
        peak, peak_burst, peak_src = 1400.0, 1590.0, "fallback"
    hbm_peak = float(peaks["hbm_gbs"]) if peaks else 6650.0
    fwd_tf = fwd_fl / (fwd_ms * 1e-3) / 1e12
    bwd_tf = bwd_exec_fl / (bwd_ms * 1e-3) / 1e12
    traffic = _load_json(os.path.join(ROOT, "profiles", "traffic.json")) or {}

    def roof(kernel, call, achieved):
        rec = traffic.get(kernel) or {}
        t = None
        if rec.get("workload") == w.name and os.path.exists(os.path.join(ROOT, rec.get("source", "-"))):
            import hashlib
            with open(os.path.join(ROOT, rec["source"]), "rb") as f:
                if hashlib.sha1(f.read()).hexdigest()[:12] == rec.get("source_sha1"):
                    t = rec.get("bytes_per_launch")
        return {"bound": "tensor", "kernel": kernel, "timed": call, "achieved": achieved,
                "peak": peak, "peak_source": peak_src + " bf16, sustained (the kernel runs inside "
                "a long back-to-back step under the power cap)", "unit": "TFLOP/s",
                "frac": achieved / peak, "peak_burst": peak_burst, "frac_burst": achieved / peak_burst,
                "traffic": t}

    roof_fwd = roof("attn_fwd_kernel", "lf_attn_fwd (one kernel)", fwd_tf)
    roof_bwd = roof("attn_bwd_kernel", "the lf_attn_bwd call (memsets and the small dQ kernels "
                    "around attn_bwd_kernel included; the kernel is ~97%% of the call in the ncu "
                    "launch list); FLOPs: executed tile FLOPs of the kept query tiles", bwd_tf)
    sel_bytes = 2 * w.total_tokens * w.hq * w.d * 2 + w.total_tokens * w.hq * 4
    line = {
        "metric": args.metric, "value": value, "unit": "TFLOP/s",
        "value_is": "LazyFlash backward (lf_attn_bwd) executed TFLOP/s, whole job; "
                    "ms_per_step is the whole step (fwd + select + bwd)",
        "n_gpus": n, "steps": K,
        "warmup": max(3, args.warmup), "ms_per_step": total_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_of(w, args),
        "phases_ms": {"fwd": fwd_ms, "select": sel_ms, "bwd": bwd_ms},
        "bwd_ms": bwd_ms, "bwd_tflops_executed": bwd_tf,
        "bwd_tflops_dense_equiv": bwd_dense_fl / (bwd_ms * 1e-3) / 1e12,
        "fwd_tflops": fwd_tf,
        "step_tflops_executed": whole_job_tflops(n, K, step_fl, total_ms),
        "select_gbs": {"achieved": sel_bytes / (sel_ms * 1e-3) / 1e9, "peak": hbm_peak,
                       "frac": sel_bytes / (sel_ms * 1e-3) / 1e9 / hbm_peak,
                       "bytes": sel_bytes, "timed": "the lf_block_select call (norm pass and "
                       "selection kernels)"},
        "flops_per_step": {"fwd": fwd_fl, "bwd_executed": bwd_exec_fl, "bwd_dense": bwd_dense_fl},
        "kept_fraction": telemetry["kept_fraction"],
        "bwd_executed_fraction": bwd_exec_fl / bwd_dense_fl,
        "telemetry": telemetry,
        "roofline": roof_bwd,
        "roofline_fwd": roof_fwd,
        "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / Ke, "steps": Ke,
                "is": "backward executed FLOPs per second of data-fed step time (fwd, select, "
                      "bwd and the host copies of inputs and results)",
                "copies": "pinned host buffers; uploads and downloads on two side streams, "
                          "device inputs and outputs double-buffered; the forward starts once "
                          "q, k, v are in (dout follows under it) and O, LSE leave under the "
                          "backward"},
        "gpu_launches": kernels_per_step(w) * K,
        "clocks": clk,
    }
    if dense_arm is not None:
        dense_arm["time_ratio"] = bwd_ms / dense_arm["bwd_ms"]
        dense_arm["executed_fraction"] = bwd_exec_fl / bwd_dense_fl
        dense_arm["speedup"] = dense_arm["bwd_ms"] / bwd_ms
        line["vs_delta0"] = dense_arm
    if rank == 0 and n == 1 and not args.no_cpu_baseline:
        r = oracle_sample(w, inp, min(args.cpu_prefix, w.seqlens[0]))
        line["cpu_baseline"] = {
            "value": r["bwd_flops"] / r["bwd_s"] / 1e12, "unit": "TFLOP/s", "cores": r["threads"],
            "kind": "oracle", "seconds": r["step_s"], "bwd_seconds": r["bwd_s"],
            "sample": "oracle backward (executed tile FLOPs over its time) on the first %d tokens "
                      "of the %s workload, all %d heads; its forward and selection ran untimed"
                      % (min(args.cpu_prefix, w.seqlens[0]), w.name, w.hq)}
    if rank == 0 and n == 1 and args.workload == "headline" and not args.no_dense_arm:
        # the other configurations of the measurement plan, each at its own delta (the
        # Long workload also at delta 0, the dense backward): context beside the headline
        others = {}
        for name, ww in (("gqa_mid", synthetic.GQA_MID),
                         ("long_delta0", synthetic.LONG.with_(delta=0.0)),
                         ("long_delta0.05", synthetic.LONG.with_(delta=0.05)),
                         ("long_delta0.2", synthetic.LONG.with_(delta=0.2)),
                         ("varlen", synthetic.VARLEN)):
            others[name] = measure_workload(lf, ww, dev)
        base = others["long_delta0"]["bwd_ms"]
        for name in ("long_delta0.05", "long_delta0.2"):
            others[name]["bwd_time_vs_delta0"] = others[name]["bwd_ms"] / base
        line["other_workloads"] = others
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
