#!/usr/bin/env python
"""Benchmark: memory-efficient exact attention on B200 through libmea's C ABI.

Headline (one JSON line on rank 0): prefill TFLOP/s on the non-causal sequence
sweep B=8, H=16, K=64, fp16, M=N in {512, 1024, 2048, 4096} -- one step is one
mea_fwd call per sequence length.  The same line carries the roofline of the
prefill kernel, the KV-cache GB/s of a decode step (B=64, cached lengths
U[512, 8192], Hq=32, Hkv=8, K=128, bf16) with its own roofline, the other
prefill workloads (packed variable-length causal; GQA + ALiBi causal; the small
causal example), peak memory against a materialised-score baseline, clocks
sampled during the timed region, an end-to-end number with host buffers, and
the fp64 oracle timed on the host cores as a CPU baseline.

FLOPs count only visible (unmasked) query/key pairs: 4 * K * Hq * pairs.
Decode bytes are the cache rows read once (K and V) plus q and out.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU: launched by torchrun, each rank runs the same workload on its own
GPU (independent batches, weak scaling, no data-path collective); time is the
max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

METRIC = "attention TFLOP/s (prefill) and KV-cache GB/s (decode) on 1 B200, % of roofline"
WORKLOAD = "noncausal_fwd_sweep B=8 H=16 K=64 fp16 M=N in {512,1024,2048,4096}"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
CSRC = os.path.join(ROOT, "memory_efficient_exact_mea_b200", "csrc")


# ---------------------------------------------------------------------------
# Work accounting
# ---------------------------------------------------------------------------
def visible_pairs(M: int, N: int, causal: bool) -> int:
    if not causal:
        return M * N
    off = N - M
    return sum(max(0, min(N, i + off + 1)) for i in range(M))


def prefill_flops(p: synth.Prefill) -> float:
    causal = p.bias in ("causal", "blockdiag_causal")
    if p.seq_lens_q is not None:
        lk = p.seq_lens_k if p.seq_lens_k is not None else p.seq_lens_q
        pairs = sum(visible_pairs(m, n, causal) for m, n in zip(p.seq_lens_q, lk))
    else:
        pairs = p.B * visible_pairs(p.M, p.N, causal)
    return 4.0 * p.K * p.Hq * pairs


def block_sparse_flops(p: synth.Prefill, mask, block: int = 128) -> float:
    """4*K per visible (query, key) pair inside the kept blocks (causal pairs
    only under a causal mask); left-out blocks are not credited."""
    mb, nb = mask.shape[2], mask.shape[3]
    off = p.N - p.M
    pairs = np.zeros((mb, nb))
    for a in range(mb):
        rows = np.arange(a * block, min(p.M, (a + 1) * block))
        for c in range(nb):
            c0, c1 = c * block, min(p.N, (c + 1) * block)
            if p.bias == "causal":
                pairs[a, c] = np.clip(rows + off + 1 - c0, 0, c1 - c0).sum()
            else:
                pairs[a, c] = len(rows) * (c1 - c0)
    m = mask.expand(p.B, p.Hq, mb, nb).to(torch.float64).sum(dim=(0, 1)).numpy()
    return 4.0 * p.K * float((m * pairs).sum())


def chunk_flops(c: synth.Chunk) -> float:
    """4*K*Hq per visible pair: every cached row, plus the chunk's own rows up to
    the diagonal (all of them without the causal mask)."""
    pairs = 0
    for p, n in zip(c.past, c.q_lens):
        pairs += p * n + (n * (n + 1) // 2 if c.causal else n * n)
    return 4.0 * c.K * c.Hq * pairs


def decode_bytes(d: synth.Decode) -> float:
    el = 2
    cache = 2.0 * sum(d.kv_lens) * d.Hkv * d.K * el
    return cache + 2.0 * d.B * d.Hq * d.K * el


# Exponentials per clock per SM of the special-function unit (ex2.approx.f32),
# measured on this B200 with a microbenchmark; clocks.max.sm of the part.
EX2_PER_CLK_PER_SM = 16
SM_MAX_MHZ = 1965.0


def ex2_roofline(achieved_tflops: float, sms: int, K: int, sm_mhz: float | None = None) -> dict:
    """The prefill's second ceiling: one exponential per score, 4*K FLOP per score,
    so the exponential unit alone allows sms * 16 * f * 4K FLOP/s at SM clock f
    (the median sampled during the timed region when known, else the maximum)."""
    f = SM_MAX_MHZ if not sm_mhz else float(sm_mhz)
    peak = sms * EX2_PER_CLK_PER_SM * f * 1e6 * 4 * K / 1e12
    return {"bound": "ex2 (special-function unit)", "achieved": round(achieved_tflops, 1),
            "peak": round(peak, 1), "unit": "TFLOP/s", "frac": round(achieved_tflops / peak, 4),
            "peak_kind": f"derived: {sms} SMs x {EX2_PER_CLK_PER_SM} ex2/clk/SM (measured) x "
                         f"{f:.0f} MHz ({'sampled median' if sm_mhz else 'maximum'} SM clock) x "
                         f"{4 * K} FLOP per score"}


def load_peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


# The sources a kernel's compiled code depends on (for matching a recorded ncu
# capture to the current build).
KERNEL_SOURCES = {"fwd_sweep": ["mea_fwd_sm100.cu", "mea_internal.h", "sm100.cuh"]}


def kernel_source_hash(kernel: str = "fwd_sweep") -> str:
    h = hashlib.sha256()
    for name in sorted(KERNEL_SOURCES[kernel]):
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the kernel's current sources."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        t = json.load(f)
    e = t.get("kernels", {}).get(kernel)
    if e is None or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    return e.get("bytes_per_launch")


# ---------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.device_index = device_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.device_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9], float(parts[3])))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [r for r in rows if r[3] > 250.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[2])
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded),
                "sm_mhz_min": min(r[0] for r in loaded),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows), "samples_under_load": len(loaded)}


# ---------------------------------------------------------------------------
# Distributed plumbing (one process per GPU; timing reduction only)
# ---------------------------------------------------------------------------
def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world <= 1:
        return x
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# The measured path
# ---------------------------------------------------------------------------
def run_ours(args, rank, world, local):
    import memory_efficient_exact_mea_b200 as mea

    dev = torch.device("cuda", local if world > 1 else 0)
    stream = torch.cuda.current_stream(dev)
    peaks, peaks_kind = load_peaks()
    hbm_peak = float(peaks["hbm_gbs"])
    tc_peak = float(peaks["bf16_tflops"])  # fp16 and bf16 share the nominal dense rate

    # ---- headline workload: the sweep --------------------------------------
    sweep = [synth.noncausal_sweep(M) for M in synth.SWEEP_M]
    dev_in = [(p.q.to(dev), p.k.to(dev), p.v.to(dev)) for p in sweep]
    outs = [torch.empty_like(q) for (q, _, _) in dev_in]
    lses = [torch.empty((p.B, p.Hq, p.M), dtype=torch.float32, device=dev) for p in sweep]
    flops = [prefill_flops(p) for p in sweep]

    def step(events=None):
        for i, (p, (q, k, v)) in enumerate(zip(sweep, dev_in)):
            if events is not None:
                events[i][0].record(stream)
            mea.mea_fwd(q, k, v, bias="none", scale=p.scale, out=outs[i], lse=lses[i])
            if events is not None:
                events[i][1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert mea.read_device_status() == 0

    per_launch = [[] for _ in sweep]
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(torch.cuda.current_device()) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in sweep]
               for _ in range(args.steps)]
        t0.record(stream)
        for s in range(args.steps):
            step(evs[s])
        t1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    elapsed_ms = t0.elapsed_time(t1)
    for s in range(args.steps):
        for i in range(len(sweep)):
            per_launch[i].append(evs[s][i][0].elapsed_time(evs[s][i][1]))
    clocks = clk.summary()
    elapsed_ms = max_over_ranks(elapsed_ms, world)
    ms_per_step = elapsed_ms / args.steps
    total_flops = sum(flops) * args.steps * world
    value = total_flops / (elapsed_ms * 1e-3) / 1e12

    kernel_ms = [statistics.mean(x) for x in per_launch]
    achieved = sum(flops) / (sum(kernel_ms) * 1e-3) / 1e12
    sweep_detail = []
    for p, f, ms in zip(sweep, flops, kernel_ms):
        sweep_detail.append({"M": p.M, "ms": round(ms, 4), "tflops": round(f / ms / 1e9, 1)})

    # ---- peak memory vs a materialised-score baseline (context) ------------
    if rank == 0 and not args.no_memory:
        for d, p, (q, k, v) in zip(sweep_detail, sweep, dev_in):
            d.update(memory_report(mea, p, q, k, v, dev))

    # ---- end to end: host buffers through the public call ------------------
    e2e = measure_e2e(mea, sweep, dev, stream, args, world)

    # ---- the other workloads (secondary measurements) -----------------------
    also = {}
    also_clk = ClockSampler(torch.cuda.current_device()) if not args.quick else None
    if also_clk is not None:
        also_clk.__enter__()
    if not args.quick:
        also["varlen_causal"] = measure_prefill(mea, synth.varlen_causal(), dev, stream, tc_peak)
        also["gqa_alibi_causal"] = measure_prefill(mea, synth.gqa_alibi_causal(), dev, stream,
                                                   tc_peak)
        also["causal_small"] = measure_prefill(mea, synth.causal_small(), dev, stream, tc_peak,
                                               iters=50, host_paths=True)
        also["decode"] = measure_decode(mea, synth.decode_step(), dev, stream, hbm_peak)
        also["chunk_prefill"] = measure_chunk(mea, synth.chunk_prefill(), dev, stream, tc_peak)
        bs_p, bs_mask = synth.block_sparse_noncausal()
        also["block_sparse"] = measure_block_sparse(mea, bs_p, bs_mask, dev, stream, tc_peak)
        also["bwd_noncausal_m2048"] = measure_backward(mea, synth.noncausal_sweep(2048), dev,
                                                       stream, tc_peak)
        also["bwd_gqa_alibi_causal"] = measure_backward(mea, synth.gqa_alibi_causal(), dev,
                                                        stream, tc_peak)
    if also_clk is not None:
        also_clk.__exit__(None, None, None)
        also["clocks"] = also_clk.summary()  # sampled over these secondary measurements
    assert mea.read_device_status() == 0

    traffic = traffic_for("fwd_sweep")
    roofline = {
        "kernel": "fwd_kernel<K=64,f16,no mask> (sweep launches)",
        "bound": "tensor", "achieved": round(achieved, 1), "peak": tc_peak,
        "unit": "TFLOP/s", "frac": round(achieved / tc_peak, 4),
        "peak_kind": f"{peaks_kind} bf16 burst (fp16 nominal rate = bf16)",
        "traffic": traffic,
        "traffic_note": "mean DRAM read+write bytes per sweep launch (ncu, profiles/traffic.json);"
                        " algorithmic q+k+v+out = 65536*M bytes, mean 125.8 MB",
        "algorithmic": "4*K*H*B*M*N FLOP per launch",
        "second_ceiling": ex2_roofline(achieved,
                                       torch.cuda.get_device_properties(dev).multi_processor_count,
                                       64, clocks.get("sm_mhz")),
    }
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": 8, "H": 16, "K": 64, "seq_lens": list(synth.SWEEP_M),
                   "bias": "none", "global_batch": 8 * world,
                   "l2": "inputs exceed L2: 502 MB read per step in a fixed order",
                   "parallelism": f"replica x{world}"},
        "roofline": roofline, "sweep": sweep_detail, "also": also, "e2e": e2e,
        "gpu_launches": len(sweep) * args.steps, "clocks": clocks,
        "impl": "ours",
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(sweep[-1], args.cpu_seconds)
    return line


def memory_report(mea, p, q, k, v, dev):
    """Peak device MB of one call: ours vs the plain materialised-score attention."""
    torch.cuda.synchronize(dev)
    base = torch.cuda.memory_allocated(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    out, lse = mea.mea_fwd(q, k, v, scale=p.scale)
    torch.cuda.synchronize(dev)
    ours = (torch.cuda.max_memory_allocated(dev) - base) / 1e6
    del out, lse
    torch.cuda.synchronize(dev)
    torch.cuda.reset_peak_memory_stats(dev)
    # Materialised scores (the pages' naive attention), [B, H, M, N] in fp16.
    qt, kt, vt = (x.permute(0, 2, 1, 3) for x in (q, k, v))

    def naive():
        s = torch.matmul(qt, kt.transpose(-1, -2)) * p.scale
        return torch.matmul(torch.softmax(s, dim=-1), vt)

    naive()
    torch.cuda.synchronize(dev)
    naive_mb = (torch.cuda.max_memory_allocated(dev) - base) / 1e6
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(3):
        naive()
    e1.record()
    torch.cuda.synchronize(dev)
    return {"peak_mb_ours": round(ours, 1), "peak_mb_materialised": round(naive_mb, 1),
            "scores_mb_analytic": round(p.B * p.Hq * p.M * p.N * 2 / 1e6, 1),
            "materialised_ms": round(e0.elapsed_time(e1) / 3, 3)}


def measure_e2e(mea, sweep, dev, stream, args, world):
    """Same metric through the public call with host buffers: pinned H2D of q,k,v,
    the kernel, D2H of out and lse, every step, inside the timed region.  Uploads,
    kernels and downloads go on three streams, so the kernel of one sequence
    length overlaps the upload of the next and the download of the previous."""
    host = [(p.q.pin_memory(), p.k.pin_memory(), p.v.pin_memory()) for p in sweep]
    dbuf = [(torch.empty_like(hq, device=dev), torch.empty_like(hk, device=dev),
             torch.empty_like(hv, device=dev)) for (hq, hk, hv) in host]
    houts = [torch.empty_like(p.q).pin_memory() for p in sweep]
    hlses = [torch.empty((p.B, p.Hq, p.M), dtype=torch.float32).pin_memory() for p in sweep]
    dout = [torch.empty_like(d[0]) for d in dbuf]
    dlse = [torch.empty((p.B, p.Hq, p.M), dtype=torch.float32, device=dev) for p in sweep]
    h2d = sum(x.numel() * x.element_size() for t in host for x in t)
    d2h = sum(x.numel() * x.element_size() for x in houts) + sum(
        x.numel() * x.element_size() for x in hlses)
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    n = len(sweep)
    ev_in = [torch.cuda.Event() for _ in range(n)]
    ev_kern = [torch.cuda.Event() for _ in range(n)]
    ev_out = [torch.cuda.Event() for _ in range(n)]
    first = [True]

    def step():
        for i, p in enumerate(sweep):
            if not first[0]:
                s_up.wait_event(ev_kern[i])      # inputs i consumed by the previous step
                stream.wait_event(ev_out[i])     # outputs i downloaded by the previous step
            with torch.cuda.stream(s_up):
                for dst, src in zip(dbuf[i], host[i]):
                    dst.copy_(src, non_blocking=True)
                ev_in[i].record(s_up)
            stream.wait_event(ev_in[i])
            mea.mea_fwd(*dbuf[i], scale=p.scale, out=dout[i], lse=dlse[i], stream=stream)
            ev_kern[i].record(stream)
            s_down.wait_event(ev_kern[i])
            with torch.cuda.stream(s_down):
                houts[i].copy_(dout[i], non_blocking=True)
                hlses[i].copy_(dlse[i], non_blocking=True)
                ev_out[i].record(s_down)
        first[0] = False

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    n_steps = max(1, min(args.steps, 10))
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    for _ in range(n_steps):
        step()
    s_up.wait_stream(s_down)
    s_up.wait_stream(stream)
    e1.record(s_up)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    flops = sum(prefill_flops(p) for p in sweep) * n_steps * world
    return {"value": round(flops / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_steps,
            "ms_per_step": round(ms / n_steps, 3),
            "overlap": "uploads, kernels and downloads on three streams"}


def _time(fn, stream, iters, warmup=3, rounds=3):
    """Mean time of one call over `iters` back-to-back calls, the best of `rounds`
    such runs (a run that a clock dip or another tenant slowed is not the
    kernel's time)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(rounds):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(iters):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1) / iters)
    return best


def measure_prefill(mea, p, dev, stream, tc_peak, iters=10, host_paths=False):
    q, k, v = p.q.to(dev), p.k.to(dev), p.v.to(dev)
    kw = {}
    if p.seq_lens_q is not None:
        kw = dict(seqstart_q=p.seqstart_q.to(dev), seqstart_k=p.seqstart_k.to(dev),
                  max_seqlen_q=max(p.seq_lens_q),
                  max_seqlen_k=max(p.seq_lens_k or p.seq_lens_q))
    out = torch.empty_like(q)
    lse = torch.empty((p.B, p.Hq, p.M), dtype=torch.float32, device=dev)
    ms = _time(lambda: mea.mea_fwd(q, k, v, bias=p.bias, scale=p.scale, alibi=p.alibi, out=out,
                                   lse=lse, **kw), stream, iters)
    f = prefill_flops(p)
    tf = f / (ms * 1e-3) / 1e12
    r = {"workload": p.name, "ms": round(ms, 4), "tflops": round(tf, 1),
         "frac": round(tf / tc_peak, 4), "flop": f, "bound": "tensor"}
    if host_paths:
        # Calls back to back on one stream, three ways: the plain binding call
        # above (Python marshalling every call), a prepared call (the C entry
        # point only), and prepared calls captured in a CUDA graph (launch gaps
        # only: close to the kernel's own time).
        call = mea.mea_fwd(q, k, v, bias=p.bias, scale=p.scale, alibi=p.alibi, out=out, lse=lse,
                           prepare=True, **kw)
        r["ms_prepared"] = round(_time(call, stream, iters), 4)
        g = torch.cuda.CUDAGraph()
        torch.cuda.synchronize()
        with torch.cuda.graph(g):  # prepared on the capturing stream
            gcall = mea.mea_fwd(q, k, v, bias=p.bias, scale=p.scale, alibi=p.alibi, out=out,
                                lse=lse, prepare=True, **kw)
            for _ in range(20):
                gcall()
        torch.cuda.synchronize()
        r["ms_graph"] = round(_time(g.replay, torch.cuda.current_stream(), 5) / 20, 4)
        r["host_note"] = "ms: plain binding call; ms_prepared: marshalled once; ms_graph: 20 calls per CUDA graph"
    return r


def measure_block_sparse(mea, p, mask, dev, stream, tc_peak, iters=10):
    q, k, v = p.q.to(dev), p.k.to(dev), p.v.to(dev)
    bm = mask.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((p.B, p.Hq, p.M), dtype=torch.float32, device=dev)
    ms = _time(lambda: mea.mea_fwd_block_sparse(q, k, v, bm, bias=p.bias, scale=p.scale,
                                                alibi=p.alibi, out=out, lse=lse), stream, iters)
    f = block_sparse_flops(p, mask)
    tf = f / (ms * 1e-3) / 1e12
    kept = float(mask.to(torch.float64).mean())
    return {"workload": p.name, "ms": round(ms, 4), "tflops": round(tf, 1),
            "frac": round(tf / tc_peak, 4), "flop": f, "bound": "tensor",
            "kept_block_fraction": round(kept, 4)}


def measure_chunk(mea, c: synth.Chunk, dev, stream, tc_peak, iters=10):
    """mea_prefill_chunk: attention of the chunk plus the fused append, timed
    together (the same chunk re-appended each iteration)."""
    q, kn, vn = c.q.to(dev), c.k_new.to(dev), c.v_new.to(dev)
    kc, vc = c.k_cache.to(dev), c.v_cache.to(dev)
    cl = torch.tensor(c.past, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty((c.B, c.Hq, c.M), dtype=torch.float32, device=dev)
    ms = _time(lambda: mea.mea_prefill_chunk(q, kn, vn, kc, vc, cl, causal=c.causal,
                                             scale=c.scale, alibi=c.alibi, out=out, lse=lse),
               stream, iters)
    f = chunk_flops(c)
    tf = f / (ms * 1e-3) / 1e12
    return {"workload": c.name, "ms": round(ms, 4), "tflops": round(tf, 1),
            "frac": round(tf / tc_peak, 4), "flop": f, "bound": "tensor",
            "note": "includes the append of 512 rows x 8 kv heads per sequence"}


def measure_backward(mea, p, dev, stream, tc_peak, iters=5):
    """mea_bwd alone (the forward that makes out and lse runs once, untimed).
    Work: five contractions of 2*K FLOP per visible (query, key) pair -- S, dP,
    dV, dK, dQ -- i.e. 2.5x the forward's count."""
    q, k, v = p.q.to(dev), p.k.to(dev), p.v.to(dev)
    kw = {}
    if p.seq_lens_q is not None:
        kw = dict(seqstart_q=p.seqstart_q.to(dev), seqstart_k=p.seqstart_k.to(dev),
                  max_seqlen_q=max(p.seq_lens_q),
                  max_seqlen_k=max(p.seq_lens_k or p.seq_lens_q))
    g = synth.generator(p.seed + 17)
    dout = synth.randn(tuple(p.q.shape), p.dtype, g).to(dev)
    out, lse = mea.mea_fwd(q, k, v, bias=p.bias, scale=p.scale, alibi=p.alibi, **kw)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    B, M, Hq, K = q.shape
    ws = torch.empty(mea.lib.mea_bwd_workspace_size(B, M, Hq, K), dtype=torch.uint8, device=dev)
    def run(stages=7):
        mea.mea_bwd(q, k, v, out, dout, lse, bias=p.bias, scale=p.scale, alibi=p.alibi, dq=dq,
                    dk=dk, dv=dv, workspace=ws, stages=stages, **kw)

    ms = _time(run, stream, iters)
    # The three launches one by one (mea_bwd_stages), with events between them.
    names = ("bwd_prep", "bwd_kernel", "bwd_dq_out")
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(iters)]
    for e in evs:
        e[0].record(stream)
        for i, st in enumerate((1, 2, 4)):
            run(st)
            e[i + 1].record(stream)
    torch.cuda.synchronize()
    stage_ms = {n: round(statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs), 4)
                for i, n in enumerate(names)}
    f = 2.5 * prefill_flops(p)
    tf = f / (ms * 1e-3) / 1e12
    tf_main = f / (stage_ms["bwd_kernel"] * 1e-3) / 1e12
    return {"workload": "bwd_" + p.name, "ms": round(ms, 4), "tflops": round(tf, 1),
            "frac": round(tf / tc_peak, 4), "flop": f, "bound": "tensor",
            "stage_ms": stage_ms, "bwd_kernel_tflops": round(tf_main, 1),
            "bwd_kernel_frac": round(tf_main / tc_peak, 4),
            "kernel": "bwd_kernel (tcgen05, TMA; dq by TMA tensor reductions)"}


def measure_decode(mea, d, dev, stream, hbm_peak, iters=20):
    q, kc, vc = d.q.to(dev), d.k_cache.to(dev), d.v_cache.to(dev)
    st = d.kv_seqstart.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((d.B, d.Hq), dtype=torch.float32, device=dev)
    ws = torch.empty(mea.mea_decode_workspace_size(d.B, d.Hq, d.Hkv, d.K, d.max_kv_len),
                     dtype=torch.uint8, device=dev)
    ms = _time(lambda: mea.mea_decode(q, kc, vc, st, d.max_kv_len, scale=d.scale, out=out, lse=lse,
                                      workspace=ws), stream, iters)
    nbytes = decode_bytes(d)
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": d.name, "ms": round(ms, 4), "gbs": round(gbs, 1),
            "frac": round(gbs / hbm_peak, 4), "bytes": nbytes, "bound": "hbm",
            "peak": hbm_peak, "note": "cache larger than L2 (1.1 GB)"}


# ---------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on the host cores, bounded sample
# ---------------------------------------------------------------------------
_F64_INPUTS = {}


def cpu_baseline(p: synth.Prefill, seconds: float):
    import oracle

    orc = oracle.get()
    if p.name not in _F64_INPUTS:  # exact fp64 copies, made once per workload
        _F64_INPUTS[p.name] = tuple(t.to(torch.float64).numpy() for t in (p.q, p.k, p.v))
    qf, kf, vf = _F64_INPUTS[p.name]
    rng = np.random.default_rng(0)
    rows_done, t_used, batch = 0, 0.0, 64
    while t_used < seconds:
        rows = np.stack([rng.integers(p.B, size=batch), rng.integers(p.M, size=batch),
                         rng.integers(p.Hq, size=batch)], axis=1)
        t = time.perf_counter()
        orc.attention_rows(qf, kf, vf, rows, bias=0, scale=p.scale)
        t_used += time.perf_counter() - t
        rows_done += batch
        batch = min(batch * 2, 4096)
    flops = rows_done * 4.0 * p.K * p.N
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": round(flops / t_used / 1e12, 6), "unit": "TFLOP/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{rows_done} random query rows of M=N={p.M} (B=8,H=16,K=64) in "
                      f"{t_used:.1f} s, fp64 C oracle, OpenMP over rows"}


def run_reference(args, rank, world):
    """The reference arm for this build is the fp64 oracle on the host cores."""
    if rank != 0:
        return None
    p = synth.noncausal_sweep(4096)
    # About two minutes of oracle work in all, whatever --steps / --warmup are.
    per_step = max(0.05, min(15.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_baseline(p, per_step / 4)
    t_start = time.perf_counter()
    vals = [cpu_baseline(p, per_step) for _ in range(args.steps)]
    ms_per_step = (time.perf_counter() - t_start) * 1e3 / max(1, args.steps)
    v = statistics.mean(x["value"] for x in vals)
    cb = dict(vals[-1])
    cb["value"] = round(v, 6)
    return {"metric": METRIC, "value": round(v, 6), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": 8, "H": 16, "K": 64,
                       "seq_lens": list(synth.SWEEP_M), "bias": "none"},
            "impl": "reference", "cpu_baseline": cb,
            "e2e": {"value": round(v, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


PROFILE_CASES = {
    # small cases for ncu captures: inputs larger than L2, a few hundred MB at most
    "fwd_sweep_all": lambda: ("sweep", None),
    "fwd_sweep_m2048": lambda: ("fwd", synth.noncausal_sweep(2048)),
    "fwd_gqa_alibi_m2048": lambda: ("fwd", synth.gqa_alibi_causal(M=2048, B=2)),
    "fwd_gqa_alibi_full": lambda: ("fwd", synth.gqa_alibi_causal()),
    "bwd_gqa_alibi_full": lambda: ("bwd", synth.gqa_alibi_causal()),
    "fwd_varlen": lambda: ("fwd", synth.varlen_causal()),
    "bwd_m2048": lambda: ("bwd", synth.noncausal_sweep(2048)),
    "block_sparse_m2048": lambda: ("sparse", synth.block_sparse_noncausal(2048)),
    "chunk_prefill": lambda: ("chunk", synth.chunk_prefill()),
    "decode_b16": lambda: ("decode", synth.make_decode(
        "decode_b16", synth.decode_lengths()[:16], 32, 8, 128, "bf16", seed=1005)),
}


def run_profile(args):
    """Launch one workload W + K times (no JSON): the target of an ncu capture."""
    import memory_efficient_exact_mea_b200 as mea

    kind, w = PROFILE_CASES[args.profile]()
    dev = torch.device("cuda", 0)
    if kind == "sweep":  # one launch per sweep size per step
        sweep = [synth.noncausal_sweep(M) for M in synth.SWEEP_M]
        ins = [(p.q.to(dev), p.k.to(dev), p.v.to(dev), p.scale) for p in sweep]

        def fn():
            for q, k, v, sc in ins:
                mea.mea_fwd(q, k, v, scale=sc)
    elif kind == "fwd":
        q, k, v = w.q.to(dev), w.k.to(dev), w.v.to(dev)
        kw = {}
        if w.seq_lens_q is not None:
            kw = dict(seqstart_q=w.seqstart_q.to(dev), seqstart_k=w.seqstart_k.to(dev))

        def fn():
            mea.mea_fwd(q, k, v, bias=w.bias, scale=w.scale, alibi=w.alibi, **kw)
    elif kind == "sparse":
        w, mask = w
        q, k, v, bm = w.q.to(dev), w.k.to(dev), w.v.to(dev), mask.to(dev)

        def fn():
            mea.mea_fwd_block_sparse(q, k, v, bm, bias=w.bias, scale=w.scale, alibi=w.alibi)
    elif kind == "chunk":
        q, kn, vn = w.q.to(dev), w.k_new.to(dev), w.v_new.to(dev)
        kc, vc = w.k_cache.to(dev), w.v_cache.to(dev)
        cl = torch.tensor(w.past, dtype=torch.int32, device=dev)

        def fn():
            mea.mea_prefill_chunk(q, kn, vn, kc, vc, cl, causal=w.causal, scale=w.scale)
    elif kind == "bwd":
        q, k, v = w.q.to(dev), w.k.to(dev), w.v.to(dev)
        dout = synth.randn(tuple(w.q.shape), w.dtype, synth.generator(w.seed + 17)).to(dev)
        out, lse = mea.mea_fwd(q, k, v, bias=w.bias, scale=w.scale, alibi=w.alibi)

        def fn():
            mea.mea_bwd(q, k, v, out, dout, lse, bias=w.bias, scale=w.scale, alibi=w.alibi)
    else:
        q, kc, vc = w.q.to(dev), w.k_cache.to(dev), w.v_cache.to(dev)
        st = w.kv_seqstart.to(dev)

        def fn():
            mea.mea_decode(q, kc, vc, st, w.max_kv_len, scale=w.scale)
    for _ in range(args.warmup + args.steps):
        fn()
    torch.cuda.synchronize()
    assert mea.read_device_status() == 0
    print(f"profiled {args.profile}: {args.warmup} + {args.steps} launches", flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--quick", action="store_true", help="headline only, skip other workloads")
    ap.add_argument("--no-memory", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--profile", choices=sorted(PROFILE_CASES),
                    help="launch one small workload only (target for ncu)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.profile:
        run_profile(args)
        return
    rank, world, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            line = run_reference(args, rank, world)
        else:
            line = run_ours(args, rank, world, local)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
