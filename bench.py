#!/usr/bin/env python
"""Benchmark of the quantized-attention hot path on B200.

One step = sage_quant_qkv (K/V smoothing, INT8 Q/K and FP8 V quantization) +
sage_attn_fwd over one batch of the long-video workload (B=1, H=32, N=55296,
D=128, BF16 NHD; synthetic, seeded), the largest single-GPU configuration.
Prints ONE JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload action_dit|mid_video|long_video|ragged|tiny]
                    [--q-gran block64|token|segment64] [--k-gran block64|token|segment64]
                    [--quant fused|separate] [--normrope] [--op attention|fp8_linear]

value      = attention ops (4*B*H*N^2*D, INT8 QK^T + FP8 PV) per step, all ranks,
             / device time of the whole step (quant + attention), in TOPS;
             the step's launches replayed as one CUDA graph (eager launches:
             eager_value); inputs resident in HBM, L2 flushed (256 MiB write)
             between steps, per-step CUDA events on the launching stream, max
             over ranks.
e2e        = the same metric through the Python API with pinned host inputs:
             H2D of Q, K, V + the calls + D2H of the BF16 output, every step,
             pipelined over two buffer sets (copy-in, compute, copy-out on three
             streams; one device-timed region over all K steps); the one-stream
             serial figure is reported beside it.
roofline   = the attention kernel alone: ops / its mean event-timed duration,
             against the INT8/FP8 dense peak derived from the measured BF16 peak.
workloads  = (default run, one GPU) the other large workloads, eager: attention
             time, TOPS and roofline fraction, and the GB/s of the fused
             quantization call and of sage_quant_qk and sage_quant_v standalone.
cpu_baseline (N=1, rank 0) = the CPU oracle timed on a bounded sample.
--impl reference runs the CPU oracle (the reference arm) instead.
Multi-GPU: one process per GPU (torchrun); every rank runs its own batch
(replicas, weak scaling, no collective on the data path).
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_PER_BF16 = 4.5 / 2.25  # nominal dense INT8/FP8 : BF16 tensor throughput ratio
DEFAULT_WORKLOAD = "long_video"  # the largest single-GPU workload


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def kernel_traffic(key: str, sources, workload: str):
    """DRAM bytes per launch of a kernel from the last ncu capture of it
    (profiles/ncu_counters.json), if that capture was taken on this workload
    and on the current kernel source (SHA-256 of `sources`); None otherwise."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "ncu_counters.json")) as f:
            rec = json.load(f)[key][workload]
    except (OSError, KeyError, ValueError):
        return None
    h = hashlib.sha256()
    for name in sources:
        with open(os.path.join(ROOT, "action_diffusion_transformers_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    if rec.get("source_sha256") != h.hexdigest():
        return None
    return rec.get("dram_bytes_per_launch")


ATTN_SOURCES = ("sage_attn.cuh", "sage_ptx.cuh")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=None, choices=sorted(synth.WORKLOADS),
                    help=f"default: {DEFAULT_WORKLOAD}, followed by a summary of the other large workloads")
    ap.add_argument("--no-summary", action="store_true",
                    help="skip the per-workload summary that the default run appends")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--q-gran", default="block64", choices=["block64", "token", "segment64"],
                    help="INT8 scale groups of Q (default: 64-token blocks)")
    ap.add_argument("--k-gran", default="block64", choices=["block64", "token", "segment64"],
                    help="INT8 scale groups of K (default: 64-token blocks)")
    ap.add_argument("--quant", default="fused", choices=["fused", "separate"],
                    help="fused: sage_quant_qkv (4 launches); separate: sage_quant_qk + sage_quant_v (6)")
    ap.add_argument("--op", default="attention", choices=["attention", "fp8_linear"],
                    help="attention: the quantized attention path (default); fp8_linear: the row-wise "
                         "FP8 projections of a joint block on the same tokens")
    ap.add_argument("--normrope", action="store_true",
                    help="Q and K are projection outputs: QK RMSNorm + RoPE fused into the quantization")
    ap.add_argument("--peaks", action="store_true",
                    help="measure library INT8 / FP8 / BF16 GEMM throughput at 8192^3 and exit")
    return ap.parse_args()


def quant_bytes(w, q_gran="block64", k_gran="block64"):
    """Algorithmic bytes of the two quantization calls (per step): 4 B per Q/K
    scale, one per 64-token block or one per (padded) token."""
    elems = w.B * w.N * w.H * w.D
    npad = (w.N + 127) // 128 * 128
    scales = sum(w.B * w.H * (npad // 64 if g == "block64" else npad) for g in (q_gran, k_gran))
    chans = w.B * w.H * w.D
    qk = elems * (2 + 2 + 1 + 1) + scales * 4 + chans * 2
    v = elems * (2 + 1) + chans * 8
    return qk, v


# ----------------------------------------------------------------------------- ranks
def rank_env():
    """(rank, world size, local rank) of this process, as torchrun sets them."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest x over all ranks (every rank gets it); x itself when alone."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tops(world: int, ops_per_step: float, steps: int, max_total_ms: float) -> float:
    """Whole-job throughput: every rank runs `steps` steps of its own batch
    (replicas), so the job does world * ops * steps in the slowest rank's time."""
    return world * ops_per_step * steps / (max_total_ms / 1e3) / 1e12


def pipelined_e2e(torch, n: int, stream, copy_in, compute, copy_out) -> float:
    """Device milliseconds of n end-to-end steps over two device buffer sets
    (slot = step & 1): copy_in(slot) (host -> device) runs on one stream,
    compute(slot) on `stream`, copy_out(slot) (device -> host) on a third, so
    step i+1's inputs cross PCIe while step i computes.  A slot's inputs are
    rewritten only after the step two back has computed on them, and its
    outputs only after they have been copied out.  One pair of events on
    `stream` brackets the whole region."""
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    new_ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    start, end = new_ev(), new_ev()
    computed, copied = [None] * n, [None] * n
    start.record(stream)
    s_in.wait_event(start)
    for i in range(n):
        slot = i & 1
        if i >= 2:
            s_in.wait_event(computed[i - 2])
        with torch.cuda.stream(s_in):
            copy_in(slot)
        ready = new_ev()
        ready.record(s_in)
        stream.wait_event(ready)
        if i >= 2:
            stream.wait_event(copied[i - 2])
        compute(slot)
        computed[i] = new_ev()
        computed[i].record(stream)
        s_out.wait_event(computed[i])
        with torch.cuda.stream(s_out):
            copy_out(slot)
        copied[i] = new_ev()
        copied[i].record(s_out)
    stream.wait_event(copied[n - 1])
    end.record(stream)
    torch.cuda.synchronize()
    return start.elapsed_time(end)


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.proc = None
        self.path = None
        if gpu_id is None:
            return
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = [l.split(",") for l in open(self.path).read().strip().splitlines() if l.count(",") >= 8]
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        load = [s for s in sm if mx and s > 0.3 * max(mx)] or sm
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def gpu_id_for(dev_index: int):
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev_index).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            return vis.split(",")[dev_index]
        return str(dev_index)


# ----------------------------------------------------------------------------- oracle
def oracle_sample(w, qb, kb, vb, rows: int, heads: int, q_gran="block64", k_gran="block64", normrope=None):
    """Time the CPU oracle on `heads` heads of batch 0 (full quantization of those
    heads, attention for `rows` query rows).  Returns (ops, seconds)."""
    from oracle import sage_oracle as so
    t0 = time.perf_counter()
    sl = (slice(0, 1), slice(None), slice(0, heads), slice(None))
    qk = so.quant_qk(qb[sl], kb[sl], q_gran, k_gran, w.cu_seqlens, normrope=normrope)
    vv = so.quant_v(vb[sl])
    r = synth.sample_rows(w.N, rows, 0)[:rows] if rows < w.N else None
    so.attn_fwd(qk["q_codes"], qk["q_scale"], qk["k_codes"], qk["k_scale"], vv["v_codes_t"], vv["v_scale"],
                vv["v_mean"], w.N, rows=r)
    dt = time.perf_counter() - t0
    nrows = w.N if r is None else len(r)
    return 4.0 * heads * nrows * w.N * w.D, dt


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def run_reference_fp8(args, w):
    host = []
    for i, (name, K, N) in enumerate(fp8_shapes(w)):
        xb, wb = fp8_inputs(w, K, N, w.seed * 10 + i)
        host.append((xb, wb, (K, N)))
    rows = 16
    for _ in range(args.warmup):
        fp8_oracle_sample(w, host, rows)
    times = []
    flops = 0.0
    for _ in range(args.steps):
        flops, dt = fp8_oracle_sample(w, host, rows)
        times.append(dt)
    tot = sum(times)
    value = flops * len(times) / tot / 1e12
    sample = f"{rows} tokens through each of the {len(host)} projections"
    line = {"impl": "reference", "metric": "fp8 projection TFLOPS", "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot / len(times), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64 exact (CPU oracle)", "data": "synthetic",
            "config": {"workload": f"{w.name} joint-block projections", "tokens": w.B * w.N, "hidden": w.H * w.D},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_reference(args, rank):
    if rank != 0:
        return
    w = synth.WORKLOADS[args.workload]
    if args.op == "fp8_linear":
        run_reference_fp8(args, w)
        return
    qb, kb, vb = synth.generate(w)
    rows, heads = 256, 1
    grans = (args.q_gran, args.k_gran)
    for _ in range(args.warmup):
        oracle_sample(w, qb, kb, vb, rows, heads, *grans)
    times = []
    ops = 0.0
    for _ in range(args.steps):
        ops, dt = oracle_sample(w, qb, kb, vb, rows, heads, *grans)
        times.append(dt)
    tot = sum(times)
    value = ops * len(times) / tot / 1e12
    sample = f"1 head of batch 0: full K/V quantization of that head + attention for {rows} query rows"
    line = {"impl": "reference", "metric": "quantized-attention TOPS", "value": value, "unit": "TOPS",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot / len(times), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32/f64 (CPU oracle)", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "N": w.N, "H": w.H, "D": w.D,
                       "q_gran": args.q_gran, "k_gran": args.k_gran},
            "cpu_baseline": {"value": value, "unit": "TOPS", "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- peaks
def measure_peaks(reps: int = 20):
    """Dense GEMM throughput of the libraries torch calls (cuBLAS / cuBLASLt) at
    8192^3: torch._int_mm (INT8 -> INT32), torch._scaled_mm (FP8 E4M3 -> BF16)
    and torch.matmul (BF16), best of `reps` event-timed calls.  Context for the
    attention roofline, whose peak stays the measured BF16 figure x 2."""
    import torch
    n = 8192
    torch.manual_seed(0)
    a8 = torch.randint(-127, 128, (n, n), dtype=torch.int8, device="cuda")
    b8 = torch.randint(-127, 128, (n, n), dtype=torch.int8, device="cuda").t()
    af = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
    bf = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn).t()
    one = torch.ones((), device="cuda")
    ab = torch.randn(n, n, device="cuda", dtype=torch.bfloat16)
    bb = torch.randn(n, n, device="cuda", dtype=torch.bfloat16)
    cases = {"int8_tops": lambda: torch._int_mm(a8, b8),
             "fp8_tflops": lambda: torch._scaled_mm(af, bf, scale_a=one, scale_b=one, out_dtype=torch.bfloat16),
             "bf16_tflops": lambda: ab @ bb}
    out = {}
    for name, fn in cases.items():
        for _ in range(3):
            fn()
        best = float("inf")
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1))
        out[name] = 2.0 * n ** 3 / (best / 1e3) / 1e12
    return out


# ----------------------------------------------------------------------------- FP8 projections
def fp8_shapes(w):
    """(name, K, N) of the FP8 projections of one joint block on the workload's
    tokens (hidden H*D, MLP ratio 4): attention output, MLP up, MLP down."""
    hid = w.H * w.D
    return [("attn_out", hid, hid), ("mlp_up", hid, 4 * hid), ("mlp_down", 4 * hid, hid)]


def fp8_inputs(w, K, N, seed):
    """Seeded BF16 activations [M, K] (per-token log-normal magnitude) and weights [N, K] ~ N(0, 0.02^2)."""
    rng = np.random.default_rng(70_000 + seed)
    M = w.B * w.N
    x = (rng.standard_normal((M, K), dtype=np.float32) * np.exp(rng.standard_normal((M, 1))).astype(np.float32))
    wt = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    return synth.to_bf16_bits(x), synth.to_bf16_bits(wt)


def fp8_oracle_sample(w, host, rows: int):
    """The CPU oracle on `rows` tokens of every projection (weights quantized
    once, outside the timing).  Returns (flops, seconds)."""
    from oracle import fp8_linear as fl
    wq = [fl.fp8_quant_rows(wb) for _, wb, _ in host]
    t0 = time.perf_counter()
    flops = 0.0
    for (xb, _, (K, N)), (wqc, wsc) in zip(host, wq):
        xq, sx = fl.fp8_quant_rows(xb[:rows])
        fl.fp8_linear(xq, sx, wqc, wsc)
        flops += 2.0 * rows * N * K
    return flops, time.perf_counter() - t0


def run_fp8_linear(args, rank, world, local):
    import torch
    import torch.distributed as dist

    import action_diffusion_transformers_b200 as adt

    w = synth.WORKLOADS[args.workload]
    M = w.B * w.N
    host = []
    for i, (name, K, N) in enumerate(fp8_shapes(w)):
        xb, wb = fp8_inputs(w, K, N, w.seed * 10 + i)
        host.append((xb, wb, (K, N)))
    as_dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()  # noqa: E731
    dev = []
    for xb, wb, (K, N) in host:
        x = as_dev(xb)
        wd = as_dev(wb)
        wq = torch.empty((N, K), dtype=torch.uint8, device="cuda")
        sw = torch.empty(N, dtype=torch.float32, device="cuda")
        adt.sage_fp8_quant_rows(wd, wq, sw)           # offline: the weights' E4M3 codes and row scales
        del wd
        xq = torch.empty((M, K), dtype=torch.uint8, device="cuda")
        sx = torch.empty(M, dtype=torch.float32, device="cuda")
        out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        dev.append(dict(x=x, wq=wq, sw=sw, xq=xq, sx=sx, out=out, K=K, N=N))
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    flops = sum(2.0 * M * d["N"] * d["K"] for d in dev)

    def step(evs=None):
        for i, d in enumerate(dev):
            adt.sage_fp8_quant_rows(d["x"], d["xq"], d["sx"], stream)
            if evs is not None:
                evs[i].record(stream)
            adt.sage_fp8_linear(d["xq"], d["sx"], d["wq"], d["sw"], d["out"], stream)
            if evs is not None:
                evs[len(dev) + i].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(max(3, args.warmup)):
        step()
    adt.sage_check()
    torch.cuda.synchronize()
    barrier()
    K_steps = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * len(dev) + 1)] for _ in range(K_steps)]
    sampler = ClockSampler(gpu_id_for(local))
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    for i in range(K_steps):
        flush.fill_(i & 0xFF)
        ev[i][0].record(stream)
        step(ev[i][1:])
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    adt.sage_check()
    nd = len(dev)
    step_ms = [e[0].elapsed_time(e[2 * nd]) for e in ev]
    max_total_ms = max_over_ranks(sum(step_ms), world, "cuda")
    value = job_tops(world, flops, K_steps, max_total_ms)
    quant_us, gemm_us = {}, {}
    for j, (name, _, _) in enumerate(fp8_shapes(w)):
        prev = [e[0] if j == 0 else e[nd + j] for e in ev]
        quant_us[name] = 1e3 * statistics.mean(p.elapsed_time(e[1 + j]) for p, e in zip(prev, ev))
        gemm_us[name] = 1e3 * statistics.mean(e[1 + j].elapsed_time(e[1 + nd + j]) for e in ev)

    # e2e: pinned host activations in, BF16 projection outputs back, every step
    # (serial on one stream, then pipelined over two buffer sets)
    hx = [torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).pin_memory() for xb, _, _ in host]
    hout = [[torch.empty(d["out"].shape, dtype=torch.bfloat16).pin_memory() for d in dev] for _ in range(2)]
    e2e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K_steps)]

    def e2e_step():
        for d, h in zip(dev, hx):
            d["x"].copy_(h, non_blocking=True)
        step()
        for d, h in zip(dev, hout[0]):
            h.copy_(d["out"], non_blocking=True)
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    for i in range(K_steps):
        flush.fill_(i & 0xFF)
        e2e_ev[i][0].record(stream)
        e2e_step()
        e2e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    adt.sage_check()
    e2e_serial = job_tops(world, flops, K_steps, max_over_ranks(sum(a.elapsed_time(b) for a, b in e2e_ev), world,
                                                                 "cuda"))
    dev2 = [dict(d, x=torch.empty_like(d["x"]), xq=torch.empty_like(d["xq"]), sx=torch.empty_like(d["sx"]),
                 out=torch.empty_like(d["out"])) for d in dev]
    sets = [dev, dev2]

    def copy_in(j):
        for d, h in zip(sets[j], hx):
            d["x"].copy_(h, non_blocking=True)

    def compute(j):
        for d in sets[j]:
            adt.sage_fp8_quant_rows(d["x"], d["xq"], d["sx"], stream)
            adt.sage_fp8_linear(d["xq"], d["sx"], d["wq"], d["sw"], d["out"], stream)

    def copy_out(j):
        for d, h in zip(sets[j], hout[j]):
            h.copy_(d["out"], non_blocking=True)

    pipelined_e2e(torch, 3, stream, copy_in, compute, copy_out)
    barrier()
    e2e_ms = pipelined_e2e(torch, K_steps, stream, copy_in, compute, copy_out)
    barrier()
    adt.sage_check()
    e2e_value = job_tops(world, flops, K_steps, max_over_ranks(e2e_ms, world, "cuda"))
    last = (K_steps - 1) & 1
    if not all(torch.equal(h, d["out"].cpu()) for h, d in zip(hout[last], sets[last])):
        raise RuntimeError("pipelined e2e: the copied-out output differs from the device result")
    h2d = sum(xb.nbytes for xb, _, _ in host)
    d2h = sum(d["out"].numel() * 2 for d in dev)

    peaks, src = load_peaks()
    peak = peaks["bf16_tflops"] * INT8_PER_BF16
    # the dominant launch: the MLP up-projection
    _, k_up, n_up = fp8_shapes(w)[1]
    achieved = 2.0 * M * n_up * k_up / (gemm_us["mlp_up"] / 1e6) / 1e12
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows = 16
        o_flops, o_dt = fp8_oracle_sample(w, host, rows)
        cpu = {"value": o_flops / o_dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"{rows} tokens through each of the {len(dev)} projections ({o_dt:.1f} s)"}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    x_bytes = sum(M * d["K"] * (2 + 1) + M * 4 for d in dev)
    line = {
        "metric": "fp8 projection TFLOPS", "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K_steps,
        "warmup": args.warmup, "ms_per_step": max_total_ms / K_steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3 (fp32 accumulate)", "data": "synthetic",
        "config": {"workload": f"{w.name} joint-block projections", "tokens": M, "hidden": w.H * w.D,
                   "shapes": {n: [M, N, K] for n, K, N in fp8_shapes(w)}, "global_batch": w.B * world,
                   "parallelism": f"replicas{world}", "l2": "flushed between steps (256 MiB write)"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak,
                     "traffic": kernel_traffic("fp8_gemm_kernel", ("fp8_linear.cuh", "sage_ptx.cuh"),
                                               f"{w.name} mlp_up"),
                     "kernel": "fp8_gemm_kernel (mlp_up launch)",
                     "peak_source": f"{src} bf16 burst {peaks['bf16_tflops']} x {INT8_PER_BF16} (fp8 dense)"},
        "kernels_us": {"quant_x": quant_us, "gemm": gemm_us},
        "quant_gbs": x_bytes / (sum(quant_us.values()) / 1e6) / 1e9,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "overlap": "copy-in, compute and copy-out on three streams, two buffer sets",
                "serial_value": e2e_serial},
        "gpu_launches": 2 * len(dev) * K_steps,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- ours
SUMMARY_WORKLOADS = ("mid_video", "ragged", "action_dit")


class AttnCase:
    """Device inputs, buffers and the step's calls for one workload."""

    def __init__(self, torch, adt, w, args, stream, qb, kb, vb, nr_host=None):
        as_dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()  # noqa: E731
        self.torch, self.adt, self.w, self.stream = torch, adt, w, stream
        self.q, self.k, self.v = as_dev(qb), as_dev(kb), as_dev(vb)
        self.nr = None
        if nr_host is not None:
            self.nr = dict(q_w=as_dev(nr_host["q_w"]), k_w=as_dev(nr_host["k_w"]), eps=nr_host["eps"],
                           cos=torch.from_numpy(nr_host["cos"]).cuda(), sin=torch.from_numpy(nr_host["sin"]).cuda())
        self.grans = (args.q_gran, args.k_gran)
        self.buf = self.new_buffers()
        self.fused = args.quant == "fused" and self.nr is None

    def new_buffers(self):
        w = self.w
        return self.adt.Buffers(w.B, w.N, w.H, w.D, cu_seqlens=w.cu_seqlens, q_gran=self.grans[0],
                                k_gran=self.grans[1])

    def quant_qk(self, q=None, k=None, buf=None, st=None):
        q, k, buf, st = q if q is not None else self.q, k if k is not None else self.k, buf or self.buf, st or self.stream
        if self.nr is None:
            self.adt.sage_quant_qk(q, k, buf.shape, buf.q_codes, buf.q_scale, buf.k_codes, buf.k_scale, buf.k_mean,
                                   buf.workspace, st)
        else:
            nr = self.nr
            self.adt.sage_quant_qk_normrope(q, k, buf.shape, nr["q_w"], nr["k_w"], nr["cos"], nr["sin"], nr["eps"],
                                            buf.q_codes, buf.q_scale, buf.k_codes, buf.k_scale, buf.k_mean,
                                            buf.workspace, st)

    def quant_v(self, v=None, buf=None, st=None):
        v, buf = v if v is not None else self.v, buf or self.buf
        self.adt.sage_quant_v(v, buf.shape, buf.v_codes_t, buf.v_scale, buf.v_mean, buf.workspace, st or self.stream)

    def quant_qkv(self, q=None, k=None, v=None, buf=None, st=None):
        q, k, v = (x if x is not None else d for x, d in ((q, self.q), (k, self.k), (v, self.v)))
        buf = buf or self.buf
        self.adt.sage_quant_qkv(q, k, v, buf.shape, 0, buf.q_codes, buf.q_scale, buf.k_codes, buf.k_scale,
                                buf.k_mean, buf.v_codes_t, buf.v_scale, buf.v_mean, buf.workspace, st or self.stream)

    def quant_all(self, q=None, k=None, v=None, buf=None, st=None):
        if self.fused:
            self.quant_qkv(q, k, v, buf, st)
        else:
            self.quant_qk(q, k, buf, st)
            self.quant_v(v, buf, st)

    def attn(self, buf=None, st=None):
        buf = buf or self.buf
        self.adt.sage_attn_fwd(buf.q_codes, buf.q_scale, buf.k_codes, buf.k_scale, buf.v_codes_t, buf.v_scale,
                               buf.v_mean, buf.shape, 0.0, buf.out, False, None, st or self.stream)

    def eager_loop(self, steps, flush, fused):
        """`steps` eager steps, each after an L2 flush, with events between the
        launches; returns per-step milliseconds (quant_qk, quant_v or None,
        quant total, attention, whole step)."""
        torch, stream = self.torch, self.stream
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
        for i in range(steps):
            flush.fill_(i & 0xFF)
            e = ev[i]
            e[0].record(stream)
            if fused:
                self.quant_qkv()
            else:
                self.quant_qk()
                e[1].record(stream)
                self.quant_v()
            e[2].record(stream)
            self.attn()
            e[3].record(stream)
        torch.cuda.synchronize()
        self.adt.sage_check()
        return dict(qk=None if fused else [e[0].elapsed_time(e[1]) for e in ev],
                    v=None if fused else [e[1].elapsed_time(e[2]) for e in ev],
                    quant=[e[0].elapsed_time(e[2]) for e in ev],
                    attn=[e[2].elapsed_time(e[3]) for e in ev],
                    step=[e[0].elapsed_time(e[3]) for e in ev])


def attn_roofline(w, attn_ms, peaks, src, k_blocks=True):
    peak = peaks["bf16_tflops"] * INT8_PER_BF16
    achieved = w.attn_ops / (attn_ms / 1e3) / 1e12
    return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "traffic": kernel_traffic(f"sage_attn_kernel<{w.D}, false>", ATTN_SOURCES, w.name) if k_blocks else None,
            "kernel": f"sage_attn_kernel<{w.D}, {'false' if k_blocks else 'true'}>",
            "peak_source": f"{src} bf16 burst {peaks['bf16_tflops']} x {INT8_PER_BF16} (int8/fp8 dense)"}


def workload_summary(torch, adt, name, args, stream, flush, peaks, src, gpu):
    """Eager per-kernel figures of another workload, on one GPU: the fused
    quantization call and attention (the step), then sage_quant_qk and
    sage_quant_v as standalone calls (their own GB/s)."""
    w = synth.WORKLOADS[name]
    qb, kb, vb = synth.generate(w)
    case = AttnCase(torch, adt, w, argparse.Namespace(q_gran="block64", k_gran="block64", quant="fused"),
                    stream, qb, kb, vb)
    del qb, kb, vb
    steps = max(3, min(args.steps, 10))
    for _ in range(3):
        case.quant_qkv(); case.attn(); case.quant_qk(); case.quant_v()
    torch.cuda.synchronize()
    sampler = ClockSampler(gpu)
    fused = case.eager_loop(steps, flush, True)
    sep = case.eager_loop(steps, flush, False)
    clocks = sampler.stop()
    qk_bytes, v_bytes = quant_bytes(w)
    mean = statistics.mean
    attn_ms = mean(fused["attn"] + sep["attn"])
    roof = attn_roofline(w, attn_ms, peaks, src)
    out = {"B": w.B, "N": w.N, "H": w.H, "D": w.D, "steps": steps,
           "step_tops_eager": w.attn_ops * steps / (sum(fused["step"]) / 1e3) / 1e12,
           "attn_us": 1e3 * attn_ms, "attn_tops": roof["achieved"], "attn_frac": roof["frac"],
           "attn_traffic": roof["traffic"],
           "quant_qkv_us": 1e3 * mean(fused["quant"]),
           "quant_qkv_gbs": (qk_bytes + v_bytes) / (mean(fused["quant"]) / 1e3) / 1e9,
           "quant_qk_us": 1e3 * mean(sep["qk"]), "quant_qk_gbs": qk_bytes / (mean(sep["qk"]) / 1e3) / 1e9,
           "quant_v_us": 1e3 * mean(sep["v"]), "quant_v_gbs": v_bytes / (mean(sep["v"]) / 1e3) / 1e9,
           "hbm_frac": {k: v / peaks["hbm_gbs"] for k, v in (
               ("quant_qkv", (qk_bytes + v_bytes) / (mean(fused["quant"]) / 1e3) / 1e9),
               ("quant_qk", qk_bytes / (mean(sep["qk"]) / 1e3) / 1e9),
               ("quant_v", v_bytes / (mean(sep["v"]) / 1e3) / 1e9))},
           "clocks": clocks}
    del case
    torch.cuda.empty_cache()
    return out


def main():
    args = parse()
    rank, world, local = rank_env()
    if args.peaks:
        if rank == 0:
            print(json.dumps({"peaks": measure_peaks(), "shape": "8192^3", "best_of": 20}), flush=True)
        return
    summary = args.workload is None and args.op == "attention" and not args.no_summary
    if args.workload is None:
        args.workload = DEFAULT_WORKLOAD if args.op == "attention" else "action_dit"
    if args.impl == "reference":
        run_reference(args, rank)
        return

    import datetime

    import torch
    import torch.distributed as dist

    import action_diffusion_transformers_b200 as adt

    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    if args.op == "fp8_linear":
        run_fp8_linear(args, rank, world, local)
        return
    w = synth.WORKLOADS[args.workload]
    qb, kb, vb = synth.generate(w)
    nr_host = None
    if args.normrope:
        qb, kb = synth.projection_outputs(w)
        nr_host = synth.normrope_inputs(w)
    stream = torch.cuda.current_stream()
    case = AttnCase(torch, adt, w, args, stream, qb, kb, vb, nr_host)
    q, k, v, buf, nr, fused = case.q, case.k, case.v, case.buf, case.nr, case.fused
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(max(3, args.warmup)):
        case.quant_all(); case.attn()
    adt.sage_check()
    torch.cuda.synchronize()
    barrier()

    K = args.steps
    gpu = gpu_id_for(local)
    sampler = ClockSampler(gpu)
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    eager = case.eager_loop(K, flush, fused)
    barrier()
    eager_out = buf.out.clone()

    # The same launches captured once into a CUDA graph and replayed: the
    # headline value (the per-kernel times and the roofline come from the
    # eager loop above, whose events sit between the launches).
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        case.quant_all(st=side)
        case.attn(st=side)
    torch.cuda.synchronize()
    graph.replay()
    torch.cuda.synchronize()
    barrier()
    gev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    for i in range(K):
        flush.fill_(i & 0xFF)
        gev[i][0].record(stream)
        graph.replay()
        gev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    adt.sage_check()
    if not torch.equal(buf.out, eager_out):
        raise RuntimeError("the graph replay's output differs from the eager step's")
    del graph, eager_out

    ops = w.attn_ops
    eager_value = job_tops(world, ops, K, max_over_ranks(sum(eager["step"]), world, "cuda"))
    max_total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in gev), world, "cuda")
    value = job_tops(world, ops, K, max_total_ms)

    # --------------------------------------------------------------- e2e (host buffers)
    # Every step copies its Q, K, V in from pinned host memory and its output
    # back.  Serial: copy in, compute, copy out on one stream.  Pipelined (the
    # reported figure): two device buffer sets, copies in on one stream, the
    # calls on another, copies out on a third, so step i+1's inputs cross PCIe
    # while step i computes; events order each slot's reuse.
    pin = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()  # noqa: E731
    hq, hk, hv = pin(qb), pin(kb), pin(vb)
    h2d = 3 * qb.nbytes
    del qb, kb, vb
    hout = [torch.empty(buf.out.shape, dtype=buf.out.dtype).pin_memory() for _ in range(2)]
    e2e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    for _ in range(2):
        q.copy_(hq, non_blocking=True); k.copy_(hk, non_blocking=True); v.copy_(hv, non_blocking=True)
        case.quant_all(); case.attn()
        hout[0].copy_(buf.out, non_blocking=True)
    torch.cuda.synchronize()
    barrier()
    for i in range(K):
        flush.fill_(i & 0xFF)
        e2e_ev[i][0].record(stream)
        q.copy_(hq, non_blocking=True); k.copy_(hk, non_blocking=True); v.copy_(hv, non_blocking=True)
        case.quant_all(); case.attn()
        hout[0].copy_(buf.out, non_blocking=True)
        e2e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    adt.sage_check()
    e2e_serial = job_tops(world, ops, K, max_over_ranks(sum(a.elapsed_time(b) for a, b in e2e_ev), world, "cuda"))

    buf2 = case.new_buffers()
    slots = [(q, k, v, buf), (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), buf2)]

    def copy_in(j):
        for d, h in zip(slots[j][:3], (hq, hk, hv)):
            d.copy_(h, non_blocking=True)

    def compute(j):
        case.quant_all(*slots[j])
        case.attn(slots[j][3])

    def copy_out(j):
        hout[j].copy_(slots[j][3].out, non_blocking=True)

    pipelined_e2e(torch, 3, stream, copy_in, compute, copy_out)
    barrier()
    e2e_ms = pipelined_e2e(torch, K, stream, copy_in, compute, copy_out)
    barrier()
    adt.sage_check()
    e2e_value = job_tops(world, ops, K, max_over_ranks(e2e_ms, world, "cuda"))
    out_ok = torch.equal(hout[(K - 1) & 1], buf2.out.cpu() if (K - 1) & 1 else buf.out.cpu())
    if not out_ok:
        raise RuntimeError("pipelined e2e: the copied-out output differs from the device result")
    d2h = buf.out.numel() * buf.out.element_size()
    del slots, buf2, hout

    # --------------------------------------------------------------- roofline, baseline
    peaks, src = load_peaks()
    k_blocks = args.k_gran == "block64"
    attn_mean_ms = statistics.mean(eager["attn"])
    roofline = attn_roofline(w, attn_mean_ms, peaks, src, k_blocks)
    qk_bytes, v_bytes = quant_bytes(w, args.q_gran, args.k_gran)
    if nr is not None:
        qk_bytes += w.N * w.D // 2 * 8 + 2 * w.D * 2          # cos / sin tables once, the two weights
    mean = statistics.mean
    if fused:
        quant_us = {"quant_qkv": 1e3 * mean(eager["quant"]), "attn": 1e3 * attn_mean_ms}
        quant_gbs = {"quant_qkv": (qk_bytes + v_bytes) / (mean(eager["quant"]) / 1e3) / 1e9,
                     "peak_hbm_gbs": peaks["hbm_gbs"]}
    else:
        quant_us = {"quant_qk": 1e3 * mean(eager["qk"]), "quant_v": 1e3 * mean(eager["v"]),
                    "attn": 1e3 * attn_mean_ms}
        quant_gbs = {"quant_qk": qk_bytes / (mean(eager["qk"]) / 1e3) / 1e9,
                     "quant_v": v_bytes / (mean(eager["v"]) / 1e3) / 1e9, "peak_hbm_gbs": peaks["hbm_gbs"]}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # about 10-30 s of CPU work on the host: 4 heads, 2^26 (query row, key) pairs
        heads = min(4, w.H)
        rows = max(1, min(w.N, (1 << 26) // (heads * w.N)))
        hb = lambda t: t.view(torch.int16).numpy().view(np.uint16)  # noqa: E731
        o_ops, o_dt = oracle_sample(w, hb(hq), hb(hk), hb(hv), rows, heads, args.q_gran, args.k_gran, nr_host)
        cpu = {"value": o_ops / o_dt / 1e12, "unit": "TOPS", "cores": blas_threads(), "kind": "oracle",
               "cores_note": "BLAS threads of the score products; the oracle's other steps run on one core",
               "sample": f"{heads} heads of batch 0: full K/V quantization of those heads + attention for "
                         f"{rows} query rows each ({o_dt:.1f} s)"}
    del case, q, k, v, buf, hq, hk, hv
    torch.cuda.empty_cache()
    others = None
    if summary and rank == 0 and world == 1:
        others = {name: workload_summary(torch, adt, name, args, stream, flush, peaks, src, gpu)
                  for name in SUMMARY_WORKLOADS if name != w.name}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": "quantized-attention TOPS", "value": value, "unit": "TOPS", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": max_total_ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "i8/e4m3 (fp32 softmax)", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "N": w.N, "H": w.H, "D": w.D, "global_batch": w.B * world,
                   "seq_len": w.N, "parallelism": f"replicas{world}", "l2": "flushed between steps (256 MiB write)",
                   "q_gran": args.q_gran, "k_gran": args.k_gran,
                   "qk_prologue": "rmsnorm+rope" if nr is not None else None},
        "roofline": roofline,
        "kernels_us": quant_us,
        "kernels_us_note": "per-kernel means from the eager loop (events between launches); value and "
                           "ms_per_step from graph replays, which trim the gaps between launches",
        "quant_gbs": quant_gbs,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "TOPS", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "overlap": "copy-in, compute and copy-out on three streams, two buffer sets",
                "serial_value": e2e_serial},
        "gpu_launches": (5 if fused else 7) * K,
        "launch": "the step's launches as one CUDA graph, replayed (eager launches: eager_value)",
        "eager_value": eager_value,
        "clocks": clocks,
    }
    if others is not None:
        line["workloads"] = others
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
