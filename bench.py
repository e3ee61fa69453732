#!/usr/bin/env python
"""Benchmark of the PaTH attention hot path on B200.

One step = the whole training hot path on one batch: path_attn_fwd (UT prep,
transport chain, attention forward) then path_attn_bwd reusing the
forward's workspace (attention backward, UT adjoint, gate gradient) at B=8
H=24 L=4096 d=64 bf16, inputs resident in HBM. The decode step (B=32 H=32 d=128, cache 16384 -> 16448,
64 steps) is timed after it and reported under "decode" (with the forget gate's per-key
bias under "decode.gated"), and a prefill of the same sequences (forward plus the decode
cache it leaves) under "prefill", and fwd+bwd at head dim 128 (B=8 H=12, the same model
width) under "d128". The other timed workloads: the forward latency at B=2 H=4 L=1024
("fwd_latency"), PaTH-FoX fwd+bwd at B=1 H=24 L=16384 ("fox"), and the headline step with
fp32 outputs and gradients ("f32out"), and the w / beta prologue at the headline layer
("wbeta").

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun every rank runs the same workload on its own GPU (weak
scaling: heads are independent, no collective on the data path); the step
time is the max over ranks.

Metric: algorithmic TFLOP/s = 11 * L^2 * d * B * H FLOP per step (forward
3 L^2 d: QK^T, PV and the d x d block transport at 64-position blocks;
backward 8 L^2 d) divided by the device time of a step. Also reported:
tokens/s = B * L / step time, and the FlashAttention-equivalent 7 L^2 d count.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic_inputs as si  # noqa: E402

WORKLOAD = "fwdbwd_bf16_l4096"
DECODE = "decode_bf16_c16k"
METRIC = "PaTH fwd+bwd TFLOP/s at L=4096 d=64 (algorithmic 11*L^2*d per head)"
UNIT = "TFLOP/s"


def algorithmic_flops(B, H, L, d):
    return 11.0 * L * L * d * B * H


def fa_equiv_flops(B, H, L, d):
    return 7.0 * L * L * d * B * H


# fp32 FMA peak from unit counts and clocks: 148 SMs x 128 fp32 lanes x 2 FLOP x 1965 MHz
ALU_F32_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def stage_model(name, B, H, L, d, BT=128):
    """(algorithmic FLOP of one launch, bound) of a stage; causal, leading order.

    Tensor-core stages count the products of the blockwise algorithm; the UT
    stages at head dims 64 and 128 count the 64x64x64 products their tcgen05
    kernels issue (fp16 operands), at other head dims the fp32 arithmetic of the
    per-block recurrences and closed-form adjoint ("alu")."""
    nh, nblk, HB = B * H, -(-L // BT), 64
    # 64x64x64 products per 128-block of the tcgen05 UT kernels: the prep (both
    # halves' closed-form UT, boundary terms, the block's composition; at d = 128
    # every d-wide product is two) and the adjoint (composition adjoint and both
    # halves' UT adjoints, the halves' transform read from the forward's save)
    ut_prep_products = {64: 36, 128: 74}
    ut_adj_products = {64: 52, 128: 124}
    per = {
        "attn_fwd": (2.0 * L * L * d, "tensor"),                      # QK^T + PV
        # S, dP, dV, dK, dQ recomputed / formed once per causal pair, plus the
        # key-side chain adjoint (Abar P_I and Abar^T Khat per block pair)
        "attn_bwd": (5.0 * L * L * d + 2.0 * L * L * d * d / BT, "tensor"),
        "attn_bwd_q": (3.0 * L * L * d, "tensor"),                    # S, dP, dQ (SIMT path)
        "attn_bwd_k": (4.0 * L * L * d + 2.0 * L * L * d * d / BT, "tensor"),
        "chain": (1.0 * L * L * d * d / BT, "tensor"),               # key-side block transport
        # other head dims: rank-one recurrences (keys with in-block logits, queries,
        # block product)
        "ut_prep": ((nblk * ut_prep_products[d] * 2.0 * HB ** 3, "tensor") if d in ut_prep_products
                    else (nblk * (BT * BT / 2 * 10.0 * d + BT * 4.0 * d * d), "alu")),
        "ut_adj": ((nblk * ut_adj_products[d] * 2.0 * HB ** 3, "tensor") if d in ut_adj_products
                   else (0.0, None)),
        "ut_prep_bwd": (nblk * (8 * 2.0 * HB * HB * d + 4 * HB * HB * 4.0 * d
                                + 2 * 24 * 2.0 * HB * HB * d), "alu"),
    }
    f, bound = per.get(name, (0.0, None))
    return f * nh, bound


# DRAM bytes (read + write) per launch of a kernel, from an ncu capture of the
# B=1 H=24 L=4096 d=64 case (profiles/ summaries), scaled to the benchmark's
# B=8 by the heads processed; None where the kernel changed since the capture.
DRAM_BYTES_B1H24 = {
    "attn_bwd": 325.66e6 + 94.57e6,
    "attn_fwd": 274.1e6 + 9.8e6,
    "ut_prep": 38.2e6 + 85.7e6,
    "ut_adj": 214.4e6 + 24.1e6,
}
DRAM_BYTES_PREFILL_CACHE_B4H24 = 157.2e6
# The same for the forget-gate workload's kernels, from a capture of B=1 H=6 L=16384
# d=64, scaled by the heads processed.
DRAM_BYTES_FOX_B1H6 = {
    "attn_bwd": 933.63e6 + 103.36e6,
}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained", j["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock/throttle samples of one GPU while the timed region runs."""

    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
              "utilization.gpu")

    def __init__(self, device):
        self.uuid = None
        try:
            self.uuid = str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            pass
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-f", self.path], stdout=subprocess.DEVNULL,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 11:
                    continue
                if self.uuid and self.uuid.replace("GPU-", "") not in parts[1]:
                    continue
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        busy = [r for r in rows if (num(r[10]) or 0) > 50] or rows
        sm = [num(r[2]) for r in busy if num(r[2]) is not None]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in busy:
            for n, v in zip(names, r[6:10]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": num(rows[0][3]), "reasons": sorted(reasons),
                "samples": len(rows), "samples_under_load": len(busy)}


def read_profile():
    """Stage name -> (total ms, launches) timed since the last read."""
    import softmax_attention_block_b200 as P
    return P.path_profile_read(64)


# ---------------------------------------------------------------- reference arm
def cpu_baseline_sample(w, heads=(0,)):
    """Time the fp64 oracle (as it stands) on a bounded sample: the listed heads
    of the workload, forward + backward. Returns (TFLOP/s, seconds, cores)."""
    import oracle

    x = si.workload_inputs(w.name, heads=list(heads))
    orc = oracle.default()
    t0 = time.perf_counter()
    orc.fwd(x["q"], x["k"], x["v"], x["w"], x["beta"], x["log_f"])
    orc.bwd(x["q"], x["k"], x["v"], x["w"], x["beta"], x["dout"], x["log_f"])
    dt = time.perf_counter() - t0
    flops = algorithmic_flops(1, len(heads), w.L, w.d)
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return flops / dt / 1e12, dt, cores


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = si.WORKLOADS[WORKLOAD]
    for _ in range(args.warmup):
        cpu_baseline_sample(w)
    vals, secs = [], []
    for _ in range(args.steps):
        v, s, cores = cpu_baseline_sample(w)
        vals.append(v)
        secs.append(s)
    value = statistics.mean(vals)
    sample = (f"1 of {w.B * w.H} heads (b=0,h=0) of {WORKLOAD}, fwd+bwd, fp64 oracle; "
              f"TFLOP/s on that head's 11*L^2*d FLOP")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * statistics.mean(secs), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": w.B, "H": w.H, "L": w.L, "d": w.d,
                       "sample": "1 head per step"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- our arm
def make_collectives(world, device):
    """The benchmark's only collectives, host-side timing plumbing (no data path):
    a barrier around the timed region and the max over ranks of a device time,
    a float64 all-reduce on `device` (the GPU under NCCL, the CPU under gloo)."""
    import torch.distributed as dist

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v):
        if world == 1:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    return barrier, max_over_ranks


def whole_job_rate(world, units_per_rank, ms_per_step_max):
    """Weak scaling: every rank runs the full workload, so the job processes
    world x units per step in the slowest rank's time."""
    return world * units_per_rank / (ms_per_step_max * 1e-3)


def run_ours(args):
    import torch.distributed as dist
    import softmax_attention_block_b200 as P

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    P.lib()
    peaks = load_peaks()

    w = si.WORKLOADS[WORKLOAD]
    xc = si.workload_inputs(WORKLOAD, seed=0)
    x = {k: (v.to(dev) if v is not None else None) for k, v in xc.items()}
    out = torch.empty_like(x["q"])
    lse = torch.empty((w.B, w.H, w.L), dtype=torch.float32, device=dev)
    grads = {n: torch.empty_like(x["q"]) for n in ("dq", "dk", "dv", "dw")}
    grads["dbeta"] = torch.empty_like(x["beta"])
    # one backward-sized workspace: the forward leaves its block transforms and
    # transported keys there and the backward reuses them (training usage)
    ws_bytes = P.path_attn_workspace_bytes(w.B, w.H, w.L, w.d, w.dtype, True)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

    def step(inp):
        P.path_attn_fwd(inp["q"], inp["k"], inp["v"], inp["w"], inp["beta"], inp["log_f"],
                        out=out, lse=lse, workspace=ws)
        P.path_attn_bwd(inp["q"], inp["k"], inp["v"], inp["w"], inp["beta"], out, lse,
                        inp["dout"], inp["log_f"], grads=grads, workspace=ws,
                        reuse_fwd_workspace=True)

    barrier, max_over_ranks = make_collectives(world, dev)

    for _ in range(args.warmup):
        step(x)
    torch.cuda.synchronize()
    barrier()
    clocks = ClockSampler(dev)
    clocks.start()
    launches0 = P.lib().path_kernel_launch_count()
    P.lib().path_profile_enable(1)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier()
    e0.record(stream)
    for _ in range(args.steps):
        step(x)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    P.lib().path_profile_enable(0)
    launches = P.lib().path_kernel_launch_count() - launches0
    clk = clocks.stop()
    ms_total = max_over_ranks(e0.elapsed_time(e1))
    stages = read_profile()
    ms_step = ms_total / args.steps
    flops = algorithmic_flops(w.B, w.H, w.L, w.d)
    value = whole_job_rate(world, flops, ms_step) / 1e12
    tokens = whole_job_rate(world, w.B * w.L, ms_step)

    # dominant stage -> roofline against the measured bf16 dense peak
    stage_rows = {n: {"ms_per_launch": t / c, "launches": c, "share": 0.0}
                  for n, (t, c) in stages.items()}
    tot = sum(t for t, _ in stages.values()) or 1.0
    for n, (t, _) in stages.items():
        stage_rows[n]["share"] = t / tot
    dom = max(stages, key=lambda n: stages[n][0]) if stages else None
    roofline = None
    if dom:
        per_launch_ms = stages[dom][0] / stages[dom][1]
        f, bound = stage_model(dom, w.B, w.H, w.L, w.d)
        ach = f / (per_launch_ms * 1e-3) / 1e12 if f else None
        if bound == "alu":
            peak, src = ALU_F32_TFLOPS, "fp32 FMA from unit counts and max clock"
        else:
            peak = peaks["bf16_tflops_sustained"]
            src = f"{peaks['source']} bf16 dense (sustained)"
        traffic = DRAM_BYTES_B1H24.get(dom)
        if traffic is not None:
            traffic *= (w.B * w.H) / 24.0
        roofline = {"kernel": dom, "bound": bound or "tensor", "achieved": ach, "peak": peak,
                    "unit": "TFLOP/s", "frac": (ach / peak) if ach else None, "traffic": traffic,
                    "traffic_unit": "bytes per launch", "peak_source": src}

    # end to end through the API with host buffers (pinned), copies in the timed
    # region: the batch goes through in per-sequence chunks; host->device copies
    # run ahead on one stream, fwd+bwd of each chunk follows on the launching
    # stream, device->host copies trail on a third (the copy engines are full
    # duplex), with events guarding each chunk's device buffers across steps
    e2e = None
    if not args.no_e2e:
        host = {k: (v.pin_memory() if v is not None else None) for k, v in xc.items()}
        hout = {n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                for n, t in list(grads.items()) + [("out", out), ("lse", lse)]}
        h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
        d2h = sum(v.numel() * v.element_size() for v in hout.values())
        ws1 = torch.empty(P.path_attn_workspace_bytes(1, w.H, w.L, w.d, w.dtype, True),
                          dtype=torch.uint8, device=dev)
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        computed = [None] * w.B   # chunk's fwd+bwd done: its inputs may be overwritten
        fetched = [None] * w.B    # chunk's results copied out: its outputs may be overwritten
        dev_out = list(grads.items()) + [("out", out), ("lse", lse)]

        def e2e_step():
            start = torch.cuda.Event()
            start.record(stream)
            s_in.wait_event(start)
            loaded = []
            with torch.cuda.stream(s_in):
                for b in range(w.B):
                    if computed[b] is not None:
                        s_in.wait_event(computed[b])
                    for k, v in host.items():
                        if v is not None:
                            x[k][b:b + 1].copy_(v[b:b + 1], non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(s_in)
                    loaded.append(ev)
            for b in range(w.B):
                stream.wait_event(loaded[b])
                if fetched[b] is not None:
                    stream.wait_event(fetched[b])
                xb = {k: (v[b:b + 1] if v is not None else None) for k, v in x.items()}
                P.path_attn_fwd(xb["q"], xb["k"], xb["v"], xb["w"], xb["beta"], xb["log_f"],
                                out=out[b:b + 1], lse=lse[b:b + 1], workspace=ws1)
                P.path_attn_bwd(xb["q"], xb["k"], xb["v"], xb["w"], xb["beta"], out[b:b + 1],
                                lse[b:b + 1], xb["dout"], xb["log_f"],
                                grads={n: t[b:b + 1] for n, t in grads.items()},
                                workspace=ws1, reuse_fwd_workspace=True)
                ev = torch.cuda.Event()
                ev.record(stream)
                computed[b] = ev
                s_out.wait_event(ev)
                with torch.cuda.stream(s_out):
                    for n, t in dev_out:
                        hout[n][b:b + 1].copy_(t[b:b + 1], non_blocking=True)
                    evo = torch.cuda.Event()
                    evo.record(s_out)
                    fetched[b] = evo
            stream.wait_event(fetched[w.B - 1])

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ms_e2e = max_over_ranks(e0.elapsed_time(e1)) / args.steps
        e2e = {"value": whole_job_rate(world, flops, ms_e2e) / 1e12, "unit": UNIT,
               "ms_per_step": ms_e2e, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "pipeline": f"{w.B} per-sequence chunks; copies in, compute, copies out on 3 streams"}
        del host, hout, ws1

    prefill = None if args.no_prefill else bench_prefill(P, x, w, ws, peaks, world,
                                                           max_over_ranks, barrier, args.steps)
    del out, lse, grads, ws
    torch.cuda.empty_cache()
    f32out = None if args.no_f32out else bench_f32out(P, x, w, world, max_over_ranks, barrier,
                                                      args.steps)
    del x
    torch.cuda.empty_cache()
    fwd_latency = None if args.no_fwd_latency else bench_fwd_latency(P, dev, peaks, world,
                                                                     max_over_ranks, barrier)
    wbeta = None if args.no_wbeta else bench_wbeta(P, dev, peaks, world, max_over_ranks, barrier,
                                                   args.steps)
    fox = None if args.no_fox else bench_fox(
        P, dev, peaks, world, max_over_ranks, barrier, 3,
        cpu_sample=(rank == 0 and world == 1 and not args.no_cpu_baseline))
    decode = None if args.no_decode else bench_decode(P, dev, peaks, world, max_over_ranks,
                                                       barrier)
    d128 = None if args.no_d128 else bench_d128(P, dev, peaks, world, max_over_ranks, barrier,
                                                 2)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, s, cores = cpu_baseline_sample(w)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"1 of {w.B * w.H} heads of {WORKLOAD} fwd+bwd in fp64 ({s:.1f} s)"}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": w.B, "H": w.H, "L": w.L, "d": w.d,
                       "log_f": False, "l2": "inputs larger than L2 (each [B,H,L,d] bf16 "
                       "tensor is 100.7 MB; 126 MB L2)",
                       "parallelism": f"{world} rank(s), full workload per rank"},
            "tokens_per_s": tokens,
            "tflops_fa_equiv": whole_job_rate(world, fa_equiv_flops(w.B, w.H, w.L, w.d), ms_step) / 1e12,
            "pct_bf16_peak": value / world / peaks["bf16_tflops_sustained"],
            "stages": stage_rows, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches, "clocks": clk, "decode": decode, "prefill": prefill,
            "d128": d128, "f32out": f32out, "fwd_latency": fwd_latency, "fox": fox,
            "wbeta": wbeta}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def bench_prefill(P, x, w, ws, peaks, world, max_over_ranks, barrier, steps):
    """Prefill of the headline sequences (forward + the decode cache it leaves), timed
    as a whole and, for the cache kernel, per launch against the HBM copy peak."""
    cap = w.L + 64
    kc = torch.empty((w.B, w.H, cap, w.d), dtype=w.dtype, device=x["q"].device)
    vc = torch.empty_like(kc)
    out = torch.empty_like(x["q"])
    lse = torch.empty((w.B, w.H, w.L), dtype=torch.float32, device=x["q"].device)

    def call():
        P.path_attn_prefill(x["q"], x["k"], x["v"], x["w"], x["beta"], cap, x["log_f"], out=out,
                            lse=lse, k_cache=kc, v_cache=vc, workspace=ws)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    barrier()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    P.lib().path_profile_enable(1)
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    P.lib().path_profile_enable(0)
    stages = read_profile()
    ms = max_over_ranks(e0.elapsed_time(e1)) / steps
    nh = w.B * w.H
    # cache kernel, per launch: read the transported key tiles (fp16), P_last (fp16) and
    # v; write the key and value caches (bf16)
    bytes_launch = nh * (w.L * w.d * 2 * 4 + w.d * w.d * 2)
    t, c = stages.get("prefill_cache", (0.0, 1))
    per_launch = t / max(c, 1)
    ach = bytes_launch / (per_launch * 1e-3) / 1e9 if per_launch else None
    # DRAM bytes of one launch from the ncu capture at B=4 (profiles/), scaled by heads
    traffic = DRAM_BYTES_PREFILL_CACHE_B4H24 * (w.B * w.H) / 96.0
    del kc, vc, out, lse
    return {"workload": f"prefill {WORKLOAD}, cache capacity {cap}",
            "value": whole_job_rate(world, w.B * w.L, ms), "unit": "tokens/s",
            "ms_per_call": ms, "cache_kernel_ms": per_launch,
            "roofline": {"kernel": "prefill_cache", "bound": "hbm", "achieved": ach,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / peaks["hbm_gbs"] if ach else None, "traffic": traffic,
                         "traffic_unit": "bytes per launch", "algorithmic_bytes": bytes_launch,
                         "peak_source": f"{peaks['source']} HBM copy"}}


L2_FLUSH_BYTES = 256 << 20  # twice the 126 MB L2: written between timed calls of small workloads


def timed_calls(call, n, flush, stream):
    """Device time of n calls, each preceded by an untimed write of `flush` (evicts L2):
    per-call CUDA events on the launching stream; returns ms per call."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    for a, b in evs:
        flush.zero_()
        a.record(stream)
        call()
        b.record(stream)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs) / n


def stage_roofline(stages, B, H, L, d, peaks, traffic_per_head=None):
    """Dominant stage of a timed region -> roofline object against the sustained bf16 peak.
    traffic_per_head: DRAM bytes per launch per head of the kernels captured, by stage."""
    if not stages:
        return None
    dom = max(stages, key=lambda n: stages[n][0])
    per_launch_ms = stages[dom][0] / stages[dom][1]
    f, bound = stage_model(dom, B, H, L, d)
    ach = f / (per_launch_ms * 1e-3) / 1e12 if f else None
    peak = peaks["bf16_tflops_sustained"]
    t = (traffic_per_head or {}).get(dom)
    return {"kernel": dom, "bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
            "frac": (ach / peak) if ach else None,
            "traffic": t * B * H if t is not None else None, "traffic_unit": "bytes per launch",
            "peak_source": f"{peaks['source']} bf16 dense (sustained)"}


FWD_LATENCY = "fwd_bf16_l1024"
FOX = "fox_fwdbwd_l16384"


def bench_fwd_latency(P, dev, peaks, world, max_over_ranks, barrier, calls=20):
    """Forward latency of the B=2 H=4 L=1024 bf16 workload (out + lse): one call is
    launch-bound, so each timed call follows an L2 flush and is timed on its own."""
    w = si.WORKLOADS[FWD_LATENCY]
    xc = si.workload_inputs(FWD_LATENCY, seed=0)
    x = {k: (v.to(dev) if v is not None else None) for k, v in xc.items()}
    out = torch.empty_like(x["q"])
    lse = torch.empty((w.B, w.H, w.L), dtype=torch.float32, device=dev)
    ws = torch.empty(P.path_attn_workspace_bytes(w.B, w.H, w.L, w.d, w.dtype, False),
                     dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def call():
        P.path_attn_fwd(x["q"], x["k"], x["v"], x["w"], x["beta"], None, out=out, lse=lse,
                        workspace=ws)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    barrier()
    stream = torch.cuda.current_stream()
    P.lib().path_profile_enable(1)
    ms = max_over_ranks(timed_calls(call, calls, flush, stream))
    P.lib().path_profile_enable(0)
    stages = read_profile()
    fl = 3.0 * w.L * w.L * w.d * w.B * w.H
    del x, out, lse, ws, flush
    return {"workload": f"{FWD_LATENCY}: bf16 forward B={w.B} H={w.H} L={w.L} d={w.d}, out + lse",
            "ms_per_call": ms, "value": whole_job_rate(world, fl, ms) / 1e12, "unit": UNIT,
            "flop_convention": "3 L^2 d per head (QK^T, PV, block transport)",
            "l2": "flushed (256 MB written) before every timed call",
            "stages_ms": {n: t / c for n, (t, c) in stages.items()}}


def bench_fox(P, dev, peaks, world, max_over_ranks, barrier, steps, cpu_sample):
    """PaTH-FoX fwd+bwd at B=1 H=24 L=16384 (the long-context workload): TFLOP/s by
    11 L^2 d per head, tokens/s, the dominant stage's roofline, and the oracle on a
    bounded sample (the first 4096 positions of one head)."""
    w = si.WORKLOADS[FOX]
    xc = si.workload_inputs(FOX, seed=0)
    x = {k: (v.to(dev) if v is not None else None) for k, v in xc.items()}
    out = torch.empty_like(x["q"])
    lse = torch.empty((w.B, w.H, w.L), dtype=torch.float32, device=dev)
    grads = {n: torch.empty_like(x["q"]) for n in ("dq", "dk", "dv", "dw")}
    grads["dbeta"] = torch.empty_like(x["beta"])
    grads["dlog_f"] = torch.empty_like(x["log_f"])
    ws = torch.empty(P.path_attn_workspace_bytes(w.B, w.H, w.L, w.d, w.dtype, True),
                     dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        P.path_attn_fwd(x["q"], x["k"], x["v"], x["w"], x["beta"], x["log_f"], out=out, lse=lse,
                        workspace=ws)
        P.path_attn_bwd(x["q"], x["k"], x["v"], x["w"], x["beta"], out, lse, x["dout"],
                        x["log_f"], grads=grads, workspace=ws, reuse_fwd_workspace=True)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    barrier()
    stream = torch.cuda.current_stream()
    P.lib().path_profile_enable(1)
    ms = max_over_ranks(timed_calls(step, steps, flush, stream))
    P.lib().path_profile_enable(0)
    stages = read_profile()
    fl = algorithmic_flops(w.B, w.H, w.L, w.d)
    del x, out, lse, grads, ws, flush
    torch.cuda.empty_cache()
    res = {"workload": f"{FOX}: bf16 PaTH-FoX fwd+bwd B={w.B} H={w.H} L={w.L} d={w.d}",
           "ms_per_step": ms, "value": whole_job_rate(world, fl, ms) / 1e12, "unit": UNIT,
           "tokens_per_s": whole_job_rate(world, w.B * w.L, ms),
           "pct_bf16_peak": fl / (ms * 1e-3) / 1e12 / peaks["bf16_tflops_sustained"],
           "l2": "flushed (256 MB written) before every timed step",
           "stages": {n: {"ms_per_launch": t / c, "launches": c} for n, (t, c) in stages.items()},
           "roofline": stage_roofline(stages, w.B, w.H, w.L, w.d, peaks,
                                      {k: v / 6.0 for k, v in DRAM_BYTES_FOX_B1H6.items()})}
    if cpu_sample:
        import oracle

        xs = si.workload_inputs(FOX, heads=[0])
        Ls = 4096
        xs = {k: (v[:, :, :Ls].contiguous() if v is not None else None) for k, v in xs.items()}
        t0 = time.perf_counter()
        orc = oracle.default()
        orc.fwd(xs["q"], xs["k"], xs["v"], xs["w"], xs["beta"], xs["log_f"])
        orc.bwd(xs["q"], xs["k"], xs["v"], xs["w"], xs["beta"], xs["dout"], xs["log_f"])
        dt = time.perf_counter() - t0
        res["cpu_baseline"] = {
            "value": algorithmic_flops(1, 1, Ls, w.d) / dt / 1e12, "unit": UNIT,
            "cores": int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1)), "kind": "oracle",
            "sample": f"positions 0..{Ls - 1} of head 0 of {FOX} (a causal prefix), fwd+bwd in "
                      f"fp64 ({dt:.1f} s); TFLOP/s on that prefix's 11*L^2*d FLOP"}
    return res


def bench_f32out(P, x, w, world, max_over_ranks, barrier, steps):
    """The headline step with fp32 out, dout and gradients (PATH_BF16_F32OUT): the mode
    whose outputs meet max-abs 2e-2 without the bf16 storage allowance."""
    dev = x["q"].device
    out = torch.empty(x["q"].shape, dtype=torch.float32, device=dev)
    lse = torch.empty((w.B, w.H, w.L), dtype=torch.float32, device=dev)
    dout = x["dout"].float()
    grads = {n: torch.empty(x["q"].shape, dtype=torch.float32, device=dev)
             for n in ("dq", "dk", "dv", "dw")}
    grads["dbeta"] = torch.empty_like(x["beta"])
    ws = torch.empty(P.path_attn_workspace_bytes(w.B, w.H, w.L, w.d, w.dtype, True,
                                                 torch.float32), dtype=torch.uint8, device=dev)

    def step():
        P.path_attn_fwd(x["q"], x["k"], x["v"], x["w"], x["beta"], None, out=out, lse=lse,
                        workspace=ws)
        P.path_attn_bwd(x["q"], x["k"], x["v"], x["w"], x["beta"], out, lse, dout, None,
                        grads=grads, workspace=ws, reuse_fwd_workspace=True)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    barrier()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1)) / steps
    fl = algorithmic_flops(w.B, w.H, w.L, w.d)
    del out, lse, dout, grads, ws
    torch.cuda.empty_cache()
    return {"workload": f"{WORKLOAD} with fp32 out, dout and gradients (PATH_BF16_F32OUT)",
            "ms_per_step": ms, "value": whole_job_rate(world, fl, ms) / 1e12, "unit": UNIT}


# the w / beta prologue at the headline layer: B, L, D (= H d), rank, H, d, beta clip
WBETA = (8, 4096, 1536, 64, 24, 64, 1.99)


def bench_wbeta(P, dev, peaks, world, max_over_ranks, barrier, steps):
    """The w / beta prologue (low-rank layer, short convolution, L2 norm, beta) forward and
    backward at the headline layer width, bf16 inputs and outputs. Algorithmic bytes: what
    the step must move at least (x read by both passes, w and beta written, dw and dbeta
    read, dx written), against the HBM copy peak."""
    B, L, D, r, H, d, bmax = WBETA
    g = torch.Generator().manual_seed(0)
    rn = lambda *s: torch.randn(*s, generator=g)
    x = rn(B, L, D).to(torch.bfloat16).to(dev)
    A = (rn(D, r) / D ** 0.5).to(torch.bfloat16).to(dev)
    Bw = (rn(r, H * d) / r ** 0.5).to(torch.bfloat16).to(dev)
    f = (rn(H * d, 3) * 0.5 + torch.tensor([1.0, 0.0, 0.0])).to(dev)
    U = (rn(D, H) * (2.0 / D ** 0.5)).to(torch.bfloat16).to(dev)
    b = rn(H).to(dev)
    dw = rn(B, H, L, d).to(torch.bfloat16).to(dev)
    dbeta = rn(B, H, L).to(dev)
    ws = torch.empty(P.path_wbeta_workspace_bytes(B, L, D, r, H, d, torch.bfloat16, True),
                     dtype=torch.uint8, device=dev)
    w = torch.empty((B, H, L, d), dtype=torch.bfloat16, device=dev)
    beta = torch.empty((B, H, L), dtype=torch.float32, device=dev)
    grads = dict(dx=torch.empty_like(x), dA=torch.empty((D, r), device=dev),
                 dBw=torch.empty((r, H * d), device=dev), df=torch.empty((H * d, 3), device=dev),
                 dU=torch.empty((D, H), device=dev), db=torch.empty((H,), device=dev))

    def step():
        P.path_wbeta_fwd(x, A, Bw, f, U, b, H, bmax, w=w, beta=beta, workspace=ws)
        P.path_wbeta_bwd(x, A, Bw, f, U, b, H, dw, dbeta, bmax, grads=grads, workspace=ws,
                         reuse_fwd_workspace=True)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    barrier()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    P.lib().path_profile_enable(1)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    P.lib().path_profile_enable(0)
    stages = read_profile()
    ms = max_over_ranks(e0.elapsed_time(e1)) / steps
    nbytes = 2 * x.numel() * 2 + w.numel() * 2 * 2 + beta.numel() * 4 * 2 + x.numel() * 2
    del x, A, Bw, f, U, b, dw, dbeta, ws, w, beta, grads
    torch.cuda.empty_cache()
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": f"w/beta prologue fwd+bwd bf16 B={B} L={L} D={D} rank={r} H={H} d={d}",
            "ms_per_step": ms, "value": whole_job_rate(world, B * L, ms), "unit": "tokens/s",
            "algorithmic_bytes": nbytes,
            "roofline": {"kernel": "whole step", "bound": "hbm", "achieved": gbs,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                         "traffic": None, "peak_source": f"{peaks['source']} HBM copy"},
            "stages_ms": {n: t / c for n, (t, c) in stages.items()}}


D128 = "fwdbwd_bf16_l4096_d128"  # the headline model width (24 x 64) as 12 heads of 128


def d128_flops(B, H, L, d):
    """Algorithmic FLOP of one fwd+bwd at any head dim, by the headline convention with
    its transport terms kept in d: forward 2 L^2 d + L^2 d^2 / 64, backward
    5 L^2 d + 3 L^2 d^2 / 64 (both 64-position blocks); 11 L^2 d at d = 64."""
    return B * H * (7.0 * L * L * d + 4.0 * L * L * d * d / 64)


def bench_d128(P, dev, peaks, world, max_over_ranks, barrier, steps):
    """fwd+bwd at head dim 128 (same model width as the headline), per stage."""
    w = si.WORKLOADS[D128]
    B, H, L, d = w.B, w.H, w.L, w.d
    xc = si.workload_inputs(D128)
    x = {k: (v.to(dev) if v is not None else None) for k, v in xc.items()}
    del xc
    out = torch.empty_like(x["q"])
    lse = torch.empty((B, H, L), dtype=torch.float32, device=dev)
    grads = {n: torch.empty_like(x["q"]) for n in ("dq", "dk", "dv", "dw")}
    grads["dbeta"] = torch.empty_like(x["beta"])
    ws = torch.empty(P.path_attn_workspace_bytes(B, H, L, d, torch.bfloat16, True),
                     dtype=torch.uint8, device=dev)

    def step():
        P.path_attn_fwd(x["q"], x["k"], x["v"], x["w"], x["beta"], None, out=out, lse=lse,
                        workspace=ws)
        P.path_attn_bwd(x["q"], x["k"], x["v"], x["w"], x["beta"], out, lse, x["dout"], None,
                        grads=grads, workspace=ws, reuse_fwd_workspace=True)

    step()
    torch.cuda.synchronize()
    barrier()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    P.lib().path_profile_enable(1)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    P.lib().path_profile_enable(0)
    stages = read_profile()
    ms = max_over_ranks(e0.elapsed_time(e1)) / steps
    fl = d128_flops(B, H, L, d)
    del x, out, lse, grads, ws
    torch.cuda.empty_cache()
    return {"workload": f"bf16 fwd+bwd B={B} H={H} L={L} d={d}",
            "value": whole_job_rate(world, fl, ms) / 1e12, "unit": UNIT, "ms_per_step": ms,
            "flop_convention": "7 L^2 d + 4 L^2 d^2 / 64 per head (11 L^2 d at d = 64)",
            "pct_bf16_peak": whole_job_rate(1, fl, ms) / 1e12 / peaks["bf16_tflops_sustained"],
            "stages_ms": {n: t / c for n, (t, c) in stages.items()}}


def bench_decode(P, dev, peaks, world, max_over_ranks, barrier):
    w = si.WORKLOADS[DECODE]
    cap = w.n0 + w.steps
    kc, vc, seq = si.make_decode_inputs(w.B, w.H, w.d, w.n0, cap, w.steps, w.dtype, seed=0)
    kd, vd = kc.to(dev), vc.to(dev)
    del kc, vc
    sd = [{k: v.to(dev) for k, v in s.items()} for s in seq]
    out = torch.empty((w.B, w.H, w.d), dtype=w.dtype, device=dev)
    ws = torch.empty(P.path_decode_workspace_bytes(w.B, w.H, cap, w.d, w.dtype), dtype=torch.uint8,
                     device=dev)
    # warm-up on a copy of the first steps' state would change the cache; warm up on the
    # first 3 steps then rewind n (the cache rows past n0 are overwritten by the timed run)
    for t in range(3):
        s = sd[t]
        P.path_decode_step(s["q"], s["k_new"], s["v_new"], s["w"], s["beta"], kd, vd, w.n0 + t,
                           out=out, workspace=ws)
    torch.cuda.synchronize()
    barrier()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    P.lib().path_profile_enable(1)
    e0.record(stream)
    for t, s in enumerate(sd):
        P.path_decode_step(s["q"], s["k_new"], s["v_new"], s["w"], s["beta"], kd, vd, w.n0 + t,
                           out=out, workspace=ws)
    e1.record(stream)
    torch.cuda.synchronize()
    P.lib().path_profile_enable(0)
    stages = read_profile()
    ms = max_over_ranks(e0.elapsed_time(e1)) / w.steps
    nh = w.B * w.H
    n_avg = w.n0 + (w.steps - 1) / 2.0
    bytes_step = 3.0 * nh * n_avg * w.d * 2  # read K, write K, read V (bf16)
    gbs = whole_job_rate(world, bytes_step, ms) / 1e9
    chunk_ms = stages.get("decode_chunks", (0.0, 1))
    per_launch = chunk_ms[0] / max(chunk_ms[1], 1)
    ach = bytes_step / (per_launch * 1e-3) / 1e9 if per_launch else None
    # the same steps with the forget gate (PaTH-FoX decode): the cached gate biases
    # ([B,H,cap] fp32) are read and written in place beside the keys
    gen = torch.Generator().manual_seed(1)
    lfs = [torch.nn.functional.logsigmoid(3.0 + torch.randn((w.B, w.H), generator=gen)).to(dev)
           for _ in range(w.steps)]
    gc = torch.zeros((w.B, w.H, cap), dtype=torch.float32, device=dev)
    for t in range(3):
        s = sd[t]
        P.path_decode_step(s["q"], s["k_new"], s["v_new"], s["w"], s["beta"], kd, vd, w.n0 + t,
                           out=out, workspace=ws, log_f=lfs[t], g_cache=gc)
    torch.cuda.synchronize()
    barrier()
    P.lib().path_profile_enable(1)
    e0.record(stream)
    for t, s in enumerate(sd):
        P.path_decode_step(s["q"], s["k_new"], s["v_new"], s["w"], s["beta"], kd, vd, w.n0 + t,
                           out=out, workspace=ws, log_f=lfs[t], g_cache=gc)
    e1.record(stream)
    torch.cuda.synchronize()
    P.lib().path_profile_enable(0)
    gstages = read_profile()
    gms = max_over_ranks(e0.elapsed_time(e1)) / w.steps
    gbytes = bytes_step + 2.0 * nh * n_avg * 4  # + read and write the gate biases
    gt, gcnt = gstages.get("decode_chunks", (0.0, 1))
    gper = gt / max(gcnt, 1)
    gach = gbytes / (gper * 1e-3) / 1e9 if gper else None
    gated = {"value": whole_job_rate(world, gbytes, gms) / 1e9, "unit": "GB/s",
             "us_per_step": gms * 1e3, "bytes_per_step": gbytes,
             "roofline": {"kernel": "decode_chunks (gated)", "bound": "hbm", "achieved": gach,
                          "peak": peaks["hbm_gbs"], "unit": "GB/s",
                          "frac": gach / peaks["hbm_gbs"] if gach else None, "traffic": None}}
    return {"workload": DECODE, "value": gbs, "unit": "GB/s", "us_per_step": ms * 1e3,
            "bytes_per_step": bytes_step,
            "roofline": {"kernel": "decode_chunks", "bound": "hbm", "achieved": ach,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / peaks["hbm_gbs"] if ach else None, "traffic": None,
                         "peak_source": f"{peaks['source']} HBM copy"},
            "gated": gated}


PROFILE_CASES = {
    # name: (B, H, L, d, log_f) -- one untimed fwd + bwd, for profiler captures
    "b1h24l4096": (1, 24, 4096, 64, False),
    "b1h6l16384fox": (1, 6, 16384, 64, True),
    "b1h12l4096d128": (1, 12, 4096, 128, False),
}
# name: (B, H, d, cached rows) -- two untimed decode steps on a 16K-row cache
DECODE_PROFILE_CASES = {
    "decode_b2h32c16k": (2, 32, 128, 16384),
}
# name: (B, H, L, d) -- one untimed prefill (forward + decode cache)
PREFILL_PROFILE_CASES = {
    "prefill_b4h24l4096": (4, 24, 4096, 64),
}


def run_profile_case(name):
    """One forward and one backward (reusing the forward's workspace) on a small
    shape of the benchmark workload, for ncu captures of single launches; or two
    decode steps on a smaller batch of the decode workload."""
    import softmax_attention_block_b200 as P

    if name in DECODE_PROFILE_CASES:
        B, H, d, n0 = DECODE_PROFILE_CASES[name]
        kc, vc, seq = si.make_decode_inputs(B, H, d, n0, n0 + 2, 2, torch.bfloat16, seed=0)
        kd, vd = kc.cuda(), vc.cuda()
        out = torch.empty((B, H, d), dtype=torch.bfloat16, device="cuda")
        for t, s in enumerate(seq):
            s = {k: v.cuda() for k, v in s.items()}
            P.path_decode_step(s["q"], s["k_new"], s["v_new"], s["w"], s["beta"], kd, vd, n0 + t,
                               out=out)
        torch.cuda.synchronize()
        print(json.dumps({"profile_case": name, "ok": bool(torch.isfinite(out.float()).all())}))
        return 0

    if name in PREFILL_PROFILE_CASES:
        B, H, L, d = PREFILL_PROFILE_CASES[name]
        x = si.make_inputs(B, H, L, d, torch.bfloat16, seed=0)
        dx = {k: (v.cuda() if v is not None else None) for k, v in x.items()}
        out, lse, kc, vc, _ = P.path_attn_prefill(dx["q"], dx["k"], dx["v"], dx["w"], dx["beta"],
                                                  L + 64)
        torch.cuda.synchronize()
        print(json.dumps({"profile_case": name, "ok": bool(torch.isfinite(kc.float()).all())}))
        return 0

    B, H, L, d, fox = PROFILE_CASES[name]
    x = si.make_inputs(B, H, L, d, torch.bfloat16, seed=0, fox=fox)
    dx = {k: (v.cuda() if v is not None else None) for k, v in x.items()}
    ws = torch.empty(P.path_attn_workspace_bytes(B, H, L, d, torch.bfloat16, True),
                     dtype=torch.uint8, device="cuda")
    out, lse = P.path_attn_fwd(dx["q"], dx["k"], dx["v"], dx["w"], dx["beta"], dx["log_f"],
                               workspace=ws)
    P.path_attn_bwd(dx["q"], dx["k"], dx["v"], dx["w"], dx["beta"], out, lse, dx["dout"],
                    dx["log_f"], workspace=ws, reuse_fwd_workspace=True)
    torch.cuda.synchronize()
    status = P.lib().path_attn_wait_status(ws.data_ptr(), None)
    print(json.dumps({"profile_case": name, "wait_status": status}))
    return 1 if status else 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-d128", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-f32out", action="store_true")
    ap.add_argument("--no-fwd-latency", action="store_true")
    ap.add_argument("--no-fox", action="store_true")
    ap.add_argument("--no-wbeta", action="store_true")
    ap.add_argument("--profile-case", choices=sorted(PROFILE_CASES) + sorted(DECODE_PROFILE_CASES)
                    + sorted(PREFILL_PROFILE_CASES),
                    help="run one untimed fwd+bwd on a small shape (for profiler captures)")
    args = ap.parse_args()
    if args.profile_case:
        return run_profile_case(args.profile_case)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
