#!/usr/bin/env python
"""Benchmark of the bidirectional VDA branch on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one `vda_forward` call over the full-scale workload shaped like the
paper's 14.3 s, 768p setting (B=1, H=48, T=60 interior latent frames,
U=1008 tokens per frame, d_k=d_v=128, chunk 5, window +-1 chunk, bf16 I/O,
fp32 states, text initial state from 256 prompt tokens).  Inputs are
synthetic and seeded; they are resident in HBM when the timed region starts
and far larger than L2 (about 3 GB read per step), so no L2 flush is needed.

Metric: frame-tokens/s = B*T*U / time per step (every head, both scans, the
readout and its epilogue).  With N GPUs (torchrun) every rank runs its own
problem of the same size (weak scaling, no collective on the data path) and
`value` = tokens of all ranks / max-over-ranks time.

Prints ONE JSON line on rank 0.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from frame_wise_delta_vda_b200 import inputs as gen  # noqa: E402
from frame_wise_delta_vda_b200 import ranks  # noqa: E402

WORKLOAD = "full"
METRIC = "VDA fwd+rev frame-tokens/s at H=48,U=1008,d=128; % of HBM/tensor roofline"
UNIT = "frame-tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=None,
                    help="timed steps of the host-buffer (end-to-end) measurement; 0 skips it")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(gen.WORKLOADS) + sorted(gen.PREP_WORKLOADS),
                    help="workload to run (the benchmark line is defined on 'full'; other "
                         "workloads serve profiling)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layout", choices=["replicas", "heads"], default="replicas",
                    help="replicas: every rank runs its own problem of the full size (weak scaling, no "
                         "collective); heads: one problem, each rank holding a token shard for every head, "
                         "exchanged into head shards and back by all-to-all around the forward (strong "
                         "scaling; H and T*U divisible by the rank count)")
    ap.add_argument("--scan-form", choices=["auto", "frames", "chunks"], default="auto",
                    help="scan form of the tensor-core path: per-frame chains, chunk-wise (compose the "
                         "chunks' maps, then scan them), or the library's choice")
    ap.add_argument("--heads", type=int, default=None,
                    help="run the workload with this many heads instead of its own (e.g. 6: the per-GPU "
                         "load of an 8-way head split of 48 heads)")
    ap.add_argument("--prep", action="store_true",
                    help="time the feature preparation (vda_prep) on the full-size shapes instead of the forward")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        # the raw samples go to $VDA_CLOCKS_DIR when it names a directory (kept
        # beside the run's other logs), else to a temporary file
        out_dir = os.environ.get("VDA_CLOCKS_DIR", "")
        self.path = os.path.join(out_dir, f"clocks_rank{index}.csv") if out_dir and os.path.isdir(out_dir) \
            else f"/tmp/vda_clocks_{os.getpid()}_{index}.csv"

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


def source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "frame_wise_delta_vda_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or
    None when absent or taken on a different version of the kernel source."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(kernel)
    if not d:
        return None
    if d.get("source_hash") != source_hash(*d.get("sources", [])):
        return None
    return d.get("bytes_per_launch_full")


# ----------------------------------------------------------------------------
def algorithmic(wl):
    """Per-stage algorithmic bytes and flops per launch for the workload (the
    minimal in + out traffic of each kernel at its boundary; workspace
    tensors A/M, B and the boundary states are fp32)."""
    FH, U, d, e = wl.frame_heads, wl.U, wl.d, 2 if wl.dtype == "bf16" else 4
    BH, NC = wl.B * wl.H, (wl.T + wl.chunk - 1) // wl.chunk
    dd4 = d * d * 4
    ab = FH * d * 4 if wl.alpha_mean is not None else 0   # decay gates [B, H, T, d_k] fp32
    return {
        "stats": {"bytes": FH * (2 * U * d * e + 4 * U + 2 * dd4), "flops": FH * 4 * U * d * d},
        "inverse": {"bytes": FH * 2 * dd4, "flops": FH * d ** 3},
        "scan": {"bytes": 2 * FH * 2 * dd4 + 2 * BH * (NC + 1) * dd4 + 2 * ab, "flops": 2 * FH * 2 * d ** 3},
        "readout": {"bytes": FH * 3 * U * d * e + BH * NC * 2 * dd4 + 4 * d, "flops": FH * 2 * U * d * d},
        "op": {"bytes": FH * (5 * U * d * e + 4 * U) + ab, "flops": FH * (6 * U * d * d + 5 * d ** 3)},
    }


def stage_kernels(wl):
    """(limiter, kernel name, source files) of each stage's kernel on the path
    the library takes for this workload: tensor cores for bf16 I/O at
    d_k = d_v = 128 and 64 (at 64 with the FP32 Gauss-Jordan inverse), the
    SIMT kernels otherwise.  The limiter is what sets the
    kernel's pace: "hbm" (streams its bytes near the copy bandwidth),
    "latency" (a dependent chain of small steps; its bytes are still measured
    against the HBM roofline) or "alu" (FP32 arithmetic)."""
    if wl.dtype == "bf16" and wl.d == 128:
        src = ["kernels_tc.cuh", "tc_ptx.cuh"]
        return {"stats": ("hbm", "k_stats_tc", src), "inverse": ("latency", "k_inverse_tc", src),
                "scan": ("latency", "k_scan_tc", src), "readout": ("hbm", "k_readout_tc", src)}
    if wl.dtype == "bf16" and wl.d == 64:
        src = ["kernels_tc.cuh", "tc_ptx.cuh"]
        return {"stats": ("hbm", "k_stats64_tc", src), "inverse": ("alu", "k_gj_inverse", ["kernels_simt.cuh"]),
                "scan": ("latency", "k_scan64_tc", src), "readout": ("hbm", "k_readout_tc", src)}
    src = ["kernels_simt.cuh"]
    return {"stats": ("hbm", "k_stats_simt", src), "inverse": ("alu", "k_gj_inverse", src),
            "scan": ("latency", "k_scan_simt", src), "readout": ("hbm", "k_readout_simt", src)}


def fp32_alu_peak_tflops(sm_mhz):
    # 148 SMs x 128 FP32 lanes x 2 flops (FMA) per clock
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


# ----------------------------------------------------------------------------
def cpu_baseline(wl, budget_s=15.0):
    """The float64 oracle, as it stands, on this host's cores: whole heads of
    the same workload until about `budget_s` seconds have been spent."""
    import oracle as ref
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    heads, t_total = 0, 0.0
    h = 0
    while t_total < budget_s and h < wl.H:
        x = gen.head_inputs(wl, 0, h)
        w = gen.rms_weight(wl)
        t0 = time.perf_counter()
        S0 = ref.text_state(gen.as_f64(x["k_text"]), gen.as_f64(x["v_text"]), x["beta_text"]) \
            if wl.text_tokens else None
        ref.vda_forward_head(gen.as_f64(x["q"]), gen.as_f64(x["k"]), gen.as_f64(x["v"]), x["beta"],
                             gen.as_f64(x["gate"]), w, S0, S0, wl.chunk, wl.window_chunks,
                             alpha=gen.as_f64(x["alpha"]) if "alpha" in x else None)
        t_total += time.perf_counter() - t0
        heads += 1
        h += 1
    value = wl.T * wl.U * heads / wl.H / t_total
    return {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{heads} of {wl.H} heads of the {wl.name} workload (B=1, T={wl.T}, U={wl.U}, "
                      f"d={wl.d}), fp64 NumPy, {t_total:.1f} s; value scaled to all heads"}


def run_reference(args):
    """The oracle arm: rank 0 times the fp64 oracle on one head per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle as ref
    if args.workload not in gen.WORKLOADS:
        raise SystemExit(f"{args.workload} is a feature-preparation workload; the reference arm times the forward")
    wl = gen.WORKLOADS[args.workload]
    x = gen.head_inputs(wl, 0, 0)
    w = gen.rms_weight(wl)
    args_f64 = [gen.as_f64(x["q"]), gen.as_f64(x["k"]), gen.as_f64(x["v"]), x["beta"], gen.as_f64(x["gate"])]
    S0 = ref.text_state(gen.as_f64(x["k_text"]), gen.as_f64(x["v_text"]), x["beta_text"]) \
        if wl.text_tokens else None
    alpha = gen.as_f64(x["alpha"]) if "alpha" in x else None

    def step():
        ref.vda_forward_head(*args_f64, w, S0, S0, wl.chunk, wl.window_chunks, alpha=alpha)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    value = wl.T * wl.U / wl.H / dt
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": f"{wl.name}: B={wl.B} H={wl.H} T={wl.T} U={wl.U} d={wl.d} "
                                   f"chunk={wl.chunk} window=+-{wl.window_chunks}"
                                   + (", decay gate" if alpha is not None else ""),
                       "sample": f"one head of {wl.B * wl.H} per step (oracle, host cores)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": "one head of the full workload per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
def run_prep(args):
    """One JSON line for the feature preparation step (vda_prep) at the
    full-size shapes: device time with CUDA events, HBM roofline of its
    algorithmic bytes (q, k, v in and out, bf16), and the float64 oracle on
    one head of the host as the CPU baseline."""
    import torch
    from frame_wise_delta_vda_b200 import api
    from frame_wise_delta_vda_b200._lib import lib
    lib()
    pw = gen.PREP_WORKLOADS[args.workload if args.workload in gen.PREP_WORKLOADS else "prep_full"]
    x = gen.make_prep_inputs(pw)

    def dev_t(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
        return torch.from_numpy(a).cuda()

    t = {k: dev_t(v) for k, v in x.items()}
    outs = api.vda_prep(t["q"], t["k"], t["v"], t["wk_s"], t["wk_t"], t["wv_s"], t["wv_t"], pw.Hl, pw.Wl)

    def step():
        api.vda_prep(t["q"], t["k"], t["v"], t["wk_s"], t["wk_t"], t["wv_s"], t["wv_t"], pw.Hl, pw.Wl, *outs)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    steps = min(args.steps, 50)
    sampler = ClockSampler(0)
    sampler.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1) / steps
    peaks, peak_src = load_peaks()
    byts = 6 * pw.B * pw.T * pw.U * pw.H * pw.d * 2 + 2 * pw.H * pw.d * 30 * 4
    ach = byts / (ms * 1e-3) / 1e9
    line = {"metric": "VDA-Prep frame-tokens/s", "value": pw.tokens / (ms * 1e-3), "unit": UNIT, "n_gpus": 1,
            "steps": steps, "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": True,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{pw.name}: B={pw.B} H={pw.H} T={pw.T} grid={pw.Hl}x{pw.Wl} d={pw.d}",
                       "l2": (f"inputs larger than L2 ({3 * pw.B * pw.T * pw.U * pw.H * pw.d * 2 / 1e9:.2f} GB read "
                              "per step), no flush" if 3 * pw.B * pw.T * pw.U * pw.H * pw.d * 2 > 2 * L2_BYTES else
                              "inputs fit in L2: read back from L2 between steps (not a roofline number)")},
            "roofline": {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / peaks["hbm_gbs"], "traffic": None, "kernel": "k_prep_kv + k_prep_q",
                         "algorithmic_per_launch": byts, "peak_source": f"hbm_gbs ({peak_src})"},
            "clocks": clocks, "gpu_launches": 2 * steps}
    if not args.no_cpu_baseline:
        import oracle as ref
        h0 = time.perf_counter()
        ref.prep(gen.as_f64(x["q"]), gen.as_f64(x["k"]), gen.as_f64(x["v"]), x["wk_s"], x["wk_t"], x["wv_s"],
                 x["wv_t"], pw.Hl, pw.Wl, heads=[(0, 0)])
        dt = time.perf_counter() - h0
        line["cpu_baseline"] = {"value": pw.tokens / pw.H / dt, "unit": UNIT, "kind": "oracle",
                                "cores": os.cpu_count(),
                                "sample": f"one head of {pw.H}, fp64 NumPy, {dt:.1f} s; value scaled to all heads"}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    if args.prep:
        run_prep(args)
        return

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local_rank)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)

    from frame_wise_delta_vda_b200 import api
    from frame_wise_delta_vda_b200._lib import lib
    lib()  # fail loudly without the CUDA library

    if args.workload not in gen.WORKLOADS:
        raise SystemExit(f"{args.workload} is a feature-preparation workload: use --prep")
    base = gen.WORKLOADS[args.workload]
    if args.heads is not None:
        base = gen.Workload(**{**base.__dict__, "H": args.heads, "name": f"{base.name}_H{args.heads}"})
    heads = args.layout == "heads"
    # replicas: every rank runs its own problem of the same size (weak
    # scaling); heads: every rank holds a token shard of the one problem
    wl = base if heads else gen.Workload(**{**base.__dict__, "seed": ranks.rank_seed(base.seed, rank)})

    x = gen.make_inputs(wl)
    if "k_text" not in x:
        x["k_text"], x["v_text"], x["beta_text"] = None, None, None

    def dev_t(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(a).to(dev)

    stream = torch.cuda.current_stream()
    if not heads:
        t = {k: dev_t(v) for k, v in x.items() if v is not None}
        S0 = api.vda_text_state(t["k_text"], t["v_text"], t["beta_text"]) if "k_text" in t else None
        out = torch.empty_like(t["q"])
        ws = api.workspace_for(t["q"], t["v"], wl.chunk)
        alpha = t.get("alpha")
        wl_rank = wl

        def step():
            api.vda_forward(t["q"], t["k"], t["v"], t["beta"], t["gate"], t["rms_weight"], S0, S0,
                            chunk=wl.chunk, window_chunks=wl.window_chunks, out=out, workspace=ws, alpha=alpha,
                            scan_form=args.scan_form)
    else:
        from frame_wise_delta_vda_b200 import ulysses
        if wl.H % world or (wl.T * wl.U) % world:
            raise SystemExit(f"--layout heads needs H = {wl.H} and T*U = {wl.T * wl.U} divisible by {world}")
        Hp = wl.H // world
        hs = slice(rank * Hp, (rank + 1) * Hp)
        host = {k: torch.from_numpy(v.view(np.int16) if v.dtype == np.uint16 else v)
                for k, v in x.items() if v is not None}
        for k in ("q", "k", "v", "gate", "k_text", "v_text"):
            if k in host:
                host[k] = host[k].view(torch.bfloat16)
        t = {k: ulysses.token_shard(host[k], rank, world, wl.T, wl.U).to(dev) for k in ("q", "k", "v", "gate", "beta")}
        t["rms_weight"] = host["rms_weight"].to(dev)
        S0 = (api.vda_text_state(host["k_text"][:, hs].contiguous().to(dev), host["v_text"][:, hs].contiguous().to(dev),
                                 host["beta_text"][:, hs].contiguous().to(dev)) if "k_text" in host else None)
        alpha = host["alpha"][:, hs].contiguous().to(dev) if "alpha" in host else None
        out = torch.empty((wl.B, Hp, wl.T, wl.U, wl.d), dtype=torch.bfloat16, device=dev)
        ws = api.workspace_for(out, out, wl.chunk)
        wl_rank = gen.Workload(**{**wl.__dict__, "H": Hp})
        del host

        def step():
            ulysses.vda_forward_ulysses(t["q"], t["k"], t["v"], t["beta"], t["gate"], t["rms_weight"], S0, S0,
                                        wl.T, wl.U, wl.chunk, wl.window_chunks, alpha=alpha, out=out, workspace=ws,
                                        scan_form=args.scan_form)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert api.vda_device_status() == 0

    # inputs smaller than twice the L2 (126 MB) would be served from L2 on the
    # next step: then a 256 MB buffer is written before every step and each
    # step is timed alone
    in_bytes = algorithmic(wl_rank)["op"]["bytes"]
    flush = in_bytes < 2 * L2_BYTES
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if flush else None
    sampler = ClockSampler(local_rank)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if flush:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for k, (e0, e1) in enumerate(evs):
            flush_buf.fill_(k & 0xFF)
            e0.record(stream)
            step()
            e1.record(stream)
        torch.cuda.synchronize()
        ms = sum(e0.elapsed_time(e1) for e0, e1 in evs) / args.steps
    else:
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        ms = ev0.elapsed_time(ev1) / args.steps
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    # per-kernel device time: further steps of the same workload with CUDA
    # events just before and after each launch, on its stream (kept out of the
    # region above, so that the headline time carries no extra stream work)
    kernel_steps = max(1, min(args.steps, 20))
    timer = api.StageTimer(kernel_steps)
    for _ in range(kernel_steps):
        step()
    torch.cuda.synchronize()
    stage_ms, calls = timer.read()
    status = api.vda_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")

    ms_max = ranks.max_over_ranks(ms, dist if world > 1 else None, dev)
    # a decay gate adds one launch per forward (the bridge products)
    # (the chunk-wise scans take two launches)
    per_fwd = api.vda_launches_per_forward(wl_rank.B, wl_rank.H, wl.T, wl.U, wl.d, wl.d, wl.chunk)
    if args.scan_form != "auto" and wl.d == 128 and wl.dtype == "bf16":
        per_fwd = 5 if args.scan_form == "chunks" else 4
    launches = (per_fwd + (1 if alpha is not None else 0)) * args.steps

    # ---- end to end through the host-buffer entry point ------------------------
    e2e_steps = args.e2e_steps if args.e2e_steps is not None else max(3, min(args.steps, 10))
    e2e = None
    if e2e_steps > 0 and not heads:
        e2e = run_e2e(api, x, S0, out, wl, dev, e2e_steps, world, dist)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    emit(args, wl, world, ms_max, stage_ms, calls, clocks, e2e, launches, wl_rank=wl_rank, flushed=flush)


def run_e2e(api, x, S0, out, wl, dev, e2e_steps, world, dist):
    """End-to-end timing through vda_forward_host with pinned host buffers."""
    import torch
    host = {k: torch.from_numpy(v.view(np.int16) if v.dtype == np.uint16 else v).pin_memory()
            for k, v in x.items() if k in ("q", "k", "v", "gate", "beta", "rms_weight", "alpha")}
    for k in ("q", "k", "v", "gate"):
        host[k] = host[k].view(torch.bfloat16)
    S0_host = S0.cpu().pin_memory() if S0 is not None else None
    out_host = torch.empty_like(host["q"]).pin_memory()
    hbuf = torch.empty(api.vda_forward_host_bytes(host["q"], host["v"], wl.chunk), dtype=torch.uint8, device=dev)

    def e2e_step():
        api.vda_forward_host(host["q"], host["k"], host["v"], host["beta"], host["gate"], host["rms_weight"],
                             S0_host, S0_host, out_host, wl.chunk, wl.window_chunks, hbuf, alpha=host.get("alpha"))

    e2e_step()
    if not torch.equal(out_host.view(torch.int16), out.cpu().view(torch.int16)):
        raise RuntimeError("host-buffer path disagrees with the device path")
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        e2e_step()
    torch.cuda.synchronize()
    e2e_s = (time.perf_counter() - t0) / e2e_steps
    e2e_s = ranks.max_over_ranks(e2e_s, dist if world > 1 else None, dev)
    h2d = sum(int(host[k].numel() * host[k].element_size()) for k in host)
    if S0_host is not None:
        h2d += 2 * S0_host.numel() * 4
    d2h = int(out_host.numel() * out_host.element_size())
    return {"e2e_s": e2e_s, "h2d": h2d, "d2h": d2h}


def emit(args, wl, world, ms_max, stage_ms, calls, clocks, e2e, launches, wl_rank=None, flushed=False):
    """The JSON line.  wl: the workload of the metric (each rank's own problem
    with replicas, the one sharded problem with heads); wl_rank: the problem
    one rank's kernels process (for the roofline)."""
    heads = getattr(args, "layout", "replicas") == "heads"
    wl_rank = wl_rank or wl

    # ---- roofline of the dominant kernel ------------------------------------
    peaks, peak_src = load_peaks()
    alg = algorithmic(wl_rank)
    dom = max(stage_ms, key=stage_ms.get)
    dom_ms = stage_ms[dom] / max(calls, 1)
    limiter, kname, _ = stage_kernels(wl)[dom]
    bound = "alu" if limiter == "alu" else "hbm"
    sm_mhz = (clocks or {}).get("sm_mhz") or 1965.0
    if bound == "hbm":
        achieved = alg[dom]["bytes"] / (dom_ms * 1e-3) / 1e9
        peak, unit = peaks["hbm_gbs"], "GB/s"
        peak_note = f"hbm_gbs ({peak_src})"
    else:
        achieved = alg[dom]["flops"] / (dom_ms * 1e-3) / 1e12
        peak, unit = fp32_alu_peak_tflops(sm_mhz), "TFLOP/s"
        peak_note = f"FP32 FMA peak 148 SMs x 128 lanes x 2 at the sampled {sm_mhz:.0f} MHz"
    roofline = {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
                "traffic": recorded_traffic(kname), "kernel": kname, "stage": dom, "limiter": limiter,
                "kernel_ms": dom_ms, "algorithmic_per_launch": alg[dom]["bytes" if bound == "hbm" else "flops"],
                "peak_source": peak_note}
    t_roof = max(alg["op"]["bytes"] / (peaks["hbm_gbs"] * 1e9),
                 alg["op"]["flops"] / (peaks["bf16_tflops"] * 1e12))

    tokens = wl.tokens if heads else wl.tokens * world
    line = {
        "metric": METRIC, "value": tokens / (ms_max * 1e-3), "unit": UNIT, "n_gpus": world,
        "head_tokens_per_s": tokens * wl.H / (ms_max * 1e-3),
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
        "higher_is_better": True, "scaling": "strong" if heads else "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{wl.name}: B={wl.B} H={wl.H} T={wl.T} U={wl.U} d={wl.d} chunk={wl.chunk} "
                               f"window=+-{wl.window_chunks}"
                               + (f", text S0 from {wl.text_tokens} prompt tokens" if wl.text_tokens else ", S0 = 0")
                               + (f", decay gate alpha = sigmoid(N({wl.alpha_mean}, 1))" if wl.alpha_mean is not None
                                  else ""),
                   "per_rank_problem": (f"token shard of one problem, {wl_rank.H} heads per GPU after the "
                                        "all-to-all" if heads else "independent problem of the same size per GPU"),
                   "l2": (f"inputs of {alg['op']['bytes'] / 1e6:.0f} MB fit in L2 (126 MB): a 256 MB buffer is "
                          "written before every step and each step is timed alone" if flushed else
                          f"inputs larger than L2 ({alg['op']['bytes'] / 1e9:.1f} GB read and written per step), "
                          "no flush"),
                   "kernel_timing": f"events around each launch over {calls} further steps of this workload; "
                                    "ms_per_step is timed without them",
                   "parallelism": f"heads{world} (all-to-all)" if heads else f"replicas{world}",
                   "scan_form": getattr(args, "scan_form", "auto")},
        "roofline": roofline,
        "op_roofline": {"t_roof_us": t_roof * 1e6, "frac": t_roof / (ms_max * 1e-3),
                        "bytes": alg["op"]["bytes"], "flops": alg["op"]["flops"]},
        "stage_ms": {k: v / max(calls, 1) for k, v in stage_ms.items()},
        "clocks": clocks,
        "e2e": None if e2e is None else {
            "value": tokens / e2e["e2e_s"], "unit": UNIT, "h2d_bytes_per_step": e2e["h2d"],
            "d2h_bytes_per_step": e2e["d2h"], "ms_per_step": e2e["e2e_s"] * 1e3,
            "api": "vda_forward_host (pinned host buffers)"},
        "gpu_launches": launches,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
