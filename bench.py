#!/usr/bin/env python
"""Benchmark of the FP8-moment AdamW step on a Llama2-7B-shaped parameter list.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole optimizer step over every tensor of the
layout (6,738,415,616 params, 291 tensors; fp32 params, bf16 grads, E4M3 m and
E5M2 v codes, all resident in HBM; 94.3 GB of algorithmic traffic per step,
far larger than the 126 MB L2, so no flush is needed between steps).  The
gradients are a seeded heavy-tailed draw, fixed for the timed steps; the
optimizer state evolves every step.

Multi-GPU (torchrun): each rank owns one 7B-shaped shard of the parameter
list; shards are independent (per-tensor amax and scale), so no collective is
on the data path (weak scaling); timing is the max over ranks.

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle
(the reference arm) on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "params updated/s (FP8-moment AdamW step, 7B-shaped layout)"
UNIT = "params/s"
BYTES_PER_PARAM = 14  # read p 4 + g 2 + m 1 + v 1, write p 4 + m 1 + v 1
FALLBACK_HBM_GBS = 6650.0

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per element of the
# step kernel in steady state: two consecutive launches on the pair_2x256m
# layout (536,870,912 params, 7.5 GB of traffic, far larger than L2) captured
# with --cache-control none, so the dirty L2 lines a launch leaves are written
# back inside the next one: 8.0015 B read + 5.9949 B written per param.  With
# the cache flushed before each launch instead, the writes come to 5.887 B per
# param: L2_RESIDUE bytes of a launch's writes are still dirty in L2 at its
# exit.  Both are per launch and valid while the kernel's device code hashes
# to KERNEL_SHA (null otherwise).
TRAFFIC_PER_PARAM = 13.99641
L2_RESIDUE = 60.7e6
KERNEL_SHA = "f49bdeb639a8eda0"


def _code_only(src: str) -> str:
    """C++ source without comments and blank runs (the step kernel's code is
    what the traffic figure was measured for, not its commentary)."""
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(" ".join(line.split()) for line in src.splitlines() if line.strip())


def kernel_sha() -> str:
    h = hashlib.sha256()
    for f in ("fp8adam_step.cuh", "fp8adam_step_tma.cuh", "fp8_codec.cuh"):  # the step kernel's device code
        with open(os.path.join(ROOT, "fp8_quantized_adam_b200", "csrc", f), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 50 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q, "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for k, nm in enumerate(names):
                if f[5 + k].lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- oracle leg
SINGLE_THREAD_PARAMS = 1 << 25  # the single-thread sample: about 4 s of oracle work per step


def oracle_sample_specs(specs):
    """The bounded CPU sample: the tensors of the first two transformer layers
    (18 tensors, 404 M params of the 7B layout: at least one tensor per core of
    a 16-core host); a layout without layers gives its first tensors up to
    2^26 params."""
    idx = [i for i, s in enumerate(specs) if s.name.startswith(("l0.", "l1."))]
    if not idx:
        total = 0
        for i, s in enumerate(specs):
            if idx and total + s.numel > 1 << 26:
                break
            idx.append(i)
            total += s.numel
    return idx


def single_thread_specs(specs, idx):
    """The single-thread sample: the first tensors of the all-core sample, in
    layout order, until they hold SINGLE_THREAD_PARAMS params (two 4096^2
    attention projections of the 7B layout)."""
    out, total = [], 0
    for i in idx:
        if out and total >= SINGLE_THREAD_PARAMS:
            break
        out.append(i)
        total += specs[i].numel
    return out


def run_oracle_sample(name: str, steps: int, warmup: int, single_thread: bool = False, variant: str = "default"):
    """Times the CPU oracle, as it stands, on a sample of the layout: one host
    thread per tensor on every available core (ctypes releases the GIL), or
    one thread in all.  Steps after the first are steady-state (t > 1).  A
    variant runs the oracle's extended step with the variant's options (for
    clipping, the multiplier from the sample's own gradients).  Returns
    (params/s, ms per step of the sample, threads used, sample description)."""
    from concurrent.futures import ThreadPoolExecutor

    import numpy as np
    import torch

    import oracle
    from fp8_quantized_adam_b200 import workloads

    specs = workloads.layout(name)
    cfg = workloads.CFG_ID[name]
    idx = oracle_sample_specs(specs)
    if single_thread:
        idx = single_thread_specs(specs, idx)
    sub = [specs[i] for i in idx]
    sig = workloads.tensor_sigmas(specs, cfg)
    sig = [sig[i] for i in idx]
    host = workloads.FlatModel(sub, "cpu")
    workloads.init_params_into(sub, host.views(host.p), cfg)
    workloads.grads_into(sub, host.views(host.g), cfg, 1, sig)
    states = [oracle.TensorState(host.view(host.p, k).numpy(), oracle.E4M3, oracle.E5M2) for k in range(len(sub))]
    grads = [host.view(host.g, k).view(torch.int16).numpy().view(np.uint16) for k in range(len(sub))]
    hp = workloads.HPARAMS
    threads = 1 if single_thread else min(len(sub), len(os.sched_getaffinity(0)))
    n = sum(s.numel for s in sub)
    order = sorted(range(len(sub)), key=lambda k: -sub[k].numel)

    ex_kw, ex_flags = {}, 0
    if variant in ("sr", "sr16"):
        ex_flags = oracle.FLAG_STOCHASTIC | (oracle.FLAG_SR_DRAW16 if variant == "sr16" else 0)
        ex_kw = dict(seed=1234)
    elif variant == "history":
        ex_kw = dict(hist_len=16)
    elif variant == "jit":
        ex_flags = oracle.FLAG_JIT_EVERY_STEP

    def step(t):
        gm = 1.0
        if variant == "clip":  # loss scale 1024, clip to 1.0: the multiplier from the sample's sum of squares
            sumsq, _ = oracle.grad_sumsq(grads)
            gm = oracle.grad_multiplier(sumsq, 1024.0, 1.0)

        def one(k):
            if variant == "default":
                states[k].step(grads[k], hp["lr"], hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"], t)
            else:
                states[k].step_ex(grads[k], hp["lr"], hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"], t,
                                  ex_flags, tensor_index=idx[k], grad_mult=gm, **ex_kw)
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, order))

    t = 0
    for _ in range(max(1, warmup)):  # step 1 (with its amax pre-pass) is never timed
        t += 1
        step(t)
    times = []
    for _ in range(steps):
        t += 1
        t0 = time.perf_counter()
        step(t)
        times.append(time.perf_counter() - t0)
    ms = 1e3 * sum(times) / len(times)
    desc = "%s of the %s layout (%d tensors, %d params), steady-state step (t>1)%s, %d host thread%s" % (
        "first tensors of layers 0-1" if single_thread else "layers 0-1 (or the first tensors)",
        name, len(sub), n, "" if variant == "default" else ", variant " + variant, threads,
        "" if threads == 1 else "s, one per tensor")
    return n / (ms / 1e3), ms, threads, desc


def cpu_baseline(name: str, steps: int = 1, warmup: int = 1, variant: str = "default") -> dict:
    """The oracle on every available core (the baseline's value) and on one
    thread, each on its own bounded sample of the layout, with the timed
    variant's options."""
    value, ms, threads, desc = run_oracle_sample(name, steps, warmup, variant=variant)
    v1, ms1, _, desc1 = run_oracle_sample(name, steps, warmup, single_thread=True, variant=variant)
    return {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc,
            "sample_ms_per_step": ms, "host_cores": len(os.sched_getaffinity(0)),
            "single_thread": {"value": v1, "unit": UNIT, "cores": 1, "sample": desc1, "sample_ms_per_step": ms1}}


def reference_arm(args):
    from fp8_quantized_adam_b200 import ranks, workloads

    _, rank, _ = ranks.env()
    if rank != 0:
        return
    import oracle

    oracle.build()
    value, ms, cores, desc = run_oracle_sample(args.workload, args.steps, args.warmup)
    n_full = workloads.total_params(workloads.layout(args.workload))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        # the sample's params/s carried to the whole layout; the sample's own
        # time per step is sample_ms_per_step
        "ms_per_step": n_full / value * 1e3, "sample_ms_per_step": ms,
        "ms_per_step_basis": "extrapolated to the full layout (%d params) from the sample's params/s" % n_full,
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(args.workload, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def kernel_name(args) -> str:
    """The step kernel a run times (plus the norm pre-pass for clipping)."""
    if args.variant in ("default", "jit"):
        k = "fp8adam_step_kernel<E4M3,E5M2>" if args.no_tma else "fp8adam_step_tma_kernel<E4M3,E5M2>"
        return k + (" + amax pre-pass" if args.variant == "jit" else "")
    base = ("fp8adam_step_ext_kernel<E4M3,E5M2>" if args.no_tma else
            "fp8adam_step_ext_tma_kernel<E4M3,E5M2,SRK=%d>" % {"sr": 1, "sr16": 2}.get(args.variant, 0))
    return base + (" + grad-norm pre-pass" if args.variant == "clip" else "")


def workload_config(name: str, n: int, variant: str = "default") -> dict:
    from fp8_quantized_adam_b200 import workloads

    specs = workloads.layout(name)
    n_params = workloads.total_params(specs)
    gb = BYTES_PER_PARAM * n_params / 1e9
    l2 = ("inputs larger than L2 (%.1f GB of traffic per step vs 126 MB L2), no flush" % gb if gb > 1.0 else
          "%.1f MB of traffic per step: partly L2-resident, a latency case, no flush" % (gb * 1e3))
    return {"workload": name, "params_per_gpu": n_params, "tensors": len(specs),
            "m_fmt": "e4m3", "v_fmt": "e5m2", "grads": "bf16, per-tensor N(0, 10^U(-5,-2)), 0.1% x100",
            "l2": l2,
            "parallelism": "independent shard per GPU x%d" % n, "variant": variant,
            "hparams": {"lr": 3e-4, "beta1": 0.9, "beta2": 0.95, "eps": 1e-8, "weight_decay": 0.1}}


# ----------------------------------------------------------------- our arm
def fail_on_kernel_error(opt, stream, dev, rank: int, where: str) -> None:
    """Reads the library's device error word (fp8adam_check); if any rank
    saw an error, rank 0 prints an error line and every rank exits 1.  Every
    rank takes the same collective (the max over ranks) either way."""
    from fp8_quantized_adam_b200 import ranks

    err = None
    try:
        opt.check(stream)
    except Exception as ex:  # the library's error, or a CUDA error
        err = str(ex)
    if ranks.max_over_ranks(0.0 if err is None else 1.0, dev) == 0.0:
        return
    if rank == 0:
        print(json.dumps({"metric": METRIC, "value": None, "unit": UNIT,
                          "error": "kernel error after the %s: %s" % (where, err or "on another rank")}), flush=True)
    sys.exit(1)


def our_arm(args):
    import torch

    from fp8_quantized_adam_b200 import FP8AdamW, build, capi, ranks, workloads

    world, rank, local = ranks.env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks.init("nccl", dev)
    build.build()

    def barrier():
        ranks.barrier()
        torch.cuda.synchronize()

    name = args.workload
    specs = workloads.layout(name)
    cfg = workloads.CFG_ID[name]
    n_params = workloads.total_params(specs)
    model = workloads.FlatModel(specs, dev)
    seed = ranks.shard_seed(cfg, rank)
    workloads.init_params_into(specs, model.views(model.p), seed)
    sig = workloads.tensor_sigmas(specs, cfg)
    workloads.grads_into(specs, model.views(model.g), seed, 1, sig)
    opt_kw, step_kw = {}, {}
    if args.variant == "sr":
        opt_kw = dict(stochastic_rounding=True, seed=1234)
    elif args.variant == "sr16":
        opt_kw = dict(stochastic_rounding=True, seed=1234, sr_draw_bits=16)
    elif args.variant == "history":
        opt_kw = dict(amax_history_len=16)
    elif args.variant == "jit":
        opt_kw = dict(jit_every_step=True)
    elif args.variant == "clip":
        step_kw = dict(loss_scale=1024.0, max_norm=1.0, skip_nonfinite=True)
    opt = FP8AdamW(model.views(model.p), model.views(model.g), m=model.views(model.m), v=model.views(model.v),
                   scale_m=model.scale_m, scale_v=model.scale_v, amax_m=model.amax_m, amax_v=model.amax_v,
                   chunk_elems=args.chunk_elems, tma=not args.no_tma, **opt_kw)
    stream = torch.cuda.current_stream(dev)

    for _ in range(args.warmup):
        opt.step(**step_kw)
    barrier()

    # ---- device-timed region: K steps back to back, inputs resident.  No
    # event sits between the steps, so a step's launch may overlap the
    # previous step's tail (programmatic dependent launch): the average
    # launch duration is the region's time / K.
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier()
    launches0 = capi.fp8adam_launch_count()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for k in range(args.steps):
        opt.step(**step_kw)
    t_end.record(stream)
    barrier()
    launches = capi.fp8adam_launch_count() - launches0
    clk = clocks.stop()
    # a staged kernel whose bounded wait ran out leaves its chunk undone and
    # later CTAs return at once: such a run is faster and wrong, so it ends here
    fail_on_kernel_error(opt, stream, dev, rank, "timed steps")
    elapsed = t_start.elapsed_time(t_end) / 1e3
    elapsed = ranks.max_over_ranks(elapsed, dev)
    value = world * n_params * args.steps / elapsed

    # ---- the spread of single launches: the same number of steps again, each
    # between its own pair of events (which also keeps launches from overlapping)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier()
    for k in range(args.steps):
        ev[k][0].record(stream)
        opt.step(**step_kw)
        ev[k][1].record(stream)
    barrier()
    fail_on_kernel_error(opt, stream, dev, rank, "spread steps")
    kernel_ms = [a.elapsed_time(b) for a, b in ev]

    # ---- end to end: host gradients in, amax out, through the public API
    e2e = None
    if not args.no_e2e:
        try:
            g_host = torch.empty_like(model.g, device="cpu", pin_memory=True)
            am_host = torch.empty(2 * len(specs), dtype=torch.float32, pin_memory=True)
        except RuntimeError as ex:  # pinned host memory refused (many ranks on one host)
            g_host = None
            e2e = {"value": None, "unit": UNIT, "unavailable": "pinned host buffer: %s" % str(ex)[:120]}
        ok = ranks.max_over_ranks(0.0 if g_host is not None else 1.0, dev) == 0.0  # every rank or none
        if g_host is not None and ok:
            g_host.copy_(model.g)
            e2e_steps = max(1, min(args.steps, args.e2e_steps))
            barrier()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            host_views = [g_host[o:o + sp.numel] for o, sp in zip(model.off, specs)]
            e0.record(stream)
            for _ in range(e2e_steps):
                # the library copies each tensor's gradients from the pinned
                # host buffer and steps each group of tensors as it arrives;
                # the step's amax comes back to the host
                opt.step_host(host_views, am_host, stream=stream, **step_kw)
            e1.record(stream)
            barrier()
            fail_on_kernel_error(opt, stream, dev, rank, "end-to-end steps")
            et = ranks.max_over_ranks(e0.elapsed_time(e1) / 1e3, dev)
            e2e = {"value": world * n_params * e2e_steps / et, "unit": UNIT,
                   "h2d_bytes_per_step": 2 * n_params,
                   "d2h_bytes_per_step": am_host.numel() * am_host.element_size(), "steps": e2e_steps,
                   "api": "FP8AdamW.step_host -> fp8adam_step_host (per-tensor H2D copies on the library's copy "
                          "stream, overlapping the step of earlier tensor groups)"}
        elif e2e is None:
            e2e = {"value": None, "unit": UNIT, "unavailable": "pinned host buffer refused on another rank"}
        del g_host

    peak, peak_kind = hbm_peak()
    avg_kernel_s = elapsed / args.steps  # the timed region's launches, back to back
    # bytes per param of one step: the fused clip/skip variant reads the
    # gradients once more in its norm pre-pass
    # and current scaling ("jit") runs an amax pre-pass over g, m, v first
    bpp = BYTES_PER_PARAM + {"clip": 2, "jit": 4}.get(args.variant, 0)
    achieved = bpp * n_params / avg_kernel_s / 1e9
    traffic = residue = None
    if TRAFFIC_PER_PARAM is not None and KERNEL_SHA == kernel_sha() and args.variant == "default" and not args.no_tma:
        traffic = TRAFFIC_PER_PARAM * n_params
        residue = L2_RESIDUE
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "peak_kind": peak_kind + " (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else peak_kind,
                "traffic": traffic,
                "traffic_basis": ("ncu dram__bytes_read.sum + dram__bytes_write.sum per param of a steady-state launch "
                                  "(pair_2x256m, --cache-control none) x this launch's params") if traffic else None,
                "l2_residue_bytes": residue,
                "kernel": kernel_name(args),
                "algorithmic_bytes_per_launch": bpp * n_params,
                "kernel_ms_avg": avg_kernel_s * 1e3,
                "single_launch_ms": {"min": min(kernel_ms), "p50": sorted(kernel_ms)[len(kernel_ms) // 2],
                                     "p90": sorted(kernel_ms)[min(len(kernel_ms) - 1, (9 * len(kernel_ms)) // 10)],
                                     "max": max(kernel_ms),
                                     "note": "a second pass of the same steps, each between its own CUDA events"},
                "frac_of_8TBs_nominal": achieved / 8000.0}
    if args.variant == "sr":
        roofline["note"] = ("stochastic rounding with 32-bit draws is bound by instruction issue, not DRAM "
                            "(Philox4x32-10 for every two elements and the integer SR encoder)")
    elif args.variant == "sr16":
        roofline["note"] = ("stochastic rounding with 16-bit draws: one Philox4x32-10 call per eight elements, "
                            "four codes per hardware stochastic-rounding conversion")

    cpu = None  # the CPU oracle is timed on rank 0 of a 1-GPU run only
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle

        oracle.build()
        cpu = cpu_baseline(name, variant=args.variant)

    opt.close()
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": elapsed * 1e3 / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": workload_config(name, world, args.variant), "roofline": roofline, "cpu_baseline": cpu,
                "e2e": e2e, "gpu_launches": launches, "clocks": clk,
                "gb_per_s": world * bpp * n_params * args.steps / elapsed / 1e9}
        print(json.dumps(line), flush=True)
    ranks.finish()


def ablation_report(args):
    """Moment-format ablation on the Llama2-100M layout ([EXPL] "实验证据
    (Fig. 5)"): all four (m, v) format pairs and the fp32-moment run, plus
    the four pairs with stochastic rounding on 16-bit draws, in lockstep on
    the same seeded gradients.  Per mode: step throughput, the
    per-step count of v elements flushed to zero, and the per-step max and
    mean |p_mode - p_fp32| (gradients are open-loop, so the difference is the
    optimizer's own error)."""
    import torch

    from fp8_quantized_adam_b200 import FP8AdamW, build, workloads

    build.build()
    dev = torch.device("cuda", 0)
    name = "ablation_100m"
    specs = workloads.layout(name)
    cfg = workloads.CFG_ID[name]
    n_params = workloads.total_params(specs)
    # (m format, v format, rounding): round to nearest, and stochastic rounding
    # with 16-bit draws for every FP8 pair
    modes = {"m4v4": ("e4m3", "e4m3", "rn"), "m4v5": ("e4m3", "e5m2", "rn"), "m5v4": ("e5m2", "e4m3", "rn"),
             "m5v5": ("e5m2", "e5m2", "rn"), "fp32": ("fp32", "fp32", "rn"),
             "m4v4_sr16": ("e4m3", "e4m3", "sr16"), "m4v5_sr16": ("e4m3", "e5m2", "sr16"),
             "m5v4_sr16": ("e5m2", "e4m3", "sr16"), "m5v5_sr16": ("e5m2", "e5m2", "sr16")}
    models, opts = {}, {}
    g = workloads.FlatModel(specs, dev).g  # one gradient buffer shared by all modes
    for k, (mf, vf, rnd) in modes.items():
        M = workloads.FlatModel(specs, dev, m_fp32=mf == "fp32", v_fp32=vf == "fp32")
        workloads.init_params_into(specs, M.views(M.p), cfg)
        M.g = g
        models[k] = M
        sr = dict(stochastic_rounding=True, seed=0xAB1A7E, sr_draw_bits=16) if rnd == "sr16" else {}
        opts[k] = FP8AdamW(M.views(M.p), M.views(g), m_fmt=mf, v_fmt=vf, m=M.views(M.m), v=M.views(M.v),
                           scale_m=M.scale_m, scale_v=M.scale_v, amax_m=M.amax_m, amax_v=M.amax_v,
                           stats=True, **sr)
    sig = workloads.tensor_sigmas(specs, cfg)
    off = workloads.offsets(specs)
    views = [g[off[i]:off[i] + s.numel] for i, s in enumerate(specs)]
    out = {k: {"flushed_v": [], "saturated": [], "max_abs_dp_vs_fp32": [], "mean_abs_dp_vs_fp32": [], "ms": []}
           for k in modes}
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    for t in range(1, args.steps + 1):
        workloads.grads_into(specs, views, cfg, t, sig)
        for k in modes:
            opts[k].reset_stats()
            ev[0].record()
            opts[k].step()
            ev[1].record()
            ev[1].synchronize()
            out[k]["ms"].append(ev[0].elapsed_time(ev[1]))
            f, s_ = opts[k].stats()
            out[k]["flushed_v"].append(f)
            out[k]["saturated"].append(s_)
        for k in modes:
            d = (models[k].p - models["fp32"].p).abs()
            out[k]["max_abs_dp_vs_fp32"].append(float(d.max()))
            out[k]["mean_abs_dp_vs_fp32"].append(float(d.mean(dtype=torch.float64)))
    res = {}
    for k, (mf, vf, rnd) in modes.items():
        ms = sorted(out[k]["ms"][3:] or out[k]["ms"])
        med = ms[len(ms) // 2]
        bpp = 4 + 2 + 4 + (8 if mf == "fp32" else 2) + (8 if vf == "fp32" else 2)
        res[k] = {"m_fmt": mf, "v_fmt": vf, "rounding": rnd, "params_per_s": n_params / (med / 1e3),
                  "gb_per_s": bpp * n_params / (med / 1e3) / 1e9, "bytes_per_param": bpp,
                  "flushed_v_mean": sum(out[k]["flushed_v"]) / args.steps,
                  "final_max_abs_dp_vs_fp32": out[k]["max_abs_dp_vs_fp32"][-1],
                  "final_mean_abs_dp_vs_fp32": out[k]["mean_abs_dp_vs_fp32"][-1], **out[k]}
        del res[k]["ms"]
    for k, o in opts.items():
        o.check()  # raises if a kernel's bounded wait ran out: no report from a broken run
        o.close()
    print(json.dumps({"report": "format_ablation", "workload": name, "params": n_params, "steps": args.steps,
                      "data": "synthetic", "modes": res}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="llama2_7b")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--chunk-elems", type=int, default=0, help="elements per CTA (0: chosen by the library)")
    ap.add_argument("--no-tma", action="store_true", help="per-thread vector loads instead of TMA staging")
    ap.add_argument("--variant", choices=["default", "sr", "sr16", "history", "clip", "jit"], default="default",
                    help="step options: stochastic rounding, amax history 16, fused loss-scale/clip/skip, "
                         "current scaling (amax pre-pass every step)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--report", choices=["ablation"], default=None,
                    help="ablation: the moment-format ablation on the Llama2-100M layout")
    args = ap.parse_args()
    if args.report == "ablation":
        ablation_report(args)
    elif args.impl == "reference":
        reference_arm(args)
    else:
        our_arm(args)


if __name__ == "__main__":
    main()
