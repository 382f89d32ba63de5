#!/usr/bin/env python3
"""Benchmark of the B200 Muon optimizer step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload ID]
    python bench.py --impl reference ...      # the fp64 CPU oracle arm

One step = one full Muon step over the workload's 2D parameters (momentum,
Newton-Schulz, update) through the library's C ABI, or one batched
orthogonalisation for the NS-only workloads.  Inputs are seeded synthetic
tensors resident in HBM.  The default workload is the largest set, the
Llama-8B Muon set (224 matrices, 6.98 G elements, ~56 GB of params + grads +
momentum read per step), far larger than the 126 MB L2, so no flush is
needed between steps.  A short device-timed measurement of the GPT-2 124M
set follows as an extra key (--also 0 turns it off).

Prints ONE JSON line on rank 0.  Under torchrun (N > 1) the ranks share
ONE step of the workload (strong scaling): each rank runs the library's step
on the whole matrices it owns (longest-processing-time partition on the
Newton-Schulz FLOPs) and one in-place all-gather per dtype spreads the
updated parameters (sharded.py).  --replicas runs an independent replica per
GPU instead (weak scaling, no data-path collective).  The device time is the
max over ranks.
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

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)

from matrix_orthogonalizing_optimizer_step_b200 import workloads as wl  # noqa: E402

METRIC = "Muon optimizer-step ms; Newton-Schulz bf16 TFLOP/s vs B200 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--form", default="auto", choices=["auto", "standard", "gram"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--offload-chunks", type=int, default=16,
                    help="groups of matrices the e2e leg's offload step pipelines its copies over")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-adamw", action="store_true",
                    help="skip the AdamW-lane measurement on the model's AdamW parameters")
    ap.add_argument("--soft-threshold", type=float, default=0.0,
                    help="lam of the soft-threshold split of the update (0 = plain Muon)")
    ap.add_argument("--replicas", action="store_true",
                    help="with N > 1: one independent replica of the workload per GPU instead of the sharded step")
    ap.add_argument("--also", default="2",
                    help="comma-separated workload ids timed on the device after the main one (extra key)")
    ap.add_argument("--no-spectral", action="store_true",
                    help="skip the singular-value report of orthogonalised updates")
    ap.add_argument("--subset", type=int, default=0,
                    help="use only the first N matrices of the workload (small profiling cases)")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(HERE, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# CPU oracle timing (the reported baseline; never part of the GPU path)

def _ns_form_for(n, m, form):
    from oracle import muon_oracle as orc
    if form != "auto":
        return form
    return "gram" if orc.ns_flops(n, m, 5, "gram") < orc.ns_flops(n, m, 5, "standard") else "standard"


def _host_cores():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def _distinct_shapes(w):
    """[(shape, [matrix indices])] in first-appearance order."""
    by = {}
    for i, s in enumerate(w.shapes):
        by.setdefault(s, []).append(i)
    return list(by.items())


def _oracle_seconds(w, i, form, soft_threshold):
    """Wall seconds of the fp64 oracle on matrix i of workload w (one Muon
    step of that matrix, or its orthogonalisation for the NS-only sets);
    input generation is outside the timed part."""
    import torch
    from oracle import muon_oracle as orc
    r, c = w.shapes[i]
    G = wl.make_matrix(w, i, wl.ROLE_GRAD).to(torch.float64).numpy()
    fm = _ns_form_for(min(r, c), max(r, c), form)
    if w.full_step:
        M = wl.make_matrix(w, i, wl.ROLE_MOMENTUM).to(torch.float64).numpy()
        W = wl.make_matrix(w, i, wl.ROLE_PARAM).to(torch.float64).numpy()
        t0 = time.perf_counter()
        orc.muon_step(W, G, M, 0.95, True, 6e-4, form=fm, soft_threshold=soft_threshold)
    else:
        t0 = time.perf_counter()
        orc.orthogonalize(G, form=fm)
    return time.perf_counter() - t0


def _extrapolate_ms(w, per_shape):
    return sum(1e3 * statistics.fmean(per_shape[s]) * len(idx) for s, idx in _distinct_shapes(w))


def cpu_oracle_step_ms(w, budget_s, form="auto", soft_threshold=0.0):
    """Time the fp64 oracle on a bounded sample of one step of workload w and
    scale to the whole step.  One matrix of every distinct shape is timed
    first, then further matrices in order until the time budget is spent; the
    per-shape mean time is multiplied by that shape's count."""
    groups = _distinct_shapes(w)
    order = [idx[0] for _, idx in groups] + [i for _, idx in groups for i in idx[1:]]
    per_shape = {}
    t_start = time.perf_counter()
    done = 0
    for i in order:
        if done >= len(groups) and time.perf_counter() - t_start > budget_s:
            break
        per_shape.setdefault(w.shapes[i], []).append(_oracle_seconds(w, i, form, soft_threshold))
        done += 1
    sample = (f"{done} of {w.count} matrices (one of each of {len(groups)} shapes first), "
              f"fp64 NumPy oracle, per-shape mean time x count (extrapolated to the whole step)")
    return _extrapolate_ms(w, per_shape), _host_cores(), sample


# ---------------------------------------------------------------------------
# clocks

class ClockSampler:
    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid=None):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:  # noqa: BLE001
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:  # noqa: BLE001
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as fh:
            for line in fh:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 11:
                    continue
                if self.uuid and parts[1] != self.uuid:
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
        load = [r for r in rows if (num(r[5]) or 0) > 10] or rows
        sm = [num(r[2]) for r in load if num(r[2]) is not None]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in load:
            for name, v in zip(names, r[7:11]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": num(rows[0][3]), "reasons": sorted(reasons),
                "samples": len(load)}


# ---------------------------------------------------------------------------

def dist_setup(args):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def max_over_ranks(x, world, device=None):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def kernel_sources_hash():
    """sha256 (first 16 hex digits) over every source of libmuon.so: a stored
    ncu figure is only reported while the kernels it was taken on are unchanged."""
    import glob
    import hashlib
    csrc = os.path.join(HERE, "matrix_orthogonalizing_optimizer_step_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(csrc, "*"))):
        if f.endswith((".cu", ".cuh", ".h", ".cpp")):
            h.update(os.path.basename(f).encode())
            with open(f, "rb") as fh:
                h.update(fh.read())
    return h.hexdigest()[:16]


def _slug(name):
    return name.replace("/", "-")


def traffic_from_profiles(workload_name):
    """DRAM bytes per launch of the dominant kernel for this workload, from the
    committed ncu record profiles/gemm_tc_<workload>_traffic.txt, if that
    record was taken on the current kernel sources (else None).  A record
    captured on a subset of the workload states its scaling to the full set
    and stores the scaled figure (dram_bytes_per_launch)."""
    p = os.path.join(HERE, "profiles", f"gemm_tc_{_slug(workload_name)}_traffic.txt")
    if not os.path.exists(p):
        return None
    vals = {}
    with open(p) as fh:
        for line in fh:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("workload") != workload_name:
        return None
    if vals.get("kernel_sources_sha256_16") != kernel_sources_hash():
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def time_adamw_lane(w, dev, steps, peaks, world):
    """Device time of muon_adamw_step over the model's AdamW parameters (fp32
    params and moments, bf16 grads: 26 bytes per element), after 3 warm-up
    steps; GB/s against the measured HBM copy bandwidth."""
    import torch
    import matrix_orthogonalizing_optimizer_step_b200 as mo
    numels = list(w.adamw_numels)
    mo.muon_set_config(param_dtype=mo.MUON_DTYPE_F32, grad_dtype=mo.MUON_DTYPE_BF16)
    P, G, M1, M2 = [], [], [], []
    for i, n in enumerate(numels):
        P.append(wl.make_single(1, n, 5000 + i, "params", dev, "f32").view(-1))
        G.append(wl.make_single(1, n, 6000 + i, "student_t3", dev, "bf16", 0.01).view(-1))
        M1.append(torch.zeros(n, device=dev))
        M2.append(torch.zeros(n, device=dev))
    t = 0
    for _ in range(3):
        t += 1
        mo.muon_adamw_step(P, G, M1, M2, t)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, dev)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(steps):
        t += 1
        mo.muon_adamw_step(P, G, M1, M2, t)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / steps
    elems = sum(numels)
    gbs = 26.0 * elems / (ms * 1e-3) / 1e9
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    mo.muon_reset_config()
    del P, G, M1, M2
    torch.cuda.empty_cache()
    return {"kernel": "adamw (fused decoupled-decay AdamW, one grouped launch)", "tensors": len(numels),
            "elements": elems, "ms": round(ms, 4), "bound": "hbm", "achieved": round(gbs, 1), "peak": peak,
            "unit": "GB/s", "frac": round(gbs / peak, 4) if peak else None, "bytes_per_element": 26}


def make_step(w, dev, args, sharded_over=1):
    """Seeded inputs of workload w, resident in HBM, and one step over them.
    Returns (step, inputs) where inputs holds the tensors and byte counts.
    sharded_over > 1: the step is the sharded step over that many ranks
    (whole matrices per rank, then one all-gather of the parameters)."""
    import torch
    import matrix_orthogonalizing_optimizer_step_b200 as mo
    mo.muon_reset_config()
    inp = {}
    if w.full_step:
        params = [wl.make_matrix(w, i, wl.ROLE_PARAM, device=dev) for i in range(w.count)]
        grads = [wl.make_matrix(w, i, wl.ROLE_GRAD, device=dev) for i in range(w.count)]
        moms = [wl.make_matrix(w, i, wl.ROLE_MOMENTUM, device=dev) for i in range(w.count)]
        mo.muon_set_config(mode=args.form, soft_threshold=args.soft_threshold)

        if sharded_over > 1:
            from matrix_orthogonalizing_optimizer_step_b200 import sharded
            owner = sharded.partition([tuple(p.shape) for p in params], sharded_over)
            inp["owner"] = owner

            def step():
                sharded.sharded_step(params, grads, moms, mu=0.95, nesterov=True, lr=6e-4, owner=owner)
        else:
            def step():
                mo.muon_step(params, grads, moms, mu=0.95, nesterov=True, lr=6e-4)
        inp.update(params=params, grads=grads, moms=moms)
        inp["bytes_in"] = sum(g.numel() * g.element_size() for g in grads)
        inp["resident"] = inp["bytes_in"] + sum(p.numel() * p.element_size() for p in params) + \
            sum(m.numel() * m.element_size() for m in moms)
    else:
        # NS-only workloads: one batched orthogonalisation per distinct shape,
        # in place.  Every timed step re-orthogonalises the previous step's
        # output (the work does not depend on the values; the input is
        # normalised first), so no copy runs inside the timed region.
        by_shape = {}
        for i, s in enumerate(w.shapes):
            by_shape.setdefault(s, []).append(i)
        work = {s: torch.stack([wl.make_matrix(w, i, wl.ROLE_GRAD, device=dev, dtype="bf16")
                                for i in idx]) for s, idx in by_shape.items()}

        def step():
            for s in work:
                mo.muon_orthogonalize(work[s], steps=5, mode=args.form)
        inp["work"] = work
        inp["bytes_in"] = sum(t.numel() * t.element_size() for t in work.values())
        inp["resident"] = inp["bytes_in"]
    return step, inp


def device_time(step, steps, world, dev):
    """ms of `steps` steps on the launching stream (CUDA events, barrier and
    synchronize on both sides), max over ranks."""
    import torch
    stream = torch.cuda.current_stream(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, dev)
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(world, dev)
    return max_over_ranks(ev0.elapsed_time(ev1), world, dev)


def gemm_roofline(prof, ms_total, ms_per_step, peaks, peak_src, traffic):
    gemm = prof.get("gemm_tc", {})
    gemm_tf = (gemm["flops"] / (gemm["total_ms"] * 1e-3) / 1e12) if gemm.get("total_ms") else 0.0
    # A kernel inside a long step runs at the power-capped sustained clock;
    # one inside a short step at the burst clock.
    long_step = ms_per_step >= 50.0
    peak_burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_sust = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    peak_tf = peak_sust if long_step else peak_burst
    launches = gemm.get("launches", 0)
    return {
        "kernel": "gemm_tc (tcgen05 grouped GEMM, all Newton-Schulz products)",
        "bound": "tensor", "achieved": round(gemm_tf, 2), "peak": peak_tf, "unit": "TFLOP/s",
        "frac": round(gemm_tf / peak_tf, 4) if peak_tf else None,
        "traffic": traffic,
        "peak_source": (f"{peak_src} bf16_tflops_sustained (step >= 50 ms)" if long_step else
                        f"{peak_src} bf16_tflops (burst; step < 50 ms)") +
                       "; fp16 operands run at the bf16 rate",
        "frac_of_burst": round(gemm_tf / peak_burst, 4) if peak_burst else None,
        "frac_of_sustained": round(gemm_tf / peak_sust, 4) if peak_sust else None,
        "launches": launches,
        "flops_per_launch": (gemm["flops"] / launches) if launches else None,
        "avg_launch_ms": (gemm["total_ms"] / launches) if launches else None,
        "share_of_step": round(gemm.get("total_ms", 0) / ms_total, 4) if ms_total else None,
    }


def spectral_report(w, dev, form):
    """Singular values after the Newton-Schulz iteration, the monitoring check
    of [NanoGPT-Muon] "落地监控指标" (they should sit near 1): the gradient of
    the first matrix of each distinct shape, orthogonalised by the library
    (muon_orthogonalize, 5 tuned steps, the step's form), then torch's svdvals
    in fp32.  Outside every timed region.  The tuned coefficients map input
    singular values of at least 3e-3 (normalised) into [0.68, 1.21]; smaller
    ones stay below (the iteration's small-sigma gain is a^5 ~ 487)."""
    import torch
    import matrix_orthogonalizing_optimizer_step_b200 as mo
    out = []
    seen = set()
    for i, shape in enumerate(w.shapes):
        if shape in seen:
            continue
        seen.add(shape)
        x = wl.make_matrix(w, i, wl.ROLE_GRAD, device=dev, dtype="bf16").contiguous()
        mo.muon_orthogonalize(x, steps=5, mode=form)
        sv = torch.linalg.svdvals(x.float())
        q = torch.quantile(sv, torch.tensor([0.01, 0.5, 0.99], device=sv.device)).tolist()
        out.append({"shape": list(shape), "sigma_min": round(float(sv.min()), 4),
                    "sigma_p01": round(q[0], 4), "sigma_p50": round(q[1], 4), "sigma_p99": round(q[2], 4),
                    "sigma_max": round(float(sv.max()), 4),
                    "frac_in_0.68_1.21": round(float(((sv >= 0.68) & (sv <= 1.21)).float().mean()), 4)})
        del x, sv
    torch.cuda.empty_cache()
    mo.muon_release_workspace()
    return {"check": "singular values of orthogonalised gradients (first matrix of each shape)", "shapes": out}


def measure_extra(w, dev, args, peaks, peak_src, world):
    """Device-timed step of another workload (no e2e, no CPU leg)."""
    import torch
    import matrix_orthogonalizing_optimizer_step_b200 as mo
    step, inp = make_step(w, dev, args)
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    mo.muon_profile_reset()
    mo.muon_profile_enable(True)
    ms_total = device_time(step, args.steps, world, dev)
    prof = mo.muon_profile_read()
    mo.muon_profile_enable(False)
    st, bad = mo.muon_device_status()
    if st != mo.MUON_OK:
        raise SystemExit(f"device status {mo.STATUS_NAMES.get(st, st)} (matrix {bad})")
    ms = ms_total / args.steps
    out = {"workload": w.name, "workload_id": w.wid, "matrices": w.count, "elements": w.elements,
           "ms_per_step": round(ms, 4), "steps": args.steps,
           "roofline": gemm_roofline(prof, ms_total, ms, peaks, peak_src, traffic_from_profiles(w.name))}
    del step, inp
    torch.cuda.empty_cache()
    mo.muon_release_workspace()
    return out


def time_hybrid_lane(w, dev, steps, peaks, world):
    """The hybrid step's elementwise launch (muon_hybrid_step: the Muon
    momentum pass with the model's AdamW parameters appended to its grid),
    from the library's per-launch events: GB/s of the combined launch against
    the measured HBM copy bandwidth, next to the two lanes timed as separate
    launches (muon_step's momentum launch, muon_adamw_step)."""
    import torch
    import matrix_orthogonalizing_optimizer_step_b200 as mo
    mo.muon_reset_config()
    W = [wl.make_matrix(w, i, wl.ROLE_PARAM, device=dev) for i in range(w.count)]
    G = [wl.make_matrix(w, i, wl.ROLE_GRAD, device=dev) for i in range(w.count)]
    M = [wl.make_matrix(w, i, wl.ROLE_MOMENTUM, device=dev) for i in range(w.count)]
    numels = list(w.adamw_numels)
    P = [wl.make_single(1, n, 5000 + i, "params", dev, "f32").view(-1) for i, n in enumerate(numels)]
    AG = [wl.make_single(1, n, 6000 + i, "student_t3", dev, "bf16", 0.01).view(-1) for i, n in enumerate(numels)]
    M1 = [torch.zeros(n, device=dev) for n in numels]
    M2 = [torch.zeros(n, device=dev) for n in numels]

    def measure(fn):
        for t in range(1, 4):
            fn(t)
        torch.cuda.synchronize()
        mo.muon_profile_reset()
        mo.muon_profile_enable(True)
        for t in range(4, 4 + steps):
            fn(t)
        prof = mo.muon_profile_read()
        mo.muon_profile_enable(False)
        return prof

    hyb = measure(lambda t: mo.muon_hybrid_step(W, G, M, P, AG, M1, M2, t))
    sep = measure(lambda t: (mo.muon_step(W, G, M), mo.muon_adamw_step(P, AG, M1, M2, t)))
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    k = hyb["momentum_norm"]
    gbs = k["bytes"] / (k["total_ms"] * 1e-3) / 1e9
    sep_ms = (sep["momentum_norm"]["total_ms"] + sep["adamw"]["total_ms"]) / steps
    out = {"kernel": "momentum_norm, hybrid instance (Muon momentum pass + AdamW lane, one launch)",
           "workload": w.name, "muon_elements": w.elements, "adamw_elements": sum(numels),
           "ms": round(k["total_ms"] / steps, 4), "bound": "hbm", "achieved": round(gbs, 1), "peak": peak,
           "unit": "GB/s", "frac": round(gbs / peak, 4) if peak else None,
           "separate_launches_ms": round(sep_ms, 4), "launches_per_step": k["launches"] / steps}
    mo.muon_reset_config()
    del W, G, M, P, AG, M1, M2
    torch.cuda.empty_cache()
    mo.muon_release_workspace()
    return out


def run_ours(args):
    import torch
    import matrix_orthogonalizing_optimizer_step_b200 as mo

    world, rank, local = dist_setup(args)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = wl.WORKLOADS[args.workload]
    if args.subset:
        import dataclasses
        w = dataclasses.replace(w, name=f"{w.name}-first{args.subset}", shapes=w.shapes[:args.subset])
    peaks, peak_src = load_peaks()

    # ---- inputs (seeded, resident in HBM) --------------------------------
    # N > 1: the sharded step of ONE workload over all ranks (strong scaling),
    # unless --replicas asks for one independent replica per GPU (weak)
    shard = world > 1 and not args.replicas and w.full_step
    step, inp = make_step(w, dev, args, sharded_over=world if shard else 1)
    torch.cuda.synchronize()
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()

    # ---- timed region --------------------------------------------------------
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:  # noqa: BLE001
        pass
    clocks = ClockSampler(uuid)
    clocks.start()
    time.sleep(0.3)
    mo.muon_profile_reset()
    mo.muon_profile_enable(True)
    launches0 = mo.muon_launch_count()
    ms_total = device_time(step, args.steps, world, dev)
    launches = mo.muon_launch_count() - launches0
    prof = mo.muon_profile_read()
    mo.muon_profile_enable(False)
    clk = clocks.stop()
    ms_per_step = ms_total / args.steps

    st, bad = mo.muon_device_status()
    if st != mo.MUON_OK:
        raise SystemExit(f"device status {mo.STATUS_NAMES.get(st, st)} (matrix {bad})")

    # ---- roofline of the dominant kernel -------------------------------------
    gemm = prof.get("gemm_tc", {})
    momk = prof.get("momentum_norm", {})
    roofline = gemm_roofline(prof, ms_total, ms_per_step, peaks, peak_src, traffic_from_profiles(w.name))
    mom_gbs = (momk["bytes"] / (momk["total_ms"] * 1e-3) / 1e9) if momk.get("total_ms") else 0.0
    peak_gbs = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    roofline_mom = {
        "kernel": "momentum_norm (fused momentum/Nesterov/sum-of-squares/bf16 cast)",
        "bound": "hbm", "achieved": round(mom_gbs, 1), "peak": peak_gbs, "unit": "GB/s",
        "frac": round(mom_gbs / peak_gbs, 4) if peak_gbs else None,
        "launches": momk.get("launches", 0),
        "share_of_step": round(momk.get("total_ms", 0) / ms_total, 4) if ms_total else None,
    }
    ns_tflops = gemm.get("flops", 0) / (ms_total * 1e-3) / 1e12 if ms_total else 0.0
    # the standard form's work for the same matrices (15 n^2 m + 5 n^3 each, symmetric
    # products at half cost) over the same time: comparable across NS forms
    std_flops = sum(15.0 * min(r, c) ** 2 * max(r, c) + 5.0 * min(r, c) ** 3 for r, c in w.shapes)
    ns_tflops_std = std_flops * args.steps / (ms_total * 1e-3) / 1e12 if ms_total else 0.0

    # ---- end to end through the public API, host buffers ---------------------
    e2e = None
    if not args.no_e2e:
        e2e_steps = max(1, min(args.steps, 10))
        if w.full_step:
            params, grads, moms = inp["params"], inp["grads"], inp["moms"]
            host_g = [g.detach().to("cpu").pin_memory() for g in grads]
            host_p = [torch.empty(p.shape, dtype=p.dtype, pin_memory=True) for p in params]
            # the offload step keeps one plan per group of matrices: free the
            # whole-set plan of the device-timed step first
            mo.muon_release_workspace()
            if "owner" in inp:
                from matrix_orthogonalizing_optimizer_step_b200 import sharded

                def e2e_step():
                    for h, g in zip(host_g, grads):
                        g.copy_(h, non_blocking=True)
                    sharded.sharded_step(params, grads, moms, mu=0.95, nesterov=True, lr=6e-4, owner=inp["owner"])
                    for h, p in zip(host_p, params):
                        h.copy_(p, non_blocking=True)
                note = "pinned host grads -> HBM, sharded step, params -> pinned host, per step"
            else:
                def e2e_step():
                    mo.muon_step_offload(params, grads, moms, grads_host=host_g, params_host=host_p,
                                         mu=0.95, nesterov=True, lr=6e-4, chunks=args.offload_chunks)
                note = (f"muon_step_offload: pinned host grads -> HBM and updated params -> pinned host, "
                        f"pipelined with the step over {args.offload_chunks} groups of matrices, per step")
            h2d = inp["bytes_in"]
            d2h = sum(p.numel() * p.element_size() for p in params)
        else:
            work = inp["work"]
            host_in = {s: t.detach().to("cpu").pin_memory() for s, t in work.items()}
            host_out = {s: torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for s, t in work.items()}

            def e2e_step():
                for s in work:
                    work[s].copy_(host_in[s], non_blocking=True)
                    mo.muon_orthogonalize(work[s], steps=5, mode=args.form)
                    host_out[s].copy_(work[s], non_blocking=True)
            h2d = inp["bytes_in"]
            d2h = inp["bytes_in"]
            note = "pinned host matrices -> HBM, muon_orthogonalize, results -> pinned host, per step"
        e2e_step()
        torch.cuda.synchronize()
        e2e_ms = device_time(e2e_step, e2e_steps, world, dev) / e2e_steps
        e2e = {"value": round(e2e_ms, 4), "unit": "ms", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "steps": e2e_steps, "note": note}
        del e2e_step
        if w.full_step:
            del host_g, host_p
            mo.muon_release_workspace()
        else:
            del host_in, host_out

    resident_mb = inp["resident"] / 1e6
    del step, inp
    torch.cuda.empty_cache()
    mo.muon_release_workspace()

    # ---- the hybrid optimizer's AdamW lane on the model's AdamW parameters ----
    adamw = None
    if w.adamw_numels and not args.no_adamw:
        adamw = time_adamw_lane(w, dev, max(args.steps, 5), peaks, world)

    # ---- the hybrid step's single elementwise launch (GPT-2 124M set) --------
    hybrid = None
    if world == 1 and not args.no_adamw:
        hybrid = time_hybrid_lane(wl.WORKLOADS[2], dev, max(args.steps, 5), peaks, world)

    # ---- other workloads, device-timed (extra keys) ----------------------------
    extra = {}
    also = [int(x) for x in args.also.split(",") if x.strip() and int(x) != w.wid] if world == 1 else []
    for wid in also:
        ew = wl.WORKLOADS[wid]
        extra[ew.name] = measure_extra(ew, dev, args, peaks, peak_src, world)

    spectral = None
    if world == 1 and not args.no_spectral:
        spectral = spectral_report(w, dev, args.form)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, sample = cpu_oracle_step_ms(w, args.cpu_seconds, args.form, args.soft_threshold)
        cpu = {"value": round(v, 2), "unit": "ms", "cores": cores, "kind": "oracle", "sample": sample}

    if rank == 0:
        out = {
            "metric": METRIC, "value": round(ms_per_step, 4), "unit": "ms",
            "n_gpus": world, "steps": args.steps, "warmup": max(args.warmup, 3),
            "ms_per_step": round(ms_per_step, 4), "higher_is_better": False,
            "scaling": "strong" if shard else "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; shapes of the named model family, random values)",
            "config": {"workload": w.name, "workload_id": w.wid, "matrices": w.count,
                       "elements": w.elements, "ns_steps": 5, "ns_form": args.form,
                       "coeffs": [3.4445, -4.775, 2.0315], "momentum": 0.95, "nesterov": True,
                       "lr": 6e-4, "momentum_dtype": w.momentum_dtype, "param_dtype": w.param_dtype,
                       "soft_threshold": args.soft_threshold,
                       "l2": f"inputs larger than L2: {resident_mb:.0f} MB read per step",
                       "parallelism": (f"sharded x{world} (whole matrices per rank, LPT on Newton-Schulz "
                                       f"FLOPs; one all-gather of the parameters per step)") if shard else
                                      f"replica x{world} (independent per GPU)"},
            "ns_tflops_per_step": round(ns_tflops, 2),
            "ns_tflops_standard_equivalent": round(ns_tflops_std, 2),
            "roofline": roofline, "roofline_momentum": roofline_mom,
            "gpu_launches": int(launches),
            "e2e": e2e, "cpu_baseline": cpu, "clocks": clk,
            "adamw_lane": adamw,
            "hybrid_lane": hybrid,
            "spectral": spectral,
            "also": extra,
        }
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_reference(args):
    """The oracle arm: the fp64 CPU oracle, as it stands, on the host cores.
    Each step is a bounded sample of the workload: one matrix, taken from the
    distinct shapes in rotation (and from the matrices of a shape in order),
    so K steps sample every shape about K / shapes times.  The reported step
    time is the per-shape mean oracle time x that shape's count, summed: an
    extrapolation to the whole step of the workload.  Warm-up steps run the
    cheapest shape's first matrix."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import muon_oracle as orc
    w = wl.WORKLOADS[args.workload]
    groups = _distinct_shapes(w)
    cheapest = min(groups, key=lambda g: orc.ns_flops(min(g[0]), max(g[0]), 5, "standard"))[1][0]
    for _ in range(args.warmup):
        _oracle_seconds(w, cheapest, args.form, args.soft_threshold)
    per_shape = {}
    t0 = time.perf_counter()
    for k in range(args.steps):
        s, idx = groups[k % len(groups)]
        i = idx[(k // len(groups)) % len(idx)]
        per_shape.setdefault(s, []).append(_oracle_seconds(w, i, args.form, args.soft_threshold))
    # a run with fewer steps than shapes still needs every shape once
    for s, idx in groups:
        if s not in per_shape:
            per_shape[s] = [_oracle_seconds(w, idx[0], args.form, args.soft_threshold)]
    wall = time.perf_counter() - t0
    value = _extrapolate_ms(w, per_shape)
    cores = _host_cores()
    sample = (f"{sum(len(v) for v in per_shape.values())} single-matrix samples over {len(groups)} shapes "
              f"(one matrix per step, shapes in rotation; {wall:.1f} s of oracle time), fp64 NumPy oracle, "
              f"per-shape mean time x count (extrapolated to the whole step of {w.count} matrices)")
    out = {
        "impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "ms",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(value, 2), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": w.name, "workload_id": w.wid, "matrices": w.count,
                   "elements": w.elements, "ns_steps": 5, "ns_form": args.form},
        "cpu_baseline": {"value": round(value, 2), "unit": "ms", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 2), "unit": "ms", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
