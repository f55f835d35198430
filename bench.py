#!/usr/bin/env python
"""Throughput benchmark: verified specs/sec of one full bound-propagation step on B200.

A step is one vf_verify_batch call over the whole batch: IBP over every node, CROWN passes
for the intermediate bounds, the specification pass and the decision. Headline workload:
ReLU MLP 3072-(1024 x 8)-100, 4096 centres, eps = 1/255, 99 margin rows per centre, IBP
intermediate bounds for z1..z6 and CROWN for z7, z8 and the output (synthetic, seeded; see
linear_bound_propagation_b200.synth). The same line carries that network at eps 0.5/255 and
2/255 (`eps_sweep`) and the other four workloads (`workloads`: value, ms per step, the
dominant kernel's roofline and the oracle's CPU baseline each).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config 1..5]

Prints one JSON line (rank 0). With N > 1 (torchrun) every rank runs an independent replica
of the workload on its own GPU (no collective on the data path; the barrier and the max over
ranks are for timing only), so `value` counts the specs of all ranks ("scaling": "weak").
`--impl reference` times the fp64 CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_bound_propagation_b200 import synth  # noqa: E402

METRIC = "verified specs/sec (IBP+CROWN bounds) at 1 B200; % tensor-pipe / HBM roofline"
UNIT = "specs/s"
L2_FLUSH_BYTES = 256 << 20


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}, \
            "fallback"


def threads_used():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def workload_config(w, cfg):
    R = w.C.shape[1]
    return {"workload": w.name, "centres": int(w.centres.shape[0]), "spec_rows": int(R),
            "eps": float(w.eps), "both_sides": bool(w.both_sides),
            "intermediate_bounds": "crown for relus " + (str(w.crown_relus) if w.crown_relus else "all (first layer exact by IBP)"),
            "l2": "flushed between timed steps (256 MiB write)", "parallelism": "replicas (one full workload per GPU)",
            "config_index": cfg}


def oracle_sample(w, target_s):
    """Time the oracle on the first n centres of the workload, n sized to about target_s seconds.
    Workloads whose single centre already takes minutes on the host (the residual network: 148,480
    intermediate-pass rows per centre) are timed on a row sample of one centre instead (see
    oracle_row_sample)."""
    import oracle.lbp as O
    R = w.C.shape[1] * (2 if w.both_sides else 1)
    if intermediate_rows(w) > 20000:
        return oracle_row_sample(w)

    def run(n):
        t0 = time.perf_counter()
        O.verify(w.net, w.centres[:n], w.eps, w.C[:n] if w.C.shape[0] > 1 else w.C, crown_relus=w.crown_relus,
                 both_sides=w.both_sides)
        return time.perf_counter() - t0

    B = w.centres.shape[0]
    t1 = run(1)
    n = int(max(1, min(B, target_s / max(t1, 1e-6))))
    t = run(n) if n > 1 else t1
    return {"value": n * R / t, "unit": UNIT, "cores": threads_used(), "kind": "oracle",
            "sample": f"first {n} of {B} centres of {w.name} ({n * R} specs), fp64 numpy oracle, {t:.2f} s"}, n, t


def crown_passes(w):
    """(relu node, pre-activation node, neurons) of every intermediate CROWN pass the oracle runs."""
    import oracle.lbp as O
    sh = O.shapes(w.net)
    relus = [v for v, nd in enumerate(w.net) if nd.op == "relu"]
    sel = set(relus if w.crown_relus is None else w.crown_relus)
    out = []
    for k in relus:
        p = w.net[k].src
        first_affine = w.net[p].op in ("dense", "conv") and w.net[p].src == 0
        if k in sel and not first_affine:
            out.append((k, p, int(np.prod(sh[p]))))
    return out


def intermediate_rows(w):
    return sum(2 * n for _, _, n in crown_passes(w))


def oracle_row_sample(w, rows_per_pass=32):
    """The oracle's per-centre time on one centre, from its own functions: the IBP pass and the
    specification pass in full, and for every intermediate pass the first rows_per_pass / 2 rows of
    [I] and of [-I] through crown_pass, scaled to the pass's 2n rows. A pass's cost is linear in its
    rows (rows are independent and each takes the same operations), and the relaxation values do not
    change the work, so the earlier layers' relaxations are taken from the IBP bounds."""
    import oracle.lbp as O
    R = w.C.shape[1] * (2 if w.both_sides else 1)
    c = w.centres[:1]
    t0 = time.perf_counter()
    cs, rs = O.ibp(w.net, c, w.eps)
    t_ibp = time.perf_counter() - t0
    relax = {}
    relus = [v for v, nd in enumerate(w.net) if nd.op == "relu"]
    passes = {k: (p, n) for k, p, n in crown_passes(w)}
    t_passes, sampled = 0.0, 0
    for k in relus:
        p = w.net[k].src
        if k in passes:
            n = passes[k][1]
            h = min(n, rows_per_pass // 2)
            eye = np.eye(n)[:h]
            t0 = time.perf_counter()
            O.crown_pass(w.net, p, np.concatenate([eye, -eye]), relax, c[0], w.eps)
            t_passes += (time.perf_counter() - t0) * (2 * n) / (2 * h)
            sampled += 2 * h
        relax[k] = O.relax_params(cs[p][0] - rs[p][0], cs[p][0] + rs[p][0])
    Cb = w.C[0]
    rows = np.concatenate([Cb, -Cb]) if w.both_sides else Cb
    t0 = time.perf_counter()
    O.crown_pass(w.net, len(w.net) - 1, rows, relax, c[0], w.eps)
    t_spec = time.perf_counter() - t0
    t = t_ibp + t_passes + t_spec
    return {"value": R / t, "unit": UNIT, "cores": threads_used(), "kind": "oracle",
            "sample": f"one centre of {w.name}: IBP and the {R}-row specification pass in full, and {sampled} of "
                      f"the {intermediate_rows(w)} intermediate-pass rows ({rows_per_pass} per pass) scaled "
                      f"linearly to each pass's rows; {t:.1f} s per centre, fp64 numpy oracle"}, 1, t


def start_clocks():
    path = tempfile.mktemp(suffix=".csv")
    q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")
    dev = os.environ.get("LOCAL_RANK", "0")
    try:
        f = open(path, "w")
        p = subprocess.Popen(["nvidia-smi", "-i", str(dev), f"--query-gpu={q}", "--format=csv,noheader,nounits",
                              "-lms", "20"], stdout=f, stderr=subprocess.DEVNULL)
        # start timing only once the sampler is running, so that its samples fall inside the timed region
        t0 = time.time()
        while time.time() - t0 < 3.0 and p.poll() is None and os.path.getsize(path) == 0:
            time.sleep(0.01)
        with open(path) as fh:
            first = len(fh.readlines())
        return p, f, path, first
    except Exception:
        return None, None, path, 0


def stop_clocks(handle):
    p, f, path, first = handle
    if p is None:
        return None
    p.terminate()
    try:
        p.wait(timeout=5)
    except Exception:
        p.kill()
    f.close()
    sm, mx, reasons = [], 0.0, set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    with open(path) as fh:
        lines = fh.readlines()
    if len(lines) > first:  # drop the samples taken before the timed region started
        lines = lines[first:]
    for line in lines:
        parts = [x.strip() for x in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            mx = max(mx, float(parts[2]))
        except ValueError:
            continue
        for nm, v in zip(names, parts[5:9]):
            if v.lower().startswith("active"):
                reasons.add(nm)
    os.unlink(path)
    if not sm:
        return None
    return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# Nominal dense-throughput ratios used to derive a per-dtype peak from the measured bf16 one.
TF32_OVER_BF16 = 1.1 / 2.25

# DRAM bytes per launch of the dominant kernel: dram__bytes_read.sum + dram__bytes_write.sum from one ncu
# capture of the full-size workload, summed over the six contraction launches of one timed step and divided
# by six. Keyed by workload name and kernel kind; reported only for that pair, and to be dropped whenever
# the kernel changes.
# DRAM bytes (read + write) per dense_back_tc launch, from one-pass ncu captures of the current kernel
# (profiles/dense_back_tc_wide_mlp_B4096.md section 3b): every launch of one verify call; the wide MLP measured at 256
# centres (21 launches, 48.69 GB) and scaled by rows to 4096 centres (traffic grows with the rows), over its 73
# full-size launches
TRAFFIC_PER_LAUNCH = {("mlp_784-256x3-10_B1024", 1): 1.105e9 / 6,
                      ("mlp_3072-1024x8-100_B4096", 1): 48.69e9 * 16 / 73}


def roofline(kstats, step_total_ms, n_sms, workload=None, step_ms=None):
    """Roofline entry for the dominant contraction kind of the step.

    Tensor-core steps (3xTF32, dense and convolution): algorithmic flops per launch (2*M*K*N dense;
    2*M*positions*C_in*C_out*k*k/s^2 convolution) against the tf32 peak divided by 3 (three tf32 products per
    fp32-accurate one); the tf32 peak is the measured bf16 peak times the nominal tf32/bf16 ratio, the burst
    figure for short steps and the sustained (power-capped) one for steps of 100 ms and longer. FFMA kernels:
    fp32 FFMA peak = SMs x 128 lanes x 2 flop x max SM clock ("alu")."""
    p, src = peaks()
    kind = max(kstats, key=lambda k: kstats[k][1])
    n_k, k_ms, k_flops = kstats[kind]
    avg_ms = k_ms / max(n_k, 1)
    achieved = (k_flops / max(n_k, 1)) / (avg_ms / 1000.0) / 1e12 if n_k else 0.0
    sm_mhz = float(p.get("sm_max_mhz", 1965.0))
    if kind in (1, 5, 7):
        sustained = step_ms is not None and step_ms >= 100.0 and "bf16_tflops_sustained" in p
        bf16 = float(p["bf16_tflops_sustained"] if sustained else p["bf16_tflops"])
        tf32 = bf16 * TF32_OVER_BF16
        peak = tf32 / 3.0
        bound = "tensor"
        name = {1: "dense_back_tc (tcgen05 kind::tf32, 3xTF32 CROWN Lambda.W contraction)",
                5: "conv_back_tc (tcgen05 kind::tf32 implicit GEMM, 3xTF32 transposed convolution)",
                7: "conv_back_tc on a 3-channel stem (input channels padded to 16)"}[kind]
        psrc = (f"tf32 = {src} bf16 {'sustained' if sustained else 'burst'} {bf16:.0f} TFLOP/s x nominal "
                f"1.1/2.25 = {tf32:.0f}; 3xTF32 effective = tf32 / 3")
    else:
        peak = n_sms * 128 * 2 * sm_mhz * 1e6 / 1e12
        bound = "alu"
        name = {2: "dense_back_ffma", 3: "conv_back_ffma", 4: "conv_back_win_k (receptive-field windows)"}[kind]
        psrc = f"fp32 FFMA: {n_sms} SMs x 128 lanes x 2 flop x {sm_mhz:.0f} MHz ({src} max clock)"
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "traffic": TRAFFIC_PER_LAUNCH.get((workload, kind)), "kernel": name, "launches": n_k, "avg_launch_ms": avg_ms,
            "share_of_step": k_ms / step_total_ms if step_total_ms else None, "peak_source": psrc}


def max_over_ranks(value: float, device) -> float:
    """Largest `value` over all ranks of the default process group (timing only, never data)."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_throughput(world: int, specs_per_rank_step: int, steps: int, total_ms: float) -> float:
    """Whole-job specs/s: every rank processes its own full workload each step; the job takes the
    slowest rank's time."""
    return world * specs_per_rank_step * steps / (total_ms / 1000.0)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = synth.workload(args.config)
    # each step a bounded sample: about two minutes for the whole --warmup + --steps run (at least one centre)
    per_step_s = min(args.cpu_sample_s, 120.0 / max(1, args.warmup + args.steps))
    base, n, t = oracle_sample(w, per_step_s)
    R = w.C.shape[1] * (2 if w.both_sides else 1)
    import oracle.lbp as O
    row_sampled = intermediate_rows(w) > 20000
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        if row_sampled:  # one centre's time from a row sample (see oracle_row_sample)
            dt = oracle_row_sample(w)[2]
        else:
            O.verify(w.net, w.centres[:n], w.eps, w.C[:n] if w.C.shape[0] > 1 else w.C, crown_relus=w.crown_relus,
                     both_sides=w.both_sides)
            dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    value = n * R * len(times) / sum(times)
    base["value"] = value
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * sum(times) / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, args.config), "cpu_baseline": base,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    ctx = {"world": world, "rank": rank, "dev": dev,
           "flush": torch.empty(L2_FLUSH_BYTES // 4, device=dev)}

    # the headline: the configured workload at its own radius, every step timed, with the e2e leg
    line = measure_workload(args, ctx, args.config, None, args.steps, args.warmup, headline=True)
    if args.eps_sweep and args.config == 5:
        # the same network and batch at the other two radii of the benchmark definition
        sweep = []
        for e in (0.5 / 255.0, 2.0 / 255.0):
            sweep.append(measure_workload(args, ctx, 5, e, min(args.steps, args.sub_steps), min(args.warmup, 3),
                                          headline=False))
        if line is not None:
            line["eps_sweep"] = sweep
    if args.all_workloads:
        subs = {}
        for cfg in (1, 2, 3, 4, 5):
            if cfg == args.config:
                continue
            subs[synth.WORKLOAD_NAMES[cfg]] = measure_workload(
                args, ctx, cfg, None, min(args.steps, args.sub_steps), min(args.warmup, 3), headline=False,
                legs=(cfg == 2))
        if line is not None:
            line["workloads"] = subs
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def measure_workload(args, ctx, cfg, eps, steps, warmup, headline, legs=None):
    """Time `steps` vf_verify_batch calls on workload `cfg` (radius `eps`, or the workload's own). The
    headline adds the end-to-end leg, the clocks and the launch count; `legs` the alpha-CROWN, sound and
    branch-and-bound legs. Returns the JSON object on rank 0 (None elsewhere)."""
    import torch
    import torch.distributed as dist
    from linear_bound_propagation_b200 import vf

    world, rank, dev, flush = ctx["world"], ctx["rank"], ctx["dev"], ctx["flush"]
    if legs is None:
        legs = headline and cfg == 2

    def barrier():
        if world > 1:
            dist.barrier()

    w = synth.workload(cfg, B=args.centres if headline else None, eps=eps)
    B, R = w.centres.shape[0], w.C.shape[1]
    Rs = R * (2 if w.both_sides else 1)
    net = vf.Net(w.net, workspace_bytes=int(args.workspace_gb * (1 << 30)))
    centres = torch.from_numpy(w.centres).to(dev)
    C = torch.from_numpy(w.C).to(dev)
    stream = torch.cuda.current_stream()
    out = {"lb": torch.empty(B, R, device=dev), "lb_ibp": torch.empty(B, R, device=dev),
           "verified": torch.empty(B, R, device=dev, dtype=torch.uint8)}
    if w.both_sides:
        out["ub"] = torch.empty(B, R, device=dev)
    kw = dict(crown_relus=w.crown_relus, both_sides=w.both_sides, out=out)

    for _ in range(warmup):
        net.verify(centres, w.eps, C, **kw)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()

    clk = start_clocks()
    launches0 = net.launch_count()
    net.profile(True)
    net.profile_read(reset=True)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        ev[i][0].record(stream)
        net.verify(centres, w.eps, C, **kw)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    clocks = stop_clocks(clk)
    launches = net.launch_count() - launches0
    kstats = {k: net.profile_read(kind=k, reset=False) for k in (1, 2, 3, 4, 5, 7)}
    fwd = net.profile_read(kind=vf.VF_KERNEL_DENSE_FWD_TC, reset=False)
    net.profile_read(reset=True)
    net.profile(False)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = float(sum(step_ms))
    total_ms = max_over_ranks(total_ms, dev)
    value = weak_throughput(world, B * Rs, steps, total_ms)
    verified = int(out["verified"].sum().item())
    roof = roofline(kstats, total_ms, torch.cuda.get_device_properties(dev).multi_processor_count,
                    w.name if (args.centres is None or not headline) else None, total_ms / steps)
    pad = kstats.get(7, (0, 0.0, 0.0))
    if pad[0] and roof.get("kernel", "").startswith("conv_back_tc (") and pad[1] > 0:
        # the stem on the tensor cores (its useful flops are 3/16 of the MMA work): reported beside the others
        roof["stem_tc"] = {"launches": pad[0], "ms": pad[1], "share_of_step": pad[1] / total_ms,
                           "achieved_tflops": pad[2] / (pad[1] / 1000.0) / 1e12}
    if fwd[0]:  # the alpha ascent's forward products on the tensor cores (reported beside the dominant kernel)
        roof["forward_products_tc"] = {"launches": fwd[0], "ms": fwd[1], "share_of_step": fwd[1] / total_ms,
                                       "achieved_tflops": fwd[2] / (fwd[1] / 1000.0) / 1e12 if fwd[1] else None}

    e2e = None
    if headline and not args.no_e2e:
        e2e = e2e_leg(args, w, net, centres, C, out, kw, stream, flush, dev, world, steps)
    graph = graph_leg(args, w, net, centres, C, stream, flush, dev, world, steps, warmup, B * Rs) \
        if (headline and args.graph) else None
    alpha = sound = bab = None
    if legs:
        alpha = alpha_leg(args, w, net, centres, C, stream, flush, dev, world, steps)
        sound = sound_leg(args, w, net, centres, C, out, kw, stream, flush, dev, world, B * Rs)
        if args.bab_domains > 0 and not w.both_sides and w.C.shape[1] > 1:
            bab = bab_leg(args, w, net, centres, dev, stream, world, rank)
    net.close()
    del net
    torch.cuda.empty_cache()
    if rank != 0:
        return None
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps,
            "warmup": warmup, "ms_per_step": total_ms / steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": workload_config(w, cfg), "roofline": roof, "gpu_launches": launches, "clocks": clocks,
            "verified_specs": verified, "total_specs": B * Rs}
    if headline:
        line["e2e"] = e2e
        line["graph"] = graph
    if legs:
        line.update({"alpha_crown": alpha, "bab": bab, "sound": sound})
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_sample(w, args.cpu_sample_s if headline else args.sub_cpu_sample_s)[0]
        if bab is not None:
            line["cpu_baseline"]["bab"] = oracle_bab_sample(args, w, bab["sample_centre"], bab["sample_label"])
    if not headline:  # sub-lines keep only what identifies and measures them
        for k in ("metric", "unit", "n_gpus", "higher_is_better", "scaling", "vs_baseline", "dtype", "data"):
            line.pop(k, None)
    return line


def e2e_leg(args, w, net, centres, C, out, kw, stream, flush, dev, world, steps):
    """End to end through the public API with host buffers, every step's copies inside the timed region:
    pinned H2D of the step's centres and C, the verify call, D2H of lb and verified. Two buffer sets and a
    copy stream: the H2D of step i+1 and the D2H of step i run while step i+1 / i+2 compute."""
    import torch
    import torch.distributed as dist
    B, R = w.centres.shape[0], w.C.shape[1]
    Rs = R * (2 if w.both_sides else 1)
    h_centres = torch.from_numpy(w.centres).pin_memory()
    h_C = torch.from_numpy(w.C).pin_memory()
    h_lb = [torch.empty(B, R).pin_memory() for _ in range(2)]
    h_ver = [torch.empty(B, R, dtype=torch.uint8).pin_memory() for _ in range(2)]
    d_c = [torch.empty_like(centres) for _ in range(2)]
    d_C = [torch.empty_like(C) for _ in range(2)]
    outs = [out] + [{k: torch.empty_like(v) for k, v in out.items()}]
    copy = torch.cuda.Stream(device=dev)

    def e2e_run(n):
        ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of buffer set k are on the device
        ev_done = [torch.cuda.Event() for _ in range(2)]  # the verify reading set k has finished
        ev_out = [torch.cuda.Event() for _ in range(2)]   # the results of set k have reached the host
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def h2d(k):
            with torch.cuda.stream(copy):
                d_c[k].copy_(h_centres, non_blocking=True)
                d_C[k].copy_(h_C, non_blocking=True)
                ev_in[k].record(copy)

        t0.record(copy)
        h2d(0)
        for i in range(n):
            k = i % 2
            if i + 1 < n:
                if i >= 1:
                    copy.wait_event(ev_done[1 - k])  # set 1-k is free once step i-1 has read it
                h2d(1 - k)
            stream.wait_event(ev_in[k])
            if i >= 2:
                stream.wait_event(ev_out[k])  # step i-2's results have been copied out of set k
            flush.zero_()
            net.verify(d_c[k], w.eps, d_C[k], crown_relus=w.crown_relus, both_sides=w.both_sides, out=outs[k])
            ev_done[k].record(stream)
            with torch.cuda.stream(copy):
                copy.wait_event(ev_done[k])
                h_lb[k].copy_(outs[k]["lb"], non_blocking=True)
                h_ver[k].copy_(outs[k]["verified"], non_blocking=True)
                ev_out[k].record(copy)
        t1.record(copy)
        t1.synchronize()
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    e2e_run(2)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e2e_ms = max_over_ranks(e2e_run(steps), dev)
    return {"value": weak_throughput(world, B * Rs, steps, e2e_ms), "unit": UNIT,
            "h2d_bytes_per_step": h_centres.numel() * 4 + h_C.numel() * 4,
            "d2h_bytes_per_step": h_lb[0].numel() * 4 + h_ver[0].numel(),
            "pipeline": "double-buffered: the H2D of step i+1 and the D2H of step i overlap compute on a "
                        "copy stream; all copies of every step are inside the timed region"}


def graph_leg(args, w, net, centres, C, stream, flush, dev, world, steps, warmup, specs):
    """The same verify call captured once in a CUDA graph (no host synchronisation inside) and replayed."""
    import torch
    from linear_bound_propagation_b200 import vf
    vg = vf.VerifyGraph(net, centres, w.eps, C, crown_relus=w.crown_relus, both_sides=w.both_sides)
    for _ in range(warmup):
        vg.replay()
    torch.cuda.synchronize()
    g_ms = 0.0
    for i in range(steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        vg.replay()
        e1.record(stream)
        e1.synchronize()
        g_ms += e0.elapsed_time(e1)
    g_ms = max_over_ranks(g_ms, dev)
    del vg
    return {"value": weak_throughput(world, specs, steps, g_ms), "unit": UNIT, "ms_per_step": g_ms / steps,
            "note": "vf.VerifyGraph: the verify call captured in a CUDA graph and replayed (no NaN/Inf scan, "
                    "no unstable-neuron compaction)"}


def alpha_leg(args, w, net, centres, C, stream, flush, dev, world, steps):
    """alpha-CROWN: the same workload, intermediate bounds as in verify, then per-row slope optimisation."""
    import torch
    if args.alpha_iters <= 0 or w.both_sides:
        return None
    B, R = w.centres.shape[0], w.C.shape[1]
    net.alpha_crown(centres, w.eps, C, iters=args.alpha_iters, crown_relus=w.crown_relus)  # warm-up
    torch.cuda.synchronize()
    a_ms = 0.0
    for i in range(steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        res = net.alpha_crown(centres, w.eps, C, iters=args.alpha_iters, crown_relus=w.crown_relus)
        e1.record(stream)
        e1.synchronize()
        a_ms += e0.elapsed_time(e1)
    a_ms = max_over_ranks(a_ms, dev)
    gain = (res["lb"] - res["lb_start"])
    out = {"iters": args.alpha_iters, "lr": 0.1, "value": weak_throughput(world, B * R, steps, a_ms),
           "unit": UNIT, "ms_per_step": a_ms / steps, "mean_lb_gain": float(gain.mean().item()),
           "rows_improved": float((gain > 0).float().mean().item()),
           "note": "vf_alpha_crown: intermediate bounds as in the verify step, then per-row lower-slope Adam ascent"}
    if args.alpha_inter_iters > 0:
        kw = dict(crown_relus=w.crown_relus, want_pre=True)
        plain = net.verify(centres, w.eps, C, **kw)
        net.verify(centres, w.eps, C, alpha_inter_iters=args.alpha_inter_iters, **kw)  # warm-up
        torch.cuda.synchronize()
        i_ms = 0.0
        for i in range(steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            ri = net.verify(centres, w.eps, C, alpha_inter_iters=args.alpha_inter_iters, **kw)
            e1.record(stream)
            e1.synchronize()
            i_ms += e0.elapsed_time(e1)
        i_ms = max_over_ranks(i_ms, dev)
        srcs = [nd.src for k, nd in enumerate(w.net) if nd.op == "relu" and
                (w.crown_relus is None or k in w.crown_relus) and k > 2]  # refined ReLUs (the first is exact)
        width = sum((net.node_block(plain["pre_ub"], v, B) - net.node_block(plain["pre_lb"], v, B)).sum().item()
                    for v in srcs)
        width_i = sum((net.node_block(ri["pre_ub"], v, B) - net.node_block(ri["pre_lb"], v, B)).sum().item()
                      for v in srcs)
        out["intermediate"] = {
            "iters": args.alpha_inter_iters, "lr": 0.1, "value": weak_throughput(world, B * R, steps, i_ms),
            "unit": UNIT, "ms_per_step": i_ms / steps,
            "mean_lb_gain": float((ri["lb"] - plain["lb"]).mean().item()),
            "verified_plain": int(plain["verified"].sum().item()), "verified": int(ri["verified"].sum().item()),
            "refined_width_ratio": width_i / width if width else None,
            "note": "vf_verify_batch with vf_opts.alpha_inter_iters: alpha-CROWN on every refined intermediate "
                    "bound (rows [e_j; -e_j] of the neurons still unstable after the CROWN pass), then the plain "
                    "specification pass"}
    return out


def sound_leg(args, w, net, centres, C, out, kw, stream, flush, dev, world, specs):
    """The same verify call with vf_opts.sound (FFMA contractions, rounding budgets)."""
    import torch
    if args.sound_steps <= 0:
        return None
    plain_lb = out["lb"].clone()
    so = {k: torch.empty_like(v) for k, v in out.items()}
    skw = dict(kw, out=so, sound=True)
    net.verify(centres, w.eps, C, **skw)  # warm-up
    torch.cuda.synchronize()
    s_ms = 0.0
    for i in range(args.sound_steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        net.verify(centres, w.eps, C, **skw)
        e1.record(stream)
        e1.synchronize()
        s_ms += e0.elapsed_time(e1)
    s_ms = max_over_ranks(s_ms, dev)
    gap = plain_lb - so["lb"]
    return {"value": weak_throughput(world, specs, args.sound_steps, s_ms), "unit": UNIT,
            "steps": args.sound_steps, "ms_per_step": s_ms / args.sound_steps,
            "lb_below_plain_mean": float(gap.mean().item()), "lb_below_plain_max": float(gap.max().item()),
            "verified_specs": int(so["verified"].sum().item()),
            "note": "vf_verify_batch with vf_opts.sound: directed-rounding IBP, rounded-up intercepts and a "
                    "per-row rounding budget at every node; FFMA contractions"}


def bab_leg(args, w, net, centres, dev, stream, world, rank):
    """Branch and bound (vf_bab_verify) on the workload's network: for the first --bab-centres centres,
    the margin rows of the class the network gives the centre (so the centre is no counterexample), at
    the workload's radius, a budget of --bab-domains subdomains bounded --bab-batch at a time with
    alpha-beta ascent steps. Reports subdomains bounded per second (device-timed, max over ranks)."""
    import torch
    from linear_bound_propagation_b200 import vf
    K = min(args.bab_centres, centres.shape[0])
    lbI, _ = net.ibp(centres[:K].contiguous(), 0.0)
    logits = net.node_block(lbI, len(w.net) - 1, K)
    labels = logits.argmax(dim=1).cpu().numpy()
    nL = logits.shape[1]
    specs = [torch.from_numpy(synth.margin_spec(np.array([y]), nL)[0]).to(dev) for y in labels]
    kw = dict(batch=args.bab_batch, alpha_iters=args.bab_alpha_iters, lr=0.1, crown_relus=w.crown_relus)
    for k in range(K):  # warm-up on every timed problem (a property falsified at once warms nothing else)
        net.bab(centres[k], w.eps, specs[k], max_domains=min(args.bab_batch + 1, args.bab_domains), **kw)
    torch.cuda.synchronize()
    ms, domains, statuses, per_centre = 0.0, 0, [], []
    for k in range(K):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        r = net.bab(centres[k], w.eps, specs[k], max_domains=args.bab_domains, **kw)
        e1.record(stream)
        e1.synchronize()
        ms += e0.elapsed_time(e1)
        domains += r["domains"]
        per_centre.append(int(r["domains"]))
        statuses.append(r["status"])
    ms = max_over_ranks(ms, dev)
    out = {"value": world * domains / (ms / 1e3) if ms > 0 else None, "unit": "subdomains/s", "subdomains": domains,
           "ms": ms, "centres": K, "statuses": statuses, "budget": args.bab_domains, "batch": args.bab_batch,
           "alpha_iters": args.bab_alpha_iters, "eps": w.eps,
           "note": "vf_bab_verify: best-first ReLU-split search; every subdomain bound by vf_verify_batch plus "
                   "alpha-beta ascent, decisions on the device, one host synchronisation per round"}
    # the oracle's timed sample searches the first centre whose device search bounded subdomains (a property
    # falsified at the root bounds none)
    k0 = next((k for k in range(K) if per_centre[k] > 0), 0)
    out["sample_centre"], out["sample_label"] = k0, int(labels[k0])
    return out


def oracle_bab_sample(args, w, k, label):
    """The oracle's search on centre k of the device's branch-and-bound leg (the first whose search bounded
    subdomains), same property, with a small budget (two rounds), timed on the host cores."""
    import oracle.lbp as O
    nL = w.net[-1].W.shape[0]
    budget = min(args.bab_domains, 2 * args.bab_batch + 1)
    C0 = synth.margin_spec(np.array([label]), nL)[0]
    t0 = time.perf_counter()
    o = O.bab(w.net, w.centres[k], w.eps, C0, max_domains=budget, batch=args.bab_batch, iters=args.bab_alpha_iters,
              lr=0.1, crown_relus=w.crown_relus)
    dt = time.perf_counter() - t0
    return {"value": o.domains / dt, "unit": "subdomains/s", "cores": threads_used(), "kind": "oracle",
            "sample": f"centre {k}, budget {budget} subdomains ({o.domains} bounded, {o.status}), {dt:.2f} s"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=5,
                    help="headline workload (5: MLP 3072-1024x8-100, 4096 centres, eps 1/255)")
    ap.add_argument("--no-eps-sweep", dest="eps_sweep", action="store_false",
                    help="skip workload 5 at eps 0.5/255 and 2/255 (reported under eps_sweep)")
    ap.add_argument("--no-all-workloads", dest="all_workloads", action="store_false",
                    help="skip the other four workloads (reported under workloads)")
    ap.add_argument("--sub-steps", type=int, default=5, help="timed steps of each eps_sweep / workloads entry")
    ap.add_argument("--sub-cpu-sample-s", type=float, default=6.0,
                    help="seconds of oracle time behind each workloads entry's cpu_baseline")
    ap.add_argument("--workspace-gb", type=float, default=16.0)
    ap.add_argument("--cpu-sample-s", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--centres", type=int, default=None,
                    help="use only the first N centres of the workload (profiling captures of a small case)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-staged end-to-end leg")
    ap.add_argument("--graph", action="store_true", help="also time the verify call replayed from a CUDA graph")
    ap.add_argument("--alpha-iters", type=int, default=10,
                    help="also time vf_alpha_crown with this many Adam steps (dense chains; 0 = skip)")
    ap.add_argument("--sound-steps", type=int, default=5,
                    help="also time the sound-in-fp32 verify call for this many steps (0 = skip)")
    ap.add_argument("--bab-domains", type=int, default=512,
                    help="also time vf_bab_verify with this budget of subdomains per centre (0 = skip)")
    ap.add_argument("--alpha-inter-iters", type=int, default=5,
                    help="Adam steps of the intermediate-bound alpha leg (0: skip it)")
    ap.add_argument("--bab-centres", type=int, default=2)
    ap.add_argument("--bab-batch", type=int, default=64)
    ap.add_argument("--bab-alpha-iters", type=int, default=10)
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
