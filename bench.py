#!/usr/bin/env python
"""Benchmark of the linear-memory relation-KL path (LinearARD, Phase 1 + Phase 2).

One step = forward (Phase 1) and backward (Phase 2) of the Q/Q, K/K and V/V
self-relations of one batch of synthetic RoPE-shaped projections, through
the C ABI (liblard.so).  Default workload: B=1, H=32, n=32768, d=128, bf16.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lard|reference]

Under torchrun (N > 1) every rank runs the same per-GPU workload on its own
batch (weak scaling); the relations of different ranks share nothing, so the
timed region holds no collective.  Rank 0 prints one JSON line.
"""
import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "fused KL fwd+bwd causal logits/s at n=32K; % of B200 bf16 tensor peak"
UNIT = "causal logits/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["lard", "reference"], default="lard")
    ap.add_argument("--workload", default="n32768",
                    help="one of: n32768 (default), n16384, n4096, gqa-n8000, fp32-small")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-mask", action="store_true",
                    help="bidirectional relation maps (every logit allowed); metric then counts n*n logits")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="approximate CPU time of the oracle sample")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 200 ms during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.tmp = None

    def start(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.index)], stdout=self.tmp, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        self.tmp.seek(0)
        rows = [ln.strip().split(",") for ln in self.tmp.read().splitlines() if ln.strip()]
        self.tmp.close()
        os.unlink(self.tmp.name)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
                for name, val in zip(names, r[5:9]):
                    if val.strip() == "Active":
                        reasons.add(name)
            except (ValueError, IndexError):
                continue
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm)}


def oracle_sample(w, host, seconds, rank_seed=0):
    """Time the fp64 oracle on the last R rows of head (0, 0) of every relation.

    R is sized from a short probe so that the sample costs about `seconds`.
    Returns (causal logits processed, elapsed seconds, R, threads)."""
    import oracle
    from linear_memory_attention_b200 import synth
    orc = oracle.default()
    f64 = {rel: (synth.as_f64(xt[0, 0]), synth.as_f64(xs[0, 0])) for rel, (xt, xs) in host.items()}
    n = w.n
    probe = min(8, n)
    t0 = time.perf_counter()
    xt, xs = f64[w.relations[0]]
    orc.rows(xt, xt, xs, xs, w.tau, w.causal, n - probe, n, want_dY=True)
    per_row = (time.perf_counter() - t0) / probe
    R = int(max(1, min(n, seconds / (per_row * len(w.relations)))))
    logits = 0
    t0 = time.perf_counter()
    for rel in w.relations:
        xt, xs = f64[rel]
        orc.rows(xt, xt, xs, xs, w.tau, w.causal, n - R, n, want_dY=True)
        logits += sum((i + 1) if w.causal else n for i in range(n - R, n))
    return logits, time.perf_counter() - t0, R, orc.num_threads()


def run_reference(args):
    """The oracle, as it stands, on the host cores (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from linear_memory_attention_b200 import synth
    w = synth.WORKLOADS[args.workload]
    if args.no_mask:
        w = dataclasses.replace(w, name=w.name + " no-mask", causal=False)
    unit = UNIT if w.causal else "logits/s (no mask)"
    metric = METRIC if w.causal else METRIC + " (no mask: every logit allowed)"
    host = synth.make_all(w)
    per_step = max(1.0, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(w, host, per_step)
    logits = 0
    elapsed = 0.0
    R = threads = 0
    for _ in range(args.steps):
        lg, dt, R, threads = oracle_sample(w, host, per_step)
        logits += lg
        elapsed += dt
    value = logits / elapsed
    sample = (f"per step: rows [n-{R}, n) of head (0,0) of each of {len(w.relations)} relations "
              f"({logits // max(1, args.steps)} causal logits), fp64 explicit maps")
    print(json.dumps({
        "impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * elapsed / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": w.name, "B": w.B, "heads": w.heads, "n": w.n,
                                        "d": w.d, "causal": w.causal},
        "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_lard(args):
    import torch
    import torch.distributed as dist
    from linear_memory_attention_b200 import lard, synth

    from linear_memory_attention_b200 import dist as ldist

    rank, world, local = ldist.env_ranks()
    torch.cuda.set_device(local)
    ldist.init("nccl", device=torch.device("cuda", local))
    w = synth.WORKLOADS[args.workload]
    if args.no_mask:
        w = dataclasses.replace(w, name=w.name + " no-mask", causal=False)
    unit = UNIT if w.causal else "logits/s (no mask)"
    metric = METRIC if w.causal else METRIC + " (no mask: every logit allowed)"
    wr = ldist.rank_workload(w, rank)  # each rank: its own batch
    host = synth.make_all(wr)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    f32 = dict(device=dev, dtype=torch.float32)
    B, n, d = w.B, w.n, w.d
    R = len(w.relations)
    # Two device copies of the inputs: the timed leg uses the first; the
    # end-to-end leg alternates, so one step's host copies fill one set while
    # the previous step computes on the other.
    X = [{r: (xt.to(dev), xs.to(dev)) for r, (xt, xs) in host.items()} for _ in range(2)]
    O = {}
    for r in w.relations:
        H = w.heads[r]
        O[r] = dict(lse_t=torch.empty((B, H, n), **f32), lse_s=torch.empty((B, H, n), **f32),
                    row_kl=torch.empty((B, H, n), **f32), loss_bh=torch.empty((B * H,), **f32),
                    dXs=torch.empty((B, H, n, d), **f32), dYs=torch.empty((B, H, n, d), **f32))
    loss = torch.empty((1,), **f32)  # the summed loss of the step's relations
    rels = [[dict(Xt=X[k][r][0], Xs=X[k][r][1], **O[r]) for r in w.relations] for k in range(2)]

    def step(ev=None, k=0):
        # One launch per phase for all relations (lard_kl_fwd_multi / _bwd_multi).
        if ev is not None:
            ev[0].record(stream)
        lard.lard_kl_fwd_multi(rels[k], w.tau, w.causal, loss, stream)
        if ev is not None:
            ev[1].record(stream)
        lard.lard_kl_bwd_multi(rels[k], w.tau, w.causal, 1.0, stream)
        if ev is not None:
            ev[2].record(stream)

    # Kernel launches per step: the bf16 path runs one Phase 1, one loss-rows,
    # one loss-total and one Phase 2 kernel for all relations; the fp32 path
    # runs Phase 1 per relation and three Phase 2 kernels per relation.
    launches_per_step = 4 if w.dtype == "bf16" else R + 2 + 3 * R

    def barrier():
        if world > 1:
            dist.barrier()

    # Device memory taken outside the caller's buffers: once on first use (the
    # CUDA runtime loading the library's kernels), and per step after that (the
    # library itself allocates nothing, so this should stay 0).
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info(dev)[0]
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info(dev)[0]
    step()
    torch.cuda.synchronize()
    free2 = torch.cuda.mem_get_info(dev)[0]
    lard.lard_device_status()
    # HBM state kept between the phases: LSE_t, LSE_s and row KL, 12 bytes per row.
    rows_total = sum(w.B * w.heads[r] * n for r in w.relations)
    extra_hbm = {"state_bytes": 12 * rows_total, "per_row_bytes": 12,
                 "allocated_per_step_bytes": int(free1 - free2),
                 "first_use_bytes": int(free0 - free1),
                 "explicit_maps_bytes": 2 * 4 * sum(w.B * w.heads[r] * n * n for r in w.relations),
                 "note": "state = lse_t, lse_s, row_kl (fp32, O(BHn)); explicit maps = the fp32 R_t and "
                         "R_s that a materialising implementation would hold"}

    # ---------------------------------------------------------------- device-resident leg
    K = args.steps
    mk = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    evs = [(mk(), mk(), mk()) for _ in range(K)]
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    t_start, t_end = mk(), mk()
    t_start.record(stream)
    for k in range(K):
        step(evs[k])
    t_end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier()
    lard.lard_device_status()
    elapsed_ms = t_start.elapsed_time(t_end)
    fwd_ms = [e[0].elapsed_time(e[1]) for e in evs]
    bwd_ms = [e[1].elapsed_time(e[2]) for e in evs]
    elapsed_ms = ldist.max_over_ranks(elapsed_ms, device=dev)
    logits_step = w.causal_logits()
    value = ldist.aggregate_rate(logits_step, K, world, elapsed_ms)

    # ---------------------------------------------------------------- end to end (host buffers)
    e2e = None
    if not args.no_e2e:
        pinned = {r: (xt.pin_memory(), xs.pin_memory()) for r, (xt, xs) in host.items()}
        loss_host = torch.empty((1,), dtype=torch.float32).pin_memory()
        h2d = sum(xt.numel() * xt.element_size() + xs.numel() * xs.element_size()
                  for xt, xs in pinned.values())
        d2h = loss_host.numel() * loss_host.element_size()

        # Every step copies all its inputs from pinned host memory into one of
        # the two device sets (on a copy stream, once the set's previous step has
        # finished with it), runs both phases on that set, and reads the summed
        # loss back.  So the copies of step k + 1 overlap the kernels of step k.
        copy_stream = torch.cuda.Stream(device=dev)
        released = [mk(), mk()]
        copied = [mk(), mk()]
        for ev in released:
            ev.record(stream)
        counter = [0]

        def e2e_step():
            k = counter[0] % 2
            counter[0] += 1
            copy_stream.wait_event(released[k])
            with torch.cuda.stream(copy_stream):
                for r in w.relations:
                    X[k][r][0].copy_(pinned[r][0], non_blocking=True)
                    X[k][r][1].copy_(pinned[r][1], non_blocking=True)
            copied[k].record(copy_stream)
            stream.wait_event(copied[k])
            step(k=k)
            released[k].record(stream)
            loss_host.copy_(loss, non_blocking=True)

        for _ in range(min(2, args.warmup)):
            e2e_step()
        barrier()
        torch.cuda.synchronize()
        a, b = mk(), mk()
        a.record(stream)
        copy_stream.wait_event(a)  # no copy of the timed steps starts before the region opens
        for _ in range(K):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = ldist.max_over_ranks(a.elapsed_time(b), device=dev)
        e2e = {"value": ldist.aggregate_rate(logits_step, K, world, e2e_ms), "unit": unit,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e2e_ms / K}

    # ---------------------------------------------------------------- roofline of the dominant kernel
    peaks, peak_src = load_peaks()
    dom, dom_ms = ("bwd", bwd_ms) if sum(bwd_ms) >= sum(fwd_ms) else ("fwd", fwd_ms)
    gemms = 4 if dom == "bwd" else 2
    per_launch_flops = sum(2 * gemms * d * w.B * w.heads[r] * (n * (n + 1) // 2 if w.causal else n * n)
                           for r in w.relations)
    ach = statistics.mean(per_launch_flops / (ms / 1e3) for ms in dom_ms) / 1e12
    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    step_tflops = w.algorithmic_flops() * K / (elapsed_ms / 1e3) / 1e12  # per rank
    traffic, traffic_basis = _profiled_traffic(f"lard_{dom}_tc_kernel<{d}>", w)
    # Phase 1 against the exponential unit: 2 exponentials per logit (teacher and
    # student), MUFU at 16 per clock per SM on 148 SMs, at the median SM clock
    # sampled during the timed region (a fraction of the polynomial share is on
    # the FMA pipe, so the fraction can pass 1 in principle).
    exps_per_launch = 2 * logits_step
    mufu_peak = 16 * 148 * clk["sm_mhz"] * 1e6 if clk.get("sm_mhz") else None
    mufu_ach = exps_per_launch / (statistics.mean(fwd_ms) / 1e3)
    # Phase 2 against shared-memory bandwidth, which binds it: per 128 x 128 tile
    # the four SS GEMMs read 256 KB of operands (at d = 128), TMA writes 64 KB of
    # X_t / X_s, the dZ warps store 32 KB, and the dX staging is written and read
    # (128 KB); 128 bytes per clock per SM.
    T = -(-n // 128)
    tiles = sum(w.B * w.heads[r] for r in w.relations) * (T * (T + 1) // 2 if w.causal else T * T)
    smem_per_tile = (256 + 64 + 32 + 128) * 1024 * d // 128
    smem_peak = 128 * 148 * clk["sm_mhz"] * 1e6 if clk.get("sm_mhz") else None
    smem_ach = tiles * smem_per_tile / (statistics.mean(bwd_ms) / 1e3)
    phase2_smem = {"kernel": f"lard_bwd_tc_kernel<{d}>", "bound": "shared-memory bandwidth",
                   "achieved": smem_ach / 1e9, "peak": smem_peak / 1e9 if smem_peak else None,
                   "unit": "GB/s", "frac": (smem_ach / smem_peak) if smem_peak else None,
                   "bytes_per_tile": smem_per_tile, "tiles_per_launch": tiles,
                   "basis": "modelled bytes per 128x128 tile (MMA operand reads 256 KB, TMA writes 64 KB, "
                            "dZ stores 32 KB, dX staging 128 KB at d = 128) over 128 B/clk/SM x 148 SMs "
                            "x median sampled SM clock"}
    phase1_mufu = {"kernel": f"lard_fwd_tc_kernel<{d}>", "bound": "alu (MUFU exponentials)",
                   "achieved": mufu_ach, "peak": mufu_peak, "unit": "exp2/s",
                   "frac": (mufu_ach / mufu_peak) if mufu_peak else None,
                   "peak_basis": "16 per clock per SM x 148 SMs x median sampled SM clock"}

    if rank == 0:
        out = {
            "metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": elapsed_ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "fp32",
            "data": "synthetic (seeded RoPE-shaped Q/K, Gaussian V; no weights or text)",
            "config": {"workload": w.name, "B": w.B, "heads": w.heads, "n": w.n, "d": w.d,
                       "relations": list(w.relations), "causal": w.causal,
                       "l2": "inputs larger than L2 (%d MB per tensor), no flush" %
                             (w.B * max(w.heads.values()) * n * d * 2 // 2**20),
                       "parallelism": f"dp{world} (independent batches per GPU)"},
            "tflops": step_tflops * world,
            "frac_of_bf16_peak": {"sustained": step_tflops / peak, "burst": step_tflops / burst,
                                  "source": peak_src},
            "roofline": {"kernel": f"lard_{dom}_tc_kernel<{d}>", "bound": "tensor",
                         "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
                         "peak_kind": f"bf16 dense, sustained ({peak_src})",
                         "frac_of_burst_peak": ach / burst, "traffic": traffic,
                         "traffic_basis": traffic_basis},
            "phase1_roofline": phase1_mufu if w.dtype == "bf16" else None,
            "phase2_smem_roofline": phase2_smem if w.dtype == "bf16" else None,
            "kernel_ms": {"fwd": statistics.mean(fwd_ms), "bwd": statistics.mean(bwd_ms),
                          "relations_per_launch": R if w.dtype == "bf16" else 1},
            "clocks": clk,
            "gpu_launches": launches_per_step * K,
            "extra_hbm": extra_hbm,
            "e2e": e2e,
        }
        if world == 1 and not args.no_cpu_baseline:
            lg, dt, R, thr = oracle_sample(w, host, args.cpu_seconds)
            out["cpu_baseline"] = {
                "value": lg / dt, "unit": unit, "cores": thr, "kind": "oracle",
                "sample": f"rows [n-{R}, n) of head (0,0) of each of {len(w.relations)} relations, "
                          f"{lg} causal logits in {dt:.1f} s, fp64 explicit maps"}
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def _profiled_traffic(kernel, w):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary for this workload, if one exists and was taken on the current
    kernel sources (else None: the counters no longer describe this kernel)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            tab = json.load(f)
        ent = tab[f"{kernel}:{w.name}"]
        from linear_memory_attention_b200 import build
        if ent.get("source_digest") != build.source_digest():
            return None, "kernel changed since the counters were taken"
        return ent["bytes_per_launch"], ent.get("basis")
    except (OSError, ValueError, KeyError, AttributeError):
        return None, "no capture for this kernel and workload"


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_lard(args)


if __name__ == "__main__":
    main()
