#!/usr/bin/env python
"""Benchmark of the linear-memory relation-KL path (LinearARD, Phase 1 + Phase 2).

One step = forward (Phase 1) and backward (Phase 2) of the Q/Q, K/K and V/V
self-relations of one batch of synthetic RoPE-shaped projections, through
the C ABI (liblard.so): the summed loss and each relation's student gradient
dL/dX_s (for a self-relation the sum of the two partials, formed in the
kernel), written as bf16.  Default workload: B=1, H=32, n=32768, d=128, bf16.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lard|reference]

Under torchrun (N > 1), by default every rank runs the same per-GPU workload
on its own batch (weak scaling; the timed region holds no collective).  With
--scaling strong the ranks split ONE workload's (relation, batch, head) units
into contiguous equal slices and all-reduce the summed loss (NCCL), the only
exchange.  Rank 0 prints one JSON line.
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
    ap.add_argument("--scaling", choices=["weak", "strong"], default="weak",
                    help="weak: every rank runs its own batch; strong: the ranks split one job's "
                         "(relation, b, h) units and all-reduce the loss")
    ap.add_argument("--grads", choices=["dq-bf16", "dq", "partials", "partials-bf16"], default="dq-bf16",
                    help="dq: the self-relation gradient dL/dX_s = dX_s + dY_s, fused in the kernel; "
                         "partials: dX_s and dY_s apart; -bf16: written as bf16 (fp32 accumulation, "
                         "rounded once), else fp32.  Default dq-bf16: what a bf16 training step consumes")
    ap.add_argument("--no-probe", action="store_true", help="skip the exponential-unit probe")
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
        if not rows:
            # A region shorter than the sampling period: one sample right after it.
            try:
                q = subprocess.run(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                    "-i", str(self.index)], capture_output=True, text=True, timeout=20)
                rows = [ln.strip().split(",") for ln in q.stdout.splitlines() if ln.strip()]
            except (OSError, subprocess.TimeoutExpired):
                rows = []
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
    xt, xs = f64[w.relations[0]]
    orc.rows(xt, xt, xs, xs, w.tau, w.causal, n - min(8, n), n, want_dY=True)  # threads and pages warm
    probe = min(32, n)
    t0 = time.perf_counter()
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
        "higher_is_better": True, "scaling": args.scaling, "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": w.name, "B": w.B, "heads": w.heads, "n": w.n,
                                        "d": w.d, "relations": list(w.relations), "causal": w.causal,
                                        "gradients": "dX_s and dY_s of the sampled rows, fp64",
                                        "parallelism": "rank 0 only, host cores"},
        "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def _tiles(w, units):
    """128 x 128 tiles one launch of a phase visits over ``units`` heads."""
    T = -(-w.n // 128)
    return units * (T * (T + 1) // 2 if w.causal else T * T)


def measure_exp_unit(dev, seconds=1.0):
    """The exponential rate of this GPU, measured with the probe library: MUFU
    ex2.approx (the unit Phase 1 is bound by) and, for reference, the FMA-pipe
    polynomial the kernels put part of the exponentials on.  Returns per-clock
    per-SM rates from the median SM clock sampled while the probe ran."""
    import torch
    from linear_memory_attention_b200 import probe
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    out = {}
    for kind in ("ex2_f32", "exp2_fma_pair"):
        blocks = sms * 8
        probe.exp_rate(kind, blocks, 64)                      # warm-up
        ms, _ = probe.exp_rate(kind, blocks, 1024)
        iters = max(64, int(1024 * (seconds / 4) / max(ms / 1e3, 1e-6)))
        clocks = ClockSampler(dev.index if dev.index is not None else 0)
        clocks.start()
        t_ms, t_exps = 0.0, 0.0
        for _ in range(4):
            ms, ex = probe.exp_rate(kind, blocks, iters)
            t_ms += ms
            t_exps += ex
        clk = clocks.stop()
        rate = t_exps / (t_ms / 1e3)
        mhz = clk.get("sm_mhz")
        out[kind] = {"per_s": rate, "sm_mhz": mhz,
                     "per_clk_per_sm": rate / (sms * mhz * 1e6) if mhz else None}
    out["sms"] = sms
    return out


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
    strong = args.scaling == "strong"
    fused = args.grads.startswith("dq")
    g16 = args.grads.endswith("-bf16")
    if (fused or g16) and w.dtype != "bf16":
        raise SystemExit(f"--grads {args.grads} needs bf16 inputs (the fp32 path returns fp32 partials)")
    gdt = torch.bfloat16 if g16 else torch.float32
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    f32 = dict(device=dev, dtype=torch.float32)
    B, n, d = w.B, w.n, w.d
    if strong:
        # One job: this rank's contiguous slice of the workload's (relation, b, h) units.
        host_all = synth.make_all(w)
        slices = ldist.rank_slices(w, world, rank)
        host = {r: tuple(ldist.slice_heads(t, lo, hi).contiguous() for t in host_all[r])
                for r, lo, hi in slices}
        del host_all
    else:
        host = synth.make_all(ldist.rank_workload(w, rank))  # each rank: its own batch
    rels_run = list(host)
    units_rank = sum(t[0].shape[0] * t[0].shape[1] for t in host.values())
    per_unit_logits = n * (n + 1) // 2 if w.causal else n * n
    logits_rank = units_rank * per_unit_logits
    logits_job = w.causal_logits() if strong else w.causal_logits() * world
    R = len(rels_run)

    # Caller-owned HBM state kept between the phases (lse_t, lse_s, row_kl per
    # row, loss_bh per head), measured as the device memory its allocation takes.
    torch.cuda.synchronize()
    m0 = torch.cuda.memory_allocated(dev)
    O = {}
    for r in rels_run:
        Bh, H = host[r][0].shape[:2]
        O[r] = dict(lse_t=torch.empty((Bh, H, n), **f32), lse_s=torch.empty((Bh, H, n), **f32),
                    row_kl=torch.empty((Bh, H, n), **f32), loss_bh=torch.empty((Bh * H,), **f32))
    state_bytes = torch.cuda.memory_allocated(dev) - m0
    for r in rels_run:
        Bh, H = host[r][0].shape[:2]
        O[r]["dXs"] = torch.empty((Bh, H, n, d), device=dev, dtype=gdt)
        if not fused:
            O[r]["dYs"] = torch.empty((Bh, H, n, d), device=dev, dtype=gdt)
    grad_keys = ("dXs",) if fused else ("dXs", "dYs")
    loss = torch.zeros((1,), **f32)  # the summed loss of the step's relations (the job's, after the all-reduce)
    # Two device copies of the inputs: the timed leg uses the first; the
    # end-to-end leg alternates, so one step's host copies fill one set while
    # the previous step computes on the other.
    X = [{r: (xt.to(dev), xs.to(dev)) for r, (xt, xs) in host.items()} for _ in range(2)]
    rels = [[dict(Xt=X[k][r][0], Xs=X[k][r][1], **O[r]) for r in rels_run] for k in range(2)]
    # bf16 gradient outputs: the caller-owned fp32 accumulation workspace of the call
    ws = (torch.empty((lard.lard_kl_bwd_bf16_workspace_bytes(rels[0]),), device=dev, dtype=torch.uint8)
          if (g16 and rels_run) else None)

    def step(ev=None, k=0, outs=None):
        # One launch per phase for all relations (lard_kl_fwd_multi / _bwd_multi);
        # when the ranks split one job, one all-reduce of the loss scalar.
        rk = rels[k] if outs is None else [dict(rr, **oo) for rr, oo in zip(rels[k], outs)]
        if ev is not None:
            ev[0].record(stream)
        if rk:
            lard.lard_kl_fwd_multi(rk, w.tau, w.causal, loss, stream)
        else:
            loss.zero_()
        if ev is not None:
            ev[1].record(stream)
        if rk and g16:
            lard.lard_kl_bwd_multi_bf16(rk, w.tau, w.causal, 1.0, ws, stream)
        elif rk:
            lard.lard_kl_bwd_multi(rk, w.tau, w.causal, 1.0, stream)
        if ev is not None:
            ev[2].record(stream)
        if strong:
            ldist.all_reduce_loss(loss)

    # Kernel launches per step: the bf16 path runs one Phase 1, one loss-rows,
    # one loss-total and one Phase 2 kernel for all relations (and, with bf16
    # gradient outputs, one rounding pass); the fp32 path runs Phase 1 per
    # relation and three Phase 2 kernels per relation.
    launches_per_step = ((5 if g16 else 4) if w.dtype == "bf16" else R + 2 + 3 * R) if R else 0

    def barrier():
        if world > 1:
            dist.barrier()

    # Device memory taken outside the caller's buffers: once on first use (the
    # CUDA runtime loading the library's kernels), and per step after that: the
    # torch allocator's peak above the caller's buffers and the driver-level
    # free memory, which would show a cudaMalloc inside the library.
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info(dev)[0]
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info(dev)[0]
    torch.cuda.reset_peak_memory_stats(dev)
    alloc1 = torch.cuda.memory_allocated(dev)
    step()
    torch.cuda.synchronize()
    free2 = torch.cuda.mem_get_info(dev)[0]
    peak_above = torch.cuda.max_memory_allocated(dev) - alloc1
    lard.lard_device_status()
    rows_rank = units_rank * n
    extra_hbm = {"state_bytes": int(state_bytes), "state_bytes_expected": 12 * rows_rank + 4 * units_rank,
                 "per_row_bytes": 12, "rows": rows_rank,
                 "allocated_per_step_bytes": int(free1 - free2), "torch_peak_above_buffers_bytes": int(peak_above),
                 "first_use_bytes": int(free0 - free1),
                 "explicit_maps_bytes": 2 * 4 * units_rank * n * n,
                 "note": "state = lse_t, lse_s, row_kl (fp32, O(BHn)) and loss_bh, measured as the "
                         "allocator's growth when the caller allocates them; per step = driver-level free "
                         "memory lost across one step (a library cudaMalloc would show there) and the torch "
                         "allocator's peak above the resident buffers; explicit maps = the fp32 R_t and R_s "
                         "that a materialising implementation would hold"}

    # ---------------------------------------------------------------- exponential unit (probe)
    exp_unit = measure_exp_unit(dev) if (w.dtype == "bf16" and not args.no_probe) else None

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
    value = ldist.job_rate(logits_job, K, elapsed_ms)

    # A timed region shorter than the sampler's period yields at most one sample,
    # taken after it, at the idle clock.  The per-clock figures then use the
    # clock sampled while more untimed steps run for about a second.
    # (The decision and the step count follow from the max-over-ranks time, so every
    # rank runs the same steps, and the same collectives in strong scaling.)
    clk_load = clk
    if elapsed_ms < 1000.0:
        per_step = max(elapsed_ms / K, 1e-3)
        extra = int(min(2000, max(1, 1500.0 / per_step)))
        sampler = ClockSampler(local)
        sampler.start()
        for _ in range(extra):
            step()
        torch.cuda.synchronize()
        clk_load = sampler.stop()
        clk = dict(clk, sm_mhz_under_load=clk_load.get("sm_mhz"),
                   note="timed region under a second: sm_mhz from the few samples taken in or "
                        "right after it; sm_mhz_under_load sampled over further untimed steps "
                        "(used for the per-clock figures)")

    # ---------------------------------------------------------------- end to end (host buffers)
    e2e = None
    if not args.no_e2e and R:
        e2e = _e2e_leg(args, w, host, X, O, grad_keys, loss, step, stream, dev, world, K, logits_job,
                       unit, barrier, mk)

    # ---------------------------------------------------------------- rooflines
    peaks, peak_src = load_peaks()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mhz = clk_load.get("sm_mhz")
    dom, dom_ms = ("bwd", bwd_ms) if sum(bwd_ms) >= sum(fwd_ms) else ("fwd", fwd_ms)
    gemms = 4 if dom == "bwd" else 2
    per_launch_flops = 2 * gemms * d * logits_rank
    ach = statistics.mean(per_launch_flops / (ms / 1e3) for ms in dom_ms) / 1e12 if R else 0.0
    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    step_tflops = 12 * d * logits_rank * K / (elapsed_ms / 1e3) / 1e12  # per rank
    traffic, traffic_basis = _profiled_traffic(f"lard_{dom}_tc_kernel<{d}>", w,
                                               args.grads if dom == "bwd" else "partials")
    # Algorithmic DRAM bytes of one launch of the dominant kernel: the distinct input
    # tensors once (self-relations: X_t and X_s; Y aliases X), plus for Phase 2 the
    # fp32 gradient accumulators written once (dX_s, and dY_s unless fused), plus for
    # Phase 1 the 12 bytes of state per row.
    in_bytes = sum(t.numel() * t.element_size() for xt, xs in host.values() for t in (xt, xs))
    grad_elems = units_rank * n * d
    algo_bytes = (in_bytes + grad_elems * 4 * (1 if fused else 2)) if dom == "bwd" else \
        (in_bytes + 12 * units_rank * n)
    tiles = _tiles(w, units_rank)
    # Cycles per 128 x 128 tile on one SM, from the kernel's time and the median
    # SM clock sampled during the timed region: comparable across clocks (the
    # sustained peak was measured at another clock than this run's).  The tensor
    # pipe alone needs 64 cycles per K = 16 step of a 128 x 128 MMA.
    ideal = {"fwd": 2 * (d // 16) * 64, "bwd": 4 * (d // 16) * 64}

    def cyc(ms_list):
        if not (mhz and tiles):
            return None
        return statistics.mean(ms_list) / 1e3 * mhz * 1e6 / (tiles / sms)

    cyc_fwd, cyc_bwd = cyc(fwd_ms), cyc(bwd_ms)
    # Phase 1 against the exponential unit: 2 exponentials per logit (teacher and
    # student) over the probe's measured MUFU rate per clock, at this run's
    # median clock (1/8 of the exponentials run on the FMA pipe, so the
    # fraction can reach 8/7).
    exps_per_launch = 2 * logits_rank
    mufu_clk = exp_unit["ex2_f32"]["per_clk_per_sm"] if exp_unit else None
    mufu_peak = mufu_clk * sms * mhz * 1e6 if (mufu_clk and mhz) else None
    mufu_ach = exps_per_launch / (statistics.mean(fwd_ms) / 1e3) if R else 0.0
    # Phase 2 against shared-memory bandwidth, which binds it: per 128 x 128 tile
    # the four SS GEMMs read 256 KB of operands (at d = 128), TMA writes 64 KB of
    # X_t / X_s, the dZ warps store 32 KB, and the dX staging is written and read
    # (128 KB); 128 bytes per clock per SM.
    smem_per_tile = (256 + 64 + 32 + 128) * 1024 * d // 128
    smem_peak = 128 * sms * mhz * 1e6 if mhz else None
    smem_ach = tiles * smem_per_tile / (statistics.mean(bwd_ms) / 1e3) if R else 0.0
    phase2_smem = {"kernel": f"lard_bwd_tc_kernel<{d}>", "bound": "shared-memory bandwidth",
                   "achieved": smem_ach / 1e9, "peak": smem_peak / 1e9 if smem_peak else None,
                   "unit": "GB/s", "frac": (smem_ach / smem_peak) if smem_peak else None,
                   "bytes_per_tile": smem_per_tile, "tiles_per_launch": tiles,
                   "basis": "modelled bytes per 128x128 tile (MMA operand reads 256 KB, TMA writes 64 KB, "
                            "dZ stores 32 KB, dX staging 128 KB at d = 128) over 128 B/clk/SM x SMs "
                            "x median sampled SM clock"}
    phase1_mufu = {"kernel": f"lard_fwd_tc_kernel<{d}>", "bound": "alu", "unit": "exp2/s",
                   "achieved": mufu_ach, "peak": mufu_peak,
                   "frac": (mufu_ach / mufu_peak) if mufu_peak else None,
                   "peak_basis": "MUFU ex2.approx rate per clock per SM measured by the probe "
                                 "(liblard_probe.so) x SMs x this run's median SM clock",
                   "measured_ex2_per_clk_per_sm": mufu_clk,
                   "cycles_per_tile": cyc_fwd, "mufu_cycles_per_tile": (2 * 128 * 128 / mufu_clk) if mufu_clk else None}

    if rank == 0:
        out = {
            "metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": elapsed_ms / K, "higher_is_better": True,
            "scaling": "strong" if strong else "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "fp32",
            "data": "synthetic (seeded RoPE-shaped Q/K, Gaussian V; no weights or text)",
            "config": {"workload": w.name, "B": w.B, "heads": w.heads, "n": w.n, "d": w.d,
                       "relations": list(w.relations), "causal": w.causal,
                       "gradients": ("fused dQ = dX_s + dY_s" if fused else "dX_s and dY_s") +
                                    (", bf16 (fp32 accumulation, rounded once)" if g16 else ", fp32"),
                       "l2": "inputs larger than L2 (%d MB per tensor), no flush" %
                             (w.B * max(w.heads.values()) * n * d * 2 // 2**20),
                       "parallelism": (f"units{world} (one job's (relation, b, h) units split across "
                                       "GPUs; loss all-reduced)") if strong else
                                      f"dp{world} (independent batches per GPU)"},
            "tflops": step_tflops * world,
            "frac_of_bf16_peak": {"sustained": step_tflops / peak, "burst": step_tflops / burst,
                                  "source": peak_src,
                                  "datasheet_2250": step_tflops / 2250.0},
            "roofline": {"kernel": f"lard_{dom}_tc_kernel<{d}>", "bound": "tensor",
                         "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
                         "peak_kind": f"bf16 dense, sustained ({peak_src})",
                         "frac_of_burst_peak": ach / burst, "traffic": traffic,
                         "traffic_basis": traffic_basis, "algorithmic_bytes": algo_bytes,
                         "cycles_per_tile": cyc_bwd if dom == "bwd" else cyc_fwd,
                         "tensor_cycles_per_tile": ideal[dom],
                         "frac_per_clock": (ideal[dom] / (cyc_bwd if dom == "bwd" else cyc_fwd))
                         if (cyc_bwd and cyc_fwd) else None},
            "phase1_roofline": phase1_mufu if w.dtype == "bf16" else None,
            "phase2_smem_roofline": phase2_smem if w.dtype == "bf16" else None,
            "kernel_ms": {"fwd": statistics.mean(fwd_ms) if R else 0.0,
                          "bwd": statistics.mean(bwd_ms) if R else 0.0,
                          "fwd_cycles_per_tile": cyc_fwd, "bwd_cycles_per_tile": cyc_bwd,
                          "tiles_per_launch": tiles,
                          "relations_per_launch": R if w.dtype == "bf16" else 1},
            "exp_unit": exp_unit,
            "clocks": clk,
            "gpu_launches": launches_per_step * K,
            "extra_hbm": extra_hbm,
            "e2e": e2e,
        }
        if world == 1 and not args.no_cpu_baseline:
            lg, dt, Rr, thr = oracle_sample(w, host, args.cpu_seconds)
            # The oracle builds explicit maps (every column of every row it is asked
            # about), so its time grows with the explicit logits; the whole
            # workload's oracle time is estimated from the sample's rate.
            explicit_sample = len(w.relations) * Rr * n
            explicit_all = units_rank * n * n
            out["cpu_baseline"] = {
                "value": lg / dt, "unit": unit, "cores": thr, "kind": "oracle",
                "sample": f"rows [n-{Rr}, n) of head (0,0) of each of {len(w.relations)} relations, "
                          f"{lg} causal logits in {dt:.1f} s, fp64 explicit maps",
                "whole_workload_estimate_s": dt * explicit_all / explicit_sample}
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def _e2e_leg(args, w, host, X, O, grad_keys, loss, step, stream, dev, world, K, logits_job, unit,
             barrier, mk):
    """The same step through the public calls with host buffers: every step
    copies its inputs from pinned host memory and reads its gradients and loss
    back into pinned host memory, inside the timed region.

    Two device sets (inputs and gradient outputs) alternate.  Step k's input
    copies run on an upload stream once the set's previous step has finished
    computing; its kernels run once they have landed and the set's previous
    gradients have been read out; its read-back runs on a download stream once
    its kernels are done.  So uploads, kernels and downloads of neighbouring
    steps overlap, and the timed region ends when the last download lands."""
    import torch
    from linear_memory_attention_b200 import dist as ldist
    pinned = {r: (xt.pin_memory(), xs.pin_memory()) for r, (xt, xs) in host.items()}
    # device gradient buffers: set 0 are the step's own (O), set 1 a second copy
    outs = [[{g: O[r][g] for g in grad_keys} for r in host],
            [{g: torch.empty_like(O[r][g]) for g in grad_keys} for r in host]]
    grads_host = [{g: torch.empty(O[r][g].shape, dtype=O[r][g].dtype).pin_memory() for g in grad_keys}
                  for r in host]
    loss_host = torch.empty((1,), dtype=torch.float32).pin_memory()
    h2d = sum(xt.numel() * xt.element_size() + xs.numel() * xs.element_size() for xt, xs in pinned.values())
    d2h = loss_host.numel() * loss_host.element_size() + sum(
        t.numel() * t.element_size() for gh in grads_host for t in gh.values())
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    computed = [mk(), mk()]
    copied = [mk(), mk()]
    read = [mk(), mk()]
    for ev in computed + read:
        ev.record(stream)
    counter = [0]

    def e2e_step():
        k = counter[0] % 2
        counter[0] += 1
        up.wait_event(computed[k])          # the set's previous step no longer reads its inputs
        with torch.cuda.stream(up):
            for r in host:
                X[k][r][0].copy_(pinned[r][0], non_blocking=True)
                X[k][r][1].copy_(pinned[r][1], non_blocking=True)
        copied[k].record(up)
        stream.wait_event(copied[k])
        stream.wait_event(read[k])          # the set's previous gradients have been read out
        step(k=k, outs=outs[k])
        computed[k].record(stream)
        down.wait_event(computed[k])
        with torch.cuda.stream(down):
            for gh, go in zip(grads_host, outs[k]):
                for g in grad_keys:
                    gh[g].copy_(go[g], non_blocking=True)
            loss_host.copy_(loss, non_blocking=True)
        read[k].record(down)

    for _ in range(min(2, args.warmup)):
        e2e_step()
    barrier()
    torch.cuda.synchronize()
    a, b = mk(), mk()
    a.record(stream)
    up.wait_event(a)  # no copy of the timed steps starts before the region opens
    down.wait_event(a)
    for _ in range(K):
        e2e_step()
    stream.wait_stream(down)  # the region closes when the last read-back has landed
    b.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = ldist.max_over_ranks(a.elapsed_time(b), device=dev)
    return {"value": ldist.job_rate(logits_job, K, e2e_ms), "unit": unit,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_ms / K,
            "d2h": "gradients (" + ", ".join(grad_keys) + ") of every relation and the loss"}


def _profiled_traffic(kernel, w, grads="partials"):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary for this workload, if one exists and was taken on the current
    kernel sources (else None: the counters no longer describe this kernel)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            tab = json.load(f)
        ent = tab[f"{kernel}:{w.name}" + ("" if grads == "partials" else ":" + grads)]
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
