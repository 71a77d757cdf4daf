#!/usr/bin/env python
"""Throughput of the BCJR forward-backward hot path on B200.

One step = one full pass of the path over one batch: ``bcjr_soft_codeword``
(forward + backward sweep: soft codeword and logZ) followed by ``bcjr_vjp``
(forward + backward expectation-semiring sweep: gradients w.r.t. weights and
codebook) on the QTIP-scale workload: L=16 (65536 states), k=2, V=1, a
2048x2048 fp32 matrix cut into 16384 sequences of 256 weights, T=0.05,
synthetic seeded inputs (codebook seed 0, weights seed 1, upstream gradient
seed 2).  Metric: state-updates/s = n_seq * n_steps * 2^L per step / time
(weights/s reported alongside).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload qtip|mid|mlp|layer|tiny] [--temp T] [--qat]

The default workload is the QTIP-scale one above.  ``--workload`` measures the
other seeded workloads of the inputs module with the same timing rules (``mid``
is forward only: soft codeword and logZ; ``mlp`` takes ``--temp`` from
{1, 0.1, 0.01}).  ``--qat`` times one self-reconstruction QAT step per
iteration instead (``bcjr_qat_step``: soft codeword, loss and its upstream
gradient, VJP and the in-place SGD update of the weights, lr 1e-3).

N > 1 runs under torch.distributed.run, one rank per GPU, each rank on its own
copy of the workload (weak scaling); the codebook gradient is summed across
ranks with one NCCL all-reduce per step.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "BCJR state-updates/s and weights/s (fwd+bwd+VJP) at L=16 k=2, 1 B200"
UNIT = "state-updates/s"
WORKLOAD = "qtip"

# Algorithmic work per (sequence, step, state) unit, fixed before optimisation
# (FP32-pipe ops, MUFU ex2 ops of a linear-domain sweep with one ex2 per state
# per sweep); recomputation and ALU-pipe work (max, compares, address
# arithmetic) are not counted.  k=2, V=1 (B = 4): forward 3.75 (energy FFMA,
# 0.75 gather FADD, rescale, psi*u), backward + posterior + soft codeword 6.75,
# VJP forward 7.5, VJP backward + G + gradients 16.5.  k=2, V=2 (B = 16): the
# energy, h = g.c and each gradient term take one op per component and the
# gather 15/16 per state: 4.94, 8.94, 10.88, 22.69.
LEDGERS = {
    (2, 1): {"soft": {"fp32": 3.75 + 6.75, "mufu": 2.0}, "vjp": {"fp32": 7.5 + 16.5, "mufu": 2.0}},
    (2, 2): {"soft": {"fp32": 4.94 + 8.94, "mufu": 2.0}, "vjp": {"fp32": 10.88 + 22.69, "mufu": 2.0}},
}
LEDGER = LEDGERS[(2, 1)]
# DRAM bytes per sequence (read + write) of each L=16, V=1 sweep kernel, from one
# ncu capture of 16 qtip sequences (one sequence per CTA, the same per-SM
# history traffic as a full launch); set to None whenever the kernel changes.
# (A 16-sequence capture of the V=2 kernels keeps their histories in L2, so it
# does not scale to a full launch; their traffic is reported as null.)
TRAFFIC_PER_SEQ = {"vjp": 1000.14e6 / 16, "soft": 443.19e6 / 16}
FP32_PER_CLK_SM = 128.0   # FFMA lanes per SM per clock (measured 123.5 FFMA, 126 FFMA2 on this machine)
MUFU_PER_CLK_SM = 16.0    # ex2 per SM per clock (measured 15.99 on this machine)
N_SM = 148


def peak_units_per_s(kind: str, mhz: float, ledger=None) -> float:
    ledger = ledger or LEDGER
    led = ledger[kind] if kind != "step" else {
        "fp32": ledger["soft"]["fp32"] + ledger["vjp"]["fp32"], "mufu": ledger["soft"]["mufu"] + ledger["vjp"]["mufu"]}
    clk_per_unit = max(led["fp32"] / FP32_PER_CLK_SM, led["mufu"] / MUFU_PER_CLK_SM)
    return N_SM * mhz * 1e6 / clk_per_unit


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0}, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def oracle_sample_rows(wl, n_avail: int) -> int:
    """Sequences (= oracle threads) for a timed CPU sample: one per host core, at
    most 128, and within a memory budget (each oracle thread holds about three
    n x 2^L fp64 arrays): 1/16 of physical memory, at most 32 GB."""
    cores = os.cpu_count() or 1
    per_thread = 3 * wl.n_steps * wl.S * 8
    try:
        phys = os.sysconf("SC_PAGE_SIZE") * os.sysconf("SC_PHYS_PAGES")
    except (ValueError, OSError, AttributeError):
        phys = 64 << 30
    budget = min(phys // 16, 32 << 30)
    return max(1, min(cores, 128, n_avail, budget // per_thread))


def cpu_baseline(wl, inp, n_rows: int, T: float, do_vjp: bool):
    """The oracle as it stands, on n_rows sequences of the workload, one host thread each."""
    import oracle
    rows = list(range(n_rows))
    w = inp.w[rows].contiguous()
    t0 = time.perf_counter()
    oracle.soft(w, inp.c, wl.L, wl.k, wl.V, T, nthreads=n_rows)
    if do_vjp:
        oracle.vjp(w, inp.c, wl.L, wl.k, wl.V, T, inp.g[rows].contiguous(), nthreads=n_rows)
    dt = time.perf_counter() - t0
    units = n_rows * wl.n_steps * wl.S
    what = "soft codeword + VJP" if do_vjp else "soft codeword"
    return {"value": units / dt, "unit": UNIT, "cores": n_rows, "kind": "oracle",
            "sample": f"{n_rows} of {wl.n_seq} sequences of the {wl.name} workload, {what}, "
                      f"fp64 C oracle with OpenMP over sequences; {dt:.1f} s"}


def units_e2e(wl, n_seq: int) -> int:
    return n_seq * wl.n_steps * wl.S


def describe(wl, T: float, do_vjp: bool) -> str:
    mats = ", ".join(f"{r}x{c}" for r, c in wl.matrices)
    what = "soft codeword + logZ + VJP" if do_vjp else "soft codeword + logZ"
    return (f"{wl.name}: L={wl.L} k={wl.k} V={wl.V}, fp32 matrices {mats} as {wl.n_seq} x {wl.seq_len}-weight "
            f"sequences ({wl.n_steps} steps), T={T:g}, {what} per step")


def metric_for(wl, do_vjp: bool) -> str:
    if wl.name == WORKLOAD:
        return METRIC
    return (f"BCJR state-updates/s and weights/s ({'fwd+bwd+VJP' if do_vjp else 'fwd+bwd'}) on the {wl.name} "
            f"workload (L={wl.L} k={wl.k} V={wl.V}), 1 B200")


def run_reference(args):
    """The oracle arm: rank 0 times the CPU oracle on a bounded sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from bcjr_sum_product_b200 import inputs as I
    wl = I.WORKLOADS[args.workload]
    T = args.temp if args.temp is not None else wl.temps[0]
    do_vjp = "vjp" in wl.calls
    n_rows = oracle_sample_rows(wl, wl.n_seq)   # one sequence per oracle thread
    inp = I.make(args.workload, rows=list(range(n_rows)))
    import oracle

    def step():
        oracle.soft(inp.w, inp.c, wl.L, wl.k, wl.V, T, nthreads=n_rows)
        if do_vjp:
            oracle.vjp(inp.w, inp.c, wl.L, wl.k, wl.V, T, inp.g, nthreads=n_rows)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / max(1, args.steps)
    units = n_rows * wl.n_steps * wl.S
    value = units / dt
    sample = (f"{n_rows} of {wl.n_seq} sequences of the {wl.name} workload per step "
              f"({'soft codeword + VJP' if do_vjp else 'soft codeword'})")
    line = {"impl": "reference", "metric": metric_for(wl, do_vjp), "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": describe(wl, T, do_vjp), "sample_sequences": n_rows},
            "weights_per_s": n_rows * wl.seq_len / dt,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": n_rows, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--seqs", type=int, default=0,
                    help="profiling only: run on the first N sequences of the workload (not a bench number)")
    ap.add_argument("--workload", default=WORKLOAD, choices=["qtip", "mid", "mlp", "layer", "tiny"])
    ap.add_argument("--temp", type=float, default=None, help="temperature (one of the workload's)")
    ap.add_argument("--qat", action="store_true", help="time bcjr_qat_step (self-reconstruction QAT step)")
    args = ap.parse_args()
    from bcjr_sum_product_b200 import inputs as I
    if args.temp is not None and args.temp not in I.WORKLOADS[args.workload].temps:
        ap.error(f"--temp must be one of {I.WORKLOADS[args.workload].temps}")
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist
    from bcjr_sum_product_b200 import dist as bdist
    from bcjr_sum_product_b200 import inputs as I
    from bcjr_sum_product_b200 import lib

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    lib.load()

    wl = I.WORKLOADS[args.workload]
    do_vjp = "vjp" in wl.calls or args.qat
    inp = I.make(args.workload, rows=list(range(args.seqs)) if args.seqs > 0 else None, with_grad=do_vjp)
    T = args.temp if args.temp is not None else wl.temps[0]
    L, k, V = wl.L, wl.k, wl.V
    ledger = LEDGERS.get((k, V))
    n_seq = inp.w.shape[0]
    stream = torch.cuda.current_stream(dev)
    w = inp.w.to(dev); c = inp.c.to(dev); g = inp.g.to(dev) if do_vjp else None
    soft = torch.empty_like(w); logZ = torch.empty(n_seq, device=dev)
    gw = torch.empty_like(w); gc = torch.empty_like(c)
    flush = torch.empty(256 * 1024 * 1024 // 4, device=dev)  # 256 MB > 126 MB L2

    def local_vjp(wl_, cb_, g_):
        return lib.vjp(wl_, cb_, L, k, V, T, g_, grad_w=gw, grad_codebook=gc, stream=stream)

    if args.qat:
        if world > 1:
            raise SystemExit("--qat runs on one GPU")
        w_target = w.clone()
        qloss = torch.empty(n_seq, device=dev)

    def qat_step():
        lib.qat_step(w, w_target, c, L, k, V, T, 1e-3, 0.0, out_soft=soft, out_loss=qloss, grad_w=gw,
                     grad_codebook=gc, stream=stream)

    def step():
        if args.qat:
            qat_step()
            return
        lib.soft_codeword(w, c, L, k, V, T, out_soft=soft, out_logZ=logZ, stream=stream)
        # each rank: VJP of its own sequences, then the codebook gradient summed over ranks
        if do_vjp:
            bdist.vjp_data_parallel(local_vjp, w, c, g)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()

    sampler = ClockSampler(local)
    sampler.start()
    soft_ms, vjp_ms, step_ms = [], [], []
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    wall0 = time.perf_counter()
    for _ in range(args.steps):
        flush.fill_(1.0)  # L2 flush between timed iterations (outside the events)
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record(stream)
        if args.qat:
            qat_step()
            e1.record(stream)
        else:
            lib.soft_codeword(w, c, L, k, V, T, out_soft=soft, out_logZ=logZ, stream=stream)
            e1.record(stream)
            if do_vjp:
                bdist.vjp_data_parallel(local_vjp, w, c, g)
        e2.record(stream)
        e2.synchronize()
        soft_ms.append(e0.elapsed_time(e1)); vjp_ms.append(e1.elapsed_time(e2)); step_ms.append(e0.elapsed_time(e2))
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    wall = time.perf_counter() - wall0
    clocks = sampler.stop()
    assert lib.get_device_error(stream) == 0

    total = torch.tensor([sum(step_ms), sum(soft_ms), sum(vjp_ms)], device=dev, dtype=torch.float64)
    if world > 1:
        dist.all_reduce(total, op=dist.ReduceOp.MAX)
    ms_step = float(total[0]) / args.steps
    ms_soft = float(total[1]) / args.steps
    ms_vjp = float(total[2]) / args.steps
    units = n_seq * wl.n_steps * wl.S
    value = world * units / (ms_step / 1e3)

    # e2e: through the public API with host buffers, copies inside the timed region
    e2e = None
    if not args.no_e2e and args.qat:
        hw = inp.w.pin_memory(); hc = inp.c.pin_memory()
        out_w_h = torch.empty_like(hw).pin_memory(); out_loss_h = torch.empty(n_seq).pin_memory()
        h2d = 2 * hw.numel() * 4 + hc.numel() * 4
        d2h = out_w_h.numel() * 4 + out_loss_h.numel() * 4
        times = []
        for _ in range(max(1, min(args.steps, 3))):
            flush.fill_(1.0)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            w.copy_(hw, non_blocking=True); w_target.copy_(hw, non_blocking=True); c.copy_(hc, non_blocking=True)
            qat_step()
            out_w_h.copy_(w, non_blocking=True); out_loss_h.copy_(qloss, non_blocking=True)
            b.record(stream)
            b.synchronize()
            times.append(a.elapsed_time(b))
        e2e = {"value": units_e2e(wl, n_seq) / (sum(times) / len(times) / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": sum(times) / len(times)}
    elif not args.no_e2e:
        hw = inp.w.pin_memory(); hc = inp.c.pin_memory(); hg = inp.g.pin_memory() if do_vjp else None
        out_soft_h = torch.empty_like(hw).pin_memory(); out_logZ_h = torch.empty(n_seq).pin_memory()
        out_gw_h = torch.empty_like(hw).pin_memory() if do_vjp else None
        out_gc_h = torch.empty_like(hc).pin_memory() if do_vjp else None
        h2d = hw.numel() * 4 + hc.numel() * 4 + (hg.numel() * 4 if do_vjp else 0)
        d2h = out_soft_h.numel() * 4 + out_logZ_h.numel() * 4
        if do_vjp:
            d2h += out_gw_h.numel() * 4 + out_gc_h.numel() * 4
        k_e2e = max(1, min(args.steps, 3))
        times = []
        for _ in range(k_e2e):
            flush.fill_(1.0)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            w.copy_(hw, non_blocking=True); c.copy_(hc, non_blocking=True)
            if do_vjp:
                g.copy_(hg, non_blocking=True)
            lib.soft_codeword(w, c, L, k, V, T, out_soft=soft, out_logZ=logZ, stream=stream)
            if do_vjp:
                bdist.vjp_data_parallel(local_vjp, w, c, g)
            out_soft_h.copy_(soft, non_blocking=True); out_logZ_h.copy_(logZ, non_blocking=True)
            if do_vjp:
                out_gw_h.copy_(gw, non_blocking=True); out_gc_h.copy_(gc, non_blocking=True)
            b.record(stream)
            b.synchronize()
            times.append(a.elapsed_time(b))
        te = torch.tensor([sum(times) / len(times)], device=dev, dtype=torch.float64)
        if world > 1:
            dist.all_reduce(te, op=dist.ReduceOp.MAX)
        e2e = {"value": world * units / (float(te[0]) / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": float(te[0])}

    if rank != 0:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return 0

    peaks, basis = measured_peaks()
    fmax = float(peaks.get("sm_max_mhz", 1965.0))
    dominant = "vjp" if do_vjp and ms_vjp >= ms_soft else "soft"
    if args.qat:
        dominant = "step"
    ms_dom = ms_step if args.qat else (ms_vjp if dominant == "vjp" else ms_soft)
    achieved = units / (ms_dom / 1e3)
    block_layout = (L, k, V) == (16, 2, 1)
    if args.qat:
        kernel = "bcjr_qat_step (soft codeword + loss + VJP + update, all launches)"
    elif block_layout:
        kernel = f"bcjr::l16::{dominant}_kernel"
    elif (L, k, V) == (16, 2, 2):
        kernel = f"bcjr::l16v2::{dominant}_kernel"
    else:
        kernel = f"bcjr::bcjr_sweep_kernel<{V},{k * V},{1 if dominant == 'vjp' else 0}>"
    roofline = None
    if ledger is not None:
        peak = peak_units_per_s(dominant, fmax, ledger)
        tps = TRAFFIC_PER_SEQ.get(dominant) if block_layout and not args.qat else None
        roofline = {"bound": "alu", "kernel": kernel, "achieved": achieved, "peak": peak,
                    "unit": UNIT, "frac": achieved / peak, "traffic": (tps * n_seq) if tps else None,
                    "traffic_note": "DRAM bytes per launch, scaled from an ncu capture of 16 sequences",
                    "peak_basis": (f"{N_SM} SMs x min(128 FP32 / {ledger[dominant]['fp32']}, 16 MUFU / "
                                   f"{ledger[dominant]['mufu']}) units/clk at sm_max {fmax:.0f} MHz ({basis})"
                                   if dominant != "step" else
                                   f"{N_SM} SMs, soft + VJP ledger, at sm_max {fmax:.0f} MHz ({basis})")}
        if do_vjp:
            roofline["step_frac"] = value / world / peak_units_per_s("step", fmax, ledger)
        if clocks.get("sm_mhz"):
            roofline["frac_at_sampled_clock"] = achieved / peak_units_per_s(dominant, clocks["sm_mhz"], ledger)

    cpu = None
    if args.seqs > 0:
        line_note = f"profiling subset: first {n_seq} sequences only, not a bench number"
    else:
        line_note = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, inp, oracle_sample_rows(wl, n_seq), T, do_vjp)

    metric = metric_for(wl, do_vjp)
    if args.qat:
        metric = f"BCJR-QAT self-reconstruction step (soft + loss + VJP + update): state-updates/s on the {wl.name} workload, 1 B200"
    line = {"metric": metric, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": describe(wl, T, do_vjp),
                       "n_seq_per_gpu": n_seq, "steps_per_seq": wl.n_steps, "states": wl.S,
                       "l2": "flushed between timed iterations (256 MB write outside the events)",
                       "parallelism": f"dp{world}" if world > 1 else "single"},
            "weights_per_s": world * n_seq * wl.seq_len / (ms_step / 1e3),
            "ms_soft": None if args.qat else ms_soft, "ms_vjp": None if args.qat else ms_vjp, "wall_s": wall,
            "ms_step_min_max": [min(step_ms), max(step_ms)],
            "gpu_launches": (7 if args.qat else 5 if do_vjp else 2) * args.steps,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks}
    if line_note:
        line["note"] = line_note
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
