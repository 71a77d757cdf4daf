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
                    [--workload qtip|mid|mlp|layer|tiny|long] [--temp T] [--qat | --viterbi]
                    [--replicate]

The default workload is the QTIP-scale one above.  ``--workload`` measures the
other seeded workloads of the inputs module with the same timing rules (``mid``
is forward only: soft codeword and logZ; ``mlp`` takes ``--temp`` from
{1, 0.1, 0.01}; ``long`` cuts the mlp matrix into 8192-weight rows, where the
L=16 kernels keep checkpointed histories).  ``--qat`` times one self-reconstruction QAT step per
iteration instead (``bcjr_qat_step``: soft codeword, loss and its upstream
gradient, VJP and the in-place SGD update of the weights, lr 1e-3).
``--viterbi`` times the T -> 0 hard decode (``viterbi_decode``, the
trellis-coded quantisation encode) over the workload (default ``mlp``).

N > 1 runs under torch.distributed.run, one rank per GPU.  By default the
ranks split the sequences of one workload into contiguous shards (strong
scaling: the total work is fixed) and the codebook gradient is summed across
ranks with one NCCL all-reduce per step; ``--replicate`` gives every rank its
own copy of the workload instead (weak scaling).  Rank 0 prints one JSON line.

Kernel variants of the L=16, k=2, V=1 path follow the library's selectors
(BCJR_L16_BWD=post|log, BCJR_L16_VJP=cluster); the line records them.
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

METRIC = "BCJR state-updates/s and weights/s (fwd+bwd+VJP) at L=16 k=2, 1 B200"
UNIT = "state-updates/s"
WORKLOAD = "qtip"
VITERBI_WORKLOAD = "mlp"

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
# Viterbi (min-sum in the prescribed fp32 order), per unit: the energy
# fl(fl(w - c)^2) and the add of the predecessor-group minimum, one FADD + one
# FMUL + one FADD per component-free state for V = 1 (V = 2: two FADD, two
# FMUL, one FADD for the component sum, one FADD for the minimum); the group
# minimum itself, (B - 1) / B compares per state, runs on the ALU pipe.
VITERBI_LEDGERS = {(2, 1): {"fp32": 3.0, "alu": 0.75}, (2, 2): {"fp32": 6.0, "alu": 15.0 / 16.0}}
# DRAM bytes per sequence (read + write) of each L=16, V=1 sweep kernel, from one
# ncu capture of 16 qtip sequences (one sequence per CTA, the same per-SM
# history traffic as a full launch); set to None whenever the kernel changes.
# (A 16-sequence capture of the V=2 kernels keeps their histories in L2, so it
# does not scale to a full launch; their traffic is reported as null.)
TRAFFIC_PER_SEQ = {"vjp": (457.83e6 + 548.85e6) / 16, "soft": (179.55e6 + 271.94e6) / 16}
FP32_PER_CLK_SM = 128.0   # FFMA lanes per SM per clock (measured by microbenchmark: 123.5 FFMA, 126 FFMA2)
MUFU_PER_CLK_SM = 16.0    # ex2 per SM per clock (measured by microbenchmark: 15.99)
ALU_PER_CLK_SM = 64.0     # compare / min-max lanes per SM per clock (nominal)
N_SM = 148


def peak_units_per_s(kind: str, mhz: float, ledger=None) -> float:
    ledger = ledger or LEDGER
    led = ledger[kind] if kind != "step" else {
        "fp32": ledger["soft"]["fp32"] + ledger["vjp"]["fp32"], "mufu": ledger["soft"]["mufu"] + ledger["vjp"]["mufu"]}
    clk_per_unit = max(led["fp32"] / FP32_PER_CLK_SM, led["mufu"] / MUFU_PER_CLK_SM)
    return N_SM * mhz * 1e6 / clk_per_unit


def viterbi_peak_units_per_s(mhz: float, ledger) -> float:
    clk_per_unit = max(ledger["fp32"] / FP32_PER_CLK_SM, ledger["alu"] / ALU_PER_CLK_SM)
    return N_SM * mhz * 1e6 / clk_per_unit


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0}, "fallback"


def kernel_variants() -> dict:
    """The library's kernel selectors as this process sees them (defaults spelled out)."""
    return {"l16_backward": os.environ.get("BCJR_L16_BWD", "post (soft), log (VJP)"),
            "l16_vjp": os.environ.get("BCJR_L16_VJP", "one CTA per sequence, codewords through a shared-memory ring"),
            "l16_ex2": os.environ.get("BCJR_L16_EX2", "mufu"),
            "l16_histories": os.environ.get("BCJR_L16_CKPT", "full, or sqrt(n) checkpoints beyond the scratch budget")}


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


def oracle_step(mode: str, wl, w, c, g, T: float, nthreads: int):
    """One step of the path in the CPU oracle on the rows of w (g: upstream gradient)."""
    import oracle
    if mode == "viterbi":
        oracle.viterbi(w, c, wl.L, wl.k, wl.V, nthreads=nthreads)
        return
    oracle.soft(w, c, wl.L, wl.k, wl.V, T, nthreads=nthreads)
    if g is not None:
        oracle.vjp(w, c, wl.L, wl.k, wl.V, T, g, nthreads=nthreads)


def cpu_baseline(mode: str, wl, inp, n_rows: int, T: float, do_vjp: bool):
    """The oracle as it stands on n_rows sequences, one host thread each, and on
    one sequence with one thread."""
    w = inp.w[:n_rows].contiguous()
    g = inp.g[:n_rows].contiguous() if do_vjp else None
    t0 = time.perf_counter()
    oracle_step(mode, wl, w, inp.c, g, T, n_rows)
    dt = time.perf_counter() - t0
    t1 = time.perf_counter()
    oracle_step(mode, wl, w[:1], inp.c, g[:1] if g is not None else None, T, 1)
    dt1 = time.perf_counter() - t1
    units = n_rows * wl.n_steps * wl.S
    what = {"viterbi": "Viterbi decode (fp32)", "path": "soft codeword + VJP" if do_vjp else "soft codeword"}[mode]
    return {"value": units / dt, "unit": UNIT, "cores": n_rows, "kind": "oracle", "nproc": os.cpu_count(),
            "value_1thread": wl.n_steps * wl.S / dt1,
            "sample": f"{n_rows} of {wl.n_seq} sequences of the {wl.name} workload, {what}, "
                      f"C oracle with OpenMP over sequences ({dt:.1f} s); one sequence on one thread {dt1:.1f} s"}


def describe(wl, T, what: str) -> str:
    mats = ", ".join(f"{r}x{c}" for r, c in wl.matrices)
    temp = f", T={T:g}" if T is not None else ""
    return (f"{wl.name}: L={wl.L} k={wl.k} V={wl.V}, fp32 matrices {mats} as {wl.n_seq} x {wl.seq_len}-weight "
            f"sequences ({wl.n_steps} steps){temp}, {what} per step")


def what_for(mode: str, do_vjp: bool) -> str:
    if mode == "viterbi":
        return "Viterbi decode (states + cost)"
    if mode == "qat":
        return "self-reconstruction QAT step (soft codeword + loss + VJP + update)"
    return "soft codeword + logZ + VJP" if do_vjp else "soft codeword + logZ"


def metric_for(mode: str, wl, do_vjp: bool) -> str:
    if mode == "viterbi":
        return (f"Viterbi (T -> 0 hard decode, the PTQ encode) state-updates/s on the {wl.name} workload "
                f"(L={wl.L} k={wl.k} V={wl.V}), 1 B200")
    if mode == "qat":
        return (f"BCJR-QAT self-reconstruction step (soft + loss + VJP + update): state-updates/s on the "
                f"{wl.name} workload, 1 B200")
    if wl.name == WORKLOAD:
        return METRIC
    return (f"BCJR state-updates/s and weights/s ({'fwd+bwd+VJP' if do_vjp else 'fwd+bwd'}) on the {wl.name} "
            f"workload (L={wl.L} k={wl.k} V={wl.V}), 1 B200")


def run_reference(args, mode: str):
    """The oracle arm: rank 0 times the CPU oracle on a bounded sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from bcjr_sum_product_b200 import inputs as I
    wl = I.WORKLOADS[args.workload]
    T = None if mode == "viterbi" else (args.temp if args.temp is not None else wl.temps[0])
    do_vjp = mode != "viterbi" and ("vjp" in wl.calls or mode == "qat")
    n_rows = oracle_sample_rows(wl, wl.n_seq)   # one sequence per oracle thread
    inp = I.make(args.workload, rows=list(range(n_rows)), with_grad=do_vjp)

    def step():
        oracle_step("viterbi" if mode == "viterbi" else "path", wl, inp.w, inp.c, inp.g if do_vjp else None, T,
                    n_rows)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / max(1, args.steps)
    units = n_rows * wl.n_steps * wl.S
    value = units / dt
    sample = f"{n_rows} of {wl.n_seq} sequences of the {wl.name} workload per step ({what_for(mode, do_vjp)})"
    line = {"impl": "reference", "metric": metric_for(mode, wl, do_vjp), "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": "strong" if args.gpus > 1 and not args.replicate else "weak",
            "vs_baseline": None, "dtype": "f32" if mode == "viterbi" else "f64", "data": "synthetic",
            "config": {"workload": describe(wl, T, what_for(mode, do_vjp)), "sample_sequences": n_rows},
            "weights_per_s": n_rows * wl.seq_len / dt,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": n_rows, "kind": "oracle", "nproc": os.cpu_count(),
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def local_problem(w, g, rank: int, world: int, replicate: bool):
    """The rows this rank works on: a contiguous shard of one problem, or (with
    ``replicate``) the whole workload on every rank.  Returns (w, g, start, stop)."""
    from bcjr_sum_product_b200 import dist as bdist
    if replicate or world == 1:
        return w, g, 0, w.shape[0]
    a, b = bdist.shard_rows(w.shape[0], rank, world)
    return w[a:b], (g[a:b] if g is not None else None), a, b


def path_halves(soft_fn, vjp_fn, w, c, g):
    """The two halves of one step of the path on this rank's rows: the soft
    codeword, then (when an upstream gradient is given) the VJP with the
    codebook gradient summed over the ranks (one all-reduce).  The second
    returns the VJP's (grad_w, grad_codebook), or None."""
    from bcjr_sum_product_b200 import dist as bdist

    def first():
        return soft_fn(w, c)

    def second():
        return None if g is None else bdist.vjp_data_parallel(vjp_fn, w, c, g)
    return first, second


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
    ap.add_argument("--workload", default=None, choices=["qtip", "mid", "mlp", "layer", "tiny", "long"])
    ap.add_argument("--temp", type=float, default=None, help="temperature (one of the workload's)")
    grp = ap.add_mutually_exclusive_group()
    grp.add_argument("--qat", action="store_true", help="time bcjr_qat_step (self-reconstruction QAT step)")
    grp.add_argument("--viterbi", action="store_true", help="time viterbi_decode (the T -> 0 hard decode)")
    ap.add_argument("--replicate", action="store_true",
                    help="N > 1: every rank runs the whole workload (weak scaling) instead of a shard of it")
    args = ap.parse_args()
    mode = "qat" if args.qat else "viterbi" if args.viterbi else "path"
    if args.workload is None:
        args.workload = VITERBI_WORKLOAD if mode == "viterbi" else WORKLOAD
    from bcjr_sum_product_b200 import inputs as I
    if args.temp is not None and args.temp not in I.WORKLOADS[args.workload].temps:
        ap.error(f"--temp must be one of {I.WORKLOADS[args.workload].temps}")
    if args.impl == "reference":
        return run_reference(args, mode)

    import torch
    import torch.distributed as dist
    from bcjr_sum_product_b200 import lib

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        if mode == "qat":
            raise SystemExit("--qat runs on one GPU")
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    lib.load()

    wl = I.WORKLOADS[args.workload]
    do_vjp = mode != "viterbi" and ("vjp" in wl.calls or mode == "qat")
    inp = I.make(args.workload, rows=list(range(args.seqs)) if args.seqs > 0 else None, with_grad=do_vjp)
    T = None if mode == "viterbi" else (args.temp if args.temp is not None else wl.temps[0])
    L, k, V = wl.L, wl.k, wl.V
    n_total = inp.w.shape[0]
    hw_rows, hg_rows, row0, row1 = local_problem(inp.w, inp.g, rank, world, args.replicate)
    n_seq = row1 - row0
    stream = torch.cuda.current_stream(dev)
    w = hw_rows.to(dev).contiguous(); c = inp.c.to(dev)
    g = hg_rows.to(dev).contiguous() if do_vjp else None
    soft = torch.empty_like(w); logZ = torch.empty(n_seq, device=dev)
    gw = torch.empty_like(w); gc = torch.empty_like(c)
    states = torch.empty((n_seq, wl.n_steps), device=dev, dtype=torch.int32)
    cost = torch.empty(n_seq, device=dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, device=dev)  # 256 MB > 126 MB L2

    def soft_fn(w_, c_):
        lib.soft_codeword(w_, c_, L, k, V, T, out_soft=soft, out_logZ=logZ, stream=stream)

    def vjp_fn(w_, c_, g_):
        return lib.vjp(w_, c_, L, k, V, T, g_, grad_w=gw, grad_codebook=gc, stream=stream)

    if mode == "qat":
        w_target = w.clone()
        qloss = torch.empty(n_seq, device=dev)

        def first_half():
            lib.qat_step(w, w_target, c, L, k, V, T, 1e-3, 0.0, out_soft=soft, out_loss=qloss, grad_w=gw,
                         grad_codebook=gc, stream=stream)

        def second_half():
            return None
    elif mode == "viterbi":
        def first_half():
            lib.viterbi_decode(w, c, L, k, V, out_states=states, out_cost=cost, stream=stream)

        def second_half():
            return None
    else:   # first half timed as "soft", second as "vjp"
        first_half, second_half = path_halves(soft_fn, vjp_fn, w, c, g)

    for _ in range(args.warmup):
        first_half()
        second_half()
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
    launches0 = lib.launch_count()
    for _ in range(args.steps):
        flush.fill_(1.0)  # L2 flush between timed iterations (outside the events)
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record(stream)
        first_half()
        e1.record(stream)
        second_half()
        e2.record(stream)
        e2.synchronize()
        soft_ms.append(e0.elapsed_time(e1)); vjp_ms.append(e1.elapsed_time(e2)); step_ms.append(e0.elapsed_time(e2))
    launches_timed = lib.launch_count() - launches0   # the library's own kernels (the L2 flush is torch's)
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
    units_rank = n_seq * wl.n_steps * wl.S
    units_all = (world if args.replicate else 1) * n_total * wl.n_steps * wl.S
    value = units_all / (ms_step / 1e3)

    # e2e: through the public API with host buffers, copies inside the timed region
    e2e = None
    if not args.no_e2e:
        hw = hw_rows.contiguous().pin_memory(); hc = inp.c.pin_memory()
        hg = hg_rows.contiguous().pin_memory() if do_vjp else None
        outs = []       # (device tensor, pinned host buffer) read back every step
        if mode == "qat":
            outs = [(w, torch.empty_like(hw).pin_memory()), (qloss, torch.empty(n_seq).pin_memory())]
            h2d = 2 * hw.numel() * 4 + hc.numel() * 4
        elif mode == "viterbi":
            outs = [(states, torch.empty((n_seq, wl.n_steps), dtype=torch.int32).pin_memory()),
                    (cost, torch.empty(n_seq).pin_memory())]
            h2d = hw.numel() * 4 + hc.numel() * 4
        else:
            outs = [(soft, torch.empty_like(hw).pin_memory()), (logZ, torch.empty(n_seq).pin_memory())]
            if do_vjp:
                outs += [(gw, torch.empty_like(hw).pin_memory()), (gc, torch.empty_like(hc).pin_memory())]
            h2d = hw.numel() * 4 + hc.numel() * 4 + (hg.numel() * 4 if do_vjp else 0)
        d2h = sum(hbuf.numel() * hbuf.element_size() for _, hbuf in outs)
        times = []
        for _ in range(max(1, min(args.steps, 3))):
            flush.fill_(1.0)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            w.copy_(hw, non_blocking=True); c.copy_(hc, non_blocking=True)
            if mode == "qat":
                w_target.copy_(hw, non_blocking=True)
            if do_vjp and mode == "path":
                g.copy_(hg, non_blocking=True)
            first_half()
            second_half()
            for dbuf, hbuf in outs:
                hbuf.copy_(dbuf, non_blocking=True)
            b.record(stream)
            b.synchronize()
            times.append(a.elapsed_time(b))
        te = torch.tensor([sum(times) / len(times)], device=dev, dtype=torch.float64)
        if world > 1:
            dist.all_reduce(te, op=dist.ReduceOp.MAX)
        e2e = {"value": units_all / (float(te[0]) / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": float(te[0])}

    if rank != 0:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return 0

    peaks, basis = measured_peaks()
    fmax = float(peaks.get("sm_max_mhz", 1965.0))
    roofline = None
    block_layout = (L, k, V) == (16, 2, 1)
    if mode == "viterbi":
        vled = VITERBI_LEDGERS.get((k, V))
        kernel = ("bcjr::l16::viterbi_kernel" if block_layout else f"bcjr::viterbi_kernel<{V},{k * V}>")
        if vled is not None:
            achieved = units_rank / (ms_step / 1e3)
            peak = viterbi_peak_units_per_s(fmax, vled)
            roofline = {"bound": "alu", "kernel": kernel, "achieved": achieved, "peak": peak, "unit": UNIT,
                        "frac": achieved / peak, "traffic": None,
                        "traffic_note": "backpointers and outputs; not captured for this mode",
                        "peak_basis": (f"{N_SM} SMs x min(128 FP32 / {vled['fp32']}, 64 ALU / {vled['alu']}) "
                                       f"units/clk at sm_max {fmax:.0f} MHz ({basis})")}
            if clocks.get("sm_mhz"):
                roofline["frac_at_sampled_clock"] = achieved / viterbi_peak_units_per_s(clocks["sm_mhz"], vled)
    else:
        ledger = LEDGERS.get((k, V))
        dominant = "vjp" if do_vjp and ms_vjp >= ms_soft else "soft"
        if mode == "qat":
            dominant = "step"
        ms_dom = ms_step if mode == "qat" else (ms_vjp if dominant == "vjp" else ms_soft)
        achieved = units_rank / (ms_dom / 1e3)
        if mode == "qat":
            kernel = "bcjr_qat_step (soft codeword + loss + VJP + update, all launches)"
        elif block_layout:
            kernel = f"bcjr::l16::{dominant}_kernel"
        elif (L, k, V) == (16, 2, 2):
            kernel = f"bcjr::l16v2::{dominant}_kernel"
        else:
            kernel = f"bcjr::bcjr_sweep_kernel<{V},{k * V},{1 if dominant == 'vjp' else 0}>"
        if ledger is not None:
            peak = peak_units_per_s(dominant, fmax, ledger)
            tps = TRAFFIC_PER_SEQ.get(dominant) if block_layout and mode == "path" else None
            roofline = {"bound": "alu", "kernel": kernel, "achieved": achieved, "peak": peak,
                        "unit": UNIT, "frac": achieved / peak, "traffic": (tps * n_seq) if tps else None,
                        "traffic_note": "DRAM bytes per launch, scaled from an ncu capture of 16 sequences",
                        "peak_basis": (f"{N_SM} SMs x min(128 FP32 / {ledger[dominant]['fp32']}, 16 MUFU / "
                                       f"{ledger[dominant]['mufu']}) units/clk at sm_max {fmax:.0f} MHz ({basis})"
                                       if dominant != "step" else
                                       f"{N_SM} SMs, soft + VJP ledger, at sm_max {fmax:.0f} MHz ({basis})")}
            if do_vjp:
                roofline["step_frac"] = (units_rank / (ms_step / 1e3)) / peak_units_per_s("step", fmax, ledger)
            if clocks.get("sm_mhz"):
                roofline["frac_at_sampled_clock"] = achieved / peak_units_per_s(dominant, clocks["sm_mhz"], ledger)

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline("viterbi" if mode == "viterbi" else "path", wl, inp, oracle_sample_rows(wl, n_seq), T,
                           do_vjp)

    line = {"metric": metric_for(mode, wl, do_vjp), "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak" if world == 1 or args.replicate else "strong",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": describe(wl, T, what_for(mode, do_vjp)),
                       "n_seq_per_gpu": n_seq, "n_seq_total": (world if args.replicate else 1) * n_total,
                       "steps_per_seq": wl.n_steps, "states": wl.S,
                       "l2": "flushed between timed iterations (256 MB write outside the events)",
                       "parallelism": (f"dp{world} ({'replicated' if args.replicate else 'sharded'})"
                                       if world > 1 else "single"),
                       "kernels": kernel_variants()},
            "weights_per_s": (world if args.replicate else 1) * n_total * wl.seq_len / (ms_step / 1e3),
            "ms_soft": ms_soft if mode == "path" else None, "ms_vjp": ms_vjp if mode == "path" else None,
            "wall_s": wall, "ms_step_min_max": [min(step_ms), max(step_ms)],
            "gpu_launches": launches_timed,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks}
    if args.seqs > 0:
        line["note"] = f"profiling subset: first {n_total} sequences only, not a bench number"
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
