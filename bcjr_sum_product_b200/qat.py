"""Quantisation-aware training by self-reconstruction on top of the library.

"BCJR-QAT: A Differentiable Relaxation of Trellis-Coded Weight Quantization"
(Technical Summary, "Core Mechanism" and "Key Technical Innovations"): the soft
codeword of the latent weights w stands in for the quantised weights, T is
annealed from T0 towards a near-zero T_end, and the schedule that skips the
high-T phase (T0 = 0.3 instead of 1.0) avoids drifting into a worse Voronoi
basin.  The drift-budget criterion compares the cumulative drift
eta * N * g_max with the basin radius (about 1e-3).

Each step is one ``bcjr_qat_step`` call (soft codeword, loss
sum ||w_hat - w*||^2 and its upstream gradient, VJP and the in-place update,
all in the library's kernels); this module only schedules T and reports.

    python -m bcjr_sum_product_b200.qat --workload qtip --seqs 256 --T0 0.3 --T-end 0.01 --steps 40 --lr 1e-3
"""
from __future__ import annotations

import argparse
import json
import math
from typing import Dict, List, Optional

import torch

from . import lib


def anneal(T0: float, T_end: float, steps: int) -> List[float]:
    """Geometric schedule from T0 to T_end over `steps` steps (T0 only for one step)."""
    if not (T0 > 0 and T_end > 0 and steps >= 1):
        raise ValueError("T0, T_end > 0 and steps >= 1 required")
    if steps == 1:
        return [float(T0)]
    r = (T_end / T0) ** (1.0 / (steps - 1))
    return [float(T0 * r ** i) for i in range(steps)]


def hard_mse(states: torch.Tensor, codebook: torch.Tensor, target: torch.Tensor, V: int) -> torch.Tensor:
    """Per-sequence sum of squared differences between the codewords of a
    state path and the target weights (host-side report, not the hot path)."""
    cw = codebook.reshape(codebook.shape[0], -1)[states.long()]          # [n_seq, n, V]
    return ((cw.reshape(target.shape) - target) ** 2).sum(dim=1)


def run(w_target: torch.Tensor, codebook: torch.Tensor, L: int, k: int, V: int, T0: float, T_end: float,
        steps: int, lr_w: float, lr_c: float = 0.0, stream=None) -> Dict:
    """Anneal from w = w_target; returns the loss history, the drift budget and
    how far the hard (Viterbi) code moved from the PTQ code of w_target."""
    w = w_target.clone()
    c = codebook.clone()
    temps = anneal(T0, T_end, steps)
    loss_hist, gmax_hist = [], []
    soft = torch.empty_like(w)
    loss = torch.empty(w.shape[0], device=w.device)
    gw = torch.empty_like(w)
    gc = torch.empty_like(c)
    for T in temps:
        lib.qat_step(w, w_target, c, L, k, V, T, lr_w, lr_c, out_soft=soft, out_loss=loss, grad_w=gw,
                     grad_codebook=gc, stream=stream)
        loss_hist.append(float(loss.sum()))
        gmax_hist.append(float(gw.abs().max()))
    ptq_states, ptq_cost = lib.viterbi_decode(w_target, codebook, L, k, V)
    new_states, _ = lib.viterbi_decode(w, c, L, k, V)
    mse_ptq = hard_mse(ptq_states, codebook, w_target, V)
    mse_new = hard_mse(new_states, c, w_target, V)
    changed = (new_states != ptq_states).float().mean().item()
    drift = float((w - w_target).abs().max())
    budget = lr_w * steps * max(gmax_hist)
    return {"temps": [temps[0], temps[-1]], "steps": steps, "lr_w": lr_w, "lr_c": lr_c,
            "loss_first": loss_hist[0], "loss_last": loss_hist[-1], "loss": loss_hist,
            "drift_budget": budget, "max_drift": drift, "g_max": max(gmax_hist),
            "code_changed_fraction": changed,
            "hard_mse_ptq": float(mse_ptq.sum()), "hard_mse_qat": float(mse_new.sum()),
            "w": w, "codebook": c}


def main(argv: Optional[List[str]] = None) -> int:
    from . import inputs as I
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", default="qtip", choices=sorted(I.WORKLOADS))
    ap.add_argument("--seqs", type=int, default=256)
    ap.add_argument("--T0", type=float, default=0.3)
    ap.add_argument("--T-end", type=float, default=0.01)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--lr", type=float, default=1e-3)
    ap.add_argument("--lr-c", type=float, default=0.0)
    a = ap.parse_args(argv)
    wl = I.WORKLOADS[a.workload]
    inp = I.make(a.workload, rows=list(range(min(a.seqs, wl.n_seq))), with_grad=False)
    lib.load()
    dev = torch.device("cuda")
    out = run(inp.w.to(dev), inp.c.to(dev), wl.L, wl.k, wl.V, a.T0, a.T_end, a.steps, a.lr, a.lr_c)
    rep = {k: v for k, v in out.items() if k not in ("w", "codebook", "loss")}
    rep["loss_every_10"] = out["loss"][::10]
    rep["workload"] = a.workload
    rep["sequences"] = int(inp.w.shape[0])
    print(json.dumps(rep))
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
