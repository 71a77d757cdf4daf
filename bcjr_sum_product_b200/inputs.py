"""Seeded synthetic workloads for the BCJR forward-backward path.

This module holds the workload shapes and the seeded random draws only; it
contains none of the method's arithmetic.  Both the CUDA path (through the
tests and ``bench.py``) and the CPU oracle are fed from here, so the two see
identical bytes.

Workloads (the trellis parameters follow the bitshift trellis of QTIP-style
trellis-coded quantisation named in the BCJR-QAT abstract, "BCJR-QAT: A
Differentiable Relaxation of Trellis-Coded Weight Quantization", Abstract):

* ``tiny``    L=8,  k=2, V=1, 16 sequences x 64 weights, T=0.5
* ``mid``     L=12, k=2, V=1, a 1024x1024 matrix cut into 256-weight rows, T=0.1
* ``qtip``    L=16, k=2, V=1, a 2048x2048 matrix (16384 x 256), T=0.05
* ``mlp``     L=16, k=2, V=1, an 8192x2048 matrix (65536 x 256), T in {1, 0.1, 0.01}
* ``layer``   L=16, k=2, V=2, the seven matrices of one decoder layer
              (2x 2048^2, 2x 512x2048, 2x 8192x2048, 2048x8192), 256-weight rows
              (128 steps of 2 weights), T=0.05
* ``long``    L=16, k=2, V=1, an 8192x2048 matrix cut into 8192-weight rows
              (2048 sequences, the longest supported length), T=0.05

Draw recipe: every tensor is drawn on the CPU with ``torch.Generator`` seeded
as stated and ``torch.randn(..., dtype=float32)``.  The codebook uses seed 0
(shape ``[2^L]`` for V=1, ``[2^L, 2]`` for V=2), the weights seed 1 (one
generator draws the matrices in the listed order; each is flattened row-major
and cut into consecutive ``len``-weight sequences), and the upstream gradient
of the soft codeword seed 2 (shape of the weights).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    L: int              # state bits: 2^L trellis states
    k: int              # bits per weight
    V: int              # weights per trellis step (codeword dimension)
    seq_len: int        # weights per sequence ("len"); steps n = seq_len // V
    matrices: Tuple[Tuple[int, int], ...]  # weight matrices drawn in order
    temps: Tuple[float, ...]
    calls: str          # which entry points the workload exercises

    @property
    def D(self) -> int:
        return self.k * self.V

    @property
    def S(self) -> int:
        return 1 << self.L

    @property
    def n_steps(self) -> int:
        return self.seq_len // self.V

    @property
    def n_weights(self) -> int:
        return sum(r * c for r, c in self.matrices)

    @property
    def n_seq(self) -> int:
        return self.n_weights // self.seq_len

    @property
    def units(self) -> int:
        """(sequence, step, state) triples of one full pass."""
        return self.n_seq * self.n_steps * self.S


WORKLOADS = {
    "tiny": Workload("tiny", 8, 2, 1, 64, ((16, 64),), (0.5,), "soft+vjp"),
    "mid": Workload("mid", 12, 2, 1, 256, ((1024, 1024),), (0.1,), "soft"),
    "qtip": Workload("qtip", 16, 2, 1, 256, ((2048, 2048),), (0.05,), "soft+vjp"),
    "mlp": Workload("mlp", 16, 2, 1, 256, ((8192, 2048),), (1.0, 0.1, 0.01), "soft+vjp+viterbi"),
    "layer": Workload("layer", 16, 2, 2, 256,
                      ((2048, 2048), (2048, 2048), (512, 2048), (512, 2048),
                       (8192, 2048), (8192, 2048), (2048, 8192)), (0.05,), "soft+vjp"),
    "long": Workload("long", 16, 2, 1, 8192, ((8192, 2048),), (0.05,), "soft+vjp"),
}

CODEBOOK_SEED = 0
WEIGHT_SEED = 1
GRAD_SEED = 2
SUBSET_SEED = 3


def codebook(L: int, V: int, seed: int = CODEBOOK_SEED) -> torch.Tensor:
    """Codebook c[s] (fp32): shape [2^L] for V=1, [2^L, V] otherwise."""
    g = torch.Generator().manual_seed(seed)
    shape = (1 << L,) if V == 1 else (1 << L, V)
    return torch.randn(shape, generator=g, dtype=torch.float32)


def weights(wl: Workload, seed: int = WEIGHT_SEED) -> torch.Tensor:
    """All sequences of the workload, [n_seq, seq_len] fp32."""
    g = torch.Generator().manual_seed(seed)
    parts = [torch.randn((r, c), generator=g, dtype=torch.float32).reshape(-1) for r, c in wl.matrices]
    flat = torch.cat(parts) if len(parts) > 1 else parts[0]
    return flat.reshape(wl.n_seq, wl.seq_len)


def upstream_grad(n_seq: int, seq_len: int, seed: int = GRAD_SEED) -> torch.Tensor:
    """Upstream gradient on the soft codeword, [n_seq, seq_len] fp32."""
    g = torch.Generator().manual_seed(seed)
    return torch.randn((n_seq, seq_len), generator=g, dtype=torch.float32)


def subset_rows(n_seq: int, n_first: int = 64, n_random: int = 64, seed: int = SUBSET_SEED) -> np.ndarray:
    """Sorted row indices: the first ``n_first`` sequences plus ``n_random``
    further sequences drawn without replacement (seeded)."""
    first = np.arange(min(n_first, n_seq))
    rest = np.arange(len(first), n_seq)
    if n_random > 0 and len(rest) > 0:
        g = torch.Generator().manual_seed(seed)
        perm = torch.randperm(len(rest), generator=g).numpy()[: min(n_random, len(rest))]
        picked = rest[np.sort(perm)]
    else:
        picked = np.zeros(0, dtype=np.int64)
    return np.concatenate([first, picked]).astype(np.int64)


@dataclass
class Inputs:
    wl: Workload
    w: torch.Tensor          # [n_seq, seq_len] fp32
    c: torch.Tensor          # [2^L] or [2^L, V] fp32
    g: Optional[torch.Tensor]  # [n_seq, seq_len] fp32 or None
    rows: Optional[np.ndarray] = None  # which rows of the full workload these are


def make(name: str, rows: Optional[Sequence[int]] = None, with_grad: bool = True) -> Inputs:
    """Seeded inputs of a named workload, optionally restricted to ``rows``."""
    wl = WORKLOADS[name]
    c = codebook(wl.L, wl.V)
    w = weights(wl)
    g = upstream_grad(wl.n_seq, wl.seq_len) if with_grad else None
    if rows is not None:
        idx = torch.as_tensor(np.asarray(rows, dtype=np.int64))
        w = w.index_select(0, idx).contiguous()
        g = g.index_select(0, idx).contiguous() if g is not None else None
        rows = np.asarray(rows, dtype=np.int64)
    return Inputs(wl, w, c, g, rows)


def random_case(L: int, k: int, V: int, n_seq: int, seq_len: int, seed: int,
                scale: float = 1.0) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Small ad-hoc case (w, c, g) with iid N(0, scale^2) draws from one seeded generator."""
    g = torch.Generator().manual_seed(seed)
    cshape = (1 << L,) if V == 1 else (1 << L, V)
    c = torch.randn(cshape, generator=g, dtype=torch.float32) * scale
    w = torch.randn((n_seq, seq_len), generator=g, dtype=torch.float32) * scale
    gr = torch.randn((n_seq, seq_len), generator=g, dtype=torch.float32)
    return w, c, gr
