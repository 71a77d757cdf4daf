"""Independent NumPy references that pin the C oracle -- TEST INFRASTRUCTURE ONLY.

These follow the definitions in "BCJR-QAT: A Differentiable Relaxation of
Trellis-Coded Weight Quantization" directly, without any recursion:

* brute force (Abstract: the soft codeword is the Boltzmann expectation over
  trellis paths; Technical Summary, "Core Mechanism": w_hat_t = sum_s c(s) p_T(s_t=s|w)):
  every path is enumerated, its weight exp(-E/T) formed, and the marginals
  summed;
* the transfer-matrix product (Abstract: the computation is the transfer-matrix
  computation of a 1D Ising-like spin chain): Z = 1^T D_0 M D_1 M ... M D_{n-1} 1
  with M the 0/1 adjacency of the trellis built from the successor rule and
  D_t = diag(exp(-E_t/T));
* closed forms of special cases.

The trellis rule, energy and boundaries are the readings stated in the C
oracle's header: succ(p, b) = ((p << D) mod 2^L) | b, E_t(s) = ||w_t - c(s)||^2,
free start and free end.
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np


def _as64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def successor(p: np.ndarray, b: np.ndarray, L: int, D: int) -> np.ndarray:
    return ((p << D) & ((1 << L) - 1)) | b


def energies(w_seq: np.ndarray, c: np.ndarray, V: int) -> np.ndarray:
    """E[t, s] = ||w_t - c(s)||^2 for one sequence; c is [S] or [S, V]."""
    c2 = c.reshape(c.shape[0], V)
    wt = w_seq.reshape(-1, V)
    return ((wt[:, None, :] - c2[None, :, :]) ** 2).sum(-1)


def all_paths(L: int, D: int, n: int) -> np.ndarray:
    """All state paths [S * B^(n-1), n] (int64), free start."""
    S, B = 1 << L, 1 << D
    paths = np.arange(S, dtype=np.int64)[:, None]
    for _ in range(1, n):
        last = paths[:, -1]
        nxt = successor(np.repeat(last, B), np.tile(np.arange(B, dtype=np.int64), len(last)), L, D)
        paths = np.concatenate([np.repeat(paths, B, axis=0), nxt[:, None]], axis=1)
    return paths


def _lse(x: np.ndarray) -> float:
    m = np.max(x)
    if not np.isfinite(m):
        return float(m)
    return float(m + np.log(np.sum(np.exp(x - m))))


def brute_force(w_seq, c, L: int, k: int, V: int, T: float, g_seq=None, gZ: float = 0.0):
    """Enumerate every path of one sequence.

    Returns logZ, posteriors p[t, s], the soft codeword, the path-energy
    minimum and its lowest-index argmin path (lexicographic by (s_0, b_1, ...)),
    and, if g_seq is given, the exact G[t, s] = Cov(F, 1[s_t = s]) + gZ p_t(s)
    with F = sum_t g_t . c(s_t).
    """
    w_seq = _as64(w_seq); c = _as64(c)
    D = k * V
    S = 1 << L
    n = w_seq.size // V
    E = energies(w_seq, c, V)                      # [n, S]
    paths = all_paths(L, D, n)                     # [P, n]
    Epath = E[np.arange(n)[None, :], paths].sum(1)
    logw = -Epath / T
    logZ = _lse(logw)
    prob = np.exp(logw - logZ)
    post = np.zeros((n, S))
    for t in range(n):
        post[t] = np.bincount(paths[:, t], weights=prob, minlength=S)
    c2 = c.reshape(S, V)
    soft = (post @ c2).reshape(-1)
    ibest = int(np.argmin(Epath))  # first occurrence = lowest (s_0, b_1, ...) ordering
    res = {"logZ": logZ, "post": post, "soft": soft, "Emin": float(Epath[ibest]), "argmin_path": paths[ibest],
           "Epath": Epath, "paths": paths}
    if g_seq is not None:
        g2 = _as64(g_seq).reshape(n, V)
        Hs = g2 @ c2.T                              # h_t(s) = g_t . c(s)   [n, S]
        F = Hs[np.arange(n)[None, :], paths].sum(1)
        EF = float(np.sum(prob * F))
        G = np.zeros((n, S))
        for t in range(n):
            G[t] = np.bincount(paths[:, t], weights=prob * F, minlength=S) - EF * post[t] + gZ * post[t]
        res["G"] = G
        res["EF"] = EF
    return res


def transfer_matrix(L: int, D: int) -> np.ndarray:
    """Dense 0/1 adjacency M[p, s] = 1 iff s = succ(p, b) for some b."""
    S, B = 1 << L, 1 << D
    M = np.zeros((S, S))
    p = np.repeat(np.arange(S, dtype=np.int64), B)
    b = np.tile(np.arange(B, dtype=np.int64), S)
    M[p, successor(p, b, L, D)] = 1.0
    return M


def transfer_matrix_logZ(w_seq, c, L: int, k: int, V: int, T: float, M: Optional[np.ndarray] = None) -> float:
    """log(1^T D_0 M D_1 M ... M D_{n-1} 1), evaluated left to right with a
    running normalisation (the product itself, only rescaled)."""
    w_seq = _as64(w_seq); c = _as64(c)
    D = k * V
    if M is None:
        M = transfer_matrix(L, D)
    theta = -energies(w_seq, c, V) / T
    n = theta.shape[0]
    m0 = theta[0].max()
    v = np.exp(theta[0] - m0)
    logscale = m0
    for t in range(1, n):
        v = v @ M
        mt = theta[t].max()
        v = v * np.exp(theta[t] - mt)
        logscale += mt
        s = v.sum()
        v = v / s
        logscale += math.log(s)
    return float(logscale + math.log(v.sum()))


def softmax_case(w_seq, c, L: int, V: int, T: float):
    """D = L: every state reaches every state, so the chain factorises and
    p_t = softmax_s(-E_t(s)/T), logZ = sum_t logsumexp_s(-E_t(s)/T)."""
    w_seq = _as64(w_seq); c = _as64(c)
    theta = -energies(w_seq, c, V) / T
    m = theta.max(1, keepdims=True)
    lz = (m[:, 0] + np.log(np.exp(theta - m).sum(1)))
    post = np.exp(theta - lz[:, None])
    return {"logZ": float(lz.sum()), "post": post, "soft": (post @ c.reshape(-1, V)).reshape(-1)}


def constant_codebook_logZ(w_seq, c0, L: int, D: int, V: int, T: float) -> float:
    """c(s) = c0 for every s: every one of the 2^L * 2^(D(n-1)) paths has the
    same energy sum_t ||w_t - c0||^2."""
    w_seq = _as64(w_seq).reshape(-1, V)
    n = w_seq.shape[0]
    E = ((w_seq - _as64(c0).reshape(1, V)) ** 2).sum()
    return (L + D * (n - 1)) * math.log(2.0) - E / T


def path_count_log(L: int, D: int, n: int) -> float:
    return (L + D * (n - 1)) * math.log(2.0)


def viterbi_brute(w_seq, c, L: int, k: int, V: int) -> np.ndarray:
    """Minimum-energy path by enumeration, with the energy accumulated in fp32
    left to right (q_t(s) = sum_v fl(fl(w - c)^2), components added in order),
    ties broken towards the lowest final state, then the lowest state at each
    earlier step (reverse-lexicographic order of (s_{n-1}, ..., s_0))."""
    w32 = np.asarray(w_seq.detach().cpu().numpy() if hasattr(w_seq, "detach") else w_seq, np.float32).reshape(-1, V)
    c32 = np.asarray(c.detach().cpu().numpy() if hasattr(c, "detach") else c, np.float32).reshape(-1, V)
    D = k * V
    n = w32.shape[0]
    S = 1 << L
    q = np.zeros((n, S), np.float32)
    for v in range(V):
        d = (w32[:, v][:, None] - c32[:, v][None, :]).astype(np.float32)
        sq = (d * d).astype(np.float32)
        q = sq if v == 0 else (q + sq).astype(np.float32)
    paths = all_paths(L, D, n)
    acc = q[0][paths[:, 0]].astype(np.float32)
    for t in range(1, n):
        acc = (acc + q[t][paths[:, t]]).astype(np.float32)
    best = acc.min()
    cand = paths[acc == best]
    order = np.lexsort(tuple(cand[:, t] for t in range(n)))  # last key = s_{n-1} is primary
    return cand[order[0]]
