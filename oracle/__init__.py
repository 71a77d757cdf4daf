"""CPU oracle for the BCJR forward-backward path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its
``cpu_baseline`` leg and ``--impl reference`` arm) may import this package.
The library under ``bcjr_sum_product_b200`` never does, and this package
imports nothing from it.

Two parts:

* ``bcjr_oracle.c`` (fp64, log-domain, OpenMP over sequences): soft codeword,
  logZ, posteriors and posterior argmax (``soft``), the vector-Jacobian product
  (``vjp``) and the fp32 Viterbi decode (``viterbi``).
* ``reference.py`` (NumPy): brute-force path enumeration, the dense
  transfer-matrix product and closed forms, used to pin the C oracle.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
against brute force, the transfer-matrix product, closed forms, identities
and finite differences; the pages print no worked numeric example, so no pin
comes from printed values.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bcjr_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc, OpenMP, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=gnu11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            i64, i32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_double
            lib.oracle_soft.argtypes = [P, i64, i64, i32, i32, i32, P, f64, P, P, P, P, P, i32]
            lib.oracle_vjp.argtypes = [P, i64, i64, i32, i32, i32, P, f64, P, P, P, P, P, P, i32]
            lib.oracle_viterbi.argtypes = [P, i64, i64, i32, i32, i32, P, P, P, i32]
            lib.oracle_pred_table.argtypes = [i32, i32, i32, P]
            for f in (lib.oracle_soft, lib.oracle_vjp, lib.oracle_viterbi, lib.oracle_pred_table):
                f.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f32(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _shape(w: np.ndarray, c: np.ndarray, V: int):
    n_seq, seq_len = w.shape
    if seq_len % V != 0:
        raise ValueError("sequence length must be a multiple of V")
    return n_seq, seq_len, seq_len // V


def default_threads() -> int:
    return int(os.environ.get("BCJR_ORACLE_THREADS", os.cpu_count() or 1))


def soft(w, c, L: int, k: int, V: int, T: float, posteriors: bool = False, nthreads: int = 0):
    """Soft codeword and logZ (fp64).

    Returns dict with ``soft`` [n_seq, len], ``logZ`` [n_seq], ``argmax``
    [n_seq, n] (lowest state on ties), ``top2`` [n_seq, n, 2] and, if asked,
    ``post`` [n_seq, n, 2^L].
    """
    lib = _load()
    w = _f32(w); c = _f32(c)
    n_seq, seq_len, n = _shape(w, c, V)
    S = 1 << L
    out_soft = np.zeros((n_seq, seq_len), np.float64)
    out_logZ = np.zeros(n_seq, np.float64)
    out_arg = np.zeros((n_seq, n), np.int32)
    out_top2 = np.zeros((n_seq, n, 2), np.float64)
    out_post = np.zeros((n_seq, n, S), np.float64) if posteriors else None
    rc = lib.oracle_soft(_ptr(w), n_seq, seq_len, L, k, V, _ptr(c), float(T), _ptr(out_soft), _ptr(out_logZ),
                         _ptr(out_post), _ptr(out_arg), _ptr(out_top2), nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle_soft failed ({rc})")
    res = {"soft": out_soft, "logZ": out_logZ, "argmax": out_arg, "top2": out_top2}
    if posteriors:
        res["post"] = out_post
    return res


def vjp(w, c, L: int, k: int, V: int, T: float, g, gZ=None, nthreads: int = 0):
    """VJP of sum_t g_t . w_hat_t (+ gZ . logZ): ``grad_w`` [n_seq, len] and
    ``grad_c`` (shape of c, summed over sequences), fp64; also ``logZ`` and
    ``Hbar`` (= E[sum_t g_t . c(s_t)]) per sequence."""
    lib = _load()
    w = _f32(w); c = _f32(c); g = _f32(g)
    gz = None if gZ is None else _f32(gZ).reshape(-1)
    n_seq, seq_len, n = _shape(w, c, V)
    grad_w = np.zeros((n_seq, seq_len), np.float64)
    grad_c = np.zeros(c.shape, np.float64)
    logZ = np.zeros(n_seq, np.float64)
    Hbar = np.zeros(n_seq, np.float64)
    rc = lib.oracle_vjp(_ptr(w), n_seq, seq_len, L, k, V, _ptr(c), float(T), _ptr(g), _ptr(gz),
                        _ptr(grad_w), _ptr(grad_c), _ptr(logZ), _ptr(Hbar), nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle_vjp failed ({rc})")
    return {"grad_w": grad_w, "grad_c": grad_c, "logZ": logZ, "Hbar": Hbar}


def viterbi(w, c, L: int, k: int, V: int, nthreads: int = 0):
    """fp32 Viterbi decode: ``states`` [n_seq, n] int32 and ``cost`` [n_seq] fp32."""
    lib = _load()
    w = _f32(w); c = _f32(c)
    n_seq, seq_len, n = _shape(w, c, V)
    states = np.zeros((n_seq, n), np.int32)
    cost = np.zeros(n_seq, np.float32)
    rc = lib.oracle_viterbi(_ptr(w), n_seq, seq_len, L, k, V, _ptr(c), _ptr(states), _ptr(cost),
                            nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle_viterbi failed ({rc})")
    return {"states": states, "cost": cost}


def pred_table(L: int, k: int, V: int) -> np.ndarray:
    """Predecessor lists [2^L, 2^(kV)] built from the successor rule."""
    lib = _load()
    B = 1 << (k * V)
    out = np.zeros((1 << L, B), np.int32)
    rc = lib.oracle_pred_table(L, k, V, _ptr(out))
    if rc != 0:
        raise RuntimeError(f"oracle_pred_table failed ({rc})")
    return out
