"""Thin ctypes binding of ``libbcjr.so`` (include/bcjr.h).

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels.  torch is used for device memory and streams.  There
is no CPU fallback: if the library cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbcjr.so")

BCJR_OK = 0
BCJR_ERR_INVALID_ARG = 1
BCJR_ERR_UNSUPPORTED = 2
BCJR_ERR_CUDA = 3
BCJR_ERR_TIMEOUT = 4
BCJR_ERR_NUMERIC = 5

EXPORTS = ("bcjr_soft_codeword", "bcjr_vjp", "viterbi_decode", "bcjr_posterior_argmax",
           "bcjr_get_device_error", "bcjr_launch_count", "bcjr_strerror", "bcjr_version")


class BcjrError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {strerror(status)} (status {status})")


_lock = threading.Lock()
_lib = None


def load(path: str = LIB_PATH):
    """Load the library (building it in-tree first if it is missing or stale)."""
    global _lib
    with _lock:
        if _lib is None:
            from . import build as _build
            if _build.needs_build():
                _build.build()
            if not os.path.exists(path):
                raise RuntimeError(f"libbcjr.so not found at {path}")
            lib = ctypes.CDLL(path)
            P, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
            lib.bcjr_soft_codeword.argtypes = [P, i64, i64, i32, i32, i32, P, f32, P, P, P]
            lib.bcjr_vjp.argtypes = [P, i64, i64, i32, i32, i32, P, f32, P, P, P, P, P]
            lib.viterbi_decode.argtypes = [P, i64, i64, i32, i32, i32, P, P, P, P]
            lib.bcjr_posterior_argmax.argtypes = [P, i64, i64, i32, i32, i32, P, f32, P, P]
            lib.bcjr_qat_step.argtypes = [P, P, i64, i64, i32, i32, i32, P, f32, f32, f32, P, P, P, P, P]
            lib.bcjr_get_device_error.argtypes = [P]
            lib.bcjr_strerror.argtypes = [i32]
            lib.bcjr_strerror.restype = ctypes.c_char_p
            lib.bcjr_version.argtypes = []
            lib.bcjr_version.restype = ctypes.c_char_p
            lib.bcjr_launch_count.argtypes = []
            lib.bcjr_launch_count.restype = ctypes.c_uint64
            for name in ("bcjr_soft_codeword", "bcjr_vjp", "viterbi_decode", "bcjr_posterior_argmax",
                         "bcjr_qat_step", "bcjr_get_device_error"):
                getattr(lib, name).restype = ctypes.c_int
            _lib = lib
    return _lib


def strerror(status: int) -> str:
    return load().bcjr_strerror(int(status)).decode()


def launch_count() -> int:
    """bcjr_launch_count: kernels the library has launched in this process."""
    return int(load().bcjr_launch_count())


def version() -> str:
    return load().bcjr_version().decode()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dev(t: torch.Tensor, name: str, dtype=torch.float32) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _check(rc: int, where: str):
    if rc != BCJR_OK:
        raise BcjrError(rc, where)


def soft_codeword(w: torch.Tensor, codebook: torch.Tensor, L: int, k: int, V: int, T: float,
                  out_soft: Optional[torch.Tensor] = None, out_logZ: Optional[torch.Tensor] = None,
                  stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """bcjr_soft_codeword: soft codeword [n_seq, len] and natural-log logZ [n_seq]."""
    _dev(w, "w"); _dev(codebook, "codebook")
    n_seq, seq_len = w.shape
    if out_soft is None:
        out_soft = torch.empty_like(w)
    if out_logZ is None:
        out_logZ = torch.empty(n_seq, device=w.device, dtype=torch.float32)
    rc = load().bcjr_soft_codeword(_ptr(w), n_seq, seq_len, L, k, V, _ptr(codebook), float(T), _ptr(out_soft),
                                   _ptr(out_logZ), _stream(stream))
    _check(rc, "bcjr_soft_codeword")
    return out_soft, out_logZ


def vjp(w: torch.Tensor, codebook: torch.Tensor, L: int, k: int, V: int, T: float, grad_soft: torch.Tensor,
        grad_logZ: Optional[torch.Tensor] = None, grad_w: Optional[torch.Tensor] = None,
        grad_codebook: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """bcjr_vjp: (dl/dw [n_seq, len], dl/dcodebook [2^L(, V)])."""
    _dev(w, "w"); _dev(codebook, "codebook"); _dev(grad_soft, "grad_soft")
    if grad_logZ is not None:
        _dev(grad_logZ, "grad_logZ")
    n_seq, seq_len = w.shape
    if grad_w is None:
        grad_w = torch.empty_like(w)
    if grad_codebook is None:
        grad_codebook = torch.empty_like(codebook)
    rc = load().bcjr_vjp(_ptr(w), n_seq, seq_len, L, k, V, _ptr(codebook), float(T), _ptr(grad_soft),
                         _ptr(grad_logZ), _ptr(grad_w), _ptr(grad_codebook), _stream(stream))
    _check(rc, "bcjr_vjp")
    return grad_w, grad_codebook


def qat_step(w: torch.Tensor, w_target: torch.Tensor, codebook: torch.Tensor, L: int, k: int, V: int, T: float,
             lr_w: float, lr_c: float = 0.0, out_soft: Optional[torch.Tensor] = None,
             out_loss: Optional[torch.Tensor] = None, grad_w: Optional[torch.Tensor] = None,
             grad_codebook: Optional[torch.Tensor] = None,
             stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor, torch.Tensor]:
    """bcjr_qat_step: one self-reconstruction QAT step; updates ``w`` (and the
    codebook when ``lr_c`` != 0) in place and returns (w_hat, loss per sequence,
    dl/dw, dl/dcodebook), all taken before the update."""
    _dev(w, "w"); _dev(w_target, "w_target"); _dev(codebook, "codebook")
    n_seq, seq_len = w.shape
    if tuple(w_target.shape) != (n_seq, seq_len):
        raise ValueError("w_target must have the shape of w")
    if out_soft is None:
        out_soft = torch.empty_like(w)
    if out_loss is None:
        out_loss = torch.empty(n_seq, device=w.device, dtype=torch.float32)
    if grad_w is None:
        grad_w = torch.empty_like(w)
    if grad_codebook is None:
        grad_codebook = torch.empty_like(codebook)
    rc = load().bcjr_qat_step(_ptr(w), _ptr(w_target), n_seq, seq_len, L, k, V, _ptr(codebook), float(T),
                              float(lr_w), float(lr_c), _ptr(out_soft), _ptr(out_loss), _ptr(grad_w),
                              _ptr(grad_codebook), _stream(stream))
    _check(rc, "bcjr_qat_step")
    return out_soft, out_loss, grad_w, grad_codebook


def viterbi_decode(w: torch.Tensor, codebook: torch.Tensor, L: int, k: int, V: int,
                   out_states: Optional[torch.Tensor] = None, out_cost: Optional[torch.Tensor] = None,
                   stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """viterbi_decode: (states [n_seq, n] int32, cost [n_seq] fp32)."""
    _dev(w, "w"); _dev(codebook, "codebook")
    n_seq, seq_len = w.shape
    n = seq_len // V
    if out_states is None:
        out_states = torch.empty((n_seq, n), device=w.device, dtype=torch.int32)
    if out_cost is None:
        out_cost = torch.empty(n_seq, device=w.device, dtype=torch.float32)
    rc = load().viterbi_decode(_ptr(w), n_seq, seq_len, L, k, V, _ptr(codebook), _ptr(out_states),
                               _ptr(out_cost), _stream(stream))
    _check(rc, "viterbi_decode")
    return out_states, out_cost


def posterior_argmax(w: torch.Tensor, codebook: torch.Tensor, L: int, k: int, V: int, T: float,
                     out_argmax: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """bcjr_posterior_argmax: argmax_s p_t(s) per step, [n_seq, n] int32."""
    _dev(w, "w"); _dev(codebook, "codebook")
    n_seq, seq_len = w.shape
    n = seq_len // V
    if out_argmax is None:
        out_argmax = torch.empty((n_seq, n), device=w.device, dtype=torch.int32)
    rc = load().bcjr_posterior_argmax(_ptr(w), n_seq, seq_len, L, k, V, _ptr(codebook), float(T),
                                      _ptr(out_argmax), _stream(stream))
    _check(rc, "bcjr_posterior_argmax")
    return out_argmax


def get_device_error(stream=None) -> int:
    return int(load().bcjr_get_device_error(_stream(stream)))


def soft_codeword_noalloc(w: torch.Tensor, codebook: torch.Tensor, L: int, k: int, V: int, T: float,
                          out_soft: Optional[torch.Tensor] = None, out_logZ: Optional[torch.Tensor] = None,
                          stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """bcjr_soft_codeword_noalloc: as soft_codeword, but the library allocates
    nothing (its scratch is a fixed 64 MiB device array shared by all calls on a
    device; calls that overlap on the GPU race on it).  For callers that may not
    allocate device memory; the output tensors are still the caller's."""
    _dev(w, "w"); _dev(codebook, "codebook")
    n_seq, seq_len = w.shape
    if out_soft is None:
        out_soft = torch.empty_like(w)
    if out_logZ is None:
        out_logZ = torch.empty(n_seq, device=w.device, dtype=torch.float32)
    fn = load().bcjr_soft_codeword_noalloc
    P = ctypes.c_void_p
    fn.argtypes = [P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, ctypes.c_float,
                   P, P, P]
    fn.restype = ctypes.c_int
    rc = fn(_ptr(w), n_seq, seq_len, L, k, V, _ptr(codebook), float(T), _ptr(out_soft), _ptr(out_logZ),
            _stream(stream))
    _check(rc, "bcjr_soft_codeword_noalloc")
    return out_soft, out_logZ
