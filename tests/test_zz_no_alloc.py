"""bcjr_soft_codeword_noalloc, the entry point for callers that may not
allocate device memory (a plugin whose host application owns every device
allocation, a fixed device-memory budget, a latency-critical path), called
through the C ABI and compared with bcjr_soft_codeword on the same inputs,
twice in a row (the fixed scratch array keeps the previous call's contents).

This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from bcjr_sum_product_b200 import inputs as I
from bcjr_sum_product_b200 import lib
from helpers import assert_logZ, assert_soft

pytestmark = pytest.mark.gpu


def _noalloc():
    L = lib.load()
    fn = L.bcjr_soft_codeword_noalloc
    P = ctypes.c_void_p
    fn.argtypes = [P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, ctypes.c_float,
                   P, P, P]
    fn.restype = ctypes.c_int
    return fn


def _call(fn, w, c, L, k, V, T, soft, logZ):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(ctypes.c_void_p(w.data_ptr()), w.shape[0], w.shape[1], L, k, V, ctypes.c_void_p(c.data_ptr()),
              float(T), ctypes.c_void_p(soft.data_ptr()), ctypes.c_void_p(logZ.data_ptr()), stream)


@pytest.mark.parametrize("L,k,V,n_seq,n,T", [(8, 2, 1, 16, 64, 0.5), (12, 2, 1, 300, 256, 0.1),
                                             (16, 2, 1, 20, 64, 0.05), (12, 2, 2, 9, 40, 0.05),
                                             # 2^15 groups: the per-sequence state lives in the array too
                                             (16, 1, 1, 8, 64, 0.1),
                                             # 16 branches, where bcjr_soft_codeword runs a specialised kernel
                                             (16, 2, 2, 9, 32, 0.05)])
def test_noalloc_matches_allocating_entry_point(L, k, V, n_seq, n, T):
    fn = _noalloc()
    w, c, _ = I.random_case(L, k, V, n_seq, n * V, seed=4242 + L + V)
    w, c = w.cuda(), c.cuda()
    ref_soft, ref_logZ = lib.soft_codeword(w, c, L, k, V, T)
    ref_soft, ref_logZ = ref_soft.cpu().numpy(), ref_logZ.cpu().numpy()
    for _ in range(2):
        soft = torch.full_like(w, float("nan"))
        logZ = torch.full((n_seq,), float("nan"), device="cuda")
        assert _call(fn, w, c, L, k, V, T, soft, logZ) == lib.BCJR_OK
        torch.cuda.synchronize()
        assert lib.get_device_error() == 0
        assert_logZ(logZ.cpu().numpy(), ref_logZ, L, k * V, n)
        assert_soft(soft.cpu().numpy(), ref_soft, c.cpu())


def test_noalloc_rejects_problems_beyond_its_scratch():
    fn = _noalloc()
    # one L=16 sequence of 8192 weights needs 8192 * 16384 * 4 B = 512 MiB of history
    w = torch.zeros((1, 8192), device="cuda")
    c = torch.zeros(1 << 16, device="cuda")
    soft = torch.empty_like(w)
    logZ = torch.empty(1, device="cuda")
    assert _call(fn, w, c, 16, 2, 1, 0.5, soft, logZ) == lib.BCJR_ERR_UNSUPPORTED


def test_noalloc_against_the_oracle():
    """The entry point's own results against the fp64 oracle (L=12 and L=16 V=2)."""
    fn = _noalloc()
    for L, k, V, n_seq, n, T in ((12, 2, 1, 20, 48, 0.1), (16, 2, 2, 3, 16, 0.05)):
        w, c, _ = I.random_case(L, k, V, n_seq, n * V, seed=77 + L)
        soft = torch.empty((n_seq, n * V), device="cuda")
        logZ = torch.empty(n_seq, device="cuda")
        assert _call(fn, w.cuda(), c.cuda(), L, k, V, T, soft, logZ) == lib.BCJR_OK
        torch.cuda.synchronize()
        assert lib.get_device_error() == 0
        ref = oracle.soft(w, c, L, k, V, T)
        assert_logZ(logZ.cpu().numpy(), ref["logZ"], L, k * V, n)
        assert_soft(soft.cpu().numpy(), ref["soft"], c)
