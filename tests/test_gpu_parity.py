"""GPU (C-ABI) vs CPU oracle, element by element, on small seeded cases that
span several thread tiles, ragged sequence counts, n = 1, D = L and both V.

Every call goes through libbcjr.so (include/bcjr.h) via the ctypes binding.
"""
import ctypes
import json
import os

import numpy as np
import pytest
import torch

import oracle
from bcjr_sum_product_b200 import inputs as I
from bcjr_sum_product_b200 import lib
from helpers import assert_grad, assert_logZ, assert_soft, unique_argmax_mask

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _run_all(w, c, L, k, V, T, g, gZ):
    wd, cd, gd, gzd = (x.to(DEV).contiguous() for x in (w, c, g, gZ))
    soft, logZ = lib.soft_codeword(wd, cd, L, k, V, T)
    gw, gc = lib.vjp(wd, cd, L, k, V, T, gd, gzd)
    am = lib.posterior_argmax(wd, cd, L, k, V, T)
    st, cost = lib.viterbi_decode(wd, cd, L, k, V)
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    return {k2: v.cpu().numpy() for k2, v in dict(soft=soft, logZ=logZ, gw=gw, gc=gc, am=am, st=st, cost=cost).items()}


def _compare(w, c, L, k, V, T, g, gZ, gpu):
    n = w.shape[1] // V
    D = k * V
    ref = oracle.soft(w, c, L, k, V, T)
    assert_logZ(gpu["logZ"], ref["logZ"], L, D, n)
    assert_soft(gpu["soft"], ref["soft"], c)
    rv = oracle.vjp(w, c, L, k, V, T, g, gZ)
    assert_grad(gpu["gw"], rv["grad_w"], "grad_w")
    assert_grad(gpu["gc"].reshape(rv["grad_c"].shape), rv["grad_c"], "grad_c")
    mask = unique_argmax_mask(ref["top2"])
    np.testing.assert_array_equal(gpu["am"][mask], ref["argmax"][mask])
    vt = oracle.viterbi(w, c, L, k, V)
    np.testing.assert_array_equal(gpu["st"], vt["states"])
    np.testing.assert_array_equal(gpu["cost"], vt["cost"])


def test_tiny_workload():
    """L=8, k=2, V=1, 16 x 64, T=0.5: soft codeword, logZ, VJP, argmax, Viterbi."""
    inp = I.make("tiny")
    gZ = torch.zeros(inp.w.shape[0])
    gpu = _run_all(inp.w, inp.c, 8, 2, 1, 0.5, inp.g, gZ)
    _compare(inp.w, inp.c, 8, 2, 1, 0.5, inp.g, gZ, gpu)


def test_tiny_prefix_golden():
    with open(os.path.join(os.path.dirname(__file__), "golden", "tiny_prefix6.json")) as f:
        gold = json.load(f)
    inp = I.make("tiny")
    w6 = inp.w[:, :6].contiguous().to(DEV)
    soft, logZ = lib.soft_codeword(w6, inp.c.to(DEV), 8, 2, 1, 0.5)
    assert_logZ(logZ.cpu().numpy(), gold["logZ"], 8, 2, 6)
    assert_soft(soft.cpu().numpy(), np.array(gold["soft"]), inp.c)


CASES = [
    # L, k, V, n_seq, n, T
    (4, 2, 1, 37, 9, 0.7),
    (4, 1, 2, 5, 6, 0.3),
    (5, 1, 1, 33, 17, 1.3),
    (6, 3, 2, 7, 5, 0.2),
    (6, 6, 1, 3, 8, 0.5),      # D = L: independent softmax per step
    (4, 4, 1, 3, 5, 0.4),      # D = L
    (8, 2, 1, 50, 40, 0.05),
    (10, 2, 1, 20, 64, 0.1),
    (12, 2, 2, 6, 32, 0.05),
    (6, 2, 1, 3, 1, 0.5),      # a single step
    (7, 1, 1, 9, 3, 2.0),
    (9, 2, 2, 11, 7, 0.01),    # low temperature
    (16, 2, 1, 2, 12, 0.05),   # 65536 states, short
    (16, 2, 2, 2, 6, 0.05),    # 65536 states, 16 branches
]


@pytest.mark.parametrize("L,k,V,n_seq,n,T", CASES)
def test_random_cases(L, k, V, n_seq, n, T):
    w, c, g = I.random_case(L, k, V, n_seq, n * V, seed=1000 + 31 * L + 7 * n + V)
    gZ = torch.randn(n_seq, generator=torch.Generator().manual_seed(5))
    gpu = _run_all(w, c, L, k, V, T, g, gZ)
    _compare(w, c, L, k, V, T, g, gZ, gpu)


def test_empty_sequence_count_is_noop_and_zeroes_codebook_gradient():
    c = torch.randn(256, device=DEV)
    w = torch.zeros((0, 64), device=DEV)
    soft, logZ = lib.soft_codeword(w, c, 8, 2, 1, 0.5)
    gc = torch.full_like(c, 7.0)
    gw, gc = lib.vjp(w, c, 8, 2, 1, 0.5, torch.zeros_like(w), grad_codebook=gc)
    torch.cuda.synchronize()
    assert soft.numel() == 0 and float(gc.abs().max()) == 0.0


@pytest.mark.parametrize("L,k,V", [(8, 2, 1), (16, 2, 1), (16, 2, 2)])
def test_nan_sequence_is_isolated_and_flagged(L, k, V):
    """A NaN weight makes its sequence's outputs NaN, leaves the others exact,
    and the per-step posterior-mass check records BCJR_ERR_NUMERIC, which the
    next read clears (generic, L=16 V=1 and V=2 kernels; soft and VJP)."""
    w, c, g = I.random_case(L, k, V, 5, 32 * V, seed=77)
    w[2, 5] = float("nan")
    wd, cd, gd = w.to(DEV), c.to(DEV), g.to(DEV)
    assert lib.get_device_error() == 0
    soft, logZ = lib.soft_codeword(wd, cd, L, k, V, 0.3)
    assert lib.get_device_error() == lib.BCJR_ERR_NUMERIC
    assert lib.get_device_error() == 0
    gw, _ = lib.vjp(wd, cd, L, k, V, 0.3, gd)
    assert lib.get_device_error() == lib.BCJR_ERR_NUMERIC
    soft, logZ, gw = soft.cpu().numpy(), logZ.cpu().numpy(), gw.cpu().numpy()
    assert np.isnan(logZ[2]) and np.isnan(soft[2]).any() and np.isnan(gw[2]).any()
    ok = [0, 1, 3, 4]
    ref = oracle.soft(w[ok], c, L, k, V, 0.3)
    assert_logZ(logZ[ok], ref["logZ"], L, k * V, 32)
    assert_soft(soft[ok], ref["soft"], c)
    rv = oracle.vjp(w[ok], c, L, k, V, 0.3, g[ok])
    assert_grad(gw[ok], rv["grad_w"], "grad_w")
    # a clean call afterwards leaves the flag clear
    lib.soft_codeword(wd[ok[0]:ok[0] + 1].contiguous(), cd, L, k, V, 0.3)
    assert lib.get_device_error() == 0


def test_runs_are_bit_identical():
    w, c, g = I.random_case(12, 2, 1, 40, 64, seed=88)
    wd, cd, gd = w.to(DEV), c.to(DEV), g.to(DEV)
    a = lib.soft_codeword(wd, cd, 12, 2, 1, 0.1)
    b = lib.soft_codeword(wd, cd, 12, 2, 1, 0.1)
    ga = lib.vjp(wd, cd, 12, 2, 1, 0.1, gd)
    gb = lib.vjp(wd, cd, 12, 2, 1, 0.1, gd)
    for x, y in zip(a + ga, b + gb):
        assert torch.equal(x, y)


def test_invalid_pointers_rejected():
    L = lib.load()
    host = np.zeros(64, np.float32)
    cd = torch.randn(256, device=DEV)
    out = torch.empty((1, 64), device=DEV)
    rc = L.bcjr_soft_codeword(host.ctypes.data_as(ctypes.c_void_p), 1, 64, 8, 2, 1,
                              ctypes.c_void_p(cd.data_ptr()), 0.5, ctypes.c_void_p(out.data_ptr()), None, None)
    assert rc == lib.BCJR_ERR_INVALID_ARG
    rc = L.bcjr_soft_codeword(ctypes.c_void_p(out.data_ptr() + 2), 1, 64, 8, 2, 1,
                              ctypes.c_void_p(cd.data_ptr()), 0.5, ctypes.c_void_p(out.data_ptr()), None, None)
    assert rc == lib.BCJR_ERR_INVALID_ARG


def test_forced_allocation_failure(monkeypatch):
    w, c, g = I.random_case(8, 2, 1, 2, 16, seed=3)
    monkeypatch.setenv("BCJR_FAULT_ALLOC", "1")
    with pytest.raises(lib.BcjrError) as e:
        lib.soft_codeword(w.to(DEV), c.to(DEV), 8, 2, 1, 0.5)
    assert e.value.status == lib.BCJR_ERR_CUDA
    monkeypatch.delenv("BCJR_FAULT_ALLOC")
    lib.soft_codeword(w.to(DEV), c.to(DEV), 8, 2, 1, 0.5)
    torch.cuda.synchronize()


def test_l16_block_kernel_matches_generic_kernel(monkeypatch):
    """The specialised L=16, k=2, V=1 kernels against the generic kernels on
    300 sequences (more than one per CTA) of 64 steps, T=0.05, with gZ."""
    w, c, g = I.random_case(16, 2, 1, 300, 64, seed=909)
    gZ = torch.randn(300, generator=torch.Generator().manual_seed(6))
    wd, cd, gd, gzd = w.to(DEV), c.to(DEV), g.to(DEV), gZ.to(DEV)
    fast = [x.cpu().numpy() for x in lib.soft_codeword(wd, cd, 16, 2, 1, 0.05) + lib.vjp(wd, cd, 16, 2, 1, 0.05, gd, gzd)]
    am_fast = lib.posterior_argmax(wd, cd, 16, 2, 1, 0.05).cpu().numpy()
    monkeypatch.setenv("BCJR_GENERIC_ONLY", "1")
    gen = [x.cpu().numpy() for x in lib.soft_codeword(wd, cd, 16, 2, 1, 0.05) + lib.vjp(wd, cd, 16, 2, 1, 0.05, gd, gzd)]
    am_gen = lib.posterior_argmax(wd, cd, 16, 2, 1, 0.05).cpu().numpy()
    assert_soft(fast[0], gen[0], c)
    assert_logZ(fast[1], gen[1], 16, 2, 64)
    assert_grad(fast[2], gen[2], "grad_w")
    assert_grad(fast[3], gen[3], "grad_c")
    assert (am_fast == am_gen).mean() > 0.999
    # and both against the oracle on a few rows
    rows = [0, 147, 148, 299]
    ref = oracle.soft(w[rows], c, 16, 2, 1, 0.05)
    assert_logZ(fast[1][rows], ref["logZ"], 16, 2, 64)
    assert_soft(fast[0][rows], ref["soft"], c)
    rv = oracle.vjp(w[rows], c, 16, 2, 1, 0.05, g[rows], gZ[rows])
    assert_grad(fast[2][rows], rv["grad_w"], "grad_w")


def test_l16_vector_kernel_matches_generic_kernel(monkeypatch):
    """The specialised L=16, k=2, V=2 kernels against the generic kernels on
    300 sequences (more than one per CTA) of 48 steps (96 weights), T=0.05,
    with gZ; then against the oracle on a few rows."""
    w, c, g = I.random_case(16, 2, 2, 300, 96, seed=919)
    gZ = torch.randn(300, generator=torch.Generator().manual_seed(7))
    wd, cd, gd, gzd = w.to(DEV), c.to(DEV), g.to(DEV), gZ.to(DEV)
    fast = [x.cpu().numpy() for x in lib.soft_codeword(wd, cd, 16, 2, 2, 0.05) + lib.vjp(wd, cd, 16, 2, 2, 0.05, gd, gzd)]
    am_fast = lib.posterior_argmax(wd, cd, 16, 2, 2, 0.05).cpu().numpy()
    assert lib.get_device_error() == 0
    monkeypatch.setenv("BCJR_GENERIC_ONLY", "1")
    gen = [x.cpu().numpy() for x in lib.soft_codeword(wd, cd, 16, 2, 2, 0.05) + lib.vjp(wd, cd, 16, 2, 2, 0.05, gd, gzd)]
    am_gen = lib.posterior_argmax(wd, cd, 16, 2, 2, 0.05).cpu().numpy()
    assert_soft(fast[0], gen[0], c)
    assert_logZ(fast[1], gen[1], 16, 4, 48)
    assert_grad(fast[2], gen[2], "grad_w")
    assert_grad(fast[3], gen[3], "grad_c")
    assert (am_fast == am_gen).mean() > 0.999
    rows = [0, 147, 148, 299]
    ref = oracle.soft(w[rows], c, 16, 2, 2, 0.05)
    assert_logZ(fast[1][rows], ref["logZ"], 16, 4, 48)
    assert_soft(fast[0][rows], ref["soft"], c)
    rv = oracle.vjp(w[rows], c, 16, 2, 2, 0.05, g[rows], gZ[rows])
    assert_grad(fast[2][rows], rv["grad_w"], "grad_w")
    mask = unique_argmax_mask(ref["top2"])
    np.testing.assert_array_equal(am_fast[rows][mask], ref["argmax"][mask])


def test_l16_vector_kernel_longest(monkeypatch):
    """V=2 at len = 8192 (4096 steps, the longest supported), biased upstream
    gradient: specialised against generic kernels."""
    w, c, g = I.random_case(16, 2, 2, 2, 8192, seed=929)
    g[1] += 1.0
    wd, cd, gd = w.to(DEV), c.to(DEV), g.to(DEV)
    fast = [x.cpu().numpy() for x in lib.soft_codeword(wd, cd, 16, 2, 2, 0.1) + lib.vjp(wd, cd, 16, 2, 2, 0.1, gd)]
    assert lib.get_device_error() == 0
    monkeypatch.setenv("BCJR_GENERIC_ONLY", "1")
    gen = [x.cpu().numpy() for x in lib.soft_codeword(wd, cd, 16, 2, 2, 0.1) + lib.vjp(wd, cd, 16, 2, 2, 0.1, gd)]
    assert_soft(fast[0], gen[0], c)
    assert_logZ(fast[1], gen[1], 16, 4, 4096)
    assert_grad(fast[2], gen[2], "grad_w")
    assert_grad(fast[3], gen[3], "grad_c")


def test_l16_viterbi_matches_generic_and_oracle(monkeypatch):
    """The block-layout L=16 Viterbi against the generic kernel (bit-exact) on
    40 sequences of 96 steps, including exact ties from a coarse codebook."""
    w, c, _ = I.random_case(16, 2, 1, 40, 96, seed=515)
    c[::7] = torch.round(c[::7] * 4) / 4
    w[:5] = torch.round(w[:5] * 4) / 4
    wd, cd = w.to(DEV), c.to(DEV)
    s_fast, c_fast = lib.viterbi_decode(wd, cd, 16, 2, 1)
    monkeypatch.setenv("BCJR_GENERIC_ONLY", "1")
    s_gen, c_gen = lib.viterbi_decode(wd, cd, 16, 2, 1)
    torch.cuda.synchronize()
    assert torch.equal(s_fast, s_gen) and torch.equal(c_fast, c_gen)
    ref = oracle.viterbi(w[:6], c, 16, 2, 1)
    np.testing.assert_array_equal(s_fast[:6].cpu().numpy(), ref["states"])
    np.testing.assert_array_equal(c_fast[:6].cpu().numpy(), ref["cost"])


def test_l16v2_viterbi_matches_generic_and_oracle(monkeypatch):
    """The L=16, V=2 Viterbi (16 branches, 4-bit backpointers, batched traceback)
    against the generic kernel (bit-exact) on 40 sequences of 64 steps, with exact
    ties from a coarse codebook, and against the oracle on 6 of them."""
    w, c, _ = I.random_case(16, 2, 2, 40, 128, seed=516)
    c[::5] = torch.round(c[::5] * 4) / 4
    w[:5] = torch.round(w[:5] * 4) / 4
    wd, cd = w.to(DEV), c.to(DEV)
    s_fast, c_fast = lib.viterbi_decode(wd, cd, 16, 2, 2)
    monkeypatch.setenv("BCJR_GENERIC_ONLY", "1")
    s_gen, c_gen = lib.viterbi_decode(wd, cd, 16, 2, 2)
    torch.cuda.synchronize()
    assert torch.equal(s_fast, s_gen) and torch.equal(c_fast, c_gen)
    ref = oracle.viterbi(w[:6], c, 16, 2, 2)
    np.testing.assert_array_equal(s_fast[:6].cpu().numpy(), ref["states"])
    np.testing.assert_array_equal(c_fast[:6].cpu().numpy(), ref["cost"])


def test_longest_sequences(monkeypatch):
    """len = 8192 (the largest supported): L=12 against the oracle, and L=16
    (whose per-CTA histories are 0.5-1 GB, so fewer CTAs are resident) against
    the generic kernels."""
    w, c, g = I.random_case(12, 2, 1, 3, 8192, seed=777)
    gpu = _run_all(w, c, 12, 2, 1, 0.2, g, torch.zeros(3))
    _compare(w, c, 12, 2, 1, 0.2, g, torch.zeros(3), gpu)
    # an upstream gradient with a non-zero mean makes the prefix and suffix
    # expectations grow linearly along the sequence
    gb = g[:1] + 1.0
    gpu = _run_all(w[:1], c, 12, 2, 1, 0.05, gb, torch.ones(1))
    _compare(w[:1], c, 12, 2, 1, 0.05, gb, torch.ones(1), gpu)
    # at T = 0.01 the posterior of a near tie depends on log values of a few
    # hundred, whose fp32 rounding differs between the two sweeps
    w, c, g = I.random_case(10, 2, 1, 1, 8192, seed=9)
    gb = g + 1.0
    gpu = _run_all(w, c, 10, 2, 1, 0.01, gb, torch.ones(1))
    _compare(w, c, 10, 2, 1, 0.01, gb, torch.ones(1), gpu)
    w, c, g = I.random_case(16, 2, 1, 2, 8192, seed=778)
    g[1] += 1.0
    wd, cd, gd = w.to(DEV), c.to(DEV), g.to(DEV)
    fast = [x.cpu().numpy() for x in lib.soft_codeword(wd, cd, 16, 2, 1, 0.1) + lib.vjp(wd, cd, 16, 2, 1, 0.1, gd)]
    vs_fast = lib.viterbi_decode(wd, cd, 16, 2, 1)[0].cpu()
    monkeypatch.setenv("BCJR_GENERIC_ONLY", "1")
    gen = [x.cpu().numpy() for x in lib.soft_codeword(wd, cd, 16, 2, 1, 0.1) + lib.vjp(wd, cd, 16, 2, 1, 0.1, gd)]
    vs_gen = lib.viterbi_decode(wd, cd, 16, 2, 1)[0].cpu()
    assert_soft(fast[0], gen[0], c)
    assert_logZ(fast[1], gen[1], 16, 2, 8192)
    assert_grad(fast[2], gen[2], "grad_w")
    assert_grad(fast[3], gen[3], "grad_c")
    assert torch.equal(vs_fast, vs_gen)
