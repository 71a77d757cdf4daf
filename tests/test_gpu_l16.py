"""The specialised L=16 kernels and their measured alternatives: the two-CTA
cluster VJP against the single-CTA VJP, the VJP backward's codeword ring
against codewords streamed from L2, the posterior-space backward sweeps against
the log-domain ones, all against the oracle; run-to-run bit reproducibility of
every L=16 kernel (soft codeword, VJP, posterior argmax and Viterbi; V=1 and
V=2); and the ring's bounded wait, made to run out by a test hook, reporting
BCJR_ERR_TIMEOUT with the context still usable.

All calls go through libbcjr.so (include/bcjr.h) via the ctypes binding.
"""
import numpy as np
import pytest
import torch

import oracle
from bcjr_sum_product_b200 import inputs as I
from bcjr_sum_product_b200 import lib
from helpers import assert_grad, assert_logZ, assert_soft

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_l16_cluster_vjp_matches_single_cta_vjp(monkeypatch):
    """300 sequences (several per cluster and per CTA) of 64 steps at T=0.05
    with a logZ gradient: the cluster kernel against the single-CTA kernel, and
    both against the oracle on rows that fall on different clusters."""
    w, c, g = I.random_case(16, 2, 1, 300, 64, seed=4242)
    gZ = torch.randn(300, generator=torch.Generator().manual_seed(8))
    wd, cd, gd, gzd = w.to(DEV), c.to(DEV), g.to(DEV), gZ.to(DEV)
    gw_cta, gc_cta = (x.cpu().numpy() for x in lib.vjp(wd, cd, 16, 2, 1, 0.05, gd, gzd))
    assert lib.get_device_error() == 0
    monkeypatch.setenv("BCJR_L16_VJP", "cluster")
    gw_cl, gc_cl = (x.cpu().numpy() for x in lib.vjp(wd, cd, 16, 2, 1, 0.05, gd, gzd))
    assert lib.get_device_error() == 0
    assert_grad(gw_cl, gw_cta, "grad_w")
    assert_grad(gc_cl, gc_cta, "grad_c")
    rows = [0, 1, 73, 74, 148, 299]
    rv = oracle.vjp(w[rows], c, 16, 2, 1, 0.05, g[rows], gZ[rows])
    assert_grad(gw_cl[rows], rv["grad_w"], "grad_w")
    assert_grad(gw_cta[rows], rv["grad_w"], "grad_w")
    sub = [x.to(DEV) for x in (w[rows], g[rows], gZ[rows])]
    _, gc_sub = lib.vjp(sub[0], cd, 16, 2, 1, 0.05, sub[1], sub[2])
    assert_grad(gc_sub.cpu().numpy(), rv["grad_c"], "grad_c")


@pytest.mark.parametrize("variant", [{}, {"BCJR_L16_VJP": "cluster"}, {"BCJR_L16_VJP": "l2"}, {"BCJR_L16_BWD": "post"}])
def test_l16_vjp_single_sequence_and_short(monkeypatch, variant):
    """One sequence (one CTA or cluster busy, the rest idle) and n = 1 and 2 steps."""
    for key, val in variant.items():
        monkeypatch.setenv(key, val)
    for n_seq, n, T in ((1, 40, 0.1), (3, 1, 0.5), (5, 2, 0.05)):
        w, c, g = I.random_case(16, 2, 1, n_seq, n, seed=31 + n)
        gZ = torch.randn(n_seq, generator=torch.Generator().manual_seed(n))
        gw, gc = lib.vjp(w.to(DEV), c.to(DEV), 16, 2, 1, T, g.to(DEV), gZ.to(DEV))
        assert lib.get_device_error() == 0
        rv = oracle.vjp(w, c, 16, 2, 1, T, g, gZ)
        assert_grad(gw.cpu().numpy(), rv["grad_w"], "grad_w")
        assert_grad(gc.cpu().numpy(), rv["grad_c"], "grad_c")


def _twice(fn):
    a = [x.clone() for x in fn()]
    b = [x.clone() for x in fn()]
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    return a, b


@pytest.mark.parametrize("variant", [{}, {"BCJR_L16_VJP": "cluster"}, {"BCJR_L16_VJP": "l2"}, {"BCJR_L16_BWD": "post"},
                                     {"BCJR_L16_BWD": "log"}, {"BCJR_L16_EX2": "fma"}])
def test_l16_v1_runs_are_bit_identical(monkeypatch, variant):
    """L=16, k=2, V=1: soft codeword, logZ, argmax and VJP of 200 sequences
    (more than one per CTA) give the same bits on every run."""
    for key, val in variant.items():
        monkeypatch.setenv(key, val)
    w, c, g = I.random_case(16, 2, 1, 200, 48, seed=606)
    wd, cd, gd = w.to(DEV), c.to(DEV), g.to(DEV)
    a, b = _twice(lambda: list(lib.soft_codeword(wd, cd, 16, 2, 1, 0.05)) +
                  [lib.posterior_argmax(wd, cd, 16, 2, 1, 0.05)] + list(lib.vjp(wd, cd, 16, 2, 1, 0.05, gd)))
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_l16_v2_runs_are_bit_identical():
    """L=16, k=2, V=2: soft codeword, logZ, argmax and VJP of 200 sequences."""
    w, c, g = I.random_case(16, 2, 2, 200, 64, seed=607)
    wd, cd, gd = w.to(DEV), c.to(DEV), g.to(DEV)
    a, b = _twice(lambda: list(lib.soft_codeword(wd, cd, 16, 2, 2, 0.05)) +
                  [lib.posterior_argmax(wd, cd, 16, 2, 2, 0.05)] + list(lib.vjp(wd, cd, 16, 2, 2, 0.05, gd)))
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("V", [1, 2])
def test_l16_viterbi_runs_are_bit_identical(V):
    w, c, _ = I.random_case(16, 2, V, 200, 64 * V, seed=608 + V)
    wd, cd = w.to(DEV), c.to(DEV)
    a, b = _twice(lambda: list(lib.viterbi_decode(wd, cd, 16, 2, V)))
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("T", [1.0, 0.05, 0.01, 0.001])
def test_l16_posterior_space_and_log_backward_agree_with_oracle(monkeypatch, T):
    """Both backward sweeps of the L=16 V=1 kernels (posterior space and log
    domain, each selected for the soft codeword and the VJP), and the soft
    pass with one forward exponential per group on the FMA pipe, against the oracle on 12 sequences of 80 steps,
    with a logZ gradient: soft codeword, logZ, grad_w and grad_c."""
    w, c, g = I.random_case(16, 2, 1, 12, 80, seed=700 + int(1000 * T))
    gZ = torch.randn(12, generator=torch.Generator().manual_seed(9))
    ref = oracle.soft(w, c, 16, 2, 1, T)
    rv = oracle.vjp(w, c, 16, 2, 1, T, g, gZ)
    wd, cd, gd, gzd = w.to(DEV), c.to(DEV), g.to(DEV), gZ.to(DEV)
    for bwd, ex2 in (("post", "mufu"), ("log", "mufu"), ("post", "fma")):
        monkeypatch.setenv("BCJR_L16_BWD", bwd)
        monkeypatch.setenv("BCJR_L16_EX2", ex2)
        soft, logZ = lib.soft_codeword(wd, cd, 16, 2, 1, T)
        gw, gc = lib.vjp(wd, cd, 16, 2, 1, T, gd, gzd)
        assert lib.get_device_error() == 0
        assert_logZ(logZ.cpu().numpy(), ref["logZ"], 16, 2, 80)
        assert_soft(soft.cpu().numpy(), ref["soft"], c)
        assert_grad(gw.cpu().numpy(), rv["grad_w"], "grad_w")
        assert_grad(gc.cpu().numpy(), rv["grad_c"], "grad_c")


def test_l16_block_argmax_against_oracle():
    """Posterior argmax of the L=16 V=1 block kernel against the oracle on 24
    sequences at T = 0.05 and 0.01, on every step whose oracle top-two
    posteriors differ by more than 1e-4 (elsewhere several answers are valid)."""
    w, c, _ = I.random_case(16, 2, 1, 24, 96, seed=612)
    for T in (0.05, 0.01):
        am = lib.posterior_argmax(w.to(DEV), c.to(DEV), 16, 2, 1, T).cpu().numpy()
        ref = oracle.soft(w, c, 16, 2, 1, T)
        mask = (ref["top2"][..., 0] - ref["top2"][..., 1]) > 1e-4
        assert mask.mean() > 0.5
        np.testing.assert_array_equal(am[mask], ref["argmax"][mask])


@pytest.fixture(scope="module")
def longest_low_t_case():
    """Two sequences of len 8192 (the longest supported) at T = 0.01, the
    second with a biased upstream gradient, and their oracle results (about
    13 GB of host memory and two minutes per sequence)."""
    w, c, g = I.random_case(16, 2, 1, 2, 8192, seed=781)
    g[1] += 1.0
    ref = oracle.soft(w, c, 16, 2, 1, 0.01, nthreads=2)
    rv = oracle.vjp(w, c, 16, 2, 1, 0.01, g, nthreads=2)
    return w, c, g, ref, rv


@pytest.mark.parametrize("variant", [{}, {"BCJR_L16_BWD": "post"}, {"BCJR_L16_BWD": "log"}, {"BCJR_L16_VJP": "l2"},
                                     {"BCJR_L16_EX2": "fma"}, {"BCJR_GENERIC_ONLY": "1"}])
def test_l16_variants_longest_sequences_low_temperature(monkeypatch, variant, longest_low_t_case):
    """len = 8192 at T = 0.01 with a biased upstream gradient, where the log
    values reach hundreds of bits: every L=16 V=1 kernel variant (and the
    generic kernels) against the oracle."""
    w, c, g, ref, rv = longest_low_t_case
    for key, val in variant.items():
        monkeypatch.setenv(key, val)
    wd, cd, gd = w.to(DEV), c.to(DEV), g.to(DEV)
    soft, logZ = lib.soft_codeword(wd, cd, 16, 2, 1, 0.01)
    gw, gc = lib.vjp(wd, cd, 16, 2, 1, 0.01, gd)
    assert lib.get_device_error() == 0
    assert_soft(soft.cpu().numpy(), ref["soft"], c)
    assert_logZ(logZ.cpu().numpy(), ref["logZ"], 16, 2, 8192)
    assert_grad(gw.cpu().numpy(), rv["grad_w"], "grad_w")
    assert_grad(gc.cpu().numpy(), rv["grad_c"], "grad_c")


@pytest.mark.parametrize("variant", [{}, {"BCJR_L16_BWD": "post"}, {"BCJR_L16_BWD": "log"}])
@pytest.mark.parametrize("n,K", [(100, 7), (100, 10), (37, 1), (37, 37), (64, 8)])
def test_l16_checkpointed_histories_are_bit_identical(monkeypatch, variant, n, K):
    """Segments of K steps recomputed from checkpoints (ragged last segment,
    K = 1, K = n) give the same bits as full histories: the recompute repeats
    the forward with the stored re-centring values.  Soft codeword, logZ,
    argmax and VJP; 160 sequences (more than one per CTA)."""
    for key, val in variant.items():
        monkeypatch.setenv(key, val)
    w, c, g = I.random_case(16, 2, 1, 160, n, seed=1200 + n + K)
    gZ = torch.randn(160, generator=torch.Generator().manual_seed(K))
    wd, cd, gd, gzd = w.to(DEV), c.to(DEV), g.to(DEV), gZ.to(DEV)

    def run():
        out = list(lib.soft_codeword(wd, cd, 16, 2, 1, 0.05)) + [lib.posterior_argmax(wd, cd, 16, 2, 1, 0.05)]
        out += list(lib.vjp(wd, cd, 16, 2, 1, 0.05, gd, gzd))
        torch.cuda.synchronize()
        assert lib.get_device_error() == 0
        return out

    monkeypatch.setenv("BCJR_L16_CKPT", "0")
    full = run()
    monkeypatch.setenv("BCJR_L16_CKPT", str(K))
    ck = run()
    for a, b in zip(full, ck):
        assert torch.equal(a, b)


@pytest.mark.parametrize("bwd", ["log", "post"])
def test_l16_codeword_ring_equals_l2_stream(monkeypatch, bwd):
    """The VJP backward's codewords through the shared-memory ring (default) and
    streamed from L2 (BCJR_L16_VJP=l2) are the same numbers fed to the same
    arithmetic: bit-identical dl/dw and dl/dc on 300 sequences of 37 steps (the
    ring's stages wrap within and across sequences: 8 x 37 blocks per
    sequence), with a logZ gradient, and both against the oracle on some rows."""
    monkeypatch.setenv("BCJR_L16_BWD", bwd)
    w, c, g = I.random_case(16, 2, 1, 300, 37, seed=1500)
    gZ = torch.randn(300, generator=torch.Generator().manual_seed(15))
    wd, cd, gd, gzd = w.to(DEV), c.to(DEV), g.to(DEV), gZ.to(DEV)
    ring = [x.clone() for x in lib.vjp(wd, cd, 16, 2, 1, 0.1, gd, gzd)]
    assert lib.get_device_error() == 0
    monkeypatch.setenv("BCJR_L16_VJP", "l2")
    l2 = [x.clone() for x in lib.vjp(wd, cd, 16, 2, 1, 0.1, gd, gzd)]
    assert lib.get_device_error() == 0
    for a, b in zip(ring, l2):
        assert torch.equal(a, b)
    rows = [0, 147, 148, 299]
    rv = oracle.vjp(w[rows], c, 16, 2, 1, 0.1, g[rows], gZ[rows])
    assert_grad(ring[0].cpu().numpy()[rows], rv["grad_w"], "grad_w")


def test_l16_ring_wait_runs_out_and_reports_timeout(monkeypatch):
    """With the test hook BCJR_L16_RING_TEST_NOFILL=1 no bulk copy is issued, so
    every CTA's first wait for a ring stage runs out after its 1 s bound: the call
    returns, bcjr_get_device_error reports BCJR_ERR_TIMEOUT, and the next call
    on the same context is correct (against the oracle) with the flag clear."""
    w, c, g = I.random_case(16, 2, 1, 3, 6, seed=1501)
    wd, cd, gd = w.to(DEV), c.to(DEV), g.to(DEV)
    monkeypatch.setenv("BCJR_L16_RING_TEST_NOFILL", "1")
    lib.vjp(wd, cd, 16, 2, 1, 0.2, gd)
    assert lib.get_device_error() == lib.BCJR_ERR_TIMEOUT
    assert lib.get_device_error() == 0
    monkeypatch.delenv("BCJR_L16_RING_TEST_NOFILL")
    gw, gc = lib.vjp(wd, cd, 16, 2, 1, 0.2, gd)
    assert lib.get_device_error() == 0
    rv = oracle.vjp(w, c, 16, 2, 1, 0.2, g)
    assert_grad(gw.cpu().numpy(), rv["grad_w"], "grad_w")
    assert_grad(gc.cpu().numpy(), rv["grad_c"], "grad_c")


def test_launch_count_per_call(monkeypatch):
    """bcjr_launch_count over single calls at L=16, k=2, V=1: the soft codeword
    is the block-codebook staging plus the sweep (2); the VJP adds the ring's
    codebook copy and the gradient reduction (4), or 3 with BCJR_L16_VJP=l2."""
    w, c, g = I.random_case(16, 2, 1, 4, 16, seed=1502)
    wd, cd, gd = w.to(DEV), c.to(DEV), g.to(DEV)
    n0 = lib.launch_count()
    lib.soft_codeword(wd, cd, 16, 2, 1, 0.5)
    n1 = lib.launch_count()
    lib.vjp(wd, cd, 16, 2, 1, 0.5, gd)
    n2 = lib.launch_count()
    monkeypatch.setenv("BCJR_L16_VJP", "l2")
    lib.vjp(wd, cd, 16, 2, 1, 0.5, gd)
    n3 = lib.launch_count()
    assert lib.get_device_error() == 0
    assert (n1 - n0, n2 - n1, n3 - n2) == (2, 4, 3)
