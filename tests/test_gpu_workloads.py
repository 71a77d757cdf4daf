"""The five seeded workloads at full size, run through the C ABI exactly as
bench.py launches them, checked against the CPU oracle on sampled sequences
(the oracle computes sequences independently) and, at full size, against
identities that hold for any size.

Workloads (bcjr_sum_product_b200/inputs.py): tiny (L=8), mid (L=12), qtip
(L=16, 16384 x 256), mlp (L=16, 65536 x 256, T in {1, 0.1, 0.01}), layer
(L=16, V=2, 237,568 sequences of 128 steps).
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


def _rows(n_seq, n_first, n_random):
    return I.subset_rows(n_seq, n_first, n_random)


def _soft_vjp(inp, T, w=None, g=None):
    wl = inp.wl
    w = inp.w if w is None else w
    g = inp.g if g is None else g
    wd, cd, gd = w.to(DEV), inp.c.to(DEV), g.to(DEV)
    soft, logZ = lib.soft_codeword(wd, cd, wl.L, wl.k, wl.V, T)
    gw, gc = lib.vjp(wd, cd, wl.L, wl.k, wl.V, T, gd)
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    return soft.cpu().numpy(), logZ.cpu().numpy(), gw.cpu().numpy(), gc.cpu().numpy()


def _check_rows(inp, T, res, rows, check_vjp=True):
    wl = inp.wl
    soft, logZ, gw, _ = res
    w, g = inp.w[rows], inp.g[rows]
    ref = oracle.soft(w, inp.c, wl.L, wl.k, wl.V, T)
    assert_logZ(logZ[rows], ref["logZ"], wl.L, wl.D, wl.n_steps)
    assert_soft(soft[rows], ref["soft"], inp.c)
    if check_vjp:
        rv = oracle.vjp(w, inp.c, wl.L, wl.k, wl.V, T, g)
        assert_grad(gw[rows], rv["grad_w"], "grad_w")
        return rv
    return None


def _translation_identity(inp, res):
    """sum_s dl/dc(s) + sum_{seq,t} dl/dw = sum g (componentwise), gZ = 0."""
    V = inp.wl.V
    _, _, gw, gc = res
    lhs = gc.reshape(-1, V).astype(np.float64).sum(0) + gw.reshape(-1, V).astype(np.float64).sum(0)
    rhs = inp.g.double().reshape(-1, V).sum(0).numpy()
    scale = np.abs(gw).astype(np.float64).sum() + np.abs(gc).astype(np.float64).sum()
    assert np.all(np.abs(lhs - rhs) <= 1e-5 * scale), (lhs, rhs, scale)


def test_mid_workload():
    inp = I.make("mid", with_grad=False)
    wl = inp.wl
    soft, logZ = lib.soft_codeword(inp.w.to(DEV), inp.c.to(DEV), wl.L, wl.k, wl.V, wl.temps[0])
    soft, logZ = soft.cpu().numpy(), logZ.cpu().numpy()
    rows = _rows(wl.n_seq, 64, 64)
    ref = oracle.soft(inp.w[rows], inp.c, wl.L, wl.k, wl.V, wl.temps[0])
    assert_logZ(logZ[rows], ref["logZ"], wl.L, wl.D, wl.n_steps)
    assert_soft(soft[rows], ref["soft"], inp.c)


def test_qtip_workload():
    inp = I.make("qtip")
    wl, T = inp.wl, inp.wl.temps[0]
    res = _soft_vjp(inp, T)
    rows = _rows(wl.n_seq, 16, 16)
    _check_rows(inp, T, res, rows)
    _translation_identity(inp, res)
    # codebook gradient restricted to the sampled rows: GPU VJP on those rows vs the oracle
    sub = I.make("qtip", rows=rows)
    _, _, _, gc_sub = _soft_vjp(sub, T)
    rv = oracle.vjp(sub.w, sub.c, wl.L, wl.k, wl.V, T, sub.g)
    assert_grad(gc_sub, rv["grad_c"], "grad_c")


@pytest.mark.parametrize("T", [1.0, 0.1, 0.01])
def test_mlp_workload_temperature(T):
    inp = I.make("mlp")
    wl = inp.wl
    res = _soft_vjp(inp, T)
    rows = _rows(wl.n_seq, 8, 8)
    _check_rows(inp, T, res, rows)
    _translation_identity(inp, res)


def test_mlp_workload_viterbi_and_argmax():
    inp = I.make("mlp", with_grad=False)
    wl = inp.wl
    wd, cd = inp.w.to(DEV), inp.c.to(DEV)
    states, cost = lib.viterbi_decode(wd, cd, wl.L, wl.k, wl.V)
    am = lib.posterior_argmax(wd, cd, wl.L, wl.k, wl.V, 0.01)
    torch.cuda.synchronize()
    states, cost, am = states.cpu().numpy(), cost.cpu().numpy(), am.cpu().numpy()
    # every decoded sequence is a trellis path
    st = states.astype(np.int64)
    assert ((st[:, 1:] >> 2) == (st[:, :-1] & ((1 << 14) - 1))).all()
    rows = _rows(wl.n_seq, 16, 16)
    ref = oracle.viterbi(inp.w[rows], inp.c, wl.L, wl.k, wl.V)
    np.testing.assert_array_equal(states[rows], ref["states"])
    np.testing.assert_array_equal(cost[rows], ref["cost"])
    # posterior argmax at T = 0.01 equals the Viterbi state wherever the
    # oracle's posterior of the Viterbi state exceeds 1/2 (then it is the unique argmax)
    po = oracle.soft(inp.w[rows[:8]], inp.c, wl.L, wl.k, wl.V, 0.01)
    vt = ref["states"][:8]
    top = po["top2"][..., 0]
    sure = (po["argmax"] == vt) & (top > 0.5 + 1e-4)
    assert sure.mean() > 0.5
    np.testing.assert_array_equal(am[rows[:8]][sure], vt[sure])
    # on the whole workload, the agreement rate is reported by the GPU alone
    agree = (am == states).mean()
    assert agree > 0.9, agree


def test_layer_workload():
    inp = I.make("layer")
    wl, T = inp.wl, inp.wl.temps[0]
    res = _soft_vjp(inp, T)
    rows = _rows(wl.n_seq, 8, 8)
    _check_rows(inp, T, res, rows)
    _translation_identity(inp, res)
    # the hard limit over the whole workload, bit-exact on the sampled rows
    states, cost = lib.viterbi_decode(inp.w.to(DEV), inp.c.to(DEV), wl.L, wl.k, wl.V)
    torch.cuda.synchronize()
    ref = oracle.viterbi(inp.w[rows], inp.c, wl.L, wl.k, wl.V)
    np.testing.assert_array_equal(states.cpu().numpy()[rows], ref["states"])
    np.testing.assert_array_equal(cost.cpu().numpy()[rows], ref["cost"])
