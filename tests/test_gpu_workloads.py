"""The five seeded workloads at full size, run through the C ABI exactly as
bench.py launches them, checked against the CPU oracle on the parity subset
(the first 64 sequences plus 64 drawn with seed 3; the oracle computes
sequences independently) and, at full size, against identities that hold for
any size.

On the subset: logZ, soft codeword, posterior argmax (on steps whose oracle
top-two posteriors differ by more than 1e-4), dl/dw, and dl/dc restricted to
the subset's contribution (the GPU VJP run on those rows alone, against the
oracle's VJP of the same rows).

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
from helpers import assert_grad, assert_logZ, assert_soft, unique_argmax_mask

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _rows(n_seq):
    return I.subset_rows(n_seq, 64, 64)


def _soft_vjp(inp, T, argmax=True):
    wl = inp.wl
    wd, cd, gd = inp.w.to(DEV), inp.c.to(DEV), inp.g.to(DEV)
    soft, logZ = lib.soft_codeword(wd, cd, wl.L, wl.k, wl.V, T)
    gw, gc = lib.vjp(wd, cd, wl.L, wl.k, wl.V, T, gd)
    am = lib.posterior_argmax(wd, cd, wl.L, wl.k, wl.V, T) if argmax else None
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    out = [soft.cpu().numpy(), logZ.cpu().numpy(), gw.cpu().numpy(), gc.cpu().numpy()]
    return out + [am.cpu().numpy() if am is not None else None]


def _check_subset(inp, T, res, rows):
    """Every output on the parity subset against the oracle; returns the oracle's soft result."""
    wl = inp.wl
    soft, logZ, gw, _, am = res
    w, g = inp.w[rows], inp.g[rows]
    ref = oracle.soft(w, inp.c, wl.L, wl.k, wl.V, T)
    assert_logZ(logZ[rows], ref["logZ"], wl.L, wl.D, wl.n_steps)
    assert_soft(soft[rows], ref["soft"], inp.c)
    mask = unique_argmax_mask(ref["top2"])   # at T = 1 only about 1 step in 8 has a unique argmax
    assert mask.sum() >= 1000
    np.testing.assert_array_equal(am[rows][mask], ref["argmax"][mask])
    rv = oracle.vjp(w, inp.c, wl.L, wl.k, wl.V, T, g)
    assert_grad(gw[rows], rv["grad_w"], "grad_w")
    # the codebook gradient restricted to the subset: the GPU VJP on those rows alone
    sub = I.make(wl.name, rows=rows)
    _, gc_sub = lib.vjp(sub.w.to(DEV), sub.c.to(DEV), wl.L, wl.k, wl.V, T, sub.g.to(DEV))
    assert_grad(gc_sub.cpu().numpy().reshape(rv["grad_c"].shape), rv["grad_c"], "grad_c")
    return ref


def _translation_identity(inp, res):
    """sum_s dl/dc(s) + sum_{seq,t} dl/dw = sum g (componentwise), gZ = 0."""
    V = inp.wl.V
    gw, gc = res[2], res[3]
    lhs = gc.reshape(-1, V).astype(np.float64).sum(0) + gw.reshape(-1, V).astype(np.float64).sum(0)
    rhs = inp.g.double().reshape(-1, V).sum(0).numpy()
    scale = np.abs(gw).astype(np.float64).sum() + np.abs(gc).astype(np.float64).sum()
    assert np.all(np.abs(lhs - rhs) <= 1e-5 * scale), (lhs, rhs, scale)


def test_mid_workload():
    inp = I.make("mid", with_grad=False)
    wl = inp.wl
    T = wl.temps[0]
    wd, cd = inp.w.to(DEV), inp.c.to(DEV)
    soft, logZ = lib.soft_codeword(wd, cd, wl.L, wl.k, wl.V, T)
    am = lib.posterior_argmax(wd, cd, wl.L, wl.k, wl.V, T)
    soft, logZ, am = soft.cpu().numpy(), logZ.cpu().numpy(), am.cpu().numpy()
    rows = _rows(wl.n_seq)
    ref = oracle.soft(inp.w[rows], inp.c, wl.L, wl.k, wl.V, T)
    assert_logZ(logZ[rows], ref["logZ"], wl.L, wl.D, wl.n_steps)
    assert_soft(soft[rows], ref["soft"], inp.c)
    mask = unique_argmax_mask(ref["top2"])
    np.testing.assert_array_equal(am[rows][mask], ref["argmax"][mask])


def test_qtip_workload():
    inp = I.make("qtip")
    T = inp.wl.temps[0]
    res = _soft_vjp(inp, T)
    _check_subset(inp, T, res, _rows(inp.wl.n_seq))
    _translation_identity(inp, res)


@pytest.mark.parametrize("T", [1.0, 0.1, 0.01])
def test_mlp_workload_temperature(T):
    inp = I.make("mlp")
    wl = inp.wl
    res = _soft_vjp(inp, T)
    rows = _rows(wl.n_seq)
    ref = _check_subset(inp, T, res, rows)
    _translation_identity(inp, res)
    if T == 0.01:
        # posterior argmax at T = 0.01 equals the Viterbi state wherever the
        # oracle's posterior of the Viterbi state exceeds 1/2 (then it is the
        # unique argmax); the remaining steps are counted, not compared
        vt = oracle.viterbi(inp.w[rows], inp.c, wl.L, wl.k, wl.V)["states"]
        sure = (ref["argmax"] == vt) & (ref["top2"][..., 0] > 0.5 + 1e-4)
        assert sure.mean() > 0.5
        np.testing.assert_array_equal(res[4][rows][sure], vt[sure])


def test_mlp_workload_viterbi():
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
    rows = _rows(wl.n_seq)
    ref = oracle.viterbi(inp.w[rows], inp.c, wl.L, wl.k, wl.V)
    np.testing.assert_array_equal(states[rows], ref["states"])
    np.testing.assert_array_equal(cost[rows], ref["cost"])
    # on the whole workload, the agreement rate is reported by the GPU alone
    agree = (am == states).mean()
    assert agree > 0.9, agree


def test_layer_workload():
    inp = I.make("layer")
    wl, T = inp.wl, inp.wl.temps[0]
    res = _soft_vjp(inp, T)
    rows = _rows(wl.n_seq)
    _check_subset(inp, T, res, rows)
    _translation_identity(inp, res)
    # the hard limit over the whole workload, bit-exact on the subset
    states, cost = lib.viterbi_decode(inp.w.to(DEV), inp.c.to(DEV), wl.L, wl.k, wl.V)
    torch.cuda.synchronize()
    ref = oracle.viterbi(inp.w[rows], inp.c, wl.L, wl.k, wl.V)
    np.testing.assert_array_equal(states.cpu().numpy()[rows], ref["states"])
    np.testing.assert_array_equal(cost.cpu().numpy()[rows], ref["cost"])
    st = states.cpu().numpy().astype(np.int64)
    assert ((st[:, 1:] >> 4) == (st[:, :-1] & ((1 << 12) - 1))).all()


def test_long_workload_checkpointed_equals_full(monkeypatch):
    """The long workload (2048 sequences of 8192 weights): with histories beyond
    the scratch budget the L=16 kernels keep sqrt(n)-step checkpoints and
    recompute segments; soft codeword, logZ and dl/dw equal the full-history
    run bit for bit (each sequence's arithmetic is the same), dl/dc agrees to
    fp64 summation order, and the translation identity holds."""
    inp = I.make("long")
    wl, T = inp.wl, inp.wl.temps[0]
    ck = _soft_vjp(inp, T, argmax=False)
    monkeypatch.setenv("BCJR_L16_CKPT", "0")   # full histories, fewer resident CTAs
    full = _soft_vjp(inp, T, argmax=False)
    for i in range(3):
        np.testing.assert_array_equal(ck[i], full[i])
    np.testing.assert_allclose(ck[3], full[3], rtol=1e-6, atol=1e-6 * np.abs(full[3]).max())
    _translation_identity(inp, ck)
