"""Pins of the CPU oracle against what the pages and the mathematics fix.

Source: "BCJR-QAT: A Differentiable Relaxation of Trellis-Coded Weight
Quantization" -- Abstract (Boltzmann expectation over trellis paths, exact
differentiability, T -> 0 recovers the hard code, identity with the transfer
matrix of a 1D Ising-like chain) and Technical Summary, "Core Mechanism"
(w_hat_t = sum_s c(s) p_T(s_t = s | w)).

Each pin is independent of the oracle's recursions: brute-force path
enumeration, the dense transfer-matrix product, closed forms, identities of
the Gibbs distribution and finite differences.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import reference as R
from bcjr_sum_product_b200 import inputs as I


def _tiny(L, k, V, n_seq, n, seed, scale=1.0):
    return I.random_case(L, k, V, n_seq, n * V, seed, scale)


# ---------------------------------------------------------------- trellis rule
@pytest.mark.parametrize("L,k,V", [(3, 1, 1), (4, 2, 1), (6, 2, 1), (8, 2, 1), (8, 2, 2), (5, 5, 1), (6, 3, 2)])
def test_predecessors_follow_successor_rule(L, k, V):
    D = k * V
    pt = oracle.pred_table(L, k, V)
    S, B = 1 << L, 1 << D
    assert pt.shape == (S, B)
    for s in range(S):
        expect = sorted(((s >> D) | (b << (L - D))) for b in range(B))
        assert list(pt[s]) == expect
        for p in pt[s]:
            assert ((int(p) << D) & (S - 1)) | (s & (B - 1)) == s


# ---------------------------------------------------------------- brute force
def test_brute_force_tiny_config_prefix():
    """The tiny workload (L=8, k=2, V=1, T=0.5) solved on its first 6 steps by
    enumerating all 256 * 4^5 paths of each of its 16 sequences."""
    inp = I.make("tiny")
    w6 = inp.w[:, :6].contiguous()
    r = oracle.soft(w6, inp.c, 8, 2, 1, 0.5, posteriors=True)
    for q in range(w6.shape[0]):
        b = R.brute_force(w6[q], inp.c, 8, 2, 1, 0.5)
        assert abs(r["logZ"][q] - b["logZ"]) <= 1e-10 * max(1.0, abs(b["logZ"]))
        np.testing.assert_allclose(r["post"][q], b["post"], atol=1e-12)
        np.testing.assert_allclose(r["soft"][q], b["soft"], atol=1e-12)


@pytest.mark.parametrize("L,k,V,n,T", [(4, 2, 1, 5, 0.7), (4, 1, 2, 4, 0.3), (5, 1, 1, 6, 1.3), (4, 2, 2, 3, 0.2),
                                       (3, 3, 1, 4, 0.5)])
def test_brute_force_small(L, k, V, n, T):
    w, c, _ = _tiny(L, k, V, 3, n, seed=11 + L + 7 * k + 3 * V)
    r = oracle.soft(w, c, L, k, V, T, posteriors=True)
    for q in range(3):
        b = R.brute_force(w[q], c, L, k, V, T)
        assert abs(r["logZ"][q] - b["logZ"]) <= 1e-11 * max(1.0, abs(b["logZ"]))
        np.testing.assert_allclose(r["post"][q], b["post"], atol=1e-12)
        np.testing.assert_allclose(r["soft"][q], b["soft"], atol=1e-12)


# ---------------------------------------------------------------- transfer matrix
def test_transfer_matrix_tiny_config():
    inp = I.make("tiny")
    r = oracle.soft(inp.w, inp.c, 8, 2, 1, 0.5)
    M = R.transfer_matrix(8, 2)
    for q in range(inp.w.shape[0]):
        tm = R.transfer_matrix_logZ(inp.w[q], inp.c, 8, 2, 1, 0.5, M)
        assert abs(r["logZ"][q] - tm) <= 1e-10 * abs(tm)


def test_transfer_matrix_mid_config():
    """L=12 (4096 states) on the first sequence of the mid workload, T=0.1."""
    inp = I.make("mid", rows=[0, 1])
    r = oracle.soft(inp.w, inp.c, 12, 2, 1, 0.1)
    M = R.transfer_matrix(12, 2)
    tm = R.transfer_matrix_logZ(inp.w[0], inp.c, 12, 2, 1, 0.1, M)
    assert abs(r["logZ"][0] - tm) <= 1e-10 * abs(tm)


# ---------------------------------------------------------------- closed forms
@pytest.mark.parametrize("L,k,V", [(6, 2, 1), (8, 2, 2), (4, 1, 1)])
def test_constant_codebook(L, k, V):
    w, c, _ = _tiny(L, k, V, 2, 20, seed=5)
    c0 = torch.tensor([0.3, -0.8][:V], dtype=torch.float32)
    cc = c0.expand(1 << L, V).clone() if V > 1 else torch.full((1 << L,), 0.3)
    T = 0.37
    r = oracle.soft(w, cc, L, k, V, T)
    for q in range(2):
        ref = R.constant_codebook_logZ(w[q], cc[0], L, k * V, V, T)
        assert abs(r["logZ"][q] - ref) <= 1e-11 * abs(ref)
    # the soft codeword is the constant itself
    np.testing.assert_allclose(r["soft"].reshape(2, -1, V), np.broadcast_to(cc[0].numpy().reshape(1, 1, V),
                               (2, 20, V)), atol=1e-6)


@pytest.mark.parametrize("L,k,V", [(4, 4, 1), (4, 2, 2), (6, 3, 2)])
def test_full_shift_is_independent_softmax(L, k, V):
    """D = L: every state reaches every state, so the posteriors are the
    per-step softmax and logZ the sum of per-step log-partition functions."""
    w, c, _ = _tiny(L, k, V, 2, 7, seed=13)
    T = 0.41
    r = oracle.soft(w, c, L, k, V, T, posteriors=True)
    for q in range(2):
        ref = R.softmax_case(w[q], c, L, V, T)
        assert abs(r["logZ"][q] - ref["logZ"]) <= 1e-11 * abs(ref["logZ"])
        np.testing.assert_allclose(r["post"][q], ref["post"], atol=1e-12)
        np.testing.assert_allclose(r["soft"][q], ref["soft"], atol=1e-12)


def test_high_temperature_uniform():
    """T -> infinity: every path has weight 1, so logZ -> log(#paths) and, the
    de Bruijn trellis being regular, every posterior -> 1/2^L."""
    L, k, V, n = 6, 2, 1, 12
    w, c, _ = _tiny(L, k, V, 2, n, seed=3)
    T = 1e12
    r = oracle.soft(w, c, L, k, V, T, posteriors=True)
    np.testing.assert_allclose(r["post"], 1.0 / (1 << L), rtol=1e-9)
    np.testing.assert_allclose(r["logZ"], R.path_count_log(L, k * V, n), rtol=1e-9)
    np.testing.assert_allclose(r["soft"], float(c.double().mean()), atol=1e-9)


def test_posteriors_sum_to_one():
    inp = I.make("tiny")
    r = oracle.soft(inp.w[:4], inp.c, 8, 2, 1, 0.5, posteriors=True)
    np.testing.assert_allclose(r["post"].sum(-1), 1.0, atol=1e-12)
    assert (r["post"] >= 0).all()


def test_logZ_bounds_against_viterbi():
    """0 <= logZ + E*/T <= log(#paths), E* the minimum path energy."""
    inp = I.make("tiny")
    for T in (0.05, 0.5, 5.0):
        r = oracle.soft(inp.w, inp.c, 8, 2, 1, T)
        v = oracle.viterbi(inp.w, inp.c, 8, 2, 1)
        for q in range(inp.w.shape[0]):
            st = v["states"][q]
            E = float(((inp.w[q].double().numpy() - inp.c.double().numpy()[st]) ** 2).sum())
            gap = r["logZ"][q] + E / T
            assert -1e-9 <= gap <= R.path_count_log(8, 2, 64) + 1e-9


# ---------------------------------------------------------------- symmetries
def test_scale_invariance():
    inp = I.make("tiny")
    w, c = inp.w[:4], inp.c
    a = oracle.soft(w, c, 8, 2, 1, 0.5)
    b = oracle.soft(2 * w, 2 * c, 8, 2, 1, 2.0)
    np.testing.assert_allclose(a["logZ"], b["logZ"], rtol=1e-12)
    np.testing.assert_allclose(2 * a["soft"], b["soft"], atol=1e-11)


def test_translation_equivariance():
    L, k, V = 6, 2, 2
    w, c, _ = _tiny(L, k, V, 3, 16, seed=21)
    a = oracle.soft(w, c, L, k, V, 0.3)
    shift = torch.tensor([0.25, -0.5])
    w2 = (w.reshape(3, -1, 2) + shift).reshape(3, -1)
    b = oracle.soft(w2, c + shift, L, k, V, 0.3)
    np.testing.assert_allclose(a["logZ"], b["logZ"], rtol=1e-6)
    np.testing.assert_allclose((a["soft"].reshape(3, -1, 2) + shift.numpy()).reshape(3, -1), b["soft"], atol=1e-6)


def test_soft_codeword_is_logZ_gradient():
    """w_hat_t = w_t + (T/2) dlogZ/dw_t (the Gibbs mean of the energy gradient),
    checked with central differences of the oracle's logZ in fp64."""
    L, k, V, n = 6, 2, 1, 10
    w, c, _ = _tiny(L, k, V, 1, n, seed=9)
    T = 0.6
    base = oracle.soft(w, c, L, k, V, T)["soft"][0]
    wd = w.double()
    h = 1e-3
    for t in range(n):
        # evaluate logZ in fp64 via the dense transfer matrix on perturbed fp64 weights
        wp = wd.clone(); wp[0, t] += h
        wm = wd.clone(); wm[0, t] -= h
        lp = R.transfer_matrix_logZ(wp[0], c, L, k, V, T)
        lm = R.transfer_matrix_logZ(wm[0], c, L, k, V, T)
        fd = (lp - lm) / (2 * h)
        assert abs(base[t] - (float(w[0, t]) + 0.5 * T * fd)) < 1e-6


def test_zero_temperature_limit():
    """T -> 0: the soft codeword approaches c at the Viterbi path."""
    L, k, V, n = 6, 2, 1, 24
    w, c, _ = _tiny(L, k, V, 4, n, seed=17)
    v = oracle.viterbi(w, c, L, k, V)
    errs, meds = [], []
    for T in (0.1, 0.01, 1e-3, 1e-5):
        r = oracle.soft(w, c, L, k, V, T)
        hard = c.double().numpy()[v["states"]]
        e = np.abs(r["soft"] - hard)
        errs.append(e.max())
        meds.append(np.median(e))
    # near-degenerate paths (energy gap ~1e-4 in this case) need T well below the gap
    assert errs[-1] < 1e-6
    assert meds[1] <= meds[0] and meds[2] < 1e-9 and meds[3] < 1e-9


def test_posterior_argmax_matches_posteriors():
    inp = I.make("tiny")
    r = oracle.soft(inp.w[:3], inp.c, 8, 2, 1, 0.5, posteriors=True)
    np.testing.assert_array_equal(r["argmax"], r["post"].argmax(-1))
    srt = np.sort(r["post"], -1)
    np.testing.assert_allclose(r["top2"][..., 0], srt[..., -1])
    np.testing.assert_allclose(r["top2"][..., 1], srt[..., -2])


# ---------------------------------------------------------------- VJP
def _chain_rule_from_G(G, w_seq, c, g_seq, post, T, V):
    """grad_w and grad_c from G_t(s) = dl/dtheta_t(s) with theta = -||w - c||^2/T."""
    n, S = G.shape
    w2 = w_seq.double().numpy().reshape(n, V)
    c2 = c.double().numpy().reshape(S, V)
    g2 = g_seq.double().numpy().reshape(n, V)
    gw = (2.0 / T) * (G @ c2 - G.sum(1, keepdims=True) * w2)
    gc = post.T @ g2 + (2.0 / T) * (G.T @ w2 - G.sum(0)[:, None] * c2)
    return gw.reshape(-1), gc


@pytest.mark.parametrize("L,k,V,n,T,gz", [(4, 2, 1, 5, 0.7, 0.0), (4, 1, 2, 4, 0.3, 0.0), (5, 1, 1, 5, 1.1, 0.8),
                                          (4, 2, 2, 3, 0.25, -0.6)])
def test_vjp_against_brute_force_covariance(L, k, V, n, T, gz):
    w, c, g = _tiny(L, k, V, 2, n, seed=31 + L)
    gZ = torch.full((2,), gz)
    gz = float(gZ[0])  # the oracle reads gZ as fp32
    r = oracle.vjp(w, c, L, k, V, T, g, gZ)
    gc_tot = np.zeros((1 << L, V))
    for q in range(2):
        b = R.brute_force(w[q], c, L, k, V, T, g_seq=g[q], gZ=gz)
        gw, gc = _chain_rule_from_G(b["G"], w[q], c, g[q], b["post"], T, V)
        np.testing.assert_allclose(r["grad_w"][q], gw, atol=1e-10)
        gc_tot += gc
        assert abs(r["Hbar"][q] - b["EF"]) < 1e-10
        np.testing.assert_allclose(b["G"].sum(1), gz, atol=1e-10)
    np.testing.assert_allclose(r["grad_c"].reshape(-1, V), gc_tot, atol=1e-10)


def _loss(w, c, g, gZ, L, k, V, T):
    r = oracle.soft(w, c, L, k, V, T)
    return float((r["soft"] * g.double().numpy()).sum() + (r["logZ"] * gZ.double().numpy()).sum())


@pytest.mark.parametrize("L,k,V,n,T", [(6, 2, 1, 8, 0.5), (4, 1, 2, 6, 0.4), (8, 2, 1, 6, 0.5)])
def test_vjp_finite_differences(L, k, V, n, T):
    """The VJP is the exact gradient of l = sum g . w_hat + gZ . logZ."""
    w, c, g = _tiny(L, k, V, 2, n, seed=41 + L)
    gZ = torch.tensor([0.3, -0.2])
    r = oracle.vjp(w, c, L, k, V, T, g, gZ)
    rng = np.random.default_rng(0)
    # the oracle reads fp32 inputs, so differences use an fp32-representable
    # step large enough to dominate input rounding; compare with a loose bound
    h = 2.0 ** -10
    for _ in range(6):
        q, t = int(rng.integers(2)), int(rng.integers(n * V))
        wp = w.clone(); wp[q, t] += h
        wm = w.clone(); wm[q, t] -= h
        fd = (_loss(wp, c, g, gZ, L, k, V, T) - _loss(wm, c, g, gZ, L, k, V, T)) / (2 * h)
        assert abs(fd - r["grad_w"][q, t]) < 2e-4 * max(1.0, abs(fd))
    cflat = c.reshape(-1)
    gcf = r["grad_c"].reshape(-1)
    for _ in range(6):
        i = int(rng.integers(cflat.numel()))
        cp = cflat.clone(); cp[i] += h
        cm = cflat.clone(); cm[i] -= h
        fd = (_loss(w, cp.reshape(c.shape), g, gZ, L, k, V, T) - _loss(w, cm.reshape(c.shape), g, gZ, L, k, V, T)) / (2 * h)
        assert abs(fd - gcf[i]) < 2e-4 * max(1.0, abs(fd))


def test_vjp_logZ_only_closed_form():
    """With g = 0 and gZ = 1 the VJP is dlogZ/dw = (2/T)(w_hat - w)."""
    L, k, V, n, T = 6, 2, 1, 12, 0.35
    w, c, _ = _tiny(L, k, V, 3, n, seed=51)
    r = oracle.vjp(w, c, L, k, V, T, torch.zeros_like(w), torch.ones(3))
    s = oracle.soft(w, c, L, k, V, T)
    np.testing.assert_allclose(r["grad_w"], (2.0 / T) * (s["soft"] - w.double().numpy()), atol=1e-9)


def test_vjp_translation_identity():
    """sum_s dl/dc(s) + sum_t dl/dw_t = sum_t g_t (componentwise), gZ = 0."""
    inp = I.make("tiny")
    r = oracle.vjp(inp.w, inp.c, 8, 2, 1, 0.5, inp.g)
    lhs = r["grad_c"].sum() + r["grad_w"].sum()
    assert abs(lhs - float(inp.g.double().sum())) < 1e-8 * max(1.0, float(inp.g.abs().sum()))
    L, k, V = 6, 1, 2
    w, c, g = _tiny(L, k, V, 3, 9, seed=61)
    r = oracle.vjp(w, c, L, k, V, 0.4, g)
    lhs = r["grad_c"].sum(0) + r["grad_w"].reshape(3, -1, 2).sum((0, 1))
    np.testing.assert_allclose(lhs, g.double().reshape(3, -1, 2).sum((0, 1)).numpy(), atol=1e-9)


def test_vjp_jacobian_symmetry():
    """J = dw_hat/dw = I + (T/2) Hess(logZ) is symmetric: <v, J^T g> = <J^T v, g>."""
    L, k, V, n, T = 6, 2, 1, 10, 0.5
    w, c, g = _tiny(L, k, V, 1, n, seed=71)
    v = torch.randn(w.shape, generator=torch.Generator().manual_seed(72))
    a = oracle.vjp(w, c, L, k, V, T, g)["grad_w"]
    b = oracle.vjp(w, c, L, k, V, T, v)["grad_w"]
    lhs = float((v.double().numpy() * a).sum())
    rhs = float((g.double().numpy() * b).sum())
    assert abs(lhs - rhs) < 1e-9 * max(1.0, abs(lhs))


def test_vjp_Hbar_is_expected_upstream_dot():
    inp = I.make("tiny")
    r = oracle.vjp(inp.w[:4], inp.c, 8, 2, 1, 0.5, inp.g[:4])
    s = oracle.soft(inp.w[:4], inp.c, 8, 2, 1, 0.5)
    np.testing.assert_allclose(r["Hbar"], (s["soft"] * inp.g[:4].double().numpy()).sum(1), atol=1e-9)
    np.testing.assert_allclose(r["logZ"], s["logZ"], rtol=1e-13)


# ---------------------------------------------------------------- Viterbi
@pytest.mark.parametrize("L,k,V,n,dup", [(4, 2, 1, 5, False), (4, 1, 2, 4, False), (3, 1, 1, 7, False),
                                         (4, 2, 1, 5, True), (4, 1, 2, 4, True), (5, 1, 1, 6, True)])
def test_viterbi_against_enumeration(L, k, V, n, dup):
    w, c, _ = _tiny(L, k, V, 6, n, seed=81 + L + n)
    if dup:
        # force exact ties: few distinct codewords, weights on a coarse grid
        c = torch.round(c * 2) / 2
        w = torch.round(w * 2) / 2
    r = oracle.viterbi(w, c, L, k, V)
    for q in range(6):
        ref = R.viterbi_brute(w[q], c, L, k, V)
        np.testing.assert_array_equal(r["states"][q], ref)


def test_viterbi_path_is_a_trellis_path_and_cost():
    inp = I.make("tiny")
    r = oracle.viterbi(inp.w, inp.c, 8, 2, 1)
    st = r["states"].astype(np.int64)
    assert ((st[:, 1:] >> 2) == (st[:, :-1] & ((1 << 6) - 1))).all()
    w32 = inp.w.numpy(); c32 = inp.c.numpy()
    for q in range(inp.w.shape[0]):
        acc = np.float32(0)
        for t in range(64):
            d = np.float32(w32[q, t] - c32[st[q, t]])
            acc = np.float32(acc + np.float32(d * d)) if t else np.float32(d * d)
        assert acc == r["cost"][q]


def test_posterior_argmax_equals_viterbi_at_low_temperature():
    """At small T the posterior mass concentrates on the minimum-energy path:
    wherever the oracle's top posterior exceeds 1/2 it is the Viterbi state."""
    L, k, V, n = 8, 2, 1, 64
    inp = I.make("tiny")
    v = oracle.viterbi(inp.w, inp.c, L, k, V)
    r = oracle.soft(inp.w, inp.c, L, k, V, 0.01)
    mask = r["top2"][..., 0] > 0.5 + 1e-4
    assert mask.mean() > 0.9
    np.testing.assert_array_equal(r["argmax"][mask], v["states"][mask])


def test_golden_tiny_prefix_fixture():
    """The stored brute-force fixture (tests/golden/make_golden.py) and the C
    oracle agree on the tiny workload's 6-step prefix."""
    import json, os
    with open(os.path.join(os.path.dirname(__file__), "golden", "tiny_prefix6.json")) as f:
        gold = json.load(f)
    inp = I.make("tiny")
    r = oracle.soft(inp.w[:, :6].contiguous(), inp.c, 8, 2, 1, 0.5)
    np.testing.assert_allclose(r["logZ"], gold["logZ"], rtol=1e-12)
    np.testing.assert_allclose(r["soft"], np.array(gold["soft"]), atol=1e-12)
