"""Pins of the fp64 CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a
hand-derived closed form stored under ``tests/golden/`` (with its citation), a
library routine (numpy SVD / norms / sort, scipy softmax), an exact scaling
law or invariant that follows from the page's formulas, or brute force on a
tiny input.  They are chosen so that a dropped term, a wrong sign or index or a
transposed operand in the oracle fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")
L3 = math.log(3.0)


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _rand_layer(rng, E=4, d=48, m=24, scale=0.2):
    gamma = rng.uniform(0.5, 1.5, d)
    wr = rng.normal(0, 0.2, (E, d)).astype(np.float32)
    wg = rng.normal(0, scale, (E, m, d)).astype(np.float32)
    wu = rng.normal(0, scale, (E, m, d)).astype(np.float32)
    wd = rng.normal(0, scale, (E, d, m)).astype(np.float32)
    return dict(gamma=gamma, wr=wr, bias=None, wg=wg, wu=wu, wd=wd, k=2, E=E, d=d, m=m)


def _page(layer, e):
    """The page's matrices for expert e: Gamma W^gate (d x m), Gamma W^up,
    W^down (m x d)."""
    G = np.diag(layer["gamma"])
    Wg = layer["wg"][e].astype(np.float64).T
    Wu = layer["wu"][e].astype(np.float64).T
    Wd = layer["wd"][e].astype(np.float64).T
    return G @ Wg, G @ Wu, Wd


# --------------------------------------------------------------------- SwiGLU
def test_swiglu_closed_form_ln3():
    """Hand-derived values of eq. f at gate pre-activations +-ln 3."""
    g = _gold("swiglu_ln3.json")
    z = np.array([L3 if v == "ln3" else float(v) for v in g["z"]])
    wg = np.array(g["page_W_gate"], dtype=np.float32).T.copy()   # stored [m][d]
    wu = np.array(g["page_W_up"], dtype=np.float32).T.copy()
    wd = np.array(g["page_W_down"], dtype=np.float32).T.copy()   # stored [d][m]
    h, f = oracle.swiglu(z, wg, wu, wd)
    assert np.allclose(h, np.array(g["expected_h_in_units_of_ln3"]) * L3, rtol=1e-14, atol=0)
    assert np.allclose(f, np.array(g["expected_f_in_units_of_ln3"]) * L3, rtol=1e-14, atol=0)


def test_swiglu_upper_bound_spectral():
    """||f(x)|| <= ||xbar||^2 ||Gamma W^gate||_2 ||Gamma W^up||_2 ||W^down||_2
    (ACE, 'Theoretical Foundation'), sigma_1 from numpy's SVD."""
    rng = np.random.default_rng(1)
    layer = _rand_layer(rng, E=3, d=40, m=24)
    u = rng.normal(0, 1, (200, 40)) * rng.uniform(0.1, 5.0, (200, 1))
    xbar, x = oracle.rmsnorm(u, layer["gamma"])
    worst = 0.0
    for e in range(3):
        A, B, D = _page(layer, e)
        s = [np.linalg.svd(M, compute_uv=False)[0] for M in (A, B, D)]
        for t in range(200):
            _, f = oracle.swiglu(x[t], layer["wg"][e], layer["wu"][e], layer["wd"][e])
            bound = np.dot(xbar[t], xbar[t]) * s[0] * s[1] * s[2]
            assert np.linalg.norm(f) <= bound * (1 + 1e-12)
            worst = max(worst, np.linalg.norm(f) / bound)
    assert worst > 1e-3  # the bound is exercised, not vacuous


def test_swiglu_linear_regime_matches_relu_bilinear():
    """For gate pre-activations far from 0, SiLU(a) = ReLU(a) within e^-|a||a|,
    so f reduces to (ReLU(x Gamma W^gate) (.) x Gamma W^up) W^down, evaluated
    here with numpy matmuls in the page's orientation."""
    rng = np.random.default_rng(2)
    d, m = 16, 8
    z = rng.normal(0, 1, d)
    # gate columns aligned (+/-) with z so that |a_j| >= 60
    sgn = np.where(np.arange(m) % 2 == 0, 1.0, -1.0)
    Wg_page = np.outer(z / np.dot(z, z), sgn * (60.0 + np.arange(m)))
    Wg_page = Wg_page.astype(np.float32).astype(np.float64)
    Wu_page = rng.normal(0, 1, (d, m)).astype(np.float32).astype(np.float64)
    Wd_page = rng.normal(0, 1, (m, d)).astype(np.float32).astype(np.float64)
    a = z @ Wg_page
    assert np.all(np.abs(a) > 50)
    ref = (np.maximum(a, 0) * (z @ Wu_page)) @ Wd_page
    _, f = oracle.swiglu(z, Wg_page.T.astype(np.float32), Wu_page.T.astype(np.float32),
                         Wd_page.T.astype(np.float32))
    assert np.allclose(f, ref, rtol=1e-12, atol=1e-12)


# -------------------------------------------------------------------- RMSNorm
def test_rmsnorm_closed_form_and_scale_invariance():
    d = 8
    gamma = np.arange(1, d + 1) / 4.0
    u = np.full((1, d), 3.0)
    xbar, x = oracle.rmsnorm(u, gamma, eps_rms=0.0)
    assert np.allclose(xbar, 1.0, rtol=1e-15)           # RMS(u) = 3
    assert np.allclose(x, gamma, rtol=1e-15)
    # eps sits under the root with the mean square: mean(u^2) = 1, eps = 3
    xbar, x = oracle.rmsnorm(np.ones((1, d)), gamma, eps_rms=3.0)
    assert np.allclose(xbar, 0.5, rtol=1e-15)
    assert np.allclose(x, 0.5 * gamma, rtol=1e-15)
    rng = np.random.default_rng(3)
    u = rng.normal(0, 1, (5, 32))
    xb1, _ = oracle.rmsnorm(u, np.ones(32), eps_rms=0.0)
    xb2, _ = oracle.rmsnorm(u * 8.0, np.ones(32), eps_rms=0.0)
    assert np.allclose(xb1, xb2, rtol=1e-14)
    assert np.allclose(np.sqrt(np.mean(xb1 ** 2, axis=1)), 1.0, rtol=1e-14)


# ------------------------------------------------------------- router / top-k
def test_router_topk_matches_library_sort_and_softmax():
    rng = np.random.default_rng(4)
    T, d, E, k = 50, 24, 16, 5
    x = rng.normal(0, 1, (T, d))
    wr = rng.normal(0, 0.3, (E, d)).astype(np.float32)
    bias = rng.normal(0, 1, E).astype(np.float32)
    logits, idx, gate = oracle.router(x, wr, bias, k, renorm=False)
    ref_logits = x @ wr.astype(np.float64).T + bias.astype(np.float64)
    assert np.allclose(logits, ref_logits, rtol=1e-12, atol=1e-12)
    from scipy.special import softmax
    p = softmax(ref_logits, axis=1)
    for t in range(T):
        order = np.lexsort((np.arange(E), -ref_logits[t]))  # logit desc, index asc
        assert list(idx[t]) == list(order[:k])
        assert np.allclose(gate[t], p[t, order[:k]], rtol=1e-12)
    _, idx2, g2 = oracle.router(x, wr, bias, k, renorm=True)
    assert (idx2 == idx).all()
    assert np.allclose(g2.sum(1), 1.0, rtol=1e-14)
    assert np.allclose(g2, gate / gate.sum(1, keepdims=True), rtol=1e-13)


def test_router_tie_break_lower_index_first():
    x = np.ones((1, 2))
    wr = np.array([[1, 0], [0, 1], [2, 0], [1, 1]], dtype=np.float32)  # logits 1,1,2,2
    _, idx, gate = oracle.router(x, wr, None, 3)
    assert list(idx[0]) == [2, 3, 0]
    assert gate[0, 0] == gate[0, 1]


def test_router_translation_invariance():
    """Softmax routing is invariant to a shared translation of the router rows
    (ACE, 'RCR' and 'Theoretical Contributions')."""
    rng = np.random.default_rng(5)
    x = rng.normal(0, 1, (30, 16))
    wr = (rng.integers(-64, 64, (8, 16)) / 1024.0).astype(np.float32)
    v = (rng.integers(-64, 64, 16) / 1024.0).astype(np.float32)
    _, i1, g1 = oracle.router(x, wr, None, 3)
    _, i2, g2 = oracle.router(x, wr + v, None, 3)
    assert (i1 == i2).all()
    assert np.allclose(g1, g2, rtol=1e-12)


# -------------------------------------------------------------- power iteration
def _with_singular_values(rng, rows, cols, s):
    U, _ = np.linalg.qr(rng.normal(size=(rows, rows)))
    V, _ = np.linalg.qr(rng.normal(size=(cols, cols)))
    S = np.zeros((rows, cols))
    S[: len(s), : len(s)] = np.diag(s)
    return U @ S @ V.T


def test_power_iteration_matches_svd_with_gap():
    rng = np.random.default_rng(6)
    E, d, m = 2, 20, 12
    s = np.linspace(1.0, 0.2, m)
    s[0] = 2.0
    wg = np.stack([_with_singular_values(rng, d, m, s).T for _ in range(E)]).astype(np.float32)
    wu = np.stack([_with_singular_values(rng, d, m, s * 0.5).T for _ in range(E)]).astype(np.float32)
    wd = np.stack([_with_singular_values(rng, m, d, s * 3).T for _ in range(E)]).astype(np.float32)
    gamma = np.ones(d)
    layer = dict(gamma=gamma, wg=wg, wu=wu, wd=wd)
    sig = oracle.sigma_factors(gamma, wg, wu, wd, iters=200)
    for e in range(E):
        A, B, D = _page(layer, e)
        ref = [np.linalg.svd(M, compute_uv=False)[0] for M in (A, B, D)]
        assert np.allclose(sig[e], ref, rtol=1e-10)
    # spectral GSP products against numpy SVD of the explicit d x d products
    gs = oracle.gsp(gamma, wg, wu, wd, spectral=True, iters=400)
    for e in range(E):
        A, B, D = _page(layer, e)
        ref = [np.linalg.svd(M, compute_uv=False)[0] for M in (B, A @ D, A, B @ D)]
        assert np.allclose(gs["norms"][e], ref, rtol=1e-8)


def test_power_iteration_monotone_and_below_sigma1():
    rng = np.random.default_rng(7)
    d, m = 30, 16
    wg = rng.normal(0, 1, (1, m, d)).astype(np.float32)
    gamma = rng.uniform(0.5, 1.5, d)
    layer = dict(gamma=gamma, wg=wg, wu=wg, wd=rng.normal(0, 1, (1, d, m)).astype(np.float32))
    s1 = np.linalg.svd(_page(layer, 0)[0], compute_uv=False)[0]
    prev = 0.0
    for it in range(0, 40):
        s = oracle.sigma_factors(gamma, wg, wg, layer["wd"], iters=it)[0, 0]
        assert s <= s1 * (1 + 1e-12)
        assert s >= prev * (1 - 1e-12)
        prev = s
    assert abs(prev - s1) / s1 < 1e-2


# ------------------------------------------------------------------------ GSP
def _identity_experts(g, abc, n=4):
    E = len(abc)
    I = np.eye(n, dtype=np.float32)
    wg = np.stack([a * I for a, b, c in abc]).astype(np.float32)
    wu = np.stack([b * I for a, b, c in abc]).astype(np.float32)
    wd = np.stack([c * I for a, b, c in abc]).astype(np.float32)
    return np.full(n, g), wg, wu, wd, E


def test_gsp_closed_form_scaled_identities():
    gd = _gold("gsp_scaled_identity.json")
    gamma, wg, wu, wd, E = _identity_experts(gd["g"], gd["experts_abc"])
    fro = oracle.gsp(gamma, wg, wu, wd, spectral=False, eps=0.0)
    assert np.allclose(fro["a_tilde"], gd["expected_a_tilde_fro"], rtol=1e-14)
    assert np.allclose(fro["A"], gd["expected_A"], rtol=1e-14)
    spec = oracle.gsp(gamma, wg, wu, wd, spectral=True, iters=50, eps=0.0)
    assert np.allclose(spec["a_tilde"], gd["expected_a_tilde_spectral"], rtol=1e-12)
    assert np.allclose(spec["A"], gd["expected_A"], rtol=1e-12)


def test_gsp_closed_form_unequal_views():
    """Diagonal experts whose two views differ (a^up != a^gate), so the
    combination of the views and its normalisation are pinned by hand values."""
    gd = _gold("gsp_diagonal_views.json")
    diag = lambda rows: np.stack([np.diag(r) for r in rows]).astype(np.float32)
    wg, wu, wd = diag(gd["w_gate_diag"]), diag(gd["w_up_diag"]), diag(gd["w_down_diag"])
    gamma = np.ones(wg.shape[1])
    fro = oracle.gsp(gamma, wg, wu, wd, spectral=False, eps=0.0)
    assert np.allclose(fro["a_up"], gd["expected_a_up_fro"], rtol=1e-15)
    assert np.allclose(fro["a_gate"], gd["expected_a_gate_fro"], rtol=1e-15)
    assert np.allclose(fro["a_tilde"], gd["expected_a_tilde_fro"], rtol=1e-15)
    assert np.allclose(fro["A"], gd["expected_A_fro"], rtol=1e-14)
    spec = oracle.gsp(gamma, wg, wu, wd, spectral=True, iters=50, eps=0.0)
    assert np.allclose(spec["a_tilde"], gd["expected_a_tilde_spectral"], rtol=1e-12)
    assert np.allclose(spec["A"], gd["expected_A_spectral"], rtol=1e-12)


def test_gsp_frobenius_products_match_library_and_gram_identity():
    rng = np.random.default_rng(8)
    layer = _rand_layer(rng, E=3, d=20, m=12)
    r = oracle.gsp(layer["gamma"], layer["wg"], layer["wu"], layer["wd"], eps=1e-6)
    for e in range(3):
        A, B, D = _page(layer, e)
        ref = [np.linalg.norm(B, "fro"), np.linalg.norm(A @ D, "fro"),
               np.linalg.norm(A, "fro"), np.linalg.norm(B @ D, "fro")]
        assert np.allclose(r["norms"][e], ref, rtol=1e-12)
        # ||AD||_F^2 = <A^T A, D D^T>
        assert np.isclose(r["norms"][e][1] ** 2, np.sum((A.T @ A) * (D @ D.T)), rtol=1e-12)
    at = r["a_tilde"]
    assert np.allclose(r["A"], at / (at.mean() + 1e-6), rtol=1e-15)


@pytest.mark.parametrize("which", ["wg", "wu", "wd", "gamma"])
def test_gsp_exact_scaling_laws(which):
    """Scaling W^gate, W^up or W^down of one expert by 2 scales that expert's
    a~ by exactly 2 (each path has one factor of each matrix under the square
    root); scaling Gamma by 2 scales every a~ by 4 and leaves A^GSP fixed up
    to eps."""
    rng = np.random.default_rng(9)
    layer = _rand_layer(rng, E=3, d=16, m=8)
    base = oracle.gsp(layer["gamma"], layer["wg"], layer["wu"], layer["wd"], eps=0.0)
    mod = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in layer.items()}
    if which == "gamma":
        mod["gamma"] = mod["gamma"] * 2.0
    else:
        mod[which][1] *= np.float32(2.0)
    r = oracle.gsp(mod["gamma"], mod["wg"], mod["wu"], mod["wd"], eps=0.0)
    if which == "gamma":
        assert np.allclose(r["a_tilde"], 4.0 * base["a_tilde"], rtol=1e-14)
        assert np.allclose(r["A"], base["A"], rtol=1e-14)
    else:
        ratio = r["a_tilde"] / base["a_tilde"]
        assert np.allclose(ratio, [1.0, 2.0, 1.0], rtol=1e-14)
        if which == "wd":
            assert np.allclose(r["a_up"][1] / base["a_up"][1], 2.0, rtol=1e-14)
            assert np.allclose(r["a_gate"][1] / base["a_gate"][1], 2.0, rtol=1e-14)
        else:  # one path scales by 2, the other by 2 through its product norm
            assert np.allclose(r["a_up"][1] * r["a_gate"][1] /
                               (base["a_up"][1] * base["a_gate"][1]), 4.0, rtol=1e-14)


def test_gsp_permutation_equivariance():
    rng = np.random.default_rng(10)
    layer = _rand_layer(rng, E=4, d=12, m=6)
    perm = np.array([2, 0, 3, 1])
    a = oracle.gsp(layer["gamma"], layer["wg"], layer["wu"], layer["wd"])
    b = oracle.gsp(layer["gamma"], layer["wg"][perm], layer["wu"][perm], layer["wd"][perm])
    assert np.allclose(b["A"], a["A"][perm], rtol=1e-14)


# ------------------------------------------------------------------------ RCR
def test_rcr_closed_form_ln3():
    gd = _gold("rcr_ln3.json")
    d = m = 4
    wr = np.array([[0.5, -0.5, 0.5, -0.5], [-0.5, 0.5, -0.5, 0.5]], dtype=np.float32)
    I = np.eye(4, dtype=np.float32)
    wg = np.stack([I, I])
    wu = np.stack([I, I])
    wd = np.stack([I, 2 * I])
    r = oracle.rcr(np.full(d, L3), wr, wg, wu, wd, rho=1.0, eps=0.0)
    assert np.allclose(r["q"][0], [1, -1, 1, -1], rtol=0, atol=1e-15)
    assert np.allclose(r["a_tilde"], np.array(gd["expected_a_tilde_over_L2"]) * L3 ** 2, rtol=1e-14)
    assert np.allclose(r["A"], gd["expected_A"], rtol=1e-14)


def test_rcr_translation_invariance_and_scaling():
    rng = np.random.default_rng(11)
    layer = _rand_layer(rng, E=4, d=16, m=8)
    layer["wr"] = (rng.integers(-64, 64, (4, 16)) / 256.0).astype(np.float32)
    v = (rng.integers(-64, 64, 16) / 256.0).astype(np.float32)
    a = oracle.rcr(layer["gamma"], layer["wr"], layer["wg"], layer["wu"], layer["wd"])
    b = oracle.rcr(layer["gamma"], layer["wr"] + v, layer["wg"], layer["wu"], layer["wd"])
    assert np.array_equal(a["q"], b["q"])
    assert np.array_equal(a["A"], b["A"])
    for which in ("wu", "wd"):
        w = layer[which].copy()
        w[2] *= np.float32(2.0)
        args = dict(wg=layer["wg"], wu=layer["wu"], wd=layer["wd"])
        args[which] = w
        c = oracle.rcr(layer["gamma"], layer["wr"], args["wg"], args["wu"], args["wd"], eps=0.0)
        a0 = oracle.rcr(layer["gamma"], layer["wr"], layer["wg"], layer["wu"], layer["wd"], eps=0.0)
        assert np.allclose(c["a_tilde"] / a0["a_tilde"], [1, 1, 2, 1], rtol=1e-14)


def test_rcr_prototype_rms_is_rho():
    rng = np.random.default_rng(12)
    layer = _rand_layer(rng, E=5, d=32, m=8)
    r = oracle.rcr(layer["gamma"], layer["wr"], layer["wg"], layer["wu"], layer["wd"], rho=1.0, eps=0.0)
    assert np.allclose(np.sqrt(np.mean(r["q"] ** 2, axis=1)), 1.0, rtol=1e-14)
    centred = layer["wr"].astype(np.float64) - layer["wr"].astype(np.float64).mean(0)
    cos = np.sum(r["q"] * centred, 1) / np.linalg.norm(r["q"], axis=1) / np.linalg.norm(centred, axis=1)
    assert np.allclose(cos, 1.0, rtol=1e-14)            # q_e points along w_e - mean_j w_j
    r2 = oracle.rcr(layer["gamma"], layer["wr"], layer["wg"], layer["wu"], layer["wd"], rho=2.0, eps=0.0)
    assert np.allclose(r2["q"], 2.0 * r["q"], rtol=1e-15)


# ------------------------------------------------------------------ skip rule
def test_mask_rules():
    rng = np.random.default_rng(13)
    T, k, E = 400, 8, 16
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    g = np.sort(rng.dirichlet(np.ones(k), T), axis=1)[:, ::-1].copy()
    A_gsp = rng.uniform(0.5, 1.5, E)
    A_rcr = rng.uniform(0.5, 1.5, E)
    prev_skips = -1
    for tau in [-1.0, 0.0, 0.05, 0.1, 0.2, 0.5, 2.0]:
        r = oracle.mask(idx, g, A_gsp, A_rcr, tau)
        assert r["disagree"] == 0                      # max rule == intersection
        assert (r["keep"][:, 0] == 1).all()            # top-1 always retained
        assert np.allclose(r["c"], np.maximum(r["s_gsp"], r["s_rcr"]))
        assert np.allclose(r["s_gsp"], g * A_gsp[idx])
        skipped = (r["keep"] == 0)
        expect = (g * A_gsp[idx] < tau) & (g * A_rcr[idx] < tau)
        expect[:, 0] = False
        assert (skipped == expect).all()
        n = int(skipped.sum())
        assert n >= prev_skips                         # raising tau only adds skips
        prev_skips = n
    assert prev_skips == T * (k - 1)                   # tau = 2 skips every non-top-1


def test_fusion_ablation_rules():
    """The pages' fusion ablation (Min, Mean against ACE's Max) and the single
    views: set identities and closed forms, not the formulas retyped."""
    rng = np.random.default_rng(16)
    T, k, E = 300, 8, 16
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    g = np.sort(rng.dirichlet(np.ones(k), T), axis=1)[:, ::-1].copy()
    A_gsp = rng.uniform(0.5, 1.5, E)
    A_rcr = rng.uniform(0.5, 1.5, E)
    low_g = g * A_gsp[idx]
    low_r = g * A_rcr[idx]
    for tau in [0.0, 0.05, 0.1, 0.2, 2.0]:
        r = {f: oracle.mask(idx, g, A_gsp, A_rcr, tau, f) for f in oracle.FUSIONS}
        sk = {f: v["keep"] == 0 for f, v in r.items()}
        for v in r.values():
            assert (v["keep"][:, 0] == 1).all()          # top-1 retained under every rule
            assert v["disagree"] == 0
        lg, lr = low_g < tau, low_r < tau
        lg[:, 0] = lr[:, 0] = False
        assert (sk["min"] == (lg | lr)).all()            # Min: either view low (union)
        assert (sk["max"] == (lg & lr)).all()            # Max: both low (intersection)
        assert (sk["gsp"] == lg).all() and (sk["rcr"] == lr).all()
        assert not (sk["max"] & ~sk["mean"]).any()       # max-skips within mean-skips
        assert not (sk["mean"] & ~sk["min"]).any()       # mean-skips within min-skips
    # equal views: every rule is the same rule
    same = {f: oracle.mask(idx, g, A_gsp, A_gsp, 0.1, f) for f in oracle.FUSIONS}
    for f in oracle.FUSIONS:
        assert np.array_equal(same[f]["keep"], same["max"]["keep"])
        assert np.array_equal(same[f]["c"], same["gsp"]["c"])
    # A^RCR = 3 A^GSP: mean = 2 s^GSP, min = s^GSP, max = s^RCR, exactly
    m3 = {f: oracle.mask(idx, g, A_gsp, 3.0 * A_gsp, 0.1, f) for f in oracle.FUSIONS}
    assert np.allclose(m3["mean"]["c"], 2.0 * m3["gsp"]["c"], rtol=1e-15, atol=0)
    assert np.array_equal(m3["min"]["c"], m3["gsp"]["c"])
    assert np.array_equal(m3["max"]["c"], m3["rcr"]["c"])


def test_tau_quantile_skips_exactly_n():
    rng = np.random.default_rng(14)
    T, k = 100, 4
    c = rng.uniform(0, 1, (T, k))
    N = T * (k - 1)
    # slot r of every token routes to expert r with both tables at 1, so the
    # fused score of a slot is its gate, here c
    idx = np.tile(np.arange(k, dtype=np.int32), (T, 1))
    ones = np.ones(k)
    for n in [0, 1, 7, 150, N - 1, N]:
        tau = oracle.tau_quantile(c, n)
        assert int((c[:, 1:] < tau).sum()) == n
        # the mask's rule with the mapped tau skips exactly those n slots (the
        # candidate equal to tau is kept)
        mk = oracle.mask(idx, c, ones, ones, tau)
        assert int((mk["keep"] == 0).sum()) == n
    assert oracle.n_skip_for(1024, 8, 0.6) == 4915
    assert oracle.n_skip_for(64, 2, 0.5, of="nontop1") == 32
    # halves round up: 0.25 of 10 slots asks for 3, 0.5 of 3 non-top-1 slots for 2
    assert oracle.n_skip_for(10, 1, 0.25) == 3
    assert oracle.n_skip_for(3, 2, 0.5, of="nontop1") == 2


def test_compaction_order_and_bijection():
    rng = np.random.default_rng(15)
    T, k, E = 70, 4, 9
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    keep = (rng.uniform(size=(T, k)) < 0.6).astype(np.uint8)
    keep[:, 0] = 1
    r = oracle.compact(idx, keep, E)
    assert r["S"] == int(keep.sum())
    assert (r["counts"] == np.bincount(idx[keep == 1], minlength=E)).all()
    assert (np.diff(r["offsets"]) == r["counts"]).all() and r["offsets"][0] == 0
    e_of_slot = idx[r["slot_token"], r["slot_rank"]]
    key = e_of_slot.astype(np.int64) * T + r["slot_token"]
    assert (np.diff(key) > 0).all()                    # (expert, token) strictly increasing
    for s in range(r["S"]):
        assert r["slot_of"][r["slot_token"][s], r["slot_rank"][s]] == s
    assert (r["slot_of"][keep == 0] == -1).all()


# --------------------------------------------------------------- whole layer
def test_zero_skip_is_dense_topk_and_k_equals_E_is_softmax_mixture():
    rng = np.random.default_rng(16)
    E, d, m = 4, 12, 6
    layer = _rand_layer(rng, E=E, d=d, m=m)
    u = rng.normal(0, 1, (6, d))
    A = np.ones(E)
    # tau <= 0: nothing is skipped -> identical to the all-kept combine
    k = 2
    layer["k"] = k
    r = oracle.moe_forward(layer, u, 0.0, A, A)
    assert (r["keep"] == 1).all()
    dense = oracle.combine(r["x"], r["idx"], r["gate"], np.ones_like(r["keep"]),
                           layer["wg"], layer["wu"], layer["wd"])
    assert np.array_equal(r["y"], dense)
    # k = E with renormalisation: the dense softmax mixture of all experts
    layer["k"] = E
    r = oracle.moe_forward(layer, u, 0.0, A, A)
    from scipy.special import softmax
    p = softmax(r["x"] @ layer["wr"].astype(np.float64).T, axis=1)
    for t in range(6):
        ref = np.zeros(d)
        for e in range(E):
            _, f = oracle.swiglu(r["x"][t], layer["wg"][e], layer["wu"][e], layer["wd"][e])
            ref += p[t, e] * f
        assert np.allclose(r["y"][t], ref, rtol=1e-11, atol=1e-14)


def test_skipped_slots_drop_out_without_renormalisation():
    rng = np.random.default_rng(17)
    E, d, m = 5, 10, 4
    layer = _rand_layer(rng, E=E, d=d, m=m)
    layer["k"] = 3
    u = rng.normal(0, 1, (8, d))
    A = np.ones(E)
    r = oracle.moe_forward(layer, u, 0.3, A, A)
    for t in range(8):
        ref = np.zeros(d)
        for i in range(3):
            if r["keep"][t, i]:
                e = r["idx"][t, i]
                _, f = oracle.swiglu(r["x"][t], layer["wg"][e], layer["wu"][e], layer["wd"][e])
                ref += r["gate"][t, i] * f
        assert np.allclose(r["y"][t], ref, rtol=1e-13, atol=1e-15)
