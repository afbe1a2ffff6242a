"""Pins for the float64 oracle: closed forms, brute force, limits, finite differences.

None of these re-types the oracle's own formula. Each checks the oracle
against something the mathematics fixes independently of it, chosen so that
a dropped term, a wrong sign or index, or a transposed operand fails.
"""
import json
import os

import numpy as np
import pytest
from scipy.optimize import brentq

from oracle import attention as oa
from oracle import entmax as oe

ALPHAS = [1.25, 1.5, 2.0, 3.0]
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "entmax_rows.json")


def _rows(seed, r=64, n=40, scale=3.0):
    rng = np.random.default_rng(seed)
    return scale * rng.standard_normal((r, n))


# --- golden rows (hand-derived closed forms) --------------------------------

def test_golden_rows():
    with open(GOLDEN) as fh:
        cases = json.load(fh)["cases"]
    for c in cases:
        z = np.array(c["z"])[None, :]
        tau = oe.tau_bisect(z, None, c["alpha"])
        p = oe.probs(z, None, tau, c["alpha"])
        assert abs(tau[0] - c["tau"]) <= 1e-11, c
        np.testing.assert_allclose(p[0], c["p"], atol=1e-11)


# --- normalisation, sign, bracket -------------------------------------------

@pytest.mark.parametrize("alpha", ALPHAS)
def test_normalised_nonnegative_in_bracket(alpha):
    z = _rows(1)
    valid = np.random.default_rng(2).random(z.shape) < 0.7
    valid[:, 0] = True
    tau = oe.tau_bisect(z, valid, alpha)
    p = oe.probs(z, valid, tau, alpha)
    assert np.all(p >= 0)
    assert np.all(p[~valid] == 0)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-10)
    lo, hi = oe.bracket(z, valid, alpha)
    assert np.all(tau >= lo - 1e-12) and np.all(tau <= hi + 1e-12)
    # bracket ends are the pages' [(alpha-1) max s - 1, (alpha-1) max s - n^(1-alpha)]
    m = np.where(valid, z, -np.inf).max(axis=1)
    np.testing.assert_allclose(lo, m - 1.0)
    np.testing.assert_allclose(hi, m - valid.sum(axis=1) ** (1.0 - alpha))


# --- alpha = 2: sparsemax, sort-based closed form -----------------------------

def _sparsemax_sort(zrow):
    zs = np.sort(zrow)[::-1]
    cs = np.cumsum(zs)
    ks = np.arange(1, len(zs) + 1)
    kstar = ks[1.0 + ks * zs > cs].max()
    return (cs[kstar - 1] - 1.0) / kstar


def test_sparsemax_closed_form():
    z = _rows(3, r=50, n=25)
    tau = oe.tau_bisect(z, None, 2.0)
    ref = np.array([_sparsemax_sort(row) for row in z])
    np.testing.assert_allclose(tau, ref, atol=1e-11, rtol=0)


# --- alpha = 1.5: sort-based quadratic closed form ----------------------------

def _entmax15_sort(zrow):
    zs = np.sort(zrow)[::-1]
    best = None
    for K in range(1, len(zs) + 1):
        top = zs[:K]
        mu = top.mean()
        ss = ((top - mu) ** 2).sum()
        disc = (1.0 - ss) / K
        if disc < 0:
            break
        t = mu - np.sqrt(disc)
        if t < zs[K - 1]:
            best = t
    return best


def test_entmax15_closed_form():
    z = _rows(4, r=50, n=25)
    tau = oe.tau_bisect(z, None, 1.5)
    ref = np.array([_entmax15_sort(row) for row in z])
    np.testing.assert_allclose(tau, ref, atol=1e-11, rtol=0)


# --- alpha -> 1: softmax limit -------------------------------------------------

def test_softmax_limit():
    s = _rows(5, r=20, n=30, scale=1.5)
    sm = np.exp(s - s.max(axis=1, keepdims=True))
    sm /= sm.sum(axis=1, keepdims=True)
    errs = []
    for eps in (1e-2, 1e-3, 1e-4):
        alpha = 1.0 + eps
        z = eps * s
        tau = oe.tau_bisect(z, None, alpha)
        p = oe.probs(z, None, tau, alpha)
        errs.append(np.abs(p - sm).max())
    assert errs[1] < errs[0] / 5 and errs[2] < errs[1] / 5, errs
    assert errs[2] < 1e-3


# --- brute force over supports on tiny rows ----------------------------------

@pytest.mark.parametrize("alpha", ALPHAS)
def test_brute_force_supports(alpha):
    k = 1.0 / (alpha - 1.0)
    z = _rows(6, r=40, n=7, scale=1.0)
    tau = oe.tau_bisect(z, None, alpha)
    for row, t in zip(z, tau):
        zs = np.sort(row)[::-1]
        found = []
        for K in range(1, len(zs) + 1):
            lo_edge = zs[K] if K < len(zs) else zs[K - 1] - 1.0
            hi_edge = zs[K - 1]
            g = lambda x: np.sum((zs[:K] - x) ** k) - 1.0
            if g(lo_edge) >= 0 and g(hi_edge) <= 0:
                found.append(brentq(g, lo_edge, hi_edge, xtol=1e-14, rtol=1e-14))
        assert len(found) >= 1
        assert min(abs(f - t) for f in found) <= 1e-10


# --- special rows --------------------------------------------------------------

@pytest.mark.parametrize("alpha", ALPHAS)
def test_special_rows(alpha):
    # one allowed key: p = 1, tau = z - 1
    z = np.array([[0.7, 5.0, -2.0]])
    valid = np.array([[True, False, False]])
    tau = oe.tau_bisect(z, valid, alpha)
    assert abs(tau[0] - (0.7 - 1.0)) < 1e-11
    np.testing.assert_allclose(oe.probs(z, valid, tau, alpha), [[1.0, 0, 0]], atol=1e-11)
    # equal scores: uniform over the allowed keys
    z = np.full((1, 9), 0.3)
    tau = oe.tau_bisect(z, None, alpha)
    np.testing.assert_allclose(oe.probs(z, None, tau, alpha), np.full((1, 9), 1 / 9), atol=1e-11)
    assert abs(tau[0] - (0.3 - 9.0 ** (1 - alpha))) < 1e-11


# --- histogram lower bound -----------------------------------------------------

@pytest.mark.parametrize("alpha", ALPHAS)
@pytest.mark.parametrize("bins", [64, 256])
def test_histogram_bound(alpha, bins):
    z = _rows(7, r=200, n=300, scale=4.0)
    valid = np.random.default_rng(8).random(z.shape) < 0.8
    valid[:, 0] = True
    tau = oe.tau_bisect(z, valid, alpha)
    tau_h, tau_H = oe.histogram_tau(z, valid, alpha, bins)
    w = 1.0 / (bins - 1)
    # lower bound, upper bound, and within one bin width
    assert np.all(tau_h <= tau + 1e-12)
    assert np.all(tau_H >= tau - 1e-12)
    assert np.all(tau - tau_h <= w + 1e-12)
    # the support at tau_h contains the true support
    assert np.all(((z > tau_h[:, None]) & valid) | ~((z > tau[:, None]) & valid))


def test_histogram_counts_window():
    # top bin holds the max; entries below m - 1 are dropped; bins are left edges
    z = np.array([[1.0, 0.999, 0.5, -0.01, -0.5]])
    top, counts = oe.histogram_counts(z, None, bins=256)
    assert top[0] == 255
    assert counts[0, 0] == 1          # z = 1.0 in bin 255
    assert counts[0, 1] == 1          # 0.999 * 255 = 254.7 -> bin 254
    assert counts[0].sum() == 3       # -0.01 falls in bin -3, below the window
    assert counts[0, 255 - 127] == 1  # 0.5 * 255 = 127.5 -> bin 127


# --- hybrid solver ---------------------------------------------------------------

@pytest.mark.parametrize("alpha", ALPHAS)
def test_hybrid_solver_matches_bisection(alpha):
    z = _rows(9, r=300, n=200, scale=4.0)
    tau = oe.tau_bisect(z, None, alpha)
    t2, steps, fb = oe.hybrid_solve(z, None, alpha)
    assert np.all(np.abs(t2 - tau) <= 2e-6 * np.maximum(1.0, np.abs(tau)))
    assert np.all(steps <= 12)
    if alpha <= 2.0:
        # 1-2 steps from the histogram start for the smooth branches
        assert steps.mean() <= 2.5


def test_method_choice():
    assert oe.method_for_alpha(1.25) == "halley"
    assert oe.method_for_alpha(1.5) == "halley"
    assert oe.method_for_alpha(1.75) == "newton"
    assert oe.method_for_alpha(2.0) == "newton"
    assert oe.method_for_alpha(3.0) == "secant"


# --- attention forward -----------------------------------------------------------

def test_forward_identity_values_gives_p():
    # V = I makes O = P: checks the orientation of P V and the causal set
    rng = np.random.default_rng(10)
    n = 6
    Q = rng.standard_normal((1, 1, n, n))
    K = rng.standard_normal((1, 1, n, n))
    V = np.eye(n)[None, None]
    out = oa.forward(Q, K, V, 2.0, causal=True, block=2)
    s = (Q[0, 0] @ K[0, 0].T) / np.sqrt(n)
    for i in range(n):
        z = (2.0 - 1.0) * s[i, : i + 1]
        t = _sparsemax_sort(z)
        p = np.maximum(z - t, 0)
        np.testing.assert_allclose(out["O"][0, 0, i, : i + 1], p, atol=1e-11)
        np.testing.assert_allclose(out["O"][0, 0, i, i + 1:], 0, atol=0)


def test_causal_first_row():
    rng = np.random.default_rng(11)
    Q, K, V = (rng.standard_normal((2, 2, 10, 4)) for _ in range(3))
    out = oa.forward(Q, K, V, 1.5, causal=True, block=4)
    np.testing.assert_allclose(out["O"][:, :, 0], V[:, :, 0], atol=1e-12)
    z00 = 0.5 * (Q[:, :, 0] * K[:, :, 0]).sum(-1) / 2.0
    np.testing.assert_allclose(out["tau"][:, :, 0], z00 - 1.0, atol=1e-11)


def test_pack_bits():
    bits = np.zeros((2, 33), dtype=bool)
    bits[0, [0, 2]] = True
    bits[1, 32] = True
    words = oa.pack_bits(bits)
    assert words.tolist() == [[5, 0], [0, 1]]


def test_block_mask_block_diagonal():
    # keys of block J point along e_J; queries of block I along e_I, so only
    # the diagonal blocks carry weight. 40 blocks of 4 (two mask words).
    nb, bs = 40, 4
    n = nb * bs
    d = nb
    Q = np.zeros((1, 1, n, d))
    K = np.zeros((1, 1, n, d))
    rng = np.random.default_rng(12)
    for i in range(n):
        Q[0, 0, i, i // bs] = 20.0
        K[0, 0, i, i // bs] = 20.0 + rng.random()
    V = rng.standard_normal((1, 1, n, 3))
    out = oa.forward(Q, K, V, 1.5, causal=False, block=bs)
    assert np.array_equal(out["bits"][0, 0], np.eye(nb, dtype=bool))
    assert out["mask"].shape == (1, 1, nb, 2)
    assert out["mask"][0, 0, 33].tolist() == [0, 1 << 1]


def test_row_subset_matches_full():
    rng = np.random.default_rng(13)
    Q, K, V = (rng.standard_normal((1, 2, 50, 8)) for _ in range(3))
    full = oa.forward(Q, K, V, 1.5, causal=True, block=16)
    rows = np.array([0, 7, 31, 49])
    sub = oa.forward(Q, K, V, 1.5, causal=True, block=16, rows=rows)
    np.testing.assert_allclose(sub["O"], full["O"][:, :, rows], atol=1e-13)
    np.testing.assert_allclose(sub["tau"], full["tau"][:, :, rows], atol=1e-13)


# --- gradients: central finite differences -------------------------------------------

def _loss(Q, K, V, dO, alpha, causal):
    return float((oa.forward(Q, K, V, alpha, causal, block=4)["O"] * dO).sum())


@pytest.mark.parametrize("alpha", ALPHAS)
@pytest.mark.parametrize("causal", [False, True])
def test_gradients_finite_differences(alpha, causal):
    n, d = 6, 3
    for seed in range(100, 200):
        rng = np.random.default_rng(seed)
        Q, K, V, dO = (rng.standard_normal((1, 1, n, d)) for _ in range(4))
        Q *= 2.0
        out = oa.forward(Q, K, V, alpha, causal, block=4)
        s = (Q[0, 0] @ K[0, 0].T) / np.sqrt(d)
        z = (alpha - 1) * s
        valid = oa.allowed(np.arange(n), n, causal)
        gap = np.abs(z - out["tau"][0, 0][:, None])[valid]
        if gap.min() > 1e-3:
            break
    dQ, dK, dV = oa.backward(Q, K, V, dO, alpha, causal, chunk=4)
    h = 1e-6
    for X, G in ((Q, dQ), (K, dK), (V, dV)):
        num = np.zeros_like(X)
        for idx in np.ndindex(X.shape):
            old = X[idx]
            X[idx] = old + h
            lp = _loss(Q, K, V, dO, alpha, causal)
            X[idx] = old - h
            lm = _loss(Q, K, V, dO, alpha, causal)
            X[idx] = old
            num[idx] = (lp - lm) / (2 * h)
        err = np.abs(num - G).max() / max(1.0, np.abs(num).max())
        assert err < 1e-6, (alpha, causal, err)


def test_row_gradients_match_full():
    rng = np.random.default_rng(14)
    Q, K, V, dO = (rng.standard_normal((1, 2, 40, 8)) for _ in range(4))
    dQ, _, _ = oa.backward(Q, K, V, dO, 1.5, True, chunk=16)
    rows = np.array([0, 5, 39])
    np.testing.assert_allclose(oa.row_gradients(Q, K, V, dO, 1.5, True, rows), dQ[:, :, rows], atol=1e-13)


def test_key_column_subset_matches_full():
    rng = np.random.default_rng(15)
    Q, K, V, dO = (rng.standard_normal((1, 1, 30, 4)) for _ in range(4))
    _, dK, dV = oa.backward(Q, K, V, dO, 2.0, True, chunk=8)
    cols = np.array([0, 13, 29])
    _, dKs, dVs = oa.backward(Q, K, V, dO, 2.0, True, chunk=8, key_cols=cols)
    np.testing.assert_allclose(dKs, dK[:, :, cols], atol=1e-13)
    np.testing.assert_allclose(dVs, dV[:, :, cols], atol=1e-13)


@pytest.mark.parametrize("alpha", ALPHAS)
def test_hybrid_solver_plain_start(alpha):
    # the plain-bracket start (no histogram) converges to the same root, in more steps
    z = _rows(16, r=200, n=150, scale=4.0)
    tau = oe.tau_bisect(z, None, alpha)
    t2, steps, _ = oe.hybrid_solve(z, None, alpha, init="plain")
    assert np.all(np.abs(t2 - tau) <= 2e-5 * np.maximum(1.0, np.abs(tau)))
    _, steps_h, _ = oe.hybrid_solve(z, None, alpha)
    assert steps.mean() > steps_h.mean()


def test_secant_near_kink_converges():
    # alpha = 3 rows whose second key sits just above tau*: the bracketing secant still converges
    rng = np.random.default_rng(17)
    rows = []
    for _ in range(50):
        z = rng.standard_normal(30) * 0.3
        z[0] = 2.0
        rows.append(z)
    z = np.array(rows)
    tau = oe.tau_bisect(z, None, 3.0)
    # move the second largest entry to 1e-6 above the root (the root then shifts a little)
    order = np.argsort(-z, axis=1)
    z[np.arange(50), order[:, 1]] = tau + 1e-6
    tau = oe.tau_bisect(z, None, 3.0)
    t2, steps, _ = oe.hybrid_solve(z, None, 3.0)
    # |f| <= ftol = 1e-5 is accepted; on the flat side of the kink |f'| >= 1/2, so |tau - tau*| <= 2e-5
    assert np.all(np.abs(t2 - tau) <= 2.5e-5)


# --- softmax reference (for the dense baseline) ----------------------------------------------

def test_softmax_oracle_is_entmax_limit():
    # alpha -> 1 entmax (independent code) converges to the softmax oracle's output
    from oracle import softmax as osm
    rng = np.random.default_rng(20)
    Q, K, V = (rng.standard_normal((1, 1, 24, 4)) for _ in range(3))
    O_sm, lse = osm.forward(Q, K, V, causal=True)
    errs = []
    for eps in (1e-2, 1e-3):
        O_e = oa.forward(Q / eps, K, V, 1.0 + eps, causal=True, scale=eps / 2.0, block=8)["O"]
        errs.append(np.abs(O_e - O_sm).max())
    assert errs[1] < errs[0] / 5 and errs[1] < 2e-3, errs
    # lse of row 0 is its single score
    np.testing.assert_allclose(lse[0, 0, 0], (Q[0, 0, 0] @ K[0, 0, 0]) / 2.0, atol=1e-12)


def test_softmax_oracle_gradients_fd():
    from oracle import softmax as osm
    rng = np.random.default_rng(21)
    Q, K, V, dO = (rng.standard_normal((1, 1, 5, 3)) for _ in range(4))
    dQ, dK, dV = osm.backward(Q, K, V, dO, causal=True)
    h = 1e-6
    for X, G in ((Q, dQ), (K, dK), (V, dV)):
        num = np.zeros_like(X)
        for idx in np.ndindex(X.shape):
            old = X[idx]
            X[idx] = old + h
            lp = (osm.forward(Q, K, V, True)[0] * dO).sum()
            X[idx] = old - h
            lm = (osm.forward(Q, K, V, True)[0] * dO).sum()
            X[idx] = old
            num[idx] = (lp - lm) / (2 * h)
        assert np.abs(num - G).max() < 1e-7
