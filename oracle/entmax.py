"""Row-wise alpha-entmax in float64: normaliser, histogram bound, hybrid solver.

Test infrastructure only (see the package docstring).

Notation. For one query row, z_j = (alpha - 1) s_j over the allowed keys j,
k = 1 / (alpha - 1), and

    f(tau) = sum_j [z_j - tau]_+^k - 1 .

alpha-entmax gives p_j = [z_j - tau*]_+^k where f(tau*) = 0. f is
continuous and strictly decreasing wherever it is positive, and with
m = max_j z_j and n_i allowed keys the root lies in

    [m - 1, m - n_i^{1 - alpha}]

(at tau = m - 1 the top term alone is 1; at tau = m - n_i^{1-alpha} every
term is at most 1/n_i). Sources: alpha-entmax replaces softmax and needs a
root search for tau ("AdaSplash-2: Faster Differentiable Sparse
Attention", gist.science (de), section 1 "Problemstellung"; euno.news
summary, "方法论" item 1).

Rows are passed as 2-D arrays `z[r, n]` with a boolean `valid[r, n]` that
marks the allowed keys (causal masking, ragged rows). Entries outside
`valid` are ignored.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "row_max",
    "bracket",
    "tau_bisect",
    "probs",
    "histogram_counts",
    "histogram_tau",
    "hybrid_solve",
    "method_for_alpha",
]


def _as_rows(z, valid):
    z = np.asarray(z, dtype=np.float64)
    if z.ndim == 1:
        z = z[None, :]
    if valid is None:
        valid = np.ones(z.shape, dtype=bool)
    valid = np.asarray(valid, dtype=bool)
    if valid.ndim == 1:
        valid = valid[None, :]
    if not np.all(valid.any(axis=1)):
        raise ValueError("every row needs at least one allowed key")
    return z, valid


def row_max(z, valid=None):
    z, valid = _as_rows(z, valid)
    return np.where(valid, z, -np.inf).max(axis=1)


def bracket(z, valid, alpha):
    """The interval [m - 1, m - n_i^(1 - alpha)] that holds tau*."""
    z, valid = _as_rows(z, valid)
    m = row_max(z, valid)
    n_i = valid.sum(axis=1).astype(np.float64)
    return m - 1.0, m - n_i ** (1.0 - alpha)


def _candidates(z, valid, floor):
    """Compact each row to the entries above `floor` (a per-row value).

    For tau >= floor an entry z_j <= floor gives [z_j - tau]_+ = 0 exactly,
    so dropping it leaves f unchanged on that range. Returns a padded
    [r, c] array with -inf padding.
    """
    keep = valid & (z > floor[:, None])
    counts = keep.sum(axis=1)
    c = max(int(counts.max()), 1)
    out = np.full((z.shape[0], c), -np.inf)
    rr, cc = np.nonzero(keep)                  # row-major: entries of each row are contiguous
    starts = np.concatenate([[0], np.cumsum(counts)[:-1]])
    pos = np.arange(len(rr)) - starts[rr]
    out[rr, pos] = z[rr, cc]
    return out


def _f(zc, tau, k):
    """f(tau) = sum_j [z_j - tau]_+^k - 1 on compacted rows."""
    x = np.maximum(zc - tau[:, None], 0.0)
    return np.power(x, k).sum(axis=1) - 1.0


def tau_bisect(z, valid=None, alpha=1.5, tol=1e-12, max_iter=400):
    """tau* by bisection on [m - 1, m - n_i^(1-alpha)] until hi - lo <= tol * max(1, |tau|).

    Plain definition of the alpha-entmax normaliser: f(lo) >= 0 >= f(hi)
    holds at the start and is kept by every halving.
    """
    if not alpha > 1.0:
        raise ValueError("alpha must exceed 1")
    z, valid = _as_rows(z, valid)
    k = 1.0 / (alpha - 1.0)
    lo, hi = bracket(z, valid, alpha)
    zc = _candidates(z, valid, lo)
    for _ in range(max_iter):
        mid = 0.5 * (lo + hi)
        width_ok = (hi - lo) <= tol * np.maximum(1.0, np.abs(mid))
        if np.all(width_ok):
            break
        fm = _f(zc, mid, k)
        pos = fm > 0.0
        lo = np.where(pos & ~width_ok, mid, lo)
        hi = np.where(~pos & ~width_ok, mid, hi)
    return 0.5 * (lo + hi)


def probs(z, valid, tau, alpha):
    """p_j = [z_j - tau]_+^(1/(alpha-1)) on allowed keys, 0 elsewhere."""
    z, valid = _as_rows(z, valid)
    k = 1.0 / (alpha - 1.0)
    x = np.where(valid, np.maximum(z - np.asarray(tau, dtype=np.float64)[:, None], 0.0), 0.0)
    return np.power(x, k)


# ---------------------------------------------------------------------------
# Histogram lower bound.
#
# The pages describe a B-bin histogram of the scores built on chip while the
# key blocks stream past, and a conservative left-edge discretisation whose
# root tau_h is a provable lower bound on tau* (gist.science (de), section 2,
# "Streaming & Histogramm-Erstellung", "Theoretische Garantie"; euno.news
# summary, "方法论" item 2, "e.g. 256 bins"). The bin width, range and anchor
# are not stated. Reading used here:
#   * bins over z, width w = 1 / (B - 1);
#   * bin index b = floor(z / w), left edge e_b = b * w <= z;
#   * the window holds the B bins top - (B-1) .. top with top = floor(m / w),
#     i.e. it spans [e_top - 1, e_top + w) and so every z >= m - 1;
#   * entries below the window are dropped (they lie below m - 1 <= tau*).
# Replacing each z by e_b <= z and dropping entries can only lower f, so the
# root of the binned function is <= tau*. Raising each edge by w gives an
# upper bound tau_H = tau_h + w.
# ---------------------------------------------------------------------------


def histogram_counts(z, valid, bins=256):
    """Per row: (top bin index, counts[r, B]) with counts[:, j] for bin top - j."""
    z, valid = _as_rows(z, valid)
    w_inv = float(bins - 1)
    m = row_max(z, valid)
    top = np.floor(m * w_inv)
    b = np.floor(np.where(valid, z, -np.inf) * w_inv)
    j = top[:, None] - b  # offset below the top bin
    counts = np.zeros((z.shape[0], bins), dtype=np.int64)
    inwin = valid & (j >= 0) & (j <= bins - 1)
    rr, cc = np.nonzero(inwin)
    np.add.at(counts, (rr, j[rr, cc].astype(np.int64)), 1)
    return top, counts


def histogram_tau(z, valid=None, alpha=1.5, bins=256, tol=1e-13):
    """(tau_h, tau_H): root of the left-edge binned f, and tau_h + w.

    The binned function f_h(tau) = sum_b c_b [e_b - tau]_+^k - 1 is solved
    by bisection on [e_top - 1, e_top], where f_h(e_top - 1) >= c_top - 1 >= 0
    and f_h(e_top) = -1.
    """
    z, valid = _as_rows(z, valid)
    k = 1.0 / (alpha - 1.0)
    w = 1.0 / (bins - 1)
    top, counts = histogram_counts(z, valid, bins)
    edges = (top[:, None] - np.arange(bins)[None, :]) * w  # e_b for offset j
    lo = top * w - 1.0
    hi = top * w
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if np.all(hi - lo <= tol * np.maximum(1.0, np.abs(mid))):
            break
        x = np.maximum(edges - mid[:, None], 0.0)
        fm = (counts * np.power(x, k)).sum(axis=1) - 1.0
        pos = fm >= 0.0
        lo = np.where(pos, mid, lo)
        hi = np.where(pos, hi, mid)
    return lo, lo + w


# ---------------------------------------------------------------------------
# Safeguarded hybrid solver.
#
# Method by alpha (gist.science (de), "Hybrid Solver & Sparsity-Awareness";
# gist.science (hi) technical summary, section 2, hybrid solver strategy):
# Halley for alpha <= 1.5, Newton for 1.5 < alpha <= 2, secant above 2 (the
# two pages disagree on alpha = 2 itself; Newton is used there, where f is
# piecewise linear). A step that leaves the current bracket is replaced by
# bisection.
#
# Readings where the pages are silent:
#  * start: lo = max(tau_h, m - 1), hi = min(tau_h + w, m - n_i^(1-alpha)),
#    first evaluation at lo; with the plain-bracket start (no histogram)
#    lo = m - 1, hi = m - n_i^(1-alpha);
#  * Halley / Newton stop when |f(tau)| <= ftol, or when a step moves tau by at
#    most xtol * max(1, |tau|), or after max_iter steps;
#  * the secant is the bracketing (Illinois) form: the first step is the
#    secant through both bracket ends (f evaluated at both in one sweep), each
#    later step the secant through the current ends, halving the f value of
#    an end that is kept twice in a row; it stops when |f| <= ftol, when the
#    bracket is narrower than xtol_bracket * max(1, |tau|) (about four float32
#    ulps), or after max_iter steps.
# ---------------------------------------------------------------------------

HALLEY, NEWTON, SECANT = "halley", "newton", "secant"
XTOL_BRACKET = 4.8e-7


def method_for_alpha(alpha):
    if alpha <= 1.5:
        return HALLEY
    if alpha <= 2.0:
        return NEWTON
    return SECANT


def _sums(zc, tau, k):
    """F_r = sum over the support of (z - tau)^(k - r), r = 0, 1, 2."""
    x = zc - tau[:, None]
    sup = x > 0.0
    xs = np.where(sup, x, 1.0)
    F0 = np.where(sup, np.power(xs, k), 0.0).sum(axis=1)
    F1 = np.where(sup, np.power(xs, k - 1.0), 0.0).sum(axis=1)
    F2 = np.where(sup, np.power(xs, k - 2.0), 0.0).sum(axis=1)
    return F0, F1, F2


def hybrid_solve(z, valid=None, alpha=1.5, bins=256, ftol=1e-5, xtol=1e-6, max_iter=None, init="histogram"):
    """Returns (tau, steps, fallbacks) per row.

    `steps` counts solver updates of tau after the start; `fallbacks` counts
    the updates that were bisection because the method's step left the
    bracket (or was not finite).
    """
    z, valid = _as_rows(z, valid)
    if max_iter is None:
        max_iter = 12 if init == "histogram" else 24
    k = 1.0 / (alpha - 1.0)
    method = method_for_alpha(alpha)
    lo0, hi0 = bracket(z, valid, alpha)
    zc = _candidates(z, valid, lo0)
    r = z.shape[0]
    if init == "histogram":
        tau_h, tau_H = histogram_tau(z, valid, alpha, bins)
        lo = np.maximum(tau_h, lo0)
        hi = np.minimum(tau_H, hi0)
        bad = lo > hi
        lo = np.where(bad, lo0, lo)
        hi = np.where(bad, hi0, hi)
    else:
        lo, hi = lo0.copy(), hi0.copy()
    steps = np.zeros(r, dtype=np.int64)
    fallbacks = np.zeros(r, dtype=np.int64)
    done = np.zeros(r, dtype=bool)

    if method == SECANT:
        flo = _f(zc, lo, k)
        fhi = _f(zc, hi, k)
        tau = lo.copy()
        # an end whose sign contradicts the bracket is off only by rounding: accept it
        stop_lo = (np.abs(flo) <= ftol) | (flo < 0.0)
        stop_hi = ~stop_lo & ((np.abs(fhi) <= ftol) | (fhi > 0.0))
        tau = np.where(stop_hi, hi, tau)
        done = stop_lo | stop_hi
        side = np.zeros(r, dtype=np.int64)
        first = True
        for _ in range(max_iter + 1):
            if not first:
                fc = _f(zc, tau, k)
                conv = ~done & (np.abs(fc) <= ftol)
                done |= conv
                act = ~done
                pos = fc > 0.0
                up = act & pos
                dn = act & ~pos
                lo = np.where(up, tau, lo)
                flo = np.where(up, fc, flo)
                fhi = np.where(up & (side == 1), 0.5 * fhi, fhi)
                hi = np.where(dn, tau, hi)
                fhi = np.where(dn, fc, fhi)
                flo = np.where(dn & (side == -1), 0.5 * flo, flo)
                side = np.where(up, 1, np.where(dn, -1, side))
            first = False
            act = ~done & (steps < max_iter)
            if not act.any():
                break
            with np.errstate(divide="ignore", invalid="ignore"):
                cand = hi - fhi * (hi - lo) / (fhi - flo)
            ok = np.isfinite(cand) & (cand > lo) & (cand < hi)
            new = np.where(ok, cand, 0.5 * (lo + hi))
            fallbacks += (act & ~ok).astype(np.int64)
            steps += act.astype(np.int64)
            tau = np.where(act, new, tau)
            narrow = (hi - lo) <= XTOL_BRACKET * np.maximum(1.0, np.abs(tau))
            done |= act & (narrow | (steps >= max_iter))
        return tau, steps, fallbacks

    tau = lo.copy()
    for _ in range(max_iter + 1):
        F0, F1, F2 = _sums(zc, tau, k)
        f = F0 - 1.0
        done |= ~done & (np.abs(f) <= ftol)
        if np.all(done):
            break
        pos = f > 0.0
        lo = np.where(~done & pos, np.maximum(lo, tau), lo)
        hi = np.where(~done & ~pos, np.minimum(hi, tau), hi)
        fp = -k * F1
        with np.errstate(divide="ignore", invalid="ignore"):
            if method == HALLEY:
                fpp = k * (k - 1.0) * F2
                cand = tau - 2.0 * f * fp / (2.0 * fp * fp - f * fpp)
            else:
                cand = tau - f / fp
        ok = np.isfinite(cand) & (cand > lo) & (cand < hi)
        new = np.where(ok, cand, 0.5 * (lo + hi))
        active = ~done & (steps < max_iter)
        fallbacks += (active & ~ok).astype(np.int64)
        steps += active.astype(np.int64)
        small = np.abs(new - tau) <= xtol * np.maximum(1.0, np.abs(tau))
        tau = np.where(active, new, tau)
        done |= active & small
        done |= steps >= max_iter
        if np.all(done):
            break
    return tau, steps, fallbacks
