"""alpha-entmax attention forward and backward in float64 (test infrastructure only).

Definition (the plainest reading of the AdaSplash-2 pages, which state that
alpha-entmax replaces the softmax normaliser, yields exact zeros and needs a
root search for tau; the formula is the standard alpha-entmax one):

    s_ij = scale * q_i . k_j          (scale = 1/sqrt(d) unless given)
    z_ij = (alpha - 1) * s_ij         for allowed j (j <= i when causal)
    p_ij = [z_ij - tau_i]_+^(1/(alpha-1)),  sum_j p_ij = 1
    O_i  = sum_j p_ij v_j

Backward, with g_ij = dO_i . v_j and u_ij = p_ij^(2 - alpha) on the support
(= [z_ij - tau_i]_+^(k-1), k = 1/(alpha-1)), 0 elsewhere:

    delta_i = sum_j u_ij g_ij / sum_j u_ij
    dS_ij   = u_ij (g_ij - delta_i)        (gradient with respect to s_ij)
    dQ = scale * dS K,   dK = scale * dS^T Q,   dV = P^T dO

Block mask: bit (I, J) is set when some entry of query block I and key
block J is nonzero, packed 32 key blocks per uint32, bit J % 32 of word
J // 32 ("AdaSplash-2", gist.science (de), section 2, "Bit-Packed Block
Mask"; gist.science (hi) technical summary, section 2, bit-packed block
masking).

Rows are independent in the forward, so they may be computed in chunks of
rows; every sum over keys is taken whole. p, u and dS vanish off the support
{j : z_ij > tau_i}, so every sum that involves them runs over the support
entries only (exact). The key-side sums of dK and dV accumulate over row
chunks in float64.
"""
from __future__ import annotations

import numpy as np

from . import entmax

__all__ = ["allowed", "scores", "forward", "backward", "row_gradients", "block_mask", "pack_bits"]


def allowed(rows: np.ndarray, n: int, causal: bool) -> np.ndarray:
    """valid[r, j]: key j is visible to query row rows[r]."""
    j = np.arange(n)[None, :]
    if causal:
        return j <= np.asarray(rows)[:, None]
    return np.ones((len(rows), n), dtype=bool)


def scores(q: np.ndarray, k: np.ndarray, scale: float) -> np.ndarray:
    """s = scale * q k^T in float64 for one head; q [r, d], k [n, d]."""
    return scale * (np.asarray(q, np.float64) @ np.asarray(k, np.float64).T)


def _row_forward(q, k, v, rows, alpha, causal, scale):
    """Forward for query rows `rows` of one head.

    The support S_i = {j : p_ij > 0} is kept as coordinate lists (rr, cc);
    p, u and every product with them are summed over the support only,
    which is exact because p_ij = u_ij = 0 off the support.
    """
    n = k.shape[0]
    valid = allowed(rows, n, causal)
    z = (alpha - 1.0) * scores(q[rows], k, scale)
    tau = entmax.tau_bisect(z, valid, alpha)
    kk = 1.0 / (alpha - 1.0)
    x = np.where(valid, z - tau[:, None], 0.0)
    rr, cc = np.nonzero(x > 0.0)
    xs = x[rr, cc]
    p_s = np.power(xs, kk)
    u_s = np.power(xs, kk - 1.0)
    v64 = np.asarray(v, np.float64)
    r = len(rows)
    dv = v64.shape[1]
    o = np.zeros((r, dv))
    obar = np.zeros((r, dv))
    np.add.at(o, rr, p_s[:, None] * v64[cc])
    np.add.at(obar, rr, u_s[:, None] * v64[cc])
    sum_u = np.bincount(rr, weights=u_s, minlength=r)
    return dict(z=z, valid=valid, tau=tau, rr=rr, cc=cc, p_s=p_s, u_s=u_s, O=o, Obar=obar, sum_u=sum_u, n=n)


def _dense(res, vals):
    """Scatter support values into a dense [r, n] array."""
    out = np.zeros((len(res["tau"]), res["n"]))
    out[res["rr"], res["cc"]] = vals
    return out


def pack_bits(bits: np.ndarray) -> np.ndarray:
    """Pack a boolean [..., nb] array into uint32 words, 32 blocks per word."""
    bits = np.asarray(bits, dtype=bool)
    nb = bits.shape[-1]
    nw = (nb + 31) // 32
    padded = np.zeros(bits.shape[:-1] + (nw * 32,), dtype=np.uint64)
    padded[..., :nb] = bits
    padded = padded.reshape(bits.shape[:-1] + (nw, 32))
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    return (padded * weights).sum(axis=-1).astype(np.uint32)


def block_mask(p: np.ndarray, block: int):
    """(bits[nqb, nkb], block max p[nqb, nkb]) for one head's full P [n, n]."""
    n_q, n_k = p.shape
    nqb = (n_q + block - 1) // block
    nkb = (n_k + block - 1) // block
    pad = np.zeros((nqb * block, nkb * block))
    pad[:n_q, :n_k] = p
    bmax = pad.reshape(nqb, block, nkb, block).max(axis=(1, 3))
    return bmax > 0.0, bmax


def forward(Q, K, V, alpha, causal, scale=None, block=64, rows=None, chunk=256):
    """Forward for every (b, h); returns a dict of float64 arrays.

    Q, K, V: [B, H, n, d]. With `rows` given (sorted indices), only those
    query rows are computed: O, tau and mask rows are then [B, H, len(rows), ...]
    and the mask is the per-row key-block bits (not packed into query blocks).
    """
    Q = np.asarray(Q)
    B, H, n, d = Q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    full = rows is None
    rows = np.arange(n) if full else np.asarray(rows)
    r = len(rows)
    nkb = (n + block - 1) // block
    dv = np.asarray(V).shape[-1]
    O = np.zeros((B, H, r, dv))
    Obar = np.zeros((B, H, r, dv))
    tau = np.zeros((B, H, r))
    sum_u = np.zeros((B, H, r))
    row_bits = np.zeros((B, H, r, nkb), dtype=bool)
    row_bmax = np.zeros((B, H, r, nkb))
    support = np.zeros((B, H, r), dtype=np.int64)
    for b in range(B):
        for h in range(H):
            for c0 in range(0, r, chunk):
                sel = rows[c0:c0 + chunk]
                res = _row_forward(Q[b, h], K[b, h], V[b, h], sel, alpha, causal, scale)
                sl = slice(c0, c0 + len(sel))
                O[b, h, sl] = res["O"]
                Obar[b, h, sl] = res["Obar"]
                tau[b, h, sl] = res["tau"]
                sum_u[b, h, sl] = res["sum_u"]
                bm = np.zeros((len(sel), nkb))
                np.maximum.at(bm, (res["rr"], res["cc"] // block), res["p_s"])
                row_bmax[b, h, sl] = bm
                row_bits[b, h, sl] = bm > 0.0
                support[b, h, sl] = np.bincount(res["rr"], minlength=len(sel))
    out = dict(O=O, Obar=Obar, tau=tau, sum_u=sum_u, row_bits=row_bits, row_bmax=row_bmax,
               support=support, rows=rows, scale=scale)
    if full:
        nqb = (n + block - 1) // block
        padb = np.zeros((B, H, nqb * block, nkb), dtype=bool)
        padm = np.zeros((B, H, nqb * block, nkb))
        padb[:, :, :n] = row_bits
        padm[:, :, :n] = row_bmax
        bits = padb.reshape(B, H, nqb, block, nkb).any(axis=3)
        bmax = padm.reshape(B, H, nqb, block, nkb).max(axis=3)
        out["bits"] = bits
        out["bmax"] = bmax
        out["mask"] = pack_bits(bits)
    return out


def _row_backward(q, k, v, do, res, scale):
    """delta, dS on the support, and dQ rows for one chunk (res from _row_forward)."""
    rr, cc = res["rr"], res["cc"]
    g_s = np.einsum("ij,ij->i", do[res_rows(res)][rr], v[cc])          # g_ij = dO_i . v_j on the support
    r = len(res["tau"])
    delta = np.bincount(rr, weights=res["u_s"] * g_s, minlength=r) / res["sum_u"]
    ds_s = res["u_s"] * (g_s - delta[rr])
    dq = np.zeros((r, q.shape[1]))
    np.add.at(dq, rr, ds_s[:, None] * k[cc])
    return delta, ds_s, scale * dq


def res_rows(res):
    return res["rows"]


def backward(Q, K, V, dO, alpha, causal, scale=None, chunk=256, key_cols=None):
    """(dQ, dK, dV) in float64 for every (b, h).

    tau is recomputed here by `entmax.tau_bisect` (every row is needed for
    the key-side sums). With `key_cols` given, dK and dV are returned only
    for those key columns; dQ is returned for all rows.
    """
    Q = np.asarray(Q)
    B, H, n, d = Q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    cols = np.arange(n) if key_cols is None else np.asarray(key_cols)
    col_of = np.full(n, -1)
    col_of[cols] = np.arange(len(cols))
    dv_ = np.asarray(V).shape[-1]
    dQ = np.zeros((B, H, n, d))
    dK = np.zeros((B, H, len(cols), d))
    dV = np.zeros((B, H, len(cols), dv_))
    rows_all = np.arange(n)
    for b in range(B):
        for h in range(H):
            q = np.asarray(Q[b, h], np.float64)
            k = np.asarray(K[b, h], np.float64)
            v = np.asarray(V[b, h], np.float64)
            do = np.asarray(dO[b, h], np.float64)
            for c0 in range(0, n, chunk):
                sel = rows_all[c0:c0 + chunk]
                res = _row_forward(q, k, v, sel, alpha, causal, scale)
                res["rows"] = sel
                _, ds_s, dq = _row_backward(q, k, v, do, res, scale)
                dQ[b, h, sel] = dq
                rr, cc = res["rr"], res["cc"]
                m = col_of[cc] >= 0                       # support entries in the requested columns
                ci = col_of[cc[m]]
                np.add.at(dK[b, h], ci, scale * ds_s[m][:, None] * q[sel][rr[m]])
                np.add.at(dV[b, h], ci, res["p_s"][m][:, None] * do[sel][rr[m]])
    return dQ, dK, dV


def row_gradients(Q, K, V, dO, alpha, causal, rows, scale=None):
    """dQ for selected query rows only (each row's dQ needs only its own row)."""
    Q = np.asarray(Q)
    B, H, n, d = Q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    rows = np.asarray(rows)
    dQ = np.zeros((B, H, len(rows), d))
    for b in range(B):
        for h in range(H):
            q = np.asarray(Q[b, h], np.float64)
            k = np.asarray(K[b, h], np.float64)
            v = np.asarray(V[b, h], np.float64)
            do = np.asarray(dO[b, h], np.float64)
            res = _row_forward(q, k, v, rows, alpha, causal, scale)
            res["rows"] = rows
            _, _, dq = _row_backward(q, k, v, do, res, scale)
            dQ[b, h] = dq
    return dQ
