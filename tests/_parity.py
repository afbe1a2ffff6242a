"""Helpers for GPU-vs-oracle parity tests (inputs from adaptive_sparse_flash_b200.inputs)."""
import numpy as np

# tolerances fixed by the benchmark spec for this path
TAU_REL = 1e-3
BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
FP32_ABS = 1e-4
MASK_EXEMPT_P = 1e-3


def to_torch(arrs, dtype, device="cuda"):
    import torch
    out = {}
    for k, v in arrs.items():
        t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32))
        out[k] = t.to(device=device, dtype=dtype).contiguous()
    return out


def unpack_mask(words: np.ndarray, nkb: int) -> np.ndarray:
    """uint32 words [..., nw] -> bool [..., nkb]."""
    w = np.asarray(words).astype(np.uint32)
    bits = (w[..., :, None] >> np.arange(32, dtype=np.uint32)) & 1
    return bits.reshape(w.shape[:-1] + (w.shape[-1] * 32,))[..., :nkb].astype(bool)


def check_tau(tau_gpu, tau_ref, where=""):
    tau_gpu = np.asarray(tau_gpu, np.float64)
    err = np.abs(tau_gpu - tau_ref) / np.maximum(1.0, np.abs(tau_ref))
    assert np.all(np.isfinite(tau_gpu)), where
    assert err.max() <= TAU_REL, f"{where} tau rel err {err.max():.3e}"
    return err.max()


def check_close(gpu, ref, max_abs, mean_abs=None, where=""):
    gpu = np.asarray(gpu, np.float64)
    diff = np.abs(gpu - ref)
    assert np.all(np.isfinite(gpu)), f"{where}: non-finite output"
    assert diff.max() <= max_abs, f"{where}: max abs err {diff.max():.3e} > {max_abs}"
    if mean_abs is not None:
        assert diff.mean() <= mean_abs, f"{where}: mean abs err {diff.mean():.3e} > {mean_abs}"
    return diff.max(), diff.mean()


def check_mask(mask_gpu_words, bits_ref, bmax_ref, where=""):
    """Bit-exact except blocks whose oracle max p < 1e-3."""
    nkb = bits_ref.shape[-1]
    g = unpack_mask(mask_gpu_words, nkb)
    bad = (g != bits_ref) & ~(bmax_ref < MASK_EXEMPT_P)
    assert not bad.any(), f"{where}: {int(bad.sum())} mask bits differ (of {bits_ref.size})"
    return int((g != bits_ref).sum())


def grad_sensitivity(q, k, v, do, alpha, causal, scale=None):
    """Bounds on the output and gradient error that float32 scores alone can cause, for one head (float64).

    Returns (dQ per query row, dK per key column, dV per key column, O per query row) bounds of the max abs
    change of each row / column when every score z_ij moves by up to

        eps_ij = 2^-21 |z|_ij  +  1e-5 / (k sum_j u_ij)  +  4 ulp_f32(tau_i)

    the accumulation error of a float32 dot product of d exact products (|z|_ij = (alpha - 1) scale
    sum_d |q_id k_jd|), plus the error of tau that the solver's stop |f| <= 1e-5 leaves (f' = -k sum u)
    and its float32 rounding. With u = x^(k-1) and p = x^k (x = z - tau, k = 1 / (alpha - 1)):
      * du_ij, dp_ij: the largest change of u, p over x +- eps_ij (an entry may leave or join the support);
      * delta_i = sum u g / sum u is a u-weighted mean of g = dO v^T: it moves by at most the range R_i of g
        over the entries that are or may become support, and by M_i R_i / (sum u - M_i) while the unstable
        u mass M_i = sum_j du_ij is below half of sum u;
      * dS_ij = u_ij (g_ij - delta_i) then moves by du_ij |g_ij - delta_i| + (u_ij + du_ij) d delta_i, and
        dQ_i = scale sum_j dS_ij k_j, dK_j = scale sum_i dS_ij q_i, dV_j = sum_i p_ij dO_i, O_i = sum_j p_ij v_j
        by the sums of those changes times the max-norm of k_j, q_i, dO_i, v_j.
    For alpha < 2 u is continuous in x and the bounds are tiny; for alpha > 2 u = x^(k-1) is unbounded as
    x -> 0+ (alpha = 3: u = x^-1/2), so a row with a support entry within rounding of tau has gradients
    that no float32 computation of the scores determines.
    """
    from oracle import attention as oa
    from oracle import entmax as oe
    n, d = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    kk = 1.0 / (alpha - 1.0)
    q64, k64 = np.asarray(q, np.float64), np.asarray(k, np.float64)
    z = (alpha - 1.0) * scale * (q64 @ k64.T)
    valid = oa.allowed(np.arange(n), n, causal)
    tau = oe.tau_bisect(z, valid, alpha)
    x = np.where(valid, z - tau[:, None], -1.0)

    def ufun(t, power):
        tp = np.where(t > 0, t, 1.0)
        return np.where(valid & (t > 0), tp ** power, 0.0)

    u = ufun(x, kk - 1.0)
    p = ufun(x, kk)
    g = np.asarray(do, np.float64) @ np.asarray(v, np.float64).T
    su = u.sum(1)
    delta = (u * g).sum(1) / np.maximum(su, 1e-300)
    eps = 2.0 ** -21 * (alpha - 1.0) * scale * (np.abs(q64) @ np.abs(k64).T)
    eps += (1e-5 / np.maximum(kk * su, 1e-300) +
            4.0 * np.spacing(np.abs(tau).astype(np.float32)).astype(np.float64))[:, None]
    du = np.maximum(np.abs(ufun(x + eps, kk - 1.0) - u), np.abs(ufun(x - eps, kk - 1.0) - u))
    dp = np.maximum(np.abs(ufun(x + eps, kk) - p), np.abs(ufun(x - eps, kk) - p))
    near = valid & (x > -eps)
    R = np.where(near.any(1), np.where(near, g, -np.inf).max(1) - np.where(near, g, np.inf).min(1), 0.0)
    M = du.sum(1)
    ddelta = np.where(M >= 0.5 * su, R, np.minimum(R, M * R / np.maximum(su - M, 1e-300)))
    dds = du * np.abs(g - delta[:, None]) + (u + du) * ddelta[:, None]
    kinf = np.abs(k64).max(1)
    qinf = np.abs(q64).max(1)
    doinf = np.abs(np.asarray(do, np.float64)).max(1)
    vinf = np.abs(np.asarray(v, np.float64)).max(1)
    return scale * dds @ kinf, scale * qinf @ dds, doinf @ dp, dp @ vinf


def check_grads_bounded(gpu, ref, sens, where, max_abs=BF16_MAX_ABS, mean_abs=BF16_MEAN_ABS, cap=None):
    """Gradient rows (dQ) or columns (dK, dV) against the oracle where float32 scores cannot fix them all.

    Every row must lie within max_abs plus twice its sensitivity bound (grad_sensitivity); the rows whose
    bound is below max_abs keep the mean bound; with `cap`, at most that fraction of the rows may exceed
    max_abs at all (callers may instead cap the total over several heads).
    Returns (rows over max_abs, rows whose bound exceeds max_abs, rows).
    """
    gpu = np.asarray(gpu, np.float64)
    diff = np.abs(gpu - ref)
    assert np.all(np.isfinite(gpu)), f"{where}: non-finite output"
    err = diff.max(axis=-1)
    assert np.all(err <= max_abs + 2.0 * sens), (
        f"{where}: {int((err > max_abs + 2.0 * sens).sum())} rows beyond their bound, worst "
        f"{float((err / (max_abs + 2.0 * sens)).max()):.2f}x")
    over = int((err > max_abs).sum())
    if cap is not None:
        assert over <= cap * len(err), f"{where}: {over} of {len(err)} rows over {max_abs} (cap {cap})"
    well = sens <= max_abs
    if well.any():
        assert diff[well].mean() <= mean_abs, f"{where}: mean abs err {diff[well].mean():.3e} on resolvable rows"
    return over, int((~well).sum()), len(err)
