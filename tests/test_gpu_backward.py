"""GPU backward parity (dQ, dK, dV) against the float64 oracle, and the dense softmax baseline."""
import numpy as np
import pytest

from adaptive_sparse_flash_b200 import inputs
from oracle import attention as oa
from oracle import softmax as osm

from _parity import BF16_MAX_ABS, BF16_MEAN_ABS, check_close, check_mask, check_tau, conditioning, to_torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from adaptive_sparse_flash_b200 import build
    build.build()
    return torch


def _fwd_bwd(torch_cuda, arr, alpha, causal):
    from adaptive_sparse_flash_b200 import binding as b
    t = to_torch(arr, torch_cuda.bfloat16)
    f = b.forward(t["Q"], t["K"], t["V"], alpha, causal)
    dQ, dK, dV = b.backward(t["Q"], t["K"], t["V"], f, t["dO"])
    torch_cuda.cuda.synchronize()
    assert b.entmax_attn_check() == 0
    return (f.O.float().cpu().numpy(), f.tau.cpu().numpy(), f.mask.cpu().numpy().view(np.uint32),
            dQ.cpu().numpy(), dK.cpu().numpy(), dV.cpu().numpy())


def _check_grads(g, ref, where, max_abs=BF16_MAX_ABS, mean_abs=BF16_MEAN_ABS):
    for name, x, y in zip(("dQ", "dK", "dV"), g, ref):
        check_close(x, y, max_abs, mean_abs, f"{where} {name}")


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0, 3.0])
@pytest.mark.parametrize("causal", [True, False])
def test_bwd_small(torch_cuda, alpha, causal):
    arr = inputs.clustered(1, 2, 640, 64, centres=32, beta_q=2.0, seed=21)
    O, tau, mask, dQ, dK, dV = _fwd_bwd(torch_cuda, arr, alpha, causal)
    ref = oa.forward(arr["Q"], arr["K"], arr["V"], alpha, causal)
    check_tau(tau, ref["tau"], "bwd small")
    check_close(O, ref["O"], BF16_MAX_ABS, BF16_MEAN_ABS, "bwd small O")
    rdQ, rdK, rdV = oa.backward(arr["Q"], arr["K"], arr["V"], arr["dO"], alpha, causal)
    _check_grads_conditioned(arr, alpha, causal, (dQ, dK, dV), (rdQ, rdK, rdV), f"bwd small a={alpha} c={causal}")


# reading for alpha >= 2 (see _parity.conditioning): alpha = 2 rows with an entry within float32 rounding
# of tau (flip), alpha > 2 rows with a support entry below 1e-2 are reported and left out of the gradient
# comparison; alpha > 2 rows with a support entry below 1e-4 are left out of the O comparison.
GRAD_FLIP = 2e-6
GRAD_XMIN = "grad"  # per-row bound from _parity.grad_xmin
FWD_XMIN = 1e-4


def _grad_conditioning(arr, alpha, causal):
    if alpha > 2.0:
        return conditioning(arr, alpha, causal, xmin=GRAD_XMIN)
    return conditioning(arr, alpha, causal, xmin=0.0, flip=GRAD_FLIP)


def _check_grads_conditioned(arr, alpha, causal, g, ref, where):
    if alpha < 2.0:
        _check_grads(g, ref, where)
        return
    bad_r, bad_c = _grad_conditioning(arr, alpha, causal)
    print(f"{where}: ill-conditioned rows {bad_r.mean():.3f}, touched key columns {bad_c.mean():.3f}")
    check_close(g[0][~bad_r], ref[0][~bad_r], BF16_MAX_ABS, BF16_MEAN_ABS, where + " dQ (conditioned rows)")
    for name, x, y in zip(("dK", "dV"), g[1:], ref[1:]):
        check_close(x[~bad_c], y[~bad_c], BF16_MAX_ABS, BF16_MEAN_ABS, f"{where} {name} (untouched columns)")


@pytest.mark.parametrize("n", [1, 77, 200])
def test_bwd_ragged_d128(torch_cuda, n):
    arr = inputs.iid(1, 2, n, 128, seed=n + 3, beta=2.0)
    O, tau, mask, dQ, dK, dV = _fwd_bwd(torch_cuda, arr, 1.5, True)
    rdQ, rdK, rdV = oa.backward(arr["Q"], arr["K"], arr["V"], arr["dO"], 1.5, True)
    _check_grads((dQ, dK, dV), (rdQ, rdK, rdV), f"ragged d128 n={n}")


# ---- configuration 3: 2 x 16 x 4096 x 128, causal, alpha 1.5, beta in {2, 8}: every row ----------------

@pytest.mark.parametrize("beta", [2.0, 8.0])
def test_cfg3_full(torch_cuda, beta):
    from _oracle_pool import per_head
    arr = inputs.iid(2, 16, 4096, 128, seed=0, beta=beta)
    O, tau, mask, dQ, dK, dV = _fwd_bwd(torch_cuda, arr, 1.5, True)
    res = per_head("bwd_full", arr, 1.5, True)
    B, H = 2, 16
    rdQ = np.stack([r[0] for r in res]).reshape(dQ.shape)
    rdK = np.stack([r[1] for r in res]).reshape(dK.shape)
    rdV = np.stack([r[2] for r in res]).reshape(dV.shape)
    _check_grads((dQ, dK, dV), (rdQ, rdK, rdV), f"cfg3 beta={beta}")
    rows = np.arange(4096)
    fw = per_head("fwd_rows", arr, 1.5, True, rows=rows)
    check_tau(tau, np.stack([r["tau"] for r in fw]).reshape(tau.shape), "cfg3 tau")
    check_close(O, np.stack([r["O"] for r in fw]).reshape(O.shape), BF16_MAX_ABS, BF16_MEAN_ABS, "cfg3 O")


# ---- dense softmax baseline -----------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("d", [64, 128])
def test_softmax_baseline(torch_cuda, causal, d):
    from adaptive_sparse_flash_b200 import binding as b
    arr = inputs.iid(1, 2, 700, d, seed=31)
    t = to_torch(arr, torch_cuda.bfloat16)
    O, lse = b.softmax_forward(t["Q"], t["K"], t["V"], causal)
    dQ, dK, dV = b.softmax_backward(t["Q"], t["K"], t["V"], O, lse, t["dO"], causal)
    torch_cuda.cuda.synchronize()
    assert b.entmax_attn_check() == 0
    rO, rlse = osm.forward(arr["Q"], arr["K"], arr["V"], causal)
    check_close(O.float().cpu().numpy(), rO, BF16_MAX_ABS, BF16_MEAN_ABS, "softmax O")
    check_close(lse.cpu().numpy(), rlse, 1e-3, None, "softmax lse")
    rdQ, rdK, rdV = osm.backward(arr["Q"], arr["K"], arr["V"], arr["dO"], causal)
    # the baseline keeps standard flash-attention numerics (bf16 P and dS): a looser bound
    for name, x, y in zip(("dQ", "dK", "dV"), (dQ, dK, dV), (rdQ, rdK, rdV)):
        check_close(x.cpu().numpy(), y, 5e-2, 5e-3, f"softmax {name}")


# ---- configuration 4: 1 x 16 x 16384 x 64 (the bench workload): sampled rows and key columns ------------

def test_cfg4_sampled(torch_cuda):
    from _oracle_pool import per_head
    arr = inputs.clustered(1, 16, 16384, 64, centres=256, beta_q=6.0, seed=0)
    O, tau, mask, dQ, dK, dV = _fwd_bwd(torch_cuda, arr, 1.5, True)
    rows = inputs.sample_rows(16384, 512, seed=0)
    cols = inputs.sample_rows(16384, 512, seed=1)
    fw = per_head("fwd_rows", arr, 1.5, True, rows=rows)
    check_tau(tau[:, :, rows], np.stack([r["tau"] for r in fw]).reshape(1, 16, -1), "cfg4 tau")
    check_close(O[:, :, rows], np.stack([r["O"] for r in fw]).reshape(1, 16, len(rows), 64),
                BF16_MAX_ABS, BF16_MEAN_ABS, "cfg4 O")
    from _parity import unpack_mask
    nkb = 256
    g_bits = unpack_mask(mask, nkb)[:, :, rows // 64]          # the 64-row mask block of each sampled row
    r_bits = np.stack([r["row_bits"] for r in fw]).reshape(1, 16, len(rows), nkb)
    r_bmax = np.stack([r["row_bmax"] for r in fw]).reshape(1, 16, len(rows), nkb)
    # a sampled row's nonzero blocks must be set in its block row (the block row may have more)
    missing = r_bits & ~g_bits & (r_bmax >= 1e-3)
    assert not missing.any(), f"cfg4 mask: {int(missing.sum())} nonzero blocks of sampled rows not set"
    bw = per_head("bwd_full", arr, 1.5, True, cols=cols)
    rdQ = np.stack([r[0] for r in bw]).reshape(dQ.shape)
    rdK = np.stack([r[1] for r in bw]).reshape(1, 16, len(cols), 64)
    rdV = np.stack([r[2] for r in bw]).reshape(1, 16, len(cols), 64)
    _check_grads((dQ[:, :, rows], dK[:, :, cols], dV[:, :, cols]), (rdQ[:, :, rows], rdK, rdV), "cfg4")


# ---- configuration 5: 8 x 12 x 2048 x 64 alpha sweep, every solver branch ------------------------------

@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0, 3.0])
@pytest.mark.parametrize("beta", [1.0, 4.0])
def test_cfg5_alpha_sweep(torch_cuda, alpha, beta):
    from adaptive_sparse_flash_b200 import binding as b
    from _oracle_pool import per_head
    arr = inputs.clustered(8, 12, 2048, 64, centres=64, beta_q=beta, seed=0)
    t = to_torch(arr, torch_cuda.bfloat16)
    f = b.forward(t["Q"], t["K"], t["V"], alpha, True, with_stats=True)
    dQ, dK, dV = b.backward(t["Q"], t["K"], t["V"], f, t["dO"])
    torch_cuda.cuda.synchronize()
    assert b.entmax_attn_check() == 0
    st = b.stats_dict(f.stats)
    print(f"cfg5 alpha={alpha} beta={beta}: mean steps {st['steps'] / st['rows']:.3f}, "
          f"fallback rate {st['fallbacks'] / max(1, st['steps']):.4f}, hist {[st[f'step_hist_{i}'] for i in range(9)]}")
    cols = inputs.sample_rows(2048, 256, seed=2)
    bw = per_head("bwd_full", arr, alpha, True, cols=cols)
    rows = np.arange(2048)
    fw = per_head("fwd_rows", arr, alpha, True, rows=rows)
    O, tau = f.O.float().cpu().numpy(), f.tau.cpu().numpy()
    check_tau(tau, np.stack([r["tau"] for r in fw]).reshape(tau.shape), "cfg5 tau")
    rO = np.stack([r["O"] for r in fw]).reshape(O.shape)
    if alpha > 2.0:
        bad_o, _ = conditioning(arr, alpha, True, xmin=FWD_XMIN)
        print(f"cfg5 a={alpha} b={beta}: O rows with a support entry below {FWD_XMIN}: {bad_o.mean():.4f}")
        check_close(O[~bad_o], rO[~bad_o], BF16_MAX_ABS, BF16_MEAN_ABS, "cfg5 O (conditioned rows)")
    else:
        check_close(O, rO, BF16_MAX_ABS, BF16_MEAN_ABS, "cfg5 O")
    rdQ = np.stack([r[0] for r in bw]).reshape(dQ.shape)
    rdK = np.stack([r[1] for r in bw]).reshape(8, 12, len(cols), 64)
    rdV = np.stack([r[2] for r in bw]).reshape(8, 12, len(cols), 64)
    g = (dQ.cpu().numpy(), dK.cpu().numpy()[:, :, cols], dV.cpu().numpy()[:, :, cols])
    if alpha < 2.0:
        _check_grads(g, (rdQ, rdK, rdV), f"cfg5 a={alpha} b={beta}")
    else:
        bad_r, bad_c = _grad_conditioning(arr, alpha, True)
        bad_c = bad_c[:, :, cols]
        print(f"cfg5 a={alpha} b={beta}: ill-conditioned rows {bad_r.mean():.3f}, columns {bad_c.mean():.3f}")
        check_close(g[0][~bad_r], rdQ[~bad_r], BF16_MAX_ABS, BF16_MEAN_ABS, "cfg5 dQ (conditioned rows)")
        check_close(g[1][~bad_c], rdK[~bad_c], BF16_MAX_ABS, BF16_MEAN_ABS, "cfg5 dK (untouched columns)")
        check_close(g[2][~bad_c], rdV[~bad_c], BF16_MAX_ABS, BF16_MEAN_ABS, "cfg5 dV (untouched columns)")
