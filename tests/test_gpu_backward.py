"""GPU backward parity (dQ, dK, dV) against the float64 oracle, and the dense softmax baseline."""
import numpy as np
import pytest

from adaptive_sparse_flash_b200 import inputs
from oracle import attention as oa
from oracle import softmax as osm

from _parity import BF16_MAX_ABS, BF16_MEAN_ABS, check_close, check_mask, check_tau, to_torch

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
    _check_grads((dQ, dK, dV), (rdQ, rdK, rdV), f"bwd small a={alpha} causal={causal}")


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
