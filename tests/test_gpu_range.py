"""GPU: inputs beyond the fp16 range (the fp16 operand path, d = 64, alpha <= 2).

Q, V and dO multiplied by 2^16 and the score scale by 2^-16 leave every score unchanged, so tau and the block
mask must match the unscaled run, O, dQ and dV must scale by 2^16 and dK by 2^32 (power-of-two factors are
exact in floating point). Q, V and dO then exceed the fp16 range, and dP exceeds it many times over, so
this drives every range exponent of the fp16 copies and the scaled storage of dS.
"""
import numpy as np
import pytest

from adaptive_sparse_flash_b200 import inputs

from _parity import to_torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from adaptive_sparse_flash_b200 import build
    build.build()
    return torch


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_power_of_two_scaled_inputs(torch_cuda, alpha):
    from adaptive_sparse_flash_b200 import binding as b
    torch = torch_cuda
    arr = inputs.clustered(1, 4, 1024, 64, centres=16, beta_q=4.0, seed=7)
    t = to_torch(arr, torch.bfloat16)
    f0 = b.forward(t["Q"], t["K"], t["V"], alpha, True)
    dQ0, dK0, dV0 = b.backward(t["Q"], t["K"], t["V"], f0, t["dO"])
    s16 = 2.0 ** 16
    Qs, Vs, dOs = t["Q"] * s16, t["V"] * s16, t["dO"] * s16  # exact in bf16
    assert float(Qs.abs().max()) >= 2.0 ** 15 and float(Vs.abs().max()) >= 2.0 ** 15
    f1 = b.forward(Qs, t["K"], Vs, alpha, True, scale=b.default_scale(64) / s16)
    dQ1, dK1, dV1 = b.backward(Qs, t["K"], Vs, f1, dOs)
    torch.cuda.synchronize()
    assert b.entmax_attn_check() == 0

    tau0, tau1 = f0.tau.cpu().numpy(), f1.tau.cpu().numpy()
    assert np.abs(tau1 - tau0).max() <= 1e-5 * max(1.0, np.abs(tau0).max())
    assert np.array_equal(f0.mask.cpu().numpy(), f1.mask.cpu().numpy())

    def close(x1, x0, factor, rel, what):
        x1 = x1.double().cpu().numpy() / factor
        x0 = x0.double().cpu().numpy()
        err = np.abs(x1 - x0).max()
        assert np.all(np.isfinite(x1)), what
        assert err <= rel * max(1.0, np.abs(x0).max()), f"{what}: {err:.3e}"

    close(f1.O, f0.O, s16, 1e-2, "O")       # bf16 output: one rounding either way
    close(dV1, dV0, s16, 1e-4, "dV")
    close(dQ1, dQ0, s16, 1e-4, "dQ")
    close(dK1, dK0, s16 * s16, 1e-4, "dK")


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_keys_beyond_unit_scale(torch_cuda, alpha):
    """K multiplied by 16 and the score scale divided by 16 leave every score unchanged. With |k| >= 8 the dQ
    kernel leaves its two-accumulator form (one fp16 term of u g and of u, for unit-scale keys) for a delta
    pass followed by dS = u (g - delta) in two fp16 terms: both routes must give the same gradients within the
    parity bound (dQ and dV unchanged, dK divided by 16), tau and mask unchanged."""
    from adaptive_sparse_flash_b200 import binding as b
    torch = torch_cuda
    arr = inputs.clustered(2, 3, 777, 64, centres=16, beta_q=4.0, seed=9)
    t = to_torch(arr, torch.bfloat16)
    f0 = b.forward(t["Q"], t["K"], t["V"], alpha, True)
    g0 = b.backward(t["Q"], t["K"], t["V"], f0, t["dO"])
    Ks = t["K"] * 16.0
    assert float(Ks.abs().max()) >= 8.0 and float(t["K"].abs().max()) < 8.0
    f1 = b.forward(t["Q"], Ks, t["V"], alpha, True, scale=b.default_scale(64) / 16.0)
    g1 = b.backward(t["Q"], Ks, t["V"], f1, t["dO"])
    torch.cuda.synchronize()
    assert b.entmax_attn_check() == 0
    tau0, tau1 = f0.tau.cpu().numpy(), f1.tau.cpu().numpy()
    assert np.abs(tau1 - tau0).max() <= 1e-5 * max(1.0, np.abs(tau0).max())
    assert np.array_equal(f0.mask.cpu().numpy(), f1.mask.cpu().numpy())
    for name, x1, x0, factor in (("dQ", g1[0], g0[0], 1.0), ("dK", g1[1], g0[1], 1.0 / 16.0),
                                 ("dV", g1[2], g0[2], 1.0)):
        a1 = x1.double().cpu().numpy() / factor
        a0 = x0.double().cpu().numpy()
        err = np.abs(a1 - a0).max()
        assert np.all(np.isfinite(a1)), name
        # the two routes round differently (one fp16 term of u g and u, against two of dS): both within the
        # parity bound of the oracle, so within it of each other
        assert err <= 2e-2, f"{name}: {err:.3e}"
