"""The autograd function and the multi-head attention module (adaptive_sparse_flash_b200.module) on the GPU,
against the float64 oracle: gradients through torch.autograd, an nn.MultiheadAttention-shaped module with
and without grouped key / value heads, and a few training steps."""
import numpy as np
import pytest

from adaptive_sparse_flash_b200 import inputs
from oracle import attention as oa

from _parity import BF16_MAX_ABS, BF16_MEAN_ABS, check_close, to_torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from adaptive_sparse_flash_b200 import build
    build.build()
    return torch


@pytest.mark.parametrize("alpha,causal", [(1.5, True), (2.0, False), (1.25, True)])
def test_function_gradients_match_oracle(torch_cuda, alpha, causal):
    torch = torch_cuda
    from adaptive_sparse_flash_b200.module import entmax_attention
    arr = inputs.clustered(2, 2, 300, 64, centres=16, beta_q=3.0, seed=51)
    t = to_torch(arr, torch.bfloat16)
    q, k, v = (t[x].clone().requires_grad_(True) for x in "QKV")
    o = entmax_attention(q, k, v, alpha, causal=causal)
    o.backward(t["dO"])
    torch.cuda.synchronize()
    ref = oa.forward(arr["Q"], arr["K"], arr["V"], alpha, causal)
    rdQ, rdK, rdV = oa.backward(arr["Q"], arr["K"], arr["V"], arr["dO"], alpha, causal)
    check_close(o.detach().float().cpu().numpy(), ref["O"], BF16_MAX_ABS, BF16_MEAN_ABS, "function O")
    # autograd hands back gradients in the bf16 dtype of q, k, v: on top of the kernel tolerance, each
    # value carries its bf16 rounding (at most 2^-9 of its magnitude)
    for name, x, r in (("dQ", q, rdQ), ("dK", k, rdK), ("dV", v, rdV)):
        g = x.grad.float().cpu().numpy()
        err = np.abs(g - r)
        assert np.all(err <= BF16_MAX_ABS + 2.0 ** -8 * np.abs(r)), f"{name}: {err.max():.3e}"
        assert err.mean() <= BF16_MEAN_ABS + 2.0 ** -9 * np.abs(r).mean(), name


class _OracleAttn:
    """float64 CPU attention core from the oracle, as a torch.autograd.Function (reference only)."""

    @staticmethod
    def make(torch, alpha, causal):
        class F(torch.autograd.Function):
            @staticmethod
            def forward(ctx, q, k, v):
                ctx.save_for_backward(q, k, v)
                out = oa.forward(q.numpy(), k.numpy(), v.numpy(), alpha, causal)
                return torch.from_numpy(out["O"])

            @staticmethod
            def backward(ctx, dO):
                q, k, v = ctx.saved_tensors
                g = oa.backward(q.numpy(), k.numpy(), v.numpy(), dO.numpy(), alpha, causal)
                return tuple(torch.from_numpy(x) for x in g)
        return F


def _reference_mha(torch, m, x, alpha, causal):
    """The module's computation in float64 on the CPU with the oracle as the attention core. The projected
    heads are rounded to bf16 as the module rounds them before the library call."""
    F = _OracleAttn.make(torch, alpha, causal)
    p = {n: w.detach().double().cpu().requires_grad_(True) for n, w in m.named_parameters()}
    xd = x.detach().double().cpu().requires_grad_(True)
    Bsz, n, E = xd.shape
    hd, nh, nkv = m.head_dim, m.num_heads, m.num_kv_heads

    def proj(name, nheads):
        y = xd @ p[name + ".weight"].T + p[name + ".bias"]
        y = y.view(Bsz, n, nheads, hd).transpose(1, 2)
        return y + (y.to(torch.bfloat16).double() - y).detach()  # bf16 values, identity gradient

    q, k, v = proj("q_proj", nh), proj("k_proj", nkv), proj("v_proj", nkv)
    if nh > nkv:
        k = k.repeat_interleave(nh // nkv, dim=1)
        v = v.repeat_interleave(nh // nkv, dim=1)
    o = F.apply(q.contiguous(), k.contiguous(), v.contiguous())
    o = o.transpose(1, 2).reshape(Bsz, n, E)
    out = o @ p["out_proj.weight"].T + p["out_proj.bias"]
    return out, xd, p


@pytest.mark.parametrize("num_kv_heads", [None, 1])
def test_module_matches_float64_reference(torch_cuda, num_kv_heads):
    torch = torch_cuda
    from adaptive_sparse_flash_b200.module import EntmaxMultiheadAttention
    torch.manual_seed(0)
    E, nh, n, Bsz, alpha = 128, 2, 192, 2, 1.5
    m = EntmaxMultiheadAttention(E, nh, alpha=alpha, num_kv_heads=num_kv_heads, device="cuda",
                                 dtype=torch.float32)
    x = (2.0 * torch.randn(Bsz, n, E, device="cuda")).requires_grad_(True)
    out, w = m(x, x, x, is_causal=True)
    assert w is None
    g = torch.randn_like(out)
    out.backward(g)
    torch.cuda.synchronize()
    ref, xd, p = _reference_mha(torch, m, x, alpha, True)
    ref.backward(g.double().cpu())
    # the module rounds the attention output and its incoming gradient to bf16 (2^-9 relative each); the
    # comparison is relative to the scale of each tensor, or for a bias to that of its layer's weight
    # gradient: the key bias has an exactly zero gradient (a shift of every score of a row by q . b leaves
    # entmax unchanged), so its computed value is pure rounding of sums of terms of the weight's scale
    def close(a, r, name, scale=None, rel=2e-2):
        a, r = a.detach().double().cpu(), r.detach()
        scale = float(r.abs().max()) if scale is None else scale
        err = float((a - r).abs().max())
        assert err <= rel * max(scale, 1e-3), f"{name}: max err {err:.3e} at scale {scale:.3e}"
    close(out, ref, "output")
    close(x.grad, xd.grad, "d input")
    for name, prm in m.named_parameters():
        layer = name.rsplit(".", 1)[0]
        wscale = float(p[layer + ".weight"].grad.abs().max())
        close(prm.grad, p[name].grad, "d " + name, scale=wscale if name.endswith("bias") else None)


def test_module_training_steps(torch_cuda):
    torch = torch_cuda
    from adaptive_sparse_flash_b200.module import EntmaxMultiheadAttention
    torch.manual_seed(1)
    m = EntmaxMultiheadAttention(128, 2, alpha=1.5, device="cuda", dtype=torch.float32)
    x = torch.randn(2, 256, 128, device="cuda")
    target = torch.randn(2, 256, 128, device="cuda")
    opt = torch.optim.SGD(m.parameters(), lr=0.5)
    losses = []
    for _ in range(5):
        opt.zero_grad()
        out, _ = m(x, x, x, is_causal=True)
        loss = torch.nn.functional.mse_loss(out, target)
        loss.backward()
        opt.step()
        losses.append(float(loss))
    assert all(np.isfinite(losses))
    assert losses[-1] < losses[0], losses
