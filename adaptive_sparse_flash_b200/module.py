"""PyTorch front end over the C ABI: an autograd function and a multi-head attention module.

The AdaSplash-2 pages present the method as a drop-in replacement for standard multi-head attention: the
same interface as torch.nn.MultiheadAttention, where only the normaliser changes from softmax to alpha-entmax
(euno.news summary, practical implications, "即插即用"; limitations section, multi-query attention as future
work). This module keeps that interface and runs the attention core through entmax_attn_fwd /
entmax_attn_bwd: the projections are ordinary torch layers, every step of the attention itself runs in the
library's kernels. Grouped-query attention maps each query head to its key / value head by index; the
key / value heads are expanded before the call and their gradients summed over each group after it.
"""
from __future__ import annotations

import math

import torch
from torch import nn

from . import binding as _b

__all__ = ["EntmaxAttnFunction", "entmax_attention", "EntmaxMultiheadAttention"]


class EntmaxAttnFunction(torch.autograd.Function):
    """O = alpha-entmax(scale Q K^T) V for bf16 [B, H, n, d] tensors on a CUDA device (d in {64, 128}).

    Besides q, k, v and O, the forward keeps tau, the block mask and the saved part of the library's
    workspace for the backward: sum u and the transposed mask (plus U V in fp32 where the bf16 kernels serve
    the call, d = 128 or alpha > 2); the fp16 operand copies live in a per-call scratch buffer, so they are
    not activation memory. Gradients come back in the inputs' dtype (the library computes them in fp32).
    """

    @staticmethod
    def forward(ctx, q, k, v, alpha: float, causal: bool, scale: float, hist_bins: int):
        for t in (q, k, v):
            if not t.is_cuda or t.dtype != torch.bfloat16:
                raise TypeError("entmax attention takes bf16 CUDA tensors")
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        f = _b.forward(q, k, v, alpha, causal, scale=scale, hist_bins=hist_bins, separate_scratch=True)
        ctx.save_for_backward(q, k, v, f.O, f.tau, f.mask, f.workspace)
        ctx.alpha, ctx.causal, ctx.scale, ctx.hist_bins = alpha, causal, scale, hist_bins
        return f.O

    @staticmethod
    def backward(ctx, dO):
        q, k, v, O, tau, mask, ws = ctx.saved_tensors
        dO = dO.to(torch.bfloat16).contiguous()
        Bsz, H, n, d = q.shape
        probe = _b.make_opts(scale=ctx.scale, hist_bins=ctx.hist_bins)
        scratch = _b.alloc_workspace(Bsz, H, n, d, _b.ENTMAX_BF16, q.device, probe, part="scratch")
        opts = _b.make_opts(ws, scale=ctx.scale, hist_bins=ctx.hist_bins, scratch=scratch)
        dQ, dK, dV = (torch.empty(x.shape, dtype=torch.float32, device=x.device) for x in (q, k, v))
        _b.entmax_attn_bwd(q, k, v, O, dO, tau, mask, dQ, dK, dV, ctx.alpha, ctx.causal, opts)
        return dQ.to(q.dtype), dK.to(k.dtype), dV.to(v.dtype), None, None, None, None


def entmax_attention(q, k, v, alpha: float = 1.5, causal: bool = False, scale: float | None = None,
                     hist_bins: int = 0):
    """Differentiable alpha-entmax attention on [B, H, n, d] bf16 CUDA tensors (scale defaults to 1/sqrt(d))."""
    s = 0.0 if scale is None else float(scale)
    return EntmaxAttnFunction.apply(q, k, v, float(alpha), bool(causal), s, int(hist_bins))


class EntmaxMultiheadAttention(nn.Module):
    """Multi-head attention with the alpha-entmax normaliser, in the shape of torch.nn.MultiheadAttention.

    forward(query, key, value, key_padding_mask=None, need_weights=False, attn_mask=None, is_causal=False)
    returns (output, None) like nn.MultiheadAttention with need_weights=False. Inputs are [B, n, E] with
    batch_first=True (the default here), else [n, B, E]. Query and key sequences must have the same length
    (the library's attention is square); masking is causal or none. `num_kv_heads` < num_heads gives
    grouped-query attention (1: multi-query). The head size E / num_heads must be 64 or 128.
    Parameters keep their own dtype; the attention core runs on bf16 copies of the projected heads.
    """

    def __init__(self, embed_dim: int, num_heads: int, alpha: float = 1.5, bias: bool = True,
                 batch_first: bool = True, num_kv_heads: int | None = None, hist_bins: int = 0,
                 device=None, dtype=None):
        super().__init__()
        if embed_dim % num_heads:
            raise ValueError("embed_dim must be divisible by num_heads")
        self.embed_dim, self.num_heads = embed_dim, num_heads
        self.head_dim = embed_dim // num_heads
        if self.head_dim not in (64, 128):
            raise ValueError(f"head size {self.head_dim} is not supported (64 or 128)")
        self.num_kv_heads = num_kv_heads or num_heads
        if num_heads % self.num_kv_heads:
            raise ValueError("num_heads must be a multiple of num_kv_heads")
        if not alpha > 1.0:
            raise ValueError("alpha must be > 1 (alpha -> 1 is softmax)")
        self.alpha, self.batch_first, self.hist_bins = float(alpha), batch_first, hist_bins
        kv_dim = self.num_kv_heads * self.head_dim
        fk = {"device": device, "dtype": dtype}
        self.q_proj = nn.Linear(embed_dim, embed_dim, bias=bias, **fk)
        self.k_proj = nn.Linear(embed_dim, kv_dim, bias=bias, **fk)
        self.v_proj = nn.Linear(embed_dim, kv_dim, bias=bias, **fk)
        self.out_proj = nn.Linear(embed_dim, embed_dim, bias=bias, **fk)
        self.reset_parameters()

    def reset_parameters(self):
        for lin in (self.q_proj, self.k_proj, self.v_proj):
            nn.init.xavier_uniform_(lin.weight, gain=1.0 / math.sqrt(2.0))
            if lin.bias is not None:
                nn.init.zeros_(lin.bias)
        nn.init.xavier_uniform_(self.out_proj.weight)
        if self.out_proj.bias is not None:
            nn.init.zeros_(self.out_proj.bias)

    def _heads(self, x, nh):
        Bsz, n, _ = x.shape
        return x.view(Bsz, n, nh, self.head_dim).transpose(1, 2).to(torch.bfloat16).contiguous()

    def forward(self, query, key, value, key_padding_mask=None, need_weights=False, attn_mask=None,
                is_causal=False):
        if key_padding_mask is not None:
            raise ValueError("key_padding_mask is not supported: pass equal-length sequences")
        if need_weights:
            raise ValueError("need_weights=True is not supported: the attention matrix is never formed")
        if attn_mask is not None and not is_causal:
            raise ValueError("attn_mask is not supported; use is_causal=True for a causal mask")
        if not self.batch_first:
            query, key, value = (x.transpose(0, 1) for x in (query, key, value))
        if query.shape[1] != key.shape[1] or key.shape[1] != value.shape[1]:
            raise ValueError("query, key and value must have the same sequence length")
        q = self._heads(self.q_proj(query), self.num_heads)
        k = self._heads(self.k_proj(key), self.num_kv_heads)
        v = self._heads(self.v_proj(value), self.num_kv_heads)
        g = self.num_heads // self.num_kv_heads
        if g > 1:  # grouped-query attention: query head h reads key / value head h // g
            k = k.repeat_interleave(g, dim=1)
            v = v.repeat_interleave(g, dim=1)
        o = entmax_attention(q, k, v, self.alpha, bool(is_causal), None, self.hist_bins)
        Bsz, _, n, _ = o.shape
        o = o.transpose(1, 2).reshape(Bsz, n, self.embed_dim).to(self.out_proj.weight.dtype)
        out = self.out_proj(o)
        if not self.batch_first:
            out = out.transpose(0, 1)
        return out, None
