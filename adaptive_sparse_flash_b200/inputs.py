"""Seeded synthetic workloads for alpha-entmax attention.

This module only draws random numbers and rounds them to the storage type.
It holds none of the attention arithmetic. Both the float64 oracle tests and
the CUDA path take their inputs from here, so that they see the same values.

Workloads follow the shapes of the AdaSplash-2 pages: long-context attention
up to 16k tokens, with sparsity swept from near-dense to highly sparse
("AdaSplash-2: Faster Differentiable Sparse Attention", results section).

Random draws use numpy's PCG64 (`default_rng(seed)`) in float32. Draw order:
  * i.i.d. workloads: Q, K, V, dO;
  * clustered workloads: centres, assignments, key noise, query noise, V, dO.
Tensors are [B, H, n, d], d fastest.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "round_to_bf16",
    "bf16_bits",
    "iid",
    "clustered",
    "sample_rows",
    "sample_blocks",
]


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even).

    Returns float32 values that are exactly representable in bfloat16.
    Inputs must be finite.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + lsb) >> 16) << 16
    return rounded.astype(np.uint32).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The bfloat16 bit patterns (uint16) of bf16-representable float32 values."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32)
    if np.any(bits & 0xFFFF):
        raise ValueError("values are not bf16-representable; call round_to_bf16 first")
    return (bits >> 16).astype(np.uint16)


def _finish(arrs: dict, dtype: str) -> dict:
    if dtype == "bf16":
        return {k: round_to_bf16(v) for k, v in arrs.items()}
    if dtype == "fp32":
        return {k: np.ascontiguousarray(v, dtype=np.float32) for k, v in arrs.items()}
    raise ValueError(f"unknown dtype {dtype!r}")


def iid(B: int, H: int, n: int, d: int, *, seed: int = 0, beta: float = 1.0,
        dtype: str = "bf16", with_dO: bool = True) -> dict:
    """Q, K, V (and dO) drawn i.i.d. N(0, 1); Q multiplied by `beta`.

    A larger `beta` sharpens the scores and so raises the sparsity of the
    entmax probabilities.
    """
    rng = np.random.default_rng(seed)
    shape = (B, H, n, d)
    out = {}
    out["Q"] = rng.standard_normal(shape, dtype=np.float32) * np.float32(beta)
    out["K"] = rng.standard_normal(shape, dtype=np.float32)
    out["V"] = rng.standard_normal(shape, dtype=np.float32)
    if with_dO:
        out["dO"] = rng.standard_normal(shape, dtype=np.float32)
    return _finish(out, dtype)


def clustered(B: int, H: int, n: int, d: int, *, centres: int, beta_q: float,
              seed: int = 0, noise: float = 0.3, run: int = 0,
              dtype: str = "bf16", with_dO: bool = True) -> dict:
    """Keys and queries grouped around random cluster centres.

    Each position i of each (b, h) is assigned a centre a_i uniformly from
    `centres` centres c ~ N(0, I). The key is c_{a_i} + noise * N(0, I); the
    query is beta_q * c_{a_i} + N(0, I). V and dO are N(0, 1).

    With `run` > 0, positions come in contiguous runs of `run` tokens that
    share one assignment (a_i = a_run[i // run]). That places the support of
    each row in a few contiguous key ranges, so whole key blocks become zero;
    fewer centres give denser attention.
    """
    rng = np.random.default_rng(seed)
    c = rng.standard_normal((B, H, centres, d), dtype=np.float32)
    if run > 0:
        nruns = (n + run - 1) // run
        a_run = rng.integers(0, centres, size=(B, H, nruns))
        a = np.repeat(a_run, run, axis=2)[:, :, :n]
    else:
        a = rng.integers(0, centres, size=(B, H, n))
    key_noise = rng.standard_normal((B, H, n, d), dtype=np.float32)
    query_noise = rng.standard_normal((B, H, n, d), dtype=np.float32)
    bidx = np.arange(B)[:, None, None]
    hidx = np.arange(H)[None, :, None]
    cent = c[bidx, hidx, a]  # [B, H, n, d]
    out = {}
    out["Q"] = np.float32(beta_q) * cent + query_noise
    out["K"] = cent + np.float32(noise) * key_noise
    out["V"] = rng.standard_normal((B, H, n, d), dtype=np.float32)
    if with_dO:
        out["dO"] = rng.standard_normal((B, H, n, d), dtype=np.float32)
    return _finish(out, dtype)


def sample_rows(n: int, count: int, *, seed: int = 0) -> np.ndarray:
    """Sorted distinct row (or key-column) indices, drawn from default_rng(seed + 1).

    Always includes row 0 and row n - 1 (the first causal row and the ragged
    tail), so the sampled checks cover both ends of the sequence.
    """
    rng = np.random.default_rng(seed + 1)
    count = min(count, n)
    picks = rng.choice(n, size=count, replace=False)
    picks = np.unique(np.concatenate([picks, [0, n - 1]]))
    return picks.astype(np.int64)


def sample_blocks(n: int, block: int, count: int, *, seed: int = 0) -> np.ndarray:
    """Every row of `count` distinct whole query blocks of `block` rows, drawn from default_rng(seed + 1).

    Always includes the first and the last block (the first causal rows and the ragged tail). Sampling whole
    blocks lets a test check the block mask rows of the sample exactly, in both directions.
    """
    rng = np.random.default_rng(seed + 1)
    nb = (n + block - 1) // block
    count = min(count, nb)
    picks = rng.choice(nb, size=count, replace=False)
    picks = np.unique(np.concatenate([picks, [0, nb - 1]]))
    if len(picks) > count:  # keep the two ends, drop interior picks beyond the count
        inner = picks[(picks != 0) & (picks != nb - 1)][: max(0, count - 2)]
        picks = np.unique(np.concatenate([inner, [0, nb - 1]]))
    rows = (picks[:, None] * block + np.arange(block)[None, :]).ravel()
    return rows[rows < n].astype(np.int64)
