"""Run the float64 oracle over (b, h) heads in a process pool (spawned, never forked after CUDA init)."""
import multiprocessing as mp
import os

import numpy as np

_POOL = None


def pool():
    global _POOL
    if _POOL is None:
        n = max(1, min(32, (os.cpu_count() or 2) - 1))
        _POOL = mp.get_context("spawn").Pool(n)
    return _POOL


def _head_job(args):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    from oracle import attention as oa
    kind, q, k, v, do, alpha, causal, rows, cols = args
    Q, K, V = q[None, None], k[None, None], v[None, None]
    if kind == "fwd_rows":
        out = oa.forward(Q, K, V, alpha, causal, rows=rows)
        return dict(O=out["O"][0, 0], tau=out["tau"][0, 0], row_bits=out["row_bits"][0, 0],
                    row_bmax=out["row_bmax"][0, 0])
    if kind == "bwd_rows":
        return oa.row_gradients(Q, K, V, do[None, None], alpha, causal, rows)[0, 0]
    if kind == "bwd_full":
        dQ, dK, dV = oa.backward(Q, K, V, do[None, None], alpha, causal, key_cols=cols)
        return dQ[0, 0], dK[0, 0], dV[0, 0]
    if kind == "sens":
        tests = os.path.dirname(os.path.abspath(__file__))
        if tests not in sys.path:
            sys.path.insert(0, tests)
        from _parity import grad_sensitivity
        return grad_sensitivity(q, k, v, do, alpha, causal)
    raise ValueError(kind)


def per_head(kind, arr, alpha, causal, rows=None, cols=None):
    """List over heads (b-major) of the oracle job's result."""
    B, H = arr["Q"].shape[:2]
    jobs = []
    for b in range(B):
        for h in range(H):
            do = arr["dO"][b, h] if "dO" in arr else None
            jobs.append((kind, arr["Q"][b, h], arr["K"][b, h], arr["V"][b, h], do, alpha, causal, rows, cols))
    return pool().map(_head_job, jobs)
