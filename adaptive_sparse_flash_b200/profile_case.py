"""Run alpha-entmax attention forward + backward on a synthetic case a few times (for profilers).

    python -m adaptive_sparse_flash_b200.profile_case [--B 2] [--H 16] [--n 16384] [--d 64] [--alpha 1.5]
                                                      [--centres 256] [--beta 6] [--reps 2]

Keys cluster on `centres` random centres, queries are `beta` times their centre plus noise (the long-context
workload of the benchmark); V and dO are N(0, 1). The device status is checked at the end.
"""
from __future__ import annotations

import argparse
import os
import sys


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--B", type=int, default=2)
    ap.add_argument("--H", type=int, default=16)
    ap.add_argument("--n", type=int, default=16384)
    ap.add_argument("--d", type=int, default=64)
    ap.add_argument("--alpha", type=float, default=1.5)
    ap.add_argument("--centres", type=int, default=256)
    ap.add_argument("--beta", type=float, default=6.0)
    ap.add_argument("--reps", type=int, default=2)
    ap.add_argument("--seed", type=int, default=0)
    args = ap.parse_args(argv)

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import numpy as np
    import torch

    from adaptive_sparse_flash_b200 import binding as b
    from adaptive_sparse_flash_b200 import inputs

    arr = inputs.clustered(args.B, args.H, args.n, args.d, centres=args.centres, beta_q=args.beta, seed=args.seed)
    dev = torch.device("cuda", 0)
    t = {k: torch.from_numpy(inputs.bf16_bits(v).view(np.int16)).view(torch.bfloat16).to(dev) for k, v in arr.items()}
    for _ in range(args.reps):
        f = b.forward(t["Q"], t["K"], t["V"], args.alpha, True)
        b.backward(t["Q"], t["K"], t["V"], f, t["dO"])
    torch.cuda.synchronize(dev)
    st = b.entmax_attn_check(None)
    print("status", b.entmax_status_str(st))
    return 0 if st == 0 else 1


if __name__ == "__main__":
    raise SystemExit(main())
