"""Measurement reports of the library on the GPU, printed as markdown tables.

    python -m adaptive_sparse_flash_b200.report solver   # solver iterations per configuration, and the
                                                         # plain-bracket start (no histogram) beside it
    python -m adaptive_sparse_flash_b200.report bins     # histogram size B: iterations, shared memory, time
    python -m adaptive_sparse_flash_b200.report memory   # bytes kept from forward to backward, entmax and
                                                         # the in-library dense softmax baseline
    python -m adaptive_sparse_flash_b200.report timing   # per configuration: forward / backward ms, effective
                                                         # TFLOP/s, the dense baseline on the same inputs

The solver report covers the pages' iteration claims: one or two solver steps after the histogram start,
against five to ten without it (euno.news summary, "方法论" item 3; gist.science (de), section 2,
"Schnelle Konvergenz"), and the hybrid solver's branches per alpha ("Hybrid Solver"). The histogram report
covers the bin-count trade-off (euno.news, limitations, "直方图粒度权衡"), the memory report the activation
memory claim (euno.news, results, "内存占用"). Every number comes from the library's own kernels (device
counters of entmax_stats, CUDA-event times, torch's allocator statistics).
"""
from __future__ import annotations

import argparse
import sys

# (name, generator kind, B, H, n, d, alphas, parameter sets, causal)
CONFIGS = (
    ("cfg2", "iid", 4, 8, 1024, 64, (1.5, 2.0), [{"beta": 1.0}, {"beta": 4.0}, {"beta": 16.0}]),
    ("cfg3", "iid", 2, 16, 4096, 128, (1.5,), [{"beta": 2.0}, {"beta": 8.0}]),
    ("cfg4", "clustered", 1, 16, 16384, 64, (1.5,), [{"centres": 256, "beta_q": 6.0}]),
    ("cfg5", "clustered", 8, 12, 2048, 64, (1.25, 1.5, 2.0, 3.0),
     [{"centres": 64, "beta_q": 1.0}, {"centres": 64, "beta_q": 4.0}]),
)


def _gen(kind, B, H, n, d, params, seed=0):
    from . import inputs
    if kind == "iid":
        return inputs.iid(B, H, n, d, seed=seed, beta=params["beta"])
    return inputs.clustered(B, H, n, d, centres=params["centres"], beta_q=params["beta_q"], seed=seed)


def _to_dev(arr):
    import numpy as np
    import torch
    return {k: torch.from_numpy(np.ascontiguousarray(v)).to("cuda", torch.bfloat16) for k, v in arr.items()}


def _median_ms(fn, reps=5):
    import torch
    fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return sorted(ts)[len(ts) // 2]


def _forward_stats(t, alpha, init_mode=0, hist_bins=0):
    """One forward with device counters; returns (stats dict, forward ms)."""
    import torch

    from . import binding as b
    Q, K, V = t["Q"], t["K"], t["V"]
    Bsz, H, n, d = Q.shape
    probe = b.make_opts(hist_bins=hist_bins, init_mode=init_mode)
    ws = b.alloc_workspace(Bsz, H, n, d, opts=probe)
    O = torch.empty_like(Q)
    tau = torch.empty((Bsz, H, n), dtype=torch.float32, device="cuda")
    mask = torch.empty(b.mask_shape(Bsz, H, n), dtype=torch.int32, device="cuda")
    stats = torch.zeros(b.STATS_WORDS, dtype=torch.int64, device="cuda")
    so = b.make_opts(ws, hist_bins=hist_bins, init_mode=init_mode, stats=stats)
    b.entmax_attn_fwd(Q, K, V, O, tau, mask, alpha, True, so)
    torch.cuda.synchronize()
    if b.entmax_attn_check() != 0:
        raise RuntimeError("device status after the forward")
    st = b.stats_dict(stats)
    oo = b.make_opts(ws, hist_bins=hist_bins, init_mode=init_mode)
    ms = _median_ms(lambda: b.entmax_attn_fwd(Q, K, V, O, tau, mask, alpha, True, oo))
    return st, ms


def _row(label, alpha, st, ms, extra=""):
    rows = max(1, st["rows"])
    hist = " ".join(str(st[f"step_hist_{i}"]) for i in range(9))
    return (f"| {label} | {alpha:g} | {st['rows']} | {st['steps'] / rows:.3f} | {hist} | "
            f"{st['fallbacks'] / max(1, st['steps']):.4f} | {st['overflow_rows']} | "
            f"{1 - st['support'] / max(1, st['causal_rows_keys']):.4f} | "
            f"{1 - st['nonzero_blocks'] / max(1, st['causal_blocks']):.3f} | {ms:.3f} |{extra}")


def solver_report(out=sys.stdout):
    import torch  # noqa: F401
    print("| workload | alpha | rows | mean steps | rows by steps 0..8+ | fallback rate | overflow rows | "
          "element sparsity | block sparsity | fwd ms |", file=out)
    print("|---|---|---|---|---|---|---|---|---|---|", file=out)
    for name, kind, B, H, n, d, alphas, psets in CONFIGS:
        for params in psets:
            arr = _gen(kind, B, H, n, d, params)
            t = _to_dev({k: arr[k] for k in ("Q", "K", "V")})
            for alpha in alphas:
                for init_mode in ((0, 1) if name in ("cfg4", "cfg5") else (0,)):
                    st, ms = _forward_stats(t, alpha, init_mode)
                    st["causal_rows_keys"] = B * H * n * (n + 1) // 2
                    label = f"{name} {' '.join(f'{k}={v:g}' for k, v in params.items())}" + \
                        (" plain start" if init_mode else "")
                    print(_row(label, alpha, st, ms), file=out, flush=True)
            del t


def bins_report(out=sys.stdout):
    name, kind, B, H, n, d, alphas, psets = CONFIGS[2]
    arr = _gen(kind, B, H, n, d, psets[0])
    t = _to_dev({k: arr[k] for k in ("Q", "K", "V")})
    print("| bins B | histogram bytes per CTA (u16 [B][128]) | mean steps | rows by steps 0..8+ | "
          "fallback rate | overflow rows | fwd ms |", file=out)
    print("|---|---|---|---|---|---|---|", file=out)
    for bins in (64, 128, 256, 512):
        st, ms = _forward_stats(t, alphas[0], 0, bins)
        rows = max(1, st["rows"])
        hist = " ".join(str(st[f"step_hist_{i}"]) for i in range(9))
        print(f"| {bins} | {bins * 128 * 2} | {st['steps'] / rows:.3f} | {hist} | "
              f"{st['fallbacks'] / max(1, st['steps']):.4f} | {st['overflow_rows']} | {ms:.3f} |", file=out,
              flush=True)


def memory_report(out=sys.stdout):
    """Device bytes that stay allocated between the forward and the backward (the activation memory of the
    attention), measured with torch's allocator around each call, and the peak during the backward.
    Three paths: entmax with one workspace buffer (the fp16 operand copies are kept for the backward),
    entmax with a separate per-call scratch (only the saved part is kept), and the dense softmax baseline."""
    import torch

    from . import binding as b
    print("| workload | path | kept fwd -> bwd (MiB) | of which library workspace (MiB) | "
          "peak during bwd above inputs (MiB) |", file=out)
    print("|---|---|---|---|---|", file=out)
    mib = float(1 << 20)
    for name, kind, B, H, n, d, alphas, psets in CONFIGS:
        arr = _gen(kind, B, H, n, d, psets[-1])
        t = _to_dev(arr)
        Q, K, V, dO = t["Q"], t["K"], t["V"], t["dO"]
        alpha = alphas[0]
        for path in ("entmax, one buffer", "entmax, separate scratch", "softmax"):
            torch.cuda.synchronize()
            base = torch.cuda.memory_allocated()
            if path.startswith("entmax"):
                f = b.forward(Q, K, V, alpha, True, separate_scratch=path.endswith("scratch"))
                kept = (f.O, f.tau, f.mask, f.workspace)
                ws_bytes = f.workspace.numel()
            else:
                O, lse = b.softmax_forward(Q, K, V, True)
                kept = (O, lse)
                ws_bytes = 0
            torch.cuda.synchronize()
            after_fwd = torch.cuda.memory_allocated() - base
            torch.cuda.reset_peak_memory_stats()
            if path.startswith("entmax"):
                g = b.backward(Q, K, V, f, dO)
            else:
                g = b.softmax_backward(Q, K, V, O, lse, dO, True)
            torch.cuda.synchronize()
            peak = torch.cuda.max_memory_allocated() - base
            print(f"| {name} B={B} H={H} n={n} d={d} | {path} | {after_fwd / mib:.1f} | {ws_bytes / mib:.1f} | "
                  f"{peak / mib:.1f} |", file=out, flush=True)
            del kept, g
            if path.startswith("entmax"):
                del f
            else:
                del O, lse
        del t, Q, K, V, dO


def _peak_burst():
    import json
    import os
    p = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            return float(json.load(fh).get("bf16_tflops", 1590.0)), "measured"
    return 1590.0, "fallback"


def timing_report(out=sys.stdout):
    """Per configuration: entmax forward and backward ms (median of 5 CUDA-event timed calls, L2 flushed
    before each), effective TFLOP/s (dense Q K^T over the causal entries plus the P V and, for fwd + bwd
    configurations, the five backward products of each nonzero 64 x 64 block), its fraction of the bf16
    burst peak, and the dense softmax baseline of the library on the same inputs."""
    import numpy as np
    import torch

    from . import binding as b
    peak, src = _peak_burst()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def timed(fn, reps=5):
        fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return sorted(ts)[len(ts) // 2]

    print(f"| workload | alpha | pass | entmax fwd ms | entmax bwd ms | effective TFLOP/s | frac of bf16 burst "
          f"({peak:g}, {src}) | dense fwd (+bwd) ms | block sparsity |", file=out)
    print("|---|---|---|---|---|---|---|---|---|", file=out)
    # cfg1: fp32 inputs, non-causal, mask blocks of 32 (the FMA kernel; the dense baseline takes bf16 only)
    import numpy as np
    from . import inputs as inp
    arr = inp.iid(1, 1, 256, 64, seed=0, beta=1.0, dtype="fp32", with_dO=False)
    Q1, K1, V1 = (torch.from_numpy(np.ascontiguousarray(arr[k])).cuda() for k in ("Q", "K", "V"))
    ws1 = b.alloc_workspace(1, 1, 256, 64, b.ENTMAX_FP32, opts=b.make_opts(mask_block=32))
    o1 = b.make_opts(ws1, mask_block=32)
    O1 = torch.empty_like(Q1)
    t1 = torch.empty((1, 1, 256), dtype=torch.float32, device="cuda")
    m1 = torch.empty(b.mask_shape(1, 1, 256, 32), dtype=torch.int32, device="cuda")
    f1 = timed(lambda: b.entmax_attn_fwd(Q1, K1, V1, O1, t1, m1, 1.5, False, o1))
    nnz1 = int(np.unpackbits(m1.cpu().numpy().view(np.uint8), bitorder="little").sum())
    fl1 = 2.0 * 64 * 256 * 256 + 2.0 * 64 * 32 * 32 * nnz1
    print(f"| cfg1 B=1 H=1 n=256 d=64 fp32 non-causal | 1.5 | fwd | {f1:.3f} | - | {fl1 / (f1 * 1e-3) / 1e12:.2f} | "
          f"{fl1 / (f1 * 1e-3) / 1e12 / peak:.4f} | - | {1 - nnz1 / 64:.3f} |", file=out, flush=True)
    for name, kind, B, H, n, d, alphas, psets in CONFIGS:
        for params in psets:
            arr = _gen(kind, B, H, n, d, params)
            t = _to_dev(arr)
            Q, K, V, dO = t["Q"], t["K"], t["V"], t["dO"]
            fwd_only = name == "cfg2"
            ws = b.alloc_workspace(B, H, n, d)
            opts = b.make_opts(ws)
            O = torch.empty_like(Q)
            tau = torch.empty((B, H, n), dtype=torch.float32, device="cuda")
            mask = torch.empty(b.mask_shape(B, H, n), dtype=torch.int32, device="cuda")
            gq, gk, gv = (torch.empty(Q.shape, dtype=torch.float32, device="cuda") for _ in range(3))
            lse = torch.empty((B, H, n), dtype=torch.float32, device="cuda")
            for alpha in alphas:
                fwd = lambda: b.entmax_attn_fwd(Q, K, V, O, tau, mask, alpha, True, opts)  # noqa: E731
                fms = timed(fwd)
                fwd()
                torch.cuda.synchronize()
                nnz = int(np.unpackbits(mask.cpu().numpy().view(np.uint8), bitorder="little").sum())
                nqb = (n + 63) // 64
                qk = 2.0 * d * n * (n + 1) / 2 * B * H
                blk = 2.0 * d * 64 * 64 * nnz
                if fwd_only:
                    bms = float("nan")
                    flops, ms = qk + blk, fms
                    dense = timed(lambda: b.softmax_attn_fwd(Q, K, V, O, lse, True, opts))
                else:
                    bwd = lambda: b.entmax_attn_bwd(Q, K, V, O, dO, tau, mask, gq, gk, gv, alpha, True, opts)  # noqa
                    bms = timed(lambda: (fwd(), bwd())) - fms
                    flops, ms = qk + 6 * blk, fms + bms
                    dense = timed(lambda: (b.softmax_attn_fwd(Q, K, V, O, lse, True, opts),
                                           b.softmax_attn_bwd(Q, K, V, O, dO, lse, gq, gk, gv, True, opts)))
                tf = flops / (ms * 1e-3) / 1e12
                label = f"{name} {' '.join(f'{k}={v:g}' for k, v in params.items())} B={B} H={H} n={n} d={d}"
                print(f"| {label} | {alpha:g} | {'fwd' if fwd_only else 'fwd+bwd'} | {fms:.3f} | "
                      f"{'-' if fwd_only else f'{bms:.3f}'} | {tf:.1f} | {tf / peak:.3f} | {dense:.3f} | "
                      f"{1 - nnz / (B * H * nqb * (nqb + 1) // 2):.3f} |", file=out, flush=True)
            del t, Q, K, V, dO, ws


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("what", choices=["solver", "bins", "memory", "timing"])
    args = ap.parse_args(argv)
    from . import build
    build.build()
    {"solver": solver_report, "bins": bins_report, "memory": memory_report, "timing": timing_report}[args.what]()


if __name__ == "__main__":
    main()
