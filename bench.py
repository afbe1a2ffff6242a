"""Benchmark: alpha-entmax attention forward + backward on B200, effective TFLOP/s at n = 16k.

One step = entmax_attn_fwd + entmax_attn_bwd over one batch of the long-context workload
(B=1, H=16, n=16384, d=64, bf16, causal, alpha=1.5, keys clustered around 256 centres, queries
6x their centre plus noise; V and dO ~ N(0,1)), inputs resident in HBM. Effective FLOPs count the
dense Q K^T pass over the causal entries plus the P V and backward products of the nonzero
64 x 64 mask blocks only:  2 d n(n+1)/2 + (2 + 5 * 2) d 64 64 N_nz  per head.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--no-sweep] [--no-cpu] [--oracle-table]

Prints one JSON line (rank 0). Under torchrun each rank runs its own copy of the workload (independent
heads: no data-path collective), times on its device, and the max over ranks is reported.

Every kernel of a timed step is timed on its own: the library records caller events around each of its
launches (entmax_opts.events), so the per-kernel roofline comes from CUDA events on the launching stream.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

B, H, N, D, ALPHA = 1, 16, 16384, 64, 1.5
CENTRES, BETA_Q = 256, 6.0
BLOCK = 64
METRIC = "α-entmax attn fwd+bwd effective TFLOP/s at n=16k vs sparsity; % bf16 peak"
# kernels of one call on the fp16 operand path (d = 64, alpha <= 2), in launch order (include/entmax_attn.h,
# "Per-kernel timing"); the L2 flush between steps is a torch fill and is not counted
FWD_KERNELS = ("to_f16_pass1", "to_f16_pass2", "fwd_h_kernel", "mask_transpose_kernel")
# the backward's dQ kernel has three launches, of which K's range lets one route work: for unit-scale keys (the
# bench) the first; for larger keys the delta pass and the plain pass. The others return at once.
BWD_KERNELS = ("to_f16_pass1", "to_f16_pass2", "bwd_pre_kernel", "bwd_h_dq_kernel", "bwd_h_dq_delta_pass",
               "bwd_h_dq_plain_pass", "bwd_h_dkdv_kernel")
SM_FWD_KERNELS = ("to_f16_pass1", "to_f16_pass2", "softmax_fwd_h_kernel")
SM_BWD_KERNELS = ("to_f16_pass1", "to_f16_pass2", "bwd_pre_kernel", "bwd_h_dq_kernel", "bwd_h_dkdv_kernel")
LAUNCHES_PER_STEP = len(FWD_KERNELS) + len(BWD_KERNELS)
WORKLOAD = (f"alpha-entmax attention fwd+bwd, B={B} H={H} n={N} d={D} bf16 causal alpha={ALPHA}, "
            f"keys clustered on {CENTRES} centres (noise 0.3), queries {BETA_Q:g} x centre + noise")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic_entmax_b1h16n16384d64.json")

# Supplementary sparsity sweep at the bench shape: (label, generator, parameters). The i.i.d. family
# sharpens the scores with the query scale beta; the clustered family with contiguous runs of positions
# sharing a centre places each row's support in few key blocks. Together they span dense to ~94 % zero
# 64 x 64 blocks (block sparsity is measured on the GPU's own mask at every point).
SWEEP = (
    ("iid beta=1", "iid", {"beta": 1.0}),
    ("iid beta=2", "iid", {"beta": 2.0}),
    ("clustered C=256 beta_q=4", "clustered", {"centres": 256, "beta_q": 4.0}),
    ("clustered C=256 beta_q=6 (bench)", "clustered", {"centres": 256, "beta_q": 6.0}),
    ("iid beta=4", "iid", {"beta": 4.0}),
    ("iid beta=8", "iid", {"beta": 8.0}),
    ("iid beta=16", "iid", {"beta": 16.0}),
    ("iid beta=32", "iid", {"beta": 32.0}),
    ("runs C=16 run=16", "clustered", {"centres": 16, "beta_q": 6.0, "run": 16}),
    ("runs C=1 run=128", "clustered", {"centres": 1, "beta_q": 6.0, "run": 128}),
    ("runs C=2 run=128", "clustered", {"centres": 2, "beta_q": 6.0, "run": 128}),
    ("runs C=64 run=16", "clustered", {"centres": 64, "beta_q": 6.0, "run": 16}),
    ("runs C=4 run=128", "clustered", {"centres": 4, "beta_q": 6.0, "run": 128}),
    ("runs C=8 run=128", "clustered", {"centres": 8, "beta_q": 6.0, "run": 128}),
    ("runs C=16 run=128", "clustered", {"centres": 16, "beta_q": 6.0, "run": 128}),
)


def peaks():
    """(burst bf16 TFLOP/s, sustained bf16 TFLOP/s, HBM GB/s, source) from MEASURED_PEAKS.json, else the
    pool's fallback figures."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            j = json.load(fh)
        return j.get("bf16_tflops", 1590.0), j.get("bf16_tflops_sustained", 1400.0), j.get("hbm_gbs", 6650.0), "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


def effective_flops(n, d, heads, nnz_blocks, causal=True):
    qk = 2.0 * d * (n * (n + 1) / 2 if causal else n * n) * heads
    return qk + (2.0 + 10.0) * d * BLOCK * BLOCK * nnz_blocks


def kernel_flops(n, d, heads, nnz_blocks):
    """Algorithmic FLOPs of each kernel of an entmax step and of the dense baseline's kernels.

    Entmax: the forward owns the dense Q K^T pass and the nonzero-block P V product; of the five backward
    products per nonzero block, the dK / dV kernel owns S, dP, dV and dK, the dQ kernel owns dQ (its
    recomputed S and dP, and its split of dQ into (u g) K and u K, are not counted). Dense softmax baseline: two products over every causal entry in
    the forward (S, P V), four in the dK / dV kernel and one in the dQ kernel."""
    qk = 2.0 * d * n * (n + 1) / 2 * heads
    blk = 2.0 * d * BLOCK * BLOCK * nnz_blocks
    return {"fwd_h_kernel": qk + blk, "bwd_h_dkdv_kernel": 4 * blk, "bwd_h_dq_kernel": blk,
            "softmax_fwd_h_kernel": 2 * qk, "softmax_bwd_h_dkdv_kernel": 4 * qk, "softmax_bwd_h_dq_kernel": qk}


def source_digest(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel, path=TRAFFIC_FILE):
    """DRAM bytes per launch of `kernel` from the committed ncu counters, or None when there is no capture
    or the kernel's sources changed since it was taken."""
    if not os.path.exists(path):
        return None, "no capture"
    with open(path) as fh:
        j = json.load(fh)
    k = j.get("kernels", {}).get(kernel)
    if not k:
        return None, "no capture"
    if source_digest(k["sources"]) != k["sources_sha"]:
        return None, "kernel changed since the capture"
    return float(k["dram_bytes_per_launch"]), k.get("how", "")


class ClockSampler:
    """SM clock, max clock and throttle reasons during the timed region, as CSV lines
    (index, sm, max_sm, power, active, hw_slowdown, hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap).

    NVML is read every 10 ms from a thread (so that even a short timed region gets a dozen samples);
    without NVML, nvidia-smi at its 100 ms minimum."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits (nvmlClocksEventReason*): hw_slowdown, hw_thermal, sw_thermal, sw_power_cap
    REASON_BITS = (0x8, 0x40, 0x20, 0x4)

    def __init__(self, gpu_index, uuid=None, period_s=0.01):
        self.gpu = gpu_index
        self.uuid = uuid
        self.period = period_s
        self.proc = None
        self.stop_evt = threading.Event()
        self.lines = []  # (monotonic time, csv line)

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        if self.uuid:
            try:
                return pynvml, pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(self.uuid))
            except Exception:
                pass
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def _nvml_loop(self, nv, h):
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop_evt.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                rs = int(get_reasons(h))
                flags = ["Active" if rs & bit else "Not Active" for bit in self.REASON_BITS]
                self.lines.append((time.monotonic(), ", ".join([str(self.gpu), str(sm), str(mx), f"{pw:.2f}",
                                                                hex(rs)] + flags)))
            except Exception:
                pass
            self.stop_evt.wait(self.period)

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            self.t = threading.Thread(target=self._nvml_loop, args=(nv, h), daemon=True)
            self.t.start()
            self.source = "nvml 10 ms"
        except Exception:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                     "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.t = threading.Thread(target=self._read, daemon=True)
                self.t.start()
                self.source = "nvidia-smi 100 ms"
            except OSError:
                self.proc = None
                return self
        # wait for the first sample so the window is covered
        t_end = time.monotonic() + 10.0
        while not self.lines and time.monotonic() < t_end and (self.proc is None or self.proc.poll() is None):
            time.sleep(0.005)
        self.t0 = time.monotonic()
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def stop(self):
        """Mark the end of the timed region (call right after the closing synchronize)."""
        self.t1 = time.monotonic()

    def __exit__(self, *exc):
        self.stop_evt.set()
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        t0 = getattr(self, "t0", 0.0)
        t1 = getattr(self, "t1", float("inf"))
        window = [ln for t, ln in self.lines if t0 - 0.25 <= t <= t1 + 0.25]
        for ln in window:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(mx), "reasons": sorted(reasons), "samples": len(sm)}


def gen_inputs(seed, centres=CENTRES, run=0):
    from adaptive_sparse_flash_b200 import inputs
    return inputs.clustered(B, H, N, D, centres=centres, beta_q=BETA_Q, seed=seed, run=run)


def gen_sweep_inputs(kind, params, seed):
    from adaptive_sparse_flash_b200 import inputs
    if kind == "iid":
        return inputs.iid(B, H, N, D, seed=seed, beta=params["beta"])
    return inputs.clustered(B, H, N, D, centres=params["centres"], beta_q=params["beta_q"], seed=seed,
                            run=params.get("run", 0))


def cpu_baseline(arr):
    """The float64 oracle on a bounded sample: one head, full forward + backward. Returns a dict."""
    from oracle import attention as oa
    t0 = time.perf_counter()
    sub = {k: v[:1, :1] for k, v in arr.items()}
    fw = oa.forward(sub["Q"], sub["K"], sub["V"], ALPHA, True)
    oa.backward(sub["Q"], sub["K"], sub["V"], sub["dO"], ALPHA, True)
    sec = time.perf_counter() - t0
    nnz = int(fw["bits"].sum())
    flops = effective_flops(N, D, 1, nnz)
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    return {"value": flops / sec / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"head 0 of {H}: float64 oracle forward (all {N} rows) + backward (all rows and keys), "
                      f"{sec:.1f} s, scaled by that head's effective FLOPs", "seconds": sec}


# (label, generator kind, B, H, n, d, alpha, params, causal, backward): one row per configuration of the
# parity tests, for the oracle's per-configuration CPU time
ORACLE_TABLE = (
    ("cfg1 1x1x256x64 fp32 non-causal", "iid", 1, 1, 256, 64, 1.5, {"beta": 1.0}, False, False),
    ("cfg2 4x8x1024x64 beta=4", "iid", 4, 8, 1024, 64, 1.5, {"beta": 4.0}, True, False),
    ("cfg3 2x16x4096x128 beta=8", "iid", 2, 16, 4096, 128, 1.5, {"beta": 8.0}, True, True),
    ("cfg4 1x16x16384x64 clustered", "clustered", 1, 16, 16384, 64, 1.5, {"centres": 256, "beta_q": 6.0}, True, True),
    ("cfg5 8x12x2048x64 clustered beta_q=4", "clustered", 8, 12, 2048, 64, 1.5, {"centres": 64, "beta_q": 4.0}, True, True),
)


def oracle_table():
    """The float64 oracle's CPU time per configuration: one head timed (forward, and backward where the
    configuration has one), scaled to the configuration's heads. Prints a markdown table."""
    from adaptive_sparse_flash_b200 import inputs as _inputs
    from oracle import attention as oa
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    print(f"| configuration | oracle s, one head | heads | oracle s, whole configuration ({cores} cores) |")
    print("|---|---|---|---|")
    for label, kind, Bc, Hc, n, d, alpha, params, causal, bwd in ORACLE_TABLE:
        if kind == "iid":
            arr = _inputs.iid(1, 1, n, d, seed=0, beta=params["beta"], dtype="fp32" if "fp32" in label else "bf16",
                              with_dO=bwd)
        else:
            arr = _inputs.clustered(1, 1, n, d, centres=params["centres"], beta_q=params["beta_q"], seed=0)
        t0 = time.perf_counter()
        oa.forward(arr["Q"], arr["K"], arr["V"], alpha, causal)
        if bwd:
            oa.backward(arr["Q"], arr["K"], arr["V"], arr["dO"], alpha, causal)
        sec = time.perf_counter() - t0
        print(f"| {label} ({'fwd+bwd' if bwd else 'fwd'}) | {sec:.2f} | {Bc * Hc} | {sec * Bc * Hc:.1f} |", flush=True)
    return 0


def rank_env():
    """(rank, world size, local rank) from the launcher's environment; one process per GPU."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_ranks(world, backend="nccl", timeout_s=120):
    """Join the process group when there is more than one rank (a short timeout, so that ranks waiting on
    one another end with an error)."""
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))


class RankOps:
    """The only collectives of a run: a barrier around the timed region and the max over ranks of each
    measured time. The data path has none: every rank computes its own independent heads."""

    def __init__(self, world, device):
        self.world = world
        self.device = device

    def barrier(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()

    def max(self, x):
        if self.world == 1:
            return x
        import torch
        import torch.distributed as dist
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())


def median(xs):
    """Middle value of the sorted times (the upper middle for an even count)."""
    ys = sorted(xs)
    return ys[len(ys) // 2]


def whole_job_tflops(world, flops_per_rank, step_ms_max):
    """Weak scaling: all ranks' effective FLOPs over the slowest rank's time per step."""
    return world * flops_per_rank / (step_ms_max * 1e-3) / 1e12


def per_kernel_ms(event_lists, names):
    """Mean time of each launch position over the steps: event_lists[i] holds len(names) + 1 events."""
    out = {}
    for k, nm in enumerate(names):
        ts = [ev[k].elapsed_time(ev[k + 1]) for ev in event_lists]
        key = nm
        while key in out:  # the same kernel twice in a call (the two conversion passes are distinct names)
            key += "'"
        out[key] = sum(ts) / len(ts)
    return out


def roofline_entry(name, flops, ms, peak):
    ach = flops / (ms * 1e-3) / 1e12
    return {"ms": ms, "algorithmic_tflop": flops / 1e12, "achieved": ach, "frac": ach / peak}


def run_reference(args, rank, world):
    if rank != 0:
        return
    arr = gen_inputs(seed=0)
    times = []
    for i in range(args.warmup + args.steps):
        res = cpu_baseline(arr)
        if i >= args.warmup:
            times.append(res["seconds"])
    sec = sum(times) / len(times)
    val = res["value"] * res["seconds"] / sec
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": res["sample"]},
            "cpu_baseline": {"kind": "oracle", "cores": res["cores"], "sample": res["sample"], "value": val,
                             "unit": "TFLOP/s"},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--oracle-table", action="store_true",
                    help="print the float64 oracle's CPU time per configuration and exit (no GPU)")
    args = ap.parse_args()
    if args.oracle_table:
        return oracle_table()
    if args.warmup < 3:
        args.warmup = 3

    rank, world, local = rank_env()
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import numpy as np
    import torch
    import torch.distributed as dist

    from adaptive_sparse_flash_b200 import binding as b
    from adaptive_sparse_flash_b200 import build as bld

    if world > 1:
        torch.cuda.set_device(local)
    init_ranks(world, "nccl")
    dev = torch.device("cuda", local)
    bld.build()
    b.lib()
    ops = RankOps(world, dev)
    barrier, max_over_ranks = ops.barrier, ops.max

    arr = gen_inputs(seed=rank)
    from adaptive_sparse_flash_b200 import inputs as _inputs
    host = {k: torch.from_numpy(_inputs.bf16_bits(v).view(np.int16)).view(torch.bfloat16) for k, v in arr.items()}
    dt = {k: v.to(dev) for k, v in host.items()}
    Q, K, V, dO = dt["Q"], dt["K"], dt["V"], dt["dO"]
    ws = b.alloc_workspace(B, H, N, D, device=dev)
    opts = b.make_opts(ws)
    stats = torch.zeros(b.STATS_WORDS, dtype=torch.int64, device=dev)
    sopts = b.make_opts(ws, stats=stats)
    O = torch.empty_like(Q)
    tau = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    mask = torch.empty(b.mask_shape(B, H, N), dtype=torch.int32, device=dev)
    dQ, dK, dV = (torch.empty(Q.shape, dtype=torch.float32, device=dev) for _ in range(3))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # larger than the 126 MB L2
    stream = torch.cuda.current_stream(dev)

    def new_events(k):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(k)]
        for e in evs:
            e.record(stream)  # creates the CUDA event, so the library can record it again
        return evs

    def step(fo=opts, bo=opts):
        b.entmax_attn_fwd(Q, K, V, O, tau, mask, ALPHA, True, fo, stream)
        b.entmax_attn_bwd(Q, K, V, O, dO, tau, mask, dQ, dK, dV, ALPHA, True, bo, stream)

    # warm-up; sparsity and solver statistics of this workload (one extra forward with counters)
    for _ in range(args.warmup):
        flush.zero_()
        step()
    b.entmax_attn_fwd(Q, K, V, O, tau, mask, ALPHA, True, sopts, stream)
    torch.cuda.synchronize(dev)
    st = b.entmax_attn_check(stream)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {b.entmax_status_str(st)}")
    sd = b.stats_dict(stats)
    nnz = int(np.unpackbits(mask.cpu().numpy().view(np.uint8), bitorder="little").sum())
    nqb = (N + BLOCK - 1) // BLOCK
    causal_blocks = H * B * nqb * (nqb + 1) // 2
    flops = effective_flops(N, D, B * H, nnz)
    causal_entries = B * H * N * (N + 1) // 2

    # timed region: per-step events around every kernel (L2 flushed before each step, outside the events)
    evf = [new_events(len(FWD_KERNELS) + 1) for _ in range(args.steps)]
    evb = [new_events(len(BWD_KERNELS) + 1) for _ in range(args.steps)]
    fo = [b.make_opts(ws, events=e) for e in evf]
    bo = [b.make_opts(ws, events=e) for e in evb]
    torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    uuid = getattr(torch.cuda.get_device_properties(dev), "uuid", None)
    with ClockSampler(local, uuid) as clk:
        for i in range(args.steps):
            flush.zero_()
            step(fo[i], bo[i])
        torch.cuda.synchronize(dev)
        clk.stop()
    barrier()
    st = b.entmax_attn_check(stream)
    if st != 0:
        raise RuntimeError(f"device status after timing: {b.entmax_status_str(st)}")
    fwd_ms = [e[0].elapsed_time(e[-1]) for e in evf]
    bwd_ms = [e[0].elapsed_time(e[-1]) for e in evb]
    step_ms = max_over_ranks(sum(f + g for f, g in zip(fwd_ms, bwd_ms)) / args.steps)
    value = whole_job_tflops(world, flops, step_ms)
    kf = per_kernel_ms(evf, FWD_KERNELS)
    kb = per_kernel_ms(evb, BWD_KERNELS)
    kms = {k: max_over_ranks(v) for k, v in [("fwd_h_kernel", kf["fwd_h_kernel"]),
                                               ("bwd_h_dq_kernel", kb["bwd_h_dq_kernel"]),
                                               ("bwd_h_dkdv_kernel", kb["bwd_h_dkdv_kernel"])]}

    # end to end through the public API with host buffers (pinned), copies inside the timed region
    pin = {k: v.pin_memory() for k, v in host.items()}
    out_host = {k: torch.empty(Q.shape, dtype=torch.float32).pin_memory() for k in ("dQ", "dK", "dV")}
    out_host["O"] = torch.empty(Q.shape, dtype=torch.bfloat16).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in pin.values())
    d2h = sum(v.numel() * v.element_size() for v in out_host.values())
    e2e_steps = max(2, min(args.steps, 5))
    barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        Q.copy_(pin["Q"], non_blocking=True)
        K.copy_(pin["K"], non_blocking=True)
        V.copy_(pin["V"], non_blocking=True)
        dO.copy_(pin["dO"], non_blocking=True)
        step()
        out_host["dQ"].copy_(dQ, non_blocking=True)
        out_host["dK"].copy_(dK, non_blocking=True)
        out_host["dV"].copy_(dV, non_blocking=True)
        out_host["O"].copy_(O, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps)
    e2e_val = whole_job_tflops(world, flops, e2e_ms)

    # dense softmax baseline on the same inputs, same tiling, its kernels timed the same way
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    sdQ, sdK, sdV = (torch.empty(Q.shape, dtype=torch.float32, device=dev) for _ in range(3))

    def sm_step(fo=opts, bo=opts):
        b.softmax_attn_fwd(Q, K, V, O, lse, True, fo, stream)
        b.softmax_attn_bwd(Q, K, V, O, dO, lse, sdQ, sdK, sdV, True, bo, stream)

    def timed(fn, reps):
        """Median of `reps` CUDA-event times after 3 warm-up calls, L2 flushed before each timed call."""
        for _ in range(3):
            fn()
        torch.cuda.synchronize(dev)
        ts = []
        for _ in range(reps):
            flush.zero_()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            fn()
            a1.record(stream)
            torch.cuda.synchronize(dev)
            ts.append(a0.elapsed_time(a1))
        return median(ts)

    sm_reps = 7
    sevf = [new_events(len(SM_FWD_KERNELS) + 1) for _ in range(sm_reps)]
    sevb = [new_events(len(SM_BWD_KERNELS) + 1) for _ in range(sm_reps)]
    for _ in range(3):
        sm_step()
    for i in range(sm_reps):
        flush.zero_()
        sm_step(b.make_opts(ws, events=sevf[i]), b.make_opts(ws, events=sevb[i]))
    torch.cuda.synchronize(dev)
    sm_steps_ms = sorted(f[0].elapsed_time(f[-1]) + g[0].elapsed_time(g[-1]) for f, g in zip(sevf, sevb))
    softmax_ms = max_over_ranks(sm_steps_ms[len(sm_steps_ms) // 2])
    skf = per_kernel_ms(sevf, SM_FWD_KERNELS)
    skb = per_kernel_ms(sevb, SM_BWD_KERNELS)

    # roofline: every tensor-core kernel of the step against the measured bf16 burst peak (the kernels run
    # for milliseconds each, L2 flushed between steps; fp16 operands have the bf16 nominal dense rate)
    pk_burst, pk_sust, hbm, pk_kind = peaks()
    kfl = kernel_flops(N, D, B * H, nnz)
    kernels = {nm: roofline_entry(nm, kfl[nm], kms[nm], pk_burst) for nm in kms}
    dom = max(kms, key=lambda k: kms[k])
    traffic, traffic_src = measured_traffic(dom)
    roofline = {"bound": "tensor", "achieved": kernels[dom]["achieved"], "peak": pk_burst, "unit": "TFLOP/s",
                "frac": kernels[dom]["frac"], "traffic": traffic, "kernel": dom,
                "peak_source": f"{pk_kind} bf16 burst (fp16 operands: same nominal dense rate)",
                "traffic_source": traffic_src, "kernels": kernels}
    sm_kms = {"softmax_fwd_h_kernel": skf["softmax_fwd_h_kernel"],
              "softmax_bwd_h_dkdv_kernel": skb["bwd_h_dkdv_kernel"], "softmax_bwd_h_dq_kernel": skb["bwd_h_dq_kernel"]}
    sm_flops = 7 * 2.0 * D * causal_entries
    softmax_baseline = {"ms": softmax_ms, "tflops": sm_flops / (softmax_ms * 1e-3) / 1e12,
                        "frac": sm_flops / (softmax_ms * 1e-3) / 1e12 / pk_burst,
                        "kernels": {nm: roofline_entry(nm, kfl[nm], ms, pk_burst) for nm, ms in sm_kms.items()}}

    # supplementary sweep of block sparsity (see SWEEP)
    sweep = []
    if not args.no_sweep:
        for i, (label, kind, params) in enumerate(SWEEP):
            a2 = gen_sweep_inputs(kind, params, seed=100 + i)
            for k2, v2 in a2.items():
                dt[k2].copy_(torch.from_numpy(v2).to(torch.bfloat16))
            stats.zero_()
            b.entmax_attn_fwd(Q, K, V, O, tau, mask, ALPHA, True, sopts, stream)
            torch.cuda.synchronize(dev)
            s2 = b.stats_dict(stats)
            nz = int(np.unpackbits(mask.cpu().numpy().view(np.uint8), bitorder="little").sum())
            ms_e = timed(step, 7)
            ms_s = timed(sm_step, 7)
            fl = effective_flops(N, D, B * H, nz)
            sweep.append({"point": label, "block_sparsity": 1.0 - nz / causal_blocks,
                          "element_sparsity": 1.0 - s2["support"] / causal_entries,
                          "entmax_ms": ms_e, "softmax_ms": ms_s, "eff_tflops": fl / (ms_e * 1e-3) / 1e12,
                          "mean_steps": s2["steps"] / max(1, s2["rows"]), "faster_than_dense": ms_e < ms_s})
        for k2, v2 in arr.items():
            dt[k2].copy_(torch.from_numpy(v2).to(torch.bfloat16))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(arr)
        cpu.pop("seconds", None)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "global_batch_heads": B * H * world, "seq_len": N,
                       "parallelism": f"independent heads x{world}" if world > 1 else "single GPU",
                       "l2": "flushed before every timed step (256 MiB write)",
                       "mma_operands": "fp16 copies of the bf16 inputs (exact, power-of-two range scaling), "
                                       "fp32 accumulation",
                       "block_sparsity": 1.0 - nnz / causal_blocks, "nonzero_blocks": nnz,
                       "element_sparsity": 1.0 - sd["support"] / causal_entries,
                       "solver_mean_steps": sd["steps"] / max(1, sd["rows"]),
                       "fwd_ms": sum(fwd_ms) / len(fwd_ms), "bwd_ms": sum(bwd_ms) / len(bwd_ms),
                       "softmax_fwd_bwd_ms": softmax_ms,
                       "pct_bf16_peak": value / world / pk_burst * 100.0},
            "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms},
            "gpu_launches": LAUNCHES_PER_STEP * args.steps * world,  # every rank launches its own
            "clocks": clk.summary(),
            "roofline": roofline,
            "softmax_baseline": softmax_baseline,
            "cpu_baseline": cpu,
            "sparsity_sweep": sweep,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
