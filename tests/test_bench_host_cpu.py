"""Host logic of bench.py on CPU: the multi-rank plumbing on two gloo ranks (the GPU run makes the same
calls over NCCL), the clock record and the effective-FLOP count."""
import io
import multiprocessing as mp
import os
import socket
import sys
import time
from contextlib import redirect_stdout
from types import SimpleNamespace

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import bench as bm
    try:
        r, w, local = bm.rank_env()
        bm.init_ranks(w, "gloo", timeout_s=30)
        ops = bm.RankOps(w, torch.device("cpu"))
        ops.barrier()
        step_ms = 2.0 + 3.0 * r           # this rank's time per step
        slowest = ops.max(step_ms)
        value = bm.whole_job_tflops(w, 1e12, slowest)
        # each rank computes its own independent problem: inputs seeded by rank (small shape here)
        bm.B, bm.H, bm.N = 1, 2, 256
        arr = bm.gen_inputs(seed=r)
        digest = float(np.abs(arr["Q"]).sum() + np.abs(arr["K"]).sum())
        # the reference arm runs on rank 0 only; the other ranks return at once and print nothing
        out = io.StringIO()
        t0 = time.perf_counter()
        if r != 0:
            with redirect_stdout(out):
                bm.run_reference(SimpleNamespace(steps=1, warmup=3), r, w)
        ref_sec = time.perf_counter() - t0
        ops.barrier()
        q.put((r, w, local, slowest, value, digest, out.getvalue(), ref_sec))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = []
    try:
        for _ in procs:
            res.append(q.get(timeout=120))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    res.sort()
    assert [x[0] for x in res] == [0, 1] and all(x[1] == 2 and x[2] == x[0] for x in res)
    # max over ranks: both ranks see the slowest rank's time, and the job rate uses it
    assert all(x[3] == 5.0 for x in res)
    assert all(x[4] == pytest.approx(2 * 1e12 / 5e-3 / 1e12) for x in res)
    # independent problems per rank
    assert res[0][5] != res[1][5]
    # rank 1 of the reference arm: no output, no work
    assert res[1][6] == "" and res[1][7] < 1.0


def test_single_rank_ops_are_identity():
    import torch
    ops = bench.RankOps(1, torch.device("cpu"))
    ops.barrier()
    assert ops.max(3.5) == 3.5
    assert bench.whole_job_tflops(1, 2e12, 1000.0) == pytest.approx(2.0)


def _line(sm, mx, reasons=()):
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    flags = ["Active" if nm in reasons else "Not Active" for nm in names]
    return ", ".join(["0", str(sm), str(mx), "700.00", "0x0"] + flags)


def test_clock_record_window_median_and_reasons():
    c = bench.ClockSampler(0)
    c.t0, c.t1 = 10.0, 12.0
    c.lines = [(9.0, _line(300, 1965, ["hw_slowdown"])),      # before the window: ignored
               (10.1, _line(1965, 1965)), (10.5, _line(1900, 1965, ["sw_power_cap"])),
               (11.0, _line(1950, 1965)), (11.9, _line("[N/A]", 1965)),  # unparsable: skipped
               (13.0, _line(200, 1965, ["sw_thermal_slowdown"]))]       # after the window: ignored
    s = c.summary()
    assert s == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_clock_record_without_samples():
    c = bench.ClockSampler(0)
    c.t0, c.t1 = 0.0, 1.0
    assert c.summary()["reasons"] == ["unsampled"]


def test_effective_flops():
    d, blk = 64, bench.BLOCK
    # dense causal Q K^T: 2 d flops per (row, allowed key) pair, n (n + 1) / 2 pairs per head
    assert bench.effective_flops(128, d, 3, 0) == 2.0 * d * (128 * 129 // 2) * 3
    assert bench.effective_flops(128, d, 1, 0, causal=False) == 2.0 * d * 128 * 128
    # each nonzero block adds P V (2 d per entry) and the five backward products (10 d per entry)
    assert bench.effective_flops(128, d, 1, 7) - bench.effective_flops(128, d, 1, 0) == 12.0 * d * blk * blk * 7


def test_median_of_repetitions():
    # one slow repetition (another tenant, a clock dip) does not move the reported time
    assert bench.median([2.5, 2.4, 9.0, 2.6, 2.5, 2.45, 2.55]) == 2.5
    assert bench.median([3.0]) == 3.0
