"""The multi-rank plumbing of bench.py on the CPU: two processes over gloo (world size 2)
check the barrier, the max / sum reductions, the whole-job aggregation of a
data-parallel run (sum of work over ranks / max of device time), and that under torchrun
only rank 0 of the reference arm runs and prints."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        mx = bench.max_over_ranks(world, float(rank + 1) * 10.0, device="cpu")
        sm = bench.sum_over_ranks(world, float(rank + 1), device="cpu")
        # rank r did (r + 1) * 1e12 FLOP in (r + 1) * 100 ms
        work, ms = bench.aggregate(world, (rank + 1) * 1e12, (rank + 1) * 100.0, device="cpu")
        # reference arm: rank 1 must return without work or output
        out = io.StringIO()
        if rank == 1:
            class Args:
                workload, steps, warmup, gpus = "quant_dense", 1, 1, world
            with redirect_stdout(out):
                bench.run_reference(Args, world, rank)
        results[rank] = (mx, sm, work, ms, out.getvalue())
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_rank_reductions_and_aggregation():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, results)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(results)
    for rank in range(2):
        mx, sm, work, ms, out = res[rank]
        assert mx == 20.0 and sm == 3.0
        assert work == 3e12 and ms == 200.0          # value = 3e12 FLOP / 0.2 s = 15 TFLOP/s
    assert res[1][4] == ""                            # the reference arm ran on rank 0 only


def test_single_rank_helpers_are_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1, 5.0) == 5.0
    assert bench.sum_over_ranks(1, 5.0) == 5.0
    assert bench.aggregate(1, 7.0, 3.0) == (7.0, 3.0)


def test_reference_arm_config_is_computed_without_a_gpu():
    # the reference arm prints the CUDA arm's config; it must build on a machine without a GPU
    sys.path.insert(0, ROOT)
    import bench
    for name in ("swiglu_block", "quant_dense", "quant_dense_fused", "quant_masked", "quant_silu", "grouped_moe",
                 "grouped_swiglu", "lowrank", "svdquant_linear", "pr1_linear", "bf16a_linear"):
        cfg = bench.workload_config(name, 64)
        assert isinstance(cfg["workload"], str) and cfg["workload"]
        assert "l2" in cfg
    assert "sum 8088" in bench.workload_config("grouped_swiglu", 64)["workload"]
    assert "r=32" in bench.workload_config("lowrank", 32)["workload"]


def test_reference_arm_prints_one_contract_line():
    # the reference arm at N = 1 on the smallest workload: one JSON line with the contract's
    # keys, the impl tag, and the cpu_baseline / e2e objects describing this run
    import json
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        workload, steps, warmup, gpus, rank_lr, swiglu_path = "pr1_linear", 2, 3, 1, 64, "fused"
    out = io.StringIO()
    with redirect_stdout(out):
        bench.run_reference(Args, 1, 0)
    lines = out.getvalue().strip().splitlines()
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["steps"] == 2 and line["warmup"] == 3
    assert line["value"] > 0 and line["unit"] == "TFLOP/s" and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["cores"] >= 1 and line["cpu_baseline"]["sample"]
    assert line["cpu_baseline"]["host_cpus"] >= line["cpu_baseline"]["cores"]
    assert "cpu_model" in line["cpu_baseline"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"] == bench.workload_config("pr1_linear", 64, "fused")
